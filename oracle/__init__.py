"""CPU oracle for one Orthrus decoding round and for the tiny-model consensus loop.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline leg (and its ``--impl reference`` arm) may import
this package.  The product library never imports, links or calls it, and it
imports nothing from the product package.

The arithmetic lives in ``orthrus_oracle.c`` (plain loops, double
accumulation); this module only marshals numpy arrays and runs the
consensus/greedy decoding loops, whose control flow restates the inference
procedure of the Orthrus explainer (cjcn.com.cn, on arXiv:2605.12825), §四:
diffusion draft of a 32-slot block, AR verify of the 32 positions, left-to-right
consensus with one correction token, then a KV notebook update.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "orthrus_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

F32, BF16, F64 = 0, 1, 2
BIDIR_BLOCK, CAUSAL_VERIFY = 0, 1


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB_PATH) or (
        os.path.getmtime(_LIB_PATH) < max(os.path.getmtime(_SRC),
                                          os.path.getmtime(_SRC[:-2] + ".h"))):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off",
             "-fno-fast-math", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        c = ctypes
        vp, i32p, f64p = c.c_void_p, c.POINTER(c.c_int32), c.POINTER(c.c_double)
        _lib.oracle_block_attn.argtypes = [c.c_int] * 7 + [vp] * 5 + [
            c.c_int, i32p, c.c_double, f64p, c.c_int]
        _lib.oracle_vocab_argmax.argtypes = [c.c_int, vp, c.c_int, c.c_int,
                                             c.c_int64, i32p, f64p]
        _lib.oracle_consensus.argtypes = [i32p, i32p, c.c_int, c.c_int,
                                          i32p, i32p, i32p, i32p]
        _lib.oracle_kv_commit.argtypes = [c.c_int, vp, vp, vp, vp] + [
            c.c_int] * 5 + [i32p, i32p]
        _lib.oracle_model_num_weights.argtypes = [c.POINTER(ModelCfg)]
        _lib.oracle_model_num_weights.restype = c.c_int64
        _lib.oracle_model_forward.argtypes = [
            c.POINTER(ModelCfg), f64p, c.c_int, i32p, c.c_int, f64p, f64p,
            c.c_int, c.c_int, f64p, f64p, f64p, c.c_int]
    return _lib


def _ptr(a: np.ndarray, ctype=ctypes.c_void_p):
    assert a.flags["C_CONTIGUOUS"]
    if ctype is ctypes.c_void_p:
        return ctypes.c_void_p(a.ctypes.data)
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:  # bf16 bit patterns
        return BF16
    raise TypeError(f"oracle takes float32 or bf16-as-uint16, got {a.dtype}")


def block_attn(q, k_blk, v_blk, k_cache, v_cache, ctx_lens, mask_mode,
               scale=None, nthreads=0):
    """softmax(q k^T * scale) v per (sequence, block row, q-head), double result.

    q [B, blk, Hq, D]; k_blk/v_blk [B, blk, Hkv, D]; caches [B, Hkv, cap, D];
    ctx_lens [B].  mask_mode 0 = bidirectional block, 1 = causal verify.
    """
    B, blk, Hq, D = q.shape
    Hkv, cap = k_cache.shape[1], k_cache.shape[2]
    dt = _dtype_code(q)
    for a in (k_blk, v_blk, k_cache, v_cache):
        assert _dtype_code(a) == dt
    assert k_blk.shape == (B, blk, Hkv, D) and v_blk.shape == k_blk.shape
    assert k_cache.shape == (B, Hkv, cap, D) and v_cache.shape == k_cache.shape
    lens = np.ascontiguousarray(ctx_lens, dtype=np.int32)
    out = np.zeros((B, blk, Hq, D), dtype=np.float64)
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    arrs = [np.ascontiguousarray(a) for a in (q, k_blk, v_blk, k_cache, v_cache)]
    rc = lib().oracle_block_attn(dt, int(mask_mode), B, Hq, Hkv, D, blk,
                                 *[_ptr(a) for a in arrs], cap,
                                 _ptr(lens, ctypes.c_int32), float(scale),
                                 _ptr(out, ctypes.c_double), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_block_attn: bad arguments")
    return out


def token_logprob(logits, idx, temperature=1.0, return_lse=False):
    """Log-softmax of each row of logits / temperature at idx, in float64:
    s[idx] - lse with s = x / T and lse = m + log(sum exp(s - m)), m the row
    maximum (the definition; no blocking).  bf16 bit patterns (uint16) are
    widened exactly.  idx outside [0, vocab) gives NaN."""
    x = np.asarray(logits)
    if x.dtype == np.uint16:
        x = (x.astype(np.uint32) << 16).view(np.float32)
    x = x.astype(np.float64) / temperature
    idx = np.asarray(idx, np.int64)
    rows, vocab = x.shape
    out = np.full(rows, np.nan)
    lse = np.zeros(rows)
    for r in range(rows):
        m = x[r].max()
        lse[r] = m + np.log(np.exp(x[r] - m).sum())
        k = int(idx[r])
        if 0 <= k < vocab:
            out[r] = x[r, k] - lse[r]
    return (out, lse) if return_lse else out


def vocab_argmax(logits, return_max=False):
    """Row argmax, lowest index among equal maxima; NaN never wins."""
    logits = np.ascontiguousarray(logits)
    rows, vocab = logits.shape
    code = F64 if logits.dtype == np.float64 else _dtype_code(logits)
    idx = np.zeros(rows, dtype=np.int32)
    mx = np.zeros(rows, dtype=np.float64)
    rc = lib().oracle_vocab_argmax(code, _ptr(logits), rows,
                                   vocab, vocab, _ptr(idx, ctypes.c_int32),
                                   _ptr(mx, ctypes.c_double))
    if rc != 0:
        raise ValueError("oracle_vocab_argmax: bad arguments")
    return (idx, mx) if return_max else idx


def _widen64(x):
    x = np.asarray(x)
    if x.dtype == np.uint16:  # bf16 bit patterns
        x = (x.astype(np.uint32) << 16).view(np.float32)
    return x.astype(np.float64)


def lm_head_argmax(h, w, chunk=8192):
    """The LM head feeding the round's argmax, without the logits leaving it:
    logits[r, v] = sum_k h[r, k] w[v, k] in float64 (the product of the
    final hidden states with the output embedding; bf16 bit patterns widened
    exactly), then each row's argmax with the lowest index among equal maxima
    (vocab_argmax).  Returns (idx int32 [rows], max float64 [rows], gap
    float64 [rows], mag float64 [rows]): gap = distance between the row's two
    largest logits, mag = max_v sum_k |h[r, k]| |w[v, k]|, the scale of the
    rounding error of any lower-precision evaluation of the row.  The product
    is taken over vocabulary slices of `chunk` rows (a memory bound only: each
    logit is one complete dot product)."""
    H = _widen64(h)
    rows, V = H.shape[0], np.shape(w)[0]
    logits = np.empty((rows, V))
    mag = np.zeros(rows)
    aH = np.abs(H)
    for c0 in range(0, V, chunk):
        Wc = _widen64(w[c0:c0 + chunk])
        logits[:, c0:c0 + chunk] = H @ Wc.T
        mag = np.maximum(mag, (aH @ np.abs(Wc).T).max(axis=1))
    idx, mx = vocab_argmax(logits, return_max=True)
    if V > 1:
        top2 = np.partition(logits, V - 2, axis=1)[:, -2:]
        gap = top2[:, 1] - top2[:, 0]
    else:
        gap = np.full(rows, np.inf)
    return idx, mx, gap, mag


def round_bf16(x):
    """float64 -> bf16 bit patterns (uint16), rounding once, to nearest with
    ties to even, straight from the float64 value: x = m 2^e with
    0.5 <= |m| < 1, and bf16 keeps 8 significant bits, so m is rounded to a
    multiple of 2^-8.  Finite inputs of normal bf16 range only."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    y = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)  # np.rint: ties to even
    return (y.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)


def projection(x, w, residual=None):
    """A linear layer of a bf16 model (the attention block's QKV and output
    projections around the round's attention; explainer §二: the diffusion
    view has its own copy of them): y[r, n] = sum_k x[r, k] w[n, k] in
    float64 over the exactly widened bf16 inputs, rounded to bf16; with a
    residual, y = bf16(residual + that rounded product).  x [R, K], w [N, K]
    (PyTorch Linear layout), residual [R, N], all bf16 bit patterns.  Returns
    (y bf16 bits [R, N], exact product float64 [R, N], mag float64 [R, N] =
    sum_k |x[r, k]| |w[n, k]|, the scale of any lower-precision summation's
    error)."""
    X, W = _widen64(x), _widen64(w)
    exact = X @ W.T
    mag = np.abs(X) @ np.abs(W).T
    y = round_bf16(exact)
    if residual is not None:
        y = round_bf16(_widen64(residual) + _widen64(y))
    return y, exact, mag


def consensus(draft, verify):
    """(accept_len [B], n_emit [B], emitted [B, blk] (-1 padded), next_anchor [B])."""
    d = np.ascontiguousarray(draft, dtype=np.int32)
    a = np.ascontiguousarray(verify, dtype=np.int32)
    B, blk = d.shape
    L = np.zeros(B, np.int32)
    ne = np.zeros(B, np.int32)
    em = np.zeros((B, blk), np.int32)
    na = np.zeros(B, np.int32)
    i32 = ctypes.c_int32
    rc = lib().oracle_consensus(_ptr(d, i32), _ptr(a, i32), B, blk, _ptr(L, i32),
                                _ptr(ne, i32), _ptr(em, i32), _ptr(na, i32))
    if rc != 0:
        raise ValueError("oracle_consensus: bad arguments")
    return L, ne, em, na


def kv_commit(k_cache, v_cache, k_blk, v_blk, ctx_lens, n_emit):
    """In place on the numpy caches; returns the new ctx_lens."""
    B, Hkv, cap, D = k_cache.shape
    blk = k_blk.shape[1]
    lens = np.array(ctx_lens, dtype=np.int32)
    ne = np.ascontiguousarray(n_emit, dtype=np.int32)
    for a in (k_cache, v_cache, k_blk, v_blk):
        assert a.flags["C_CONTIGUOUS"]
    i32 = ctypes.c_int32
    rc = lib().oracle_kv_commit(_dtype_code(k_cache), _ptr(k_cache), _ptr(v_cache),
                                _ptr(k_blk), _ptr(v_blk), B, Hkv, D, cap, blk,
                                _ptr(lens, i32), _ptr(ne, i32))
    if rc != 0:
        raise ValueError("oracle_kv_commit: bad arguments")
    return lens


# ----------------------------------------------------------------- tiny model

class ModelCfg(ctypes.Structure):
    _fields_ = [("V", ctypes.c_int), ("d", ctypes.c_int), ("L", ctypes.c_int),
                ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("hd", ctypes.c_int),
                ("ffn", ctypes.c_int), ("eps", ctypes.c_double),
                ("rope_theta", ctypes.c_double)]


def model_cfg(V, d, L, Hq, Hkv, hd, ffn, eps=1e-6, rope_theta=1e6) -> ModelCfg:
    return ModelCfg(V, d, L, Hq, Hkv, hd, ffn, eps, rope_theta)


def pack_weights(cfg: ModelCfg, W: dict) -> np.ndarray:
    """Flatten a weight dict into the packing order orthrus_oracle.h documents."""
    parts = [W["embed"]]
    for layer in W["layers"]:
        parts += [layer[k] for k in ("attn_norm", "wq", "wk", "wv", "wo",
                                     "dq", "dk", "dv", "do", "ffn_norm",
                                     "w_gate", "w_up", "w_down")]
    parts += [W["final_norm"], W["lm_head"]]
    flat = np.concatenate([np.asarray(p, dtype=np.float64).ravel() for p in parts])
    assert flat.size == lib().oracle_model_num_weights(ctypes.byref(cfg))
    return flat


class Sequence:
    """One sequence's double-precision KV cache [L][Hkv][cap][hd]."""

    def __init__(self, cfg: ModelCfg, cap: int):
        shape = (cfg.L, cfg.Hkv, cap, cfg.hd)
        self.k = np.zeros(shape, np.float64)
        self.v = np.zeros(shape, np.float64)
        self.cap = cap
        self.n = 0


def forward(cfg, wflat, seq: Sequence, tokens, view, nthreads=0):
    """Logits [rows, V] and block K/V [L, rows, Hkv, hd] for tokens at [n, n+rows)."""
    toks = np.ascontiguousarray(tokens, dtype=np.int32)
    rows = toks.size
    logits = np.zeros((rows, cfg.V), np.float64)
    kb = np.zeros((cfg.L, rows, cfg.Hkv, cfg.hd), np.float64)
    vb = np.zeros_like(kb)
    f64 = ctypes.c_double
    rc = lib().oracle_model_forward(ctypes.byref(cfg), _ptr(wflat, f64), int(view),
                                    _ptr(toks, ctypes.c_int32), rows,
                                    _ptr(seq.k, f64), _ptr(seq.v, f64), seq.cap,
                                    seq.n, _ptr(logits, f64), _ptr(kb, f64),
                                    _ptr(vb, f64), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_model_forward: bad arguments")
    return logits, kb, vb


def commit_rows(seq: Sequence, kb, vb, count: int):
    """Append block rows [0, count) of every layer to the cache (a copy)."""
    n = seq.n
    assert n + count <= seq.cap
    # kb [L, rows, Hkv, hd] -> cache [L, Hkv, n:n+count, hd]
    seq.k[:, :, n:n + count, :] = kb[:, :count].transpose(0, 2, 1, 3)
    seq.v[:, :, n:n + count, :] = vb[:, :count].transpose(0, 2, 1, 3)
    seq.n = n + count


def prefill(cfg, wflat, prompt, cap, nthreads=0):
    """AR causal pass over the prompt; returns (sequence, first generated token)."""
    seq = Sequence(cfg, cap)
    logits, kb, vb = forward(cfg, wflat, seq, prompt, view=0, nthreads=nthreads)
    commit_rows(seq, kb, vb, len(prompt))
    return seq, int(vocab_argmax(logits[-1:])[0])


def greedy_ar(cfg, wflat, prompt, n_new, cap=None, nthreads=0):
    """Plain greedy autoregressive decoding: n_new tokens after the prompt."""
    cap = cap or len(prompt) + n_new + 1
    seq, tok = prefill(cfg, wflat, prompt, cap, nthreads)
    out = [tok]
    while len(out) < n_new:
        logits, kb, vb = forward(cfg, wflat, seq, [tok], view=0, nthreads=nthreads)
        commit_rows(seq, kb, vb, 1)
        tok = int(vocab_argmax(logits)[0])
        out.append(tok)
    return np.array(out[:n_new], np.int32)


def consensus_decode(cfg, wflat, prompt, n_new, blk=32, mask_id=None,
                     draft_fn=None, cap=None, nthreads=0):
    """Orthrus consensus loop (explainer §四), returning (tokens, stats).

    Per round: the diffusion view reads [anchor, MASK x (blk-1)] at positions
    [n, n+blk) and its row argmaxes are the drafts d[0..blk); the AR view
    verifies [anchor, d0..d_{blk-2}] causally, giving a[0..blk); consensus
    accepts the agreeing prefix plus one correction; the accepted rows'
    AR K/V are committed.  ``draft_fn(round_idx, n, d)`` may replace the
    drafts (to check that any draft gives the greedy trajectory).
    """
    if mask_id is None:
        mask_id = cfg.V - 1
    cap = cap or len(prompt) + n_new + 2 * blk
    seq, anchor = prefill(cfg, wflat, prompt, cap, nthreads)
    out = [anchor]
    stats = {"rounds": 0, "accept_len": [], "n_emit": []}
    r = 0
    while len(out) < n_new:
        blk_tokens = [anchor] + [mask_id] * (blk - 1)
        dlog, _, _ = forward(cfg, wflat, seq, blk_tokens, view=1, nthreads=nthreads)
        d = vocab_argmax(dlog)
        if draft_fn is not None:
            d = np.asarray(draft_fn(r, seq.n, d), np.int32)
        vlog, kb, vb = forward(cfg, wflat, seq, [anchor] + list(d[:blk - 1]),
                               view=0, nthreads=nthreads)
        a = vocab_argmax(vlog)
        L, ne, em, na = consensus(d[None, :], a[None, :])
        commit_rows(seq, kb, vb, int(ne[0]))
        out += list(em[0, :ne[0]])
        anchor = int(na[0])
        stats["rounds"] += 1
        stats["accept_len"].append(int(L[0]))
        stats["n_emit"].append(int(ne[0]))
        r += 1
    return np.array(out[:n_new], np.int32), stats
