"""block_attention_b200 -- B200 (sm_100a) hot path of one Orthrus decoding round.

Thin Python binding over the C ABI in ``include/orthrus.h`` (``liborthrus.so``,
built in-tree by ``block_attention_b200.build``).  Every function here only
marshals torch tensors into pointers and sizes; all arithmetic runs in the
CUDA kernels.  There is no CPU fallback: if the library is missing or a
tensor is not on a CUDA device, the call raises.

Entry points (same names as the C ABI, minus the ``orthrus_`` prefix):
    block_attn      both views' attention over the shared GQA KV cache
    vocab_argmax    per-row argmax, lowest index on ties
    consensus       accepted prefix, tokens to emit, next anchor
    kv_commit       copy accepted block K/V rows into every layer's cache
and the row-invariant decoder building blocks of ``include/orthrus_decoder.h``
(embed, rmsnorm, linear, qkv_rope, swiglu, block_tokens) that
``block_attention_b200.decoder`` composes into the end-to-end consensus loop.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liborthrus.so")

F32, BF16 = 0, 1
BIDIR_BLOCK, CAUSAL_VERIFY = 0, 1
STATUS = {0: "ok", -1: "EINVAL", -2: "EUNSUPPORTED", -3: "EWORKSPACE", -4: "ECAPACITY",
          -5: "ECUDA", -6: "ETIMEOUT"}


class OrthrusError(RuntimeError):
    def __init__(self, fn, code):
        self.code = code
        super().__init__(f"{fn} failed: {STATUS.get(code, code)} ({code})")


class AttnArgs(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int32), ("mask_mode", ctypes.c_int32),
                ("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
                ("D", ctypes.c_int32), ("blk", ctypes.c_int32), ("cap", ctypes.c_int32),
                ("max_ctx", ctypes.c_int32), ("scale", ctypes.c_float),
                ("flags", ctypes.c_int32),
                ("q", ctypes.c_void_p), ("k_blk", ctypes.c_void_p),
                ("v_blk", ctypes.c_void_p), ("k_cache", ctypes.c_void_p),
                ("v_cache", ctypes.c_void_p), ("ctx_lens", ctypes.c_void_p),
                ("out", ctypes.c_void_p), ("err", ctypes.c_void_p),
                ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
                ("next_k_cache", ctypes.c_void_p), ("next_v_cache", ctypes.c_void_p)]


class CommitArgs(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int32), ("layers", ctypes.c_int32),
                ("B", ctypes.c_int32), ("Hkv", ctypes.c_int32), ("D", ctypes.c_int32),
                ("blk", ctypes.c_int32), ("cap", ctypes.c_int32),
                ("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p),
                ("cache_layer_stride", ctypes.c_int64),
                ("k_blk", ctypes.c_void_p), ("v_blk", ctypes.c_void_p),
                ("blk_layer_stride", ctypes.c_int64),
                ("ctx_lens", ctypes.c_void_p), ("n_emit", ctypes.c_void_p),
                ("err", ctypes.c_void_p),
                ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t)]


class SampleArgs(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int32), ("B", ctypes.c_int32), ("blk", ctypes.c_int32),
                ("vocab", ctypes.c_int32), ("row_stride", ctypes.c_int64),
                ("temperature", ctypes.c_float), ("step", ctypes.c_uint32),
                ("seed", ctypes.c_uint64),
                ("draft", ctypes.c_void_p), ("logq", ctypes.c_void_p),
                ("lse_diff", ctypes.c_void_p),
                ("logits_ar", ctypes.c_void_p), ("logits_diff", ctypes.c_void_p),
                ("logp", ctypes.c_void_p), ("lse_ar", ctypes.c_void_p),
                ("accept_len", ctypes.c_void_p), ("n_emit", ctypes.c_void_p),
                ("emitted", ctypes.c_void_p), ("next_anchor", ctypes.c_void_p),
                ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t)]


EXPORTS = ("orthrus_block_attn", "orthrus_block_attn_workspace",
           "orthrus_block_attn_launches", "orthrus_block_attn_plan", "orthrus_vocab_argmax",
           "orthrus_vocab_argmax_workspace", "orthrus_consensus", "orthrus_kv_commit",
           "orthrus_kv_commit_workspace", "orthrus_status_str", "orthrus_version",
           "orthrus_vocab_sample", "orthrus_vocab_sample_workspace", "orthrus_token_logprob", "orthrus_token_logprob_workspace",
           "orthrus_consensus_sample", "orthrus_consensus_sample_workspace",
           "orthrus_lm_head_argmax", "orthrus_lm_head_argmax_workspace",
           "orthrus_lm_head_argmax_plan",
           "orthrus_linear_tc", "orthrus_linear_tc_workspace", "orthrus_linear_tc_plan",
           "orthrus_rope_table", "orthrus_linear_tc_qkv_rope", "orthrus_selftest_bounded_wait",
           # decoder building blocks (include/orthrus_decoder.h)
           "orthrus_embed", "orthrus_rmsnorm", "orthrus_linear", "orthrus_qkv_rope",
           "orthrus_swiglu", "orthrus_block_tokens")

_lib = None


def lib() -> ctypes.CDLL:
    """Load liborthrus.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m block_attention_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        c = ctypes
        vp, i32, i64, sz = c.c_void_p, c.c_int32, c.c_int64, c.c_size_t
        L.orthrus_block_attn.argtypes = [c.POINTER(AttnArgs), vp]
        L.orthrus_block_attn_workspace.argtypes = [c.POINTER(AttnArgs)]
        L.orthrus_block_attn_workspace.restype = sz
        L.orthrus_block_attn_launches.argtypes = [c.POINTER(AttnArgs)]
        L.orthrus_block_attn_launches.restype = c.c_int
        L.orthrus_block_attn_plan.argtypes = [c.POINTER(AttnArgs), i32, vp]
        L.orthrus_block_attn_plan.restype = c.c_int
        L.orthrus_vocab_argmax.argtypes = [i32, vp, i32, i32, i64, vp, vp, vp, sz, vp]
        L.orthrus_vocab_argmax_workspace.argtypes = [i32]
        L.orthrus_vocab_argmax_workspace.restype = sz
        L.orthrus_consensus.argtypes = [vp, vp, i32, i32, vp, vp, vp, vp, vp]
        L.orthrus_kv_commit.argtypes = [c.POINTER(CommitArgs), vp]
        L.orthrus_kv_commit_workspace.argtypes = [c.POINTER(CommitArgs)]
        L.orthrus_kv_commit_workspace.restype = sz
        L.orthrus_status_str.argtypes = [c.c_int]
        L.orthrus_status_str.restype = c.c_char_p
        L.orthrus_version.restype = c.c_int
        L.orthrus_embed.argtypes = [i32, vp, i32, i32, vp, i32, vp, vp, vp]
        L.orthrus_rmsnorm.argtypes = [i32, vp, vp, i32, i32, c.c_float, vp, vp]
        L.orthrus_linear.argtypes = [i32, vp, vp, vp, i32, i32, i32, vp, vp]
        L.orthrus_qkv_rope.argtypes = [i32, vp, i32, i32, i32, i32, i32, vp, c.c_double,
                                       vp, vp, vp, vp]
        L.orthrus_swiglu.argtypes = [i32, vp, i32, i32, vp, vp]
        L.orthrus_block_tokens.argtypes = [vp, vp, i32, i32, i32, vp, vp]
        L.orthrus_token_logprob.argtypes = [i32, vp, i32, i32, i64, vp, c.c_float, vp, vp, vp,
                                            sz, vp]
        L.orthrus_token_logprob_workspace.argtypes = [i32, i32]
        L.orthrus_token_logprob_workspace.restype = sz
        L.orthrus_consensus_sample_workspace.argtypes = [i32, i32, i32]
        L.orthrus_consensus_sample_workspace.restype = sz
        L.orthrus_vocab_sample_workspace.argtypes = [i32, i32]
        L.orthrus_vocab_sample_workspace.restype = sz
        L.orthrus_vocab_sample.argtypes = [i32, vp, i32, i32, i64, c.c_float, c.c_uint64,
                                           c.c_uint32, vp, vp, vp, vp, sz, vp]
        L.orthrus_consensus_sample.argtypes = [c.POINTER(SampleArgs), vp]
        L.orthrus_linear_tc_workspace.argtypes = [i32, i32, i32]
        L.orthrus_linear_tc_workspace.restype = sz
        L.orthrus_linear_tc_plan.argtypes = [i32, i32, i32, i32, vp]
        L.orthrus_linear_tc.argtypes = [i32, vp, i32, i32, i64, vp, i32, vp, vp, i64, vp, i64,
                                        vp, vp, sz, vp]
        L.orthrus_rope_table.argtypes = [vp, i32, i32, i32, c.c_double, vp, vp]
        L.orthrus_selftest_bounded_wait.argtypes = [i32, c.c_uint32, vp, vp, vp]
        L.orthrus_linear_tc_qkv_rope.argtypes = [i32, vp, i32, i32, i64, vp, i32, i32, i32, vp,
                                                 vp, vp, vp, vp, i64, vp, vp, sz, vp]
        L.orthrus_lm_head_argmax_plan.argtypes = [i32, i32, i32, i32, vp]
        L.orthrus_lm_head_argmax_workspace.argtypes = [i32]
        L.orthrus_lm_head_argmax_workspace.restype = sz
        L.orthrus_lm_head_argmax.argtypes = [i32, vp, i32, i32, i64, vp, i32, vp, vp, vp, vp,
                                             sz, vp]
        _lib = L
    return _lib


def _check(fn, rc):
    if rc != 0:
        raise OrthrusError(fn, rc)


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _dev(*ts):
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise ValueError("tensors must be on a CUDA device (no CPU path)")
            if not t.is_contiguous():
                raise ValueError("tensors must be contiguous")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


class Workspace:
    """Zero-initialised device scratch, grown on demand and reused.

    The kernels return their ticket counters to zero, so one workspace serves
    every later call issued on the same stream."""

    def __init__(self, device=None):
        self.device = torch.device(device or "cuda")
        self.buf = torch.zeros(0, dtype=torch.uint8, device=self.device)

    def get(self, nbytes: int) -> torch.Tensor:
        if self.buf.numel() < nbytes:
            self.buf = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=self.device)
        return self.buf


_default_ws = {}


def _ws(ws, device, op):
    """Caller's workspace, else a per-(device, op) default: ops must not share
    one, since argmax/commit keep zeroed ticket counters in theirs."""
    if ws is None:
        dev = device.index if device.index is not None else torch.cuda.current_device()
        ws = _default_ws.setdefault((dev, op), Workspace(torch.device("cuda", dev)))
    return ws


ATTN_EARLY_KV = 1


def attn_args(q, k_blk, v_blk, k_cache, v_cache, ctx_lens, mask_mode, out=None,
              scale=None, max_ctx=None, err=None, flags=0, next_kv=None) -> AttnArgs:
    B, blk, Hq, D = q.shape
    Hkv, cap = k_cache.shape[1], k_cache.shape[2]
    nk = nv = None
    if next_kv is not None:
        nk, nv = next_kv
        if nk.shape != k_cache.shape or nv.shape != v_cache.shape or nk.dtype != k_cache.dtype \
                or nv.dtype != v_cache.dtype or not (nk.is_contiguous() and nv.is_contiguous()):
            raise ValueError("next_kv must be two caches shaped like k_cache and v_cache")
        nk, nv = nk.data_ptr(), nv.data_ptr()
    return AttnArgs(_dtype(q), int(mask_mode), B, Hq, Hkv, D, blk, cap,
                    cap if max_ctx is None else int(max_ctx),
                    float(D ** -0.5 if scale is None else scale), int(flags),
                    q.data_ptr(), k_blk.data_ptr(), v_blk.data_ptr(), k_cache.data_ptr(),
                    v_cache.data_ptr(), ctx_lens.data_ptr(),
                    out.data_ptr() if out is not None else None,
                    err.data_ptr() if err is not None else None, None, 0, nk, nv)


def block_attn_workspace_bytes(args: AttnArgs) -> int:
    return lib().orthrus_block_attn_workspace(ctypes.byref(args))


def block_attn(q, k_blk, v_blk, k_cache, v_cache, ctx_lens, mask_mode, *, out=None,
               scale=None, max_ctx=None, err=None, workspace=None, stream=None, flags=0,
               next_kv=None):
    """Attention of one layer for one round (see orthrus.h for the definition).

    q [B, blk, Hq, D]; k_blk/v_blk [B, blk, Hkv, D]; k_cache/v_cache
    [B, Hkv, cap, D]; ctx_lens int32 [B] on the device.  max_ctx bounds every
    ctx_lens entry (default: cap).  next_kv = (k_cache, v_cache) of the call
    that follows on the stream: warmed into L2 while this one runs (a hint;
    results unchanged).  Returns out [B, blk, Hq, D] (q's dtype)."""
    _dev(q, k_blk, v_blk, k_cache, v_cache, ctx_lens, out, err)
    if ctx_lens.dtype != torch.int32:
        raise TypeError("ctx_lens must be int32")
    if out is None:
        out = torch.empty_like(q)
    a = attn_args(q, k_blk, v_blk, k_cache, v_cache, ctx_lens, mask_mode, out, scale,
                  max_ctx, err, flags, next_kv)
    need = block_attn_workspace_bytes(a)
    if need:
        # scratch for the split partials; one default buffer per device
        buf = _ws(workspace, q.device, "attn").get(need)
        a.workspace, a.workspace_bytes = buf.data_ptr(), buf.numel()
    _check("orthrus_block_attn", lib().orthrus_block_attn(ctypes.byref(a), _stream(stream)))
    return out


def vocab_argmax(logits, *, idx=None, maxval=None, workspace=None, stream=None):
    """Row argmax of logits [rows, vocab] (row stride may exceed vocab)."""
    _dev(idx, maxval)
    if not logits.is_cuda or logits.dim() != 2 or logits.stride(1) != 1:
        raise ValueError("logits must be a 2-D CUDA tensor with unit column stride")
    rows, vocab = logits.shape
    if idx is None:
        idx = torch.empty(rows, dtype=torch.int32, device=logits.device)
    need = lib().orthrus_vocab_argmax_workspace(rows)
    buf = _ws(workspace, logits.device, "argmax").get(need)
    _check("orthrus_vocab_argmax", lib().orthrus_vocab_argmax(
        _dtype(logits), _ptr(logits), rows, vocab, logits.stride(0), _ptr(idx), _ptr(maxval),
        _ptr(buf), buf.numel(), _stream(stream)))
    return idx


def consensus(draft, verify, *, accept_len=None, n_emit=None, emitted=None,
              next_anchor=None, stream=None):
    """Returns (accept_len [B], n_emit [B], emitted [B, blk], next_anchor [B])."""
    _dev(draft, verify)
    B, blk = draft.shape
    dev = draft.device
    mk = lambda t, shp: t if t is not None else torch.empty(shp, dtype=torch.int32, device=dev)
    accept_len, n_emit, next_anchor = mk(accept_len, B), mk(n_emit, B), mk(next_anchor, B)
    emitted = mk(emitted, (B, blk))
    _check("orthrus_consensus", lib().orthrus_consensus(
        _ptr(draft), _ptr(verify), B, blk, _ptr(accept_len), _ptr(n_emit), _ptr(emitted),
        _ptr(next_anchor), _stream(stream)))
    return accept_len, n_emit, emitted, next_anchor


def kv_commit(k_cache, v_cache, k_blk, v_blk, ctx_lens, n_emit, *, err=None,
              workspace=None, stream=None):
    """Commit accepted rows for all layers and advance ctx_lens in place.

    k_cache/v_cache [layers, B, Hkv, cap, D] (or [B, Hkv, cap, D] for one
    layer); k_blk/v_blk [layers, B, blk, Hkv, D] (or [B, blk, Hkv, D])."""
    _dev(k_cache, v_cache, k_blk, v_blk, ctx_lens, n_emit, err)
    if k_cache.dim() == 4:
        k_cache, v_cache = k_cache[None], v_cache[None]
        k_blk, v_blk = k_blk[None], v_blk[None]
    layers, B, Hkv, cap, D = k_cache.shape
    blk = k_blk.shape[2]
    a = CommitArgs(_dtype(k_cache), layers, B, Hkv, D, blk, cap, k_cache.data_ptr(),
                   v_cache.data_ptr(), k_cache.stride(0), k_blk.data_ptr(), v_blk.data_ptr(),
                   k_blk.stride(0), ctx_lens.data_ptr(), n_emit.data_ptr(),
                   err.data_ptr() if err is not None else None, None, 0)
    need = lib().orthrus_kv_commit_workspace(ctypes.byref(a))
    buf = _ws(workspace, k_cache.device, "commit").get(need)
    a.workspace, a.workspace_bytes = buf.data_ptr(), buf.numel()
    _check("orthrus_kv_commit", lib().orthrus_kv_commit(ctypes.byref(a), _stream(stream)))
    return ctx_lens


# ------------------------------------------------- decoder building blocks

def embed(table, tokens, *, out=None, err=None, stream=None):
    """out [rows, d] = table[tokens] (tokens int32 [rows])."""
    _dev(table, tokens, out, err)
    V, d = table.shape
    rows = tokens.numel()
    if out is None:
        out = torch.empty(rows, d, dtype=table.dtype, device=table.device)
    _check("orthrus_embed", lib().orthrus_embed(_dtype(table), _ptr(table), V, d, _ptr(tokens),
                                                rows, _ptr(out), _ptr(err), _stream(stream)))
    return out


def rmsnorm(x, gain, eps, *, out=None, stream=None):
    """Row-wise RMSNorm of x [rows, d] with gain [d] (out may be x)."""
    _dev(x, gain, out)
    d = x.shape[-1]
    rows = x.numel() // d
    if out is None:
        out = torch.empty_like(x)
    _check("orthrus_rmsnorm", lib().orthrus_rmsnorm(_dtype(x), _ptr(x), _ptr(gain), rows, d,
                                                    float(eps), _ptr(out), _stream(stream)))
    return out


def linear(x, w, *, residual=None, out=None, stream=None):
    """out [rows, N] = residual + x [rows, K] @ w[N, K]^T (out may be residual)."""
    _dev(x, w, residual, out)
    N, K = w.shape
    rows = x.numel() // K
    if out is None:
        out = torch.empty(rows, N, dtype=x.dtype, device=x.device)
    _check("orthrus_linear", lib().orthrus_linear(_dtype(x), _ptr(x), _ptr(w), _ptr(residual),
                                                  rows, K, N, _ptr(out), _stream(stream)))
    return out


def qkv_rope(qkv, ctx_lens, B, blk, Hq, Hkv, hd, theta, *, q, k, v, stream=None):
    """Split qkv [B*blk, (Hq+2Hkv)*hd] into q/k/v with RoPE at ctx_lens[b] + j."""
    _dev(qkv, ctx_lens, q, k, v)
    _check("orthrus_qkv_rope", lib().orthrus_qkv_rope(
        _dtype(qkv), _ptr(qkv), B, blk, Hq, Hkv, hd, _ptr(ctx_lens), float(theta), _ptr(q),
        _ptr(k), _ptr(v), _stream(stream)))
    return q, k, v


def swiglu(gu, *, out=None, stream=None):
    """out [rows, F] = silu(gu[:, :F]) * gu[:, F:]."""
    _dev(gu, out)
    rows, F2 = gu.shape
    if out is None:
        out = torch.empty(rows, F2 // 2, dtype=gu.dtype, device=gu.device)
    _check("orthrus_swiglu", lib().orthrus_swiglu(_dtype(gu), _ptr(gu), rows, F2 // 2,
                                                  _ptr(out), _stream(stream)))
    return out


def block_tokens(anchor, draft, blk, mask_id, *, out=None, stream=None):
    """[anchor, MASK...] (draft None) or [anchor, draft[:, :blk-1]] as int32 [B, blk]."""
    _dev(anchor, draft, out)
    B = anchor.numel()
    if out is None:
        out = torch.empty(B, blk, dtype=torch.int32, device=anchor.device)
    _check("orthrus_block_tokens", lib().orthrus_block_tokens(
        _ptr(anchor), _ptr(draft), B, blk, int(mask_id), _ptr(out), _stream(stream)))
    return out


def token_logprob(logits, idx, *, temperature=1.0, out=None, lse=None, workspace=None,
                  stream=None):
    """float [rows]: log-softmax of logits [rows, vocab] / temperature at idx
    (int32 [rows]); fills lse [rows] with each row's log-sum-exp if given."""
    _dev(idx, out, lse)
    if not logits.is_cuda or logits.dim() != 2 or logits.stride(1) != 1:
        raise ValueError("logits must be a 2-D CUDA tensor with unit column stride")
    rows, vocab = logits.shape
    if out is None:
        out = torch.empty(rows, dtype=torch.float32, device=logits.device)
    need = lib().orthrus_token_logprob_workspace(rows, vocab)
    buf = _ws(workspace, logits.device, "logprob").get(need)
    _check("orthrus_token_logprob", lib().orthrus_token_logprob(
        _dtype(logits), _ptr(logits), rows, vocab, logits.stride(0), _ptr(idx),
        float(temperature), _ptr(out), _ptr(lse), _ptr(buf), buf.numel(), _stream(stream)))
    return out


def vocab_sample(logits, temperature, seed, step, *, idx=None, logprob=None, lse=None,
                 workspace=None, stream=None):
    """int32 [rows]: one sample per row of softmax(logits / temperature)
    (Gumbel-max, Philox stream of orthrus.h; purpose 1, x1 = row).  Given
    float32 [rows] tensors ``logprob`` / ``lse``, the same pass also writes the
    sample's log-probability and the row's log-sum-exp at that temperature."""
    _dev(idx, logprob, lse)
    if not logits.is_cuda or logits.dim() != 2 or logits.stride(1) != 1:
        raise ValueError("logits must be a 2-D CUDA tensor with unit column stride")
    rows, vocab = logits.shape
    if idx is None:
        idx = torch.empty(rows, dtype=torch.int32, device=logits.device)
    need = lib().orthrus_vocab_sample_workspace(rows, vocab)
    buf = _ws(workspace, logits.device, "sample").get(need)
    _check("orthrus_vocab_sample", lib().orthrus_vocab_sample(
        _dtype(logits), _ptr(logits), rows, vocab, logits.stride(0), float(temperature),
        int(seed) & (2 ** 64 - 1), int(step) & 0xFFFFFFFF, _ptr(idx), _ptr(logprob), _ptr(lse),
        _ptr(buf), buf.numel(), _stream(stream)))
    return idx


def consensus_sample(draft, logits_ar, logits_diff, logq, lse_diff, temperature, seed, step, *,
                     logp=None, lse_ar=None, accept_len=None, n_emit=None, emitted=None,
                     next_anchor=None, workspace=None, stream=None):
    """Stochastic consensus (see orthrus.h).  draft int32 [B, blk]; logits_*
    [B*blk, vocab]; logq / lse_diff float32 [B*blk], the logprob / lse outputs
    of vocab_sample on logits_diff at the same temperature.  Writes log p and
    the AR rows' log-sum-exp into ``logp`` / ``lse_ar`` (allocated if None).
    Returns (accept_len, n_emit, emitted, next_anchor)."""
    _dev(draft, logq, lse_diff, logp, lse_ar)
    B, blk = draft.shape
    rows, vocab = logits_ar.shape
    if logits_diff.shape != logits_ar.shape or logits_ar.stride(1) != 1 or \
            logits_diff.stride(0) != logits_ar.stride(0):
        raise ValueError("logit matrices must share shape and row stride")
    dev = draft.device
    mk = lambda t, shp, dt=torch.int32: t if t is not None else torch.empty(shp, dtype=dt,
                                                                            device=dev)
    accept_len, n_emit, next_anchor = mk(accept_len, B), mk(n_emit, B), mk(next_anchor, B)
    emitted = mk(emitted, (B, blk))
    logp, lse_ar = mk(logp, rows, torch.float32), mk(lse_ar, rows, torch.float32)
    a = SampleArgs(_dtype(logits_ar), B, blk, vocab, logits_ar.stride(0), float(temperature),
                   int(step) & 0xFFFFFFFF, int(seed) & (2 ** 64 - 1), draft.data_ptr(),
                   logq.data_ptr(), lse_diff.data_ptr(), logits_ar.data_ptr(),
                   logits_diff.data_ptr(), logp.data_ptr(), lse_ar.data_ptr(),
                   accept_len.data_ptr(), n_emit.data_ptr(), emitted.data_ptr(),
                   next_anchor.data_ptr())
    need = lib().orthrus_consensus_sample_workspace(B, blk, vocab)
    buf = _ws(workspace, dev, "consensus_sample").get(need)
    a.workspace, a.workspace_bytes = buf.data_ptr(), buf.numel()
    _check("orthrus_consensus_sample", lib().orthrus_consensus_sample(ctypes.byref(a),
                                                                      _stream(stream)))
    return accept_len, n_emit, emitted, next_anchor


def lm_head_argmax(h, w, *, idx=None, maxval=None, err=None, workspace=None, stream=None):
    """int32 [rows]: argmax_v of h @ w.T per row (lowest index on ties), the
    logits never materialised (see orthrus.h).  h bf16 [rows, d] (unit column
    stride), w bf16 [vocab, d] contiguous; ``maxval`` float32 [rows] receives
    the maximum logit when given."""
    _dev(w, idx, maxval, err)  # h may be a row-strided view
    if not h.is_cuda:
        raise ValueError("tensors must be on a CUDA device (no CPU path)")
    if h.dim() != 2 or w.dim() != 2 or h.stride(1) != 1 or not w.is_contiguous():
        raise ValueError("h must be 2-D with unit column stride, w 2-D contiguous")
    rows, d = h.shape
    if w.shape[1] != d:
        raise ValueError("h and w disagree on the hidden size")
    if idx is None:
        idx = torch.empty(rows, dtype=torch.int32, device=h.device)
    buf = _ws(workspace, h.device, "lm_head").get(lib().orthrus_lm_head_argmax_workspace(rows))
    _check("orthrus_lm_head_argmax", lib().orthrus_lm_head_argmax(
        _dtype(h), _ptr(h), rows, d, h.stride(0), _ptr(w), w.shape[0], _ptr(idx),
        _ptr(maxval), _ptr(err), _ptr(buf), buf.numel(), _stream(stream)))
    return idx


def rope_table(ctx_lens, B, blk, hd, theta, *, out=None, stream=None):
    """float32 [B*blk, hd/2, 2] (cos, sin) of RoPE at positions ctx_lens[b] + j
    (orthrus_rope_table)."""
    _dev(out)
    if not ctx_lens.is_cuda or ctx_lens.dtype != torch.int32:
        raise ValueError("ctx_lens must be an int32 CUDA tensor")
    if out is None:
        out = torch.empty(B * blk, hd // 2, 2, dtype=torch.float32, device=ctx_lens.device)
    if out.numel() != B * blk * hd or not out.is_contiguous() or out.dtype != torch.float32:
        raise ValueError("out must be contiguous float32 with B*blk*hd elements")
    _check("orthrus_rope_table", lib().orthrus_rope_table(
        _ptr(ctx_lens), B, blk, hd, ctypes.c_double(theta), _ptr(out), _stream(stream)))
    return out


def _l2_hint(t):
    """(pointer, bytes) of an optional L2 warm-up hint tensor."""
    if t is None:
        return None, 0
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("l2_next must be a contiguous CUDA tensor")
    return _ptr(t), t.numel() * t.element_size() // 16 * 16


def linear_tc_qkv_rope(x, w, Hq, Hkv, cos_sin, *, q, k, v, l2_next=None, err=None,
                       workspace=None, stream=None):
    """The QKV projection of x (bf16 [rows, K]) by w (bf16 [(Hq + 2 Hkv) * 128, K])
    with RoPE (table `cos_sin` from rope_table) and the head split in its
    epilogue: q [rows, Hq, 128], k / v [rows, Hkv, 128] (see orthrus.h).
    l2_next: a tensor a later call reads, to warm L2 with (a hint)."""
    _dev(w, cos_sin, q, k, v, err)
    if not x.is_cuda:
        raise ValueError("tensors must be on a CUDA device (no CPU path)")
    if x.dim() != 2 or w.dim() != 2 or x.stride(1) != 1 or not w.is_contiguous():
        raise ValueError("x must be 2-D with unit column stride, w 2-D contiguous")
    rows, K = x.shape
    hd = 128
    N = (Hq + 2 * Hkv) * hd
    if tuple(w.shape) != (N, K):
        raise ValueError("w must be [(Hq + 2 Hkv) * 128, K]")
    for t, h in ((q, Hq), (k, Hkv), (v, Hkv)):
        if t.numel() != rows * h * hd or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous [rows, heads, 128]")
    buf = _ws(workspace, x.device, "linear").get(lib().orthrus_linear_tc_workspace(rows, K, N))
    hp, hb = _l2_hint(l2_next)
    _check("orthrus_linear_tc_qkv_rope", lib().orthrus_linear_tc_qkv_rope(
        _dtype(x), _ptr(x), rows, K, x.stride(0), _ptr(w), Hq, Hkv, hd, _ptr(cos_sin), _ptr(q),
        _ptr(k), _ptr(v), hp, hb, _ptr(err), _ptr(buf), buf.numel(), _stream(stream)))
    return q, k, v


def selftest_bounded_wait(which, timeout_us, *, err, never=None, stream=None):
    """Run one wait that never completes (0: an mbarrier phase, 1: the
    generation word `never`) and let it give up after timeout_us: err (int32
    CUDA tensor) receives ORTHRUS_ETIMEOUT (see orthrus.h)."""
    _dev(err, never)
    _check("orthrus_selftest_bounded_wait", lib().orthrus_selftest_bounded_wait(
        which, timeout_us, _ptr(never), _ptr(err), _stream(stream)))
    return err


def linear_tc(x, w, *, residual=None, out=None, l2_next=None, err=None, workspace=None,
              stream=None):
    """bf16 [rows, N] = x @ w.T on the tensor cores (plus the residual, each
    sum rounded to bf16 first; see orthrus.h).  x bf16 [rows, K] (unit
    column stride), w bf16 [N, K] contiguous, residual/out bf16 [rows, N]
    with unit column stride (out may be the residual).  l2_next: a tensor a
    later call reads, to warm L2 with (a hint)."""
    _dev(w, residual, out, err)
    if not x.is_cuda:
        raise ValueError("tensors must be on a CUDA device (no CPU path)")
    if x.dim() != 2 or w.dim() != 2 or x.stride(1) != 1 or not w.is_contiguous():
        raise ValueError("x must be 2-D with unit column stride, w 2-D contiguous")
    rows, K = x.shape
    N = w.shape[0]
    if w.shape[1] != K:
        raise ValueError("x and w disagree on K")
    if out is None:
        out = torch.empty(rows, N, dtype=x.dtype, device=x.device)
    if out.shape != (rows, N) or out.stride(1) != 1:
        raise ValueError("out must be [rows, N] with unit column stride")
    if residual is not None and (residual.shape != (rows, N) or residual.stride() != out.stride()):
        raise ValueError("residual must be laid out like out")
    buf = _ws(workspace, x.device, "linear").get(lib().orthrus_linear_tc_workspace(rows, K, N))
    hp, hb = _l2_hint(l2_next)
    _check("orthrus_linear_tc", lib().orthrus_linear_tc(
        _dtype(x), _ptr(x), rows, K, x.stride(0), _ptr(w), N, _ptr(residual), _ptr(out),
        out.stride(0), hp, hb, _ptr(err), _ptr(buf), buf.numel(), _stream(stream)))
    return out
