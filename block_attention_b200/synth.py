"""Seeded synthetic inputs for the decoding-round workloads.

This module only draws numbers and lays them out; it holds none of the
method's arithmetic, so the CUDA path and the CPU oracle can both be fed from
it.  All draws go through numpy's PCG64 seeded by (seed, stream id) so that a
tensor does not change when another one is added.

Workloads (shapes follow Qwen3 attention layers; values are synthetic because
no checkpoint or dataset is used):

* ``tiny``        B=1, Hq=4, Hkv=2, D=64, context 256, block 32, fp32,
                  vocab 1024 logits ~ N(0, 3).
* ``qwen3_1p7b``  B=1, Hq=16, Hkv=8, D=128, context 2048, block 32,
                  bf16 or fp32, vocab 151936.
* ``qwen3_8b``    36 layers, B=1, Hq=32, Hkv=8, D=128, context 8192, block 32,
                  bf16 KV cache, vocab 151936, accepted prefix ~ Geometric(mean 5.4).
* ``ragged``      B=16, context ~ U{1024..32768}, Hq=32, Hkv=8, D=128, bf16.
"""
from __future__ import annotations

import numpy as np

WORKLOADS = {
    "tiny": dict(B=1, Hq=4, Hkv=2, D=64, ctx=256, blk=32, vocab=1024),
    "qwen3_1p7b": dict(B=1, Hq=16, Hkv=8, D=128, ctx=2048, blk=32, vocab=151936),
    "qwen3_8b": dict(B=1, Hq=32, Hkv=8, D=128, ctx=8192, blk=32, vocab=151936,
                     layers=36),
    "ragged": dict(B=16, Hq=32, Hkv=8, D=128, ctx_lo=1024, ctx_hi=32768, blk=32,
                   vocab=151936),
    # end-to-end consensus loop on a random-init Qwen3-style decoder
    "e2e_decoder": dict(V=8192, d=512, L=4, Hq=8, Hkv=4, hd=64, ffn=1536, std=0.02,
                        prompts=256, prompt_lo=64, prompt_hi=512, n_new=256, blk=32),
}

# Stream ids, one per kind of tensor.
S_Q, S_KBLK, S_VBLK, S_KC, S_VC, S_LOGIT, S_TOK, S_LEN, S_ACC, S_W, S_PROMPT = range(11)


def rng(seed: int, *stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, *stream])))


def normal(g: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    x = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def to_bf16(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest even; NaN kept quiet."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    nan = (u & 0x7FFFFFFF) > 0x7F800000
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    r[nan] = ((u[nan] >> 16) | 0x40).astype(np.uint16)
    return r


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def cast(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f32":
        return np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "bf16":
        return to_bf16(x)
    raise ValueError(dtype)


def lm_head_inputs(rows, d, V, seed=0, std_h=1.0, std_w=0.02, slice_rows=8192):
    """Final hidden states h [rows, d] ~ N(0, std_h) and an output embedding
    w [V, d] ~ N(0, std_w) (the usual init scale: logits of std
    sqrt(d) std_h std_w), both as bf16 bit patterns; w is drawn in row slices
    so a vocabulary-sized matrix needs no full-size float32 temporary."""
    h = to_bf16(normal(rng(seed, S_W, 0), (rows, d), std_h))
    w = np.empty((V, d), np.uint16)
    g = rng(seed, S_W, 1)
    for r0 in range(0, V, slice_rows):
        r1 = min(V, r0 + slice_rows)
        w[r0:r1] = to_bf16(normal(g, (r1 - r0, d), std_w))
    return h, w


def attn_inputs(B, Hq, Hkv, D, blk, ctx_lens, cap, dtype="f32", seed=0, layer=0,
                std=1.0, with_cache=True):
    """Q/K/V for one layer of one round: all entries ~ N(0, std).

    Returns q [B, blk, Hq, D], k_blk/v_blk [B, blk, Hkv, D],
    k_cache/v_cache [B, Hkv, cap, D] (rows >= ctx_len are zero), ctx_lens [B].
    """
    ctx_lens = np.asarray(ctx_lens, dtype=np.int32)
    assert ctx_lens.shape == (B,) and int(ctx_lens.max(initial=0)) <= cap
    out = {
        "q": cast(normal(rng(seed, S_Q, layer), (B, blk, Hq, D), std), dtype),
        "k_blk": cast(normal(rng(seed, S_KBLK, layer), (B, blk, Hkv, D), std), dtype),
        "v_blk": cast(normal(rng(seed, S_VBLK, layer), (B, blk, Hkv, D), std), dtype),
        "ctx_lens": ctx_lens,
    }
    if not with_cache:
        return out
    kc = np.zeros((B, Hkv, cap, D), np.float32)
    vc = np.zeros((B, Hkv, cap, D), np.float32)
    gk, gv = rng(seed, S_KC, layer), rng(seed, S_VC, layer)
    for b in range(B):
        n = int(ctx_lens[b])
        kc[b, :, :n] = normal(gk, (Hkv, n, D), std)
        vc[b, :, :n] = normal(gv, (Hkv, n, D), std)
    out["k_cache"] = cast(kc, dtype)
    out["v_cache"] = cast(vc, dtype)
    return out


def ragged_lens(B, lo, hi, seed) -> np.ndarray:
    return rng(seed, S_LEN).integers(lo, hi + 1, size=B).astype(np.int32)


def geometric_accept(g: np.random.Generator, size, mean=5.4, blk=32) -> np.ndarray:
    """Planted accepted-prefix lengths: min(failures before first success, blk)
    with success probability 1/(mean+1), so the uncapped mean is `mean`."""
    p = 1.0 / (mean + 1.0)
    return np.minimum(g.geometric(p, size=size) - 1, blk).astype(np.int32)


def planted_tokens(g: np.random.Generator, B, blk, vocab, accept):
    """(draft, verify) token ids [B, blk] that agree exactly on [0, accept[b])
    and differ at position accept[b] (when < blk); elsewhere independent."""
    accept = np.asarray(accept, np.int32)
    verify = g.integers(0, vocab, size=(B, blk)).astype(np.int32)
    draft = g.integers(0, vocab, size=(B, blk)).astype(np.int32)
    for b in range(B):
        L = int(accept[b])
        draft[b, :L] = verify[b, :L]
        if L < blk:
            shift = int(g.integers(1, vocab))
            draft[b, L] = (verify[b, L] + shift) % vocab
    return draft, verify


def planted_logits(g: np.random.Generator, targets, vocab, std=3.0, spike=40.0,
                   dtype="f32"):
    """Logits ~ N(0, std) per row, with `spike` written at each row's target id,
    so each row's maximum sits at its target (N(0,3) over 151936 draws stays
    below ~20)."""
    t = np.asarray(targets, np.int64).ravel()
    x = normal(g, (t.size, vocab), std)
    x[np.arange(t.size), t] = np.float32(spike)
    return cast(x, dtype)


def logits(g: np.random.Generator, rows, vocab, std=3.0, dtype="f32"):
    return cast(normal(g, (rows, vocab), std), dtype)


# ----------------------------------------------------------- tiny decoder

TINY_DECODER = dict(V=8192, d=512, L=4, Hq=8, Hkv=4, hd=64, ffn=1536)


def decoder_weights(V, d, L, Hq, Hkv, hd, ffn, seed=0, std=0.02):
    """Random-init Qwen3-style decoder: matrices ~ N(0, std) stored W[out][in];
    RMSNorm gains 1 + N(0, std); each layer also has a separate-weight copy of
    the attention projections for the diffusion view (dq, dk, dv, do)."""
    g = rng(seed, S_W)
    qd, kd = Hq * hd, Hkv * hd

    def mat(o, i):
        return normal(g, (o, i), std)

    def gain():
        return (1.0 + normal(g, (d,), std)).astype(np.float32)

    W = {"embed": normal(g, (V, d), std), "layers": []}
    for _ in range(L):
        W["layers"].append({
            "attn_norm": gain(),
            "wq": mat(qd, d), "wk": mat(kd, d), "wv": mat(kd, d), "wo": mat(d, qd),
            "dq": mat(qd, d), "dk": mat(kd, d), "dv": mat(kd, d), "do": mat(d, qd),
            "ffn_norm": gain(),
            "w_gate": mat(ffn, d), "w_up": mat(ffn, d), "w_down": mat(d, ffn),
        })
    W["final_norm"] = gain()
    W["lm_head"] = mat(V, d)
    return W


def prompts(n, vocab, lo, hi, seed, exclude=None):
    """n prompts of uniform-random token ids, lengths ~ U{lo..hi}."""
    g = rng(seed, S_PROMPT)
    lens = g.integers(lo, hi + 1, size=n)
    hi_tok = vocab - 1 if exclude == vocab - 1 else vocab
    return [g.integers(0, hi_tok, size=int(m)).astype(np.int32) for m in lens]
