"""Oracle for the stochastic (temperature) variant of the Orthrus consensus.

TEST INFRASTRUCTURE ONLY: imported by tests/, never by the product path.

The cjcn.com.cn explainer of "Orthrus" (section 四) states that for sampling
with a temperature the framework aligns the distributions by strict
rejection sampling, which keeps decoding lossless.  The plainest reading is
standard speculative sampling with the diffusion view as the draft model:

  drafts      d_j ~ q_j = softmax(z_diff[j] / T)            (j = 0 .. blk-1)
  verify      p_j = softmax(z_ar[j] / T), row j of the AR pass over
              [anchor, d_0 .. d_{blk-2}]
  accept      d_j while u_j < p_j(d_j) / q_j(d_j), left to right
  correction  at the first rejected position L: c ~ normalize(max(0, p_L - q_L))
  emit        d_0 .. d_{L-1}, c  (n_emit = L + 1); if every draft is accepted
              the blk drafts (no distribution exists past the block, so no
              bonus token) -- n_emit = min(L + 1, blk) as in the greedy rule

Sampling from a softmax uses the Gumbel-max identity: argmax_k (x_k + g_k),
g_k = -log(-log u_k) with u_k uniform, is distributed as softmax(x).  The
uniforms come from Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel
random numbers: as easy as 1, 2, 3", SC'11), written here from that
definition: key = the 64-bit seed (low word, high word); counter = (x0, x1,
purpose, step) with purpose 1 for draft noise (x0 = vocab index / 4, x1 =
row, word = vocab index % 4), purpose 2 for acceptance (x0 = block position,
x1 = sequence, word 0) and purpose 3 for the correction's noise (x0 = vocab
index / 4, x1 = sequence); a 32-bit word w becomes u = ((w >> 9) + 1/2) 2^-23
(exact in float32, so both sides start from the same value).
Everything after the uniforms is float64, in definition order.
"""
from __future__ import annotations

import numpy as np

PURPOSE_DRAFT, PURPOSE_ACCEPT, PURPOSE_RESIDUAL = 1, 2, 3
_M0, _M1 = np.uint64(0xD2511F53), np.uint64(0xCD9E8D57)
_W0, _W1 = np.uint64(0x9E3779B9), np.uint64(0xBB67AE85)
_MASK = np.uint64(0xFFFFFFFF)


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Ten Philox rounds on (arrays of) 32-bit counters and keys."""
    c = [np.asarray(x, dtype=np.uint64) & _MASK for x in (c0, c1, c2, c3)]
    k0 = np.asarray(k0, dtype=np.uint64) & _MASK
    k1 = np.asarray(k1, dtype=np.uint64) & _MASK
    for _ in range(10):
        p0 = _M0 * c[0]
        p1 = _M1 * c[2]
        hi0, lo0 = p0 >> np.uint64(32), p0 & _MASK
        hi1, lo1 = p1 >> np.uint64(32), p1 & _MASK
        c = [hi1 ^ c[1] ^ k0, lo1, hi0 ^ c[3] ^ k1, lo0]
        k0 = (k0 + _W0) & _MASK
        k1 = (k1 + _W1) & _MASK
    return c


def uniforms(seed: int, step: int, purpose: int, x0, x1, word):
    """Uniforms in (0, 1) for counters (x0, x1, purpose, step), picking `word`."""
    x0 = np.asarray(x0, dtype=np.uint64)
    out = philox4x32_10(x0, np.broadcast_to(np.uint64(x1), x0.shape), purpose, step,
                        seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF)
    w = np.choose(np.asarray(word, dtype=np.int64), out)
    return ((w >> np.uint64(9)).astype(np.float64) + 0.5) * 2.0 ** -23


def _widen(logits):
    x = np.asarray(logits)
    if x.dtype == np.uint16:  # bf16 bit patterns
        x = (x.astype(np.uint32) << 16).view(np.float32)
    return x.astype(np.float64)


def _gumbel(seed, step, purpose, x1, vocab):
    k = np.arange(vocab, dtype=np.int64)
    u = uniforms(seed, step, purpose, k // 4, x1, k % 4)
    return -np.log(-np.log(u))


def vocab_sample(logits, temperature: float, seed: int, step: int):
    """Per row r: argmax_k z[r, k] / T + g_k (lowest index among equal keys),
    g from purpose 1 with x1 = r.  Returns (idx int32 [rows], gap float64
    [rows]) where gap is the distance between the two largest keys (a tie
    within rounding makes the winner precision-dependent)."""
    x = _widen(logits)
    rows, vocab = x.shape
    idx = np.zeros(rows, np.int32)
    gap = np.zeros(rows)
    for r in range(rows):
        key = x[r] / temperature + _gumbel(seed, step, PURPOSE_DRAFT, r, vocab)
        idx[r] = int(np.argmax(key))
        top2 = np.partition(key, -2)[-2:]
        gap[r] = top2[1] - top2[0]
    return idx, gap


def _log_softmax_at(z, k, temperature):
    s = z / temperature
    m = s.max()
    return s[k] - (m + np.log(np.exp(s - m).sum()))


def consensus_sample(draft, logits_ar, logits_diff, temperature: float, seed: int, step: int):
    """Stochastic consensus per sequence.  draft int [B, blk]; logits_* [B*blk,
    vocab] (row b*blk + j).  Returns (accept_len, n_emit, emitted (-1 past
    n_emit), next_anchor, margin) with margin [B] the smallest distance of a
    decision to its threshold: |log u_j - (log p_j - log q_j)| over the tested
    positions, and the correction's top-2 key gap."""
    draft = np.asarray(draft)
    B, blk = draft.shape
    zar, zdf = _widen(logits_ar), _widen(logits_diff)
    vocab = zar.shape[1]
    L = np.zeros(B, np.int32)
    ne = np.zeros(B, np.int32)
    em = np.full((B, blk), -1, np.int32)
    na = np.zeros(B, np.int32)
    margin = np.full(B, np.inf)
    for b in range(B):
        acc = blk
        for j in range(blk):
            r, d = b * blk + j, int(draft[b, j])
            lp = _log_softmax_at(zar[r], d, temperature)
            lq = _log_softmax_at(zdf[r], d, temperature)
            lu = np.log(uniforms(seed, step, PURPOSE_ACCEPT, np.array([j]), b, np.array([0]))[0])
            margin[b] = min(margin[b], abs(lu - (lp - lq)))
            if not lu < lp - lq:
                acc = j
                break
        L[b] = acc
        n = min(acc + 1, blk)
        ne[b] = n
        em[b, :min(acc, n)] = draft[b, :min(acc, n)]
        if acc < blk:
            r = b * blk + acc
            sp, sq = zar[r] / temperature, zdf[r] / temperature
            p = np.exp(sp - sp.max())
            p /= p.sum()
            q = np.exp(sq - sq.max())
            q /= q.sum()
            res = p - q
            g = _gumbel(seed, step, PURPOSE_RESIDUAL, b, vocab)
            pos = res > 0
            if pos.any():
                key = np.where(pos, np.log(np.where(pos, res, 1.0)) + g, -np.inf)
                c = int(np.argmax(key))
                top2 = np.partition(key[pos], -2)[-2:] if pos.sum() > 1 else np.array([-np.inf, key[c]])
                margin[b] = min(margin[b], top2[1] - top2[0])
            else:
                c = int(np.argmax(p))
            em[b, acc] = c
        na[b] = em[b, n - 1]
    return L, ne, em, na, margin
