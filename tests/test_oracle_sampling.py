"""CPU pins of the stochastic-consensus oracle (oracle/sampling.py).

Pinned to things other than the oracle itself:
  * Philox4x32-10 known-answer vectors published with the generator (Salmon,
    Moraes, Dror, Shaw, SC'11; the Random123 distribution's test vectors);
  * Gumbel-max sampling frequencies against softmax(z / T) (chi-square);
  * the defining property of speculative sampling that makes it lossless
    (cjcn.com.cn explainer of "Orthrus", section 四): whatever the draft
    distribution q, the first emitted token is distributed as the AR view's p;
  * the temperature-to-zero limit equals the greedy consensus;
  * identical views accept every draft.
"""
import numpy as np
import pytest
from scipy.stats import chi2

from oracle import sampling as S


@pytest.mark.parametrize("ctr,key,expect", [
    ((0, 0, 0, 0), (0, 0), (0x6627e8d5, 0xe169c58d, 0xbc57ac4c, 0x9b00dbd8)),
    ((0xffffffff,) * 4, (0xffffffff,) * 2, (0x408f276d, 0x41c83b0e, 0xa20bc7c6, 0x6d5451fd)),
    ((0x243f6a88, 0x85a308d3, 0x13198a2e, 0x03707344), (0xa4093822, 0x299f31d0),
     (0xd16cfe09, 0x94fdcceb, 0x5001e420, 0x24126ea1)),
])
def test_philox_known_answers(ctr, key, expect):
    got = tuple(int(w) for w in S.philox4x32_10(*ctr, *key))
    assert got == expect


def test_uniforms_in_open_unit_interval():
    u = S.uniforms(123456789012345, 3, S.PURPOSE_DRAFT, np.arange(4096), 7, np.arange(4096) % 4)
    assert (u > 0).all() and (u < 1).all()
    assert abs(u.mean() - 0.5) < 0.02


def _chi2_pvalue(counts, probs):
    n = counts.sum()
    exp = n * probs
    stat = ((counts - exp) ** 2 / exp).sum()
    return chi2.sf(stat, df=len(probs) - 1)


def _softmax(x):
    e = np.exp(x - x.max())
    return e / e.sum()


def test_gumbel_max_samples_follow_softmax():
    z = np.array([0.3, -1.2, 2.0, 0.0, 0.9, -0.4])
    T = 0.7
    rows = 20000
    idx, _ = S.vocab_sample(np.tile(z, (rows, 1)), T, seed=2024, step=5)
    counts = np.bincount(idx, minlength=z.size).astype(np.float64)
    assert _chi2_pvalue(counts, _softmax(z / T)) > 1e-4


def test_first_emitted_token_follows_ar_distribution():
    """Speculative sampling is lossless: with drafts from q and verification by
    p, the first emitted token is distributed as p (blk = 1 isolates it)."""
    zq = np.array([1.5, 0.2, -0.3, 0.9, -1.0, 0.0])   # diffusion view (draft)
    zp = np.array([-0.2, 1.1, 0.4, -0.8, 0.6, 0.1])   # AR view (verify)
    T = 0.9
    B = 20000
    draft, _ = S.vocab_sample(np.tile(zq, (B, 1)), T, seed=77, step=1)
    L, ne, em, na, _ = S.consensus_sample(draft.reshape(B, 1), np.tile(zp, (B, 1)),
                                          np.tile(zq, (B, 1)), T, seed=77, step=1)
    assert (ne == 1).all()
    counts = np.bincount(em[:, 0], minlength=6).astype(np.float64)
    assert _chi2_pvalue(counts, _softmax(zp / T)) > 1e-4
    # and it is not simply the draft distribution
    assert _chi2_pvalue(counts, _softmax(zq / T)) < 1e-6


def test_low_temperature_equals_greedy_consensus(oracle_mod):
    g = np.random.default_rng(11)
    B, blk, V = 6, 8, 50
    zq = g.normal(0, 1, (B * blk, V))
    zp = g.normal(0, 1, (B * blk, V))
    # plant agreement on a prefix so the accept length varies
    for b in range(B):
        for j in range(b):
            zp[b * blk + j] = zq[b * blk + j]
    T = 1e-3
    draft, _ = S.vocab_sample(zq, T, seed=5, step=0)
    np.testing.assert_array_equal(draft, oracle_mod.vocab_argmax(zq))
    L, ne, em, na, _ = S.consensus_sample(draft.reshape(B, blk), zp, zq, T, seed=5, step=0)
    gL, gne, gem, gna = oracle_mod.consensus(draft.reshape(B, blk),
                                             oracle_mod.vocab_argmax(zp).reshape(B, blk))
    np.testing.assert_array_equal(L, gL)
    np.testing.assert_array_equal(ne, gne)
    np.testing.assert_array_equal(em, gem)
    np.testing.assert_array_equal(na, gna)


def test_identical_views_accept_every_draft():
    g = np.random.default_rng(12)
    B, blk, V = 4, 32, 40
    z = g.normal(0, 2, (B * blk, V))
    draft, _ = S.vocab_sample(z, 1.0, seed=9, step=2)
    L, ne, em, na, _ = S.consensus_sample(draft.reshape(B, blk), z, z, 1.0, seed=9, step=2)
    assert (L == blk).all() and (ne == blk).all()
    np.testing.assert_array_equal(em, draft.reshape(B, blk))
    np.testing.assert_array_equal(na, draft.reshape(B, blk)[:, -1])


def test_token_logprob_temperature_and_lse_match_scipy(oracle_mod):
    """The temperature path of the log-probability (used by the stochastic
    consensus) against scipy's logsumexp of the scaled row."""
    from scipy.special import logsumexp
    g = np.random.default_rng(13)
    x = g.normal(0, 3, (5, 777))
    idx = g.integers(0, 777, 5)
    for T in (0.3, 1.0, 2.5):
        lp, lse = oracle_mod.token_logprob(x, idx, temperature=T, return_lse=True)
        ref_lse = logsumexp(x / T, axis=1)
        np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lp, x[np.arange(5), idx] / T - ref_lse, rtol=0, atol=1e-12)
