"""Pins of the oracle's bf16 projection (the QKV and output projections of the
attention block) and of its bf16 rounding: brute force on tiny inputs,
closed forms (identity and one-hot weights, a zero input with a residual),
rounding ties to even, and every bf16 value mapping to itself."""
import itertools

import numpy as np

from block_attention_b200 import synth


def _bits(a):
    return synth.to_bf16(np.asarray(a, np.float32))


def _f(bits):
    return (np.asarray(bits, np.uint32) << 16).view(np.float32).astype(np.float64)


def _bf16_value_brute(v):
    """Nearest bf16 to v by scanning the neighbouring representable values
    (ties to the even mantissa)."""
    if v == 0:
        return 0.0
    e = int(np.floor(np.log2(abs(v))))
    step = 2.0 ** (e - 7)
    lo = np.floor(v / step) * step
    cands = [lo - step, lo, lo + step, lo + 2 * step]
    best = min(cands, key=lambda c: (abs(c - v), int(round(abs(c) / 2.0 ** (int(np.floor(np.log2(abs(c)))) - 7))) % 2 if c else 0))
    return best


def test_round_bf16_is_identity_on_bf16_values(oracle_mod):
    bits = np.arange(0, 0x7F80, 7, dtype=np.uint16)  # positive finite normals and zero
    bits = bits[(bits >= 0x0080) | (bits == 0)]
    both = np.concatenate([bits, bits | 0x8000])
    np.testing.assert_array_equal(oracle_mod.round_bf16(_f(both)), both)


def test_round_bf16_ties_to_even_and_brute_force(oracle_mod):
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: the even mantissa (1) wins;
    # 1 + 3 * 2^-8 lies halfway between 1 + 2^-7 and 1 + 2^-6: 1 + 2^-6 wins
    np.testing.assert_array_equal(oracle_mod.round_bf16([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8]),
                                  _bits([1.0, 1 + 2.0 ** -6]))
    g = np.random.default_rng(7)
    v = g.normal(size=400) * 10.0 ** g.integers(-3, 4, size=400)
    got = _f(oracle_mod.round_bf16(v))
    want = np.array([_bf16_value_brute(x) for x in v])
    np.testing.assert_array_equal(got, want)


def test_projection_matches_brute_force_sums(oracle_mod):
    g = np.random.default_rng(3)
    R, K, N = 3, 5, 4
    x, w = _bits(g.normal(size=(R, K))), _bits(g.normal(size=(N, K)))
    res = _bits(g.normal(size=(R, N)))
    y, exact, mag = oracle_mod.projection(x, w)
    yr, _, _ = oracle_mod.projection(x, w, res)
    X, W, Rs = _f(x), _f(w), _f(res)
    for r, n in itertools.product(range(R), range(N)):
        s = sum(X[r, k] * W[n, k] for k in range(K))
        assert exact[r, n] == s
        assert mag[r, n] == sum(abs(X[r, k]) * abs(W[n, k]) for k in range(K))
        assert _f(y[r, n]) == _bf16_value_brute(s)
        assert _f(yr[r, n]) == _bf16_value_brute(Rs[r, n] + _bf16_value_brute(s))


def test_projection_closed_forms(oracle_mod):
    g = np.random.default_rng(4)
    K = 64
    x = _bits(g.normal(size=(6, K)))
    y, _, _ = oracle_mod.projection(x, _bits(np.eye(K)))       # identity weights
    np.testing.assert_array_equal(y, x)
    perm = g.permutation(K)
    y, _, _ = oracle_mod.projection(x, _bits(np.eye(K)[perm]))  # a permutation
    np.testing.assert_array_equal(y, x[:, perm])
    res = _bits(g.normal(size=(6, 8)))
    y, _, _ = oracle_mod.projection(_bits(np.zeros((6, K))), _bits(g.normal(size=(8, K))), res)
    np.testing.assert_array_equal(y, res)                       # zero input: the residual
