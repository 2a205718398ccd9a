"""CPU pins of the fused LM-head + argmax oracle (oracle.lm_head_argmax).

The operation: the LM head (the shared output projection every view ends in,
cjcn.com.cn explainer of "Orthrus", §二) followed by the row argmax that
turns the diffusion rows into drafts and the verify rows into the AR tokens
(§四 steps 1-3).  Pinned to: brute-force dot products on tiny inputs,
planted ties (lowest index), a closed form (one-hot output embedding picks
entries of h), exact bf16 widening, and the gap / magnitude properties.
"""
import numpy as np


def _brute(h, w):
    rows, d = h.shape
    V = w.shape[0]
    idx, mx = [], []
    for r in range(rows):
        best, bi = None, -1
        for v in range(V):
            s = 0.0
            for k in range(d):
                s += float(h[r, k]) * float(w[v, k])
            if best is None or s > best:
                best, bi = s, v
        idx.append(bi)
        mx.append(best)
    return np.array(idx), np.array(mx)


def test_matches_brute_force_dot_products(oracle_mod):
    g = np.random.default_rng(21)
    h = g.integers(-8, 9, (3, 8)).astype(np.float64)  # exact in any precision
    w = g.integers(-8, 9, (23, 8)).astype(np.float64)
    idx, mx, gap, mag = oracle_mod.lm_head_argmax(h, w, chunk=5)
    bi, bm = _brute(h, w)
    np.testing.assert_array_equal(idx, bi)
    np.testing.assert_array_equal(mx, bm)


def test_planted_ties_take_the_lowest_index(oracle_mod):
    g = np.random.default_rng(22)
    h = g.normal(0, 1, (4, 16))
    w = g.normal(0, 0.1, (300, 16))
    for r, (lo, hi) in enumerate([(5, 250), (0, 299), (128, 129), (77, 200)]):
        w[lo] = w[hi] = 10 * h[r] / np.linalg.norm(h[r])  # the max of row r, twice
    idx, mx, gap, _ = oracle_mod.lm_head_argmax(h, w, chunk=64)
    np.testing.assert_array_equal(idx, [5, 0, 128, 77])
    np.testing.assert_array_equal(gap, 0.0)


def test_one_hot_output_embedding_picks_entries_of_h(oracle_mod):
    """w[v] = c_v e_{k(v)} gives logits[r, v] = c_v h[r, k(v)]."""
    g = np.random.default_rng(23)
    d, V = 12, 40
    h = g.normal(0, 1, (5, d))
    k_of = g.integers(0, d, V)
    c = g.uniform(0.5, 2.0, V)
    w = np.zeros((V, d))
    w[np.arange(V), k_of] = c
    idx, mx, _, _ = oracle_mod.lm_head_argmax(h, w)
    expect = np.array([int(np.argmax(c * h[r, k_of])) for r in range(5)])
    np.testing.assert_array_equal(idx, expect)
    np.testing.assert_allclose(mx, [c[e] * h[r, k_of[e]] for r, e in enumerate(expect)],
                               rtol=0, atol=0)


def test_bf16_bit_patterns_widen_exactly(oracle_mod):
    g = np.random.default_rng(24)
    hf = g.normal(0, 1, (6, 64)).astype(np.float32)
    wf = g.normal(0, 0.05, (500, 64)).astype(np.float32)
    hb = (hf.view(np.uint32) >> 16).astype(np.uint16)  # truncation: exact bf16 values
    wb = (wf.view(np.uint32) >> 16).astype(np.uint16)
    widen = lambda b: (b.astype(np.uint32) << 16).view(np.float32)
    a = oracle_mod.lm_head_argmax(hb, wb)
    b = oracle_mod.lm_head_argmax(widen(hb), widen(wb))
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


def test_gap_and_magnitude_bound_the_logits(oracle_mod):
    g = np.random.default_rng(25)
    h = g.normal(0, 1, (7, 32))
    w = g.normal(0, 0.1, (1000, 32))
    idx, mx, gap, mag = oracle_mod.lm_head_argmax(h, w, chunk=97)
    logits = h @ w.T
    assert (gap >= 0).all()
    assert (np.abs(logits).max(axis=1) <= mag + 1e-12).all()
    srt = np.sort(logits, axis=1)
    np.testing.assert_allclose(gap, srt[:, -1] - srt[:, -2], rtol=0, atol=1e-12)


def test_every_row_can_win_under_any_slicing(oracle_mod):
    """The maximum planted at each vocabulary row in turn, for slice sizes that
    put it first, last and inside a slice: the product over slices must not
    drop or move any row."""
    g = np.random.default_rng(26)
    V, d = 23, 8
    h = g.normal(0, 1, (1, d))
    base = g.normal(0, 0.1, (V, d))
    for v in range(V):
        w = base.copy()
        w[v] = 10 * h[0] / np.linalg.norm(h[0])
        want = float(h[0] @ w[v])
        for chunk in (1, 2, 5, 7, V, 64):
            idx, mx, _, _ = oracle_mod.lm_head_argmax(h, w, chunk=chunk)
            assert int(idx[0]) == v, (v, chunk)
            # float64 summation order of the library product depends on the slice
            assert abs(mx[0] - want) <= 1e-12 * abs(want), (v, chunk)
