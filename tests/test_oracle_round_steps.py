"""Pins for the oracle's vocab argmax, prefix consensus and KV commit.

* argmax: numpy's argmax (a library routine that returns the first maximum)
  on finite rows, numpy's nanargmax on rows with NaN; planted ties; +0/-0.
* consensus (Orthrus explainer §四): every output is checked against the
  properties that define it -- the accepted prefix agrees, the next position
  disagrees, at least one token per round, a perfect draft takes the whole
  block -- exhaustively over every (draft, verify) pair of a tiny block.
* commit (explainer §四 notebook update, §七 constant block state): the
  accepted rows are copied, nothing else in the cache changes, and a full
  block of the 8B shape moves exactly the 4.5 MiB the explainer quotes.
"""
import itertools
import json
import os

import numpy as np
import pytest

from block_attention_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_argmax_matches_numpy_first_maximum(oracle_mod, dtype):
    g = synth.rng(21)
    x = synth.logits(g, 37, 1000, dtype=dtype)
    # plant exact ties at the max on some rows
    xf = synth.bf16_to_f32(x) if dtype == "bf16" else x
    for r in range(0, 37, 3):
        j, k = sorted(g.choice(1000, 2, replace=False))
        big = np.float32(50.0)
        if dtype == "bf16":
            x[r, j] = x[r, k] = synth.to_bf16(np.array([big]))[0]
        else:
            x[r, j] = x[r, k] = big
    xf = synth.bf16_to_f32(x) if dtype == "bf16" else x
    idx, mx = oracle_mod.vocab_argmax(x, return_max=True)
    np.testing.assert_array_equal(idx, np.argmax(xf, axis=1))
    np.testing.assert_array_equal(mx, xf.max(axis=1).astype(np.float64))


def test_argmax_all_equal_row_is_zero(oracle_mod):
    x = np.full((3, 17), 2.5, np.float32)
    assert list(oracle_mod.vocab_argmax(x)) == [0, 0, 0]


def test_argmax_signed_zero_ties_take_lower_index(oracle_mod):
    x = np.full((2, 4), -1.0, np.float32)
    x[0, 1], x[0, 2] = -0.0, 0.0
    x[1, 1], x[1, 2] = 0.0, -0.0
    assert list(oracle_mod.vocab_argmax(x)) == [1, 1]


def test_argmax_nan_never_wins(oracle_mod):
    g = synth.rng(22)
    x = synth.logits(g, 8, 64)
    x[:, ::5] = np.nan
    x[3, :] = np.nan
    x[5, 0] = np.nan
    idx = oracle_mod.vocab_argmax(x)
    for r in range(8):
        if r == 3:
            assert idx[r] == 0  # all-NaN row
        else:
            assert idx[r] == np.nanargmax(x[r])


def _check_consensus(d, a, L, ne, em, na):
    blk = d.size
    assert 0 <= L <= blk
    assert np.array_equal(d[:L], a[:L])
    if L < blk:
        assert d[L] != a[L]
    assert ne == min(L + 1, blk) and ne >= 1
    assert np.array_equal(em[:ne], a[:ne]) and np.all(em[ne:] == -1)
    assert na == a[ne - 1]


def test_consensus_exhaustive_tiny_block(oracle_mod):
    blk = 4
    seqs = np.array(list(itertools.product([0, 1], repeat=blk)), np.int32)
    D = np.repeat(seqs, len(seqs), axis=0)
    A = np.tile(seqs, (len(seqs), 1))
    L, ne, em, na = oracle_mod.consensus(D, A)
    for b in range(len(D)):
        _check_consensus(D[b], A[b], L[b], ne[b], em[b], na[b])


def test_consensus_planted_prefix(oracle_mod):
    g = synth.rng(23)
    acc = g.integers(0, 33, size=200).astype(np.int32)
    d, a = synth.planted_tokens(g, 200, 32, 1024, acc)
    L, ne, em, na = oracle_mod.consensus(d, a)
    np.testing.assert_array_equal(L, acc)
    for b in range(200):
        _check_consensus(d[b], a[b], L[b], ne[b], em[b], na[b])


def test_consensus_perfect_draft_accepts_whole_block(oracle_mod):
    a = synth.rng(24).integers(0, 151936, size=(5, 32)).astype(np.int32)
    L, ne, em, na = oracle_mod.consensus(a.copy(), a)
    assert np.all(L == 32) and np.all(ne == 32)
    np.testing.assert_array_equal(em, a)
    np.testing.assert_array_equal(na, a[:, -1])


def test_consensus_always_wrong_draft_emits_one(oracle_mod):
    a = synth.rng(25).integers(0, 100, size=(4, 32)).astype(np.int32)
    L, ne, em, na = oracle_mod.consensus((a + 1) % 100, a)
    assert np.all(L == 0) and np.all(ne == 1)
    np.testing.assert_array_equal(em[:, 0], a[:, 0])
    np.testing.assert_array_equal(na, a[:, 0])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_commit_copies_only_accepted_rows(oracle_mod, dtype):
    B, Hkv, cap, D, blk = 3, 2, 40, 8, 6
    g = synth.rng(26)
    kc = synth.cast(synth.normal(g, (B, Hkv, cap, D)), dtype)
    vc = synth.cast(synth.normal(g, (B, Hkv, cap, D)), dtype)
    kb = synth.cast(synth.normal(g, (B, blk, Hkv, D)), dtype)
    vb = synth.cast(synth.normal(g, (B, blk, Hkv, D)), dtype)
    lens = np.array([0, 17, 34], np.int32)
    ne = np.array([6, 0, 3], np.int32)
    k0, v0 = kc.copy(), vc.copy()
    new = oracle_mod.kv_commit(kc, vc, kb, vb, lens, ne)
    np.testing.assert_array_equal(new, lens + ne)
    for b in range(B):
        n, e = lens[b], ne[b]
        np.testing.assert_array_equal(kc[b, :, n:n + e], kb[b, :e].transpose(1, 0, 2))
        np.testing.assert_array_equal(vc[b, :, n:n + e], vb[b, :e].transpose(1, 0, 2))
        mask = np.ones(cap, bool)
        mask[n:n + e] = False
        np.testing.assert_array_equal(kc[b][:, mask], k0[b][:, mask])
        np.testing.assert_array_equal(vc[b][:, mask], v0[b][:, mask])


def test_commit_rejects_overflow(oracle_mod):
    kc = np.zeros((1, 1, 10, 4), np.float32)
    kb = np.zeros((1, 4, 1, 4), np.float32)
    with pytest.raises(ValueError):
        oracle_mod.kv_commit(kc, kc.copy(), kb, kb.copy(), [8], [3])


def test_commit_full_block_bytes_match_explainer_figure(oracle_mod):
    """Explainer §七: the only extra KV state is the 32-slot block, ~4.5 MiB for
    Qwen3-8B.  One full-accept commit across all layers moves exactly the block
    state: 36 layers x 32 rows x 8 kv-heads x 128 dims x (K,V) x 2 bytes."""
    fig = json.load(open(os.path.join(GOLDEN, "pages_figures.json")))
    shp = fig["qwen3_8b_shape"]
    kc = np.zeros((1, shp["Hkv"], 40, shp["D"]), np.uint16)
    vc = np.zeros_like(kc)
    g = synth.rng(27)
    kb = synth.to_bf16(synth.normal(g, (1, 32, shp["Hkv"], shp["D"])))
    vb = synth.to_bf16(synth.normal(g, (1, 32, shp["Hkv"], shp["D"])))
    before = kc.copy(), vc.copy()
    oracle_mod.kv_commit(kc, vc, kb, vb, [0], [32])
    changed_rows = (np.any(kc != before[0], axis=-1).sum()
                    + np.any(vc != before[1], axis=-1).sum())
    per_layer_bytes = int(changed_rows) * shp["D"] * 2
    assert per_layer_bytes * shp["layers"] == fig["block_state_bytes"]["value"]
    assert fig["block_state_bytes"]["value"] == 4.5 * 2 ** 20


# ---------------------------------------------------------- token log-prob

def test_token_logprob_matches_scipy_logsumexp(oracle_mod):
    from scipy.special import logsumexp
    g = np.random.default_rng(7)
    x = g.normal(0, 3, (6, 1000))
    idx = g.integers(0, 1000, 6)
    got = oracle_mod.token_logprob(x, idx)
    ref = x[np.arange(6), idx] - logsumexp(x, axis=1)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_token_logprob_closed_forms(oracle_mod):
    V = 512
    # uniform row: every token has probability 1/V
    np.testing.assert_allclose(oracle_mod.token_logprob(np.zeros((1, V)), [17]), [-np.log(V)],
                               atol=1e-12)
    # shifting a row leaves log-probabilities unchanged; a dominant logit -> ~0
    x = np.random.default_rng(8).normal(0, 1, (2, V))
    x[1] = x[0] + 123.0
    lp = oracle_mod.token_logprob(x, [5, 5])
    assert abs(lp[0] - lp[1]) < 1e-9
    y = np.zeros((1, V)); y[0, 9] = 60.0
    assert abs(oracle_mod.token_logprob(y, [9])[0]) < 1e-20 + (V - 1) * np.exp(-60)
    # probabilities of a row sum to one
    tot = np.exp(oracle_mod.token_logprob(np.repeat(x[:1], V, 0), np.arange(V))).sum()
    assert abs(tot - 1.0) < 1e-12
    # an index outside the row gives NaN
    assert np.isnan(oracle_mod.token_logprob(x[:1], [V])[0])
