"""GPU parity of vocab argmax, consensus and KV commit against the CPU oracle,
through the C ABI.  All three are integer/byte results: bit-exact."""
import numpy as np
import pytest
import torch

import block_attention_b200 as ba
from block_attention_b200 import synth
from gpu_util import to_dev, to_host

pytestmark = pytest.mark.gpu


def gpu_argmax(x, stride=None):
    t = to_dev(x)
    if stride is not None:
        big = torch.zeros(t.shape[0], stride, dtype=t.dtype, device="cuda")
        big[:, :t.shape[1]] = t
        t = big[:, :t.shape[1]]
    mx = torch.empty(t.shape[0], dtype=torch.float32, device="cuda")
    idx = ba.vocab_argmax(t, maxval=mx)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), mx.cpu().numpy()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("vocab", [1024, 8192, 151936, 100003, 300007])
def test_argmax_random_rows(oracle_mod, dtype, vocab):
    x = synth.logits(synth.rng(201, vocab), 32, vocab, std=3.0, dtype=dtype)
    idx, mx = gpu_argmax(x)
    ref, rmx = oracle_mod.vocab_argmax(x, return_max=True)
    np.testing.assert_array_equal(idx, ref)
    np.testing.assert_array_equal(mx.astype(np.float64), rmx)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("V", [151936, 300007])  # one cluster per row; atomics across CTAs
def test_argmax_ties_nan_zero_and_strides(oracle_mod, dtype, V):
    g = synth.rng(202)
    x = synth.logits(g, 24, V, dtype=dtype)
    top = synth.cast(np.array([60.0], np.float32), dtype)[0]
    for r in range(0, 8):  # planted ties across chunk boundaries
        cols = np.sort(g.choice(V, size=3, replace=False))
        x[r, cols] = top
    nan = synth.cast(np.array([np.nan], np.float32), dtype)[0]
    x[8, :] = nan                       # all NaN -> 0
    x[9, ::7] = nan                     # NaN never wins
    x[10, :] = synth.cast(np.array([-1.0], np.float32), dtype)[0]
    x[10, 5] = synth.cast(np.array([-0.0], np.float32), dtype)[0]
    x[10, 9] = synth.cast(np.array([0.0], np.float32), dtype)[0]   # -0 == +0 -> 5
    x[11, :] = synth.cast(np.array([2.5], np.float32), dtype)[0]   # all equal -> 0
    x[12, -1] = top                     # max in the last element (ragged tail)
    x[13, :] = synth.cast(np.array([-np.inf], np.float32), dtype)[0]
    x[13, :3] = nan                     # -inf everywhere else: the first -inf wins
    ref = oracle_mod.vocab_argmax(x)
    for stride in (None, V + 8, V + 3):  # aligned and unaligned row strides
        idx, _ = gpu_argmax(x, stride)
        np.testing.assert_array_equal(idx, ref)
    assert ref[8] == 0 and ref[10] == 5 and ref[11] == 0 and ref[12] == V - 1 and ref[13] == 3


def test_argmax_repeated_calls_reuse_workspace(oracle_mod):
    """The workspace's slots return to zero: many calls in a row agree."""
    for s in range(5):
        for V in (5000, 300007):
            x = synth.logits(synth.rng(203, s), 7, V)
            idx, _ = gpu_argmax(x)
            np.testing.assert_array_equal(idx, oracle_mod.vocab_argmax(x))


def _gpu_consensus(d, a):
    L, ne, em, na = ba.consensus(to_dev(d), to_dev(a))
    torch.cuda.synchronize()
    return [t.cpu().numpy() for t in (L, ne, em, na)]


@pytest.mark.parametrize("blk", [1, 4, 8, 16, 31, 32])
def test_consensus_planted(oracle_mod, blk):
    g = synth.rng(204, blk)
    B = 300
    acc = g.integers(0, blk + 1, size=B).astype(np.int32)
    d, a = synth.planted_tokens(g, B, blk, 151936, acc)
    got = _gpu_consensus(d, a)
    ref = oracle_mod.consensus(d, a)
    for x, y in zip(got, ref):
        np.testing.assert_array_equal(x, y)
    np.testing.assert_array_equal(got[0], acc)


def test_consensus_exhaustive_tiny(oracle_mod):
    import itertools
    seqs = np.array(list(itertools.product([0, 1], repeat=5)), np.int32)
    d = np.repeat(seqs, len(seqs), axis=0)
    a = np.tile(seqs, (len(seqs), 1))
    for x, y in zip(_gpu_consensus(d, a), oracle_mod.consensus(d, a)):
        np.testing.assert_array_equal(x, y)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("D", [64, 128, 6])
def test_commit_multi_layer_ragged(oracle_mod, dtype, D):
    layers, B, Hkv, cap, blk = 3, 5, 2, 90, 32
    g = synth.rng(205, D)
    kc = synth.cast(synth.normal(g, (layers, B, Hkv, cap, D)), dtype)
    vc = synth.cast(synth.normal(g, (layers, B, Hkv, cap, D)), dtype)
    kb = synth.cast(synth.normal(g, (layers, B, blk, Hkv, D)), dtype)
    vb = synth.cast(synth.normal(g, (layers, B, blk, Hkv, D)), dtype)
    lens = np.array([0, 10, 58, 33, 77], np.int32)
    ne = np.array([32, 0, 32, 1, 13], np.int32)   # rows 2 and 4 fill the cache exactly
    tk, tv = to_dev(kc), to_dev(vc)
    tl = to_dev(lens)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ba.kv_commit(tk, tv, to_dev(kb), to_dev(vb), tl, to_dev(ne), err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    new_lens = None
    for l in range(layers):
        rk, rv = kc[l].copy(), vc[l].copy()
        new_lens = oracle_mod.kv_commit(rk, rv, np.ascontiguousarray(kb[l]),
                                        np.ascontiguousarray(vb[l]), lens, ne)
        gk, gv = tk[l].cpu(), tv[l].cpu()
        if dtype == "bf16":
            gk, gv = gk.view(torch.int16).numpy().view(np.uint16), gv.view(torch.int16).numpy().view(np.uint16)
        else:
            gk, gv = gk.numpy(), gv.numpy()
        assert np.array_equal(gk, rk) and np.array_equal(gv, rv)
    np.testing.assert_array_equal(tl.cpu().numpy(), new_lens)


def test_commit_overflow_skips_sequence_and_flags(oracle_mod):
    B, Hkv, cap, D, blk = 2, 2, 20, 64, 8
    g = synth.rng(206)
    kc = synth.to_bf16(synth.normal(g, (B, Hkv, cap, D)))
    kb = synth.to_bf16(synth.normal(g, (B, blk, Hkv, D)))
    tk, tv = to_dev(kc), to_dev(kc.copy())
    lens = to_dev(np.array([5, 15], np.int32))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ba.kv_commit(tk, tv, to_dev(kb), to_dev(kb.copy()), lens, to_dev(np.array([8, 8], np.int32)),
                 err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == -4
    assert lens.cpu().tolist() == [13, 15]
    got = tk.cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got[1], kc[1])  # sequence 1 untouched
    assert np.array_equal(got[0, :, 5:13], kb[0].transpose(1, 0, 2))


def test_commit_repeated_rounds_grow_context(oracle_mod):
    """Ten rounds of commit on one workspace: lengths and bytes track the oracle."""
    layers, B, Hkv, cap, D, blk = 2, 3, 2, 400, 64, 32
    g = synth.rng(207)
    kc = np.zeros((layers, B, Hkv, cap, D), np.uint16)
    vc = np.zeros_like(kc)
    tk, tv = to_dev(kc), to_dev(vc)
    lens = np.array([0, 5, 9], np.int32)
    tl = to_dev(lens)
    rk, rv = kc.copy(), vc.copy()
    for r in range(10):
        kb = synth.to_bf16(synth.normal(g, (layers, B, blk, Hkv, D)))
        vb = synth.to_bf16(synth.normal(g, (layers, B, blk, Hkv, D)))
        ne = synth.geometric_accept(g, B) + 1
        ne = np.minimum(ne, blk).astype(np.int32)
        ba.kv_commit(tk, tv, to_dev(kb), to_dev(vb), tl, to_dev(ne))
        for l in range(layers):
            a, b_ = rk[l].copy(), rv[l].copy()
            nl = oracle_mod.kv_commit(a, b_, kb[l].copy(), vb[l].copy(), lens, ne)
            rk[l], rv[l] = a, b_
        lens = nl
    torch.cuda.synchronize()
    np.testing.assert_array_equal(tl.cpu().numpy(), lens)
    assert np.array_equal(tk.cpu().view(torch.int16).numpy().view(np.uint16), rk)
    assert np.array_equal(tv.cpu().view(torch.int16).numpy().view(np.uint16), rv)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_token_logprob_matches_oracle(oracle_mod, dtype):
    """Log-probability of a chosen token per row (precision-study input) against
    the float64 oracle, on the vocab-151936 shape and on a ragged short vocab."""
    for k, (rows, vocab) in enumerate([(32, 151936), (7, 1000)]):
        x = synth.logits(synth.rng(500 + k, len(dtype)), rows, vocab, dtype=dtype)
        idx = synth.rng(510 + k).integers(0, vocab, rows).astype(np.int32)
        t = to_dev(x)
        got = to_host(ba.token_logprob(t, to_dev(idx)))
        ref = oracle_mod.token_logprob(x, idx)
        # FP32 sums of <= 151936 exponentials in a fixed order, then a log:
        # the result is exact to ~1e-5 absolute at these magnitudes
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-4)
