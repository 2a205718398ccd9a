"""GPU parity of the LM head with the argmax in its epilogue
(orthrus_lm_head_argmax) against the float64 oracle (oracle.lm_head_argmax).

The kernel sums exact bf16 products in fp32, so a row whose two largest
logits lie within fp32 rounding of each other may legitimately pick either.
Tolerance per row: tol = 2^-12 * mag, mag = max_v sum_k |h_k w_vk| (the
worst-case error of a 4096-term fp32 sum is K * 2^-24 * mag = 2^-12 * mag at
K = 4096).  Rows whose oracle top-2 gap exceeds 2 tol must match exactly;
every row's index must be a near-maximum (its exact logit within tol of the
maximum) and maxval within tol of that logit.  Integer-valued inputs, whose
sums are exact in any order, check ties (lowest index) bit-exactly.
"""
import numpy as np
import pytest
import torch

import block_attention_b200 as ba
from block_attention_b200 import synth

pytestmark = pytest.mark.gpu


def _widen(b):
    return synth.bf16_to_f32(b).astype(np.float64)


def _run(h, w, ld=None, workspace=None):
    th = torch.from_numpy(h.view(np.int16)).view(torch.bfloat16).cuda()
    if ld is not None:  # h as a view into wider rows
        wide = torch.zeros(h.shape[0], ld, dtype=torch.bfloat16, device="cuda")
        wide[:, :h.shape[1]] = th
        th = wide[:, :h.shape[1]]
    tw = torch.from_numpy(w.view(np.int16)).view(torch.bfloat16).cuda()
    mx = torch.empty(h.shape[0], dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    idx = ba.lm_head_argmax(th, tw, maxval=mx, err=err, workspace=workspace)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return idx.cpu().numpy(), mx.cpu().numpy()


def _check(oracle_mod, h, w, got, gmax, min_sure=0.5):
    idx, mx, gap, mag = oracle_mod.lm_head_argmax(h, w)
    V = w.shape[0]
    assert ((got >= 0) & (got < V)).all()
    tol = 2.0 ** -12 * mag
    exact_at = np.einsum("rk,rk->r", _widen(h), _widen(w[got]))
    assert (exact_at >= mx - tol).all()  # a near-maximum
    np.testing.assert_allclose(gmax, exact_at, rtol=0, atol=tol.max())
    sure = gap > 2 * tol
    assert sure.mean() >= min_sure
    np.testing.assert_array_equal(got[sure], idx[sure])


@pytest.mark.parametrize("rows,d,V", [(32, 256, 3001), (7, 128, 1000), (128, 512, 5000),
                                      (33, 64, 128), (1, 64, 1), (96, 192, 40000),
                                      (64, 1024, 20000)])
def test_lm_head_argmax_matches_oracle(oracle_mod, rows, d, V):
    """Several CTAs, ragged last vocabulary tile, hidden rows from 1 to 128
    (one to four TMEM lane quadrants), tiles of 128 and 144 rows, one-tile and
    one-word vocabularies."""
    h, w = synth.lm_head_inputs(rows, d, V, seed=700 + rows, std_w=1.0 / np.sqrt(d))
    got, gmax = _run(h, w)
    _check(oracle_mod, h, w, got, gmax)


def test_hidden_rows_with_a_row_stride(oracle_mod):
    h, w = synth.lm_head_inputs(20, 256, 2000, seed=711, std_w=0.0625)
    got, gmax = _run(h, w, ld=264)
    _check(oracle_mod, h, w, got, gmax)


def test_exact_integer_inputs_take_the_lowest_index_on_ties(oracle_mod):
    """Small integers: every sum is exact in fp32 in any order, so the GPU must
    equal the oracle bit for bit, including planted ties across tiles and
    CTAs (lowest index wins)."""
    g = np.random.default_rng(712)
    rows, d, V = 40, 128, 20000
    hf = g.integers(-2, 3, (rows, d)).astype(np.float32)
    wf = g.integers(-2, 3, (V, d)).astype(np.float32)
    for r in range(rows):  # the row's maximum, planted twice (or three times)
        sites = sorted(g.choice(V, 3 if r % 4 == 0 else 2, replace=False))
        for v in sites:
            wf[v] = np.sign(hf[r]) * 2
    h, w = synth.to_bf16(hf), synth.to_bf16(wf)
    got, gmax = _run(h, w)
    idx, mx, _, _ = oracle_mod.lm_head_argmax(h, w)
    np.testing.assert_array_equal(got, idx)
    np.testing.assert_array_equal(gmax.astype(np.float64), mx)


def test_qwen3_8b_lm_head_shape(oracle_mod):
    """The Qwen3-8B LM head (d 4096, vocabulary 151936: 731 tiles of 208 rows
    over one wave of CTAs) for one 32-row block, every row against the oracle."""
    h, w = synth.lm_head_inputs(32, 4096, 151936, seed=713)
    got, gmax = _run(h, w)
    _check(oracle_mod, h, w, got, gmax, min_sure=0.75)


def test_workspace_left_zero_across_shapes(oracle_mod):
    ws = ba.Workspace("cuda")
    for i, (rows, d, V) in enumerate(((128, 64, 3000), (5, 128, 700), (64, 64, 129))):
        h, w = synth.lm_head_inputs(rows, d, V, seed=720 + i, std_w=0.125)
        got, gmax = _run(h, w, workspace=ws)
        _check(oracle_mod, h, w, got, gmax)
        assert not ws.buf.any().item()
