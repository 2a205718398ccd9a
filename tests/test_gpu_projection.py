"""GPU parity of the tensor-core projection (orthrus_linear_tc) against the
float64 oracle, through the C ABI: per output row, the largest difference
from the oracle's exact product (or, with a residual, from its bf16 result)
relative to the row's largest magnitude is within the bf16 tolerance, and
the bf16 rounding agrees with the oracle's on nearly every element.  Shapes: the Qwen3-8B attention block's QKV (6144 x 4096) and
output (4096 x 4096, with the residual) projections of a 32-row block, and
ragged ones (rows 1..128, N not a multiple of the 128-feature tile, small K,
split and unsplit K)."""
import numpy as np
import pytest
import torch

import block_attention_b200 as ba
from block_attention_b200 import synth
from gpu_util import TOL, to_dev

pytestmark = pytest.mark.gpu


def _f(bits):
    return (np.asarray(bits, np.uint32) << 16).view(np.float32).astype(np.float64)


def _host_bits(t):
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def check(oracle_mod, rows, K, N, residual, seed, std_w=0.02):
    g = synth.rng(seed, 1)
    x = synth.to_bf16(synth.normal(g, (rows, K)))
    w = synth.to_bf16(synth.normal(g, (N, K), std_w))
    res = synth.to_bf16(synth.normal(g, (rows, N))) if residual else None
    xt, wt = to_dev(x), to_dev(w)
    rt = to_dev(res) if residual else None
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = ba.linear_tc(xt, wt, residual=rt, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    got = _host_bits(y)
    ref, exact, mag = oracle_mod.projection(x, w, res)
    want = exact if res is None else _f(ref)
    # per row: max |got - oracle| over the row's largest oracle magnitude,
    # within the bf16 tolerance (fp32 accumulation in the tensor core's order,
    # then bf16 rounding); and the rounding agrees on nearly every element
    err = np.abs(_f(got) - want).max(axis=1) / np.maximum(np.abs(want).max(axis=1), 1e-6)
    assert err.max() <= TOL["bf16"], err.max()
    assert (got == ref).mean() > 0.9, (got == ref).mean()


def test_qwen3_8b_qkv_projection(oracle_mod):
    check(oracle_mod, 32, 4096, 6144, residual=False, seed=501)


def test_qwen3_8b_output_projection_with_residual(oracle_mod):
    check(oracle_mod, 32, 4096, 4096, residual=True, seed=502)


@pytest.mark.parametrize("rows,K,N", [(1, 64, 128), (7, 256, 1000), (32, 640, 300),
                                       (100, 1024, 2048), (128, 4096, 384), (16, 128, 12000)])
def test_ragged_shapes(oracle_mod, rows, K, N):
    check(oracle_mod, rows, K, N, residual=False, seed=503 + rows)
    check(oracle_mod, rows, K, N, residual=True, seed=603 + rows)


def test_deterministic_and_workspace_left_zero():
    g = synth.rng(510, 1)
    x = to_dev(synth.to_bf16(synth.normal(g, (32, 4096))))
    w = to_dev(synth.to_bf16(synth.normal(g, (6144, 4096), 0.02)))
    ws = ba.Workspace("cuda")
    a = ba.linear_tc(x, w, workspace=ws)
    b = ba.linear_tc(x, w, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    tiles = (6144 + 127) // 128
    assert int(ws.buf[:tiles * 4].count_nonzero()) == 0  # ticket counters back at zero


@pytest.mark.parametrize("B,blk,Hq,Hkv,K", [(1, 32, 32, 8, 4096),   # the Qwen3-8B block
                                            (3, 17, 4, 2, 640),     # ragged rows, one K split
                                            (4, 32, 2, 1, 256),     # 128 rows: four row chunks
                                            (2, 9, 3, 1, 64)])      # one K step: no split
def test_qkv_rope_epilogue_equals_projection_then_rope(B, blk, Hq, Hkv, K):
    """The QKV projection with RoPE and the head split in its epilogue gives
    the same bits as the projection followed by the stand-alone RoPE kernel
    (which the decoder tests check against the oracle's forward)."""
    g = torch.Generator(device="cuda").manual_seed(B * 1000 + blk)
    rows, hd, theta = B * blk, 128, 1e6
    N = (Hq + 2 * Hkv) * hd
    x = torch.randn(rows, K, generator=g, device="cuda").to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    lens = torch.tensor([8192, 5, 77, 30000][:B], dtype=torch.int32, device="cuda")
    table = ba.rope_table(lens, B, blk, hd, theta)
    mk = lambda h: torch.empty(rows, h, hd, dtype=torch.bfloat16, device="cuda")
    q, k, v = mk(Hq), mk(Hkv), mk(Hkv)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ba.linear_tc_qkv_rope(x, w, Hq, Hkv, table, q=q, k=k, v=v, err=err)
    qkv = ba.linear_tc(x, w)
    q2, k2, v2 = mk(Hq), mk(Hkv), mk(Hkv)
    ba.qkv_rope(qkv, lens, B, blk, Hq, Hkv, hd, theta, q=q2, k=k2, v=v2)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(q, q2) and torch.equal(k, k2) and torch.equal(v, v2)
    # the table holds the stand-alone kernel's angles: spot-check against float64
    pos = (lens.cpu().numpy()[:, None] + np.arange(blk)[None]).reshape(-1)
    ang = pos[:, None] * theta ** (-2.0 * np.arange(hd // 2) / hd)[None]
    t = table.cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(t[..., 0], np.cos(ang), atol=2e-7)
    np.testing.assert_allclose(t[..., 1], np.sin(ang), atol=2e-7)


def test_l2_hint_changes_nothing():
    """The L2 warm-up hint of the projections is only a hint: with it the
    outputs are as without it and the ticket counters return to zero."""
    g = torch.Generator(device="cuda").manual_seed(77)
    x = torch.randn(32, 1024, generator=g, device="cuda").to(torch.bfloat16)
    w = (torch.randn(768, 1024, generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    res = torch.randn(32, 768, generator=g, device="cuda").to(torch.bfloat16)
    nxt = torch.randn(3, 1000003, generator=g, device="cuda")  # size not a multiple of the CTAs
    ws = ba.Workspace("cuda")
    a = ba.linear_tc(x, w, residual=res, workspace=ws)
    b = ba.linear_tc(x, w, residual=res, l2_next=nxt, workspace=ws)
    table = ba.rope_table(torch.tensor([100], dtype=torch.int32, device="cuda"), 1, 32, 128, 1e4)
    mk = lambda h: torch.empty(32, h, 128, dtype=torch.bfloat16, device="cuda")
    outs = []
    for hint in (None, nxt):
        q, k, v = mk(2), mk(2), mk(2)
        ba.linear_tc_qkv_rope(x, w[:768], 2, 2, table, q=q, k=k, v=v, l2_next=hint, workspace=ws)
        outs.append((q, k, v))
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert all(torch.equal(s, t) for s, t in zip(*outs))
    assert int(ws.buf[:(768 // 128) * 4].count_nonzero()) == 0  # ticket counters
