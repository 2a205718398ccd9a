"""GPU parity of block attention (both views) against the CPU oracle, through
the C ABI.  Tolerance: per (sequence, row, head) max-abs error over the head
dim relative to the oracle row's max-abs value -- 1e-5 for FP32 tensors, 2e-2
for bf16 tensors with FP32 accumulation."""
import numpy as np
import pytest
import torch

import block_attention_b200 as ba
from block_attention_b200 import synth
from gpu_util import TOL, rel_err_rows, to_dev, to_host

pytestmark = pytest.mark.gpu


def run_gpu(inp, mode, max_ctx=None, err=None, out=None):
    t = {k: to_dev(v) for k, v in inp.items()}
    o = ba.block_attn(t["q"], t["k_blk"], t["v_blk"], t["k_cache"], t["v_cache"],
                      t["ctx_lens"], mode, max_ctx=max_ctx, err=err, out=out)
    torch.cuda.synchronize()
    return o


def check(inp, mode, dtype, max_ctx=None, oracle_mod=None):
    ref = oracle_mod.block_attn(inp["q"], inp["k_blk"], inp["v_blk"], inp["k_cache"],
                                inp["v_cache"], inp["ctx_lens"], mode)
    got = to_host(run_gpu(inp, mode, max_ctx))
    e = rel_err_rows(got, ref)
    assert np.isfinite(got).all()
    assert e.max() <= TOL[dtype], (e.max(), np.unravel_index(e.argmax(), e.shape))
    return e.max()


@pytest.mark.parametrize("mode", [0, 1])
def test_tiny_f32_workload(oracle_mod, mode):
    w = synth.WORKLOADS["tiny"]
    inp = synth.attn_inputs(w["B"], w["Hq"], w["Hkv"], w["D"], w["blk"], [w["ctx"]],
                            w["ctx"] + w["blk"], "f32", seed=101)
    check(inp, mode, "f32", oracle_mod=oracle_mod)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("mode", [0, 1])
def test_qwen3_1p7b_layer(oracle_mod, dtype, mode):
    w = synth.WORKLOADS["qwen3_1p7b"]
    inp = synth.attn_inputs(w["B"], w["Hq"], w["Hkv"], w["D"], w["blk"], [w["ctx"]],
                            w["ctx"] + w["blk"], dtype, seed=102)
    check(inp, mode, dtype, oracle_mod=oracle_mod)


EDGE = [
    # (ctx lens, blk, Hq, Hkv, D)
    ([0], 32, 4, 2, 64),          # empty context: block only
    ([1], 1, 2, 2, 64),           # one key + one row (plain decode)
    ([15, 16, 17], 8, 8, 2, 128),  # around a tile edge
    ([255, 256, 257], 32, 4, 1, 64),  # around a split edge, one kv head
    ([1000, 3, 0, 511], 16, 8, 8, 128),  # ragged, MHA
    ([700], 4, 32, 8, 128),       # small block, 8B head layout
    ([129], 32, 16, 4, 64),
]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("case", range(len(EDGE)))
def test_edge_shapes(oracle_mod, dtype, mode, case):
    lens, blk, Hq, Hkv, D = EDGE[case]
    cap = max(lens) + 40
    inp = synth.attn_inputs(len(lens), Hq, Hkv, D, blk, lens, cap, dtype, seed=103 + case)
    check(inp, mode, dtype, max_ctx=max(lens) + 7, oracle_mod=oracle_mod)


@pytest.mark.parametrize("mode", [0, 1])
def test_qwen3_8b_layer_full(oracle_mod, mode):
    w = synth.WORKLOADS["qwen3_8b"]
    inp = synth.attn_inputs(1, w["Hq"], w["Hkv"], w["D"], w["blk"], [w["ctx"]],
                            w["ctx"] + 32, "bf16", seed=104)
    check(inp, mode, "bf16", oracle_mod=oracle_mod)


@pytest.mark.parametrize("mode", [0, 1])
def test_multi_wave_grid_sorted_by_length(oracle_mod, mode):
    """A bf16 grid of more than one wave (here 20 sequences x 8 kv-heads x 2
    splits = 320 CTAs, merged by the second kernel) starts its CTAs
    longest-sequence first.  Every (sequence, kv-head, split) is still
    computed exactly once: the output matches the oracle, and the
    ORTHRUS_ATTN_EARLY_KV launch (lengths read before the dependency wait)
    gives the same bits."""
    lens = [5, 900, 0, 3000, 129, 2500, 77, 1800, 640, 1, 3333, 256, 1500, 12, 2048, 700,
            999, 9000, 31, 1024]
    inp = synth.attn_inputs(len(lens), 16, 8, 128, 16, lens, max(lens) + 20, "bf16", seed=120)
    ref = oracle_mod.block_attn(inp["q"], inp["k_blk"], inp["v_blk"], inp["k_cache"],
                                inp["v_cache"], inp["ctx_lens"], mode)
    t = {k: to_dev(v) for k, v in inp.items()}
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs = [ba.block_attn(t["q"], t["k_blk"], t["v_blk"], t["k_cache"], t["v_cache"],
                          t["ctx_lens"], mode, err=err, flags=f) for f in (0, ba.ATTN_EARLY_KV)]
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(outs[0], outs[1])
    e = rel_err_rows(to_host(outs[0]), ref)
    assert e.max() <= TOL["bf16"], (e.max(), np.unravel_index(e.argmax(), e.shape))


def test_ragged_batch_sampled_sequences(oracle_mod):
    """16 sequences, contexts ~ U{1024..32768}; the GPU runs the whole batch,
    the oracle checks three of them (first, longest, shortest)."""
    w = synth.WORKLOADS["ragged"]
    lens = synth.ragged_lens(w["B"], w["ctx_lo"], w["ctx_hi"], seed=105)
    cap = int(lens.max()) + w["blk"]
    inp = synth.attn_inputs(w["B"], w["Hq"], w["Hkv"], w["D"], w["blk"], lens, cap, "bf16",
                            seed=105)
    picks = sorted({0, int(lens.argmax()), int(lens.argmin())})
    for mode in (0, 1):
        got = to_host(run_gpu(inp, mode, max_ctx=cap - w["blk"]))
        for b in picks:
            sub = {k: v[b:b + 1] for k, v in inp.items()}
            ref = oracle_mod.block_attn(sub["q"], sub["k_blk"], sub["v_blk"], sub["k_cache"],
                                        sub["v_cache"], sub["ctx_lens"], mode)
            e = rel_err_rows(got[b:b + 1], ref)
            assert e.max() <= TOL["bf16"], (b, mode, e.max())


@pytest.mark.parametrize("B,Hkv", [(32, 8), (40, 4)])
def test_many_sequences_multi_wave(oracle_mod, B, Hkv):
    """More kv-head rows than SMs (one split each, two launches): 32
    sequences take the length-sorted launch order, 40 the grid order; every
    sequence matches the oracle in both views."""
    lens = [int(x) for x in np.random.default_rng(B).integers(0, 600, B)]
    lens[3] = 0
    inp = synth.attn_inputs(B, 2 * Hkv, Hkv, 128, 8, lens, max(lens) + 10, "bf16", seed=130 + B)
    for mode in (0, 1):
        ref = oracle_mod.block_attn(inp["q"], inp["k_blk"], inp["v_blk"], inp["k_cache"],
                                    inp["v_cache"], inp["ctx_lens"], mode)
        got = to_host(run_gpu(inp, mode))
        e = rel_err_rows(got, ref)
        assert e.max() <= TOL["bf16"], (mode, e.max(), np.unravel_index(e.argmax(), e.shape))


def test_f32_causal_row_equals_single_token_decode_bitwise():
    """Verify row i over (cache n, block) == one-row decode at n+i over
    (cache n+i, block of 1), bit for bit, across split and tile boundaries."""
    n, blk, Hq, Hkv, D = 250, 32, 4, 2, 64
    inp = synth.attn_inputs(1, Hq, Hkv, D, blk, [n], n + blk, "f32", seed=106)
    full = to_host(run_gpu(inp, 1, max_ctx=n))
    for i in range(blk):
        kc, vc = inp["k_cache"].copy(), inp["v_cache"].copy()
        kc[0, :, n:n + i] = inp["k_blk"][0, :i].transpose(1, 0, 2)
        vc[0, :, n:n + i] = inp["v_blk"][0, :i].transpose(1, 0, 2)
        one = {"q": inp["q"][:, i:i + 1], "k_blk": inp["k_blk"][:, i:i + 1],
               "v_blk": inp["v_blk"][:, i:i + 1], "k_cache": kc, "v_cache": vc,
               "ctx_lens": np.array([n + i], np.int32)}
        # a different max_ctx (grid size) must not change the result either
        dec = to_host(run_gpu(one, 1, max_ctx=n + blk))
        assert np.array_equal(dec[0, 0], full[0, i]), i


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_deterministic(dtype):
    inp = synth.attn_inputs(2, 32, 8, 128, 32, [3000, 777], 3100, dtype, seed=107)
    a = to_host(run_gpu(inp, 0))
    b = to_host(run_gpu(inp, 0))
    assert np.array_equal(a, b)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_device_length_over_bound_sets_error_word(oracle_mod, dtype):
    inp = synth.attn_inputs(2, 8, 2, 64, 8, [40, 100], 128, dtype, seed=108)
    inp["ctx_lens"] = np.array([40, 100], np.int32)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.full((2, 8, 8, 64), 7.0, device="cuda",
                     dtype=torch.float32 if dtype == "f32" else torch.bfloat16)
    run_gpu(inp, 0, max_ctx=64, err=err, out=out)  # sequence 1 exceeds max_ctx
    assert int(err.item()) == -4  # ORTHRUS_ECAPACITY
    got = to_host(out)
    sub = {k: v[:1] for k, v in inp.items()}
    ref = oracle_mod.block_attn(sub["q"], sub["k_blk"], sub["v_blk"], sub["k_cache"],
                                sub["v_cache"], sub["ctx_lens"], 0)
    assert rel_err_rows(got[:1], ref).max() <= TOL[dtype]
    assert np.all(got[1] == 7.0)  # skipped sequence left untouched


def test_multi_wave_grid_with_lengths_over_bound(oracle_mod):
    """The length-sorted launch order of a multi-wave grid ranks sequences
    whose length is out of bounds last; they report ORTHRUS_ECAPACITY and
    are left untouched, the others match the oracle (20 sequences x 8
    kv-heads: 160 CTAs, more than one wave)."""
    lens = [5, 900, 0, 3000, 129, 2500, 77, 1800, 640, 1, 3333, 256, 1500, 12, 2048, 700,
            999, 4000, 31, 1024]
    inp = synth.attn_inputs(len(lens), 16, 8, 128, 16, lens, 4100, "bf16", seed=121)
    bad = [3, 17]
    lens_dev = np.array(lens, np.int32)
    lens_dev[bad] = [3500, 4050]  # over max_ctx = 3400
    inp_dev = dict(inp, ctx_lens=lens_dev)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.full((len(lens), 16, 16, 128), 7.0, device="cuda", dtype=torch.bfloat16)
    run_gpu(inp_dev, 0, max_ctx=3400, err=err, out=out)
    assert int(err.item()) == -4  # ORTHRUS_ECAPACITY
    got = to_host(out)
    good = [i for i in range(len(lens)) if i not in bad]
    sub = {k: v[good] for k, v in inp.items()}
    ref = oracle_mod.block_attn(sub["q"], sub["k_blk"], sub["v_blk"], sub["k_cache"],
                                sub["v_cache"], sub["ctx_lens"], 0)
    assert rel_err_rows(got[good], ref).max() <= TOL["bf16"]
    assert np.all(got[bad] == 7.0)


def test_one_workspace_reused_across_shapes(oracle_mod):
    """One bf16 workspace serves calls of different shapes in any order.  The
    in-launch merge keeps one 64-bit word per (sequence, kv-head) in the
    buffer's first 2048 bytes (these shapes all fit one wave): the arrival
    count (low half) is back at zero after every call and the generation
    (high half) of every head the call covers has moved on by exactly one;
    no partial is ever written there."""
    ws = ba.Workspace("cuda")
    shapes = [(2, 32, 8, 128, 32, [3000, 500]), (1, 4, 1, 64, 32, [100]),
              (1, 16, 8, 128, 32, [2048]), (1, 8, 8, 128, 4, [0]),
              (3, 32, 8, 128, 32, [900, 10, 4000]), (1, 16, 8, 128, 32, [2048])]
    gens = np.zeros(256, np.int64)
    for k, (B, Hq, Hkv, D, blk, lens) in enumerate(shapes):
        inp = synth.attn_inputs(B, Hq, Hkv, D, blk, lens, max(lens) + 8, "bf16", seed=300 + k)
        t = {kk: to_dev(v) for kk, v in inp.items()}
        for mode in (0, 1):
            ptr = ws.buf.data_ptr()
            out = ba.block_attn(t["q"], t["k_blk"], t["v_blk"], t["k_cache"], t["v_cache"],
                                t["ctx_lens"], mode, workspace=ws)
            torch.cuda.synchronize()
            ref = oracle_mod.block_attn(inp["q"], inp["k_blk"], inp["v_blk"], inp["k_cache"],
                                        inp["v_cache"], inp["ctx_lens"], mode)
            e = rel_err_rows(to_host(out), ref)
            assert e.max() <= TOL["bf16"], (k, mode, e.max())
            words = ws.buf[:2048].cpu().numpy().view(np.uint64)
            assert not (words & 0xFFFFFFFF).any(), (k, mode)  # counts back at zero
            if ws.buf.data_ptr() != ptr:
                gens[:] = 0  # the workspace grew: a new zeroed buffer
            gens[:B * Hkv] += 1
            assert np.array_equal((words >> 32).astype(np.int64), gens), (k, mode)


@pytest.mark.parametrize("mode", [0, 1])
def test_early_kv_flag_same_result(oracle_mod, mode):
    """ORTHRUS_ATTN_EARLY_KV only moves when the cache is read: same output."""
    inp = synth.attn_inputs(2, 32, 8, 128, 32, [4000, 1500], 4100, "bf16", seed=109)
    t = {k: to_dev(v) for k, v in inp.items()}
    a = ba.block_attn(t["q"], t["k_blk"], t["v_blk"], t["k_cache"], t["v_cache"],
                      t["ctx_lens"], mode)
    b = ba.block_attn(t["q"], t["k_blk"], t["v_blk"], t["k_cache"], t["v_cache"],
                      t["ctx_lens"], mode, flags=ba.ATTN_EARLY_KV)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("blk", [4, 8, 16])
def test_block_size_variants(oracle_mod, dtype, mode, blk):
    """Block sizes K in {4, 8, 16} (the explainer's ablation, section 六) at the
    Qwen3-8B head layout, with a ragged pair of contexts."""
    inp = synth.attn_inputs(2, 32, 8, 128, blk, [2000, 333], 2000 + blk, dtype, seed=150 + blk)
    check(inp, mode, dtype, oracle_mod=oracle_mod)


@pytest.mark.parametrize("mode", [0, 1])
def test_next_call_l2_prefetch_same_result(oracle_mod, mode):
    """Naming the next call's caches (an L2 warm-up hint) leaves the output
    bit-identical, for a one-wave grid (merge inside the launch) and a larger
    one (separate merge kernel)."""
    for B, lens in ((1, [8192]), (8, [3000, 500, 8000, 1, 0, 4096, 2048, 7777])):
        inp = synth.attn_inputs(B, 32, 8, 128, 32, lens, max(lens) + 32, "bf16", seed=160 + B)
        t = {k: to_dev(v) for k, v in inp.items()}
        nk, nv = torch.randn_like(t["k_cache"]), torch.randn_like(t["v_cache"])
        a = ba.block_attn(t["q"], t["k_blk"], t["v_blk"], t["k_cache"], t["v_cache"],
                          t["ctx_lens"], mode)
        b = ba.block_attn(t["q"], t["k_blk"], t["v_blk"], t["k_cache"], t["v_cache"],
                          t["ctx_lens"], mode, next_kv=(nk, nv), flags=ba.ATTN_EARLY_KV)
        torch.cuda.synchronize()
        assert torch.equal(a, b), B
        if B == 1:
            ref = oracle_mod.block_attn(inp["q"], inp["k_blk"], inp["v_blk"], inp["k_cache"],
                                        inp["v_cache"], inp["ctx_lens"], mode)
            assert rel_err_rows(to_host(b), ref).max() <= TOL["bf16"]
