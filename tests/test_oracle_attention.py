"""Pins for the oracle's block attention (both mask modes).

The oracle is checked against things other than itself:
* torch's scaled_dot_product_attention in float64 (a library routine) for the
  cases where the round reduces to ordinary attention: empty context with a
  bidirectional block (full attention), empty context with the causal mask,
  and a context folded into the key sequence with a visibility mask;
* closed forms (equal keys -> mean of V; one dominant key -> that V);
* the mask rule of the Orthrus explainer §三 as invariants: perturbing keys a
  query must not see leaves its output bit-identical, perturbing keys it sees
  changes it;
* verify row i equals a single-token decode at position ctx+i (same key set).
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from block_attention_b200 import synth


def _case(B=1, Hq=4, Hkv=2, D=16, blk=8, ctx=(12,), cap=20, dtype="f32", seed=1):
    return synth.attn_inputs(B, Hq, Hkv, D, blk, list(ctx), cap, dtype, seed)


def _f64(a):
    a = np.asarray(a)
    if a.dtype == np.uint16:
        a = synth.bf16_to_f32(a)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))


def _sdpa_ref(inp, mask_mode, scale=None):
    """Fold cache + block into one key sequence per sequence and call SDPA."""
    q = _f64(inp["q"])  # [B, blk, Hq, D]
    B, blk, Hq, D = q.shape
    outs = []
    for b in range(B):
        n = int(inp["ctx_lens"][b])
        kc = _f64(inp["k_cache"])[b, :, :n]  # [Hkv, n, D]
        vc = _f64(inp["v_cache"])[b, :, :n]
        kb = _f64(inp["k_blk"])[b].transpose(0, 1)  # [Hkv, blk, D]
        vb = _f64(inp["v_blk"])[b].transpose(0, 1)
        k = torch.cat([kc, kb], 1)[None]
        v = torch.cat([vc, vb], 1)[None]
        qq = q[b].transpose(0, 1)[None]  # [1, Hq, blk, D]
        if mask_mode == 0:
            o = F.scaled_dot_product_attention(qq, k, v, scale=scale, enable_gqa=True)
        else:
            keypos = torch.arange(n + blk)
            rowpos = n + torch.arange(blk)
            allowed = keypos[None, :] <= rowpos[:, None]
            o = F.scaled_dot_product_attention(qq, k, v, attn_mask=allowed,
                                               scale=scale, enable_gqa=True)
        outs.append(o[0].transpose(0, 1).numpy())
    return np.stack(outs)


@pytest.mark.parametrize("mask_mode", [0, 1])
def test_empty_context_is_textbook_attention(oracle_mod, mask_mode):
    inp = _case(ctx=(0,), cap=4, blk=8)
    got = oracle_mod.block_attn(**{k: inp[k] for k in ("q", "k_blk", "v_blk", "k_cache",
                                                        "v_cache", "ctx_lens")},
                                mask_mode=mask_mode)
    q = _f64(inp["q"])[0].transpose(0, 1)[None]
    k = _f64(inp["k_blk"])[0].transpose(0, 1)[None]
    v = _f64(inp["v_blk"])[0].transpose(0, 1)[None]
    ref = F.scaled_dot_product_attention(q, k, v, is_causal=bool(mask_mode),
                                         enable_gqa=True)[0].transpose(0, 1).numpy()
    np.testing.assert_allclose(got[0], ref, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("mask_mode", [0, 1])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_context_plus_block_matches_sdpa(oracle_mod, mask_mode, dtype):
    inp = _case(B=3, Hq=6, Hkv=2, D=32, blk=8, ctx=(0, 5, 29), cap=33, dtype=dtype,
                seed=7)
    got = oracle_mod.block_attn(inp["q"], inp["k_blk"], inp["v_blk"], inp["k_cache"],
                                inp["v_cache"], inp["ctx_lens"], mask_mode, scale=0.3)
    ref = _sdpa_ref(inp, mask_mode, scale=0.3)
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)


def test_mha_when_hkv_equals_hq(oracle_mod):
    inp = _case(Hq=3, Hkv=3, D=8, blk=4, ctx=(6,), cap=6, seed=3)
    got = oracle_mod.block_attn(inp["q"], inp["k_blk"], inp["v_blk"], inp["k_cache"],
                                inp["v_cache"], inp["ctx_lens"], 0)
    np.testing.assert_allclose(got, _sdpa_ref(inp, 0), rtol=1e-11, atol=1e-12)


def test_gqa_grouping_is_consecutive_heads(oracle_mod):
    """q-head h reads kv-head h // G: zeroing kv-head 1's values zeroes exactly
    the outputs of q-heads G..2G-1."""
    inp = _case(Hq=6, Hkv=3, D=8, blk=4, ctx=(5,), cap=5, seed=4)
    inp["v_cache"][:, 1] = 0
    inp["v_blk"][:, :, 1] = 0
    got = oracle_mod.block_attn(inp["q"], inp["k_blk"], inp["v_blk"], inp["k_cache"],
                                inp["v_cache"], inp["ctx_lens"], 0)
    assert np.all(got[:, :, 2:4] == 0)
    assert np.all(np.abs(got[:, :, [0, 1, 4, 5]]).max(axis=-1) > 0)


@pytest.mark.parametrize("mask_mode", [0, 1])
def test_equal_keys_give_mean_of_values(oracle_mod, mask_mode):
    """All keys identical -> uniform weights -> o = mean of the visible V rows."""
    inp = _case(Hq=2, Hkv=1, D=8, blk=4, ctx=(5,), cap=8, seed=5)
    key = synth.normal(synth.rng(9), (8,))
    inp["k_cache"][:] = key
    inp["k_blk"][:] = key
    got = oracle_mod.block_attn(inp["q"], inp["k_blk"], inp["v_blk"], inp["k_cache"],
                                inp["v_cache"], inp["ctx_lens"], mask_mode)
    vc = inp["v_cache"][0, 0, :5].astype(np.float64)
    vb = inp["v_blk"][0, :, 0].astype(np.float64)
    for i in range(4):
        vis = np.concatenate([vc, vb if mask_mode == 0 else vb[:i + 1]])
        for h in range(2):
            np.testing.assert_allclose(got[0, i, h], vis.mean(0), rtol=1e-13, atol=1e-14)


def test_dominant_key_selects_its_value(oracle_mod):
    inp = _case(Hq=1, Hkv=1, D=8, blk=2, ctx=(6,), cap=6, seed=6)
    q = inp["q"][0, :, 0]  # [blk, D]
    # cache key 3 is 60 * q of row 0 -> score ~ 60 |q|^2 / sqrt(8) >> others
    inp["k_cache"][0, 0, 3] = 60.0 * q[0]
    got = oracle_mod.block_attn(inp["q"], inp["k_blk"], inp["v_blk"], inp["k_cache"],
                                inp["v_cache"], inp["ctx_lens"], 0)
    np.testing.assert_allclose(got[0, 0, 0], inp["v_cache"][0, 0, 3], rtol=1e-9, atol=1e-9)


def test_bidir_ignores_cache_rows_past_context(oracle_mod):
    inp = _case(B=2, ctx=(7, 12), cap=20, seed=8)
    base = oracle_mod.block_attn(inp["q"], inp["k_blk"], inp["v_blk"], inp["k_cache"],
                                 inp["v_cache"], inp["ctx_lens"], 0)
    for b, n in enumerate((7, 12)):
        inp["k_cache"][b, :, n:] = 1e3
        inp["v_cache"][b, :, n:] = -1e3
    again = oracle_mod.block_attn(inp["q"], inp["k_blk"], inp["v_blk"], inp["k_cache"],
                                  inp["v_cache"], inp["ctx_lens"], 0)
    assert np.array_equal(base, again)


def test_bidir_every_row_sees_every_block_row(oracle_mod):
    """Explainer §三: inside its block a diffusion query attends in both directions."""
    inp = _case(blk=6, ctx=(4,), cap=4, seed=10)
    base = oracle_mod.block_attn(inp["q"], inp["k_blk"], inp["v_blk"], inp["k_cache"],
                                 inp["v_cache"], inp["ctx_lens"], 0)
    for j in range(6):
        pert = {k: v.copy() for k, v in inp.items()}
        pert["v_blk"][0, j] += 1.0
        out = oracle_mod.block_attn(pert["q"], pert["k_blk"], pert["v_blk"],
                                    pert["k_cache"], pert["v_cache"], pert["ctx_lens"], 0)
        changed = np.abs(out - base).max(axis=(2, 3))[0]  # per row
        assert np.all(changed > 0), (j, changed)


def test_causal_row_sees_only_earlier_block_rows(oracle_mod):
    inp = _case(blk=6, ctx=(4,), cap=4, seed=11)
    base = oracle_mod.block_attn(inp["q"], inp["k_blk"], inp["v_blk"], inp["k_cache"],
                                 inp["v_cache"], inp["ctx_lens"], 1)
    for j in range(6):
        pert = {k: v.copy() for k, v in inp.items()}
        pert["k_blk"][0, j] += 0.5
        pert["v_blk"][0, j] += 1.0
        out = oracle_mod.block_attn(pert["q"], pert["k_blk"], pert["v_blk"],
                                    pert["k_cache"], pert["v_cache"], pert["ctx_lens"], 1)
        changed = np.abs(out - base).max(axis=(2, 3))[0]
        assert np.all(changed[:j] == 0) and np.all(changed[j:] > 0), (j, changed)


def test_context_perturbation_changes_every_row(oracle_mod):
    """Context before the anchor is visible to every row in both views."""
    inp = _case(blk=4, ctx=(6,), cap=6, seed=12)
    for mode in (0, 1):
        base = oracle_mod.block_attn(inp["q"], inp["k_blk"], inp["v_blk"], inp["k_cache"],
                                     inp["v_cache"], inp["ctx_lens"], mode)
        pert = {k: v.copy() for k, v in inp.items()}
        pert["v_cache"][0, :, 2] += 1.0
        out = oracle_mod.block_attn(pert["q"], pert["k_blk"], pert["v_blk"],
                                    pert["k_cache"], pert["v_cache"], pert["ctx_lens"], mode)
        assert np.all(np.abs(out - base).max(axis=(2, 3))[0] > 0)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_causal_row_equals_single_token_decode(oracle_mod, dtype):
    """Verify row i over cache[0,n) + block[0..i] == decode at n+i over a cache
    holding n+i rows plus the row itself as a 1-row block: bit-identical."""
    n, blk = 9, 5
    inp = _case(Hq=4, Hkv=2, D=16, blk=blk, ctx=(n,), cap=n + blk, dtype=dtype, seed=13)
    full = oracle_mod.block_attn(inp["q"], inp["k_blk"], inp["v_blk"], inp["k_cache"],
                                 inp["v_cache"], inp["ctx_lens"], 1)
    for i in range(blk):
        kc = inp["k_cache"].copy()
        vc = inp["v_cache"].copy()
        kc[0, :, n:n + i] = inp["k_blk"][0, :i].transpose(1, 0, 2)
        vc[0, :, n:n + i] = inp["v_blk"][0, :i].transpose(1, 0, 2)
        one = oracle_mod.block_attn(
            np.ascontiguousarray(inp["q"][:, i:i + 1]),
            np.ascontiguousarray(inp["k_blk"][:, i:i + 1]),
            np.ascontiguousarray(inp["v_blk"][:, i:i + 1]), kc, vc, [n + i], 1)
        assert np.array_equal(one[0, 0], full[0, i])


def test_bf16_is_exact_widening(oracle_mod):
    inp = _case(dtype="bf16", seed=14)
    wide = {k: (synth.bf16_to_f32(v) if v.dtype == np.uint16 else v) for k, v in inp.items()}
    a = oracle_mod.block_attn(inp["q"], inp["k_blk"], inp["v_blk"], inp["k_cache"],
                              inp["v_cache"], inp["ctx_lens"], 1)
    b = oracle_mod.block_attn(wide["q"], wide["k_blk"], wide["v_blk"], wide["k_cache"],
                              wide["v_cache"], wide["ctx_lens"], 1)
    assert np.array_equal(a, b)


def test_bad_arguments_rejected(oracle_mod):
    inp = _case()
    with pytest.raises(ValueError):
        oracle_mod.block_attn(inp["q"], inp["k_blk"], inp["v_blk"], inp["k_cache"],
                              inp["v_cache"], [21], 0)  # ctx > cap
    with pytest.raises(ValueError):
        oracle_mod.block_attn(inp["q"], inp["k_blk"], inp["v_blk"], inp["k_cache"],
                              inp["v_cache"], inp["ctx_lens"], 2)
