"""A round with the attention block's projections and the LM head on the path
(block_attention_b200.projected), at the Qwen3-8B head layout with two layers,
a 1000-key context and a 16384-entry vocabulary, checked op by op against the
float64 oracle on the GPU's own inputs: the QKV projection and the output
projection with its residual (per row within the bf16 tolerance, the bf16
rounding agreeing on nearly every element), the round's QKV projection with
RoPE in its epilogue (the same bits as the projection followed by RoPE), the
attention of both views (bf16 tolerance), the LM head's argmax
(bit-exact wherever the top-2 gap exceeds the fp32 error scale), consensus and
commit bit-exact; and the graph replay equals the eager round."""
import numpy as np
import pytest
import torch

import block_attention_b200 as ba
from block_attention_b200.projected import ProjectedRound
from gpu_util import TOL, rel_err_rows

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _f(bits):
    return (np.asarray(bits, np.uint32) << 16).view(np.float32).astype(np.float64)


def _check_projection(oracle_mod, x, w, y, residual=None):
    ref, exact, _ = oracle_mod.projection(_bits(x), _bits(w),
                                          None if residual is None else _bits(residual))
    got = _bits(y)
    want = exact if residual is None else _f(ref)
    err = np.abs(_f(got) - want).max(axis=1) / np.maximum(np.abs(want).max(axis=1), 1e-6)
    assert err.max() <= TOL["bf16"], err.max()
    assert (got == ref).mean() > 0.9


def test_projected_round_op_by_op(oracle_mod):
    rnd = ProjectedRound(layers=2, ctx=1000, vocab=16384, seed=21, prefetch="both")
    blk, L = rnd.blk, rnd.L
    mode = {0: ba.BIDIR_BLOCK, 1: ba.CAUSAL_VERIFY}
    lens0 = rnd.ctx_base.cpu().numpy()
    kc0 = {l: _bits(rnd.k_cache[l]) for l in range(L)}
    vc0 = {l: _bits(rnd.v_cache[l]) for l in range(L)}
    rnd.ctx_lens.copy_(rnd.ctx_base)
    table = ba.rope_table(rnd.ctx_lens, 1, blk, rnd.D, rnd.theta)
    for v in (0, 1):
        draft = None if v == 0 else rnd.tok_out[0].view(1, blk)
        ba.block_tokens(rnd.anchor, draft, blk, rnd.mask_id, out=rnd.tok_in[v])
        ba.embed(rnd.embed_w, rnd.tok_in[v].view(-1), out=rnd.x, err=rnd.err)
        for l in range(L):
            ba.rmsnorm(rnd.x, rnd.gain[l], rnd.eps, out=rnd.h)
            h = rnd.h.clone()
            ba.linear_tc(rnd.h, rnd.wqkv[v, l], out=rnd.qkv, err=rnd.err)
            torch.cuda.synchronize()
            _check_projection(oracle_mod, h, rnd.wqkv[v, l], rnd.qkv)
            ba.qkv_rope(rnd.qkv, rnd.ctx_lens, 1, blk, rnd.Hq, rnd.Hkv, rnd.D, rnd.theta,
                        q=rnd.q, k=rnd.k_blk[v, l], v=rnd.v_blk[v, l])
            fq, fk, fv = (torch.empty_like(t) for t in (rnd.q, rnd.k_blk[v, l], rnd.v_blk[v, l]))
            ba.linear_tc_qkv_rope(h, rnd.wqkv[v, l], rnd.Hq, rnd.Hkv, table, q=fq, k=fk, v=fv,
                                  err=rnd.err)
            torch.cuda.synchronize()
            assert torch.equal(fq, rnd.q) and torch.equal(fk, rnd.k_blk[v, l])
            assert torch.equal(fv, rnd.v_blk[v, l])
            ba.block_attn(rnd.q, rnd.k_blk[v, l], rnd.v_blk[v, l], rnd.k_cache[l],
                          rnd.v_cache[l], rnd.ctx_lens, mode[v], out=rnd.attn, max_ctx=rnd.ctx,
                          err=rnd.err)
            torch.cuda.synchronize()
            ref = oracle_mod.block_attn(_bits(rnd.q), _bits(rnd.k_blk[v, l]),
                                        _bits(rnd.v_blk[v, l]), kc0[l], vc0[l], lens0, mode[v])
            got = (_bits(rnd.attn).astype(np.uint32) << 16).view(np.float32)
            assert rel_err_rows(got, ref).max() <= TOL["bf16"], (v, l)
            x_in = rnd.x.clone()
            ba.linear_tc(rnd.attn.view(blk, -1), rnd.wo[v, l], residual=rnd.x, out=rnd.x,
                         err=rnd.err)
            torch.cuda.synchronize()
            _check_projection(oracle_mod, rnd.attn.view(blk, -1), rnd.wo[v, l], rnd.x, x_in)
        ba.rmsnorm(rnd.x, rnd.gain_final, rnd.eps, out=rnd.h)
        ba.lm_head_argmax(rnd.h, rnd.embed_w, idx=rnd.tok_out[v], err=rnd.err)
        torch.cuda.synchronize()
        idx, _, gap, mag = oracle_mod.lm_head_argmax(_bits(rnd.h), _bits(rnd.embed_w))
        clear = gap > 2 * 2.0 ** -12 * mag
        got = rnd.tok_out[v].cpu().numpy()
        np.testing.assert_array_equal(got[clear], idx[clear])
        assert clear.mean() > 0.9
    tok = [rnd.tok_out[v].cpu().numpy() for v in (0, 1)]
    ba.consensus(rnd.tok_out[0].view(1, blk), rnd.tok_out[1].view(1, blk),
                 accept_len=rnd.accept_len, n_emit=rnd.n_emit, emitted=rnd.emitted,
                 next_anchor=rnd.next_anchor)
    torch.cuda.synchronize()
    L_, ne, em, na = oracle_mod.consensus(tok[0][None], tok[1][None])
    np.testing.assert_array_equal(rnd.accept_len.cpu().numpy(), L_)
    np.testing.assert_array_equal(rnd.n_emit.cpu().numpy(), ne)
    np.testing.assert_array_equal(rnd.next_anchor.cpu().numpy(), na)
    assert int(rnd.err.item()) == 0

    # the captured round (graph, PDL, early K/V, next-layer L2 warm-up) gives
    # the same tokens as the eager ops above, every time it is replayed
    rnd.capture()
    for _ in range(2):
        rnd.replay()
        torch.cuda.synchronize()
        for v in (0, 1):
            np.testing.assert_array_equal(rnd.tok_out[v].cpu().numpy(), tok[v])
        np.testing.assert_array_equal(rnd.n_emit.cpu().numpy(), ne)
    assert int(rnd.err.item()) == 0
