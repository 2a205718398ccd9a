"""Whole-round parity in the launch configuration bench.py times: the
DecodeRound driver (all layers, both views, argmax of both views, consensus,
commit) captured as CUDA graphs with programmatic dependent launch and early
K/V streaming, replayed, then checked against the CPU oracle: attention of
sampled layers within the bf16 tolerance, every integer result and every
committed cache byte bit-exact."""
import numpy as np
import pytest
import torch

import oracle
from block_attention_b200 import synth
from block_attention_b200.round import DecodeRound
from gpu_util import TOL, rel_err_rows

pytestmark = pytest.mark.gpu


def _np(t):
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def _check_round(rnd, sample_layers, oracle_mod):
    # snapshot what the oracle needs before the round mutates the cache
    lens0 = rnd.ctx_base.cpu().numpy()
    pre = {l: (_np(rnd.k_cache[l]).copy(), _np(rnd.v_cache[l]).copy()) for l in sample_layers}
    rnd.capture()      # one eager round, then graphs (each replay restarts from lens0)
    rnd.replay()
    rnd.replay()
    torch.cuda.synchronize()
    assert int(rnd.err.item()) == 0
    for l in sample_layers:
        kc, vc = pre[l]
        for view in (0, 1):
            ref = oracle_mod.block_attn(_np(rnd.q[view, l]), _np(rnd.k_blk[view, l]),
                                        _np(rnd.v_blk[view, l]), kc, vc, lens0, view)
            got = synth.bf16_to_f32(_np(rnd.out[view, l]))
            e = rel_err_rows(got, ref)
            assert e.max() <= TOL["bf16"], (l, view, e.max())
    # argmax of both views, consensus
    B, blk = rnd.B, rnd.blk
    tok_ref = [oracle_mod.vocab_argmax(_np(rnd.logits[v])) for v in (0, 1)]
    for v in (0, 1):
        np.testing.assert_array_equal(_np(rnd.tok[v]), tok_ref[v])
    np.testing.assert_array_equal(tok_ref[0].reshape(B, blk), rnd.draft_planted)
    np.testing.assert_array_equal(tok_ref[1].reshape(B, blk), rnd.verify_planted)
    L, ne, em, na = oracle_mod.consensus(tok_ref[0].reshape(B, blk), tok_ref[1].reshape(B, blk))
    np.testing.assert_array_equal(_np(rnd.accept_len), L)
    np.testing.assert_array_equal(_np(rnd.n_emit), ne)
    np.testing.assert_array_equal(_np(rnd.emitted), em)
    np.testing.assert_array_equal(_np(rnd.next_anchor), na)
    # commit: every sampled layer's cache equals the oracle's commit of the
    # verify block, bytes past the accepted rows untouched
    for l in sample_layers:
        kc, vc = pre[l]
        # the oracle commits in place: kc/vc now hold the expected caches
        new = oracle_mod.kv_commit(kc, vc, np.ascontiguousarray(_np(rnd.k_blk[1, l])),
                                   np.ascontiguousarray(_np(rnd.v_blk[1, l])), lens0, ne)
        assert np.array_equal(_np(rnd.k_cache[l]), kc)
        assert np.array_equal(_np(rnd.v_cache[l]), vc)
    np.testing.assert_array_equal(_np(rnd.ctx_lens), new)


def test_qwen3_8b_round_as_benchmarked(oracle_mod):
    w = synth.WORKLOADS["qwen3_8b"]
    rnd = DecodeRound(layers=w["layers"], B=1, Hq=w["Hq"], Hkv=w["Hkv"], D=w["D"],
                      blk=w["blk"], vocab=w["vocab"], ctx_lens=[w["ctx"]], seed=1003,
                      device="cuda")
    _check_round(rnd, [0, 17, 35], oracle_mod)


def test_ragged_batch_round(oracle_mod):
    lens = synth.ragged_lens(5, 300, 5000, seed=1004)
    rnd = DecodeRound(layers=3, B=5, Hq=32, Hkv=8, D=128, blk=32, vocab=4096,
                      ctx_lens=lens, seed=1004, device="cuda")
    _check_round(rnd, [0, 2], oracle_mod)
