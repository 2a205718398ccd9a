"""Pins for the oracle's tiny decoder and its consensus loop.

* The AR view of the oracle's decoder is checked against Hugging Face's
  LlamaForCausalLM in float64 (an independent library implementation of the
  same architecture: RMSNorm, RoPE with half-split pairs, GQA, SwiGLU, untied
  LM head).  Its RMSNorm and RoPE tables run in float32 internally, hence the
  1e-4 tolerance: a structural mistake (dropped term, wrong sign, wrong index,
  transposed weight) shows up at order 1.
* The diffusion view is checked the same way with the diffusion attention copy
  swapped in, the AR prefix cache kept, and an all-visible 4-D mask over the
  block (Orthrus explainer §二: Q_diff over the AR cache and the block's own
  K_diff/V_diff; §三: bidirectional inside the block).
* Row invariance: a multi-row causal pass equals single-token decoding bitwise.
* Losslessness (explainer §四 and Q1; FP32 result in the reproduction's
  abstract): the consensus loop's output equals greedy AR decoding exactly,
  for the model's own drafts and for perfect, always-wrong, random and
  planted-prefix drafts; every round emits >= 1 token; a perfect draft takes
  whole blocks; tokens per forward >= 0.5.
"""
import json
import os

import numpy as np
import pytest
import torch

from block_attention_b200 import synth

SMALL = dict(V=256, d=64, L=2, Hq=4, Hkv=2, hd=16, ffn=96)
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def small(oracle_mod):
    cfg = oracle_mod.model_cfg(**SMALL)
    W = synth.decoder_weights(**SMALL, seed=3, std=0.2)
    return cfg, W, oracle_mod.pack_weights(cfg, W)


def _hf_model(W, view):
    from transformers import LlamaConfig, LlamaForCausalLM
    c = LlamaConfig(vocab_size=SMALL["V"], hidden_size=SMALL["d"],
                    intermediate_size=SMALL["ffn"], num_hidden_layers=SMALL["L"],
                    num_attention_heads=SMALL["Hq"], num_key_value_heads=SMALL["Hkv"],
                    head_dim=SMALL["hd"], rms_norm_eps=1e-6,
                    rope_parameters={"rope_type": "default", "rope_theta": 1e6},
                    tie_word_embeddings=False, attention_bias=False, mlp_bias=False,
                    max_position_embeddings=512, attn_implementation="eager")
    m = LlamaForCausalLM(c).to(torch.float64).eval()
    t = lambda a: torch.from_numpy(np.asarray(a, np.float64))
    with torch.no_grad():
        m.model.embed_tokens.weight.copy_(t(W["embed"]))
        for l, lw in enumerate(W["layers"]):
            L = m.model.layers[l]
            L.input_layernorm.weight.copy_(t(lw["attn_norm"]))
            pre = "d" if view == 1 else "w"
            L.self_attn.q_proj.weight.copy_(t(lw[pre + "q"]))
            L.self_attn.k_proj.weight.copy_(t(lw[pre + "k"]))
            L.self_attn.v_proj.weight.copy_(t(lw[pre + "v"]))
            L.self_attn.o_proj.weight.copy_(t(lw["do" if view == 1 else "wo"]))
            L.post_attention_layernorm.weight.copy_(t(lw["ffn_norm"]))
            L.mlp.gate_proj.weight.copy_(t(lw["w_gate"]))
            L.mlp.up_proj.weight.copy_(t(lw["w_up"]))
            L.mlp.down_proj.weight.copy_(t(lw["w_down"]))
        m.model.norm.weight.copy_(t(W["final_norm"]))
        m.lm_head.weight.copy_(t(W["lm_head"]))
    return m


def _close(a, b, tol=1e-4):
    err = np.abs(a - b).max() / max(np.abs(b).max(), 1e-30)
    assert err < tol, err


def test_ar_view_matches_hf_llama(oracle_mod, small):
    cfg, W, wf = small
    toks = synth.rng(31).integers(0, SMALL["V"], size=11).astype(np.int32)
    seq = oracle_mod.Sequence(cfg, 16)
    logits, _, _ = oracle_mod.forward(cfg, wf, seq, toks, view=0)
    hf = _hf_model(W, 0)
    with torch.no_grad():
        ref = hf(torch.from_numpy(toks.astype(np.int64))[None]).logits[0].numpy()
    _close(logits, ref)


def test_diffusion_view_matches_hf_with_swapped_attention(oracle_mod, small):
    cfg, W, wf = small
    g = synth.rng(32)
    prefix = g.integers(0, SMALL["V"], size=9).astype(np.int32)
    block = np.array([7] + [SMALL["V"] - 1] * 5, np.int32)
    seq, _ = oracle_mod.prefill(cfg, wf, prefix, cap=20)
    dlog, _, _ = oracle_mod.forward(cfg, wf, seq, block, view=1)

    from transformers import DynamicCache
    ar = _hf_model(W, 0)
    diff = _hf_model(W, 1)
    with torch.no_grad():
        cache = DynamicCache(config=ar.config)
        ar(torch.from_numpy(prefix.astype(np.int64))[None], past_key_values=cache,
           use_cache=True)
        n, r = len(prefix), len(block)
        mask = torch.zeros(1, 1, r, n + r, dtype=torch.float64)  # all visible
        out = diff(torch.from_numpy(block.astype(np.int64))[None], past_key_values=cache,
                   attention_mask=mask, position_ids=torch.arange(n, n + r)[None],
                   use_cache=True)
    _close(dlog, out.logits[0].numpy())


def test_multi_row_pass_equals_token_by_token_decode(oracle_mod, small):
    cfg, W, wf = small
    toks = synth.rng(33).integers(0, SMALL["V"], size=7).astype(np.int32)
    seq = oracle_mod.Sequence(cfg, 10)
    full, kb, vb = oracle_mod.forward(cfg, wf, seq, toks, view=0)
    seq2 = oracle_mod.Sequence(cfg, 10)
    for i, t in enumerate(toks):
        one, k1, v1 = oracle_mod.forward(cfg, wf, seq2, [t], view=0)
        assert np.array_equal(one[0], full[i])
        assert np.array_equal(k1[:, 0], kb[:, i]) and np.array_equal(v1[:, 0], vb[:, i])
        oracle_mod.commit_rows(seq2, k1, v1, 1)


DRAFTS = ["model", "perfect", "wrong", "random", "planted"]


@pytest.mark.parametrize("blk", [8, 32])
@pytest.mark.parametrize("kind", DRAFTS)
def test_consensus_loop_equals_greedy_for_any_draft(oracle_mod, small, kind, blk):
    cfg, W, wf = small
    fig = json.load(open(os.path.join(GOLDEN, "pages_figures.json")))
    n_new = 40
    for p, prompt in enumerate(synth.prompts(2, SMALL["V"], 3, 10, seed=34 + blk,
                                             exclude=SMALL["V"] - 1)):
        ref = oracle_mod.greedy_ar(cfg, wf, prompt, n_new + blk + 1)
        g = synth.rng(35, p, blk)

        def draft_fn(r, n, d):
            # position n is the anchor; d[j] predicts the token at n + j + 1
            pos0 = n - len(prompt)  # index of the anchor in ref
            truth = ref[pos0 + 1: pos0 + 1 + blk]
            if kind == "model":
                return d
            if kind == "perfect":
                return truth
            if kind == "wrong":
                return (truth + 1) % SMALL["V"]
            if kind == "random":
                return g.integers(0, SMALL["V"], size=blk)
            L = int(g.integers(0, blk + 1))
            out = g.integers(0, SMALL["V"], size=blk)
            out[:L] = truth[:L]
            if L < blk and out[L] == truth[L]:
                out[L] = (truth[L] + 1) % SMALL["V"]
            return out

        got, st = oracle_mod.consensus_decode(cfg, wf, prompt, n_new, blk=blk,
                                              draft_fn=draft_fn)
        np.testing.assert_array_equal(got, ref[:n_new])
        assert min(st["n_emit"]) >= fig["min_tokens_per_round"]["value"]
        tpf = sum(st["n_emit"]) / (2.0 * st["rounds"])
        assert tpf >= fig["tpf_lower_bound"]["value"]
        if kind == "perfect":
            assert all(e == blk for e in st["n_emit"])
        if kind == "wrong":
            assert all(e == 1 for e in st["n_emit"])
