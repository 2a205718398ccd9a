"""GPU parity of the stochastic consensus (cjcn.com.cn explainer of "Orthrus",
section 四: strict rejection sampling for sampling with a temperature) against
the float64 oracle in oracle/sampling.py, through the C ABI.

Sampled indices depend on floating point only through near-ties; each
comparison skips the rows whose oracle margin (gap between the two best
Gumbel keys, or distance of an acceptance test to its threshold) is below a
few units of FP32 rounding, and checks that what it skips is still valid."""
import numpy as np
import pytest
import torch
from scipy.stats import chi2

import block_attention_b200 as ba
from block_attention_b200 import synth
from gpu_util import to_dev, to_host
from oracle import sampling as S

pytestmark = pytest.mark.gpu

SAFE = 1e-3  # margin (in log units) beyond FP32 rounding of the keys


@pytest.mark.parametrize("dtype,rows,vocab,T", [("f32", 32, 151936, 0.8), ("bf16", 7, 1000, 1.3),
                                                ("f32", 5, 1001, 1.0), ("bf16", 3, 6, 0.7)])
def test_vocab_sample_matches_oracle(oracle_mod, dtype, rows, vocab, T):
    for step in (0, 3):
        x = synth.logits(synth.rng(600 + step, len(dtype)), rows, vocab, dtype=dtype)
        lp = torch.empty(rows, dtype=torch.float32, device="cuda")
        lse = torch.empty_like(lp)
        plain = to_host(ba.vocab_sample(to_dev(x), T, seed=2025, step=step))
        got = to_host(ba.vocab_sample(to_dev(x), T, seed=2025, step=step, logprob=lp, lse=lse))
        np.testing.assert_array_equal(got, plain)  # the fused log-prob leaves the draw alone
        ref, gap = S.vocab_sample(x, T, seed=2025, step=step)
        ref_lp, ref_lse = oracle_mod.token_logprob(x, got, temperature=T, return_lse=True)
        np.testing.assert_allclose(to_host(lp), ref_lp, rtol=0, atol=1e-4)
        np.testing.assert_allclose(to_host(lse), ref_lse, rtol=1e-6, atol=1e-4)
        safe = gap > SAFE
        assert safe.mean() > 0.9
        np.testing.assert_array_equal(got[safe], ref[safe])
        assert ((got >= 0) & (got < vocab)).all()


@pytest.mark.parametrize("dtype,rows,vocab", [("f32", 16, 5000), ("bf16", 16, 5000),
                                              ("bf16", 6, 151936), ("f32", 3, 100)])
def test_token_logprob_temperature_and_lse(oracle_mod, dtype, rows, vocab):
    """Rows of one, two (ragged) and 38 (Qwen3 vocabulary, ragged) 4096-chunks."""
    x = synth.logits(synth.rng(620, len(dtype)), rows, vocab, dtype=dtype)
    idx = synth.rng(621).integers(0, vocab, rows).astype(np.int32)
    lse = torch.empty(rows, dtype=torch.float32, device="cuda")
    got = to_host(ba.token_logprob(to_dev(x), to_dev(idx), temperature=0.7, lse=lse))
    ref, ref_lse = oracle_mod.token_logprob(x, idx, temperature=0.7, return_lse=True)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-4)
    np.testing.assert_allclose(to_host(lse), ref_lse, rtol=1e-6, atol=1e-4)


def test_token_logprob_workspace_reused_across_shapes(oracle_mod):
    """One workspace for calls of different row counts: a small call's chunk
    pairs lie where a larger call keeps its tickets, so every call must leave
    the buffer zero."""
    ws = ba.Workspace("cuda")
    for i, rows in enumerate((8, 256, 3, 256, 40)):
        x = synth.logits(synth.rng(650 + i), rows, 8192)
        idx = synth.rng(660 + i).integers(0, 8192, rows).astype(np.int32)
        lse = torch.empty(rows, dtype=torch.float32, device="cuda")
        got = to_host(ba.token_logprob(to_dev(x), to_dev(idx), temperature=0.9, lse=lse,
                                       workspace=ws))
        ref, ref_lse = oracle_mod.token_logprob(x, idx, temperature=0.9, return_lse=True)
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-4)
        np.testing.assert_allclose(to_host(lse), ref_lse, rtol=1e-6, atol=1e-4)
        assert not ws.buf.any().item()


def test_sampling_workspaces_left_zero_across_shapes():
    """vocab_sample and consensus_sample leave their workspaces all zero, so
    one buffer serves calls of any shape (pair offsets move with the shape)."""
    ws_s, ws_c = ba.Workspace("cuda"), ba.Workspace("cuda")
    f32 = dict(dtype=torch.float32, device="cuda")
    for i, (B, blk, V) in enumerate(((1, 32, 151936), (8, 4, 9000), (3, 32, 151936),
                                     (40, 8, 5000))):
        g = np.random.default_rng(670 + i)
        zq = torch.from_numpy(g.normal(0, 2, (B * blk, V)).astype(np.float32)).cuda()
        zp = zq + torch.from_numpy(g.normal(0, 1, (B * blk, V)).astype(np.float32)).cuda()
        logq, lse_q = torch.empty(B * blk, **f32), torch.empty(B * blk, **f32)
        d = ba.vocab_sample(zq, 0.9, 5, i, logprob=logq, lse=lse_q, workspace=ws_s)
        ba.consensus_sample(d.view(B, blk), zp, zq, logq, lse_q, 0.9, 5, i, workspace=ws_c)
        torch.cuda.synchronize()
        assert not ws_s.buf.any().item() and not ws_c.buf.any().item()


def _gpu_round(zp, zq, B, blk, T, seed, step, logs=None):
    """The stochastic round's kernels on device logits: drafts with their log q,
    then the consensus (log p, acceptance, correction)."""
    tq, tp = to_dev(zq), to_dev(zp)
    f32 = dict(dtype=torch.float32, device="cuda")
    logq, lse_q, logp, lse_p = (torch.empty(B * blk, **f32) for _ in range(4))
    d = ba.vocab_sample(tq, T, seed, step, logprob=logq, lse=lse_q)
    out = ba.consensus_sample(d.view(B, blk), tp, tq, logq, lse_q, T, seed, step, logp=logp,
                              lse_ar=lse_p)
    if logs is not None:
        logs.update(logq=to_host(logq), lse_q=to_host(lse_q), logp=to_host(logp),
                    lse_p=to_host(lse_p))
    return to_host(d).reshape(B, blk), [to_host(o) for o in out]


@pytest.mark.parametrize("B,blk,V,T", [(8, 32, 4096, 1.0), (3, 8, 151936, 0.8),
                                       (4, 16, 1000, 1.2)])
def test_consensus_sample_matches_oracle(oracle_mod, B, blk, V, T):
    """Correction rows of one, 38 (Qwen3 vocabulary, ragged) and a partial chunk."""
    g = np.random.default_rng(630 + V)
    zq = g.normal(0, 2, (B * blk, V)).astype(np.float32)
    # the AR view drifts away from the draft view along the block, faster for
    # later sequences: accept lengths spread over the block
    sig = np.array([[0.64 / blk * (b + 1) * (j + 1) for j in range(blk)] for b in range(B)])
    zp = (zq + g.normal(0, 1, (B * blk, V)) * sig.reshape(-1, 1)).astype(np.float32)
    for step in (1, 2):
        logs = {}
        draft, (L, ne, em, na) = _gpu_round(zp, zq, B, blk, T, seed=31, step=step, logs=logs)
        rL, rne, rem, rna, margin = S.consensus_sample(draft, zp, zq, T, seed=31, step=step)
        for z, lp, ls in ((zq, "logq", "lse_q"), (zp, "logp", "lse_p")):
            ref_lp, ref_lse = oracle_mod.token_logprob(z, draft.reshape(-1), temperature=T,
                                                       return_lse=True)
            np.testing.assert_allclose(logs[lp], ref_lp, rtol=0, atol=1e-4)
            np.testing.assert_allclose(logs[ls], ref_lse, rtol=1e-6, atol=1e-4)
        for b in range(B):
            assert 0 <= L[b] <= blk and ne[b] == min(L[b] + 1, blk)
            np.testing.assert_array_equal(em[b, :min(L[b], ne[b])], draft[b, :min(L[b], ne[b])])
            assert (em[b, ne[b]:] == -1).all() and 0 <= em[b, ne[b] - 1] < V
            assert na[b] == em[b, ne[b] - 1]
            if margin[b] > SAFE:
                assert (L[b], ne[b]) == (rL[b], rne[b]), (step, b)
                np.testing.assert_array_equal(em[b], rem[b])
        if B >= 8:
            assert len(set(L.tolist())) > 2  # the planted drift spreads the accept lengths
        assert (L < blk).any()  # a correction was drawn


def test_first_emitted_token_follows_ar_distribution_on_gpu():
    """Lossless: drafts from q, verification by p -- the first emitted token
    is distributed as p (blk = 1), through the GPU kernels end to end."""
    zq = np.array([1.5, 0.2, -0.3, 0.9, -1.0, 0.0], np.float32)
    zp = np.array([-0.2, 1.1, 0.4, -0.8, 0.6, 0.1], np.float32)
    B, T = 16384, 0.9
    _, (L, ne, em, na) = _gpu_round(np.tile(zp, (B, 1)), np.tile(zq, (B, 1)), B, 1, T, 99, 0)
    counts = np.bincount(em[:, 0], minlength=6).astype(np.float64)

    def pval(probs):
        e = B * probs
        return chi2.sf(((counts - e) ** 2 / e).sum(), df=5)
    soft = lambda z: np.exp(z / T - (z / T).max()) / np.exp(z / T - (z / T).max()).sum()
    assert pval(soft(zp.astype(np.float64))) > 1e-4
    assert pval(soft(zq.astype(np.float64))) < 1e-6


def test_low_temperature_equals_greedy_consensus():
    B, blk, V, T = 4, 32, 1000, 1e-6
    g = np.random.default_rng(640)
    zq = g.normal(0, 1, (B * blk, V)).astype(np.float32)
    zp = g.normal(0, 1, (B * blk, V)).astype(np.float32)
    for b in range(B):
        zp[b * blk:b * blk + 5 * b] = zq[b * blk:b * blk + 5 * b]
    draft, (L, ne, em, na) = _gpu_round(zp, zq, B, blk, T, seed=4, step=0)
    d = to_dev(draft.astype(np.int32))
    a = ba.vocab_argmax(to_dev(zp)).view(B, blk)
    np.testing.assert_array_equal(draft.reshape(-1), to_host(ba.vocab_argmax(to_dev(zq))))
    gL, gne, gem, gna = [to_host(o) for o in ba.consensus(d, a)]
    np.testing.assert_array_equal(L, gL)
    np.testing.assert_array_equal(ne, gne)
    np.testing.assert_array_equal(em, gem)
    np.testing.assert_array_equal(na, gna)
