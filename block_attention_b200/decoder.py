"""The Orthrus consensus loop end to end on a small Qwen3-style decoder.

A frozen autoregressive decoder and, per layer, a separate-weight copy of the
attention projections for the diffusion view; both views share one KV cache
(cjcn.com.cn explainer of "Orthrus", §二).  A round (§四): the diffusion view
reads [anchor, MASK x 31] at positions [n, n+32) with bidirectional
attention inside the block and drafts one token per position; the AR view
verifies [anchor, d_0..d_30] causally; consensus accepts the agreeing prefix
plus one AR correction, and only the accepted rows' AR K/V enter the cache.

Every step runs in the library's kernels (include/orthrus.h and
include/orthrus_decoder.h); this module only allocates tensors, orders the
calls and keeps the per-sequence token lists on the host.  Batches hold
independent sequences of ragged lengths.

Exactness: in FP32 every kernel is row-invariant and the attention reduces in
an order fixed by absolute key position, so a verify row computes bitwise the
same logits as a one-token greedy decode of that position.  The consensus
loop therefore emits exactly the greedy AR tokens, for any draft (the
explainer's lossless claim, §四).  In BF16 the tensor-core attention's
reduction order depends on where keys sit (cache tile or block) and
trajectories may drift from FP32 (the reproduction study "How Lossless Is
Lossless Speculative Decoding? The Role of Numerical Precision in Orthrus",
abstract); ``trajectory_report`` measures how often.
"""
from __future__ import annotations

import numpy as np
import torch

import block_attention_b200 as ba

AR_VIEW, DIFFUSION_VIEW = 0, 1
_MASK_MODE = {AR_VIEW: ba.CAUSAL_VERIFY, DIFFUSION_VIEW: ba.BIDIR_BLOCK}


class DecodeState:
    """Per-batch KV cache [L, B, Hkv, cap, hd] (k and v) and device lengths."""

    def __init__(self, model: "TinyDecoder", B: int, cap: int):
        shape = (model.L, B, model.Hkv, cap, model.hd)
        self.k = torch.zeros(shape, dtype=model.dtype, device=model.device)
        self.v = torch.zeros(shape, dtype=model.dtype, device=model.device)
        self.ctx_lens = torch.zeros(B, dtype=torch.int32, device=model.device)
        self.err = torch.zeros(1, dtype=torch.int32, device=model.device)
        self.B, self.cap = B, cap


class TinyDecoder:
    """Random-init Qwen3-style decoder on the GPU, in FP32 or BF16.

    ``W`` is the weight dict of ``synth.decoder_weights`` (float32 arrays,
    matrices stored [out][in]); BF16 weights are its round-to-nearest-even
    bf16 values."""

    def __init__(self, W: dict, Hq: int, Hkv: int, hd: int, dtype=torch.float32,
                 device="cuda", eps: float = 1e-6, rope_theta: float = 1e6):
        self.dtype, self.device = dtype, torch.device(device)
        self.Hq, self.Hkv, self.hd, self.eps, self.theta = Hq, Hkv, hd, eps, rope_theta
        self.L = len(W["layers"])
        self.V, self.d = W["embed"].shape

        def t(*arrs):
            a = np.concatenate(arrs) if len(arrs) > 1 else arrs[0]
            return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(
                device=self.device, dtype=dtype)

        self.embed_w = t(W["embed"])
        self.layers = []
        for lw in W["layers"]:
            self.layers.append({
                "attn_norm": t(lw["attn_norm"]),
                "qkv": (t(lw["wq"], lw["wk"], lw["wv"]), t(lw["dq"], lw["dk"], lw["dv"])),
                "o": (t(lw["wo"]), t(lw["do"])),
                "ffn_norm": t(lw["ffn_norm"]),
                "gu": t(lw["w_gate"], lw["w_up"]),
                "down": t(lw["w_down"]),
            })
        self.final_norm = t(W["final_norm"])
        self.lm_head = t(W["lm_head"])
        self.mask_id = self.V - 1

    # ------------------------------------------------------------ forward
    def forward(self, st: DecodeState, tokens: torch.Tensor, view: int):
        """tokens int32 [B, R] at positions [ctx_lens[b], ctx_lens[b] + R).

        Returns logits [B*R, V] and this block's K/V [L, B, R, Hkv, hd]; the
        cache is read, never written."""
        B, R = tokens.shape
        rows = B * R
        Hq, Hkv, hd = self.Hq, self.Hkv, self.hd
        kb = torch.empty(self.L, B, R, Hkv, hd, dtype=self.dtype, device=self.device)
        vb = torch.empty_like(kb)
        q = torch.empty(B, R, Hq, hd, dtype=self.dtype, device=self.device)
        x = ba.embed(self.embed_w, tokens, err=st.err)
        mode = _MASK_MODE[view]
        for l, lw in enumerate(self.layers):
            h = ba.rmsnorm(x, lw["attn_norm"], self.eps)
            qkv = ba.linear(h, lw["qkv"][view])
            ba.qkv_rope(qkv, st.ctx_lens, B, R, Hq, Hkv, hd, self.theta, q=q, k=kb[l], v=vb[l])
            att = ba.block_attn(q, kb[l], vb[l], st.k[l], st.v[l], st.ctx_lens, mode,
                                err=st.err)
            ba.linear(att.view(rows, Hq * hd), lw["o"][view], residual=x, out=x)
            h = ba.rmsnorm(x, lw["ffn_norm"], self.eps)
            a = ba.swiglu(ba.linear(h, lw["gu"]))
            ba.linear(a, lw["down"], residual=x, out=x)
        h = ba.rmsnorm(x, self.final_norm, self.eps)
        return ba.linear(h, self.lm_head), kb, vb

    def commit(self, st: DecodeState, kb, vb, n_emit: torch.Tensor):
        ba.kv_commit(st.k, st.v, kb, vb, st.ctx_lens, n_emit, err=st.err)

    def check(self, st: DecodeState):
        e = int(st.err.item())
        if e != 0:
            raise ba.OrthrusError("device error word", e)

    # ------------------------------------------------------------ prefill
    def prefill(self, prompts, cap: int, chunk: int = 32):
        """Causal AR pass over every prompt in blocks of ``chunk`` rows.

        Returns the state (cache holding each prompt), the first generated
        token per sequence (host int32 [B]) and its log-probability (host
        float32 [B]).  Rows past a prompt's end are computed but never
        committed; causal masking keeps them from influencing the prompt's own
        rows."""
        B = len(prompts)
        lens = np.array([len(p) for p in prompts], np.int64)
        if lens.min() < 1 or lens.max() + chunk > cap:
            raise ValueError("prompt lengths must lie in [1, cap - chunk]")
        nchunks = int(-(-lens.max() // chunk))
        toks = np.zeros((B, nchunks * chunk), np.int32)
        for b, p in enumerate(prompts):
            toks[b, :len(p)] = p
        st = DecodeState(self, B, cap)
        first = np.zeros(B, np.int32)
        first_lp = np.zeros(B, np.float32)
        last_chunk, last_row = (lens - 1) // chunk, (lens - 1) % chunk
        for c in range(nchunks):
            t = torch.from_numpy(np.ascontiguousarray(toks[:, c * chunk:(c + 1) * chunk]))
            logits, kb, vb = self.forward(st, t.to(self.device), AR_VIEW)
            here = np.nonzero(last_chunk == c)[0]  # prompts that end in this chunk
            if here.size:
                idx = ba.vocab_argmax(logits)
                idx_h = idx.view(B, chunk).cpu().numpy()
                lp_h = ba.token_logprob(logits, idx).view(B, chunk).cpu().numpy()
                first[here] = idx_h[here, last_row[here]]
                first_lp[here] = lp_h[here, last_row[here]]
            valid = np.clip(lens - c * chunk, 0, chunk).astype(np.int32)
            self.commit(st, kb, vb, torch.from_numpy(valid).to(self.device))
        self.check(st)
        return st, first, first_lp

    # ---------------------------------------------------------- greedy AR
    def greedy(self, prompts, n_new: int, cap: int | None = None, logprob: bool = False):
        """Plain greedy autoregressive decoding, one token per forward:
        int32 [B, n_new] (the first token comes from the prefill); with
        ``logprob`` also each chosen token's log-probability, float32 [B, n_new]."""
        cap = cap or max(len(p) for p in prompts) + n_new + 64
        st, first, first_lp = self.prefill(prompts, cap)
        B = st.B
        out = torch.empty(n_new, B, dtype=torch.int32, device=self.device)
        out[0].copy_(torch.from_numpy(first))
        lp = torch.empty(n_new, B, dtype=torch.float32, device=self.device)
        lp[0].copy_(torch.from_numpy(first_lp))
        ones = torch.ones(B, dtype=torch.int32, device=self.device)
        for t in range(1, n_new):
            logits, kb, vb = self.forward(st, out[t - 1].view(B, 1), AR_VIEW)
            ba.vocab_argmax(logits, idx=out[t])
            if logprob:
                ba.token_logprob(logits, out[t], out=lp[t])
            self.commit(st, kb, vb, ones)
        self.check(st)
        toks = out.t().contiguous().cpu().numpy()
        return (toks, lp.t().contiguous().cpu().numpy()) if logprob else toks

    def sample_ar(self, prompts, n_new: int, temperature: float, seed: int,
                  cap: int | None = None) -> np.ndarray:
        """Plain autoregressive sampling at ``temperature``, one token per
        forward (the first token is the prefill's greedy one, as in the
        loop): int32 [B, n_new].  Step t uses Philox step t of ``seed``."""
        cap = cap or max(len(p) for p in prompts) + n_new + 64
        st, first, _ = self.prefill(prompts, cap)
        B = st.B
        out = torch.empty(n_new, B, dtype=torch.int32, device=self.device)
        out[0].copy_(torch.from_numpy(first))
        ones = torch.ones(B, dtype=torch.int32, device=self.device)
        for t in range(1, n_new):
            logits, kb, vb = self.forward(st, out[t - 1].view(B, 1), AR_VIEW)
            ba.vocab_sample(logits, temperature, seed, t, idx=out[t])
            self.commit(st, kb, vb, ones)
        self.check(st)
        return out.t().contiguous().cpu().numpy()

    # ----------------------------------------------------- consensus loop
    def consensus(self, prompts, n_new: int, blk: int = 32, draft_fn=None,
                  cap: int | None = None, temperature: float = 0.0, seed: int = 0):
        """The Orthrus loop: int32 [B, n_new] tokens and per-round stats.

        ``draft_fn(counts, d)`` may replace the diffusion drafts d (device
        int32 [B, blk]) given each sequence's emitted-token count, to show
        that any draft gives the greedy trajectory.  With ``temperature`` > 0
        the round samples instead (explainer §四): drafts d_j ~ softmax of the
        diffusion logits / T, and the stochastic consensus accepts d_j with
        probability min(1, p_j(d_j) / q_j(d_j)) and draws the correction from
        normalize(max(0, p - q)); round r uses Philox step r of ``seed``.
        Sequences that reach n_new tokens stop committing; the loop ends when
        all have."""
        cap = cap or max(len(p) for p in prompts) + n_new + 2 * blk
        st, first, _ = self.prefill(prompts, cap)
        B = st.B
        out = [[int(f)] for f in first]
        counts = np.ones(B, np.int64)
        anchor = torch.from_numpy(first).to(self.device)
        stats = {"rounds": 0, "seq_rounds": 0, "emitted": 0, "accept_len": []}
        while counts.min() < n_new:
            active = counts < n_new
            dtok = ba.block_tokens(anchor, None, blk, self.mask_id)
            dlog, _, _ = self.forward(st, dtok, DIFFUSION_VIEW)
            step = stats["rounds"]
            if temperature > 0:
                rows = B * blk
                logq = torch.empty(rows, dtype=torch.float32, device=self.device)
                lse_d = torch.empty_like(logq)
                d = ba.vocab_sample(dlog, temperature, seed, step, logprob=logq,
                                    lse=lse_d).view(B, blk)
            else:
                d = ba.vocab_argmax(dlog).view(B, blk)
            if draft_fn is not None:
                d = draft_fn(counts, d)
            vtok = ba.block_tokens(anchor, d, blk, self.mask_id)
            vlog, kb, vb = self.forward(st, vtok, AR_VIEW)
            if temperature > 0:
                if draft_fn is not None:  # replaced drafts: their log q under the diffusion view
                    ba.token_logprob(dlog, d.reshape(-1).contiguous(), temperature=temperature,
                                     out=logq, lse=lse_d)
                acc, ne, em, na = ba.consensus_sample(d.contiguous(), vlog, dlog, logq, lse_d,
                                                      temperature, seed, step)
            else:
                a = ba.vocab_argmax(vlog).view(B, blk)
                acc, ne, em, na = ba.consensus(d, a)
            ne_h, em_h, acc_h = ne.cpu().numpy(), em.cpu().numpy(), acc.cpu().numpy()
            commit = np.where(active, ne_h, 0).astype(np.int32)
            self.commit(st, kb, vb, torch.from_numpy(commit).to(self.device))
            anchor = na
            for b in np.nonzero(active)[0]:
                out[b] += em_h[b, :ne_h[b]].tolist()
            counts += commit
            stats["rounds"] += 1
            stats["seq_rounds"] += int(active.sum())
            stats["emitted"] += int(commit.sum())
            stats["accept_len"] += acc_h[active].tolist()
        self.check(st)
        stats["tokens_per_forward"] = stats["emitted"] / (2.0 * stats["seq_rounds"])
        return np.array([o[:n_new] for o in out], np.int32), stats


def teacher_drafts(ref: np.ndarray, device, wrong: bool = False, vocab: int | None = None):
    """draft_fn giving each sequence the reference trajectory's next tokens
    (every draft accepted), or, with ``wrong``, a token that differs from
    each of them (no draft accepted)."""
    B, n_new = ref.shape

    def fn(counts, d):
        blk = d.shape[1]
        out = np.zeros((B, blk), np.int32)
        for b in range(B):
            c = int(counts[b])
            seg = ref[b, c:c + blk]
            out[b, :seg.size] = seg
        if wrong:
            out = (out + 1) % (vocab - 1)
        return torch.from_numpy(out).to(device)

    return fn


def trajectory_report(test: np.ndarray, ref: np.ndarray) -> dict:
    """Exact-trajectory match rate of ``test`` against ``ref`` (rows =
    sequences) and where they first diverge."""
    eq = test == ref
    exact = eq.all(axis=1)
    first_div = np.where(exact, ref.shape[1], np.argmin(eq, axis=1))
    return {"sequences": int(ref.shape[0]), "tokens": int(ref.shape[1]),
            "exact_match_rate": float(exact.mean()),
            "token_match_rate": float(eq.mean()),
            "mean_first_divergence": float(first_div.mean())}


def perplexity_report(test: np.ndarray, ref: np.ndarray, ref_logprob: np.ndarray,
                      groups: int = 4) -> dict:
    """Exact-trajectory match of ``test`` against ``ref`` within groups of
    sequences ordered by the reference's response-conditional perplexity
    exp(-mean log p(token)) (the reproduction study finds exact matching
    strongly associated with it), plus the rank correlation between that
    perplexity and where the trajectories first diverge."""
    ppl = np.exp(-ref_logprob.astype(np.float64).mean(axis=1))
    eq = test == ref
    exact = eq.all(axis=1)
    first_div = np.where(exact, ref.shape[1], np.argmin(eq, axis=1))
    order = np.argsort(ppl, kind="stable")
    rows = []
    for gi, part in enumerate(np.array_split(order, groups)):
        rows.append({"group": gi, "sequences": int(part.size),
                     "perplexity_min": float(ppl[part].min()),
                     "perplexity_max": float(ppl[part].max()),
                     "exact_match_rate": float(exact[part].mean()),
                     "mean_first_divergence": float(first_div[part].mean())})
    rank = lambda a: np.argsort(np.argsort(a, kind="stable"), kind="stable").astype(np.float64)
    rho = float(np.corrcoef(rank(ppl), rank(first_div))[0, 1]) if ref.shape[0] > 1 else 0.0
    return {"groups": rows, "spearman_perplexity_vs_first_divergence": rho}
