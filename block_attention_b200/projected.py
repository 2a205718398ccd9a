"""One Orthrus decoding round at the Qwen3-8B shape with the attention block's
projections and the LM head on the path.

The round of ``round.DecodeRound`` takes each layer's Q and block K/V, and each
view's logits, as synthetic inputs.  Here they are computed, as in the model
the pages describe (cjcn.com.cn explainer of "Orthrus", §二: the diffusion view
has its own copy of the attention projections; the embedding, norms and LM head
are shared; both views read the one KV cache; §四: draft, verify, consensus,
update):

  per view v (0 = diffusion over [anchor, MASK x (blk-1)], 1 = AR verify over
  [anchor, d0 .. d_{blk-2}]):
      x = embed[block tokens]
      per layer l:  h = RMSNorm(x)
                    q, k, v = RoPE split of h Wqkv[v, l]^T at positions
                              n .. n+blk-1  (tensor cores, RoPE in the epilogue)
                    a = block attention over cache_l ‖ block k/v  (mask of v)
                    x = x + a Wo[v, l]^T                          (tensor cores)
      tokens_v = argmax_V RMSNorm(x) E^T                (LM head, argmax fused)
  consensus(tokens_0, tokens_1); commit the AR view's accepted K/V rows.

The FFN of each layer is not on this path (its weights do not meet the
method's attention or its round structure); everything else of the attention
path is.  The embedding doubles as the LM head (tied).  Weights are random
(N(0, 0.02), norm gains 1 + N(0, 0.02)) in bf16; the caches are N(0, 1).  Every
kernel is this library's, through the C ABI, on the current stream; the round
is captured as one CUDA graph.

L2 warm-up (`prefetch`, off by default): "weights" has each QKV projection
warm L2 with the same layer's output-projection weights (34 MB, needed one
attention later) and each output projection with the next layer's QKV
weights (50 MB); "kv" has each attention warm L2 with the next layer's
cache; "both".  Measured at the Qwen3-8B shape every variant was slower
than none (4.76 ms per round; "kv" 4.96, "weights" 5.08-5.14, "both"
5.38): the prefetches compete with the stream on the critical path.
"""
from __future__ import annotations

import torch

from . import (ATTN_EARLY_KV, BIDIR_BLOCK, CAUSAL_VERIFY, Workspace, block_attn,
               block_tokens, consensus, embed, kv_commit, linear_tc, linear_tc_qkv_rope,
               lm_head_argmax, rmsnorm, rope_table)


class ProjectedRound:
    def __init__(self, *, layers=36, Hq=32, Hkv=8, D=128, d_model=4096, blk=32, vocab=151936,
                 ctx=8192, seed=0, device="cuda", eps=1e-6, theta=1e6, prefetch=None):
        self.dev = torch.device(device)
        self.L, self.Hq, self.Hkv, self.D, self.d, self.blk, self.V = (
            layers, Hq, Hkv, D, d_model, blk, vocab)
        if prefetch is True:
            prefetch = "weights"
        if prefetch not in (None, False, "weights", "kv", "both"):
            raise ValueError("prefetch: None, 'weights', 'kv' or 'both'")
        self.ctx, self.eps, self.theta, self.prefetch = ctx, eps, theta, prefetch or None
        self.cap = ctx + blk
        dev, bf = self.dev, torch.bfloat16
        g = torch.Generator(device=dev).manual_seed(seed)
        rnd = lambda *shape, std=1.0: (torch.randn(*shape, generator=g, device=dev) * std).to(bf)
        nqkv = (Hq + 2 * Hkv) * D
        self.embed_w = rnd(vocab, d_model, std=0.02)  # also the LM head
        self.gain = 1 + rnd(layers, d_model, std=0.02).float()
        self.gain = self.gain.to(bf)
        self.gain_final = (1 + rnd(d_model, std=0.02).float()).to(bf)
        self.wqkv = rnd(2, layers, nqkv, d_model, std=0.02)
        self.wo = rnd(2, layers, d_model, Hq * D, std=0.02)
        self.k_cache = rnd(layers, 1, Hkv, self.cap, D)
        self.v_cache = rnd(layers, 1, Hkv, self.cap, D)
        i32 = dict(dtype=torch.int32, device=dev)
        self.ctx_base = torch.full((1,), ctx, **i32)
        self.ctx_lens = self.ctx_base.clone()
        self.anchor = torch.randint(0, vocab - 1, (1,), generator=g, device=dev,
                                    dtype=torch.int32)
        self.mask_id = vocab - 1
        # per-round state
        self.tok_in = torch.empty(2, 1, blk, **i32)     # block tokens of each view
        self.tok_out = torch.empty(2, blk, **i32)       # each view's argmax tokens
        self.x = torch.empty(blk, d_model, dtype=bf, device=dev)
        self.h = torch.empty_like(self.x)
        self.qkv = torch.empty(blk, nqkv, dtype=bf, device=dev)
        self.rope_cs = torch.empty(blk, D // 2, 2, dtype=torch.float32, device=dev)
        self.q = torch.empty(1, blk, Hq, D, dtype=bf, device=dev)
        self.k_blk = torch.empty(2, layers, 1, blk, Hkv, D, dtype=bf, device=dev)
        self.v_blk = torch.empty_like(self.k_blk)
        self.attn = torch.empty(1, blk, Hq, D, dtype=bf, device=dev)
        self.accept_len = torch.empty(1, **i32)
        self.n_emit = torch.empty(1, **i32)
        self.emitted = torch.empty(1, blk, **i32)
        self.next_anchor = torch.empty(1, **i32)
        self.err = torch.zeros(1, **i32)
        self.ws = {k: Workspace(dev) for k in ("attn0", "attn1", "linear", "lm", "commit")}
        self.graph = None

    # ------------------------------------------------------------ one view
    def view(self, v):
        blk, L = self.blk, self.L
        draft = None if v == 0 else self.tok_out[0].view(1, blk)
        block_tokens(self.anchor, draft, blk, self.mask_id, out=self.tok_in[v])
        embed(self.embed_w, self.tok_in[v].view(-1), out=self.x, err=self.err)
        # the block's positions are the same in every layer: one cos/sin table
        rope_table(self.ctx_lens, 1, blk, self.D, self.theta, out=self.rope_cs)
        mode = BIDIR_BLOCK if v == 0 else CAUSAL_VERIFY
        for l in range(L):
            rmsnorm(self.x, self.gain[l], self.eps, out=self.h)
            w_pf = self.prefetch in ("weights", "both")
            linear_tc_qkv_rope(self.h, self.wqkv[v, l], self.Hq, self.Hkv, self.rope_cs,
                               q=self.q, k=self.k_blk[v, l], v=self.v_blk[v, l],
                               l2_next=self.wo[v, l] if w_pf else None, err=self.err,
                               workspace=self.ws["linear"])
            nxt = (l + 1) % L
            # the kernel before the attention (the QKV projection) writes
            # neither a cache nor the lengths: the cache may stream while it
            # finishes
            block_attn(self.q, self.k_blk[v, l], self.v_blk[v, l], self.k_cache[l],
                       self.v_cache[l], self.ctx_lens, mode, out=self.attn, max_ctx=self.ctx,
                       err=self.err, workspace=self.ws[f"attn{v}"], flags=ATTN_EARLY_KV,
                       next_kv=(self.k_cache[nxt], self.v_cache[nxt])
                       if self.prefetch in ("kv", "both") else None)
            linear_tc(self.attn.view(blk, -1), self.wo[v, l], residual=self.x, out=self.x,
                      l2_next=self.wqkv[v, l + 1] if w_pf and l + 1 < L else None,
                      err=self.err, workspace=self.ws["linear"])
        rmsnorm(self.x, self.gain_final, self.eps, out=self.h)
        lm_head_argmax(self.h, self.embed_w, idx=self.tok_out[v], err=self.err,
                       workspace=self.ws["lm"])

    def step(self):
        """One round: both views, consensus, commit; the lengths then return
        to the base context so that every step is the same round."""
        self.ctx_lens.copy_(self.ctx_base)
        self.view(0)
        self.view(1)
        blk = self.blk
        consensus(self.tok_out[0].view(1, blk), self.tok_out[1].view(1, blk),
                  accept_len=self.accept_len, n_emit=self.n_emit, emitted=self.emitted,
                  next_anchor=self.next_anchor)
        kv_commit(self.k_cache, self.v_cache, self.k_blk[1], self.v_blk[1], self.ctx_lens,
                  self.n_emit, err=self.err, workspace=self.ws["commit"])

    def capture(self):
        side = torch.cuda.Stream(device=self.dev)
        side.wait_stream(torch.cuda.current_stream(self.dev))
        with torch.cuda.stream(side):
            self.step()
        torch.cuda.current_stream(self.dev).wait_stream(side)
        torch.cuda.synchronize(self.dev)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.step()
        torch.cuda.synchronize(self.dev)

    def replay(self):
        self.graph.replay()

    # ------------------------------------------------------------ accounting
    def bytes_per_round(self) -> dict:
        """Algorithmic HBM bytes of one round by kind: the projection
        weights, the KV cache both views read, the LM head (both views)."""
        L, d, D = self.L, self.d, self.D
        w = 2 * L * (self.wqkv.shape[2] * d + d * self.Hq * D) * 2
        kv = 2 * L * 2 * self.ctx * self.Hkv * D * 2
        lm = 2 * self.V * d * 2
        return {"projection_weights": w, "kv_cache": kv, "lm_head": lm}

    def kernels_per_round(self) -> int:
        # per view: block tokens, embed, RoPE table, per layer (norm, QKV with
        # RoPE, attention (1 launch at the one-wave batch-1 shape), out),
        # final norm, LM head; then consensus and commit
        return 2 * (3 + 4 * self.L + 2) + 2
