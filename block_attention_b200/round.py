"""One Orthrus decoding round over an L-layer model, on one GPU.

The round's launch sequence (Orthrus explainer on arXiv:2605.12825, §四):

  A  diffusion view: per layer, block attention with the bidirectional block
     mask over the layer's KV cache (anchor + 31 [MASK] rows)
  B  argmax of the diffusion logits -> drafts d[b, 0..blk)
  C  AR verify view: per layer, causal block attention over the same cache
  D  argmax of the verify logits -> a[b, 0..blk); consensus; commit of the
     accepted rows' K/V into every layer's cache (ctx_lens advance on device)

Only those kernels are on the path; the projections, FFN and LM head that sit
between them in a full model are out of scope, so each layer's Q and block K/V
and each view's logits are synthetic per-round inputs (``synth``), with the
logits' row maxima planted so the accepted prefix follows the configured
distribution.  Every call goes through the C ABI binding, on the current
stream, and the four segments can be captured as CUDA graphs.
"""
from __future__ import annotations

import numpy as np
import torch

from . import ATTN_EARLY_KV, BIDIR_BLOCK, CAUSAL_VERIFY
from . import attn_args, block_attn, consensus, kv_commit, lib, vocab_argmax, Workspace
from . import synth

_TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def _dev(a: np.ndarray, device) -> torch.Tensor:
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(a).to(device)


class DecodeRound:
    def __init__(self, *, layers, B, Hq, Hkv, D, blk, vocab, ctx_lens, cap=None,
                 dtype="bf16", logits_dtype="f32", accept_mean=5.4, seed=0,
                 device="cuda", prefetch=True):
        self.dev = torch.device(device)
        self.L, self.B, self.Hq, self.Hkv, self.D, self.blk, self.V = (
            layers, B, Hq, Hkv, D, blk, vocab)
        self.dtype, self.logits_dtype = dtype, logits_dtype
        lens = np.asarray(ctx_lens, np.int32)
        self.max_ctx = int(lens.max())
        self.cap = int(cap or self.max_ctx + blk)
        dt = _TORCH_DT[dtype]
        dev = self.dev
        self.k_cache = torch.empty(layers, B, Hkv, self.cap, D, dtype=dt, device=dev)
        self.v_cache = torch.empty_like(self.k_cache)
        # per-round inputs: view 0 = diffusion, view 1 = AR verify
        self.q = torch.empty(2, layers, B, blk, Hq, D, dtype=dt, device=dev)
        self.k_blk = torch.empty(2, layers, B, blk, Hkv, D, dtype=dt, device=dev)
        self.v_blk = torch.empty_like(self.k_blk)
        self.out = torch.empty_like(self.q)
        self.host = {}
        for l in range(layers):
            for v in (0, 1):
                inp = synth.attn_inputs(B, Hq, Hkv, D, blk, lens, self.cap, dtype, seed=seed,
                                        layer=2 * l + v, with_cache=v == 0)
                self.q[v, l].copy_(_dev(inp["q"], dev))
                self.k_blk[v, l].copy_(_dev(inp["k_blk"], dev))
                self.v_blk[v, l].copy_(_dev(inp["v_blk"], dev))
                if v == 0:  # one cache per layer, shared by both views
                    self.k_cache[l].copy_(_dev(inp["k_cache"], dev))
                    self.v_cache[l].copy_(_dev(inp["v_cache"], dev))
        g = synth.rng(seed, synth.S_ACC)
        self.accept = synth.geometric_accept(g, B, mean=accept_mean, blk=blk)
        d_tok, a_tok = synth.planted_tokens(g, B, blk, vocab, self.accept)
        self.draft_planted, self.verify_planted = d_tok, a_tok
        self.logits = torch.empty(2, B * blk, vocab, dtype=_TORCH_DT[logits_dtype], device=dev)
        self.logits[0].copy_(_dev(synth.planted_logits(g, d_tok, vocab, dtype=logits_dtype), dev))
        self.logits[1].copy_(_dev(synth.planted_logits(g, a_tok, vocab, dtype=logits_dtype), dev))
        self.ctx_base = torch.from_numpy(lens).to(dev)
        self.ctx_lens = self.ctx_base.clone()
        i32 = dict(dtype=torch.int32, device=dev)
        self.tok = torch.empty(2, B * blk, **i32)  # draft, verify argmax
        self.accept_len = torch.empty(B, **i32)
        self.n_emit = torch.empty(B, **i32)
        self.emitted = torch.empty(B, blk, **i32)
        self.next_anchor = torch.empty(B, **i32)
        self.err = torch.zeros(1, **i32)
        self.ws = {k: Workspace(dev) for k in ("attn0", "attn1", "argmax", "commit")}
        self.graphs = None
        self.prefetch = prefetch

    # ------------------------------------------------------------ segments
    def _attn(self, view):
        # ATTN_EARLY_KV promises that the work right before the call writes
        # neither a cache nor the lengths.  It holds for every layer after the
        # first (the previous layer's attention) and for the verify view's
        # first layer (the diffusion argmax).  The diffusion view's first
        # layer follows the copy that resets ctx_lens, so it waits for it.
        # With `prefetch`, each call warms L2 with the cache the next
        # attention call reads: the next layer's, and after the last layer
        # the first layer's (the other view's pass, or the next round's).
        mode = BIDIR_BLOCK if view == 0 else CAUSAL_VERIFY
        for l in range(self.L):
            early = not (view == 0 and l == 0)
            nxt = (l + 1) % self.L
            block_attn(self.q[view, l], self.k_blk[view, l], self.v_blk[view, l],
                       self.k_cache[l], self.v_cache[l], self.ctx_lens, mode,
                       out=self.out[view, l], max_ctx=self.max_ctx, err=self.err,
                       workspace=self.ws[f"attn{view}"], flags=ATTN_EARLY_KV if early else 0,
                       next_kv=(self.k_cache[nxt], self.v_cache[nxt]) if self.prefetch else None)

    def seg_a(self):
        self.ctx_lens.copy_(self.ctx_base)  # same round every step
        self._attn(0)

    def seg_b(self):
        vocab_argmax(self.logits[0], idx=self.tok[0], workspace=self.ws["argmax"])

    def seg_c(self):
        self._attn(1)

    def seg_d(self):
        vocab_argmax(self.logits[1], idx=self.tok[1], workspace=self.ws["argmax"])
        blk = self.blk
        consensus(self.tok[0].view(self.B, blk), self.tok[1].view(self.B, blk),
                  accept_len=self.accept_len, n_emit=self.n_emit, emitted=self.emitted,
                  next_anchor=self.next_anchor)
        kv_commit(self.k_cache, self.v_cache, self.k_blk[1], self.v_blk[1], self.ctx_lens,
                  self.n_emit, err=self.err, workspace=self.ws["commit"])

    SEGMENTS = ("seg_a", "seg_b", "seg_c", "seg_d")

    def step_eager(self):
        for s in self.SEGMENTS:
            getattr(self, s)()

    def capture(self):
        """Record each segment as a CUDA graph (after one eager warm-up step,
        so every workspace is allocated before capture)."""
        side = torch.cuda.Stream(device=self.dev)
        side.wait_stream(torch.cuda.current_stream(self.dev))
        with torch.cuda.stream(side):
            self.step_eager()
        torch.cuda.current_stream(self.dev).wait_stream(side)
        torch.cuda.synchronize(self.dev)
        self.graphs = []
        for s in self.SEGMENTS:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                getattr(self, s)()
            self.graphs.append(g)
        torch.cuda.synchronize(self.dev)

    def replay(self, events=None):
        """One round from the captured graphs; events[i] recorded before segment i
        and events[4] after the last (on the current stream)."""
        for i, g in enumerate(self.graphs):
            if events is not None:
                events[i].record()
            g.replay()
        if events is not None:
            events[4].record()

    # ------------------------------------------------------------ accounting
    def kernels_per_round(self) -> int:
        per = []
        for view in (0, 1):
            a = attn_args(self.q[view, 0], self.k_blk[view, 0], self.v_blk[view, 0],
                          self.k_cache[0], self.v_cache[0], self.ctx_lens, view,
                          self.out[view, 0], None, self.max_ctx)
            per.append(lib().orthrus_block_attn_launches(a))
        return self.L * sum(per) + 2 + 1 + 1  # argmax x2, consensus, commit

    def attn_bytes_per_launch(self, lens=None) -> int:
        """Algorithmic HBM bytes of one block_attn launch: the visible K/V cache
        rows once, plus Q, the block K/V and the output."""
        lens = np.asarray(lens if lens is not None else self.ctx_base.cpu().numpy())
        es = 2 if self.dtype == "bf16" else 4
        kv = 2 * int(lens.sum()) * self.Hkv * self.D * es
        qo = 2 * self.B * self.blk * self.Hq * self.D * es
        blkkv = 2 * self.B * self.blk * self.Hkv * self.D * es
        return kv + qo + blkkv

    def round_bytes(self) -> dict:
        es_l = 4 if self.logits_dtype == "f32" else 2
        es = 2 if self.dtype == "bf16" else 4
        n_emit = np.minimum(self.accept + 1, self.blk)
        commit = 2 * 2 * int(n_emit.sum()) * self.Hkv * self.D * es * self.L  # K,V read+write
        return {"attn": 2 * self.L * self.attn_bytes_per_launch(),
                "argmax": 2 * self.B * self.blk * self.V * es_l,
                "commit": commit}

    # ------------------------------------------------------------ host I/O
    INPUTS = ("q", "k_blk", "v_blk", "logits")

    def pinned_inputs(self):
        """Pinned host copies of one round's inputs (for the end-to-end path)."""
        return {k: getattr(self, k).cpu().pin_memory() for k in self.INPUTS}

    def h2d(self, host, into=None):
        """Copy a round's inputs from (pinned) host memory into the current
        input set, or into input set `into` (see add_input_set)."""
        bufs = self.input_sets[into][0] if into is not None else {
            k: getattr(self, k) for k in self.INPUTS}
        for k, t in host.items():
            bufs[k].copy_(t, non_blocking=True)
        return sum(t.numel() * t.element_size() for t in host.values())

    def add_input_set(self):
        """A second set of per-round input buffers with graphs of its own
        (after capture()), so that one set's inputs can be copied in while
        the round on the other set runs.  Caches, lengths, outputs and
        workspaces stay shared: rounds still run one after another."""
        first = ({k: getattr(self, k) for k in self.INPUTS}, self.graphs)
        for k in self.INPUTS:
            setattr(self, k, first[0][k].clone())
        self.capture()
        self.input_sets = [first, ({k: getattr(self, k) for k in self.INPUTS}, self.graphs)]
        self.use_set(0)

    def use_set(self, s):
        bufs, graphs = self.input_sets[s]
        for k, t in bufs.items():
            setattr(self, k, t)
        self.graphs = graphs

    def pinned_outputs(self):
        return {k: torch.empty(getattr(self, k).shape, dtype=torch.int32).pin_memory()
                for k in ("accept_len", "n_emit", "emitted", "next_anchor")}

    def d2h(self, host):
        for k, t in host.items():
            t.copy_(getattr(self, k), non_blocking=True)
        return sum(t.numel() * t.element_size() for t in host.values())
