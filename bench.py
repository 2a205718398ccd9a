"""Benchmark of one Orthrus decoding round on B200 (Qwen3-8B attention shape).

A step = one full round (both attention views over 36 layers, argmax of both
views' logits, consensus, KV commit of the accepted rows), replayed from CUDA
graphs with every input resident in HBM.  Prints ONE JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N > 1) every rank runs its own replica of the round on its own
GPU (independent sequences; no data-path collective): weak scaling, value =
rounds completed by all ranks / max-over-ranks device time.

--impl reference times the CPU oracle (the only reference that exists for this
method: its pages carry no code) on this host's cores, on a bounded sample of
the same workload, rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "block-attn HBM GB/s (% of peak) and consensus rounds/s, Qwen3-8B shape"
WORKLOAD = dict(name="qwen3_8b_round", layers=36, B=1, Hq=32, Hkv=8, D=128, ctx=8192,
                blk=32, vocab=151936, dtype="bf16", logits_dtype="f32", accept_mean=5.4)
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20  # written between cold timings: twice the 126 MB L2
# DRAM bytes (read + write) of one block-attention call at this workload, from
# an ncu capture of the benchmarked call.  Valid only for the kernel source it
# was measured on: reported as null once attn_tc.cu changes.
TRAFFIC = {"attn_tc_sha256_prefix": "3acaf7a96dbdf4df", "bytes_per_call": 34023168}


def measured_traffic():
    import hashlib
    src = os.path.join(ROOT, "block_attention_b200", "csrc", "attn_tc.cu")
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    return TRAFFIC["bytes_per_call"] if h == TRAFFIC["attn_tc_sha256_prefix"] else None


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], "measured"
    return FALLBACK_HBM_GBS, "fallback"


def config_dict():
    w = WORKLOAD
    return {"workload": w["name"], "layers": w["layers"], "B": w["B"], "Hq": w["Hq"],
            "Hkv": w["Hkv"], "D": w["D"], "ctx": w["ctx"], "blk": w["blk"],
            "vocab": w["vocab"], "kv_dtype": w["dtype"], "logits_dtype": w["logits_dtype"],
            "accept_len": f"Geometric(mean {w['accept_mean']}) planted",
            "l2": "inputs larger than L2: 1.21 GB KV cache, 2.46 GB of K/V streamed per round"}


# ---------------------------------------------------------------- ranks

def max_over_ranks(values, device):
    """Element-wise maximum of per-rank device times (ms) over every rank of
    the initialised process group (identity without one): a multi-GPU number
    is the slowest rank's."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def bind_host_to_gpu(dev_index):
    """Run this process on the CPUs nearest the GPU (NVML's affinity for the
    GPU's PCI address), so that pinned host buffers allocated afterwards sit
    on the GPU's NUMA node and host-device copies do not cross the socket
    interconnect.  A setting of this process only (nothing of the GPU is
    changed).  Returns (previous CPU set, description), or (None, None)
    where the affinity cannot be read."""
    try:
        import pynvml
        import torch
        prop = torch.cuda.get_device_properties(dev_index)
        bus = f"{prop.pci_domain_id:08x}:{prop.pci_bus_id:02x}:{prop.pci_device_id:02x}.0"
        pynvml.nvmlInit()
        try:
            handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            words = pynvml.nvmlDeviceGetCpuAffinity(handle, ((os.cpu_count() or 64) + 63) // 64)
        finally:
            pynvml.nvmlShutdown()
        before = os.sched_getaffinity(0)
        near = {64 * i + b for i, w in enumerate(words) for b in range(64) if (w >> b) & 1}
        near &= before
        if not near or near == before:
            return None, None
        os.sched_setaffinity(0, near)
        return before, f"{len(near)} of {len(before)} cpus, the GPU's NUMA node"
    except Exception:
        return None, None


def whole_job_rate(world, steps, ms):
    """Units per second completed by all ranks together: every rank runs
    `steps` units of its own (weak scaling), in at most `ms` milliseconds."""
    return world * steps / (ms * 1e-3)


# ---------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid, self.proc, self.path = uuid, None, None

    def start(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(prefix="orthrus_clocks_", suffix=".csv")
        os.close(fd)
        try:
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                   "-lms", "100"]
            if self.uuid:
                cmd[1:1] = ["-i", self.uuid]
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"),
                                         stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 10:
                    rows.append(parts)
        try:
            os.unlink(self.path)
        except OSError:
            pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        smax = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[6 + i] == "Active"})
        load = [s for s in sm if s > 0.5 * max(smax or [1])] or sm
        return {"sm_mhz": statistics.median(load) if load else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
                "samples": len(rows)}


# ---------------------------------------------------------------- CPU oracle leg

def oracle_round_sample(heads=1, layers_timed=1):
    """Time the oracle on a bounded sample of one round and extrapolate to the
    whole round: `layers_timed` layer(s) per view restricted to `heads` kv-head
    group(s) (x 36 layers x 8/heads groups), plus the full argmax of both
    views' 32 x 151936 logits, consensus and one layer's commit (x 36)."""
    import oracle
    from block_attention_b200 import synth
    w = WORKLOAD
    G = w["Hq"] // w["Hkv"]
    cap = w["ctx"] + w["blk"]
    nthreads = os.cpu_count() or 1
    t_attn = 0.0
    for v in (0, 1):
        for l in range(layers_timed):
            inp = synth.attn_inputs(1, G * heads, heads, w["D"], w["blk"], [w["ctx"]], cap,
                                    w["dtype"], seed=7, layer=2 * l + v)
            t0 = time.perf_counter()
            oracle.block_attn(inp["q"], inp["k_blk"], inp["v_blk"], inp["k_cache"],
                              inp["v_cache"], inp["ctx_lens"], v, nthreads=nthreads)
            t_attn += time.perf_counter() - t0
    t_attn *= (w["layers"] / layers_timed) * (w["Hkv"] / heads)
    g = synth.rng(8)
    acc = synth.geometric_accept(g, 1)
    d, a = synth.planted_tokens(g, 1, w["blk"], w["vocab"], acc)
    ld = synth.planted_logits(g, d, w["vocab"])
    la = synth.planted_logits(g, a, w["vocab"])
    t0 = time.perf_counter()
    di, ai = oracle.vocab_argmax(ld), oracle.vocab_argmax(la)
    L, ne, em, na = oracle.consensus(di[None], ai[None])
    t_mid = time.perf_counter()
    kc = np.zeros((1, w["Hkv"], cap, w["D"]), np.uint16)
    vc = np.zeros_like(kc)
    kb = np.zeros((1, w["blk"], w["Hkv"], w["D"]), np.uint16)
    oracle.kv_commit(kc, vc, kb, kb.copy(), [w["ctx"]], ne)
    t_end = time.perf_counter()
    t_round = t_attn + (t_mid - t0) + w["layers"] * (t_end - t_mid)
    sample = (f"{layers_timed} layer(s) per view x {heads} of {w['Hkv']} kv-head groups timed, "
              f"extrapolated x{w['layers'] // layers_timed * w['Hkv'] // heads}; "
              "full argmax (2 x 32 x 151936), consensus, 1-layer commit x36")
    return 1.0 / t_round, nthreads, sample


def reference_arm(args, rank, world):
    if rank != 0:
        return
    for _ in range(args.warmup):
        oracle_round_sample()
    vals, t0 = [], time.perf_counter()
    for _ in range(args.steps):
        v, cores, sample = oracle_round_sample()
        vals.append(v)
    wall = time.perf_counter() - t0
    value = float(np.mean(vals))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "rounds/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 / value, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(),
            "cpu_baseline": {"value": value, "unit": "rounds/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "rounds/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "wall_s": wall}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- one kernel alone

def kernel_alone(args):
    """Block attention alone at the Qwen3-8B layer shape, bidirectional view:
    B sequences of context 8192 (--attn-batch; 8 by default: 269 MB of K/V,
    over twice the L2; 1: the call the round makes, whose 34 MB stay in L2
    across launches, so only a cold-cache profile reads them from HBM).
    W warm-up launches, then K launches captured in one CUDA graph."""
    import torch
    import block_attention_b200 as ba
    from block_attention_b200.round import _dev
    from block_attention_b200 import synth
    w = WORKLOAD
    B, ctx = args.attn_batch, w["ctx"]
    cap = ctx + w["blk"]
    dev = torch.device("cuda", 0)
    inp = synth.attn_inputs(B, w["Hq"], w["Hkv"], w["D"], w["blk"], [ctx] * B, cap, "bf16",
                            seed=11)
    t = {k: _dev(v, dev) for k, v in inp.items()}
    out = torch.empty_like(t["q"])
    call = lambda: ba.block_attn(t["q"], t["k_blk"], t["v_blk"], t["k_cache"], t["v_cache"],
                                 t["ctx_lens"], ba.BIDIR_BLOCK, out=out, max_ctx=ctx)
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(args.steps):
            call()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g.replay()
    torch.cuda.synchronize()
    e0.record()
    g.replay()
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / args.steps
    nbytes = 2 * B * ctx * w["Hkv"] * w["D"] * 2 + 2 * B * w["blk"] * w["Hq"] * w["D"] * 2 \
        + 2 * B * w["blk"] * w["Hkv"] * w["D"] * 2
    hbm, src = peaks()
    print(json.dumps({"kernel": "block_attn", "case": f"B={B} ctx={ctx} Hq=32 Hkv=8 D=128 blk=32 bf16 bidir",
                      "us_per_launch": us, "bytes_per_launch": nbytes,
                      "gbs": nbytes / us / 1e3, "frac": nbytes / us / 1e3 / hbm,
                      "peak": hbm, "peak_source": src}), flush=True)


def sampling_kernels(args):
    """The stochastic round's kernels one at a time at the Qwen3-8B shape (32
    rows x vocab 151936, fp32 logits, T = 1): draft sampling with and without
    the fused log-sum-exp, the stand-alone log-probability pass, and the
    consensus (log p + acceptance, then the correction).  Each is captured
    `steps` times in its own CUDA graph; the logits stay L2-resident."""
    import torch
    import block_attention_b200 as ba
    dev = torch.device("cuda", 0)
    w = WORKLOAD
    rows, V, B, blk = w["B"] * w["blk"], w["vocab"], w["B"], w["blk"]
    g = torch.Generator(device=dev).manual_seed(1005)
    zq = torch.randn(rows, V, generator=g, device=dev) * 3
    zp = zq + torch.randn(rows, V, generator=g, device=dev) * 0.5
    f32 = dict(dtype=torch.float32, device=dev)
    lq, lp, sq, sp = (torch.empty(rows, **f32) for _ in range(4))
    d = torch.empty(rows, dtype=torch.int32, device=dev)
    outs = [torch.empty(B, dtype=torch.int32, device=dev) for _ in range(3)]
    em = torch.empty(B, blk, dtype=torch.int32, device=dev)
    ops = {
        "vocab_sample": lambda k: ba.vocab_sample(zq, 1.0, 7, k, idx=d),
        "vocab_sample_with_lse": lambda k: ba.vocab_sample(zq, 1.0, 7, k, idx=d, logprob=lq,
                                                           lse=sq),
        "token_logprob": lambda k: ba.token_logprob(zq, d, temperature=1.0, out=lq, lse=sq),
        "consensus_sample": lambda k: ba.consensus_sample(
            d.view(B, blk), zp, zq, lq, sq, 1.0, 7, k, logp=lp, lse_ar=sp, accept_len=outs[0],
            n_emit=outs[1], emitted=em, next_anchor=outs[2]),
    }
    res = {}
    for name, f in ops.items():
        for k in range(args.warmup):
            f(k)
        torch.cuda.synchronize()
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            for k in range(args.steps):
                f(k)
        gr.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        gr.replay()
        e1.record()
        torch.cuda.synchronize()
        res[name] = e0.elapsed_time(e1) * 1e3 / args.steps
        del gr
    print(json.dumps({"kernel": "stochastic round kernels",
                      "case": f"{rows} rows x vocab {V}, fp32 logits, T = 1, L2-resident",
                      "us_per_launch": res}), flush=True)


def lm_head_leg(dev, steps=10, warmup=3):
    """The Qwen3-8B LM head with the argmax fused in its epilogue (d 4096,
    vocabulary 151936, bf16) for 32 and 128 hidden rows (one and four
    32-row blocks), against the unfused pair a round would otherwise run: a
    cuBLAS bf16 GEMM writing the logits, then this library's vocab_argmax.
    The 1.24 GB output embedding is larger than L2, so every launch streams
    it from HBM.  Algorithmic bytes: the embedding once plus h."""
    import torch
    import block_attention_b200 as ba
    d, V = 4096, WORKLOAD["vocab"]
    g = torch.Generator(device=dev).manual_seed(1006)
    w = (torch.randn(V, d, generator=g, device=dev) * 0.02).to(torch.bfloat16)
    hbm, src = peaks()
    out = {}
    for rows in (32, 128):
        h = torch.randn(rows, d, generator=g, device=dev).to(torch.bfloat16)
        idx = torch.empty(rows, dtype=torch.int32, device=dev)
        fused = lambda: ba.lm_head_argmax(h, w, idx=idx)
        logits = torch.empty(rows, V, dtype=torch.bfloat16, device=dev)
        unfused = lambda: (torch.matmul(h, w.t(), out=logits), ba.vocab_argmax(logits, idx=idx))
        res = {}
        for name, f in (("fused", fused), ("cublas_gemm_then_argmax", unfused)):
            for _ in range(warmup):
                f()
            torch.cuda.synchronize()
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr):
                for _ in range(steps):
                    f()
            gr.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            gr.replay()
            e1.record()
            torch.cuda.synchronize()
            res[name] = e0.elapsed_time(e1) * 1e3 / steps
            del gr
        nbytes = V * d * 2 + rows * d * 2
        out[f"rows_{rows}"] = {"us_fused": res["fused"],
                               "us_unfused": res["cublas_gemm_then_argmax"],
                               "bytes": nbytes, "gbs_fused": nbytes / res["fused"] / 1e3,
                               "frac_fused": nbytes / res["fused"] / 1e3 / hbm}
    del w
    return {"kernel": "lm_head_argmax", "case": f"d {d}, vocab {V}, bf16",
            "peak": hbm, "peak_source": src, **out}


def projection_kernels(args):
    """The attention block's projections alone at the Qwen3-8B shape: a
    32-row block through the QKV (4096 -> 6144) and output (4096 -> 4096)
    weights of 36 layers in turn (beyond the L2), `steps` graph replays."""
    import torch
    import block_attention_b200 as ba
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(1010)
    L, blk, d = WORKLOAD["layers"], WORKLOAD["blk"], 4096
    hbm, src = peaks()
    res = {}
    for name, N in (("qkv_projection", 6144), ("output_projection", 4096)):
        W = (torch.randn(L, N, d, generator=g, device=dev) * 0.02).to(torch.bfloat16)
        x = torch.randn(blk, d, generator=g, device=dev).to(torch.bfloat16)
        y = torch.empty(blk, N, dtype=torch.bfloat16, device=dev)
        ws = ba.Workspace(dev)
        seq = lambda: [ba.linear_tc(x, W[l], out=y, workspace=ws) for l in range(L)]
        for _ in range(args.warmup):
            seq()
        torch.cuda.synchronize()
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            seq()
        gr.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            gr.replay()
        e1.record()
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / (args.steps * L)
        nbytes = N * d * 2 + blk * (d + N) * 2
        res[name] = {"us_per_call": us, "gbs": nbytes / us / 1e3, "frac": nbytes / us / 1e3 / hbm}
        del gr, W
    print(json.dumps({"kernel": "linear_tc", "case": f"{blk} rows, Qwen3-8B projections, "
                      f"{L} layers' weights in turn", "peak": hbm, "peak_source": src, **res}),
          flush=True)


def lm_head_kernel(args):
    import torch
    print(json.dumps(lm_head_leg(torch.device("cuda", 0), args.steps, args.warmup)), flush=True)


def block_size_sweep(args):
    """Block attention at the Qwen3-8B layer shape (B=1, ctx 8192) for block
    sizes K in {4, 8, 16, 32}, both views, 72 calls per CUDA graph chained as in
    a round: the explainer's ablation (section 六) finds per-round latency
    roughly constant in K; this checks it at the kernel level."""
    import torch
    import block_attention_b200 as ba
    w = WORKLOAD
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(1002)
    rnd = lambda *shape: torch.randn(*shape, generator=g, device=dev).to(torch.bfloat16)
    ctx, Hq, Hkv, D, layers = w["ctx"], w["Hq"], w["Hkv"], w["D"], w["layers"]
    cap = ctx + 32
    kc, vc = rnd(layers, 1, Hkv, cap, D), rnd(layers, 1, Hkv, cap, D)
    lens = torch.full((1,), ctx, dtype=torch.int32, device=dev)
    res = {}
    for K in (4, 8, 16, 32):
        q, kb, vb = rnd(2, layers, 1, K, Hq, D), rnd(2, layers, 1, K, Hkv, D), rnd(2, layers, 1, K, Hkv, D)
        out = torch.empty_like(q)
        ws = ba.Workspace(dev)

        def seq():
            for view in (0, 1):
                for l in range(layers):
                    ba.block_attn(q[view, l], kb[view, l], vb[view, l], kc[l], vc[l], lens, view,
                                  out=out[view, l], max_ctx=ctx, workspace=ws, flags=ba.ATTN_EARLY_KV)
        seq()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            seq()
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(max(args.steps, 1)):
            graph.replay()
        e1.record()
        torch.cuda.synchronize()
        res[K] = e0.elapsed_time(e1) * 1e3 / (max(args.steps, 1) * 2 * layers)
        del graph
    print(json.dumps({"kernel": "block_attn", "sweep": "block size K",
                      "case": f"B=1 ctx={ctx} Hq={Hq} Hkv={Hkv} D={D} bf16, both views, "
                              f"{2 * layers} chained calls per graph",
                      "us_per_call": res}), flush=True)


# ---------------------------------------------------------------- GPU arm

def batched_ragged_leg(dev, hbm, launches=10):
    """Block attention of the batched ragged Qwen3-8B configuration: 16
    sequences with contexts ~ U{1k..32k}, Hq 32, Hkv 8, head dim 128, block 32,
    bf16, both views alternating.  Seeded random bf16 tensors are generated on
    the device (values do not change the work; parity for this shape is in the
    tests).  The K/V caches hold about 2.2 GB, far beyond the L2.  Runs after the
    timed round; it reports its own time and roofline fraction."""
    import torch
    import block_attention_b200 as ba
    from block_attention_b200 import synth
    B, Hq, Hkv, D, blk = 16, 32, 8, 128, 32
    lens = synth.ragged_lens(B, 1024, 32768, seed=1004)
    cap = int(lens.max()) + blk
    g = torch.Generator(device=dev).manual_seed(1004)
    rnd = lambda *shape: torch.randn(*shape, generator=g, device=dev).to(torch.bfloat16)
    q, kb, vb = rnd(B, blk, Hq, D), rnd(B, blk, Hkv, D), rnd(B, blk, Hkv, D)
    kc, vc = rnd(B, Hkv, cap, D), rnd(B, Hkv, cap, D)
    ctx = torch.from_numpy(lens.astype(np.int32)).to(dev)
    out = torch.empty_like(q)
    ws = ba.Workspace(dev)

    def call(k):
        ba.block_attn(q, kb, vb, kc, vc, ctx, k % 2, out=out, max_ctx=cap - blk, workspace=ws,
                      flags=ba.ATTN_EARLY_KV)
    for k in range(4):
        call(k)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for k in range(launches):
            call(k)
    graph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    graph.replay()
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / launches
    nbytes = 2 * int(lens.sum()) * Hkv * D * 2 + 2 * B * blk * Hq * D * 2 + 2 * B * blk * Hkv * D * 2
    gbs = nbytes / (us * 1e-6) / 1e9
    del graph
    return {"workload": "batched ragged Qwen3-8B layer: 16 sequences, ctx ~ U{1024..32768} "
                        f"(sum {int(lens.sum())}), Hq 32, Hkv 8, D 128, block 32, bf16, both views",
            "us_per_launch": us, "bytes_per_launch": nbytes, "gbs": gbs, "peak": hbm,
            "frac": gbs / hbm, "launches": launches, "l2": "inputs larger than L2"}


def attn_flops(Hq, blk, lens, D, mode):
    """Multiply-adds x 2 of one block-attention call: Q K^T and P V over the
    visible keys of every query row (bidir: n + blk keys per row; causal:
    n + i + 1 for block row i)."""
    keys = 0
    for n in lens:
        keys += blk * (n + blk) if mode == 0 else blk * n + blk * (blk + 1) // 2
    return 4 * Hq * keys * D


def ffma_peak_tflops(sm_mhz):
    """FP32 fused multiply-add peak: 148 SMs x 4 sub-partitions x 32 FP32
    lanes, 2 FLOP per FMA, at the given SM clock."""
    return 148 * 128 * 2 * sm_mhz * 1e6 / 1e12


def small_config_legs(dev, hbm, sm_max_mhz=1965.0, reps=4):
    """Block attention of the two smaller configurations, both views chained
    layer after layer as in a round:
      tiny: B 1, Hq 4, Hkv 2, D 64, ctx 256, block 32, FP32, one layer (its
            0.3 MB of K/V stay in L2; the number is launch-bound);
      qwen3_1p7b: B 1, Hq 16, Hkv 8, D 128, ctx 2048, block 32, 28 layers
            (Qwen3-1.7B depth) so the caches (238 MB bf16, 477 MB FP32)
            exceed the L2; bf16 (tensor cores) and FP32 (CUDA cores).
    FP32 runs are reported as a fraction of the FP32 FMA peak, bf16 runs as a
    fraction of the measured HBM bandwidth."""
    import torch
    import block_attention_b200 as ba
    out = {}
    cases = (("tiny_f32", 1, 4, 2, 64, 256, 32, 1, torch.float32),
             ("qwen3_1p7b_bf16", 1, 16, 8, 128, 2048, 32, 28, torch.bfloat16),
             ("qwen3_1p7b_f32", 1, 16, 8, 128, 2048, 32, 28, torch.float32))
    for name, B, Hq, Hkv, D, ctx, blk, layers, dt in cases:
        g = torch.Generator(device=dev).manual_seed(1001)
        rnd = lambda *shape: torch.randn(*shape, generator=g, device=dev).to(dt)
        cap = ctx + blk
        kc, vc = rnd(layers, B, Hkv, cap, D), rnd(layers, B, Hkv, cap, D)
        q = rnd(2, layers, B, blk, Hq, D)
        kb, vb = rnd(2, layers, B, blk, Hkv, D), rnd(2, layers, B, blk, Hkv, D)
        o = torch.empty_like(q)
        lens = torch.full((B,), ctx, dtype=torch.int32, device=dev)
        ws = ba.Workspace(dev)

        def seq():
            for view in (0, 1):
                for l in range(layers):
                    ba.block_attn(q[view, l], kb[view, l], vb[view, l], kc[l], vc[l], lens, view,
                                  out=o[view, l], max_ctx=ctx, workspace=ws,
                                  flags=ba.ATTN_EARLY_KV)
        seq()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            seq()
        graph.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            graph.replay()
        e1.record()
        torch.cuda.synchronize()
        calls = reps * 2 * layers
        us = e0.elapsed_time(e1) * 1e3 / calls
        es = 4 if dt == torch.float32 else 2
        nbytes = 2 * B * ctx * Hkv * D * es + 2 * B * blk * Hq * D * es + 2 * B * blk * Hkv * D * es
        flops = (attn_flops(Hq, blk, [ctx] * B, D, 0) + attn_flops(Hq, blk, [ctx] * B, D, 1)) / 2
        rec = {"us_per_call": us, "bytes_per_call": nbytes, "gbs": nbytes / us / 1e3,
               "tflops": flops / us / 1e6, "calls_timed": calls,
               "l2": "L2-resident" if layers == 1 else "inputs larger than L2"}
        if dt == torch.float32:
            peak = ffma_peak_tflops(sm_max_mhz)
            rec.update(bound="fp32 FMA", peak_tflops=peak, frac=rec["tflops"] / peak,
                       peak_note=f"148 SMs x 128 FP32 lanes x 2 FLOP x {sm_max_mhz:.0f} MHz")
        else:
            rec.update(bound="hbm", peak_gbs=hbm, frac=rec["gbs"] / hbm)
        out[name] = rec
        del graph
    return out


def argmax_leg(dev, hbm, buffers=8, reps=5):
    """The vocabulary argmax of one view at the Qwen3-8B shape (32 rows x
    151936 fp32 logits = 19.45 MB), alone: `buffers` distinct logit matrices
    (156 MB together, beyond the L2) read in turn, buffers x reps launches in
    one CUDA graph.  Algorithmic bytes: the logits once."""
    import torch
    import block_attention_b200 as ba
    rows, V = WORKLOAD["B"] * WORKLOAD["blk"], WORKLOAD["vocab"]
    g = torch.Generator(device=dev).manual_seed(1007)
    logits = [torch.randn(rows, V, generator=g, device=dev) * 3 for _ in range(buffers)]
    idx = torch.empty(rows, dtype=torch.int32, device=dev)
    ws = ba.Workspace(dev)
    calls = lambda: [ba.vocab_argmax(x, idx=idx, workspace=ws) for x in logits]
    for _ in range(3):
        calls()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(reps):
            calls()
    graph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    graph.replay()
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / (buffers * reps)
    nbytes = rows * V * 4
    del graph
    return {"workload": f"{rows} rows x vocab {V}, fp32 logits, {buffers} buffers in turn "
                        "(inputs larger than L2)",
            "us_per_launch": us, "bytes_per_launch": nbytes, "gbs": nbytes / us / 1e3,
            "peak": hbm, "frac": nbytes / us / 1e3 / hbm}


def projected_round_leg(dev, hbm, steps=10, warmup=3):
    """A round with the attention block's projections and the LM head on the
    path (block_attention_b200.projected): Qwen3-8B shape, 36 layers, both
    views each computing Q and the block K/V from the hidden states (RMSNorm,
    QKV projection, RoPE), attending, projecting back with the residual,
    then the LM head with the argmax fused; consensus and commit.  Reported:
    rounds/s of the captured round, its algorithmic bytes, and the projection
    kernels alone (36 layers' weights in turn, beyond the L2) against the
    measured HBM bandwidth."""
    import torch
    import block_attention_b200 as ba
    from block_attention_b200.projected import ProjectedRound
    rnd = ProjectedRound(layers=WORKLOAD["layers"], ctx=WORKLOAD["ctx"], seed=1009,
                         device=dev)
    rnd.capture()
    for _ in range(warmup):
        rnd.replay()
    torch.cuda.synchronize()
    ev = lambda: torch.cuda.Event(enable_timing=True)
    e0, e1 = ev(), ev()
    e0.record()
    for _ in range(steps):
        rnd.replay()
    e1.record()
    torch.cuda.synchronize()
    assert int(rnd.err.item()) == 0
    ms = e0.elapsed_time(e1) / steps
    rb = rnd.bytes_per_round()
    out = {"workload": "Qwen3-8B attention path: 36 layers x 2 views of RMSNorm, QKV "
                       "projection (4096 -> 6144), RoPE, block attention (ctx 8192), output "
                       "projection (4096 -> 4096) with residual; LM head (vocab 151936) with "
                       "the argmax fused; bf16 random weights",
           "rounds_per_s": 1e3 / ms, "ms_per_round": ms, "bytes_per_round": rb,
           "round_gbs": sum(rb.values()) / (ms * 1e-3) / 1e9,
           "kernels_per_round": rnd.kernels_per_round()}
    # the projections alone, each layer's weights in turn (graph of 36 calls)
    x = torch.randn(WORKLOAD["blk"], rnd.d, device=dev).to(torch.bfloat16)
    for name, W, N in (("qkv_projection", rnd.wqkv[1], rnd.wqkv.shape[2]),
                       ("output_projection", rnd.wo[1], rnd.d)):
        y = torch.empty(WORKLOAD["blk"], N, dtype=torch.bfloat16, device=dev)
        ws = ba.Workspace(dev)
        # (the output projection's input is [blk, Hq * D] = [blk, 4096], like x)
        seq = lambda: [ba.linear_tc(x, W[l], out=y, workspace=ws) for l in range(rnd.L)]
        seq()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            seq()
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = ev(), ev()
        e0.record()
        for _ in range(3):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / (3 * rnd.L)
        nbytes = N * rnd.d * 2 + WORKLOAD["blk"] * (rnd.d + N) * 2
        out[name] = {"us_per_call": us, "bytes_per_call": nbytes, "gbs": nbytes / us / 1e3,
                     "frac": nbytes / us / 1e3 / hbm,
                     "shape": f"{WORKLOAD['blk']} x {rnd.d} -> {N}"}
        del g
    del rnd
    torch.cuda.empty_cache()
    return out


def stochastic_round_leg(dev, hbm, iters=20):
    """The stochastic consensus step of one round at the Qwen3-8B shape (B = 1,
    block 32, vocab 151936, fp32 logits of both views): draft sampling with the
    drafts' log q and log-sum-exp from the same pass, then the consensus (log p
    over the AR logits with the acceptance test, and the correction), three
    launches in one CUDA graph.  Algorithmic bytes: one read of each logit
    matrix plus the two rows of the correction.  Timed twice: 20 rounds back
    to back (the logits stay L2-resident, as right after the LM head writes
    them), and rounds that each follow an L2 flush (HBM reads; the fraction
    of peak refers to these): a graph of `iters` x (flush, round) less a
    graph of `iters` flushes, so no host launch gap enters the figure."""
    import torch
    import block_attention_b200 as ba
    w = WORKLOAD
    rows, V, B, blk = w["B"] * w["blk"], w["vocab"], w["B"], w["blk"]
    g = torch.Generator(device=dev).manual_seed(1005)
    zq = torch.randn(rows, V, generator=g, device=dev) * 3
    zp = zq + torch.randn(rows, V, generator=g, device=dev) * 0.5
    f32 = dict(dtype=torch.float32, device=dev)
    lq, lp, sq, sp = (torch.empty(rows, **f32) for _ in range(4))
    d = torch.empty(rows, dtype=torch.int32, device=dev)
    outs = [torch.empty(B, dtype=torch.int32, device=dev) for _ in range(3)]
    em = torch.empty(B, blk, dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step(k):
        ba.vocab_sample(zq, 1.0, 7, k, idx=d, logprob=lq, lse=sq)
        ba.consensus_sample(d.view(B, blk), zp, zq, lq, sq, 1.0, 7, k, logp=lp, lse_ar=sp,
                            accept_len=outs[0], n_emit=outs[1], emitted=em,
                            next_anchor=outs[2])
    for k in range(3):
        step(k)
    torch.cuda.synchronize()
    graph, cold_g, flush_g = (torch.cuda.CUDAGraph() for _ in range(3))
    with torch.cuda.graph(graph):
        for k in range(iters):
            step(k)
    with torch.cuda.graph(cold_g):
        for k in range(iters):
            flush.fill_(k & 0xFF)
            step(k)
    with torch.cuda.graph(flush_g):
        for k in range(iters):
            flush.fill_(k & 0xFF)
    for g_ in (graph, cold_g, flush_g):
        g_.replay()
    torch.cuda.synchronize()
    ev = lambda: torch.cuda.Event(enable_timing=True)

    def timed(g_):
        e0, e1 = ev(), ev()
        e0.record()
        g_.replay()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) * 1e3

    hot = timed(graph) / iters
    cold = sorted((timed(cold_g) - timed(flush_g)) / iters for _ in range(3))[1]
    nbytes = 2 * rows * V * 4 + 2 * V * 4
    del graph, cold_g, flush_g
    return {"workload": f"stochastic consensus, B=1 block 32, vocab {V}, fp32 logits, T = 1",
            "kernels_per_round": 3, "bytes_per_round": nbytes,
            "us_per_round_l2_resident": hot, "us_per_round_cold": cold,
            "gbs_cold": nbytes / (cold * 1e-6) / 1e9, "peak": hbm,
            "frac_cold": nbytes / (cold * 1e-6) / 1e9 / hbm}


def decoder_report():
    """The end-to-end consensus loop on the random-init decoder (4 layers,
    d_model 512, Hq 8, Hkv 4, head dim 64, SwiGLU 1536, vocab 8192; 256
    prompts of U{64..512} random tokens, 256 greedy tokens each): FP32 loop
    against FP32 greedy (must be exact), BF16 trajectory-match rates, tokens
    per forward.  Runs after the timed regions; it times nothing of the bench."""
    import torch
    from block_attention_b200 import synth
    from block_attention_b200.decoder import TinyDecoder, perplexity_report, trajectory_report
    E = synth.WORKLOADS["e2e_decoder"]
    seed = 1004
    W = synth.decoder_weights(E["V"], E["d"], E["L"], E["Hq"], E["Hkv"], E["hd"], E["ffn"],
                              seed=seed, std=E["std"])
    prompts = synth.prompts(E["prompts"], E["V"], E["prompt_lo"], E["prompt_hi"], seed=seed,
                            exclude=E["V"] - 1)
    t0 = time.perf_counter()
    rep = {"workload": "random-init decoder L4 d512 Hq8 Hkv4 hd64 ffn1536 V8192; "
                       "256 prompts U{64..512}, 256 new tokens, block 32"}
    out = {}
    for name, dt in (("fp32", torch.float32), ("bf16", torch.bfloat16)):
        m = TinyDecoder(W, E["Hq"], E["Hkv"], E["hd"], dtype=dt)
        out[name + "_greedy"], out[name + "_logprob"] = m.greedy(prompts, E["n_new"],
                                                                 logprob=True)
        toks, st = m.consensus(prompts, E["n_new"], blk=E["blk"])
        out[name + "_loop"] = toks
        rep.setdefault("tokens_per_forward", {})[name] = st["tokens_per_forward"]
        del m
    rep["fp32_loop_vs_fp32_greedy"] = trajectory_report(out["fp32_loop"], out["fp32_greedy"])
    rep["bf16_loop_vs_fp32_greedy"] = trajectory_report(out["bf16_loop"], out["fp32_greedy"])
    rep["bf16_loop_vs_bf16_greedy"] = trajectory_report(out["bf16_loop"], out["bf16_greedy"])
    rep["bf16_greedy_vs_fp32_greedy"] = trajectory_report(out["bf16_greedy"],
                                                          out["fp32_greedy"])
    rep["bf16_loop_vs_fp32_greedy_by_reference_perplexity"] = perplexity_report(
        out["bf16_loop"], out["fp32_greedy"], out["fp32_logprob"])
    rep["seconds"] = time.perf_counter() - t0
    return rep, {"prompts": prompts, "weights": W, "fp32_greedy": out["fp32_greedy"]}


def oracle_decoder_leg(dec_raw, prompts_n=8, n_new=64):
    """CPU baseline of the end-to-end configuration: the float64 oracle's
    greedy AR decoding of the first `prompts_n` prompts (`n_new` tokens each)
    and its consensus loop on the first two, timed on this host's cores, and
    the GPU FP32 greedy trajectories' match against the oracle's on that
    subset (different summation orders may flip a true near-tie, so the match
    is reported, not assumed)."""
    import oracle
    E = synth_workload("e2e_decoder")
    cfg = oracle.model_cfg(E["V"], E["d"], E["L"], E["Hq"], E["Hkv"], E["hd"], E["ffn"])
    wflat = oracle.pack_weights(cfg, dec_raw["weights"])
    nthreads = os.cpu_count() or 1
    sub = dec_raw["prompts"][:prompts_n]
    t0 = time.perf_counter()
    ref = [oracle.greedy_ar(cfg, wflat, p, n_new, nthreads=nthreads) for p in sub]
    t_greedy = time.perf_counter() - t0
    gpu = dec_raw["fp32_greedy"][:prompts_n, :n_new]
    exact = [bool(np.array_equal(gpu[b], ref[b])) for b in range(len(sub))]
    tok = [float(np.mean(gpu[b] == ref[b])) for b in range(len(sub))]
    n_cons = 32
    t0 = time.perf_counter()
    cons, _ = oracle.consensus_decode(cfg, wflat, sub[-1], n_cons, blk=E["blk"],
                                      nthreads=nthreads)
    t_cons = time.perf_counter() - t0
    return {"subset": f"first {len(sub)} prompts (lengths {[len(p) for p in sub]}), "
                      f"{n_new} greedy tokens each; consensus loop on the last of them, "
                      f"{n_cons} tokens",
            "cores": nthreads,
            "greedy_tokens_per_s": len(sub) * n_new / t_greedy,
            "consensus_tokens_per_s": n_cons / t_cons,
            "consensus_equals_greedy": bool(np.array_equal(cons, ref[-1][:n_cons])),
            "gpu_fp32_greedy_vs_oracle_exact_match_rate": float(np.mean(exact)),
            "gpu_fp32_greedy_vs_oracle_token_match_rate": float(np.mean(tok))}


def synth_workload(name):
    from block_attention_b200 import synth
    return synth.WORKLOADS[name]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e-decoder", action="store_true",
                    help="skip the end-to-end decoder report (runs after the timing)")
    ap.add_argument("--no-batched", action="store_true",
                    help="skip the batched ragged attention, stochastic consensus and LM-head "
                         "legs (they run after the timing)")
    ap.add_argument("--attn-batch", type=int, default=8,
                    help="sequences of the --kernel attn case (8: larger than L2; 1: the "
                         "round's call)")
    ap.add_argument("--kernel", choices=["attn", "blk", "sample", "lmhead", "proj", "argmax",
                                         "projround", "small"], default=None,
                    help="attn: time block attention alone on a case larger than L2 (for "
                         "profiling); blk: block-size sweep K in {4, 8, 16, 32}; sample: "
                         "the stochastic round's kernels one at a time; lmhead: the LM head "
                         "with the argmax in its epilogue against GEMM + argmax; proj: the "
                         "attention block's projections alone; argmax: the vocabulary argmax "
                         "alone; projround: the Qwen3-8B round with the projections and the "
                         "LM head on the path; small: the tiny and Qwen3-1.7B attention "
                         "configurations")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.kernel == "attn":
        return kernel_alone(args)
    if args.kernel == "blk":
        return block_size_sweep(args)
    if args.kernel == "sample":
        return sampling_kernels(args)
    if args.kernel == "lmhead":
        return lm_head_kernel(args)
    if args.kernel == "proj":
        return projection_kernels(args)
    if args.kernel == "argmax":
        import torch
        hbm, _ = peaks()
        print(json.dumps({"kernel": "vocab_argmax",
                          **argmax_leg(torch.device("cuda", 0), hbm, reps=args.steps)}))
        return
    if args.kernel == "small":
        import torch
        hbm, _ = peaks()
        print(json.dumps({"kernel": "block_attn_small_configs",
                          **small_config_legs(torch.device("cuda", 0), hbm)}))
        return
    if args.kernel == "projround":
        import torch
        hbm, _ = peaks()
        print(json.dumps({"kernel": "projected_round",
                          **projected_round_leg(torch.device("cuda", 0), hbm, steps=args.steps,
                                                warmup=args.warmup)}))
        return

    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        return reference_arm(args, rank, world)

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", device_id=dev, timeout=timedelta(seconds=120))

    import block_attention_b200 as ba
    from block_attention_b200.round import DecodeRound
    ba.lib()
    w = WORKLOAD
    rnd = DecodeRound(layers=w["layers"], B=w["B"], Hq=w["Hq"], Hkv=w["Hkv"], D=w["D"],
                      blk=w["blk"], vocab=w["vocab"], ctx_lens=[w["ctx"]] * w["B"],
                      dtype=w["dtype"], logits_dtype=w["logits_dtype"],
                      accept_mean=w["accept_mean"], seed=1000 + 3 + rank, device=dev)
    rnd.capture()

    for _ in range(args.warmup):
        rnd.replay()
    torch.cuda.synchronize()
    expect_ne = np.minimum(rnd.accept + 1, w["blk"])
    assert np.array_equal(rnd.n_emit.cpu().numpy(), expect_ne), "round result mismatch"
    assert int(rnd.err.item()) == 0
    # The kernels are deterministic: a sampled layer's attention output of both
    # views, poisoned before each measured loop, must come back bit-identical.
    probe_layer = w["layers"] // 2
    attn_ref = rnd.out[:, probe_layer].clone()

    def poison_probe():
        rnd.out[:, probe_layer].fill_(float("nan"))
        torch.cuda.synchronize()

    def check_probe(where):
        torch.cuda.synchronize()
        assert int(rnd.err.item()) == 0, f"device error word set during the {where}"
        assert torch.equal(rnd.out[:, probe_layer], attn_ref), \
            f"layer {probe_layer} attention differs after the {where}"
    poison_probe()

    # ---- timed region: K rounds from the graphs, inputs resident in HBM
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
        uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    except Exception:
        uuid = None
    clocks = ClockSampler(uuid)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    for k in range(args.steps):
        rnd.replay(ev[k])
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    time.sleep(0.2)
    clk = clocks.stop()

    check_probe("timed rounds")
    step_ms = [e[0].elapsed_time(e[4]) for e in ev]
    attn_ms = [e[0].elapsed_time(e[1]) + e[2].elapsed_time(e[3]) for e in ev]
    total_ms = ev[0][0].elapsed_time(ev[-1][4])
    total_ms, attn_total_ms = max_over_ranks([total_ms, sum(attn_ms)], dev)

    launches_attn = 2 * w["layers"] * args.steps
    attn_launch_us = attn_total_ms * 1e3 / launches_attn
    bytes_per_launch = rnd.attn_bytes_per_launch()
    hbm, src = peaks()
    achieved = bytes_per_launch / (attn_launch_us * 1e-6) / 1e9
    rounds_per_s = whole_job_rate(world, args.steps, total_ms)
    gpu_launches = rnd.kernels_per_round() * args.steps

    # ---- end to end: per-round inputs from pinned host memory, results back.
    # Two input sets: round i+1's inputs are copied in on a second stream
    # while round i runs on the other set; every round's copy, graph and
    # result read-back are inside the timed region.
    cpus_before, host_cpus = bind_host_to_gpu(local)
    h_in, h_out = rnd.pinned_inputs(), rnd.pinned_outputs()
    rnd.add_input_set()
    comp, copy = torch.cuda.current_stream(dev), torch.cuda.Stream(device=dev)
    copied = [torch.cuda.Event() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]

    def e2e_rounds_run(n):
        copy.wait_stream(comp)
        with torch.cuda.stream(copy):
            bi = rnd.h2d(h_in, into=0)
        copied[0].record(copy)
        bo = 0
        for i in range(n):
            s = i % 2
            comp.wait_event(copied[s])
            rnd.use_set(s)
            rnd.replay()
            done[s].record(comp)
            bo = rnd.d2h(h_out)
            if i + 1 < n:
                t = 1 - s
                if i >= 1:
                    copy.wait_event(done[t])  # the round that last read set t
                with torch.cuda.stream(copy):
                    rnd.h2d(h_in, into=t)
                copied[t].record(copy)
        comp.wait_stream(copy)
        return bi, bo

    e2e_rounds_run(3)
    torch.cuda.synchronize()
    poison_probe()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    bi, bo = e2e_rounds_run(args.steps)
    e1.record()
    torch.cuda.synchronize()
    rnd.use_set(0)
    (e2e_ms,) = max_over_ranks([e0.elapsed_time(e1)], dev)
    e2e_rounds = whole_job_rate(world, args.steps, e2e_ms)
    if cpus_before:
        os.sched_setaffinity(0, cpus_before)  # the CPU legs below use every core
    assert np.array_equal(h_out["n_emit"].numpy(), expect_ne)
    check_probe("end-to-end rounds")

    dec = dec_raw = None
    if rank == 0 and world == 1 and not args.no_e2e_decoder:
        dec, dec_raw = decoder_report()

    # ---- the same rounds without the next-layer L2 warm-up (for comparison)
    nopf = None
    if not args.no_batched:
        rnd.prefetch = False
        rnd.capture()
        for _ in range(args.warmup):
            rnd.replay()
        poison_probe()
        ev2 = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
        for k in range(args.steps):
            rnd.replay(ev2[k])
        check_probe("rounds without prefetch")
        a2 = max_over_ranks([sum(e[0].elapsed_time(e[1]) + e[2].elapsed_time(e[3]) for e in ev2),
                             ev2[0][0].elapsed_time(ev2[-1][4])], dev)
        us2 = a2[0] * 1e3 / launches_attn
        nopf = {"us_per_launch": us2, "gbs": bytes_per_launch / us2 / 1e3,
                "pct_of_peak": 100.0 * bytes_per_launch / us2 / 1e3 / hbm,
                "rounds_per_s": whole_job_rate(world, args.steps, a2[1])}
        rnd.prefetch = True

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, sample = oracle_round_sample(heads=WORKLOAD["Hkv"], layers_timed=4)
        cpu = {"value": v, "unit": "rounds/s", "cores": cores, "kind": "oracle",
               "sample": sample}
        if dec_raw is not None:
            cpu["e2e_decoder"] = oracle_decoder_leg(dec_raw)
    batched = stochastic = lm_head = small = amax = proj = None
    if rank == 0 and world == 1 and not args.no_batched:
        small = small_config_legs(dev, hbm)
        amax = argmax_leg(dev, hbm)
        proj = projected_round_leg(dev, hbm)
        batched = batched_ragged_leg(dev, hbm)
        stochastic = stochastic_round_leg(dev, hbm)
        lm_head = lm_head_leg(dev)

    if world > 1:
        dist.barrier()
        rnd.graphs = None
        dist.destroy_process_group()
    if rank != 0:
        return
    rb = rnd.round_bytes()
    line = {
        "metric": METRIC, "value": rounds_per_s, "unit": "rounds/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": config_dict(),
        "block_attn": {"gbs": achieved, "pct_of_peak": 100.0 * achieved / hbm,
                       "us_per_launch": attn_launch_us, "bytes_per_launch": bytes_per_launch,
                       "launches_per_round": 2 * w["layers"],
                       "next_layer_l2_prefetch": True},
        "block_attn_without_prefetch": nopf,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "peak_source": src, "traffic": measured_traffic(),
                     "kernel": "block_attn (both views, per-layer launches)"},
        "round_bytes": rb,
        "round_hbm_gbs": sum(rb.values()) / (total_ms / args.steps * 1e-3) / 1e9,
        "step_ms_median": statistics.median(step_ms),
        "e2e": {"value": e2e_rounds, "unit": "rounds/s", "h2d_bytes_per_step": bi,
                "d2h_bytes_per_step": bo, "host_cpus": host_cpus or "unbound"},
        "gpu_launches": gpu_launches,
        "clocks": clk,
        "cpu_baseline": cpu,
        "e2e_decoder": dec,
        "block_attn_small_configs": small,
        "vocab_argmax": amax,
        "projected_round": proj,
        "block_attn_batched_ragged": batched,
        "stochastic_consensus": stochastic,
        "lm_head_argmax": lm_head,
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
