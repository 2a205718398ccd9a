"""CPU-only checks of the C ABI: the library loads, exports every function
the headers under include/ declare, the ctypes structs match the C layout, and
host-side argument checks return their status codes without launching
anything (no GPU is touched by these calls)."""
import ctypes
import os
import re
import subprocess

import pytest

import block_attention_b200 as ba
from block_attention_b200 import build as ba_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
HEADERS = sorted(os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h"))


@pytest.fixture(scope="module")
def L():
    ba_build.build()
    return ba.lib()


def _declared_functions():
    names = set()
    for h in HEADERS:
        src = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names |= set(re.findall(r"\b(orthrus_\w+)\s*\(", src))
    return sorted(names)


def test_exports_every_declared_symbol(L):
    names = _declared_functions()
    assert set(names) >= set(ba.EXPORTS)
    out = subprocess.run(["nm", "-D", "--defined-only", ba.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r" T (\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        getattr(L, n)


def test_version_and_status_strings(L):
    assert L.orthrus_version() == 10000
    assert L.orthrus_status_str(0) == b"ok"
    for code in (-1, -2, -3, -4, -5):
        assert L.orthrus_status_str(code) not in (b"ok", b"unknown status")


def test_struct_layout_matches_c(tmp_path):
    prog = tmp_path / "layout.c"
    prog.write_text(r'''
#include <stddef.h>
#include <stdio.h>
#include "orthrus.h"
#define F(T, m) printf(#T " " #m " %zu\n", offsetof(T, m))
int main(void) {
  printf("orthrus_attn_args size %zu\n", sizeof(orthrus_attn_args));
  F(orthrus_attn_args, scale); F(orthrus_attn_args, flags); F(orthrus_attn_args, q);
  F(orthrus_attn_args, ctx_lens);
  F(orthrus_attn_args, err); F(orthrus_attn_args, workspace_bytes);
  F(orthrus_attn_args, next_k_cache); F(orthrus_attn_args, next_v_cache);
  printf("orthrus_commit_args size %zu\n", sizeof(orthrus_commit_args));
  F(orthrus_commit_args, k_cache); F(orthrus_commit_args, cache_layer_stride);
  F(orthrus_commit_args, blk_layer_stride); F(orthrus_commit_args, n_emit);
  F(orthrus_commit_args, workspace_bytes);
  printf("orthrus_sample_args size %zu\n", sizeof(orthrus_sample_args));
  F(orthrus_sample_args, row_stride); F(orthrus_sample_args, temperature);
  F(orthrus_sample_args, step); F(orthrus_sample_args, seed); F(orthrus_sample_args, draft);
  F(orthrus_sample_args, logq); F(orthrus_sample_args, lse_diff);
  F(orthrus_sample_args, logits_ar); F(orthrus_sample_args, logits_diff);
  F(orthrus_sample_args, logp); F(orthrus_sample_args, lse_ar);
  F(orthrus_sample_args, accept_len); F(orthrus_sample_args, n_emit);
  F(orthrus_sample_args, emitted); F(orthrus_sample_args, next_anchor);
  F(orthrus_sample_args, workspace); F(orthrus_sample_args, workspace_bytes);
  return 0;
}''')
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(prog), "-o", str(exe)],
                   check=True)
    got = {}
    for line in subprocess.run([str(exe)], capture_output=True, text=True).stdout.splitlines():
        t, m, v = line.split()
        got[(t, m)] = int(v)
    cls = {"orthrus_attn_args": ba.AttnArgs, "orthrus_commit_args": ba.CommitArgs,
           "orthrus_sample_args": ba.SampleArgs}
    for (t, m), v in got.items():
        c = cls[t]
        assert (ctypes.sizeof(c) if m == "size" else getattr(c, m).offset) == v, (t, m)


@pytest.mark.parametrize("compiler,std", [("gcc", "-std=c99"), ("g++", "-std=c++17")])
def test_headers_compile_as_strict_c_and_cpp(tmp_path, compiler, std):
    """Both public headers stand alone in C99 and C++17 (the ABI is plain C:
    no C++ types leak into the declarations)."""
    src = tmp_path / ("hdr.c" if compiler == "gcc" else "hdr.cpp")
    src.write_text('#include "orthrus.h"\n#include "orthrus_decoder.h"\n'
                   'int main(void) { return orthrus_version() > 0 ? 0 : 1; }\n')
    subprocess.run([compiler, std, "-Wall", "-Wextra", "-pedantic", "-Werror", "-fsyntax-only",
                    "-I", os.path.join(ROOT, "include"), str(src)], check=True)


def _args(**kw):
    base = dict(dtype=0, mask_mode=0, B=1, Hq=4, Hkv=2, D=64, blk=32, cap=300, max_ctx=256,
                scale=0.125)
    base.update(kw)
    a = ba.AttnArgs()
    for k, v in base.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw,code", [
    (dict(dtype=7), -1), (dict(mask_mode=2), -1), (dict(Hq=5), -1), (dict(blk=0), -1),
    (dict(D=96), -2), (dict(blk=33), -2), (dict(Hq=16, Hkv=2, blk=32), -2),
    (dict(max_ctx=301), -4), (dict(scale=float("inf")), -1),
    (dict(scale=0.0), -1), (dict(scale=-0.125), -1),
])
def test_block_attn_rejects_bad_shapes_without_launch(L, kw, code):
    a = _args(**kw)
    assert L.orthrus_block_attn(ctypes.byref(a), None) == code
    assert L.orthrus_block_attn_workspace(ctypes.byref(a)) == 0


def test_block_attn_null_pointers_and_workspace(L):
    a = _args()
    assert L.orthrus_block_attn(ctypes.byref(a), None) == -1  # null tensors
    for f in ("q", "k_blk", "v_blk", "k_cache", "v_cache", "out", "ctx_lens"):
        setattr(a, f, 4096)  # aligned fake addresses: never dereferenced
    need = L.orthrus_block_attn_workspace(ctypes.byref(a))
    assert need > 0
    assert L.orthrus_block_attn(ctypes.byref(a), None) == -3  # no workspace
    a.workspace, a.workspace_bytes = 8192, need - 1
    assert L.orthrus_block_attn(ctypes.byref(a), None) == -3
    a.q = 4100  # misaligned
    assert L.orthrus_block_attn(ctypes.byref(a), None) == -1
    b = _args(B=0)
    assert L.orthrus_block_attn(ctypes.byref(b), None) == 0  # nothing to do


def test_argmax_consensus_commit_host_checks(L):
    assert L.orthrus_vocab_argmax(0, None, 4, 0, 0, None, None, None, 0, None) == -1
    assert L.orthrus_vocab_argmax(0, None, 4, 10, 5, None, None, None, 0, None) == -1
    assert L.orthrus_vocab_argmax(3, None, 4, 10, 10, None, None, None, 0, None) == -1
    assert L.orthrus_vocab_argmax(0, None, 0, 10, 10, None, None, None, 0, None) == 0
    assert L.orthrus_vocab_argmax(0, 4096, 4, 10, 10, 4096, None, None, 0, None) == -3
    assert L.orthrus_vocab_argmax_workspace(32) >= 32 * 12
    assert L.orthrus_consensus(None, None, 1, 0, None, None, None, None, None) == -1
    assert L.orthrus_consensus(None, None, 1, 33, None, None, None, None, None) == -2
    assert L.orthrus_consensus(None, None, 0, 32, None, None, None, None, None) == 0
    assert L.orthrus_consensus(None, None, 2, 32, None, None, None, None, None) == -1
    c = ba.CommitArgs(dtype=1, layers=2, B=1, Hkv=8, D=128, blk=32, cap=100,
                      cache_layer_stride=10, blk_layer_stride=10)
    assert L.orthrus_kv_commit(ctypes.byref(c), None) == -1  # strides too small
    c.cache_layer_stride, c.blk_layer_stride = 8 * 100 * 128, 32 * 8 * 128
    for f in ("k_cache", "v_cache", "k_blk", "v_blk", "ctx_lens", "n_emit"):
        setattr(c, f, 4096)
    assert L.orthrus_kv_commit(ctypes.byref(c), None) == -3  # no workspace
    assert L.orthrus_kv_commit_workspace(ctypes.byref(c)) >= 4


def test_python_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(2, 8)
    with pytest.raises(ValueError):
        ba.vocab_argmax(x)


def test_decoder_entry_points_host_checks(L):
    c = ctypes
    vp = c.c_void_p
    # bad dtype, negative sizes and null pointers are refused before any launch
    assert L.orthrus_embed(5, vp(256), 10, 8, vp(256), 2, vp(256), None, None) == -1
    assert L.orthrus_embed(0, None, 10, 8, None, 0, None, None, None) == 0
    assert L.orthrus_embed(0, None, 10, 8, vp(256), 2, vp(256), None, None) == -1
    assert L.orthrus_rmsnorm(0, vp(256), vp(256), 2, 0, c.c_float(1e-6), vp(256), None) == -1
    assert L.orthrus_rmsnorm(0, vp(256), vp(256), 2, 8, c.c_float(float("nan")), vp(256),
                             None) == -1
    assert L.orthrus_rmsnorm(1, None, None, 0, 8, c.c_float(1e-6), None, None) == 0
    assert L.orthrus_linear(0, vp(256), vp(512), None, 4, 0, 8, vp(1024), None) == -1
    assert L.orthrus_linear(0, vp(256), vp(512), None, 4, 8, 8, vp(256), None) == -1  # out == x
    assert L.orthrus_linear(0, None, None, None, 0, 8, 8, None, None) == 0
    assert L.orthrus_linear(0, vp(256), vp(512), None, 128 * 65536, 8, 8, vp(1024),
                            None) == -2
    assert L.orthrus_qkv_rope(0, vp(256), 1, 4, 2, 1, 7, vp(256), c.c_double(1e6), vp(256),
                              vp(256), vp(256), None) == -1  # odd head dim
    assert L.orthrus_qkv_rope(0, vp(256), 1, 4, 2, 1, 8, vp(256), c.c_double(0.0), vp(256),
                              vp(256), vp(256), None) == -1  # theta <= 0
    assert L.orthrus_swiglu(0, vp(256), 2, 0, vp(256), None) == -1
    assert L.orthrus_swiglu(0, None, 0, 8, None, None) == 0
    assert L.orthrus_block_tokens(vp(256), None, 1, 33, 0, vp(256), None) == -1
    assert L.orthrus_block_tokens(None, None, 1, 32, 0, vp(256), None) == -1
    assert L.orthrus_block_tokens(None, None, 0, 32, 0, None, None) == 0


def test_sampling_entry_points_host_checks(L):
    c = ctypes
    vp = c.c_void_p
    ws = L.orthrus_vocab_sample_workspace(4, 10)
    assert ws >= 4 * 8 + 4 * 4 + 4 * 8  # keys, tickets, one chunk pair per row
    # temperature must be positive and finite
    for T in (0.0, -1.0, float("inf"), float("nan")):
        assert L.orthrus_vocab_sample(0, vp(256), 4, 10, 10, c.c_float(T), 1, 0, vp(256),
                                      None, None, vp(256), ws, None) == -1
        assert L.orthrus_token_logprob(0, vp(256), 4, 10, 10, vp(256), c.c_float(T), vp(256),
                                       None, vp(256), 1 << 20, None) == -1
    assert L.orthrus_vocab_sample(0, vp(256), 4, 10, 10, c.c_float(1.0), 1, 0, vp(256),
                                  None, None, vp(256), ws - 1, None) == -3  # workspace
    assert L.orthrus_vocab_sample(0, vp(256), 4, 10, 10, c.c_float(1.0), 1, 0, vp(256),
                                  None, None, vp(264), ws, None) == -3  # 16-byte alignment
    assert L.orthrus_vocab_sample(0, None, 0, 10, 10, c.c_float(1.0), 1, 0, None, None, None,
                                  None, 0, None) == 0
    assert L.orthrus_vocab_sample(0, vp(256), 4, (1 << 30) + 1, (1 << 30) + 1, c.c_float(1.0),
                                  1, 0, vp(256), None, None, vp(256), 1 << 40, None) == -2
    a = ba.SampleArgs(dtype=0, B=1, blk=33, vocab=10, row_stride=10, temperature=1.0)
    assert L.orthrus_consensus_sample(ctypes.byref(a), None) == -2  # blk > 32
    a.blk = 4
    assert L.orthrus_consensus_sample(ctypes.byref(a), None) == -1  # null tensors
    for f in ("draft", "logq", "lse_diff", "logits_ar", "logits_diff", "logp", "lse_ar",
              "n_emit"):
        setattr(a, f, 4096)
    assert L.orthrus_consensus_sample(ctypes.byref(a), None) == -1  # accept_len is required
    a.accept_len = 4096
    assert L.orthrus_consensus_sample(ctypes.byref(a), None) == -3  # no workspace
    a.workspace, a.workspace_bytes = 4096, L.orthrus_consensus_sample_workspace(1, 4, 10)
    a.B, a.blk = 2048, 32
    assert L.orthrus_consensus_sample(ctypes.byref(a), None) == -3  # too small for B = 2048
    a.workspace_bytes = L.orthrus_consensus_sample_workspace(2048, 32, 10)
    assert L.orthrus_consensus_sample(ctypes.byref(a), None) == -2  # B * blk > 65535
    a.B, a.blk = 1, 4
    assert L.orthrus_token_logprob(0, vp(256), 4, 10, 10, vp(256), c.c_float(1.0), vp(256),
                                   None, None, 0, None) == -3
    assert L.orthrus_consensus_sample_workspace(4, 8, 10) >= 4 * 24 + 32 * 4 + 32 * 8
    a.B = 0
    assert L.orthrus_consensus_sample(ctypes.byref(a), None) == 0


def test_lm_head_argmax_host_checks(L):
    c = ctypes
    vp = c.c_void_p
    ws = L.orthrus_lm_head_argmax_workspace(32)
    assert ws >= 32 * 8 + 4
    args = lambda dtype=1, h=256, rows=32, d=4096, ld=4096, w=512, V=151936, idx=1024, \
        wsp=2048, wsb=ws: (dtype, vp(h) if h else None, rows, d, ld, vp(w) if w else None, V,
                          vp(idx) if idx else None, None, None, vp(wsp) if wsp else None, wsb,
                          None)
    assert L.orthrus_lm_head_argmax(*args(dtype=7)) == -1          # unknown dtype
    assert L.orthrus_lm_head_argmax(*args(dtype=0)) == -2          # fp32: not implemented
    assert L.orthrus_lm_head_argmax(*args(rows=-1)) == -1
    assert L.orthrus_lm_head_argmax(*args(ld=100, d=128)) == -1    # row stride < d
    assert L.orthrus_lm_head_argmax(*args(rows=0, h=0, w=0, idx=0, wsp=0)) == 0
    assert L.orthrus_lm_head_argmax(*args(rows=129)) == -2         # more rows than TMEM lanes
    assert L.orthrus_lm_head_argmax(*args(d=4000, ld=4000)) == -2  # d not a multiple of 64
    assert L.orthrus_lm_head_argmax(*args(ld=4100)) == -2          # pitch not 16-byte
    assert L.orthrus_lm_head_argmax(*args(V=(1 << 30) + 1)) == -2
    assert L.orthrus_lm_head_argmax(*args(h=0)) == -1
    assert L.orthrus_lm_head_argmax(*args(w=520)) == -1            # w not 16-byte aligned
    assert L.orthrus_lm_head_argmax(*args(wsb=ws - 1)) == -3
    assert L.orthrus_lm_head_argmax(*args(wsp=2056)) == -3         # workspace alignment


def test_lm_head_plan_respects_hardware_limits(L):
    """The LM head's launch shape over a sweep of sizes and SM counts (host
    only): tiles within the UMMA N range and the TMA box limit, the stage ring
    and TMEM within the SM's 227 KB and 512 columns, at least one slot of look
    ahead, every vocabulary row covered, the grid within the SMs."""
    out = (ctypes.c_int32 * 8)()
    for sms in (148, 132, 16, 1):
        for rows in (1, 7, 32, 33, 64, 96, 128):
            for d in (64, 128, 192, 256, 1024, 4096, 8192):
                for V in (1, 100, 128, 3001, 32000, 151936, 262144, 1 << 20):
                    assert L.orthrus_lm_head_argmax_plan(rows, d, V, sms, out) == 0
                    nv, kb, stages, aslots, smem, grid, tiles, tmem = list(out)
                    assert nv % 16 == 0 and 128 <= nv <= 256, (rows, d, V, nv)
                    assert kb in (1, 2, 4) and (d // 64) % kb == 0
                    assert kb > 1 or (d // 64) % 2 == 1  # one box only for an odd K
                    assert stages >= 2 and aslots >= 1 and min(aslots, stages) >= 1
                    assert smem <= 227 * 1024, (rows, d, V, smem)
                    nvp = (nv + 31) // 32 * 32
                    assert nvp + aslots * 32 * kb <= tmem == 512
                    assert tiles * nv >= V > (tiles - 1) * nv
                    assert 1 <= grid <= min(sms, tiles)
    # the Qwen3-8B LM head as measured: 176-row tiles, four boxes per stage and
    # two stages for one block; 208-row tiles, two boxes per stage and three
    # stages for four blocks (their h boxes, 16 KB each, in the separate h ring)
    assert L.orthrus_lm_head_argmax_plan(32, 4096, 151936, 148, out) == 0
    assert list(out)[:4] == [176, 4, 2, 2]
    assert L.orthrus_lm_head_argmax_plan(128, 4096, 151936, 148, out) == 0
    assert list(out)[:4] == [208, 2, 3, 4]
    for bad in ((0, 4096, 100, 148), (129, 4096, 100, 148), (32, 100, 100, 148),
                (32, 4096, 0, 148), (32, 4096, 100, 0)):
        assert L.orthrus_lm_head_argmax_plan(*bad, out) == -1


def test_tensor_core_attention_plan(L):
    """Launch plan of the bf16 tensor-core path over a sweep of shapes and SM
    counts: S splits per (sequence, kv-head) with 1 <= S <= min(24, tiles / 2)
    (at least two tiles a split; 24: the merge stages a split per lane of a
    warp and a bounded staging area), one wave of CTAs
    when the batch is small, no split longer than 64 tiles unless S is
    capped, the shared memory within the 227 KB a CTA may use, the merge
    inside the launch exactly when the grid fits one wave, and a workspace
    that holds the 2048-byte counter head plus every split's fp32 partial for
    any GPU of up to 256 SMs."""
    out = (ctypes.c_int32 * 8)()
    for D in (64, 128):
        for Hq, Hkv, blk in ((32, 8, 32), (16, 8, 32), (8, 8, 16), (32, 8, 4), (64, 2, 2)):
            for B in (1, 2, 8, 16, 64, 512):
                for max_ctx in (0, 1, 100, 8192, 32768, 131072):
                    a = _args(dtype=1, B=B, Hq=Hq, Hkv=Hkv, D=D, blk=blk, max_ctx=max_ctx,
                              cap=max_ctx + blk, scale=D ** -0.5)
                    ws = L.orthrus_block_attn_workspace(ctypes.byref(a))
                    assert L.orthrus_block_attn_plan(ctypes.byref(a), 256, out) == 0
                    part = (128 + 24) * (D // 2 + 4) * 4  # bf16 O + fp32 (max, sum) per row
                    assert ws == 2048 + B * Hkv * out[0] * part, (D, Hq, Hkv, blk, B, max_ctx)
                    assert L.orthrus_block_attn_launches(ctypes.byref(a)) in (1, 2)
                    for sms in (132, 148, 160, 256):
                        key = (D, Hq, Hkv, blk, B, max_ctx, sms)
                        assert L.orthrus_block_attn_plan(ctypes.byref(a), sms, out) == 0, key
                        S, gx, gy, gz, thr, smem, most, fused = list(out)
                        tiles = -(-max_ctx // 128) + 1
                        heads = B * Hkv
                        assert 1 <= S <= min(24, max(1, tiles // 2)), key
                        assert 2048 + heads * S * part <= ws, key  # fits the sized buffer
                        assert (gx, gy, gz) == (Hkv, B, S), key
                        assert most == -(-tiles // S), key
                        assert most <= 64 or S == 24, key
                        if heads < sms:  # a small batch fills the SMs as far as it can
                            assert S >= min(24, max(1, tiles // 2), sms // heads), key
                        # more CTAs than SMs only where long sequences need the splits
                        assert heads * S <= sms or S == min(24, tiles, -(-tiles // 64)), key
                        assert fused == int(heads * S <= sms and heads <= 256), key
                        assert thr % 32 == 0 and 0 < smem <= 227 * 1024, key
    # the fp32 path has no such plan
    a = _args(dtype=0, B=1, Hq=32, Hkv=8, D=128, blk=32, max_ctx=64, cap=96, scale=0.1)
    assert L.orthrus_block_attn_plan(ctypes.byref(a), 148, out) == -2
    a = _args(dtype=1, B=1, Hq=32, Hkv=8, D=128, blk=32, max_ctx=8192, cap=8224, scale=0.1)
    assert L.orthrus_block_attn_plan(ctypes.byref(a), 0, out) == -1
    # the Qwen3-8B round shape on 148 SMs: 18 splits per kv-head, 144 CTAs,
    # at most 4 of the 65 tiles each, merged inside the launch
    assert L.orthrus_block_attn_plan(ctypes.byref(a), 148, out) == 0
    assert list(out)[:4] == [18, 8, 1, 18] and out[6] == 4 and out[7] == 1
    # the Qwen3-1.7B layer (ctx 2048, 17 tiles): 8 splits of two or three
    # tiles rather than 17 of one, merged inside the launch
    a = _args(dtype=1, B=1, Hq=16, Hkv=8, D=128, blk=32, max_ctx=2048, cap=2080, scale=0.1)
    assert L.orthrus_block_attn_plan(ctypes.byref(a), 148, out) == 0
    assert list(out)[:4] == [8, 8, 1, 8] and out[6] == 3 and out[7] == 1


def test_linear_tc_plan_and_rejections(L):
    """Launch plan of the tensor-core projection over a sweep: tiles of 128
    features, K splits that fill the SMs without exceeding 16 or the K steps,
    at least two ring stages within the shared memory a CTA may use, TMEM
    columns a power of two holding the rows; and the host-side rejections."""
    out = (ctypes.c_int32 * 8)()
    for rows in (1, 16, 17, 32, 100, 128):
        for K in (64, 640, 4096):
            for N in (1, 128, 300, 4096, 6144, 151936):
                for sms in (132, 148, 160):
                    key = (rows, K, N, sms)
                    assert L.orthrus_linear_tc_plan(rows, K, N, sms, out) == 0, key
                    tiles, ksplit, stages, sb, smem, grid, tcols, rp = list(out)
                    assert tiles == -(-N // 128) and grid == tiles * ksplit, key
                    assert 1 <= ksplit <= min(16, K // 64), key
                    assert tiles * ksplit <= max(sms, tiles), key
                    assert stages >= 2 and smem <= 227 * 1024, key
                    assert rp == -(-rows // 16) * 16 and sb >= 128 * 128 + rp * 128, key
                    assert tcols >= rp and tcols & (tcols - 1) == 0 and tcols <= 512, key
                    assert L.orthrus_linear_tc_workspace(rows, K, N) >= tiles * 4, key
    assert L.orthrus_linear_tc_plan(129, 64, 128, 148, out) == -1
    assert L.orthrus_linear_tc_plan(32, 100, 128, 148, out) == -1
    vp = ctypes.c_void_p
    ws = L.orthrus_linear_tc_workspace(32, 4096, 6144)
    call = lambda dtype=1, x=256, rows=32, K=4096, ldx=4096, w=512, N=6144, y=1024, ldy=6144, \
        hint=0, hint_bytes=0, wsp=2048, wsb=ws: L.orthrus_linear_tc(
            dtype, vp(x) if x else None, rows, K, ldx, vp(w) if w else None, N, None,
            vp(y) if y else None, ldy, vp(hint) if hint else None, ctypes.c_int64(hint_bytes),
            None, vp(wsp) if wsp else None, wsb, None)
    assert call(dtype=0) == -2           # fp32: unsupported
    assert call(dtype=5) == -1
    assert call(rows=0) == 0             # nothing to do
    assert call(rows=129) == -2
    assert call(K=100, ldx=100) == -2    # K not a multiple of 64
    assert call(ldx=4100) == -2          # row pitch not 16-byte aligned
    assert call(ldx=10) == -1            # pitch below K
    assert call(x=0) == -1 and call(w=0) == -1 and call(y=0) == -1
    assert call(x=264) == -1             # x not 16-byte aligned
    assert call(wsp=0) == -3 and call(wsb=ws - 1) == -3 and call(wsp=2056) == -3
    # the L2 hint: 16-byte address and size, no negative size
    assert call(hint=4104, hint_bytes=4096) == -1 and call(hint=4096, hint_bytes=100) == -1
    assert call(hint=4096, hint_bytes=-16) == -1

def test_qkv_rope_projection_and_table_rejections(L):
    """Host-side checks of the QKV projection with RoPE in its epilogue and of
    the RoPE table (nothing here reaches a launch)."""
    vp = ctypes.c_void_p
    ws = L.orthrus_linear_tc_workspace(32, 4096, 6144)
    assert ws == L.orthrus_linear_tc_workspace(32, 4096, (32 + 2 * 8) * 128)
    call = lambda dtype=1, x=256, rows=32, K=4096, ldx=4096, w=512, Hq=32, Hkv=8, hd=128, \
        cs=1024, q=2048, k=4096, v=8192, wsp=16384, wsb=ws: L.orthrus_linear_tc_qkv_rope(
            dtype, vp(x) if x else None, rows, K, ldx, vp(w) if w else None, Hq, Hkv, hd,
            vp(cs) if cs else None, vp(q) if q else None, vp(k) if k else None,
            vp(v) if v else None, None, ctypes.c_int64(0), None, vp(wsp) if wsp else None, wsb,
            None)
    assert call(dtype=0) == -2           # fp32: unsupported
    assert call(hd=64) == -2             # a head must be one 128-feature tile
    assert call(hd=127) == -1 and call(Hq=0) == -1 and call(Hkv=-1) == -1
    assert call(rows=0) == 0
    assert call(rows=129) == -2 and call(K=100, ldx=100) == -2
    assert call(cs=0) == -1 and call(q=0) == -1 and call(k=0) == -1 and call(v=0) == -1
    assert call(cs=1028) == -1           # the table holds float pairs: 8-byte aligned
    assert call(x=264) == -1
    assert call(wsp=0) == -3 and call(wsb=ws - 1) == -3
    rt = lambda lens=256, B=1, blk=32, hd=128, theta=1e6, out=512: L.orthrus_rope_table(
        vp(lens) if lens else None, B, blk, hd, ctypes.c_double(theta), vp(out) if out else None,
        None)
    assert rt(B=0) == 0
    assert rt(lens=0) == -1 and rt(out=0) == -1 and rt(out=516) == -1
    assert rt(hd=127) == -1 and rt(blk=0) == -1 and rt(theta=0.0) == -1 and rt(B=-1) == -1


def test_selftest_bounded_wait_rejections(L):
    """Host-side checks of the bounded-wait self-test (no launch here)."""
    vp = ctypes.c_void_p
    st = lambda which=0, us=1000, never=256, err=512: L.orthrus_selftest_bounded_wait(
        which, ctypes.c_uint32(us), vp(never) if never else None, vp(err) if err else None, None)
    assert st(which=2) == -1 and st(which=-1) == -1
    assert st(us=0) == -1 and st(us=10_000_001) == -1
    assert st(err=0) == -1
    assert st(which=1, never=0) == -1 and st(which=1, never=258) == -1
