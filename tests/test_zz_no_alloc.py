"""The scratch-free argmax entry point, for callers that cannot allocate.

Some users of this library run where they cannot call cudaMalloc (no
allocator available or allowed: code handed only the tensors it works on, or
a process whose device memory is fully reserved).  orthrus_vocab_argmax_noalloc
serves them from a static device array instead of a caller workspace.  This
test calls it through the C ABI and checks that it returns exactly what the
workspace-based orthrus_vocab_argmax returns (argmax indices are integer
results: bit-exact), on two calls in a row, and that a row count beyond the
static scratch is refused.  It lives in its own file, collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import block_attention_b200 as ba
from block_attention_b200 import synth

pytestmark = pytest.mark.gpu

MAX_ROWS = 4096  # ORTHRUS_NOALLOC_ARGMAX_MAX_ROWS in include/orthrus.h


def _noalloc():
    L = ba.lib()
    fn = L.orthrus_vocab_argmax_noalloc
    c = ctypes
    fn.argtypes = [c.c_int32, c.c_void_p, c.c_int32, c.c_int32, c.c_int64, c.c_void_p,
                   c.c_void_p, c.c_void_p]
    fn.restype = c.c_int
    return fn


def _call_noalloc(fn, logits, idx, maxval):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rows, vocab = logits.shape
    return fn(ba.F32 if logits.dtype == torch.float32 else ba.BF16,
              ctypes.c_void_p(logits.data_ptr()), rows, vocab, logits.stride(0),
              ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(maxval.data_ptr()), stream)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_noalloc_argmax_matches_workspace_argmax_twice(dtype):
    fn = _noalloc()
    # 151936 and 8192: one cluster per row; 300007 (19 chunks): the scratch's
    # atomic slots and tickets
    for call, (rows, vocab) in enumerate([(32, 151936), (200, 8192), (9, 300007)]):
        x = synth.logits(synth.rng(400 + call, len(dtype)), rows, vocab, dtype=dtype)
        if dtype == "bf16":
            t = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
        else:
            t = torch.from_numpy(x).cuda()
        idx_a = torch.full((rows,), -7, dtype=torch.int32, device="cuda")
        max_a = torch.empty(rows, dtype=torch.float32, device="cuda")
        assert _call_noalloc(fn, t, idx_a, max_a) == 0
        max_b = torch.empty(rows, dtype=torch.float32, device="cuda")
        idx_b = ba.vocab_argmax(t, maxval=max_b)
        torch.cuda.synchronize()
        assert torch.equal(idx_a, idx_b), call
        assert torch.equal(max_a, max_b), call


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_noalloc_argmax_unaligned_row_stride(dtype):
    """Rows that do not start on a 16-byte boundary take the kernel's scalar
    path: vocab 100003 with a row stride of 100003 elements."""
    fn = _noalloc()
    rows, vocab = 24, 100003
    x = synth.logits(synth.rng(410, len(dtype)), rows, vocab, dtype=dtype)
    if dtype == "bf16":
        t = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    else:
        t = torch.from_numpy(x).cuda()
    assert t.stride(0) == vocab
    for _ in range(2):
        idx_a = torch.full((rows,), -7, dtype=torch.int32, device="cuda")
        max_a = torch.empty(rows, dtype=torch.float32, device="cuda")
        assert _call_noalloc(fn, t, idx_a, max_a) == 0
        max_b = torch.empty(rows, dtype=torch.float32, device="cuda")
        idx_b = ba.vocab_argmax(t, maxval=max_b)
        torch.cuda.synchronize()
        assert torch.equal(idx_a, idx_b)
        assert torch.equal(max_a, max_b)


def test_noalloc_argmax_allocates_no_device_memory():
    """After a first call (which looks up the static array), further calls
    leave the device's free memory unchanged."""
    fn = _noalloc()
    rows, vocab = 64, 151936
    t = torch.from_numpy(synth.logits(synth.rng(420, 3), rows, vocab, dtype="f32")).cuda()
    idx = torch.empty(rows, dtype=torch.int32, device="cuda")
    mx = torch.empty(rows, dtype=torch.float32, device="cuda")
    assert _call_noalloc(fn, t, idx, mx) == 0
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(5):
        assert _call_noalloc(fn, t, idx, mx) == 0
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0


def test_noalloc_argmax_refuses_rows_beyond_its_scratch():
    fn = _noalloc()
    t = torch.zeros(MAX_ROWS + 1, 16, device="cuda")
    idx = torch.zeros(MAX_ROWS + 1, dtype=torch.int32, device="cuda")
    mx = torch.zeros(MAX_ROWS + 1, device="cuda")
    assert _call_noalloc(fn, t, idx, mx) == -2  # ORTHRUS_EUNSUPPORTED
    assert _call_noalloc(fn, t[:MAX_ROWS], idx, mx) == 0
    torch.cuda.synchronize()
    assert int(idx[:MAX_ROWS].max()) == 0  # all-equal rows -> lowest index
