"""Failure detection without a fault (orthrus_selftest_bounded_wait): a wait
that never completes -- an mbarrier phase nothing arrives on, or a
generation word nothing advances, the two forms every kernel of the library
waits in -- gives up after its limit, the caller's error word reads
ORTHRUS_ETIMEOUT, and the context keeps working for the calls after it."""
import time

import numpy as np
import pytest
import torch

import block_attention_b200 as ba

pytestmark = pytest.mark.gpu

ETIMEOUT = -6


@pytest.mark.parametrize("which", [0, 1])
def test_bounded_wait_gives_up_and_the_context_stays_usable(which):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    never = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    ba.selftest_bounded_wait(which, 200_000, err=err, never=never)  # 0.2 s limit
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert int(err.item()) == ETIMEOUT
    assert elapsed >= 0.15, elapsed
    # later work on the same context is unaffected
    g = torch.Generator(device="cuda").manual_seed(which)
    x = torch.randn(8, 5000, generator=g, device="cuda")
    idx = ba.vocab_argmax(x)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(idx.cpu().numpy(), x.argmax(dim=1).cpu().numpy())
