"""Failure detection on the GPU without a GPU fault.

* A bounded wait that runs out: the test hook ``qmoe_debug_skip_stage`` makes the next
  streaming-kernel launch leave one pipeline stage of its last CTA unissued (nothing
  ever lands there).  The kernel must flag QMOE_DEV_TIMEOUT in its status word, stop all
  its roles and return; the call returns normally, and the next call on the same stream
  is correct and flags nothing.  No trap, no assert, no bad address: the waits are the
  library's ordinary bounded waits (about a second each).
* A broken ``sorted_indices`` promise (rhs decreasing somewhere) sets QMOE_DEV_UNSORTED,
  and the result is still the gather_qmm of the given indices (the rows are sorted by
  expert on the device either way; nuvec-core 0.4.0 tests/quantized.rs,
  gather_qmm_selects_batches: sorted and unsorted indices give the same products).
"""

import time

import numpy as np
import pytest
import torch

import oracle as O
from gpu_util import assert_close, dev_bf16, dev_u32
from inputs import normal_bf16, random_qweight

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_sets_status_and_the_next_call_is_clean(gpu_lib):
    q = gpu_lib
    rng = np.random.default_rng(123)
    M, N, K, group, bits = 2, 4096, 2048, 64, 4
    w, s, b = random_qweight(rng, 1, N, K, group, bits)
    x = normal_bf16(rng, (M, K))
    args = (dev_u32(w[0]), dev_bf16(s[0]), dev_bf16(b[0]), group, bits)
    xd = dev_bf16(x)
    want = O.qmm(x, w[0], s[0], b[0], group, bits)

    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    q.qmoe_debug_skip_stage(0)
    t0 = time.time()
    q.qmoe_qmm(xd, *args, status=status)
    torch.cuda.synchronize()
    waited = time.time() - t0
    assert int(status.item()) & q.QMOE_DEV_TIMEOUT, "the skipped stage's wait did not run out"
    assert waited < 60.0

    status2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = q.qmoe_qmm(xd, *args, status=status2)
    torch.cuda.synchronize()
    assert int(status2.item()) == 0
    assert_close("qmm after a timed-out launch", y, want)


def test_broken_sorted_promise_is_flagged_and_result_unchanged(gpu_lib):
    q = gpu_lib
    rng = np.random.default_rng(9)
    E, N, K, group, bits, B = 8, 64, 256, 64, 4, 40
    w, s, b = random_qweight(rng, E, N, K, group, bits)
    x = normal_bf16(rng, (B, 1, K))
    W = (dev_u32(w), dev_bf16(s), dev_bf16(b))
    ids = rng.integers(0, E, size=B).astype(np.uint32)
    for rhs, broken in ((np.sort(ids), False), (ids, True)):
        assert broken == bool(np.any(np.diff(rhs.astype(np.int64)) < 0))
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        y = q.qmoe_gather_qmm(dev_bf16(x), *W, None, dev_u32(rhs), group, bits,
                              sorted_indices=True, status=status)
        torch.cuda.synchronize()
        assert bool(int(status.item()) & q.QMOE_DEV_UNSORTED) == broken
        assert_close("gather_qmm with a sorted promise", y,
                     O.gather_qmm(x, w, s, b, group, bits, None, rhs))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    q.qmoe_gather_qmm(dev_bf16(x), *W, None, dev_u32(ids), group, bits, sorted_indices=False,
                      status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0  # no promise, nothing to flag
