"""The device-side launch timing hook records one slot per launch, eagerly and
inside a captured CUDA graph."""

import numpy as np
import pytest
import torch

from gpu_util import dev_bf16, dev_u32
from inputs import normal_bf16, random_qweight

pytestmark = pytest.mark.gpu


def test_timing_slots_eager_and_graph(gpu_lib):
    q = gpu_lib
    rng = np.random.default_rng(0)
    w, s, b = random_qweight(rng, 1, 4096, 4096, 64, 4)
    args = (dev_u32(w[0]), dev_bf16(s[0]), dev_bf16(b[0]), 64, 4)
    x = dev_bf16(normal_bf16(rng, (4, 4096)))
    y = torch.empty((4, 4096), dtype=torch.bfloat16, device="cuda")
    slots = torch.zeros(16 * 8, dtype=torch.uint8, device="cuda")
    q.qmoe_qmm(x, *args, out=y)          # eager warm-up outside timing
    torch.cuda.synchronize()
    q.qmoe_timing_enable(slots)
    try:
        q.qmoe_qmm(x, *args, out=y)
        torch.cuda.synchronize()
        ms, n = q.qmoe_timing_read("qmv")
        assert n == 1 and 0.0 < ms < 50.0
        assert q.qmoe_timing_read("combine") == (0.0, 0)
        q.qmoe_timing_enable(slots)       # clears the records
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            q.qmoe_qmm(x, *args, out=y)
        for _ in range(2):
            g.replay()
            torch.cuda.synchronize()
            ms, n = q.qmoe_timing_read("qmv")
            assert n == 1 and 0.0 < ms < 50.0
    finally:
        q.qmoe_timing_enable(None)


def test_forced_kernels_really_run(gpu_lib, monkeypatch):
    """QMOE_FORCE_KERNEL selects the streaming or a tensor-core kernel (QMOE_PREFILL=tc
    picks the one that stages weights in shared memory over the one that keeps them in
    tensor memory): the launch records prove which one ran (so the parity tests cover
    each)."""
    q = gpu_lib
    rng = np.random.default_rng(3)
    w, s, b = random_qweight(rng, 1, 256, 512, 64, 4)
    args = (dev_u32(w[0]), dev_bf16(s[0]), dev_bf16(b[0]), 64, 4)
    x = dev_bf16(normal_bf16(rng, (200, 512)))
    slots = torch.zeros(16 * 8, dtype=torch.uint8, device="cuda")
    for forced, prefill, name in (("qmv", None, "qmv"), ("tc", None, "ts"), ("tc", "tc", "tc")):
        monkeypatch.setenv("QMOE_FORCE_KERNEL", forced)
        if prefill is None:
            monkeypatch.delenv("QMOE_PREFILL", raising=False)
        else:
            monkeypatch.setenv("QMOE_PREFILL", prefill)
        q.qmoe_qmm(x, *args)  # warm-up outside timing
        torch.cuda.synchronize()
        q.qmoe_timing_enable(slots)
        try:
            q.qmoe_qmm(x, *args)
            torch.cuda.synchronize()
            assert q.qmoe_timing_read(name)[1] == 1, forced
        finally:
            q.qmoe_timing_enable(None)
