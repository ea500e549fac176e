"""qmoe_gather_qmm_noalloc: gather_qmm without any device allocation.

It exists for callers that cannot allocate device memory or pass a workspace (a
plugin handed only its input and output tensors by a framework that owns all device
memory; a serving loop that must not call cudaMalloc between requests).  It keeps
its routing metadata in a fixed array inside the library, so its results must match
the ordinary, workspace-based qmoe_gather_qmm, including on back-to-back calls that
reuse that array.  This file sorts last so that a run stopping at the first failure
has already run every other test."""

import ctypes

import numpy as np
import pytest
import torch

import quantized_moe_expert_gather_b200 as q
from gpu_util import assert_close, dev_bf16, dev_u32
from inputs import distinct_sorted_experts, normal_bf16, random_qweight


def test_noalloc_rejects_problems_beyond_its_capacity():
    lib = q.load()
    fake = 1 << 20  # never dereferenced: the size check fails first
    too_many_rows = lib.qmoe_gather_qmm_noalloc(fake, 4097, 1, 64, fake, fake, fake, 8, 16, 64,
                                                4, None, fake, 4097, 0, fake, None, None)
    too_many_experts = lib.qmoe_gather_qmm_noalloc(fake, 4, 1, 64, fake, fake, fake, 1025, 16,
                                                   64, 4, None, fake, 4, 0, fake, None, None)
    assert too_many_rows == too_many_experts == -6
    assert "QMOE_ERR_TOO_LARGE" in q.qmoe_status_string(-6)


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_consecutive_calls(gpu_lib):
    rng = np.random.default_rng(77)
    E, N, K, group, bits = 64, 512, 1024, 64, 4
    w, s, b = random_qweight(rng, E, N, K, group, bits)
    W = (dev_u32(w), dev_bf16(s), dev_bf16(b))
    for call, T in enumerate((4, 16)):          # two calls in a row, different routings
        x = dev_bf16(normal_bf16(rng, (T, 1, K)))
        rhs = dev_u32(distinct_sorted_experts(rng, T, E, 8).reshape(-1))
        want = gpu_lib.qmoe_gather_qmm(x, *W, None, rhs, group, bits)
        out = torch.empty_like(want)
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        got = gpu_lib.qmoe_gather_qmm_noalloc(x, *W, None, rhs, group, bits, out=out,
                                              status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert_close(f"noalloc call {call}", got, want.float().cpu().numpy())
