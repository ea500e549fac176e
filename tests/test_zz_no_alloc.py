"""qmoe_gather_qmm_noalloc: gather_qmm without any device allocation.

It exists for callers that cannot allocate device memory or pass a workspace (a
plugin handed only its input and output tensors by a framework that owns all device
memory; a serving loop that must not call cudaMalloc between requests).  It keeps
its routing metadata in a fixed array inside the library.  Its results are checked
against the oracle and against the ordinary, workspace-based qmoe_gather_qmm,
on back-to-back calls that reuse that array, up to the array's capacity (4096
routed rows over 1024 experts, where the routing runs its multi-chunk path).
This file sorts last so that a run stopping at the first failure has already run
every other test."""

import numpy as np
import pytest
import torch

import oracle as O
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
    two_bit = lib.qmoe_gather_qmm_noalloc(fake, 4, 1, 64, fake, fake, fake, 8, 16, 64,
                                          2, None, fake, 4, 0, fake, None, None)
    assert too_many_rows == too_many_experts == -6
    assert two_bit == -3  # 4- and 8-bit codes only
    assert "QMOE_ERR_TOO_LARGE" in q.qmoe_status_string(-6)


def _case(rng, E, N, K, group, bits, T, top_k, lhs_perm, unsorted):
    """(x [T,1,K], weights, lhs or None, rhs): top_k distinct experts per token."""
    w, s, b = random_qweight(rng, E, N, K, group, bits)
    x = normal_bf16(rng, (T, 1, K))
    rhs = distinct_sorted_experts(rng, T, E, top_k).reshape(-1)
    lhs = None
    if lhs_perm:  # explicit lhs: batch b reads token b // top_k, batches shuffled
        perm = rng.permutation(rhs.size)
        lhs = (np.arange(rhs.size) // top_k)[perm].astype(np.uint32)
        rhs = rhs[perm]
    elif unsorted:
        rhs = rhs[rng.permutation(rhs.size)]
    return x, (w, s, b), lhs, rhs.astype(np.uint32)


# (E, N, K, group, bits, T, top_k, explicit lhs, unsorted rhs)
CASES = [
    (64, 512, 1024, 64, 4, 4, 8, False, False),
    (1024, 64, 512, 64, 4, 512, 8, False, True),      # 4096 routed rows, 1024 experts
    (48, 256, 1024, 128, 8, 37, 8, True, True),       # 8-bit group 128, explicit lhs
    (16, 128, 256, 32, 4, 300, 2, False, True),       # several rows per expert
]


@pytest.mark.gpu
def test_noalloc_matches_oracle_and_workspace_entry_point_on_consecutive_calls(gpu_lib):
    rng = np.random.default_rng(77)
    for call, (E, N, K, group, bits, T, top_k, lhs_perm, unsorted) in enumerate(CASES):
        x, (w, s, b), lhs, rhs = _case(rng, E, N, K, group, bits, T, top_k, lhs_perm, unsorted)
        B = rhs.size
        xd, W = dev_bf16(x), (dev_u32(w), dev_bf16(s), dev_bf16(b))
        lhs_d = None if lhs is None else dev_u32(lhs)
        rhs_d = dev_u32(rhs)
        out = torch.empty((B, 1, N), dtype=torch.bfloat16, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        got = gpu_lib.qmoe_gather_qmm_noalloc(xd, *W, lhs_d, rhs_d, group, bits, out=out,
                                              status=status)
        ref = gpu_lib.qmoe_gather_qmm(xd, *W, lhs_d, rhs_d, group, bits)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, f"call {call}: device status {int(status.item())}"
        want = O.gather_qmm(x, w, s, b, group, bits, lhs, rhs)
        assert_close(f"noalloc call {call} vs oracle", got, want)
        assert_close(f"noalloc call {call} vs qmoe_gather_qmm", got, ref.float().cpu().numpy())
