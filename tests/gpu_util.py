"""Helpers of the GPU parity tests: host<->device copies of the seeded inputs and the
comparison rule.  No arithmetic of the method lives here."""

import numpy as np
import torch

TOL = 8e-3  # |got - want| <= TOL * max|want| for bf16 outputs with fp32 accumulation


def dev_u32(a):
    """uint32 numpy -> int32 CUDA tensor holding the same bits."""
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int32)).cuda()


def dev_bf16(a):
    """bf16 bit patterns (uint16 numpy) -> torch.bfloat16 CUDA tensor."""
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


def dev_f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def host_bits16(t):
    """torch.bfloat16 tensor -> uint16 numpy bit patterns."""
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def host_u32(t):
    return t.detach().cpu().numpy().view(np.uint32)


def host_f32_from_bf16(t):
    return t.detach().float().cpu().numpy()


def assert_close(name, got_bf16, want, tol=TOL):
    got = host_f32_from_bf16(got_bf16).astype(np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, f"{name}: shape {got.shape} vs {want.shape}"
    scale = float(np.max(np.abs(want))) if want.size else 0.0
    err = np.abs(got - want)
    worst = float(err.max()) if err.size else 0.0
    assert np.all(np.isfinite(got)), f"{name}: non-finite output"
    assert worst <= tol * scale + 1e-30, (
        f"{name}: max |got-want| = {worst:.4g} > {tol} * {scale:.4g}")
    return worst / scale if scale else 0.0


def qweight(w, s, b, group, bits):
    """Device copies of a packed weight stack for the binding's QWeight."""
    import quantized_moe_expert_gather_b200 as q
    return q.QWeight(dev_u32(w), dev_bf16(s), dev_bf16(b), group, bits)


def select_experts(wt, experts):
    """Host slice of the given experts of a (codes, scales, biases) stack: input
    selection for the oracle, so it only dequantises what the routing touches."""
    w, s, b = wt
    return w[experts], s[experts], b[experts]
