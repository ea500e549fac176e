"""Seeded synthetic inputs shared by the oracle tests, the GPU parity tests and
bench.py.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no quantisation, no matmul, no routing maths beyond drawing
indices).  Every array is host numpy; bf16 tensors are uint16 bit patterns, made
by truncating-free round-to-nearest-even of float32 draws (a plain bit operation
written out here, so this module imports nothing from the oracle or the library).

Workloads (shapes and distributions of the pages' benchmarks):

* ``tiny_gather``   E=8, W [8, 256, 512] 4-bit g64, x [4, 512], top-2 experts.
* ``decode_layer``  SwitchGLU decode: hidden 4096, intermediate 2048, E=288, top-8,
                    4-bit g64, M tokens with 8 distinct sorted experts each
                    (MLX issue #4509 repro script).
* ``dense_layer``   decoder-block projections of hidden 2560 (Qwen3-4B shapes of
                    MLX PR #4787's chained benchmark), W ~ N(0,1)/sqrt(K) in bf16.
* ``prefill_routing`` top-8 of a softmax over N(0,1) gating logits plus a
                    per-expert Zipf(1.1) popularity offset (skewed expert loads).
"""

from __future__ import annotations

import numpy as np


def bf16_bits(f: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round-to-nearest-even (inputs are finite)."""
    u = np.ascontiguousarray(np.asarray(f, np.float32)).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    return (((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)) & np.uint64(0xFFFF)).astype(np.uint16)


def random_qweight(rng: np.random.Generator, E: int, N: int, K: int, group: int, bits: int):
    """Packed codes uniform over [0, 2^bits), bf16 scales ~ U(0.005, 0.02) and
    biases ~ U(-0.1, 0.1).  Codes are drawn as 32-bit words: every bit pattern of a
    word is a valid set of codes, so uniform words give uniform codes."""
    words = rng.integers(0, 1 << 32, size=(E, N, K * bits // 32), dtype=np.uint32)
    s = bf16_bits(rng.uniform(0.005, 0.02, size=(E, N, K // group)).astype(np.float32))
    b = bf16_bits(rng.uniform(-0.1, 0.1, size=(E, N, K // group)).astype(np.float32))
    return words, s, b


def normal_bf16(rng: np.random.Generator, shape, scale: float = 1.0) -> np.ndarray:
    return bf16_bits((rng.standard_normal(size=shape) * scale).astype(np.float32))


def distinct_sorted_experts(rng: np.random.Generator, T: int, E: int, top_k: int) -> np.ndarray:
    """Each token draws ``top_k`` distinct experts uniformly, sorted ascending
    (the decode repro's ``sorted(random.sample(range(E), TOPK))``)."""
    out = np.empty((T, top_k), np.uint32)
    for t in range(T):
        out[t] = np.sort(rng.choice(E, size=top_k, replace=False))
    return out


def tiny_gather(seed: int = 0):
    rng = np.random.default_rng(seed)
    E, N, K, group, bits = 8, 256, 512, 64, 4
    w, s, b = random_qweight(rng, E, N, K, group, bits)
    x = normal_bf16(rng, (4, K))
    idx = np.empty((4, 2), np.uint32)
    for t in range(4):
        idx[t] = rng.choice(E, size=2, replace=False)
    return dict(E=E, N=N, K=K, group=group, bits=bits, w=w, s=s, b=b, x=x, idx=idx)


DECODE = dict(H=4096, I=2048, E=288, top_k=8, group=64, bits=4)


def decode_weights(seed: int = 0, H=4096, I=2048, E=288, group=64, bits=4):
    rng = np.random.default_rng(seed)
    up = random_qweight(rng, E, I, H, group, bits)
    gate = random_qweight(rng, E, I, H, group, bits)
    down = random_qweight(rng, E, H, I, group, bits)
    return up, gate, down


def decode_tokens(seed: int, M: int, H=4096, E=288, top_k=8):
    rng = np.random.default_rng(1000 + seed)
    x = normal_bf16(rng, (M, H))
    idx = distinct_sorted_experts(rng, M, E, top_k)
    return x, idx


def decode_scores(seed: int, M: int, top_k=8):
    """Positive combine weights per token summing to 1 (the decode repro has no
    router; any normalised scores serve the combine)."""
    rng = np.random.default_rng(2000 + seed)
    w = rng.random((M, top_k)).astype(np.float32) + np.float32(0.05)
    return (w / w.sum(axis=1, keepdims=True)).astype(np.float32)


DENSE = dict(hidden=2560, q_out=4096, kv_out=1024, inter=9728, layers=36, sets=8)


def dense_projections(hidden=2560, q_out=4096, kv_out=1024, inter=9728):
    """(name, N, K) of the decoder-block projections (MLX PR #4787 script)."""
    return [("q", q_out, hidden), ("k", kv_out, hidden), ("v", kv_out, hidden),
            ("o", hidden, q_out), ("g", inter, hidden), ("u", inter, hidden),
            ("dn", hidden, inter)]


def dense_weight_f32(rng: np.random.Generator, N: int, K: int) -> np.ndarray:
    """W = N(0,1)/sqrt(K) rounded to bf16, returned as float32 values."""
    w = (rng.standard_normal(size=(N, K)) / np.sqrt(K)).astype(np.float32)
    return (bf16_bits(w).astype(np.uint32) << np.uint32(16)).view(np.float32)


PREFILL = dict(H=2048, I=512, E=256, top_k=8, group=64, bits=4)


def prefill_routing(seed: int, T: int, E: int = 256, top_k: int = 8, zipf_a: float = 1.1):
    """Routing of the prefill workloads.

    logit[t, e] = N(0,1) - zipf_a * ln(rank[e]) where ``rank`` is a seeded
    permutation of 1..E (a Zipf popularity prior); scores are the float32 softmax
    over all E, and each token keeps its ``top_k`` largest probabilities (not
    renormalised).  Returns ``(idx uint32 [T, top_k], scores float32 [T, top_k])``.
    """
    rng = np.random.default_rng(seed)
    rank = rng.permutation(E) + 1
    logits = rng.standard_normal(size=(T, E)) - zipf_a * np.log(rank)[None, :]
    logits = logits.astype(np.float32)
    z = logits - logits.max(axis=1, keepdims=True)
    p = np.exp(z)
    p = (p / p.sum(axis=1, keepdims=True)).astype(np.float32)
    idx = np.argsort(-p, axis=1, kind="stable")[:, :top_k].astype(np.uint32)
    scores = np.take_along_axis(p, idx.astype(np.int64), axis=1).astype(np.float32)
    return idx, scores


def prefill_layer(seed: int, T: int, H=2048, I=512, E=256, top_k=8, group=64, bits=4,
                  shared: bool = False):
    """Routed-expert weights, activations and routing for the prefill workloads;
    with ``shared`` also a shared SwiGLU expert (E=1, intermediate I) and a bf16
    shared-gate vector."""
    rng = np.random.default_rng(10_000 + seed)
    up = random_qweight(rng, E, I, H, group, bits)
    gate = random_qweight(rng, E, I, H, group, bits)
    down = random_qweight(rng, E, H, I, group, bits)
    x = normal_bf16(rng, (T, H))
    idx, scores = prefill_routing(seed, T, E, top_k)
    out = dict(up=up, gate=gate, down=down, x=x, idx=idx, scores=scores,
               H=H, I=I, E=E, top_k=top_k, group=group, bits=bits)
    if shared:
        out["sh_up"] = random_qweight(rng, 1, I, H, group, bits)
        out["sh_gate"] = random_qweight(rng, 1, I, H, group, bits)
        out["sh_down"] = random_qweight(rng, 1, H, I, group, bits)
        out["w_sg"] = normal_bf16(rng, (H,), scale=1.0 / np.sqrt(H))
    return out
