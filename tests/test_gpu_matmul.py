"""GPU parity of the floating-point steps against the fp64 oracle:
|got - want| <= 8e-3 * max|want| for bf16 outputs with fp32 accumulation.

Covers qmm (dense, the decoder-block shapes and the kernel-coverage shapes of
nuvec-core 0.4.0 tests/quantized.rs), gather_qmm (explicit and default indices,
sorted and unsorted, bad indices), SwitchGLU (decode and prefill workloads, both
output modes) and the one-pass combine."""

import os

import numpy as np
import pytest
import torch

import oracle as O
from gpu_util import (assert_close, dev_bf16, dev_f32, dev_u32, host_bits16, host_u32,
                      qweight, select_experts)
from inputs import (bf16_bits, decode_tokens, decode_weights, dense_projections,
                    dense_weight_f32, normal_bf16, prefill_layer, prefill_routing, random_qweight,
                    tiny_gather)

pytestmark = pytest.mark.gpu


@pytest.fixture(params=["qmv", "tc", "tc_smem", "auto"])
def kernel(request, monkeypatch):
    """Kernel choice: forced streaming, forced tensor-core tiles (weights in tensor
    memory where the shape allows, or staged in shared memory), or the library's own
    plan (chosen from the most rows one expert can receive)."""
    monkeypatch.delenv("QMOE_PREFILL", raising=False)
    if request.param == "auto":
        monkeypatch.delenv("QMOE_FORCE_KERNEL", raising=False)
    elif request.param == "tc_smem":
        monkeypatch.setenv("QMOE_FORCE_KERNEL", "tc")
        monkeypatch.setenv("QMOE_PREFILL", "tc")
    else:
        monkeypatch.setenv("QMOE_FORCE_KERNEL", request.param)
    return request.param


# ------------------------------------------------------------------------- qmm
QMM_CASES = [  # (M, N, K, bits, group)
    (1, 64, 512, 4, 64), (5, 64, 512, 4, 64), (4, 36, 1024, 4, 32), (8, 16, 512, 4, 128),
    (3, 36, 1024, 4, 32), (1, 13, 96, 8, 32), (4, 24, 256, 8, 128), (40, 64, 256, 4, 64),
    (33, 50, 128, 8, 32), (64, 96, 4096, 4, 128), (16, 40, 64, 4, 64), (2, 1, 128, 8, 64),
    (17, 300, 640, 4, 64), (130, 256, 512, 4, 64), (300, 384, 1024, 8, 64),
    # tensor-memory kernel edges: N not a multiple of 8 (element stores), several
    # 192-row tiles with a ragged last one (TMA-stored full pieces), groups 32 and 128
    (40, 37, 512, 4, 64), (200, 128, 1024, 4, 32), (400, 136, 2048, 4, 128),
    # 2-bit codes (streaming kernel, one and two token sets, groups 64 and 128)
    (1, 64, 512, 2, 64), (5, 96, 1024, 2, 128), (12, 64, 512, 2, 64), (40, 37, 1024, 2, 128),
]


@pytest.mark.parametrize("M,N,K,bits,group", QMM_CASES)
def test_qmm_matches_oracle(gpu_lib, kernel, M, N, K, bits, group):
    q = gpu_lib
    rng = np.random.default_rng(M * 7 + N + K + bits)
    w, s, b = random_qweight(rng, 1, N, K, group, bits)
    x = normal_bf16(rng, (M, K))
    want = O.qmm(x, w[0], s[0], b[0], group, bits)
    y = q.qmoe_qmm(dev_bf16(x), dev_u32(w[0]), dev_bf16(s[0]), dev_bf16(b[0]), group, bits)
    torch.cuda.synchronize()
    assert_close(f"qmm {M}x{N}x{K} {bits}/{group}", y, want)


@pytest.mark.parametrize("bits", [4, 8])
def test_qmm_decoder_block_shapes(gpu_lib, bits):
    """Hidden 2560 projections (q/k/v/o/gate/up/down) at every row count of the
    small-M benchmark, W = N(0,1)/sqrt(K) quantised on the GPU."""
    q = gpu_lib
    rng = np.random.default_rng(bits)
    for name, N, K in dense_projections():
        wb16 = bf16_bits(dense_weight_f32(rng, N, K))
        wc, ws, wb = O.quantize(O.f32_from_bf16(wb16), 64, bits)   # oracle-quantised weights
        codes, s, b = dev_u32(wc), dev_bf16(ws), dev_bf16(wb)
        rows = np.arange(0, N, max(1, N // 512))                     # sampled output channels
        for M in (1, 2, 3, 4, 5, 6, 7, 8, 10, 12, 16):
            x = normal_bf16(rng, (M, K))
            y = q.qmoe_qmm(dev_bf16(x), codes, s, b, 64, bits)
            want = O.qmm(x, wc[rows], ws[rows], wb[rows], 64, bits)
            assert_close(f"{name} M={M}", y[:, torch.from_numpy(rows).cuda()], want)


def test_qmm_few_rows_equal_one_row_bitwise(gpu_lib):
    """nuvec-core quantized.rs few_row_products_equal_one_row_products_bit_for_bit:
    each row of a few-row product equals that row's one-row product."""
    q = gpu_lib
    rng = np.random.default_rng(1)
    for M, K, N, group in [(6, 4096, 512, 64), (5, 1024, 1000, 32), (4, 2048, 256, 128)]:
        w, s, b = random_qweight(rng, 1, N, K, group, 4)
        x = dev_bf16(normal_bf16(rng, (M, K)))
        args = (dev_u32(w[0]), dev_bf16(s[0]), dev_bf16(b[0]), group, 4)
        allr = host_bits16(q.qmoe_qmm(x, *args))
        for r in range(M):
            one = host_bits16(q.qmoe_qmm(x[r:r + 1].contiguous(), *args))
            assert np.array_equal(one[0], allr[r]), (M, K, N, group, r)


@pytest.mark.parametrize("plan", ["tmem", "smem"])
def test_prefill_kernels_row_bits_independent_of_tile_companions(gpu_lib, monkeypatch, plan):
    """The invariant lane of MTPLX PR #558 (Summary) asks that a row's result not depend
    on the batch it runs in; nuvec-core quantized.rs few_row_products_equal_one_row_
    products_bit_for_bit states it for the few-row kernels.  On the tensor-core kernels
    (forced, weights in tensor memory or staged in shared memory) a row's output bits
    are the same alone in its tile, among 17 or 100 rows, and in a full 192-row tile,
    at any position; for the dense product and the SwitchGLU chain."""
    q = gpu_lib
    monkeypatch.setenv("QMOE_FORCE_KERNEL", "tc")
    if plan == "smem":
        monkeypatch.setenv("QMOE_PREFILL", "tc")
    else:
        monkeypatch.delenv("QMOE_PREFILL", raising=False)
    rng = np.random.default_rng(31)
    for bits, group, N, K in ((4, 64, 256, 2048), (8, 128, 136, 1024)):
        w, s, b = random_qweight(rng, 1, N, K, group, bits)
        args = (dev_u32(w[0]), dev_bf16(s[0]), dev_bf16(b[0]), group, bits)
        X = normal_bf16(rng, (192, K))
        full = host_bits16(q.qmoe_qmm(dev_bf16(X), *args))
        for n in (1, 17, 100):
            rows = rng.choice(192, size=n, replace=False)
            sub = host_bits16(q.qmoe_qmm(dev_bf16(X[rows]), *args))
            assert np.array_equal(sub, full[rows]), (plan, bits, n)
    # SwitchGLU (fused up/gate + silu*mul, then down): a token's output bits with the
    # other tokens of the call removed
    E, H, I, T, top_k = 4, 512, 256, 160, 2
    up, gate, down = (random_qweight(rng, E, nn, kk, 64, 4) for nn, kk in ((I, H), (I, H), (H, I)))
    W = [qweight(*t, 64, 4) for t in (up, gate, down)]
    x = normal_bf16(rng, (T, H))
    idx = np.stack([rng.choice(E, size=top_k, replace=False) for _ in range(T)]).astype(np.uint32)
    full = host_bits16(q.qmoe_switch_glu(dev_bf16(x), dev_u32(idx), *W, mode=0))
    for n in (1, 33):
        toks = np.sort(rng.choice(T, size=n, replace=False))
        sub = host_bits16(q.qmoe_switch_glu(dev_bf16(x[toks]), dev_u32(idx[toks]), *W, mode=0))
        assert np.array_equal(sub, full[toks]), (plan, "switch_glu", n)


# bit-stream widths (1, 3, 5, 6 bits; 2 bits in groups of 32): the CUDA-core kernel
BITSTREAM_QMM = [  # (M, N, K, bits, group)
    (1, 64, 512, 3, 64), (5, 33, 256, 5, 32), (17, 40, 384, 6, 128), (3, 64, 256, 1, 64),
    (4, 48, 320, 2, 32), (40, 37, 512, 3, 32), (2, 16, 1024, 6, 64), (9, 24, 128, 5, 128),
]


@pytest.mark.parametrize("M,N,K,bits,group", BITSTREAM_QMM)
def test_qmm_bitstream_widths(gpu_lib, M, N, K, bits, group):
    """quantized_matmul over the widths of nuvec-core quantized.rs `const BITS` whose codes
    straddle words (3, 5, 6) or have no MMA kernel here (1; 2 in groups of 32): ragged N,
    several 16-row tiles."""
    q = gpu_lib
    rng = np.random.default_rng(M * 11 + N + K + bits)
    w, s, b = random_qweight(rng, 1, N, K, group, bits)
    x = normal_bf16(rng, (M, K))
    want = O.qmm(x, w[0], s[0], b[0], group, bits)
    y = q.qmoe_qmm(dev_bf16(x), dev_u32(w[0]), dev_bf16(s[0]), dev_bf16(b[0]), group, bits)
    assert_close(f"qmm {M}x{N}x{K} {bits}-bit g{group}", y, want)


@pytest.mark.parametrize("bits,group", [(1, 32), (2, 32), (3, 64), (5, 128), (6, 32)])
def test_gather_qmm_bitstream_widths(gpu_lib, bits, group):
    """gather_qmm over the bit-stream widths: sorted and unsorted indices give the same
    bits; rows of one x batch broadcast over its experts."""
    q = gpu_lib
    rng = np.random.default_rng(bits * 7 + group)
    E, N, K = 8, 48, 256
    w, s, b = random_qweight(rng, E, N, K, group, bits)
    x = normal_bf16(rng, (12, 1, K))
    rhs = np.stack([rng.choice(E, size=3, replace=False) for _ in range(12)]).reshape(-1)
    rhs = rhs.astype(np.uint32)
    W = (dev_u32(w), dev_bf16(s), dev_bf16(b))
    want = O.gather_qmm(x, w, s, b, group, bits, None, rhs)
    y = q.qmoe_gather_qmm(dev_bf16(x), *W, None, dev_u32(rhs), group, bits)
    assert_close(f"gather {bits}-bit g{group}", y, want)
    perm = np.argsort(rhs, kind="stable")
    lhs = (np.arange(rhs.size) // 3)[perm].astype(np.uint32)
    ys = q.qmoe_gather_qmm(dev_bf16(x), *W, dev_u32(lhs), dev_u32(rhs[perm]), group, bits,
                           sorted_indices=True)
    assert np.array_equal(host_bits16(ys), host_bits16(y)[perm])


@pytest.mark.parametrize("T,bits,group", [(4, 3, 64), (64, 5, 32), (24, 6, 128), (8, 1, 64)])
def test_switch_glu_bitstream_widths(gpu_lib, T, bits, group):
    """SwitchGLU with bit-stream codes (fused up/gate + silu*mul, then down), decode- and
    prefill-sized rows per expert."""
    q = gpu_lib
    rng = np.random.default_rng(T + bits + group)
    E, H, I, top_k = 8, 512, 256, 2
    up, gate, down = (random_qweight(rng, E, n, k, group, bits) for n, k in ((I, H), (I, H), (H, I)))
    x = normal_bf16(rng, (T, H))
    idx = np.stack([rng.choice(E, size=top_k, replace=False) for _ in range(T)]).astype(np.uint32)
    W = [qweight(*t, group, bits) for t in (up, gate, down)]
    y = q.qmoe_switch_glu(dev_bf16(x), dev_u32(idx), *W, mode=0)
    want, _ = O.switch_glu(x, idx, (*up, group, bits), (*gate, group, bits), (*down, group, bits))
    assert_close(f"switch_glu {bits}-bit g{group} T={T}", y, want)


def test_qmm_empty(gpu_lib):
    q = gpu_lib
    x = torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((16, 8), dtype=torch.int32, device="cuda")
    s = torch.zeros((16, 1), dtype=torch.bfloat16, device="cuda")
    y = q.qmoe_qmm(x, w, s, s.clone(), 64, 4)
    assert tuple(y.shape) == (0, 16)


# ------------------------------------------------------------------- gather_qmm
def test_tiny_gather_sorted_and_unsorted(gpu_lib, kernel):
    q = gpu_lib
    d = tiny_gather(0)
    T, K = d["x"].shape
    x3 = d["x"].reshape(T, 1, K)
    rhs = d["idx"].reshape(-1)
    want = O.gather_qmm(x3, d["w"], d["s"], d["b"], d["group"], d["bits"], None, rhs)
    args = (dev_u32(d["w"]), dev_bf16(d["s"]), dev_bf16(d["b"]))
    y = q.qmoe_gather_qmm(dev_bf16(x3), *args, None, dev_u32(rhs), d["group"], d["bits"])
    assert_close("tiny unsorted", y.reshape(T, 2, -1), want.reshape(T, 2, -1))
    perm = np.argsort(rhs, kind="stable")
    lhs = (np.arange(rhs.size) // 2)[perm].astype(np.uint32)
    ys = q.qmoe_gather_qmm(dev_bf16(x3), *args, dev_u32(lhs), dev_u32(rhs[perm]), d["group"],
                           d["bits"], sorted_indices=True)
    assert np.array_equal(host_bits16(ys), host_bits16(y)[perm])


GATHER_CASES = [  # (E, N, K, M, batches, sorted, bits, group)
    (8, 64, 512, 1, 6, False, 4, 64), (8, 36, 192, 1, 5, False, 4, 32),
    (4, 64, 256, 40, 3, False, 4, 64), (4, 40, 128, 33, 2, False, 8, 32),
    (8, 64, 256, 1, 100, True, 4, 64), (8, 64, 256, 1, 20, True, 8, 128),
    (16, 48, 192, 1, 70, True, 4, 32), (32, 128, 1024, 2, 300, False, 4, 64),
    (8, 64, 512, 1, 20, False, 2, 64), (4, 48, 1024, 3, 30, True, 2, 128),
]


@pytest.mark.parametrize("E,N,K,M,batches,sorted_,bits,group", GATHER_CASES)
def test_gather_qmm_matches_oracle(gpu_lib, kernel, E, N, K, M, batches, sorted_, bits, group):
    q = gpu_lib
    rng = np.random.default_rng(E + N + K + M + batches)
    w, s, b = random_qweight(rng, E, N, K, group, bits)
    x = normal_bf16(rng, (batches, M, K))
    ids = np.array([(i * 7 + 3) % E for i in range(batches)], np.uint32)
    if sorted_:
        ids.sort()
    want = O.gather_qmm(x, w, s, b, group, bits, None, ids)
    y = q.qmoe_gather_qmm(dev_bf16(x), dev_u32(w), dev_bf16(s), dev_bf16(b), None, dev_u32(ids),
                          group, bits, sorted_indices=sorted_)
    assert_close("gather", y, want)


def test_gather_qmm_explicit_and_default_indices(gpu_lib):
    q = gpu_lib
    rng = np.random.default_rng(0x71)
    E, N, K, group, bits = 3, 8, 64, 32, 4
    w, s, b = random_qweight(rng, E, N, K, group, bits)
    x = normal_bf16(rng, (4, 2, K))
    lhs, rhs = np.array([3, 0, 2], np.uint32), np.array([1, 2, 0], np.uint32)
    args = (dev_u32(w), dev_bf16(s), dev_bf16(b))
    y = q.qmoe_gather_qmm(dev_bf16(x), *args, dev_u32(lhs), dev_u32(rhs), group, bits)
    assert_close("explicit", y, O.gather_qmm(x, w, s, b, group, bits, lhs, rhs))
    x1 = x[:1, :1]
    y = q.qmoe_gather_qmm(dev_bf16(x1), *args, None, None, group, bits)
    assert_close("default", y, O.gather_qmm(x1, w, s, b, group, bits))


def test_gather_qmm_bad_indices_zero_rows(gpu_lib):
    q = gpu_lib
    rng = np.random.default_rng(5)
    E, N, K, group, bits = 4, 32, 128, 64, 4
    w, s, b = random_qweight(rng, E, N, K, group, bits)
    x = normal_bf16(rng, (3, 1, K))
    rhs = np.array([1, 7, 2, 0, 3, 9], np.uint32)  # 7 and 9 are out of range
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = q.qmoe_gather_qmm(dev_bf16(x), dev_u32(w), dev_bf16(s), dev_bf16(b), None, dev_u32(rhs),
                          group, bits, status=status)
    got = y.float().cpu().numpy()
    ok = rhs < E
    want = O.gather_qmm(x, w, s, b, group, bits, np.arange(6) // 2, np.where(ok, rhs, 0))
    assert np.all(got[~ok] == 0)
    assert_close("valid rows", y[torch.from_numpy(ok).cuda()], want[ok])
    assert int(status.item()) & q.QMOE_DEV_BAD_INDEX


# ------------------------------------------------------------------- switch_glu
def _switch_oracle(x, idx, up, gate, down, group, bits):
    experts = np.unique(idx)
    remap = np.searchsorted(experts, idx)
    sel = lambda wt: (*select_experts(wt, experts), group, bits)
    return O.switch_glu(x, remap, sel(up), sel(gate), sel(down))


def test_switch_glu_decode_rows_bitwise_across_unit_shapes(gpu_lib, monkeypatch):
    """A decode token's SwitchGLU output bits are the same in a 4-token call (the streaming
    kernel's four-block units) as alone (two-block units): MTPLX PR #558, Summary (the
    invariant lane); nuvec-core quantized.rs few_row_products_equal_one_row_products_bit_for_bit."""
    q = gpu_lib
    monkeypatch.setenv("QMOE_FORCE_KERNEL", "qmv")
    up, gate, down = _decode_weights()
    x, idx = decode_tokens(3, 4)
    W = [qweight(*t, 64, 4) for t in (up, gate, down)]
    together = host_bits16(q.qmoe_switch_glu(dev_bf16(x), dev_u32(idx), *W, mode=0))
    for t in range(4):
        alone = host_bits16(q.qmoe_switch_glu(dev_bf16(x[t:t + 1]), dev_u32(idx[t:t + 1]), *W,
                                              mode=0))
        assert np.array_equal(alone[0], together[t]), t


@pytest.mark.parametrize("M", [1, 4])
def test_switch_glu_decode_layer(gpu_lib, kernel, M):
    """Decode layer at full size: hidden 4096, intermediate 2048, E=288, top-8."""
    q = gpu_lib
    up, gate, down = _decode_weights()
    x, idx = decode_tokens(0, M)
    W = [qweight(*t, 64, 4) for t in (up, gate, down)]
    y = q.qmoe_switch_glu(dev_bf16(x), dev_u32(idx), *W, mode=0)
    want, _ = _switch_oracle(x, idx, up, gate, down, 64, 4)
    assert_close(f"decode M={M}", y, want)


_DECODE = {}


def _decode_weights():
    if "w" not in _DECODE:
        _DECODE["w"] = decode_weights(0)
    return _DECODE["w"]


@pytest.mark.parametrize("T,mode", [(64, 0), (512, 1), (713, 0)])
def test_switch_glu_prefill(gpu_lib, kernel, T, mode):
    """Prefill SwitchGLU with Zipf-skewed routing (hidden 2048, intermediate 512,
    E=256, top-8), token-order and expert-sorted outputs."""
    q = gpu_lib
    d = _prefill(T)
    W = [qweight(*d[k], 64, 4) for k in ("up", "gate", "down")]
    want, _ = _switch_oracle(d["x"], d["idx"], d["up"], d["gate"], d["down"], 64, 4)
    if mode == 0:
        y = q.qmoe_switch_glu(dev_bf16(d["x"]), dev_u32(d["idx"]), *W, mode=0)
        assert_close(f"prefill T={T}", y, want)
    else:
        ys, inv = q.qmoe_switch_glu(dev_bf16(d["x"]), dev_u32(d["idx"]), *W, mode=1)
        inv = host_u32(inv)
        _, w_inv, _ = O.sort_by_expert(d["idx"].reshape(-1), d["E"])
        assert np.array_equal(inv, w_inv)
        assert_close(f"prefill sorted T={T}", ys[torch.from_numpy(inv.astype(np.int64)).cuda()],
                     want.reshape(T * d["top_k"], -1))


@pytest.mark.parametrize("T,group", [(4, 64), (24, 128)])
def test_switch_glu_2bit(gpu_lib, T, group):
    """SwitchGLU with 2-bit codes (hidden 512, intermediate 256, 16 experts, top-2):
    the fused up/gate and the down launch on the streaming kernel."""
    q = gpu_lib
    rng = np.random.default_rng(T + group)
    E, H, I, top_k = 16, 512, 256, 2
    up, gate, down = (random_qweight(rng, E, n, k, group, 2) for n, k in ((I, H), (I, H), (H, I)))
    x = normal_bf16(rng, (T, H))
    idx = np.stack([rng.choice(E, size=top_k, replace=False) for _ in range(T)]).astype(np.uint32)
    W = [qweight(*t, group, 2) for t in (up, gate, down)]
    y = q.qmoe_switch_glu(dev_bf16(x), dev_u32(idx), *W, mode=0)
    want, _ = O.switch_glu(x, idx, (*up, group, 2), (*gate, group, 2), (*down, group, 2))
    assert_close(f"switch_glu 2-bit T={T} g{group}", y, want)


@pytest.mark.parametrize("bits", [4, 8])
def test_switch_glu_prefill_rows_of_few_groups(gpu_lib, bits):
    """Prefill SwitchGLU whose up/gate rows (hidden 512, group 128) and down rows
    (intermediate 256) hold fewer than 8 groups: the tensor-memory kernel takes both
    projections' scales and biases by whole-unit bulk copies (two stacks, then one)."""
    q = gpu_lib
    rng = np.random.default_rng(bits)
    E, H, I, T, top_k, group = 4, 512, 256, 96, 2, 128
    up, gate, down = (random_qweight(rng, E, n, k, group, bits) for n, k in ((I, H), (I, H), (H, I)))
    x = normal_bf16(rng, (T, H))
    idx = np.stack([rng.choice(E, size=top_k, replace=False) for _ in range(T)]).astype(np.uint32)
    W = [qweight(*t, group, bits) for t in (up, gate, down)]
    slots = torch.zeros(16 * 16, dtype=torch.uint8, device="cuda")
    q.qmoe_timing_enable(slots)
    try:
        y = q.qmoe_switch_glu(dev_bf16(x), dev_u32(idx), *W, mode=0)
        torch.cuda.synchronize()
        assert q.qmoe_timing_read("ts_glu")[1] == 1 and q.qmoe_timing_read("ts")[1] == 1
    finally:
        q.qmoe_timing_enable(None)
    want, _ = O.switch_glu(x, idx, (*up, group, bits), (*gate, group, bits), (*down, group, bits))
    assert_close(f"switch_glu {bits}-bit g{group} few groups", y, want)


@pytest.mark.parametrize("T", [40, 331])
def test_switch_glu_prefill_8bit_g128(gpu_lib, kernel, T):
    """8-bit group-128 prefill SwitchGLU with Zipf-skewed routing: the down projection's
    rows (K = 512) hold only 4 groups, so on the tensor-core path their scales and
    biases arrive by 1-D bulk copies of whole 128-row blocks."""
    q = gpu_lib
    d = prefill_layer(2, T, group=128, bits=8)
    W = [qweight(*d[k], 128, 8) for k in ("up", "gate", "down")]
    want, _ = _switch_oracle(d["x"], d["idx"], d["up"], d["gate"], d["down"], 128, 8)
    y = q.qmoe_switch_glu(dev_bf16(d["x"]), dev_u32(d["idx"]), *W, mode=0)
    assert_close(f"prefill 8-bit g128 T={T}", y, want)


_PREFILL = {}


def _prefill(T):
    if T not in _PREFILL:
        _PREFILL[T] = prefill_layer(0, T)
    return _PREFILL[T]


# ------------------------------------------------------------------- gather_mm
GATHER_MM_CASES = [  # (x_batches, M, K, E, N, B)
    (300, 1, 512, 8, 200, 300),   # rows across three 128-row tiles; N not a multiple of 128
    (40, 1, 256, 5, 384, 320),    # x broadcast over 8 experts per token
    (3, 7, 128, 4, 64, 3),        # several rows per batch, one tile
    (1000, 1, 256, 3, 136, 1000), # several 128-row tiles per expert with ragged tails
    (50, 2, 192, 6, 128, 50),     # K of three 64-k stages
]


@pytest.mark.parametrize("xb,M,K,E,N,B", GATHER_MM_CASES)
def test_gather_mm(gpu_lib, xb, M, K, E, N, B):
    """Unquantized gather_mm on the tensor-core kernel (no dequant stage) against the
    oracle; sorted and unsorted indices give the same bits."""
    q = gpu_lib
    rng = np.random.default_rng(1000 + K + N)
    w = normal_bf16(rng, (E, N, K), 1 / np.sqrt(K))
    x = normal_bf16(rng, (xb, M, K))
    rhs = rng.integers(0, E, size=B).astype(np.uint32)
    lhs = None if xb != B else rng.permutation(B).astype(np.uint32)
    want = O.gather_mm(x, w, lhs, rhs)
    got = q.qmoe_gather_mm(dev_bf16(x), dev_bf16(w), None if lhs is None else dev_u32(lhs),
                           dev_u32(rhs))
    assert_close(f"gather_mm {xb}x{M}x{K} E={E} N={N} B={B}", got, want)
    if lhs is None:
        lhs_b = ((np.arange(B) * xb) // B).astype(np.uint32)
        order = np.argsort(rhs, kind="stable")
        srt = q.qmoe_gather_mm(dev_bf16(x), dev_bf16(w), dev_u32(lhs_b[order]),
                               dev_u32(rhs[order]), sorted_indices=True)
        assert np.array_equal(host_bits16(srt), host_bits16(got)[order])


def test_gather_mm_bad_index_zeroes_row(gpu_lib):
    q = gpu_lib
    rng = np.random.default_rng(5)
    E, N, K, B = 4, 128, 256, 150
    w = normal_bf16(rng, (E, N, K), 1 / np.sqrt(K))
    x = normal_bf16(rng, (B, 1, K))
    rhs = rng.integers(0, E, size=B).astype(np.uint32)
    rhs[17] = E + 3
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = q.qmoe_gather_mm(dev_bf16(x), dev_bf16(w), None, dev_u32(rhs), status=status)
    assert int(status.item()) & q.QMOE_DEV_BAD_INDEX
    assert not torch.any(got[17].float() != 0)
    keep = np.arange(B) != 17
    want = O.gather_mm(x[keep], w, None, rhs[keep])
    assert_close("gather_mm rows with valid indices", got[torch.from_numpy(keep).cuda()], want)


def test_gather_mm_prefill_shape(gpu_lib):
    """Prefill-shaped unquantized expert projection: hidden 2048 -> 512, 256 experts,
    Zipf-skewed top-8 routing of 512 tokens (x broadcast over each token's experts)."""
    q = gpu_lib
    T, E, K, N = 512, 256, 2048, 512
    rng = np.random.default_rng(9)
    idx, _ = prefill_routing(3, T, E, 8)
    w = normal_bf16(rng, (E, N, K), 1 / np.sqrt(K))
    x = normal_bf16(rng, (T, 1, K))
    rhs = idx.reshape(-1).astype(np.uint32)
    got = q.qmoe_gather_mm(dev_bf16(x), dev_bf16(w), None, dev_u32(rhs))
    want = O.gather_mm(x, w, None, rhs)
    assert_close("gather_mm prefill shape", got, want)


# --------------------------------------------------------------------- combine
@pytest.mark.parametrize("T", [128, 331])
@pytest.mark.parametrize("gated", [True, False])
def test_moe_combine(gpu_lib, T, gated):
    q = gpu_lib
    rng = np.random.default_rng(T)
    K, H, E = 8, 2048, 256
    keys = rng.integers(0, E, size=T * K)
    order, inv, _ = O.sort_by_expert(keys, E)
    y_sorted = normal_bf16(rng, (T * K, H))
    scores = rng.random((T, K)).astype(np.float32) / K
    shared = normal_bf16(rng, (T, H))
    x = normal_bf16(rng, (T, H))
    wsg = normal_bf16(rng, (H,), 1 / np.sqrt(H))
    want = O.moe_combine(y_sorted, inv, scores, shared, x if gated else None,
                         wsg if gated else None)
    out = q.qmoe_moe_combine(dev_bf16(y_sorted), dev_u32(inv.astype(np.uint32)), dev_f32(scores),
                             dev_bf16(shared), dev_bf16(x) if gated else None,
                             dev_bf16(wsg) if gated else None)
    assert_close(f"combine T={T}", out, want)


def _stock_case(T, seed):
    rng = np.random.default_rng(seed)
    K, H, E = 8, 2048, 256
    keys = rng.integers(0, E, size=T * K)
    _, inv, _ = O.sort_by_expert(keys, E)
    y_sorted = normal_bf16(rng, (T * K, H))
    p = rng.random((T, K)).astype(np.float32)
    scores = (p / p.sum(axis=1, keepdims=True)).astype(np.float32)
    shared = normal_bf16(rng, (T, H))
    logits = normal_bf16(rng, (T,), 2.0)
    return y_sorted, inv.astype(np.uint32), scores, shared, logits


@pytest.mark.parametrize("T", [128, 331])
@pytest.mark.parametrize("variant", ["gated", "ungated", "no_shared"])
def test_moe_combine_stock_bit_exact(gpu_lib, T, variant):
    """Stock-tail combine: every rounding point is fixed, so the GPU result equals the
    oracle's bit for bit (MoE block sizes: top-8, hidden 2048)."""
    q = gpu_lib
    y_sorted, inv, scores, shared, logits = _stock_case(T, 100 + T)
    sh = None if variant == "no_shared" else shared
    z = logits if variant == "gated" else None
    want = O.moe_combine_stock(y_sorted, inv, scores, sh, z)
    out = q.qmoe_moe_combine_stock(dev_bf16(y_sorted), dev_u32(inv), dev_f32(scores),
                                   None if sh is None else dev_bf16(sh),
                                   None if z is None else dev_bf16(z))
    got = host_bits16(out)
    assert np.array_equal(got, want), f"{int((got != want).sum())} of {got.size} differ"


def test_moe_combine_stock_bad_index_and_batch_invariance(gpu_lib):
    """An out-of-range position contributes nothing and flags the status word (the
    same bits as a zero score); a token's output does not depend on the other tokens
    of the call."""
    q = gpu_lib
    T, K = 96, 8
    y_sorted, inv, scores, shared, logits = _stock_case(T, 7)
    bad = inv.copy()
    bad[5 * K + 3] = T * K + 11
    zeroed = scores.copy()
    zeroed[5, 3] = 0.0
    want = O.moe_combine_stock(y_sorted, inv, zeroed, shared, logits)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = q.qmoe_moe_combine_stock(dev_bf16(y_sorted), dev_u32(bad), dev_f32(scores),
                                   dev_bf16(shared), dev_bf16(logits), status=status)
    assert np.array_equal(host_bits16(out), want)
    assert int(status.item()) & q.QMOE_DEV_BAD_INDEX
    full = host_bits16(q.qmoe_moe_combine_stock(dev_bf16(y_sorted), dev_u32(inv), dev_f32(scores),
                                                dev_bf16(shared), dev_bf16(logits)))
    a, b = 17, 60  # tokens a..b-1 on their own: their rows, in k order, positions 0..
    rows = inv.reshape(T, K)[a:b].reshape(-1).astype(np.int64)
    sub = q.qmoe_moe_combine_stock(dev_bf16(y_sorted[rows]),
                                   dev_u32(np.arange((b - a) * K, dtype=np.uint32)),
                                   dev_f32(scores[a:b]), dev_bf16(shared[a:b]), dev_bf16(logits[a:b]))
    assert np.array_equal(host_bits16(sub), full[a:b])


def test_moe_block_prefill_with_shared_expert(gpu_lib):
    """MoE block: routed experts in expert order + shared SwiGLU + sigmoid gate, one
    combine pass (T = 128)."""
    q = gpu_lib
    T = 128
    d = prefill_layer(1, T, shared=True)
    W = [qweight(*d[k], 64, 4) for k in ("up", "gate", "down")]
    S = [qweight(*d[k], 64, 4) for k in ("sh_up", "sh_gate", "sh_down")]
    xd = dev_bf16(d["x"])
    ys, inv = q.qmoe_switch_glu(xd, dev_u32(d["idx"]), *W, mode=1)
    zeros = torch.zeros((T, 1), dtype=torch.int32, device="cuda")
    sh = q.qmoe_switch_glu(xd, zeros, *S, mode=0).reshape(T, -1)
    out = q.qmoe_moe_combine(ys, inv, dev_f32(d["scores"]), sh, xd, dev_bf16(d["w_sg"]))
    # oracle chain: its own bf16 expert outputs and shared output feed its combine
    y_tok, _ = _switch_oracle(d["x"], d["idx"], d["up"], d["gate"], d["down"], 64, 4)
    sh_want, _ = O.switch_glu(d["x"], np.zeros((T, 1), np.int64),
                              (*d["sh_up"], 64, 4), (*d["sh_gate"], 64, 4), (*d["sh_down"], 64, 4))
    order, w_inv, _ = O.sort_by_expert(d["idx"].reshape(-1), d["E"])
    y_sorted = O.bf16_from_f32(y_tok.reshape(T * d["top_k"], -1)[order].astype(np.float32))
    sh_b = O.bf16_from_f32(sh_want[:, 0].astype(np.float32))
    want = O.moe_combine(y_sorted, w_inv, d["scores"], sh_b, d["x"], d["w_sg"])
    assert_close("moe block", out, want)
