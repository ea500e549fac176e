"""GPU parity of the integer and bit-exact steps: quantize / dequantize, the expert
sort and the tile table, each compared with the CPU oracle bit for bit."""

import json
import os

import numpy as np
import pytest
import torch

import oracle as O
from gpu_util import assert_close, dev_bf16, dev_u32, host_bits16, host_u32
from inputs import bf16_bits, normal_bf16

pytestmark = pytest.mark.gpu
GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _weights(rng, rows, cols, group):
    w = rng.standard_normal((rows, cols)).astype(np.float32)
    w[0, :group] = 0.75                                    # constant group
    w[1, :group] = -1.0 - np.arange(group) / 8             # all negative
    w[2, :group] = np.arange(group) / (group - 1) - 0.25   # spans zero
    w[3, :group] = rng.random(group) / 4                   # U[0, 0.25)
    return w


@pytest.mark.parametrize("bits", O.CODE_BITS)
@pytest.mark.parametrize("group", [32, 64, 128])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_quantize_dequantize_bit_exact(gpu_lib, bits, group, dtype):
    q = gpu_lib
    rng = np.random.default_rng(bits * 1000 + group)
    w = _weights(rng, 37, 4 * group, group)
    if dtype == "bf16":
        wb = bf16_bits(w)
        w_host = O.f32_from_bf16(wb)
        w_dev = torch.from_numpy(wb.view(np.int16)).cuda().view(torch.bfloat16)
    else:
        w_host = w
        w_dev = torch.from_numpy(w).cuda()
    codes, s, b = q.qmoe_quantize(w_dev, group, bits)
    want_codes, want_s, want_b = O.quantize(w_host, group, bits, scale_dtype=dtype)
    assert np.array_equal(host_u32(codes), want_codes)
    if dtype == "bf16":
        assert np.array_equal(host_bits16(s), want_s)
        assert np.array_equal(host_bits16(b), want_b)
    else:
        assert np.array_equal(s.cpu().numpy().view(np.uint32), want_s.view(np.uint32))
        assert np.array_equal(b.cpu().numpy().view(np.uint32), want_b.view(np.uint32))
    want_d = O.dequantize(want_codes, want_s, want_b, group, bits)
    d32 = q.qmoe_dequantize(codes, s, b, group, bits, out_dtype=torch.float32)
    assert np.array_equal(d32.cpu().numpy().view(np.uint32), want_d.view(np.uint32))
    d16 = q.qmoe_dequantize(codes, s, b, group, bits, out_dtype=torch.bfloat16)
    assert np.array_equal(host_bits16(d16), O.bf16_from_f32(want_d))


def test_seven_bits_rejected_and_quantised_3bit_weights_multiply(gpu_lib):
    """7 bits is rejected by the codec and the matmuls ([P3] rejected_arguments); 3-bit
    weights quantised on the GPU go straight into qmoe_qmm (the bit-stream layout is the
    matmul's input layout) and match the oracle's product of the same codes."""
    q = gpu_lib
    w = torch.zeros((2, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(RuntimeError, match="UNSUPPORTED"):
        q.qmoe_quantize(w, 64, 7)
    rng = np.random.default_rng(3)
    wb = torch.from_numpy(rng.standard_normal((40, 192)).astype(np.float32)).cuda().to(torch.bfloat16)
    codes, s, b = q.qmoe_quantize(wb, 64, 3)
    assert codes.shape == (40, 18)
    xh = normal_bf16(rng, (3, 192))
    y = q.qmoe_qmm(dev_bf16(xh), codes, s, b, 64, 3)
    want = O.qmm(xh, host_u32(codes), host_bits16(s), host_bits16(b), 64, 3)
    assert_close("3-bit qmm of GPU-quantised weights", y, want)
    with pytest.raises(RuntimeError, match="UNSUPPORTED"):
        q.qmoe_qmm(dev_bf16(xh), codes, s, b, 64, 7)


@pytest.mark.parametrize("R,E", [(1, 1), (37, 5), (1024, 288), (1025, 256), (4099, 8),
                                 (20000, 256), (131072, 256)])
def test_sort_by_expert_bit_exact(gpu_lib, R, E):
    q = gpu_lib
    rng = np.random.default_rng(R + E)
    keys = rng.integers(0, E, size=R).astype(np.uint32)
    order, inv, offsets = q.qmoe_sort_by_expert(dev_u32(keys), E)
    w_order, w_inv, w_off = O.sort_by_expert(keys, E)
    assert np.array_equal(host_u32(order), w_order)
    assert np.array_equal(host_u32(inv), w_inv)
    assert np.array_equal(host_u32(offsets), w_off)


def test_sort_by_expert_flags_bad_indices(gpu_lib):
    q = gpu_lib
    keys = np.array([3, 9, 1, 3, 0, 12, 1], np.uint32)    # E = 4: 9 and 12 are invalid
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    order, inv, offsets = q.qmoe_sort_by_expert(dev_u32(keys), 4, status=status)
    valid = keys < 4
    w_order, _, w_off = O.sort_by_expert(keys[valid], 4)
    got = host_u32(order)
    assert np.array_equal(got[: valid.sum()], np.nonzero(valid)[0][w_order])
    assert np.array_equal(got[valid.sum():], np.nonzero(~valid)[0])
    assert np.array_equal(host_u32(offsets), w_off)
    assert np.array_equal(host_u32(inv)[got], np.arange(len(keys)))
    assert int(status.item()) & q.QMOE_DEV_BAD_INDEX


def test_tile_table_worked_example(gpu_lib):
    q = gpu_lib
    g = json.load(open(os.path.join(GOLD, "p2_tile_example.json")))
    offsets = np.concatenate([[0], np.cumsum(g["counts"])]).astype(np.uint32)
    tiles, num = q.qmoe_tile_table(dev_u32(offsets), g["bm"], 16)
    n = int(num.item())
    assert n == g["aligned_passes"]
    assert host_u32(tiles)[:n].tolist() == g["aligned_tiles"]


@pytest.mark.parametrize("bm", [8, 16, 128, 192])
def test_tile_table_random_bit_exact(gpu_lib, bm):
    q = gpu_lib
    rng = np.random.default_rng(bm)
    for E in (1, 7, 256, 1500):
        counts = rng.integers(0, 300, size=E) * (rng.random(E) < 0.6)
        offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.uint32)
        want = O.tile_table(offsets, bm)
        max_tiles = len(want) + 5
        tiles, num = q.qmoe_tile_table(dev_u32(offsets), bm, max_tiles)
        assert int(num.item()) == len(want)
        assert host_u32(tiles)[: len(want)].tolist() == [list(t) for t in want]
