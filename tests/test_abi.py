"""The C-ABI library loads without a GPU, exports every symbol include/qmoe.h
declares, and rejects invalid arguments on the host before any launch (the
rejected cases of nuvec-core 0.4.0 tests/quantized.rs, invalid_arguments_are_rejected
and gather_qmm_selects_batches)."""

import ctypes
import os
import re

import pytest

import quantized_moe_expert_gather_b200 as q
from quantized_moe_expert_gather_b200 import build as qbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ERR_ARG, ERR_DTYPE, ERR_UNSUPPORTED, ERR_WORKSPACE = -1, -2, -3, -4


@pytest.fixture(scope="module")
def lib():
    qbuild.build()
    return q.load()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "qmoe.h")).read()
    return set(re.findall(r"QMOE_API[^;(]*?\b(qmoe_\w+)\s*\(", text))


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert len(names) >= 13
    assert names == set(q.EXPORTED)
    raw = ctypes.CDLL(q.library_path())
    for n in names:
        assert hasattr(raw, n), n


def test_timing_hook_off_without_gpu(lib):
    assert lib.qmoe_timing_enable(None, 0) == 0
    ms, n = ctypes.c_double(1.0), ctypes.c_uint64(7)
    assert lib.qmoe_timing_read(b"qmv", ctypes.byref(ms), ctypes.byref(n)) == 0
    assert ms.value == 0.0 and n.value == 0
    assert lib.qmoe_timing_read(b"qmv", None, None) == ERR_ARG


def test_status_strings(lib):
    for s in (0, -1, -2, -3, -4, -5):
        assert q.qmoe_status_string(s).startswith("QMOE_")


def test_quantize_rejects_bad_arguments_on_host(lib):
    fake = 1 << 20  # never dereferenced: validation fails first
    assert lib.qmoe_quantize(fake, 1, 2, 64, 48, 4, fake, fake, fake, None) == ERR_UNSUPPORTED
    assert lib.qmoe_quantize(fake, 1, 2, 64, 64, 7, fake, fake, fake, None) == ERR_UNSUPPORTED
    assert lib.qmoe_quantize(fake, 1, 2, 64, 64, 0, fake, fake, fake, None) == ERR_UNSUPPORTED
    assert lib.qmoe_quantize(fake, 1, 2, 64, 64, 9, fake, fake, fake, None) == ERR_UNSUPPORTED
    assert lib.qmoe_dequantize(fake, fake, fake, 1, 2, 64, 64, 7, fake, 1, None) == ERR_UNSUPPORTED
    assert lib.qmoe_quantize(fake, 1, 2, 96, 64, 4, fake, fake, fake, None) == ERR_ARG
    assert lib.qmoe_quantize(fake, 5, 2, 64, 64, 4, fake, fake, fake, None) == ERR_DTYPE
    assert lib.qmoe_quantize(fake, 1, 0, 64, 64, 4, None, None, None, None) == 0  # empty
    assert lib.qmoe_dequantize(fake, fake, fake, 1, 2, 64, 32, 4, fake, 7, None) == ERR_DTYPE


def test_matmuls_reject_bad_arguments_on_host(lib):
    fake = 1 << 20
    # inner-size mismatch (K not a multiple of the group)
    assert lib.qmoe_qmm(fake, 3, fake, fake, fake, 8, 63, 64, 4, fake, None, None) == ERR_ARG
    # unsupported codec
    assert lib.qmoe_qmm(fake, 3, fake, fake, fake, 8, 96, 48, 4, fake, None, None) == ERR_UNSUPPORTED
    # every width of the quantisation tests has a matmul; 7 bits (rejected there), 0 and
    # 9 bits do not
    assert lib.qmoe_qmm(fake, 3, fake, fake, fake, 8, 96, 32, 7, fake, None, None) == ERR_UNSUPPORTED
    assert lib.qmoe_qmm(fake, 3, fake, fake, fake, 8, 64, 32, 0, fake, None, None) == ERR_UNSUPPORTED
    assert lib.qmoe_qmm(fake, 3, fake, fake, fake, 8, 64, 64, 9, fake, None, None) == ERR_UNSUPPORTED
    assert lib.qmoe_qmm(fake, 0, fake, fake, fake, 8, 64, 64, 4, fake, None, None) == 0
    # gather: workspace too small
    need = lib.qmoe_gather_qmm_workspace_size(4, 1, 8, 16, 64)
    assert need > 0
    assert lib.qmoe_gather_qmm(fake, 4, 1, 64, fake, fake, fake, 8, 16, 64, 4, None, fake, 4, 0,
                               fake, need - 1, fake, None, None) == ERR_WORKSPACE
    assert lib.qmoe_gather_qmm(fake, 4, 1, 64, fake, fake, fake, 8, 16, 64, 7, None, fake, 4, 0,
                               fake, need, fake, None, None) == ERR_UNSUPPORTED
    # combine: hidden size not a multiple of 8, and a gate without a shared expert
    assert lib.qmoe_moe_combine(fake, fake, fake, fake, None, None, 2, 2, 12, fake, None, None) == ERR_UNSUPPORTED
    assert lib.qmoe_moe_combine(fake, fake, fake, None, fake, fake, 2, 2, 16, fake, None, None) == ERR_ARG
    assert lib.qmoe_moe_combine(fake, fake, fake, fake, fake, None, 2, 2, 16, fake, None, None) == ERR_ARG


def test_switch_glu_rejects_mismatched_weights_on_host(lib):
    fake = 1 << 20
    W = q._QWeight
    up = W(fake, fake, fake, 4, 32, 64, 64, 4)
    gate = W(fake, fake, fake, 4, 32, 64, 64, 4)
    down_bad = W(fake, fake, fake, 4, 64, 64, 64, 4)   # K must equal up.N = 32
    down = W(fake, fake, fake, 4, 64, 32, 32, 4)
    need = lib.qmoe_switch_glu_workspace_size(2, 2, ctypes.byref(up), ctypes.byref(gate), ctypes.byref(down))
    assert need > 0
    assert lib.qmoe_switch_glu(fake, fake, 2, 2, ctypes.byref(up), ctypes.byref(gate),
                               ctypes.byref(down_bad), 0, fake, need, fake, None, None, None) == ERR_ARG
    assert lib.qmoe_switch_glu(fake, fake, 2, 2, ctypes.byref(up), ctypes.byref(gate),
                               ctypes.byref(down), 2, fake, need, fake, None, None, None) == ERR_ARG
    assert lib.qmoe_switch_glu(fake, fake, 2, 2, ctypes.byref(up), ctypes.byref(gate),
                               ctypes.byref(down), 0, fake, need - 1, fake, None, None, None) == ERR_WORKSPACE


def test_workspace_sizes_grow_with_rows(lib):
    small = lib.qmoe_gather_qmm_workspace_size(8, 1, 288, 2048, 4096)
    large = lib.qmoe_gather_qmm_workspace_size(4096, 1, 288, 2048, 4096)
    assert large > small > 0
    assert lib.qmoe_sort_by_expert_workspace_size(131072, 256) > lib.qmoe_sort_by_expert_workspace_size(8, 256)


def test_gather_mm_and_ep_pack_reject_bad_arguments_on_host(lib):
    fake = 1 << 20  # never dereferenced: validation fails first
    # gather_mm: K a whole number of 64-k stages; workspace; 16-byte aligned operands
    need = lib.qmoe_gather_mm_workspace_size(4, 1, 8, 16, 64)
    assert need > 0
    assert lib.qmoe_gather_mm(fake, 4, 1, 96, fake, 8, 16, None, fake, 4, 0, fake, need,
                              fake, None, None) == ERR_UNSUPPORTED
    assert lib.qmoe_gather_mm(fake, 4, 1, 64, fake, 8, 16, None, fake, 4, 0, fake, need - 1,
                              fake, None, None) == ERR_WORKSPACE
    assert lib.qmoe_gather_mm(fake + 2, 4, 1, 64, fake, 8, 16, None, fake, 4, 0, fake, need,
                              fake, None, None) == ERR_ARG
    assert lib.qmoe_gather_mm(fake, 4, 1, 64, fake, 8, 16, None, fake, 0, 0, None, 0,
                              fake, None, None) == 0  # no batches: nothing to do
    # ep_pack: hidden size a multiple of 8, positive sizes, aligned rows; no rows is a no-op
    assert lib.qmoe_ep_pack(fake, 2, 12, 2, fake, fake, 4, fake, fake, None, None) == ERR_UNSUPPORTED
    assert lib.qmoe_ep_pack(fake, -1, 16, 2, fake, fake, 4, fake, fake, None, None) == ERR_ARG
    assert lib.qmoe_ep_pack(fake, 2, 16, 2, fake, fake, 0, fake, fake, None, None) == ERR_ARG
    assert lib.qmoe_ep_pack(fake + 2, 2, 16, 2, fake, fake, 4, fake, fake, None, None) == ERR_ARG
    assert lib.qmoe_ep_pack(fake, 2, 16, 2, None, fake, 4, fake, fake, None, None) == ERR_ARG
    assert lib.qmoe_ep_pack(None, 0, 16, 2, None, None, 4, None, None, None, None) == 0
