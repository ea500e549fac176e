"""Python binding of the qmoe C ABI (``include/qmoe.h``).

Argument marshalling only: every function here checks tensor shapes, dtypes and
devices, allocates outputs and workspaces with torch (device memory plumbing), and
calls the function of the same name in ``libqmoe.so`` on torch's current CUDA
stream.  All arithmetic runs in the library's CUDA kernels; there is no CPU or
PyTorch fallback, and every call raises if the library cannot be loaded.

Tensors: bf16 data as ``torch.bfloat16``; packed codes as ``torch.int32`` or
``torch.uint32`` (bit patterns); indices as ``torch.int32``/``torch.uint32``.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

__all__ = [
    "QmoeError", "load", "library_path", "qmoe_status_string", "qmoe_launch_count", "qmoe_timing_enable", "qmoe_timing_read",
    "qmoe_quantize", "qmoe_dequantize", "qmoe_qmm", "qmoe_gather_qmm",
    "qmoe_gather_qmm_workspace_size", "qmoe_gather_qmm_noalloc", "qmoe_sort_by_expert", "qmoe_tile_table",
    "qmoe_ep_pack",
    "qmoe_switch_glu", "qmoe_switch_glu_workspace_size", "qmoe_moe_combine",
    "qmoe_moe_combine_stock", "qmoe_gather_mm", "qmoe_gather_mm_workspace_size", "QWeight",
    "QMOE_DEV_BAD_INDEX", "QMOE_DEV_TIMEOUT", "QMOE_DEV_UNSORTED", "qmoe_debug_skip_stage",
    "EXPORTED",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB: Optional[ctypes.CDLL] = None

QMOE_DTYPE_BF16, QMOE_DTYPE_F32 = 0, 1
QMOE_DEV_BAD_INDEX, QMOE_DEV_TIMEOUT, QMOE_DEV_UNSORTED = 1, 2, 4

_p = ctypes.c_void_p
_i64 = ctypes.c_int64
_i32 = ctypes.c_int
_sz = ctypes.c_size_t


class _QWeight(ctypes.Structure):
    _fields_ = [("codes", _p), ("scales", _p), ("biases", _p), ("E", _i64), ("N", _i64),
                ("K", _i64), ("group", ctypes.c_int32), ("bits", ctypes.c_int32)]


# name -> (restype, argtypes); the exact list of symbols include/qmoe.h declares.
_SIGS = {
    "qmoe_status_string": (ctypes.c_char_p, [_i32]),
    "qmoe_debug_skip_stage": (_i32, [_i64]),
    "qmoe_launch_count": (ctypes.c_uint64, []),
    "qmoe_timing_enable": (_i32, [_p, _i64]),
    "qmoe_timing_read": (_i32, [ctypes.c_char_p, ctypes.POINTER(ctypes.c_double),
                                ctypes.POINTER(ctypes.c_uint64)]),
    "qmoe_quantize": (_i32, [_p, _i32, _i64, _i64, _i32, _i32, _p, _p, _p, _p]),
    "qmoe_dequantize": (_i32, [_p, _p, _p, _i32, _i64, _i64, _i32, _i32, _p, _i32, _p]),
    "qmoe_qmm": (_i32, [_p, _i64, _p, _p, _p, _i64, _i64, _i32, _i32, _p, _p, _p]),
    "qmoe_gather_qmm_workspace_size": (_sz, [_i64, _i64, _i64, _i64, _i64]),
    "qmoe_gather_qmm": (_i32, [_p, _i64, _i64, _i64, _p, _p, _p, _i64, _i64, _i32, _i32,
                               _p, _p, _i64, _i32, _p, _sz, _p, _p, _p]),
    "qmoe_gather_qmm_noalloc": (_i32, [_p, _i64, _i64, _i64, _p, _p, _p, _i64, _i64, _i32,
                                       _i32, _p, _p, _i64, _i32, _p, _p, _p]),
    "qmoe_sort_by_expert_workspace_size": (_sz, [_i64, _i64]),
    "qmoe_sort_by_expert": (_i32, [_p, _i64, _i64, _p, _p, _p, _p, _sz, _p, _p]),
    "qmoe_tile_table": (_i32, [_p, _i64, _i32, _p, _i64, _p, _p, _p]),
    "qmoe_ep_pack": (_i32, [_p, _i64, _i64, _i32, _p, _p, _i64, _p, _p, _p, _p]),
    "qmoe_switch_glu_workspace_size": (_sz, [_i64, _i32, ctypes.POINTER(_QWeight),
                                             ctypes.POINTER(_QWeight), ctypes.POINTER(_QWeight)]),
    "qmoe_switch_glu": (_i32, [_p, _p, _i64, _i32, ctypes.POINTER(_QWeight),
                               ctypes.POINTER(_QWeight), ctypes.POINTER(_QWeight), _i32, _p, _sz,
                               _p, _p, _p, _p]),
    "qmoe_moe_combine": (_i32, [_p, _p, _p, _p, _p, _p, _i64, _i32, _i64, _p, _p, _p]),
    "qmoe_moe_combine_stock": (_i32, [_p, _p, _p, _p, _p, _i64, _i32, _i64, _p, _p, _p]),
    "qmoe_gather_mm_workspace_size": (_sz, [_i64, _i64, _i64, _i64, _i64]),
    "qmoe_gather_mm": (_i32, [_p, _i64, _i64, _i64, _p, _i64, _i64, _p, _p, _i64, _i32, _p, _sz,
                              _p, _p, _p]),
}
EXPORTED = tuple(_SIGS)


class QmoeError(RuntimeError):
    def __init__(self, fn: str, status: int):
        msg = load().qmoe_status_string(status).decode()
        super().__init__(f"{fn} failed: {msg} ({status})")
        self.status = status


def library_path() -> str:
    return os.path.join(_HERE, "libqmoe.so")


def load() -> ctypes.CDLL:
    """Loads libqmoe.so (built in-tree by ``build.py``); raises if it is missing."""
    global _LIB
    if _LIB is None:
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: run `python -m quantized_moe_expert_gather_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in _SIGS.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _LIB = lib
    return _LIB


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    return t.data_ptr()


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _check(name: str, status: int):
    if status != 0:
        raise QmoeError(name, status)


def _need(t: torch.Tensor, name: str, dtypes, shape=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype not in dtypes:
        raise TypeError(f"{name}: dtype {t.dtype} not in {dtypes}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)} != {tuple(shape)}")


_CODES = (torch.int32, torch.uint32)
_IDX = (torch.int32, torch.uint32)
_BF16 = (torch.bfloat16,)


def qmoe_status_string(status: int) -> str:
    return load().qmoe_status_string(status).decode()


def qmoe_debug_skip_stage(stage: int) -> None:
    """Test hook of the bounded waits: the next streaming-kernel launch leaves pipeline
    stage ``stage`` of its last CTA unissued (its waits run out, QMOE_DEV_TIMEOUT);
    a negative stage disarms it."""
    _check("qmoe_debug_skip_stage", load().qmoe_debug_skip_stage(stage))


def qmoe_launch_count() -> int:
    return int(load().qmoe_launch_count())


def qmoe_timing_enable(slots: Optional[torch.Tensor]) -> None:
    """Time every following library kernel launch into ``slots`` (a CUDA uint8
    tensor of 16 bytes per launch); ``None`` turns timing off."""
    if slots is None:
        _check("qmoe_timing_enable", load().qmoe_timing_enable(None, 0))
        return
    _need(slots, "slots", (torch.uint8,))
    _check("qmoe_timing_enable", load().qmoe_timing_enable(_ptr(slots), slots.numel() // 16))


def qmoe_timing_read(kernel: str):
    """``(total_ms, launches)`` of the recorded launches of one kernel name."""
    ms = ctypes.c_double(0.0)
    n = ctypes.c_uint64(0)
    _check("qmoe_timing_read", load().qmoe_timing_read(kernel.encode(), ctypes.byref(ms),
                                                       ctypes.byref(n)))
    return ms.value, int(n.value)


def qmoe_quantize(w: torch.Tensor, group: int = 64, bits: int = 4):
    """Affine group quantisation of a 2-D bf16 or float32 matrix.  Returns
    ``(codes int32 [rows, cols*bits/32], scales, biases)``, scales/biases in w's dtype."""
    _need(w, "w", (torch.bfloat16, torch.float32))
    rows, cols = w.shape
    codes = torch.empty((rows, cols * bits // 32), dtype=torch.int32, device=w.device)
    s = torch.empty((rows, cols // group), dtype=w.dtype, device=w.device)
    b = torch.empty_like(s)
    dt = QMOE_DTYPE_F32 if w.dtype == torch.float32 else QMOE_DTYPE_BF16
    _check("qmoe_quantize", load().qmoe_quantize(_ptr(w), dt, rows, cols, group, bits, _ptr(codes),
                                                 _ptr(s), _ptr(b), _stream()))
    return codes, s, b


def qmoe_dequantize(codes, scales, biases, group: int = 64, bits: int = 4,
                    out_dtype=torch.float32) -> torch.Tensor:
    _need(codes, "codes", _CODES)
    _need(scales, "scales", (torch.bfloat16, torch.float32))
    _need(biases, "biases", (scales.dtype,), scales.shape)
    rows = codes.shape[0]
    cols = codes.shape[1] * 32 // bits
    out = torch.empty((rows, cols), dtype=out_dtype, device=codes.device)
    sdt = QMOE_DTYPE_F32 if scales.dtype == torch.float32 else QMOE_DTYPE_BF16
    odt = QMOE_DTYPE_F32 if out_dtype == torch.float32 else QMOE_DTYPE_BF16
    _check("qmoe_dequantize", load().qmoe_dequantize(_ptr(codes), _ptr(scales), _ptr(biases), sdt,
                                                     rows, cols, group, bits, _ptr(out), odt,
                                                     _stream()))
    return out


def qmoe_qmm(x, codes, scales, biases, group: int = 64, bits: int = 4, out=None, status=None):
    """y = x . dequantize(W)^T for x [M, K] bf16 and W [N, K*bits/32]."""
    _need(x, "x", _BF16)
    _need(codes, "codes", _CODES)
    M, K = x.shape
    N = codes.shape[-2]
    y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _check("qmoe_qmm", load().qmoe_qmm(_ptr(x), M, _ptr(codes), _ptr(scales), _ptr(biases), N, K,
                                       group, bits, _ptr(y), _ptr(status), _stream()))
    return y


def qmoe_gather_qmm_workspace_size(B: int, M: int, E: int, N: int, K: int) -> int:
    return int(load().qmoe_gather_qmm_workspace_size(B, M, E, N, K))


def qmoe_gather_qmm(x, codes, scales, biases, lhs_indices=None, rhs_indices=None, group: int = 64,
                    bits: int = 4, sorted_indices: bool = False, out=None, workspace=None,
                    status=None):
    """gather_qmm with transpose=True: x [x_batches, M, K] bf16, W [E, N, K*bits/32];
    index tensors are 1-D (flatten broadcast shapes first).  Returns [B, M, N]."""
    _need(x, "x", _BF16)
    _need(codes, "codes", _CODES)
    xb, M, K = x.shape
    E, N = codes.shape[0], codes.shape[1]
    if lhs_indices is not None:
        _need(lhs_indices, "lhs_indices", _IDX)
    if rhs_indices is not None:
        _need(rhs_indices, "rhs_indices", _IDX)
    if lhs_indices is None and rhs_indices is None:
        B = max(xb, E)
    elif rhs_indices is not None:
        B = rhs_indices.numel()
    else:
        B = lhs_indices.numel()
    if lhs_indices is not None and lhs_indices.numel() != B:
        raise ValueError("lhs_indices and rhs_indices have different sizes")
    y = out if out is not None else torch.empty((B, M, N), dtype=torch.bfloat16, device=x.device)
    need = qmoe_gather_qmm_workspace_size(B, M, E, N, K)
    ws = workspace if workspace is not None else torch.empty(need, dtype=torch.uint8, device=x.device)
    _check("qmoe_gather_qmm", load().qmoe_gather_qmm(
        _ptr(x), xb, M, K, _ptr(codes), _ptr(scales), _ptr(biases), E, N, group, bits,
        _ptr(lhs_indices), _ptr(rhs_indices), B, int(bool(sorted_indices)), _ptr(ws), ws.numel(),
        _ptr(y), _ptr(status), _stream()))
    return y


def qmoe_gather_qmm_noalloc(x, codes, scales, biases, lhs_indices=None, rhs_indices=None,
                            group: int = 64, bits: int = 4, sorted_indices: bool = False,
                            out=None, status=None):
    """As :func:`qmoe_gather_qmm`, for callers that cannot allocate device scratch:
    the library keeps the routing metadata in its own fixed device array (B*M <= 4096,
    E <= 1024; overlapping calls race on it).  4- and 8-bit codes in groups of 32, 64
    or 128; it runs the streaming kernel at every row count.  Pass ``out`` to
    allocate nothing here."""
    _need(x, "x", _BF16)
    _need(codes, "codes", _CODES)
    xb, M, K = x.shape
    E, N = codes.shape[0], codes.shape[1]
    if lhs_indices is not None:
        _need(lhs_indices, "lhs_indices", _IDX)
    if rhs_indices is not None:
        _need(rhs_indices, "rhs_indices", _IDX)
    if rhs_indices is not None:
        B = rhs_indices.numel()
    elif lhs_indices is not None:
        B = lhs_indices.numel()
    else:
        B = max(xb, E)
    if lhs_indices is not None and lhs_indices.numel() != B:
        raise ValueError("lhs_indices and rhs_indices have different sizes")
    if out is not None:
        _need(out, "out", _BF16, (B, M, N))
    y = out if out is not None else torch.empty((B, M, N), dtype=torch.bfloat16, device=x.device)
    _check("qmoe_gather_qmm_noalloc", load().qmoe_gather_qmm_noalloc(
        _ptr(x), xb, M, K, _ptr(codes), _ptr(scales), _ptr(biases), E, N, group, bits,
        _ptr(lhs_indices), _ptr(rhs_indices), B, int(bool(sorted_indices)), _ptr(y),
        _ptr(status), _stream()))
    return y


def qmoe_sort_by_expert(indices, E: int, status=None):
    """Returns ``(order, inv_order, offsets)`` as int32 tensors (bit patterns of uint32)."""
    _need(indices, "indices", _IDX)
    R = indices.numel()
    dev = indices.device
    order = torch.empty(R, dtype=torch.int32, device=dev)
    inv = torch.empty(R, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    need = int(load().qmoe_sort_by_expert_workspace_size(R, E))
    ws = torch.empty(need, dtype=torch.uint8, device=dev)
    _check("qmoe_sort_by_expert", load().qmoe_sort_by_expert(
        _ptr(indices), R, E, _ptr(order), _ptr(inv), _ptr(offsets), _ptr(ws), need, _ptr(status),
        _stream()))
    return order, inv, offsets


def qmoe_ep_pack(x, indices, order, E_local: int, x_send=None, e_send=None, status=None):
    """Expert-parallel send buffers: ``x_send[p] = x[order[p] // top_k]`` and
    ``e_send[p] = indices.flat[order[p]] % E_local`` for the rows in expert order.
    Returns ``(x_send [T*top_k, H] bf16, e_send [T*top_k] int32)``."""
    _need(x, "x", _BF16)
    _need(indices, "indices", _IDX)
    _need(order, "order", _IDX)
    T, H = x.shape
    top_k = indices.shape[1]
    R = T * top_k
    if order.numel() != R:
        raise ValueError("order must hold T*top_k entries")
    if x_send is None:
        x_send = torch.empty((R, H), dtype=torch.bfloat16, device=x.device)
    if e_send is None:
        e_send = torch.empty(R, dtype=torch.int32, device=x.device)
    _check("qmoe_ep_pack", load().qmoe_ep_pack(
        _ptr(x), T, H, top_k, _ptr(indices), _ptr(order), E_local, _ptr(x_send), _ptr(e_send),
        _ptr(status), _stream()))
    return x_send, e_send


def qmoe_tile_table(offsets, bm: int, max_tiles: int, status=None):
    """Returns ``(tiles int32 [max_tiles, 3], num_tiles int32 [1])``."""
    _need(offsets, "offsets", _IDX)
    E = offsets.numel() - 1
    tiles = torch.zeros((max_tiles, 3), dtype=torch.int32, device=offsets.device)
    num = torch.zeros(1, dtype=torch.int32, device=offsets.device)
    _check("qmoe_tile_table", load().qmoe_tile_table(_ptr(offsets), E, bm, _ptr(tiles), max_tiles,
                                                     _ptr(num), _ptr(status), _stream()))
    return tiles, num


class QWeight:
    """A quantised weight stack: codes [E, N, K*bits/32], scales/biases [E, N, K/group]."""

    def __init__(self, codes, scales, biases, group: int, bits: int):
        _need(codes, "codes", _CODES)
        _need(scales, "scales", _BF16)
        _need(biases, "biases", _BF16, scales.shape)
        if codes.dim() == 2:
            codes, scales, biases = codes[None], scales[None], biases[None]
        self.codes, self.scales, self.biases = codes, scales, biases
        self.group, self.bits = group, bits
        self.E, self.N = codes.shape[0], codes.shape[1]
        self.K = codes.shape[2] * 32 // bits

    def c_struct(self) -> _QWeight:
        return _QWeight(_ptr(self.codes), _ptr(self.scales), _ptr(self.biases), self.E, self.N,
                        self.K, self.group, self.bits)


def qmoe_switch_glu_workspace_size(T: int, top_k: int, up: QWeight, gate: QWeight, down: QWeight) -> int:
    u, g, d = up.c_struct(), gate.c_struct(), down.c_struct()
    return int(load().qmoe_switch_glu_workspace_size(T, top_k, ctypes.byref(u), ctypes.byref(g),
                                                     ctypes.byref(d)))


def qmoe_switch_glu(x, indices, up: QWeight, gate: QWeight, down: QWeight, mode: int = 0,
                    out=None, inv_order=None, workspace=None, status=None):
    """SwitchGLU over routed rows.  mode 0: y [T, top_k, H] in token order; mode 1:
    ``(y_sorted [T*top_k, H], inv_order [T*top_k])``."""
    _need(x, "x", _BF16)
    _need(indices, "indices", _IDX)
    T, H = x.shape
    top_k = indices.shape[1]
    u, g, d = up.c_struct(), gate.c_struct(), down.c_struct()
    if out is None:
        shape = (T, top_k, H) if mode == 0 else (T * top_k, H)
        out = torch.empty(shape, dtype=torch.bfloat16, device=x.device)
    if mode == 1 and inv_order is None:
        inv_order = torch.empty(T * top_k, dtype=torch.int32, device=x.device)
    need = int(load().qmoe_switch_glu_workspace_size(T, top_k, ctypes.byref(u), ctypes.byref(g),
                                                     ctypes.byref(d)))
    ws = workspace if workspace is not None else torch.empty(need, dtype=torch.uint8, device=x.device)
    _check("qmoe_switch_glu", load().qmoe_switch_glu(
        _ptr(x), _ptr(indices), T, top_k, ctypes.byref(u), ctypes.byref(g), ctypes.byref(d), mode,
        _ptr(ws), ws.numel(), _ptr(out), _ptr(inv_order), _ptr(status), _stream()))
    return out if mode == 0 else (out, inv_order)


def qmoe_moe_combine(y_sorted, inv_order, scores, shared=None, x=None, w_shared_gate=None,
                     out=None, status=None):
    """out[t] = sum_k scores[t,k]*y_sorted[inv_order[t*top_k+k]] + sigmoid(x[t].w)*shared[t]."""
    _need(y_sorted, "y_sorted", _BF16)
    _need(scores, "scores", (torch.float32,))
    T, top_k = scores.shape
    H = y_sorted.shape[-1]
    out = out if out is not None else torch.empty((T, H), dtype=torch.bfloat16, device=y_sorted.device)
    _check("qmoe_moe_combine", load().qmoe_moe_combine(
        _ptr(y_sorted), _ptr(inv_order), _ptr(scores), _ptr(shared), _ptr(x), _ptr(w_shared_gate),
        T, top_k, H, _ptr(out), _ptr(status), _stream()))
    return out


def qmoe_moe_combine_stock(y_sorted, inv_order, scores, shared=None, shared_gate_logit=None,
                           out=None, status=None):
    """The MoE tail with the stock block's bf16 rounding at every step: out[t] =
    bf16(bf16(sum_k bf16(y_sorted[inv_order[t*top_k+k]] * bf16(scores[t,k])))
    + bf16(bf16(sigmoid(z[t])) * shared[t])), z = shared_gate_logit (bf16 [T])."""
    _need(y_sorted, "y_sorted", _BF16)
    _need(scores, "scores", (torch.float32,))
    T, top_k = scores.shape
    H = y_sorted.shape[-1]
    out = out if out is not None else torch.empty((T, H), dtype=torch.bfloat16, device=y_sorted.device)
    _check("qmoe_moe_combine_stock", load().qmoe_moe_combine_stock(
        _ptr(y_sorted), _ptr(inv_order), _ptr(scores), _ptr(shared), _ptr(shared_gate_logit),
        T, top_k, H, _ptr(out), _ptr(status), _stream()))
    return out


def qmoe_gather_mm_workspace_size(B: int, M: int, E: int, N: int, K: int) -> int:
    return int(load().qmoe_gather_mm_workspace_size(B, M, E, N, K))


def qmoe_gather_mm(x, w, lhs_indices=None, rhs_indices=None, sorted_indices: bool = False,
                   out=None, workspace=None, status=None):
    """Unquantized gather_mm: y[b] = x[lhs[b]] . W[rhs[b]]^T for x [x_batches, M, K] bf16
    and W [E, N, K] bf16; 1-D index tensors.  Returns [B, M, N] bf16."""
    _need(x, "x", _BF16)
    _need(w, "w", _BF16)
    xb, M, K = x.shape
    E, N = w.shape[0], w.shape[1]
    if lhs_indices is not None:
        _need(lhs_indices, "lhs_indices", _IDX)
    if rhs_indices is not None:
        _need(rhs_indices, "rhs_indices", _IDX)
    if lhs_indices is None and rhs_indices is None:
        B = max(xb, E)
    elif rhs_indices is not None:
        B = rhs_indices.numel()
    else:
        B = lhs_indices.numel()
    if lhs_indices is not None and lhs_indices.numel() != B:
        raise ValueError("lhs_indices and rhs_indices have different sizes")
    y = out if out is not None else torch.empty((B, M, N), dtype=torch.bfloat16, device=x.device)
    need = qmoe_gather_mm_workspace_size(B, M, E, N, K)
    ws = workspace if workspace is not None else torch.empty(need, dtype=torch.uint8, device=x.device)
    _check("qmoe_gather_mm", load().qmoe_gather_mm(
        _ptr(x), xb, M, K, _ptr(w), E, N, _ptr(lhs_indices), _ptr(rhs_indices), B,
        int(bool(sorted_indices)), _ptr(ws), ws.numel(), _ptr(y), _ptr(status), _stream()))
    return y
