"""Plain CPU oracle of the affine group-quantised MoE gather path.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Sources, by page and section:

[P1] MLX issue #4509, "gather_qmm at M=1 streams 4-bit expert weights at ~half the
     bandwidth of M=4 (MoE decode)": the repro script (expert shapes, the SwitchGLU
     order up, gate, silu(gate)*up, down).
[P2] MLX PR #4567, "[Metal] Gather mm improvement": Description and Proposed
     changes (expert-aligned row tiles built from offsets of rhs_indices; the
     BM = 16, counts 13/8/2/10 example).
[P3] nuvec-core 0.4.0, tests/quantized.rs: the semantic contract of quantize,
     dequantize, quantized_matmul and gather_qmm (tests
     ``round_trip_error_is_about_half_a_step``,
     ``quantize_snaps_zero_and_handles_constant_and_one_signed_groups``,
     ``quantized_matmul_equals_the_dequantized_product``,
     ``gather_qmm_selects_batches``).
[P5] MTPLX PR #558, "One-kernel MoE combine for Qwen3.5/3.6 MoE prefill on the
     invariant lane": Summary and Motivation (unsort, weight by the routing
     scores, sum over top_k, add the gated shared expert).

Conventions.  bf16 tensors are carried as ``uint16`` bit patterns.  Packed codes
are ``uint32`` words.  Every helper returns fresh arrays and mutates nothing.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "CODE_BITS", "bf16_from_f32", "bf16_from_f64", "f32_from_bf16", "pack_codes", "unpack_codes", "quantize",
    "dequantize", "qmm", "gather_qmm", "gather_mm", "sort_by_expert", "tile_table",
    "silu", "switch_glu", "moe_combine", "moe_combine_stock", "sigmoid",
]


# ----------------------------------------------------------------------------- bf16

def bf16_from_f64(v: np.ndarray) -> np.ndarray:
    """float64 -> bf16 bit patterns rounded ONCE to nearest, ties to even (finite
    inputs).

    The value is first rounded to float32 with round-to-odd (truncate toward zero,
    then set the last significand bit when anything was dropped) and that float32 is
    rounded to bf16 to nearest-even.  Round-to-odd at 24 bits keeps every bit the
    second rounding to 8 bits needs, so the result equals one direct rounding of the
    float64 value; plain float32 rounding first would double-round (1 + 2^-8 + 2^-30
    would land on the tie 1 + 2^-8 and go down to 1 instead of up to 1 + 2^-7).
    """
    v = np.ascontiguousarray(np.asarray(v, dtype=np.float64))
    f = v.astype(np.float32)
    too_big = np.abs(f.astype(np.float64)) > np.abs(v)
    f = np.where(too_big, np.nextafter(f, np.float32(0)), f).astype(np.float32)
    inexact = f.astype(np.float64) != v
    u = f.view(np.uint32) | np.where(inexact, np.uint32(1), np.uint32(0))
    return bf16_from_f32(u.view(np.float32))


def f32_from_bf16(u16: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float32 values (exact: bf16 is the top half of fp32)."""
    u16 = np.asarray(u16, dtype=np.uint16)
    return (u16.astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_from_f32(f: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest, ties to even; NaN stays a
    quiet NaN of the same sign."""
    f = np.ascontiguousarray(np.asarray(f, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    rounded = ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint32)
    nan = np.isnan(f)
    quiet = ((u >> np.uint64(16)).astype(np.uint32) | np.uint32(0x0040))
    out = np.where(nan, quiet, rounded)
    return (out & np.uint32(0xFFFF)).astype(np.uint16)


# -------------------------------------------------------------------------- packing

# Bit widths of [P3] (``const BITS``); 7 is rejected there (``quantize(64, 7)`` fails).
CODE_BITS = (1, 2, 3, 4, 5, 6, 8)


def pack_codes(codes: np.ndarray, bits: int) -> np.ndarray:
    """Pack integer codes along the last axis into uint32 words.

    The codes of a row form one least-significant-bit-first bit stream: code j
    occupies stream bits [j*bits, (j+1)*bits), and stream bit i is bit (i mod 32) of
    word i // 32.  For widths that divide 32 this is "code j of a word in bits
    [(j mod 32/bits)*bits, ...)"; for 3, 5 and 6 bits a code may straddle two words.
    The packed shape is ``[..., cols*bits/32]`` for every width, as [P3]
    ``round_trip_error_is_about_half_a_step`` asserts.
    """
    assert bits in CODE_BITS
    codes = np.asarray(codes, dtype=np.int64)
    assert (codes.shape[-1] * bits) % 32 == 0
    assert codes.min(initial=0) >= 0 and codes.max(initial=0) < (1 << bits)
    # stream[..., j*bits + i] = bit i of code j
    shifts = np.arange(bits, dtype=np.int64)
    stream = ((codes[..., :, None] >> shifts) & 1).reshape(codes.shape[:-1] + (-1,))
    stream = stream.reshape(stream.shape[:-1] + (stream.shape[-1] // 32, 32)).astype(np.uint64)
    weights = np.left_shift(np.uint64(1), np.arange(32, dtype=np.uint64))
    return (stream * weights).sum(axis=-1).astype(np.uint32)


def unpack_codes(words: np.ndarray, bits: int) -> np.ndarray:
    """Inverse of :func:`pack_codes`; returns int64 codes.

    For widths that divide 32 no code straddles a word, so code j of a word is
    simply ``(word >> (j*bits)) & (2^bits - 1)``; other widths walk the bit stream.
    """
    assert bits in CODE_BITS
    if 32 % bits == 0:
        w = np.asarray(words, dtype=np.uint32)
        shifts = (np.arange(32 // bits, dtype=np.uint32) * np.uint32(bits))
        codes = (w[..., :, None] >> shifts) & np.uint32((1 << bits) - 1)
        return codes.reshape(w.shape[:-1] + (-1,)).astype(np.int64)
    w = np.asarray(words, dtype=np.uint64)
    stream = (w[..., :, None] >> np.arange(32, dtype=np.uint64)) & np.uint64(1)
    stream = stream.reshape(w.shape[:-1] + (-1,))
    per_code = stream.reshape(stream.shape[:-1] + (stream.shape[-1] // bits, bits))
    weights = np.left_shift(np.uint64(1), np.arange(bits, dtype=np.uint64))
    return (per_code * weights).sum(axis=-1).astype(np.int64)


# ---------------------------------------------------------------------- quantisation

_EPS = np.float32(1e-7)


def quantize(w: np.ndarray, group: int, bits: int, scale_dtype: str = "bf16"):
    """Affine group quantisation of a 2-D float32 matrix along its last axis.

    Returns ``(packed, scales, biases)``; scales and biases are bf16 bit patterns
    (``scale_dtype="bf16"``) or float32 (``"f32"``), shape ``[rows, cols/group]``.

    Per group G of ``group`` consecutive values, with n = 2**bits - 1, every
    operation in float32 and correctly rounded (numpy's float32 arithmetic):

    1. lo = min G, hi = max G; delta = max((hi - lo) / n, 1e-7).
    2. The edge of larger magnitude is snapped to a code so that zero is exactly
       representable ([P3] quantize_snaps_zero...): if |lo| > |hi| the edge is lo
       and the trial step is +delta, otherwise the edge is hi and the step -delta.
    3. q0 = rint(edge / step).  If q0 != 0 the stored step is edge / q0 and the
       bias is the edge, so the edge is restored exactly and zero sits on code
       -q0; snapping can clip the far end of the range by up to one step ([P3]
       round_trip_error_is_about_half_a_step).  If q0 == 0 the trial step is kept
       and the bias is 0.
    4. Step and bias are rounded to the storage type; codes are
       clamp(rint((w - bias) / step), 0, n) with the STORED step and bias.

    The pages fix the invariants, not these constants (1e-7 floor, the tie rule of
    step 2, half-even rint, codes from stored values): they are the plainest
    reading that meets every invariant the pages state.
    """
    assert bits in CODE_BITS and group in (32, 64, 128)
    w = np.asarray(w, dtype=np.float32)
    assert w.ndim == 2 and w.shape[1] % group == 0
    rows, cols = w.shape
    n = np.float32((1 << bits) - 1)
    g = w.reshape(rows, cols // group, group)
    lo = g.min(axis=-1)
    hi = g.max(axis=-1)
    delta = np.maximum((hi - lo) / n, _EPS).astype(np.float32)
    neg = np.abs(lo) > np.abs(hi)
    edge = np.where(neg, lo, hi).astype(np.float32)
    step0 = np.where(neg, delta, -delta).astype(np.float32)
    q0 = np.rint(edge / step0).astype(np.float32)
    nz = q0 != 0
    with np.errstate(divide="ignore", invalid="ignore"):
        snapped = (edge / np.where(nz, q0, np.float32(1))).astype(np.float32)
    scale = np.where(nz, snapped, step0).astype(np.float32)
    bias = np.where(nz, edge, np.float32(0)).astype(np.float32)
    if scale_dtype == "bf16":
        s_store, b_store = bf16_from_f32(scale), bf16_from_f32(bias)
        s_val, b_val = f32_from_bf16(s_store), f32_from_bf16(b_store)
    elif scale_dtype == "f32":
        s_store, b_store = scale, bias
        s_val, b_val = scale, bias
    else:
        raise ValueError(scale_dtype)
    codes = np.rint((g - b_val[..., None]) / s_val[..., None]).astype(np.float32)
    codes = np.clip(codes, np.float32(0), n).astype(np.int64).reshape(rows, cols)
    return pack_codes(codes, bits), s_store, b_store


def _as_f32(v: np.ndarray) -> np.ndarray:
    v = np.asarray(v)
    return f32_from_bf16(v) if v.dtype == np.uint16 else v.astype(np.float32)


def dequantize(packed: np.ndarray, scales: np.ndarray, biases: np.ndarray,
               group: int, bits: int) -> np.ndarray:
    """w = q*scale + bias per group, in float32 ([P3] ``reference`` helper and
    round-trip tests).  Leading (expert) dimensions are kept.

    The product is rounded to float32 before the bias is added.  With bf16 scales
    the product of a <=8-bit code and an 8-bit significand is exact, so this equals
    a fused multiply-add; with float32 scales it is the two-rounding form.
    """
    q = unpack_codes(packed, bits).astype(np.float32)
    s = _as_f32(scales)
    b = _as_f32(biases)
    shp = q.shape
    qg = q.reshape(shp[:-1] + (shp[-1] // group, group))
    prod = (qg * s[..., None]).astype(np.float32)
    return (prod + b[..., None]).astype(np.float32).reshape(shp)


# ------------------------------------------------------------------------- matmuls

def qmm(x: np.ndarray, packed, scales, biases, group: int, bits: int) -> np.ndarray:
    """quantized_matmul with transpose=True: ``x . dequantize(W)^T`` in fp64.

    ``x`` is bf16 bits (uint16) or float; W is ``[N, K*bits/32]``.
    [P3] quantized_matmul_equals_the_dequantized_product.
    """
    xf = _as_f32(x).astype(np.float64)
    wd = dequantize(packed, scales, biases, group, bits).astype(np.float64)
    return xf @ wd.T


def gather_qmm(x, packed, scales, biases, group: int, bits: int,
               lhs_indices=None, rhs_indices=None) -> np.ndarray:
    """gather_qmm with transpose=True ([P3] gather_qmm_selects_batches;
    [P1] repro script ``gq``).

    ``x``: ``[x_batches, M, K]``; W: ``[E, N, K*bits/32]``.  Batch b of the result
    is ``x[lhs[b]] . dequantize(W[rhs[b]])^T``.  Missing indices default to every
    batch in order, x's batch broadcast against the weights'.  Returns fp64
    ``[B, M, N]``.  Sorted and unsorted index lists take the same path.
    """
    x = np.asarray(x)
    E = packed.shape[0]
    xb = x.shape[0]
    if lhs_indices is None and rhs_indices is None:
        B = max(xb, E)
        lhs = np.arange(B) % xb if xb == B else np.zeros(B, np.int64)
        rhs = np.arange(B) % E if E == B else np.zeros(B, np.int64)
    else:
        rhs = np.asarray(rhs_indices, np.int64).reshape(-1) if rhs_indices is not None else None
        lhs = np.asarray(lhs_indices, np.int64).reshape(-1) if lhs_indices is not None else None
        if lhs is None:
            B = rhs.size
            lhs = (np.arange(B) * xb) // B
        if rhs is None:
            B = lhs.size
            rhs = (np.arange(B) * E) // B
        assert lhs.size == rhs.size
    xf = _as_f32(x).astype(np.float64)
    out = np.empty((lhs.size, x.shape[1], packed.shape[1]), np.float64)
    for e in np.unique(rhs):  # dequantise each selected expert once
        wd = dequantize(packed[e], scales[e], biases[e], group, bits).astype(np.float64)
        for b in np.nonzero(rhs == e)[0]:
            out[b] = xf[lhs[b]] @ wd.T
    return out


def gather_mm(x, w, lhs_indices=None, rhs_indices=None) -> np.ndarray:
    """Unquantized gathered matmul ([P2] Description: the gather_mm whose row tiles the
    page reorganises).

    ``x``: bf16 ``[x_batches, M, K]``; ``w``: bf16 ``[E, N, K]``.  Batch b of the result
    is ``x[lhs[b]] . w[rhs[b]]^T``, with the index defaults of :func:`gather_qmm`.
    Returns fp64 ``[B, M, N]``.
    """
    x = np.asarray(x)
    w = np.asarray(w)
    E, xb = w.shape[0], x.shape[0]
    if lhs_indices is None and rhs_indices is None:
        B = max(xb, E)
        lhs = np.arange(B) % xb if xb == B else np.zeros(B, np.int64)
        rhs = np.arange(B) % E if E == B else np.zeros(B, np.int64)
    else:
        rhs = np.asarray(rhs_indices, np.int64).reshape(-1) if rhs_indices is not None else None
        lhs = np.asarray(lhs_indices, np.int64).reshape(-1) if lhs_indices is not None else None
        if lhs is None:
            B = rhs.size
            lhs = (np.arange(B) * xb) // B
        if rhs is None:
            B = lhs.size
            rhs = (np.arange(B) * E) // B
        assert lhs.size == rhs.size
    xf = _as_f32(x).astype(np.float64)
    out = np.empty((lhs.size, x.shape[1], w.shape[1]), np.float64)
    for b in range(lhs.size):
        out[b] = xf[lhs[b]] @ _as_f32(w[rhs[b]]).astype(np.float64).T
    return out


# --------------------------------------------------------------- route metadata

def sort_by_expert(indices: np.ndarray, num_experts: int):
    """Stable sort of routed rows by expert ([P5] Change: the sorted chain's
    ``_gather_sort`` and its inverse permutation; [P2] offsets from rhs_indices).

    ``indices``: expert id per routed row r (r = token*top_k + k when flattened).
    Returns ``order`` (sorted position -> r), ``inv_order`` (r -> sorted position)
    and ``offsets`` (``[E+1]``, exclusive prefix sums of the per-expert counts).
    Ties keep ascending r.
    """
    keys = np.asarray(indices, np.int64).reshape(-1)
    assert keys.size == 0 or (keys.min() >= 0 and keys.max() < num_experts)
    order = np.argsort(keys, kind="stable").astype(np.int64)
    inv = np.empty_like(order)
    inv[order] = np.arange(order.size)
    counts = np.bincount(keys, minlength=num_experts)
    offsets = np.zeros(num_experts + 1, np.int64)
    offsets[1:] = np.cumsum(counts)
    return order, inv, offsets


def tile_table(offsets: np.ndarray, bm: int):
    """Expert-aligned row tiles ([P2] Proposed changes: each tile gets the row to
    start from, the expert to load and the number of valid rows; no tile spans two
    experts).

    Experts are visited in order; expert e with c_e rows gets ceil(c_e/bm) tiles
    starting at offsets[e] + i*bm.  Returns a list of ``(row_start, expert,
    valid)`` triples.
    """
    tiles = []
    for e in range(len(offsets) - 1):
        start, end = int(offsets[e]), int(offsets[e + 1])
        r = start
        while r < end:
            tiles.append((r, e, min(bm, end - r)))
            r += bm
    return tiles


# ------------------------------------------------------------------ MoE blocks

def sigmoid(v):
    v = np.asarray(v, np.float64)
    return 1.0 / (1.0 + np.exp(-v))


def silu(v):
    """silu(g) = g * sigmoid(g) ([P1] repro script ``moe``: ``g * mx.sigmoid(g)``)."""
    v = np.asarray(v, np.float64)
    return v * sigmoid(v)


def switch_glu(x, indices, up, gate, down):
    """SwitchGLU over routed rows ([P1] repro script ``moe``):
    u = x.Wup[e]^T, g = x.Wgate[e]^T, h = silu(g)*u, y = h.Wdown[e]^T.

    ``x``: bf16 ``[T, H]``; ``indices``: ``[T, top_k]``; each weight is a tuple
    ``(packed [E,N,K*bits/32], scales, biases, group, bits)``.  u and g are fp64;
    h is rounded from fp64 to bf16 once (it is the bf16 input of the down
    projection); y is fp64.  The rows routed to one expert go through its three
    matrices together (one fp64 matrix product per matrix).  Returns
    ``(y [T, top_k, H], h_bits [T, top_k, I])``.
    """
    idx = np.asarray(indices, np.int64)
    T, top_k = idx.shape
    xf = _as_f32(x).astype(np.float64)

    def dq(wt, e):
        packed, s, b, gs, bits = wt
        return dequantize(packed[e], s[e], b[e], gs, bits).astype(np.float64)

    inter = up[0].shape[1]
    hid_out = down[0].shape[1]
    y = np.empty((T, top_k, hid_out), np.float64)
    h_bits = np.empty((T, top_k, inter), np.uint16)
    for e in np.unique(idx):  # dequantise each routed expert once
        wu, wg, wd = dq(up, e), dq(gate, e), dq(down, e)
        ts, ks = np.nonzero(idx == e)
        xe = xf[ts]                      # [rows, H]
        u = xe @ wu.T
        g = xe @ wg.T
        h = bf16_from_f64(silu(g) * u)
        h_bits[ts, ks] = h
        y[ts, ks] = f32_from_bf16(h).astype(np.float64) @ wd.T
    return y, h_bits


def moe_combine(y_sorted, inv_order, scores, shared=None, x=None, w_shared_gate=None):
    """One-pass MoE combine ([P5] Summary / Motivation):

    out[t] = sum_k scores[t,k] * y_sorted[inv_order[t*top_k + k]]
             + sigmoid(x[t] . w_shared_gate) * shared[t]

    ``y_sorted``: bf16 ``[T*top_k, H]`` in expert-sorted order; ``scores``: float32
    ``[T, top_k]``; ``shared``/``x``: bf16 ``[T, H]``; ``w_shared_gate``: bf16
    ``[H]``.  The shared term is omitted when ``shared`` is None; the gate is 1
    when ``w_shared_gate`` is None.  Everything in fp64; returns ``[T, H]`` fp64.
    """
    ys = _as_f32(y_sorted).astype(np.float64)
    sc = np.asarray(scores, np.float32).astype(np.float64)
    T, top_k = sc.shape
    inv = np.asarray(inv_order, np.int64).reshape(T, top_k)
    out = np.zeros((T, ys.shape[1]), np.float64)
    for t in range(T):
        for k in range(top_k):
            out[t] += sc[t, k] * ys[inv[t, k]]
    if shared is not None:
        sh = _as_f32(shared).astype(np.float64)
        if w_shared_gate is not None:
            xf = _as_f32(x).astype(np.float64)
            wg = _as_f32(w_shared_gate).astype(np.float64)
            gate = sigmoid(xf @ wg)
        else:
            gate = np.ones(T)
        out += gate[:, None] * sh
    return out


def _bf16_round(v: np.ndarray) -> np.ndarray:
    """float32 values rounded to bf16 (round to nearest even), returned as float32."""
    return f32_from_bf16(bf16_from_f32(np.asarray(v, np.float32)))


def moe_combine_stock(y_sorted, inv_order, scores, shared=None, shared_gate_logit=None):
    """The MoE block tail step by step, each step rounded to bf16 as the stock block
    materialises it ([P5] Motivation: unsort to token order, multiply by the scores,
    sum over top_k, each writing a bf16 tensor, then add the shared expert).

    Reading of the steps (the page names them, not their arithmetic):
      s_k   = bf16(scores[t, k])                        (routing scores as bf16)
      p_k   = bf16(y_sorted[inv_order[t*top_k + k]] * s_k)   (fp32 product, exact)
      r     = bf16(p_0 + p_1 + ... + p_{top_k-1})       (fp32 sum in k order)
      g     = bf16(float32(sigmoid(z_t)))               (z_t: bf16 gate logit, sigmoid
                                                          in fp64; g = 1 without logits)
      out   = bf16(r + bf16(g * shared[t]))             (fp32 product and sum)
    Every operand of a product is bf16, so each fp32 product is exact and every
    rounding point is fixed: the result is defined to the bit.  ``y_sorted``,
    ``shared``, ``shared_gate_logit``: bf16 bit patterns; ``scores`` float32
    ``[T, top_k]``.  Returns bf16 bits ``[T, H]``.
    """
    ys = f32_from_bf16(np.asarray(y_sorted, np.uint16))
    sc = _bf16_round(np.asarray(scores, np.float32))
    T, top_k = sc.shape
    inv = np.asarray(inv_order, np.int64).reshape(T, top_k)
    r = np.zeros((T, ys.shape[1]), np.float32)
    for k in range(top_k):
        p = _bf16_round(ys[inv[:, k]] * sc[:, k:k + 1])
        r = (r + p).astype(np.float32)
    r = _bf16_round(r)
    if shared is None:
        return bf16_from_f32(r)
    sh = f32_from_bf16(np.asarray(shared, np.uint16))
    if shared_gate_logit is None:
        g = np.ones((T, 1), np.float32)
    else:
        z = f32_from_bf16(np.asarray(shared_gate_logit, np.uint16)).astype(np.float64)
        g = _bf16_round((1.0 / (1.0 + np.exp(-z))).astype(np.float32)).reshape(T, 1)
    return bf16_from_f32((r + _bf16_round(g * sh)).astype(np.float32))
