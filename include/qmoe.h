/*
 * qmoe: affine group-quantised MoE expert gather on NVIDIA B200 (sm_100a).
 *
 * A C ABI over hand-written CUDA kernels.  Sources of each operation, by page and
 * section:
 *   [P1] MLX issue #4509 "gather_qmm at M=1 streams 4-bit expert weights at ~half
 *        the bandwidth of M=4 (MoE decode)", repro script.
 *   [P2] MLX PR #4567 "[Metal] Gather mm improvement", Description / Proposed changes.
 *   [P3] nuvec-core 0.4.0 tests/quantized.rs (the quantize / quantized_matmul /
 *        gather_qmm contract and its rejected arguments).
 *   [P5] MTPLX PR #558 "One-kernel MoE combine for Qwen3.5/3.6 MoE prefill on the
 *        invariant lane", Summary / Motivation.
 *
 * Conventions for every call:
 *   - Pointers are DEVICE pointers owned by the caller, unless a comment says
 *     otherwise.  The library never allocates, frees or synchronises; every call is
 *     asynchronous on `stream` (a cudaStream_t / CUstream handle; NULL = the legacy
 *     default stream).
 *   - bf16 tensors are 16-bit bit patterns (qmoe_bf16).  Tensors are dense and
 *     row-major with the shapes given; codes, scales and biases must be 16-byte
 *     aligned (any cudaMalloc / torch allocation is).
 *   - Host-side validation runs before any launch and returns a negative status;
 *     nothing is launched then.  QMOE_ERR_CUDA reports a launch failure.
 *   - Errors found on the device never trap: they are OR-ed into the optional
 *     `int* d_status` (device memory, caller-zeroed) as QMOE_DEV_* bits, and the
 *     rows concerned are written as zeros.
 *   - Supported codecs: group in {32, 64, 128}; bits in {1, 2, 3, 4, 5, 6, 8} (the widths
 *     of nuvec-core's quantisation tests; 7 is rejected there and here) for every call.
 *     4- and 8-bit codes run on the MMA kernels (streaming and tensor-core), 2-bit codes
 *     in groups of 64 or 128 on the streaming MMA kernel, and 1-, 3-, 5- and 6-bit codes
 *     and 2-bit codes in groups of 32 on a CUDA-core streaming kernel at every row count
 *     (supported for completeness, not tuned); K a positive
 *     multiple of the group.  Packed layout: the codes of a row form one
 *     least-significant-bit-first bit stream, code j at stream bits [j*bits, (j+1)*bits)
 *     and stream bit i in bit (i mod 32) of word i/32 -- for 4 and 8 bits, code j of a
 *     word in bits [(j mod 32/bits)*bits, ...); 3-, 5- and 6-bit codes may straddle two
 *     words -- so W [rows, K] packs to [rows, K*bits/32].
 *   - Kernel choice (results agree within the bf16 tolerance whichever runs): the matmul
 *     calls plan from the most routed rows one expert can receive -- up to 16 a streaming
 *     kernel, beyond a tensor-core kernel.  Environment overrides, read at every call:
 *     QMOE_FORCE_KERNEL=qmv|tc pins the plan; QMOE_PREFILL=tc uses the tensor-core kernel
 *     that stages weights in shared memory instead of the one that keeps them in tensor
 *     memory; QMOE_PDL=0 (read once) launches without programmatic dependent launch.
 */
#ifndef QMOE_H_
#define QMOE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QMOE_API __attribute__((visibility("default")))
#else
#define QMOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t qmoe_bf16;   /* bf16 bit pattern */
typedef void* qmoe_stream;    /* cudaStream_t */

enum {
  QMOE_OK = 0,
  QMOE_ERR_ARG = -1,          /* bad shape, size, pointer or index count        */
  QMOE_ERR_DTYPE = -2,        /* unsupported dtype code                          */
  QMOE_ERR_UNSUPPORTED = -3,  /* bits / group / K combination not supported     */
  QMOE_ERR_WORKSPACE = -4,    /* workspace missing or smaller than required      */
  QMOE_ERR_CUDA = -5,         /* a kernel launch failed                          */
  QMOE_ERR_TOO_LARGE = -6     /* beyond the fixed capacity of qmoe_gather_qmm_noalloc */
};

enum { QMOE_DTYPE_BF16 = 0, QMOE_DTYPE_F32 = 1 };

/* Bits OR-ed into *d_status by kernels. */
enum {
  QMOE_DEV_BAD_INDEX = 1,     /* an expert or row index was out of range; its rows are zero */
  QMOE_DEV_TIMEOUT = 2,       /* a bounded wait ran out; the call's outputs are undefined    */
  QMOE_DEV_UNSORTED = 4       /* sorted_indices was set but rhs decreases somewhere; the
                                 result is still correct (rows are sorted by expert anyway) */
};

/* One quantised weight stack: codes [E, N, K*bits/32] uint32, scales and biases
 * [E, N, K/group] bf16.  Row n of expert e holds output channel n (transpose=True). */
typedef struct {
  const uint32_t* codes;
  const qmoe_bf16* scales;
  const qmoe_bf16* biases;
  int64_t E, N, K;
  int32_t group, bits;
} qmoe_qweight;

/*
 * qmoe_debug_skip_stage -- test hook of the bounded waits (no page counterpart).  The
 * next launch of the streaming kernel (qmoe_qmm / qmoe_gather_qmm / qmoe_switch_glu on
 * few rows per expert) leaves the copies of pipeline stage `stage` of its last CTA
 * unissued, so the waits for that stage run out: the kernel sets QMOE_DEV_TIMEOUT in
 * its d_status, stops every role, lets its issued copies land and returns, leaving
 * its outputs undefined; the next call is unaffected.  A wait runs out after about a
 * second.  stage < 0 disarms the hook.  Host state, one-shot; returns QMOE_OK.
 */
QMOE_API int qmoe_debug_skip_stage(int64_t stage);

/* Human-readable name of a status code (static string; never NULL). */
QMOE_API const char* qmoe_status_string(int status);

/* Number of kernels launched by this process through the library so far (host
 * counter, for benchmark bookkeeping). */
QMOE_API uint64_t qmoe_launch_count(void);

/*
 * Kernel timing (benchmark instrumentation, works inside CUDA graphs).
 *   qmoe_timing_enable(slots, capacity): from now on every kernel launch of the
 *     library takes the next of `capacity` 16-byte slots of the caller's DEVICE
 *     buffer `slots`, zeroes it in stream order and records in it the earliest CTA
 *     start and the latest CTA end (the GPU's global nanosecond timer), keyed on the
 *     host by the kernel's name ("route", "gather_rows", "qmv", "qmv_glu", "tc",
 *     "tc_glu", "combine").  Launches beyond `capacity` are not timed.  Earlier
 *     records are cleared.  slots = NULL turns timing off.
 *   qmoe_timing_read(kernel, &ms, &n): copies the slots back (synchronously: call it
 *     after the timed work has finished) and returns the summed durations and the
 *     number of timed launches of that kernel name.  Replaying a captured graph
 *     rewrites the same slots, so read after each replay.
 * Returns QMOE_ERR_ARG for a null output pointer, QMOE_ERR_CUDA if the copy fails.
 */
QMOE_API int qmoe_timing_enable(void* slots, int64_t capacity);
QMOE_API int qmoe_timing_read(const char* kernel, double* total_ms, uint64_t* launches);

/*
 * qmoe_quantize -- affine group quantisation along the last axis ([P3]
 * round_trip_error_is_about_half_a_step, quantize_snaps_zero_and_handles_constant_
 * and_one_signed_groups).
 *   w       [rows, cols] of dtype w_dtype (QMOE_DTYPE_BF16 or QMOE_DTYPE_F32)
 *   codes   [rows, cols*bits/32] uint32 (out)
 *   scales, biases [rows, cols/group] of dtype w_dtype (out)
 * Per group: lo/hi = min/max, delta = max((hi-lo)/(2^bits-1), 1e-7); the edge of
 * larger magnitude is snapped to a code (scale = edge/rint(edge/(+-delta)), bias =
 * edge; or scale = +-delta, bias = 0 when that code is 0), so zero is exactly
 * representable and constant groups are restored exactly; codes =
 * clamp(rint((w - bias)/scale), 0, 2^bits-1) from the STORED scale and bias.  All
 * steps are IEEE float32; the result is bit-exact with the oracle.
 * Errors: QMOE_ERR_ARG (rows < 0, cols not a multiple of group, null pointers),
 * QMOE_ERR_UNSUPPORTED (bits/group), QMOE_ERR_DTYPE.
 */
QMOE_API int qmoe_quantize(const void* w, int w_dtype, int64_t rows, int64_t cols, int group, int bits,
                  uint32_t* codes, void* scales, void* biases, qmoe_stream stream);

/*
 * qmoe_dequantize -- w = q*scale + bias ([P3] the `reference` helper):
 *   codes [rows, cols*bits/32]; scales, biases [rows, cols/group] of sb_dtype;
 *   out [rows, cols] of out_dtype (float32 or bf16, round to nearest even).
 * The product is rounded to float32 before the bias is added (for bf16 scales the
 * product is exact).  Bit-exact with the oracle.
 */
QMOE_API int qmoe_dequantize(const uint32_t* codes, const void* scales, const void* biases, int sb_dtype,
                    int64_t rows, int64_t cols, int group, int bits, void* out, int out_dtype,
                    qmoe_stream stream);

/*
 * qmoe_qmm -- quantized_matmul with transpose=True ([P3]
 * quantized_matmul_equals_the_dequantized_product): y = x . dequantize(W)^T.
 *   x [M, K] bf16; codes [N, K*bits/32]; scales, biases [N, K/group] bf16;
 *   y [M, N] bf16 (out), fp32 accumulation, one rounding at the end.
 * M = 0 is a no-op.  No workspace.
 * Ordering: the kernel may begin streaming codes, scales and biases while the kernel
 * launched just before it on the stream is still running (only x is read after that
 * kernel has completed).  The weights therefore must not be written by that kernel if
 * it is one of this library's hot-path kernels (qmm, gather_qmm, switch_glu, combine,
 * routing); weights written by qmoe_quantize, qmoe_dequantize, a copy or any kernel
 * outside this library are complete before the weights are read.
 */
QMOE_API int qmoe_qmm(const qmoe_bf16* x, int64_t M, const uint32_t* codes, const qmoe_bf16* scales,
             const qmoe_bf16* biases, int64_t N, int64_t K, int group, int bits, qmoe_bf16* y,
             int* d_status, qmoe_stream stream);

/*
 * qmoe_gather_qmm -- gather_qmm with transpose=True ([P3] gather_qmm_selects_batches;
 * [P1] repro script `gq`):  y[b] = x[lhs[b]] . dequantize(W[rhs[b]])^T, b in [0, B).
 *   x            [x_batches, M, K] bf16
 *   codes        [E, N, K*bits/32];  scales, biases [E, N, K/group] bf16
 *   lhs_indices  [B] uint32 or NULL: NULL means lhs[b] = b*x_batches/B (identity when
 *                x_batches == B; one x batch per token over its experts when
 *                B = x_batches*top_k)
 *   rhs_indices  [B] uint32 or NULL: NULL means rhs[b] = b*E/B
 *   sorted_indices  a promise that rhs is non-decreasing; results are identical
 *                either way (the rows are sorted by expert on the device), and a
 *                broken promise sets QMOE_DEV_UNSORTED
 *   workspace    device scratch of at least qmoe_gather_qmm_workspace_size() bytes
 *   y            [B, M, N] bf16 (out)
 * Rows whose rhs >= E or lhs >= x_batches are written as zeros and flag
 * QMOE_DEV_BAD_INDEX.
 */
QMOE_API size_t qmoe_gather_qmm_workspace_size(int64_t B, int64_t M, int64_t E, int64_t N, int64_t K);
QMOE_API int qmoe_gather_qmm(const qmoe_bf16* x, int64_t x_batches, int64_t M, int64_t K,
                    const uint32_t* codes, const qmoe_bf16* scales, const qmoe_bf16* biases,
                    int64_t E, int64_t N, int group, int bits, const uint32_t* lhs_indices,
                    const uint32_t* rhs_indices, int64_t B, int sorted_indices, void* workspace,
                    size_t workspace_bytes, qmoe_bf16* y, int* d_status, qmoe_stream stream);

/*
 * qmoe_gather_qmm_noalloc -- the same product as qmoe_gather_qmm for callers that
 * cannot allocate device memory.  The pages have no counterpart: this entry point
 * exists because some callers can neither call cudaMalloc nor hand the library a
 * workspace -- e.g. a plugin that is given only its input and output tensors by a
 * host framework that owns all device memory, or a serving loop that must not call
 * cudaMalloc (it can synchronise the device) between requests.
 *   Arguments as qmoe_gather_qmm, without the workspace, except that only 4- and
 *   8-bit codes in groups of 32, 64 or 128 are taken (others: QMOE_ERR_UNSUPPORTED).
 *   The routing metadata lives in a fixed 128 KiB array in device memory inside the
 *   library (one copy per GPU that loads the library, held until the process exits).
 *   The call allocates nothing and runs the streaming kernel at every row count: it
 *   reads an expert's weights once per tile of 8 or 16 routed rows, so with many rows
 *   per expert (prefill-sized calls, skewed routing) it re-reads a heavy expert's
 *   weights up to 256 times and runs far below qmoe_gather_qmm's tensor-core path.
 *   Limits: B*M <= 4096 routed rows and E <= 1024 experts; larger problems return
 *   QMOE_ERR_TOO_LARGE before any launch.
 *   The first call on a device looks up the array's device address (with that device
 *   current); make that first call before any stream capture.  The address is kept
 *   for the life of the process: after cudaDeviceReset (or anything else that
 *   destroys the device's primary context) do not call this entry point again in
 *   that process.
 *   All calls share the array: calls that overlap on the GPU (other streams, other
 *   threads) race on it and must be serialised by the caller.
 */
QMOE_API int qmoe_gather_qmm_noalloc(const qmoe_bf16* x, int64_t x_batches, int64_t M, int64_t K,
                                     const uint32_t* codes, const qmoe_bf16* scales,
                                     const qmoe_bf16* biases, int64_t E, int64_t N, int group,
                                     int bits, const uint32_t* lhs_indices,
                                     const uint32_t* rhs_indices, int64_t B, int sorted_indices,
                                     qmoe_bf16* y, int* d_status, qmoe_stream stream);

/*
 * qmoe_sort_by_expert -- stable counting sort of routed rows by expert ([P5] Change:
 * the sorted chain's `_gather_sort` and inverse permutation; [P2] offsets
 * precomputed from rhs_indices).
 *   indices    [R] uint32 expert id of routed row r (r = token*top_k + k)
 *   order      [R] uint32 (out): sorted position -> r; equal experts keep ascending r
 *   inv_order  [R] uint32 (out): r -> sorted position
 *   offsets    [E+1] uint32 (out): exclusive prefix sums of the per-expert counts
 * Rows with an index >= E are placed after offsets[E] (in ascending r) and flag
 * QMOE_DEV_BAD_INDEX.  Bit-exact with the oracle.
 */
QMOE_API size_t qmoe_sort_by_expert_workspace_size(int64_t R, int64_t E);
QMOE_API int qmoe_sort_by_expert(const uint32_t* indices, int64_t R, int64_t E, uint32_t* order,
                        uint32_t* inv_order, uint32_t* offsets, void* workspace,
                        size_t workspace_bytes, int* d_status, qmoe_stream stream);

/*
 * qmoe_ep_pack -- the send buffer of an expert-parallel dispatch ([P5] Change: the sorted
 * chain gathers routed rows in expert order and keeps the inverse permutation for the
 * combine).  With experts partitioned contiguously over ranks (expert e on rank
 * e / E_local), rows in expert order are grouped by owner rank: one all-to-all of these
 * buffers dispatches every row, the same all-to-all in reverse returns the outputs in
 * expert order for qmoe_moe_combine (with the sort's inv_order).
 *   x        [T, H] bf16 activations;  indices [T, top_k] uint32 expert ids
 *   order    [T*top_k] uint32 from qmoe_sort_by_expert(indices)
 *   x_send   [T*top_k, H] bf16 (out): x_send[p] = x[order[p] / top_k]
 *   e_send   [T*top_k] uint32 (out): indices[order[p]] mod E_local, the expert's number
 *            on its owner rank
 * H must be a multiple of 8 (QMOE_ERR_UNSUPPORTED); x and x_send 16-byte aligned.
 * Rows past the valid ones (index >= E) are packed too; a caller sends only the first
 * offsets[E] rows.  QMOE_ERR_ARG for bad sizes or pointers.
 */
QMOE_API int qmoe_ep_pack(const qmoe_bf16* x, int64_t T, int64_t H, int top_k,
                          const uint32_t* indices, const uint32_t* order, int64_t E_local,
                          qmoe_bf16* x_send, uint32_t* e_send, int* d_status, qmoe_stream stream);

/*
 * qmoe_tile_table -- expert-aligned row tiles ([P2] Proposed changes: every tile gets
 * the row to start from, the expert to load and the number of valid rows; no tile
 * spans two experts).
 *   offsets  [E+1] uint32 (from qmoe_sort_by_expert)
 *   tiles    [max_tiles, 3] uint32 (out): (row_start, expert, valid), experts in
 *            order, ceil(count_e/bm) tiles for expert e
 *   num_tiles  [1] uint32 (out)
 * max_tiles must be at least R/bm + min(E, R) rounded up (QMOE_ERR_ARG otherwise is
 * not detectable on the host: excess tiles are dropped and flag QMOE_DEV_BAD_INDEX).
 */
QMOE_API int qmoe_tile_table(const uint32_t* offsets, int64_t E, int bm, uint32_t* tiles,
                    int64_t max_tiles, uint32_t* num_tiles, int* d_status, qmoe_stream stream);

/*
 * qmoe_switch_glu -- the routed SwitchGLU chain ([P1] repro script `moe`):
 *   u = x.Wup[e]^T, g = x.Wgate[e]^T, h = bf16(silu(g)*u), y = h.Wdown[e]^T
 * for every routed row r = t*top_k + k with e = indices[t, k].
 *   x        [T, H] bf16;  indices [T, top_k] uint32
 *   up, gate  qweights with N = I, K = H;  down: N = H, K = I (host structs)
 *   mode 0   y [T, top_k, H] in token order
 *   mode 1   y [T*top_k, H] in expert-sorted order and inv_order [T*top_k]
 *            (r -> sorted row), ready for qmoe_moe_combine ([P5] Change:
 *            `sorted_experts`)
 *   workspace  at least qmoe_switch_glu_workspace_size() bytes
 */
QMOE_API size_t qmoe_switch_glu_workspace_size(int64_t T, int top_k, const qmoe_qweight* up,
                                      const qmoe_qweight* gate, const qmoe_qweight* down);
QMOE_API int qmoe_switch_glu(const qmoe_bf16* x, const uint32_t* indices, int64_t T, int top_k,
                    const qmoe_qweight* up, const qmoe_qweight* gate, const qmoe_qweight* down,
                    int mode, void* workspace, size_t workspace_bytes, qmoe_bf16* y,
                    uint32_t* inv_order, int* d_status, qmoe_stream stream);

/*
 * qmoe_gather_mm -- the unquantized gathered matmul ([P2] Description and Proposed
 * changes: gather_mm over rows routed to experts, tiles cut per expert from offsets of
 * rhs_indices, every tile running one K loop against one expert):
 *   y[b, m, :] = x[lhs[b], m, :] . W[rhs[b]]^T
 *   x   [x_batches, M, K] bf16;  w [E, N, K] bf16 (row n of expert e at (e*N + n)*K)
 *   lhs_indices, rhs_indices, B, sorted_indices as in qmoe_gather_qmm
 *   y   [B, M, N] bf16.  fp32 accumulation on the tensor cores, one rounding.
 * Routed rows are sorted by expert into 128-row tiles (the tensor-core kernel
 * without the dequant stage).  K must be a multiple of 64 (QMOE_ERR_UNSUPPORTED);
 * x, w and y 16-byte aligned (QMOE_ERR_ARG); workspace at least
 * qmoe_gather_mm_workspace_size() bytes (QMOE_ERR_WORKSPACE).  Rows with an index
 * >= E (or a bad lhs) are zeroed and flag QMOE_DEV_BAD_INDEX.
 */
QMOE_API size_t qmoe_gather_mm_workspace_size(int64_t B, int64_t M, int64_t E, int64_t N,
                                              int64_t K);
QMOE_API int qmoe_gather_mm(const qmoe_bf16* x, int64_t x_batches, int64_t M, int64_t K,
                            const qmoe_bf16* w, int64_t E, int64_t N,
                            const uint32_t* lhs_indices, const uint32_t* rhs_indices, int64_t B,
                            int sorted_indices, void* workspace, size_t workspace_bytes,
                            qmoe_bf16* y, int* d_status, qmoe_stream stream);

/*
 * qmoe_moe_combine -- one-pass MoE combine ([P5] Summary / Motivation):
 *   out[t] = sum_k scores[t,k] * y_sorted[inv_order[t*top_k+k]]
 *            + sigmoid(x[t] . w_shared_gate) * shared[t]
 *   y_sorted [T*top_k, H] bf16; inv_order [T*top_k] uint32; scores [T, top_k] float32
 *   shared [T, H] bf16 or NULL (no shared term); x [T, H] bf16 and w_shared_gate [H]
 *   bf16, both NULL for an ungated shared term (gate 1)
 *   out [T, H] bf16.  fp32 accumulation, one rounding.
 * inv_order entries >= T*top_k contribute zero and flag QMOE_DEV_BAD_INDEX.
 */
QMOE_API int qmoe_moe_combine(const qmoe_bf16* y_sorted, const uint32_t* inv_order, const float* scores,
                     const qmoe_bf16* shared, const qmoe_bf16* x, const qmoe_bf16* w_shared_gate,
                     int64_t T, int top_k, int64_t H, qmoe_bf16* out, int* d_status,
                     qmoe_stream stream);

/*
 * qmoe_moe_combine_stock -- the same tail with the stock block's rounding, in one pass
 * ([P5] Motivation: the stock block unsorts the expert outputs, multiplies by the
 * scores and sums over top_k, each step writing a bf16 tensor, then adds the gated
 * shared expert; the combine reproduces that rounding).  Reading of the steps:
 *   s_k = bf16(scores[t,k])
 *   p_k = bf16(y_sorted[inv_order[t*top_k+k]] * s_k)     (exact fp32 product)
 *   r   = bf16(p_0 + ... + p_{top_k-1})                  (fp32 sum in k order)
 *   g   = bf16(float(sigmoid(z[t])))                     (sigmoid in fp64; 1 if no z)
 *   out[t] = bf16(r + bf16(g * shared[t]))
 *   y_sorted [T*top_k, H] bf16; inv_order [T*top_k] uint32; scores [T, top_k] float32
 *   shared [T, H] bf16 or NULL (no shared term); shared_gate_logit [T] bf16 (each
 *   token's shared-gate projection z) or NULL for gate 1; out [T, H] bf16.
 * The result is fixed to the bit by these steps and does not depend on the other
 * tokens of the call.  inv_order entries >= T*top_k contribute zero and flag
 * QMOE_DEV_BAD_INDEX.  Errors: QMOE_ERR_ARG (T < 0, top_k <= 0, H <= 0, null or
 * unaligned tensors, shared_gate_logit without shared), QMOE_ERR_UNSUPPORTED (H not a
 * multiple of 8), QMOE_ERR_CUDA (launch failure).
 */
QMOE_API int qmoe_moe_combine_stock(const qmoe_bf16* y_sorted, const uint32_t* inv_order,
                                    const float* scores, const qmoe_bf16* shared,
                                    const qmoe_bf16* shared_gate_logit, int64_t T, int top_k,
                                    int64_t H, qmoe_bf16* out, int* d_status,
                                    qmoe_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* QMOE_H_ */
