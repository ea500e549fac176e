#!/usr/bin/env python
"""Benchmark of the quantized MoE expert-gather hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = a 42-layer chain of decode MoE layers (MLX issue #4509's chained
protocol): per layer, route the M=4 tokens to their 8 experts (expert sort + tile
table), up/gate gather_qmm with the fused silu*mul epilogue, down gather_qmm, and
the one-pass combine; each layer gets fresh routing and its output is the next
layer's input.  Shapes: hidden 4096, intermediate 2048, 288 experts, top-8, 4-bit
affine, group 64.  The metric is the weight bandwidth: unique expert bytes the
step touches / step time.  Weights (3.6 GB) are far larger than L2, and fresh
routing per layer keeps each layer's experts cold.

Printed on rank 0 as one JSON line, with: isolated decode layers at M=1 and M=4;
the prefill MoE layer at T = 512 ... 16384 (Zipf-skewed routing); the dense small-M
decoder-block qmm forward (1..16 rows, 4- and 8-bit); the full MoE block with a
shared expert and the combine (4-bit g64 and 8-bit g128); the roofline of the
dominant kernel (its launches timed live by the kernels' own device timers inside
the CUDA graph); an end-to-end number with host buffers; SM clocks sampled through
NVML during the timed region; and the CPU oracle timed on a bounded sample (rank 0,
N=1).

``--impl reference`` times the CPU oracle itself (the reference arm of this
repository) on the same metric.  Under torchrun each rank runs an independent
replica (weak scaling) and the time is the max over ranks.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.join(ROOT, "tests"))

H, I, E, TOP_K, GROUP, BITS = 4096, 2048, 288, 8, 64, 4
LAYERS = 42
M_CHAIN = 4

# DRAM traffic of one fused up/gate launch over its algorithmic bytes, from an ncu
# capture (dram__bytes_read.sum + dram__bytes_write.sum) of qmv_kernel<4,64,4,1> in this
# chain at 64 experts, layer 20 of the first warm-up step (28 touched experts:
# 264,368,384 B read + 3,879,424 B written for 264,241,152 algorithmic bytes).
# The per-launch traffic reported below is this ratio times the launch's algorithmic
# bytes (traffic scales with the experts touched).
UPGATE_TRAFFIC_RATIO = (264_368_384 + 3_879_424) / 264_241_152


def matrix_bytes(N, K, group=GROUP, bits=BITS):
    return N * K * bits // 8 + 2 * N * (K // group) * 2


UPGATE_BYTES = 2 * matrix_bytes(I, H)            # per expert, fused up/gate kernel
EXPERT_BYTES = UPGATE_BYTES + matrix_bytes(H, I)  # 14,155,776 per expert
PREFILL_FLOP_PER_ROW = 2 * (2 * 2048 * 512) + 2 * 512 * 2048


# --------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML every ~5 ms."""

    HW_SLOWDOWN, SW_POWER_CAP, SW_THERMAL, HW_THERMAL = 0x8, 0x4, 0x20, 0x40

    def __init__(self, torch_dev: int):
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._th = None
        try:
            import pynvml as nv
            nv.nvmlInit()
            self.nv = nv
            self.h = self._handle(torch_dev)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
        except Exception as e:  # noqa: BLE001
            self.nv, self.err = None, str(e)

    def _handle(self, torch_dev):
        import torch
        nv = self.nv
        props = torch.cuda.get_device_properties(torch_dev)
        uuid = getattr(props, "uuid", None)
        if uuid is not None:
            try:
                return nv.nvmlDeviceGetHandleByUUID(("GPU-" + str(uuid)).encode())
            except Exception:  # noqa: BLE001
                try:
                    return nv.nvmlDeviceGetHandleByUUID("GPU-" + str(uuid))
                except Exception:  # noqa: BLE001
                    pass
        return nv.nvmlDeviceGetHandleByIndex(torch_dev)

    def _reasons(self):
        nv = self.nv
        f = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        return f(self.h)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= int(self._reasons())
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self.nv is not None:
            self._th = threading.Thread(target=self._run, daemon=True)
            self._th.start()
        return self

    def __exit__(self, *exc):
        if self._th is not None:
            self._stop.set()
            self._th.join()

    def summary(self):
        if self.nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [f"nvml unavailable: {self.err}"]}
        names = []
        for bit, name in ((self.HW_SLOWDOWN, "hw_slowdown"), (self.HW_THERMAL, "hw_thermal_slowdown"),
                          (self.SW_THERMAL, "sw_thermal_slowdown"), (self.SW_POWER_CAP, "sw_power_cap")):
            if self.reasons & bit:
                names.append(name)
        med = statistics.median(self.samples) if self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


# ------------------------------------------------------------------ helpers
def dist_setup(gpus):
    import torch
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, ws, local


def max_over_ranks(value: float, ws: int) -> float:
    if ws == 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, ws: int) -> float:
    if ws == 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def job_gbs(my_bytes: float, my_ms: float, ws: int):
    """Whole-job throughput of independent replicas: the bytes every rank processed
    over the slowest rank's time.  Returns (GB/s, max ms)."""
    ms_max = max_over_ranks(my_ms, ws)
    total = sum_over_ranks(my_bytes, ws)
    return total / (ms_max * 1e-3) / 1e9, ms_max


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def measured_peaks():
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except Exception:  # noqa: BLE001
        return None


# ---------------------------------------------------------------- CPU oracle
def oracle_decode_sample(weights, seed):
    """The oracle on one decode token (8 experts): switch_glu + combine.  Returns
    (seconds, weight bytes of the sample)."""
    import oracle as O
    from inputs import decode_scores, decode_tokens
    up, gate, down = weights
    x, idx = decode_tokens(seed, 1)
    sc = decode_scores(seed, 1)
    experts = np.unique(idx)
    remap = np.searchsorted(experts, idx)
    sel = lambda wt: (wt[0][experts], wt[1][experts], wt[2][experts], GROUP, BITS)  # noqa: E731
    t0 = time.perf_counter()
    y, _ = O.switch_glu(x, remap, sel(up), sel(gate), sel(down))
    order, inv, _ = O.sort_by_expert(remap.reshape(-1), len(experts))
    ys = O.bf16_from_f32(y.reshape(TOP_K, H)[order].astype(np.float32))
    O.moe_combine(ys, inv, sc)
    return time.perf_counter() - t0, len(experts) * EXPERT_BYTES


def cpu_threads_limit():
    try:
        from threadpoolctl import threadpool_limits
        return threadpool_limits(limits=1)
    except Exception:  # noqa: BLE001
        import contextlib
        return contextlib.nullcontext()


def run_reference(args, rank, ws):
    """Reference arm: the CPU oracle, as it stands, on the host cores."""
    if rank != 0:
        return
    from inputs import decode_weights
    weights = decode_weights(0)
    times, nbytes = [], []
    with cpu_threads_limit():
        for i in range(args.warmup + args.steps):
            t, b = oracle_decode_sample(weights, 10_000 + i)
            if i >= args.warmup:
                times.append(t)
                nbytes.append(b)
    gbs = sum(nbytes) / sum(times) / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sum(times) / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": CONFIG,
        "cpu_baseline": {"kind": "oracle", "value": gbs, "unit": "GB/s", "cores": 1,
                         "nproc": os.cpu_count(), "cores_available": len(os.sched_getaffinity(0)),
                         "sample": "one decode token per step: SwitchGLU over its 8 experts "
                                   "(113 MB of packed weights) + combine, fp64, one thread"},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


METRIC = "MoE gather_qmm decode weight GB/s (42-layer SwitchGLU+combine chain, M=4)"
CONFIG = {
    "workload": "decode MoE layer chain: 42 layers x (expert sort + tile table, up/gate "
                "gather_qmm + silu*mul, down gather_qmm, combine); hidden 4096, intermediate "
                "2048, 288 experts, top-8, 4-bit affine group 64, M=4 tokens, fresh routing per layer",
    "M": M_CHAIN, "layers": LAYERS, "experts": E, "top_k": TOP_K, "hidden": H, "intermediate": I,
    "bits": BITS, "group": GROUP,
    "l2": "inputs larger than L2: 3.6 GB of expert weights, fresh routing every layer",
}


def run_prefill(q, token_counts, dev, peaks, reps=5):
    """Prefill MoE layer (Zipf-skewed routing, expert-sorted SwitchGLU, combine) at each
    token count: layer time, TFLOP/s, and the per-kernel split from the launch timing
    slots."""
    import torch
    from gpu_util import dev_bf16, dev_f32, dev_u32, qweight
    from inputs import prefill_layer
    out = {}
    for T in token_counts:
        d = prefill_layer(0, T)
        Wp = [qweight(*d[k], GROUP, BITS) for k in ("up", "gate", "down")]
        xp, ip, sp = dev_bf16(d["x"]), dev_u32(d["idx"]), dev_f32(d["scores"])
        wsp = torch.empty(q.qmoe_switch_glu_workspace_size(T, TOP_K, *Wp), dtype=torch.uint8,
                          device=dev)
        ysp = torch.empty((T * TOP_K, 2048), dtype=torch.bfloat16, device=dev)
        invp = torch.empty(T * TOP_K, dtype=torch.int32, device=dev)
        outp = torch.empty((T, 2048), dtype=torch.bfloat16, device=dev)

        def pf():
            q.qmoe_switch_glu(xp, ip, *Wp, mode=1, out=ysp, inv_order=invp, workspace=wsp)
            q.qmoe_moe_combine(ysp, invp, sp, out=outp)

        for _ in range(3):
            pf()
        torch.cuda.synchronize()
        stream = torch.cuda.current_stream()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            pf()
        e1.record(stream)
        torch.cuda.synchronize()
        t = e0.elapsed_time(e1) / reps
        slots = torch.zeros(16 * 64, dtype=torch.uint8, device=dev)
        q.qmoe_timing_enable(slots)
        pf()
        torch.cuda.synchronize()
        split = {k: q.qmoe_timing_read(k)[0] for k in
                 ("route", "gather_rows", "ts_glu", "ts", "tc_glu", "tc", "qmv_glu", "qmv",
                  "combine")}
        q.qmoe_timing_enable(None)
        flop = T * TOP_K * PREFILL_FLOP_PER_ROW
        tf = flop / (t * 1e-3) / 1e12
        bf16_peak = peaks["bf16_tflops"] if peaks else 1590.0
        glu_ms = split["ts_glu"] or split["tc_glu"] or split["qmv_glu"]
        dn_ms = split["ts"] or split["tc"] or split["qmv"]
        glu_tf = T * TOP_K * 4 * 2048 * 512 / (glu_ms * 1e-3) / 1e12 if glu_ms else None
        dn_tf = T * TOP_K * 2 * 2048 * 512 / (dn_ms * 1e-3) / 1e12 if dn_ms else None
        # bytes the layer must move at least: touched experts' weights, the activations
        # read and the expert outputs written (x once, x_s and y_sorted, h both ways)
        touched = len(np.unique(d["idx"]))
        R = T * TOP_K
        moved = touched * (2 * matrix_bytes(512, 2048) + matrix_bytes(2048, 512)) + \
            T * 2048 * 2 + R * 512 * 4 + R * 2048 * 2
        gbs = moved / (t * 1e-3) / 1e9
        hbm_peak = peaks["hbm_gbs"] if peaks else 6650.0
        out[f"T{T}"] = {"ms": t, "tflops": tf, "frac_bf16_peak": tf / bf16_peak,
                        "bytes_moved": moved, "gbs": gbs, "frac_hbm": gbs / hbm_peak,
                        "touched_experts": touched,
                        "upgate_tflops": glu_tf, "down_tflops": dn_tf,
                        "upgate_ms": glu_ms, "down_ms": dn_ms,
                        "upgate_kernel": "qmm_ts" if split["ts_glu"] else
                                         "qmm_tc" if split["tc_glu"] else "qmv",
                        **{f"{k}_ms": v for k, v in split.items() if v}}
        del Wp, d
    return out


def flat(d, sep="_"):
    """Nested result dicts -> one level of scalar values (keys joined by ``sep``):
    the form the JSON line's sub-objects keep."""
    out = {}
    for k, v in d.items():
        if isinstance(v, dict):
            for k2, v2 in flat(v, sep).items():
                out[f"{k}{sep}{k2}"] = v2
        else:
            out[k] = v
    return out


def prefill_roofline(prefill, peaks):
    """Roofline of the prefill up/gate launch at the largest token count: its FLOP per
    launch over its live launch time, against the measured bf16 peak."""
    if not prefill:
        return None
    T = max(int(k[1:]) for k in prefill)
    r = prefill[f"T{T}"]
    peak = peaks["bf16_tflops"] if peaks else 1590.0
    flop = T * TOP_K * 4 * 2048 * 512
    ach = r["upgate_tflops"]
    return {"kernel": f"{r['upgate_kernel']} up/gate gather_qmm + silu*mul, T={T}",
            "bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s",
            "frac": ach / peak if ach else None,
            "peak_source": "measured (MEASURED_PEAKS.json bf16_tflops, burst)" if peaks
                           else "fallback",
            "flop_per_launch": flop, "launch_us": 1e3 * r["upgate_ms"] if r["upgate_ms"] else None,
            "traffic": None,
            "layer_ms": r["ms"], "layer_tflops": r["tflops"], "layer_frac": r["frac_bf16_peak"]}


def _graph_time(fn, reps=8):
    """Device time of one replay of a CUDA graph of fn (ms): 3 warm replays, then reps
    replays between CUDA events on the current stream."""
    import torch
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    t = e0.elapsed_time(e1) / reps
    del g
    return t


def run_dense(q, dev, peaks, layers=36, n_sets=8):
    """Dense small-M quantised matmuls over decoder-block shapes (hidden 2560, q 4096,
    kv 1024, intermediate 9728): a forward of 36 layers of q/k/v/o/gate/up/down qmm,
    cycling over 8 weight sets so the weights (>= 454 MB) stream from HBM, for 1..16
    rows, 4-bit and 8-bit group 64.  Weights W = N(0,1)/sqrt(K) bf16, quantised by
    qmoe_quantize.  Reports forward time and weight GB/s against the HBM peak."""
    import torch
    from inputs import dense_projections
    proj = dense_projections()
    hbm = peaks["hbm_gbs"] if peaks else 6650.0
    gen = torch.Generator(device=dev)
    gen.manual_seed(3)
    out = {}
    for bits in (4, 8):
        sets = []
        for _ in range(n_sets):
            layer = []
            for _, N, K in proj:
                w = (torch.randn(N, K, generator=gen, device=dev) / K ** 0.5).to(torch.bfloat16)
                layer.append(q.qmoe_quantize(w, GROUP, bits))
                del w
            sets.append(layer)
        layer_bytes = sum(matrix_bytes(N, K, GROUP, bits) for _, N, K in proj)
        rows = {}
        for M in (1, 2, 3, 4, 5, 6, 7, 8, 10, 12, 16):
            xs = {K: torch.randn(M, K, generator=gen, device=dev).to(torch.bfloat16)
                  for K in sorted({k for _, _, k in proj})}
            ys = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for _, N, _ in proj]

            def fwd():
                for l in range(layers):
                    ws = sets[l % n_sets]
                    for i, (_, N, K) in enumerate(proj):
                        q.qmoe_qmm(xs[K], *ws[i], GROUP, bits, out=ys[i])

            t = _graph_time(fwd)
            gbs = layers * layer_bytes / (t * 1e-3) / 1e9
            rows[f"M{M}"] = {"ms": t, "weight_gbs": gbs, "frac_hbm": gbs / hbm}
        out[f"{bits}bit_g{GROUP}"] = {"bytes_per_forward": layers * layer_bytes, "rows": rows}
        del sets
    return out


def run_block(q, dev, peaks):
    """Full MoE block: the prefill routing at T in {128, 331, 2048, 4096}, expert-sorted
    routed SwitchGLU, a shared SwiGLU expert (intermediate 512, same quantisation), and
    the one-pass combine with the sigmoid-gated shared output; 4-bit group 64 and 8-bit
    group 128.  Reports block time, TFLOP/s and the weight bytes touched per second."""
    import torch
    from gpu_util import dev_bf16, dev_f32, dev_u32, qweight
    from inputs import prefill_layer
    hbm = peaks["hbm_gbs"] if peaks else 6650.0
    bf16_peak = peaks["bf16_tflops"] if peaks else 1590.0
    out = {}
    for bits, group in ((4, 64), (8, 128)):
        e_bytes = 2 * matrix_bytes(512, 2048, group, bits) + matrix_bytes(2048, 512, group, bits)
        res = {}
        for T in (128, 331, 2048, 4096):
            d = prefill_layer(0, T, group=group, bits=bits, shared=True)
            W = [qweight(*d[k], group, bits) for k in ("up", "gate", "down")]
            S = [qweight(*d[k], group, bits) for k in ("sh_up", "sh_gate", "sh_down")]
            xd, ids, sc, wsg = dev_bf16(d["x"]), dev_u32(d["idx"]), dev_f32(d["scores"]), dev_bf16(d["w_sg"])
            zeros = torch.zeros((T, 1), dtype=torch.int32, device=dev)
            ws1 = torch.empty(q.qmoe_switch_glu_workspace_size(T, TOP_K, *W), dtype=torch.uint8, device=dev)
            ws2 = torch.empty(q.qmoe_switch_glu_workspace_size(T, 1, *S), dtype=torch.uint8, device=dev)
            ys = torch.empty((T * TOP_K, 2048), dtype=torch.bfloat16, device=dev)
            inv = torch.empty(T * TOP_K, dtype=torch.int32, device=dev)
            sh = torch.empty((T, 1, 2048), dtype=torch.bfloat16, device=dev)
            ob = torch.empty((T, 2048), dtype=torch.bfloat16, device=dev)

            def blk():
                q.qmoe_switch_glu(xd, ids, *W, mode=1, out=ys, inv_order=inv, workspace=ws1)
                q.qmoe_switch_glu(xd, zeros, *S, mode=0, out=sh, workspace=ws2)
                q.qmoe_moe_combine(ys, inv, sc, sh.view(T, 2048), xd, wsg, out=ob)

            t = _graph_time(blk)
            touched = len(np.unique(d["idx"]))
            flop = (T * TOP_K + T) * PREFILL_FLOP_PER_ROW
            wbytes = (touched + 1) * e_bytes
            res[f"T{T}"] = {"ms": t, "tflops": flop / (t * 1e-3) / 1e12,
                            "frac_bf16_peak": flop / (t * 1e-3) / 1e12 / bf16_peak,
                            "touched_experts": touched,
                            "weight_gbs": wbytes / (t * 1e-3) / 1e9,
                            "frac_hbm_weights": wbytes / (t * 1e-3) / 1e9 / hbm}
            del W, S, d
        out[f"{bits}bit_g{group}"] = res
    return out


def run_combine(q, dev, peaks):
    """The one-pass combine (fp32 sum, one rounding) and the stock-tail combine (bf16
    rounding at each step) on expert-sorted outputs of hidden 2048, top-8, with a gated
    shared term.  Each must read top_k + 1 rows (and x for the gate dot, or one logit)
    and write one row per token; reported against the HBM peak."""
    import torch
    from gpu_util import dev_bf16, dev_f32, dev_u32
    from inputs import normal_bf16
    hbm = peaks["hbm_gbs"] if peaks else 6650.0
    Hh, K = 2048, TOP_K
    out = {}
    for T in (128, 331, 2048, 4096, 16384):
        rng = np.random.default_rng(T)
        y = dev_bf16(normal_bf16(rng, (T * K, Hh)))
        inv = dev_u32(rng.permutation(T * K).astype(np.uint32))
        sc = dev_f32((rng.random((T, K)) / K).astype(np.float32))
        sh, x = dev_bf16(normal_bf16(rng, (T, Hh))), dev_bf16(normal_bf16(rng, (T, Hh)))
        wsg = dev_bf16(normal_bf16(rng, (Hh,), 1 / np.sqrt(Hh)))
        z = dev_bf16(normal_bf16(rng, (T,)))
        ob = torch.empty((T, Hh), dtype=torch.bfloat16, device=dev)
        row = Hh * 2
        t_one = _graph_time(lambda: q.qmoe_moe_combine(y, inv, sc, sh, x, wsg, out=ob))
        t_stock = _graph_time(lambda: q.qmoe_moe_combine_stock(y, inv, sc, sh, z, out=ob))
        b_one = T * ((K + 3) * row + K * 8) + row          # y rows, shared, x, out; inv+scores; w
        b_stock = T * ((K + 2) * row + K * 8 + 2)           # y rows, shared, out; inv+scores; z
        out[f"T{T}"] = {
            "one_pass_us": 1e3 * t_one, "one_pass_frac_hbm": b_one / (t_one * 1e-3) / 1e9 / hbm,
            "stock_us": 1e3 * t_stock, "stock_frac_hbm": b_stock / (t_stock * 1e-3) / 1e9 / hbm}
    return out


def run_gather_mm(q, dev, peaks):
    """Unquantized gather_mm (bf16 weights, the tensor-core kernel without its dequant
    stage) on the prefill expert projection: hidden 2048 -> 512, 256 experts, Zipf-skewed
    top-8 routing, x broadcast over each token's experts.  TFLOP/s against the bf16 peak."""
    import torch
    from gpu_util import dev_bf16, dev_u32
    from inputs import normal_bf16, prefill_routing
    bf16_peak = peaks["bf16_tflops"] if peaks else 1590.0
    E, K, N = 256, 2048, 512
    rng = np.random.default_rng(21)
    w = dev_bf16(normal_bf16(rng, (E, N, K), 1 / np.sqrt(K)))
    out = {}
    for T in (4096, 16384):
        idx, _ = prefill_routing(0, T, E, TOP_K)
        x = dev_bf16(normal_bf16(rng, (T, 1, K)))
        rhs = dev_u32(idx.reshape(-1).astype(np.uint32))
        B = T * TOP_K
        ws = torch.empty(q.qmoe_gather_mm_workspace_size(B, 1, E, N, K), dtype=torch.uint8, device=dev)
        y = torch.empty((B, 1, N), dtype=torch.bfloat16, device=dev)
        t = _graph_time(lambda: q.qmoe_gather_mm(x, w, None, rhs, out=y, workspace=ws))
        tf = 2.0 * B * N * K / (t * 1e-3) / 1e12
        out[f"T{T}"] = {"ms": t, "tflops": tf, "frac_bf16_peak": tf / bf16_peak}
    return out


# ---------------------------------------------------------------------- ours
def main():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=30)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-prefill", action="store_true")
    p.add_argument("--no-cpu", action="store_true")
    p.add_argument("--experts", type=int, default=E,
                   help="number of experts (smaller for profiling captures)")
    p.add_argument("--prefill-only", type=int, default=0, metavar="T",
                   help="only time the prefill MoE layer at T tokens (profiling captures)")
    p.add_argument("--prefill-tokens", default="512,713,1024,2048,4123,8192,16384",
                   help="comma-separated token counts of the prefill measurement")
    p.add_argument("--no-dense", action="store_true",
                   help="skip the dense small-M decoder-block qmm forward")
    p.add_argument("--no-block", action="store_true",
                   help="skip the MoE block with shared expert and combine")
    args = p.parse_args()
    args.warmup = max(args.warmup, 3)
    rank, ws, local = dist_setup(args.gpus)
    if args.impl == "reference":
        run_reference(args, rank, ws)
        return

    import torch
    import quantized_moe_expert_gather_b200 as q
    from gpu_util import dev_bf16, dev_f32, dev_u32, qweight
    from inputs import decode_scores, decode_tokens, decode_weights, prefill_layer

    q.load()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    peaks = measured_peaks()
    if args.prefill_only:
        print(json.dumps({"prefill": run_prefill(q, [args.prefill_only], dev, peaks)}), flush=True)
        return
    weights = decode_weights(0, E=args.experts)
    W = [qweight(*t, GROUP, BITS) for t in weights]

    n_layers_total = (args.warmup + args.steps) * LAYERS
    routing = [decode_tokens(100 + rank * 1_000_000 + i, M_CHAIN, E=args.experts)
               for i in range(n_layers_total)]
    idx_all = dev_u32(np.stack([r[1] for r in routing]))                    # [L, M, 8]
    sc_all = dev_f32(np.stack([decode_scores(100 + i, M_CHAIN) for i in range(n_layers_total)]))
    touched = [len(np.unique(r[1])) for r in routing]

    ws_bytes = q.qmoe_switch_glu_workspace_size(M_CHAIN, TOP_K, *W)
    ws_buf = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    ys = torch.empty((M_CHAIN * TOP_K, H), dtype=torch.bfloat16, device=dev)
    inv = torch.empty(M_CHAIN * TOP_K, dtype=torch.int32, device=dev)
    hbuf = [torch.empty((M_CHAIN, H), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    # Fixed device buffers read by the captured step: this step's input and routing.
    x_in = dev_bf16(routing[0][0])
    idx_cur = torch.empty_like(idx_all[:LAYERS])
    sc_cur = torch.empty_like(sc_all[:LAYERS])

    def step_body():
        cur = x_in
        for l in range(LAYERS):
            nxt = hbuf[l % 2]
            q.qmoe_switch_glu(cur, idx_cur[l], *W, mode=1, out=ys, inv_order=inv, workspace=ws_buf)
            q.qmoe_moe_combine(ys, inv, sc_cur[l], out=nxt)
            cur = nxt
        return cur

    def load_routing(s):
        idx_cur.copy_(idx_all[s * LAYERS:(s + 1) * LAYERS], non_blocking=True)
        sc_cur.copy_(sc_all[s * LAYERS:(s + 1) * LAYERS], non_blocking=True)

    def step_bytes(s):
        return sum(touched[s * LAYERS + l] for l in range(LAYERS)) * EXPERT_BYTES

    def capture():
        g = torch.cuda.CUDAGraph()
        n0 = q.qmoe_launch_count()
        with torch.cuda.graph(g):
            step_body()
        return g, q.qmoe_launch_count() - n0

    # eager warm-up (kernel attributes, TMA descriptor encoder), then the step graph
    load_routing(0)
    step_body()
    torch.cuda.synchronize()
    graph, launches_per_step = capture()
    for s in range(args.warmup):
        load_routing(s)
        graph.replay()
    torch.cuda.synchronize()

    # timed region: K steps, each = routing copy-in + one replay of the 42-layer graph
    stream = torch.cuda.current_stream()
    barrier(ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        e0.record(stream)
        for s in range(args.warmup, args.warmup + args.steps):
            load_routing(s)
            graph.replay()
        e1.record(stream)
        torch.cuda.synchronize()
    barrier(ws)
    ms = e0.elapsed_time(e1)
    launches = launches_per_step * args.steps
    my_bytes = sum(step_bytes(s) for s in range(args.warmup, args.warmup + args.steps))
    value, ms_max = job_gbs(my_bytes, ms, ws)
    ms_per_step = ms_max / args.steps

    # instrumented graph: the kernels' device timers around every launch of the step
    slots = torch.zeros(16 * 4 * LAYERS * 4, dtype=torch.uint8, device=dev)
    q.qmoe_timing_enable(slots)
    g_timed, _ = capture()
    sums = {k: 0.0 for k in ("qmv_glu", "qmv", "route", "combine")}
    counts = {k: 0 for k in sums}
    ug_bytes = 0
    for s in range(args.warmup, args.warmup + args.steps):
        load_routing(s)
        g_timed.replay()
        torch.cuda.synchronize()
        for k in sums:
            t, n = q.qmoe_timing_read(k)
            sums[k] += t
            counts[k] += n
        ug_bytes += sum(touched[s * LAYERS + l] for l in range(LAYERS)) * UPGATE_BYTES
    q.qmoe_timing_enable(None)
    del g_timed
    k_ms, k_n = sums["qmv_glu"], counts["qmv_glu"]
    hbm_peak = peaks["hbm_gbs"] if peaks else 6650.0
    achieved = ug_bytes / (k_ms * 1e-3) / 1e9 if k_ms > 0 else None
    roofline = {
        "kernel": "qmv_glu (fused up/gate gather_qmm + silu*mul)", "bound": "hbm",
        "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
        "frac": achieved / hbm_peak if achieved else None,
        "peak_source": "measured (MEASURED_PEAKS.json hbm_gbs)" if peaks else "fallback",
        "traffic": UPGATE_TRAFFIC_RATIO * ug_bytes / k_n if k_n else None,
        "traffic_source": "ncu dram read+write of this kernel at 64 experts, scaled by "
                          "the bytes touched",
        "launch_us": 1e3 * k_ms / k_n if k_n else None,
        "bytes_per_launch": ug_bytes / k_n if k_n else None,
        **{f"{k}_ms_in_timed_steps": v for k, v in sums.items()}, "step_total_ms": ms,
    }

    # end to end through the public API with host buffers (pinned), copies timed
    x_host = torch.from_numpy(routing[0][0].view(np.int16)).view(torch.bfloat16).pin_memory()
    idx_host = idx_all.cpu().pin_memory()
    sc_host = sc_all.cpu().pin_memory()
    out_host = torch.empty((M_CHAIN, H), dtype=torch.bfloat16).pin_memory()
    last = hbuf[(LAYERS - 1) % 2]

    def e2e_step(s):
        sl = slice(s * LAYERS, (s + 1) * LAYERS)
        x_in.copy_(x_host, non_blocking=True)
        idx_cur.copy_(idx_host[sl], non_blocking=True)
        sc_cur.copy_(sc_host[sl], non_blocking=True)
        graph.replay()
        out_host.copy_(last, non_blocking=True)

    for s in range(args.warmup):
        e2e_step(s)
    torch.cuda.synchronize()
    barrier(ws)
    e0.record(stream)
    for s in range(args.warmup, args.warmup + args.steps):
        e2e_step(s)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_gbs, _ = job_gbs(my_bytes, e0.elapsed_time(e1), ws)
    e2e = {"value": e2e_gbs, "unit": "GB/s",
           "h2d_bytes_per_step": M_CHAIN * H * 2 + LAYERS * (idx_cur[0].numel() + sc_cur[0].numel()) * 4,
           "d2h_bytes_per_step": M_CHAIN * H * 2}

    # isolated decode layers (M = 1 and M = 4): independent layers, fresh routing each
    isolated = {}
    for M in (1, 4):
        chunk, chunks = 20, 10
        n = chunk * (chunks + 1)
        rt = [decode_tokens(500_000 + M * 10_000 + i, M, E=args.experts) for i in range(n)]
        xs_all = dev_bf16(np.stack([r[0] for r in rt]))
        ids_all = dev_u32(np.stack([r[1] for r in rt]))
        scs_all = dev_f32(np.stack([decode_scores(i, M) for i in range(n)]))
        xs, ids, scs = xs_all[:chunk].clone(), ids_all[:chunk].clone(), scs_all[:chunk].clone()
        wsb = torch.empty(q.qmoe_switch_glu_workspace_size(M, TOP_K, *W), dtype=torch.uint8, device=dev)
        ysm = torch.empty((M * TOP_K, H), dtype=torch.bfloat16, device=dev)
        invm = torch.empty(M * TOP_K, dtype=torch.int32, device=dev)
        outm = torch.empty((M, H), dtype=torch.bfloat16, device=dev)

        def body():
            for i in range(chunk):
                q.qmoe_switch_glu(xs[i], ids[i], *W, mode=1, out=ysm, inv_order=invm, workspace=wsb)
                q.qmoe_moe_combine(ysm, invm, scs[i], out=outm)

        body()
        torch.cuda.synchronize()
        gi = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gi):
            body()

        def load(c):
            sl = slice(c * chunk, (c + 1) * chunk)
            xs.copy_(xs_all[sl], non_blocking=True)
            ids.copy_(ids_all[sl], non_blocking=True)
            scs.copy_(scs_all[sl], non_blocking=True)

        load(0)
        gi.replay()
        torch.cuda.synchronize()
        e0.record(stream)
        for c in range(1, chunks + 1):
            load(c)
            gi.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        t = e0.elapsed_time(e1) / (chunk * chunks)
        nb = sum(len(np.unique(r[1])) for r in rt[chunk:]) * EXPERT_BYTES / (chunk * chunks)
        isolated[f"M{M}"] = {"us_per_layer": 1e3 * t, "weight_gbs": nb / (t * 1e-3) / 1e9,
                             "unique_experts": nb / EXPERT_BYTES,
                             "p1_formula_gbs": M * TOP_K * EXPERT_BYTES / (t * 1e-3) / 1e9}
        del gi

    # prefill MoE layer (routed experts, expert-sorted, combine)
    prefill = None
    if not args.no_prefill:
        prefill = run_prefill(q, [int(t) for t in args.prefill_tokens.split(",") if t], dev,
                              peaks)

    combine = run_combine(q, dev, peaks) if not args.no_block else None
    gmm = run_gather_mm(q, dev, peaks) if not args.no_block else None
    dense = run_dense(q, dev, peaks) if not args.no_dense else None
    block = run_block(q, dev, peaks) if not args.no_block else None

    # CPU oracle on a bounded sample (rank 0, N = 1)
    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu and args.experts == E:
        with cpu_threads_limit():
            t_tot, b_tot, n = 0.0, 0, 0
            while t_tot < 10.0 and n < 4:
                t, b = oracle_decode_sample(weights, 20_000 + n)
                t_tot += t
                b_tot += b
                n += 1
        cpu = {"value": b_tot / t_tot / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
               "nproc": os.cpu_count(), "cores_available": len(os.sched_getaffinity(0)),
               "sample": f"{n} decode token(s): SwitchGLU over 8 experts + combine in fp64 "
                         f"({t_tot:.1f} s), one thread (BLAS limited to 1) of the host's "
                         f"{os.cpu_count()}"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(CONFIG, experts=args.experts), "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "clocks": clk.summary(), "gpu_launches": launches,
            "roofline_prefill": prefill_roofline(prefill, peaks),
            "decode_isolated": flat(isolated),
            "prefill": flat(prefill) if prefill else None,
            "dense_qmm": flat(dense) if dense else None,
            "moe_block": flat(block) if block else None,
            "combine": flat(combine) if combine else None,
            "gather_mm_bf16": flat(gmm) if gmm else None,
            "hbm_frac_of_measured": value / hbm_peak,
        }
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
