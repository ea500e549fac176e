"""GPU parity at the benchmarked sizes, on sampled rows the oracle can afford.

* Prefill MoE layer (hidden 2048, intermediate 512, 256 experts, top-8, 4-bit group 64,
  Zipf-skewed routing) at T = 1024, 2048, 4123, 8192 and 16384 tokens: the expert-sorted
  SwitchGLU output (mode 1) is compared with the oracle on every row of the heaviest
  expert's first and last 192-row tile, the first row and the last eight rows of every
  touched expert (its ragged last tile), the last tiles of the three heaviest experts and
  1000 random rows; the inverse permutation is compared bit for bit in full.  The token
  counts are those of MLX PR #4567's Results table.
* Full MoE block (the same routed experts, a shared SwiGLU expert of intermediate 512 and
  a sigmoid-gated shared output, one-pass combine) at T = 128, 331, 2048 and 4096 rows in
  4-bit group 64 and 8-bit group 128 (MTPLX PR #558, Tests: the row counts of its block
  checks): the routed rows as above, and the block output on 160 sampled tokens, whose
  oracle chain feeds its own bf16 expert and shared outputs to its combine.
* Unquantized gather_mm on the benchmarked workload (2048 -> 512, 256 experts, Zipf top-8)
  at T = 4096 and 16384 tokens, on sampled routed rows.

Tolerance as everywhere: |got - want| <= 8e-3 * max|want| over the compared values.
"""

import numpy as np
import pytest
import torch

import oracle as O
from gpu_util import assert_close, dev_bf16, dev_f32, dev_u32, host_u32, qweight
from inputs import prefill_layer

pytestmark = pytest.mark.gpu

TOP_K = 8


PLANS = {  # name -> environment of the plan
    "auto": {},                                                   # the library's own plan
    "tc_smem": {"QMOE_FORCE_KERNEL": "tc", "QMOE_PREFILL": "tc"},  # weights staged in smem
    "qmv": {"QMOE_FORCE_KERNEL": "qmv"},                          # the streaming kernel
}


def _set_plan(monkeypatch, name):
    for k in ("QMOE_PREFILL", "QMOE_FORCE_KERNEL"):
        monkeypatch.delenv(k, raising=False)
    for k, v in PLANS[name].items():
        monkeypatch.setenv(k, v)


def sample_positions(offsets, seed, n_random=1000, tile=192):
    """Expert-sorted positions to check: tile edges of the heaviest experts, the ragged
    end of every touched expert, and random rows."""
    offsets = np.asarray(offsets, np.int64)
    counts = np.diff(offsets)
    R = int(offsets[-1])
    pos = []
    heavy = np.argsort(-counts, kind="stable")[:3]
    e0 = int(heavy[0])
    pos.append(np.arange(offsets[e0], min(offsets[e0] + tile, offsets[e0 + 1])))
    for e in heavy:
        e = int(e)
        c = int(counts[e])
        last = offsets[e] + ((c - 1) // tile) * tile if c else offsets[e]
        pos.append(np.arange(last, offsets[e + 1]))
    for e in np.nonzero(counts)[0]:
        pos.append([offsets[e]])
        pos.append(np.arange(max(offsets[e], offsets[e + 1] - 8), offsets[e + 1]))
    pos.append(np.random.default_rng(seed).choice(R, size=min(n_random, R), replace=False))
    return np.unique(np.concatenate([np.asarray(p, np.int64) for p in pos]))


def oracle_rows(d, rows, group, bits):
    """The oracle's SwitchGLU output of the given routed rows r = t*top_k + k."""
    t = rows // TOP_K
    e = d["idx"].reshape(-1)[rows].astype(np.int64)
    experts = np.unique(e)
    sel = lambda wt: (wt[0][experts], wt[1][experts], wt[2][experts], group, bits)  # noqa: E731
    y, _ = O.switch_glu(d["x"][t], np.searchsorted(experts, e)[:, None], sel(d["up"]),
                        sel(d["gate"]), sel(d["down"]))
    return y[:, 0]


_CACHE = {}


def _layer(T, group=64, bits=4, shared=False):
    key = (T, group, bits, shared)
    if key not in _CACHE:
        _CACHE.clear()  # one workload at a time (T = 16384 holds ~0.5 GB of host arrays)
        d = prefill_layer(0, T, group=group, bits=bits, shared=shared)
        order, inv, offsets = O.sort_by_expert(d["idx"].reshape(-1), d["E"])
        pos = sample_positions(offsets, seed=T)
        d.update(order=order, inv=inv, offsets=offsets, pos=pos,
                 want_pos=oracle_rows(d, order[pos], group, bits))
        _CACHE[key] = d
    return _CACHE[key]


def _check_sorted_rows(name, d, ys, inv):
    assert np.array_equal(host_u32(inv), d["inv"].astype(np.uint32)), f"{name}: inv_order"
    got = ys[torch.from_numpy(d["pos"]).cuda()]
    return assert_close(f"{name}: {d['pos'].size} sampled sorted rows", got, d["want_pos"])


@pytest.mark.parametrize("T", [1024, 2048, 4123, 8192, 16384])
def test_prefill_layer_full_size(gpu_lib, monkeypatch, T):
    """Each plan in turn on the same workload (the library's own, the shared-memory
    tensor-core kernel, the streaming kernel)."""
    q = gpu_lib
    d = _layer(T)
    W = [qweight(*d[k], 64, 4) for k in ("up", "gate", "down")]
    x, idx = dev_bf16(d["x"]), dev_u32(d["idx"])
    for name in PLANS:
        _set_plan(monkeypatch, name)
        ys, inv = q.qmoe_switch_glu(x, idx, *W, mode=1)
        torch.cuda.synchronize()
        _check_sorted_rows(f"prefill T={T} [{name}]", d, ys, inv)
        del ys, inv


@pytest.mark.parametrize("T", [128, 331, 2048, 4096])
@pytest.mark.parametrize("bits,group", [(4, 64), (8, 128)])
def test_moe_block_full_size(gpu_lib, monkeypatch, T, bits, group):
    q = gpu_lib
    _set_plan(monkeypatch, "auto")
    d = _layer(T, group, bits, shared=True)
    W = [qweight(*d[k], group, bits) for k in ("up", "gate", "down")]
    S = [qweight(*d[k], group, bits) for k in ("sh_up", "sh_gate", "sh_down")]
    xd = dev_bf16(d["x"])
    ys, inv = q.qmoe_switch_glu(xd, dev_u32(d["idx"]), *W, mode=1)
    zeros = torch.zeros((T, 1), dtype=torch.int32, device="cuda")
    sh = q.qmoe_switch_glu(xd, zeros, *S, mode=0).reshape(T, -1)
    out = q.qmoe_moe_combine(ys, inv, dev_f32(d["scores"]), sh, xd, dev_bf16(d["w_sg"]))
    torch.cuda.synchronize()
    _check_sorted_rows(f"block T={T} {bits}-bit g{group} routed", d, ys, inv)

    # the block output of sampled tokens, from the oracle's own chain
    toks = np.sort(np.random.default_rng(T + bits).choice(T, size=min(160, T), replace=False))
    rows = (toks[:, None] * TOP_K + np.arange(TOP_K)[None, :]).reshape(-1)
    y_tok = oracle_rows(d, rows, group, bits)                               # [n*top_k, H]
    sh_want, _ = O.switch_glu(d["x"][toks], np.zeros((toks.size, 1), np.int64),
                              (*d["sh_up"], group, bits), (*d["sh_gate"], group, bits),
                              (*d["sh_down"], group, bits))
    y_b = O.bf16_from_f64(y_tok)
    sh_b = O.bf16_from_f64(sh_want[:, 0])
    want = O.moe_combine(y_b, np.arange(rows.size), d["scores"][toks], sh_b, d["x"][toks],
                         d["w_sg"])
    assert_close(f"block T={T} {bits}-bit g{group} output of {toks.size} tokens",
                 out[torch.from_numpy(toks).cuda()], want)


_GMM = {}


def _gather_mm_case(T):
    """The bench's gather_mm workload (the weights, then the activations of T = 4096 and of
    T = 16384 from the same seeded stream), the sampled routed rows of T tokens and the
    oracle's values there (over the sampled rows' experts only)."""
    from inputs import normal_bf16, prefill_routing
    E, K, N = 256, 2048, 512
    if "w" not in _GMM:
        rng = np.random.default_rng(21)
        _GMM["w"] = normal_bf16(rng, (E, N, K), 1 / np.sqrt(K))
        _GMM["x"] = {t: normal_bf16(rng, (t, 1, K)) for t in (4096, 16384)}
    if _GMM.get("T") != T:
        w, x = _GMM["w"], _GMM["x"][T]
        idx, _ = prefill_routing(0, T, E, TOP_K)
        rhs = idx.reshape(-1).astype(np.uint32)
        order, _, offsets = O.sort_by_expert(rhs, E)
        b = np.sort(order[sample_positions(offsets, seed=T)].astype(np.int64))
        ue = np.unique(rhs[b])
        want = O.gather_mm(x[b // TOP_K], w[ue], np.arange(b.size), np.searchsorted(ue, rhs[b]))
        _GMM.update(T=T, case=(x, w, rhs, b, want))
    return _GMM["case"]


@pytest.mark.parametrize("T", [4096, 16384])
def test_gather_mm_full_size(gpu_lib, monkeypatch, T):
    """Unquantized gather_mm on the benchmarked workload (hidden 2048 -> 512, 256 experts,
    Zipf-skewed top-8 routing of T tokens, x broadcast over each token's experts; MLX PR
    #4567, Description: the gather_mm whose row tiles the page reorganises), compared with
    the oracle on sampled routed rows chosen as for the prefill layer."""
    q = gpu_lib
    _set_plan(monkeypatch, "auto")
    x, w, rhs, b, want = _gather_mm_case(T)
    got = q.qmoe_gather_mm(dev_bf16(x), dev_bf16(w), None, dev_u32(rhs))
    torch.cuda.synchronize()
    assert_close(f"gather_mm T={T}: {b.size} sampled rows",
                 got[torch.from_numpy(b).cuda()], want)
