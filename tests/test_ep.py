"""Expert-parallel MoE layer (``quantized_moe_expert_gather_b200.ep``).

* Two and four gloo ranks on CPU: the layer's exchange (counts, dispatch of rows and expert numbers,
  return of the outputs, reassembly in expert order) with the local steps done by the
  oracle.  Each rank's result equals, bit for bit, the single-process oracle layer on its
  own tokens with every expert (the same rounding points), so the dispatch and combine
  permutations are exact.
* One GPU (world size 1): the layer through the library's kernels (expert sort, the
  dispatch packing, SwitchGLU, combine) against the oracle.
"""

import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
E, H, I, TOP_K, GROUP, BITS = 8, 64, 32, 2, 32, 4


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


class OracleOps:
    """The layer's local steps done by the oracle, on CPU tensors (test infrastructure)."""

    def __init__(self, O):
        self.O = O

    def sort(self, indices, num_experts):
        order, inv, off = self.O.sort_by_expert(indices.numpy().reshape(-1).astype(np.int64),
                                                 num_experts)
        return (torch.from_numpy(order.astype(np.int32)), torch.from_numpy(inv.astype(np.int32)),
                torch.from_numpy(off.astype(np.int64)))

    def pack(self, x, indices, order, e_local):
        o = order.numpy().astype(np.int64)
        top_k = indices.shape[1]
        x_send = _bits(x)[o // top_k]
        e_send = indices.numpy().reshape(-1).astype(np.int64)[o] % e_local
        return _bf16(x_send), torch.from_numpy(e_send.astype(np.int32))

    def experts(self, x_recv, e_recv, up, gate, down):
        n = x_recv.shape[0]
        if n == 0:
            return torch.empty((0, H), dtype=torch.bfloat16)
        y, _ = self.O.switch_glu(_bits(x_recv), e_recv.numpy().astype(np.int64)[:, None], up,
                                 gate, down)
        return _bf16(self.O.bf16_from_f64(y[:, 0]))

    def combine(self, y_sorted, inv, scores, shared=None, x=None, w_shared_gate=None):
        return torch.from_numpy(self.O.moe_combine(_bits(y_sorted), inv.numpy(), scores.numpy()))


def _global_weights():
    from inputs import random_qweight
    rng = np.random.default_rng(5)
    return [random_qweight(rng, E, n, k, GROUP, BITS) for n, k in ((I, H), (I, H), (H, I))]


def _token_count(rank, ws):
    """Routed tokens of a rank: different on every rank; with four ranks, rank 2 has none."""
    return 0 if (ws == 4 and rank == 2) else 5 + 2 * rank


def _tokens(rank, ws):
    from inputs import normal_bf16
    rng = np.random.default_rng(100 + rank)
    T = _token_count(rank, ws)
    x = normal_bf16(rng, (T, H))
    idx = np.array([rng.choice(E, size=TOP_K, replace=False) for _ in range(T)],
                   np.uint32).reshape(T, TOP_K)
    p = rng.random((T, TOP_K)).astype(np.float32)
    return x, idx, (p / p.sum(axis=1, keepdims=True)).astype(np.float32)


def _reference(O, x, idx, scores, weights):
    """The single-process oracle layer with the same rounding points as the EP layer: each
    expert output rounded to bf16 once, then the combine in fp64."""
    up, gate, down = ((*w, GROUP, BITS) for w in weights)
    y, _ = O.switch_glu(x, idx.astype(np.int64), up, gate, down)
    order, inv, _ = O.sort_by_expert(idx.reshape(-1).astype(np.int64), E)
    y_sorted = O.bf16_from_f64(y.reshape(-1, H)[order])
    return O.moe_combine(y_sorted, inv, scores)


def _rank_main(rank, ws, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime

    import torch.distributed as dist

    import oracle as O
    from quantized_moe_expert_gather_b200.ep import ExpertParallelMoE
    dist.init_process_group("gloo", rank=rank, world_size=ws,
                            timeout=datetime.timedelta(seconds=60))
    weights = _global_weights()
    el = E // ws
    local = [(w[rank * el:(rank + 1) * el], s[rank * el:(rank + 1) * el],
              b[rank * el:(rank + 1) * el], GROUP, BITS) for (w, s, b) in weights]
    layer = ExpertParallelMoE(*local, num_experts=E, ops=OracleOps(O))
    x, idx, sc = _tokens(rank, ws)
    got = layer(_bf16(x), torch.from_numpy(idx.view(np.int32)), torch.from_numpy(sc))
    want = _reference(O, x, idx, sc, weights) if x.shape[0] else np.zeros((0, H), np.uint16)
    order, _, off = O.sort_by_expert(idx.reshape(-1).astype(np.int64), E)
    out[rank] = (bool(np.array_equal(got.numpy(), want)), layer.split_counts(torch.from_numpy(off)),
                 float(np.abs(got.numpy() - want).max()) if want.size else 0.0)
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("ws", [2, 4])
def test_expert_parallel_gloo_ranks_match_the_oracle_layer_bitwise(ws):
    """Two ranks (four experts each), and four ranks (two each) of which one routes no
    tokens but still serves its experts to the others."""
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(ws, _free_port(), out), nprocs=ws,
                           start_method="spawn", join=True)
        got = dict(out)
    for rank in range(ws):
        equal, sends, err = got[rank]
        assert equal, f"rank {rank}: max |got - want| = {err}"
        assert sum(sends) == _token_count(rank, ws) * TOP_K  # each routed row to one owner


@pytest.mark.gpu
def test_expert_parallel_layer_one_gpu(gpu_lib):
    """World size 1 through the library's kernels: the layer equals the oracle layer."""
    import oracle as O
    from gpu_util import assert_close, dev_bf16, dev_f32, dev_u32, qweight
    from quantized_moe_expert_gather_b200.ep import ExpertParallelMoE
    weights = _global_weights()
    W = [qweight(*w, GROUP, BITS) for w in weights]
    layer = ExpertParallelMoE(*W, num_experts=E)
    for rank in range(2):
        x, idx, sc = _tokens(rank, 1)
        got = layer(dev_bf16(x), dev_u32(idx), dev_f32(sc))
        torch.cuda.synchronize()
        assert_close(f"EP layer tokens {rank}", got, _reference(O, x, idx, sc, weights))
