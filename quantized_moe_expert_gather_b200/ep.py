"""Expert-parallel MoE layer over ``torch.distributed`` (one process per GPU).

The experts are partitioned contiguously over the ranks of a process group: rank r owns
experts ``[r*E_local, (r+1)*E_local)``.  A layer call on every rank, with its own tokens:

1. ``qmoe_sort_by_expert`` sorts the routed rows ``t*top_k + k`` by expert (MTPLX PR #558,
   Change: the sorted chain).  In expert order the rows are grouped by owner rank, and the
   per-rank send counts are differences of the expert offsets.
2. ``qmoe_ep_pack`` writes the rows to send (the activation row of each sorted routed
   row) and each row's expert number on its owner.
3. One ``all_to_all_single`` sends the rows, another their expert numbers, to the owners
   (the counts go first, so every rank knows what it receives).
4. The owner runs its experts on what it received: ``qmoe_switch_glu`` with one expert per
   row (top_k = 1), outputs in received order.
5. ``all_to_all_single`` with the counts reversed returns every output to its sender, in
   the sender's expert order.
6. ``qmoe_moe_combine`` unsorts with the sort's inverse permutation, weights by the
   routing scores, sums over top_k and adds the gated shared expert (MTPLX PR #558,
   Summary).

Every step on the data path is a library kernel or a collective; the Python here moves
the per-rank counts to the host (the collectives take their split sizes as integers) and
allocates buffers.  The collectives run on the process group's backend (NCCL over
NVLink on GPUs).  Routed rows whose expert index is out of range are not sent; their
outputs stay zero (and the sort flags them).
"""

from __future__ import annotations


import torch
import torch.distributed as dist

import quantized_moe_expert_gather_b200 as q


class LibraryOps:
    """The library's kernels for the local steps of the layer (the only ops the layer
    uses outside tests)."""

    def sort(self, indices: torch.Tensor, num_experts: int):
        return q.qmoe_sort_by_expert(indices.reshape(-1), num_experts)

    def pack(self, x, indices, order, e_local: int):
        return q.qmoe_ep_pack(x, indices, order, e_local)

    def experts(self, x_recv, e_recv, up, gate, down):
        n, H = x_recv.shape
        if n == 0:
            return torch.empty((0, H), dtype=torch.bfloat16, device=x_recv.device)
        y = q.qmoe_switch_glu(x_recv, e_recv.reshape(n, 1), up, gate, down, mode=0)
        return y.reshape(n, H)

    def combine(self, y_sorted, inv_order, scores, shared=None, x=None, w_shared_gate=None):
        return q.qmoe_moe_combine(y_sorted, inv_order, scores, shared, x, w_shared_gate)


class ExpertParallelMoE:
    """One MoE layer whose experts are spread over the ranks of ``group``.

    ``up``, ``gate``, ``down``: this rank's ``E_local = num_experts / world_size`` experts
    (``q.QWeight`` stacks on this rank's device; anything the ``ops`` object accepts).
    ``ops`` defaults to the library's kernels; tests substitute their own."""

    def __init__(self, up, gate, down, num_experts: int, group=None, ops=None):
        self.group = group
        self.ws = dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if self.ws > 1 else 0
        if num_experts % self.ws != 0:
            raise ValueError("num_experts must be a multiple of the world size")
        self.E = num_experts
        self.E_local = num_experts // self.ws
        self.up, self.gate, self.down = up, gate, down
        self.ops = ops if ops is not None else LibraryOps()

    def _all_to_all(self, out, inp, out_splits, in_splits):
        if self.ws == 1:
            out.copy_(inp)
        else:
            dist.all_to_all_single(out, inp, out_splits, in_splits, group=self.group)

    def split_counts(self, offsets) -> list:
        """Rows this rank sends to each rank: the rows of that rank's experts."""
        off = [int(v) for v in offsets.reshape(-1).tolist()]
        return [off[(r + 1) * self.E_local] - off[r * self.E_local] for r in range(self.ws)]

    def __call__(self, x, indices, scores, shared=None, w_shared_gate=None):
        """x [T, H] bf16, indices [T, top_k] expert ids, scores [T, top_k] float32;
        returns out [T, H] bf16 on this rank (the combine's output)."""
        T, H = x.shape
        top_k = indices.shape[1]
        R = T * top_k
        order, inv, offsets = self.ops.sort(indices, self.E)
        send = self.split_counts(offsets)
        valid = sum(send)
        x_send, e_send = self.ops.pack(x, indices, order, self.E_local)
        # counts first: what every rank receives from every other
        dev = x.device
        send_t = torch.tensor(send, dtype=torch.int64, device=dev)
        recv_t = torch.empty_like(send_t)
        self._all_to_all(recv_t, send_t, [1] * self.ws, [1] * self.ws)
        recv = [int(v) for v in recv_t.tolist()]
        n_recv = sum(recv)
        x_recv = torch.empty((n_recv, H), dtype=x_send.dtype, device=dev)
        e_recv = torch.empty(n_recv, dtype=e_send.dtype, device=dev)
        self._all_to_all(x_recv, x_send[:valid], recv, send)
        self._all_to_all(e_recv, e_send[:valid], recv, send)
        y_recv = self.ops.experts(x_recv, e_recv, self.up, self.gate, self.down)
        # outputs back to their senders, in the senders' expert order; rows with an
        # invalid expert index (sorted after the valid ones) stay zero
        y_sorted = torch.zeros((R, H), dtype=y_recv.dtype, device=dev)
        self._all_to_all(y_sorted[:valid], y_recv, send, recv)
        return self.ops.combine(y_sorted, inv, scores, shared,
                                x if w_shared_gate is not None else None, w_shared_gate)
