"""Expert-parallel MoE layer: the routed experts spread over R ranks, one GPU
each, with the tokens data-parallel ("K2 inference engineer's answer", 2.1:
EP = 128 with two or three routed experts per rank for DeepSeek-V3 and about
10 GB of expert weights per rank for K2; 2.4: n_group = 1, so any token may
select any rank's experts).

Rank q owns the routed experts [q E/R, (q+1) E/R); the router, its bias and the
shared expert are replicated; every rank routes its own tokens.  One forward
pass on every rank:

  1. moe_ep_dispatch      route, permute, gather the token rows (expert-major,
                          so the rows for rank q are one contiguous block)
  2. all-to-all           the per-expert row counts ([R, E/R] ints)
  3. all-to-all           the token rows, split by those counts
  4. moe_ep_expert_ffn    the rank's experts on the received rows
  5. all-to-all           the expert outputs back to their sources
  6. moe_ep_combine       the shared expert on the rank's own tokens, plus the
                          weighted sum of the returned rows in slot order

Every step of the layer's arithmetic runs in the library's kernels; this module
only sizes buffers and calls the exchange.  The exchange is `comm.all_to_all`:
TorchComm wraps torch.distributed (NCCL between GPUs).  Steps 3 and 5 need the
split sizes on the host, so a call reads the counts back twice (one small
device-to-host copy each).  Each rank's output equals moe_layer_forward on its
own tokens bit for bit: every row meets the same kernels in the same K order.
"""
from __future__ import annotations

import sys

import torch


class TorchComm:
    """All-to-all over a torch.distributed process group (NCCL for CUDA
    tensors, gloo for CPU tensors)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self._dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def all_to_all(self, out, inp, out_splits, in_splits):
        """Rows [sum(in_splits), ...] of `inp`, split along dim 0, go to the ranks
        in order; `out` receives [sum(out_splits), ...] rows from them."""
        self._dist.all_to_all_single(out, inp, list(out_splits), list(in_splits), group=self.group)


class ExpertParallelMoE:
    """One MoE FFN layer whose routed experts are split over `comm.world` ranks.

    w_gate_up / w_down are this rank's E/R experts ([E/R, 2*inter, d] and
    [E/R, d, inter] bf16, contiguous); w_router [E, d], bias [E] and the shared
    expert (ws_gate_up [2*inter, d], ws_down [d, inter]) are the full, replicated
    tensors.  `ops` provides the layer's kernels (default: this package's CUDA
    library)."""

    def __init__(self, comm, w_router, bias, w_gate_up, w_down, ws_gate_up, ws_down, k: int,
                 scale: float, ops=None):
        # the package's CUDA library unless the caller provides the kernels
        self.ops = ops if ops is not None else sys.modules[__package__]
        self.comm = comm
        self.R = comm.world
        self.E = w_router.shape[0]
        if self.E % self.R:
            raise ValueError(f"E = {self.E} experts do not split evenly over {self.R} ranks")
        self.El = self.E // self.R
        if w_gate_up.shape[0] != self.El or w_down.shape[0] != self.El:
            raise ValueError(f"rank holds {w_gate_up.shape[0]} experts, expected E/R = {self.El}")
        self.w_router, self.bias = w_router, bias
        self.w_gate_up, self.w_down = w_gate_up, w_down
        self.ws_gate_up, self.ws_down = ws_gate_up, ws_down
        self.k, self.scale = k, scale
        self.inter = ws_gate_up.shape[0] // 2

    def _ws(self, nbytes, dev):
        return torch.empty((max(int(nbytes), 16),), dtype=torch.uint8, device=dev)

    def forward(self, x, out):
        """out [T, d] bf16 = the layer on this rank's tokens x [T, d] bf16."""
        ops, comm, R, El, k = self.ops, self.comm, self.R, self.El, self.k
        T, d = x.shape
        dev = x.device
        # 1. route, permute, gather
        idx = torch.empty((T, k), dtype=torch.int32, device=dev)
        w = torch.empty((T, k), dtype=torch.float32, device=dev)
        counts = torch.empty((self.E,), dtype=torch.int32, device=dev)
        slot_row = torch.empty((T * k,), dtype=torch.int32, device=dev)
        send = torch.empty((T * k, d), dtype=x.dtype, device=dev)
        if T > 0:
            ops.moe_ep_dispatch(x, self.w_router, self.bias, k, self.scale, idx, w, counts,
                                slot_row, send,
                                self._ws(ops.moe_ep_dispatch_workspace_size(T, d, self.E, k), dev))
        else:
            counts.zero_()
        # 2. counts: rank q gets this rank's counts of its experts
        recv_counts = torch.empty((R, El), dtype=torch.int32, device=dev)
        comm.all_to_all(recv_counts.view(-1), counts, [El] * R, [El] * R)
        # split sizes on the host (two small reads back)
        send_splits = counts.cpu().view(R, El).sum(1).tolist()
        recv_splits = recv_counts.cpu().sum(1).tolist()
        rows = int(sum(recv_splits))
        # 3. token rows to the experts' ranks
        recv = torch.empty((rows, d), dtype=x.dtype, device=dev)
        comm.all_to_all(recv, send, recv_splits, send_splits)
        # 4. this rank's experts
        y = torch.empty((rows, d), dtype=x.dtype, device=dev)
        if rows > 0:
            ops.moe_ep_expert_ffn(
                recv, recv_counts, self.w_gate_up, self.w_down, y,
                self._ws(ops.moe_ep_expert_ffn_workspace_size(rows, d, R, El, self.inter), dev))
        # 5. outputs back to their sources, in send order
        y_back = torch.empty((T * k, d), dtype=x.dtype, device=dev)
        comm.all_to_all(y_back, y, send_splits, recv_splits)
        # 6. shared expert + combine
        if T > 0:
            ops.moe_ep_combine(y_back, x, self.ws_gate_up, self.ws_down, w, slot_row, out,
                               self._ws(ops.moe_ep_combine_workspace_size(T, d, self.inter), dev))
        return out
