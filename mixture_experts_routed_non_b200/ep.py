"""Expert-parallel dispatch and combine around the local path (non-expand),
host side: the order of the phases across ranks, the exchange of send counts
and the receive buffers.  Every data movement runs in the CUDA library
(``moe_ep_layout``, ``moe_ep_dispatch``, ``moe_ep_combine``); this module only
marshals pointers and offsets.

The dataflow is that of "End-to-end DeepEP v2 non-expand + SonicMoE
integration #68": dispatch (non-expand) -> recv_x / recv_topk_idx (local
ids, -1 for slots whose expert lives on another rank) / recv_topk_weights ->
the local expert compute (``binding.forward``) -> local_out -> combine ->
routed_out in the source's token order.

Two ways to hold the ranks:

* ``EmulatedRanks``: R ranks' buffers on one GPU.  The kernels see every
  rank's buffers as ordinary device pointers; each phase runs for every rank
  in turn, so no kernel waits on another.
* ``ProcessGroupRanks``: one process per GPU.  Send counts are all-gathered
  over the process group; receive and output buffers have a fixed capacity
  and are opened by the peers through CUDA IPC handles exchanged over the
  group; barriers separate the phases.  The kernels then store and load
  across NVLink with plain peer accesses.
"""
from __future__ import annotations

from typing import List, Optional, Sequence

import numpy as np
import torch

from . import binding


def block_offsets(counts: np.ndarray):
    """``counts[s, d]`` rows from source s to destination d -> ``off[d, s]``,
    the first receive row of source s's block on d (blocks in source order),
    and ``n_recv[d]``."""
    counts = np.asarray(counts, np.int64)
    n_recv = counts.sum(axis=0)
    off = np.zeros_like(counts)
    off[:, 1:] = np.cumsum(counts.T, axis=1)[:, :-1]
    return off, n_recv


def expert_slice(t: Optional[torch.Tensor], d: int, E_local: int) -> Optional[torch.Tensor]:
    """Rank d's experts of a global [R*E_local, ...] weight (or None)."""
    return None if t is None else t[d * E_local:(d + 1) * E_local]


class EmulatedRanks:
    """R ranks on one GPU: rank d's receive buffers and local_out live in this
    GPU's memory, and the per-rank kernels run one after another."""

    def __init__(self, R: int, E_local: int, device=None):
        if not (1 <= R <= binding.EP_MAX_RANKS):
            raise ValueError(f"EmulatedRanks: 1 <= R <= {binding.EP_MAX_RANKS}")
        self.R, self.E_local = R, E_local
        self.device = torch.device(device) if device is not None else torch.device("cuda")

    def dispatch(self, xs: Sequence[torch.Tensor], idxs: Sequence[torch.Tensor], ws: Sequence[torch.Tensor],
                 err: Optional[torch.Tensor] = None) -> dict:
        R, E_local = self.R, self.E_local
        layouts = [binding.ep_layout(idxs[s], R, E_local, err=err) for s in range(R)]
        counts = torch.stack([c for _, c in layouts]).cpu().numpy()  # the exchange of counts
        off, n_recv = block_offsets(counts)
        H, K = xs[0].shape[1], idxs[0].shape[1]
        # at least one row each, so that every pointer is valid
        recv_x = [torch.empty((max(int(n), 1), H), dtype=torch.bfloat16, device=self.device) for n in n_recv]
        recv_idx = [torch.empty((max(int(n), 1), K), dtype=torch.int32, device=self.device) for n in n_recv]
        recv_w = [torch.empty((max(int(n), 1), K), dtype=torch.float32, device=self.device) for n in n_recv]
        for s in range(R):
            peers = binding.ep_peers(recv_x, recv_idx, recv_w, off[:, s])
            binding.ep_dispatch(xs[s], idxs[s], ws[s], layouts[s][0], E_local, peers, R)
        return {"recv_x": [recv_x[d][:int(n_recv[d])] for d in range(R)],
                "recv_idx": [recv_idx[d][:int(n_recv[d])] for d in range(R)],
                "recv_w": [recv_w[d][:int(n_recv[d])] for d in range(R)],
                "send_idx": [l[0] for l in layouts], "counts": counts, "off": off, "n_recv": n_recv,
                "_bufs": (recv_x, recv_idx, recv_w)}

    def combine(self, local_outs: Sequence[torch.Tensor], state: dict, H: int) -> List[torch.Tensor]:
        R = self.R
        # a rank that received nothing still needs a valid (unread) pointer
        lo = [t if t.shape[0] else torch.empty((1, H), dtype=torch.bfloat16, device=self.device) for t in local_outs]
        return [binding.ep_combine(binding.ep_sources(lo, state["off"][:, s]), state["send_idx"][s], H)
                for s in range(R)]

    def forward(self, xs, idxs, ws, w1, w2, b1=None, b2=None, layout: int = 0) -> List[torch.Tensor]:
        """dispatch -> every rank's local forward over its experts -> combine."""
        st = self.dispatch(xs, idxs, ws)
        H = xs[0].shape[1]
        local = []
        for d in range(self.R):
            if st["recv_x"][d].shape[0] == 0:
                local.append(st["recv_x"][d])
                continue
            local.append(binding.forward(st["recv_x"][d], st["recv_idx"][d], st["recv_w"][d],
                                         expert_slice(w1, d, self.E_local), expert_slice(w2, d, self.E_local),
                                         expert_slice(b1, d, self.E_local), expert_slice(b2, d, self.E_local),
                                         layout=layout))
        return self.combine(local, st, H)


def exchange_counts(send_count: torch.Tensor, group=None) -> np.ndarray:
    """All-gather of every rank's send counts [R] -> counts [R, R] (row =
    source).  Works with gloo (CPU tensors) and NCCL (device tensors)."""
    import torch.distributed as dist
    R = dist.get_world_size(group)
    parts = [torch.empty_like(send_count) for _ in range(R)]
    dist.all_gather(parts, send_count, group=group)
    return torch.stack(parts).cpu().numpy()


class ProcessGroupRanks:
    """One process per GPU.  Buffers of ``capacity`` receive rows per rank
    (R * T_max covers any routing) are allocated once; every rank opens its
    peers' buffers through CUDA IPC handles exchanged over the group.

    Phases per call: layout -> all-gather of counts -> dispatch (peer stores)
    -> barrier -> local forward -> barrier -> combine (peer loads) -> barrier.
    Tested on one GPU with a one-rank NCCL group (count all-gather, barriers,
    buffers; no IPC), and on two gloo ranks on CPU with stand-ins for the
    library calls and file-shared buffers in place of IPC (count exchange,
    block offsets, capacity check, buffer slicing, combine sources); the tests
    do not run it on more than one GPU.
    """

    def __init__(self, E_local: int, capacity: int, H: int, K: int, group=None, device=None, opener=None):
        import torch.distributed as dist
        self.group = group
        self.R = dist.get_world_size(group)
        self.me = dist.get_rank(group)
        self.E_local, self.capacity, self.H, self.K = E_local, capacity, H, K
        self.device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.recv_x = torch.empty((capacity, H), dtype=torch.bfloat16, device=self.device)
        self.recv_idx = torch.empty((capacity, K), dtype=torch.int32, device=self.device)
        self.recv_w = torch.empty((capacity, K), dtype=torch.float32, device=self.device)
        self.local_out = torch.empty((capacity, H), dtype=torch.bfloat16, device=self.device)
        mine = (self.recv_x, self.recv_idx, self.recv_w, self.local_out)
        self.peer = self._open_peers(mine, opener)

    def _open_peers(self, mine, opener):
        """Per rank, the four buffers as tensors of this process: its own, or
        the peer's opened from the IPC handle it published."""
        import torch.distributed as dist
        from torch.multiprocessing.reductions import reduce_tensor
        if self.R == 1:
            return [mine]
        handles = [None] * self.R
        dist.all_gather_object(handles, [reduce_tensor(t) for t in mine], group=self.group)
        out = []
        for d in range(self.R):
            if d == self.me:
                out.append(mine)
            else:
                open_one = opener or (lambda h: h[0](*h[1]))
                out.append(tuple(open_one(h) for h in handles[d]))
        return out

    def _barrier(self):
        import torch.distributed as dist
        torch.cuda.synchronize(self.device)
        dist.barrier(group=self.group)

    def forward(self, x, topk_idx, topk_w, w1_local, w2_local, b1_local=None, b2_local=None, layout: int = 0):
        """This rank's routed_out [T,H] for its tokens; w*_local hold this
        rank's experts."""
        R, E_local, H = self.R, self.E_local, self.H
        send_idx, send_count = binding.ep_layout(topk_idx, R, E_local)
        counts = exchange_counts(send_count, self.group)
        off, n_recv = block_offsets(counts)
        if int(n_recv.max()) > self.capacity:
            raise ValueError("ProcessGroupRanks: receive rows exceed the capacity")
        peers = binding.ep_peers([p[0] for p in self.peer], [p[1] for p in self.peer], [p[2] for p in self.peer],
                                 off[:, self.me])
        binding.ep_dispatch(x, topk_idx, topk_w, send_idx, E_local, peers, R)
        self._barrier()  # every rank's rows have landed
        n = int(n_recv[self.me])
        if n:
            binding.forward(self.recv_x[:n], self.recv_idx[:n], self.recv_w[:n], w1_local, w2_local, b1_local,
                            b2_local, layout=layout, out=self.local_out[:n])
        self._barrier()  # every rank's local_out is complete
        out = binding.ep_combine(binding.ep_sources([p[3] for p in self.peer], off[:, self.me]), send_idx, H)
        self._barrier()  # no rank reuses its buffers while a peer still reads them
        return out
