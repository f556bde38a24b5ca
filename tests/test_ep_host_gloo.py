"""The one-process-per-GPU expert-parallel host path (``ProcessGroupRanks``)
on two gloo ranks on CPU.

The library calls are replaced by CPU stand-ins written from the oracle's
definitions (test code), and the receive and output buffers are shared
between the two processes through file-backed memory in place of CUDA IPC.
What is under test is the host side of ``ProcessGroupRanks.forward``: the
exchange of send counts, the receive-block offsets every rank derives, the
capacity check, the slicing of the receive buffers for the local forward, and
the order of the combine's sources.  Each rank's routed output must match the
oracle's forward over all experts within the expert-parallel tolerance.
"""
from __future__ import annotations

import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

R, E_LOCAL, H, I, K = 2, 4, 64, 64, 3
T_OF = (24, 17)          # tokens per source rank (ragged)
CAPACITY = 48


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(rank: int):
    """Rank ``rank``'s tokens and the global weights (seeded, bf16)."""
    import torch
    g = torch.Generator().manual_seed(100 + rank)
    T = T_OF[rank]
    x = torch.randn(T, H, generator=g).to(torch.bfloat16)
    rng = np.random.default_rng(200 + rank)
    E = R * E_LOCAL
    idx = np.full((T, K), -1, np.int32)
    for t in range(T):
        m = int(rng.integers(0, K + 1))                 # 0..K valid slots
        idx[t, rng.permutation(K)[:m]] = rng.permutation(E)[:m]
    idx[0] = [0, 1, -1]                                  # two experts of rank 0: one row
    idx[1] = [E_LOCAL, 0, E_LOCAL + 2]                   # both ranks
    idx[2] = -1                                          # sent nowhere
    w = rng.random((T, K)).astype(np.float32)
    w[idx < 0] = np.nan                                  # never used
    gw = torch.Generator().manual_seed(7)
    w1 = (torch.randn(E, H, 2 * I, generator=gw) / np.sqrt(H)).to(torch.bfloat16)
    w2 = (torch.randn(E, I, H, generator=gw) / np.sqrt(I)).to(torch.bfloat16)
    return x, torch.from_numpy(idx), torch.from_numpy(w), w1, w2


class _CpuLibrary:
    """CPU stand-ins for the library calls ProcessGroupRanks makes."""

    @staticmethod
    def ep_layout(topk_idx, R_, E_local, err=None):
        import torch
        from oracle import ep as oep
        si, cnt = oep.ep_layout(topk_idx.numpy(), R_, E_local)
        return torch.from_numpy(si), torch.from_numpy(cnt.astype(np.int32))

    @staticmethod
    def ep_peers(recv_x, recv_idx, recv_w, row_off, recv_rows=None, err=None):
        return {"x": recv_x, "idx": recv_idx, "w": recv_w, "off": [int(o) for o in row_off]}

    @staticmethod
    def ep_dispatch(x, topk_idx, topk_w, send_idx, E_local, peers, R_):
        for t in range(x.shape[0]):
            for d in range(R_):
                j = int(send_idx[t, d])
                if j < 0:
                    continue
                row = peers["off"][d] + j
                peers["x"][d][row] = x[t]
                for k in range(topk_idx.shape[1]):
                    e = int(topk_idx[t, k])
                    mine = 0 <= e < R_ * E_local and e // E_local == d
                    peers["idx"][d][row, k] = e - d * E_local if mine else -1
                    peers["w"][d][row, k] = float(topk_w[t, k]) if mine else 0.0

    @staticmethod
    def forward(x, topk_idx, topk_w, w1, w2, b1=None, b2=None, layout=0, out=None):
        import torch
        import oracle
        y = oracle.forward_rows(oracle.Weights(x, w1, b1, w2, b2), topk_idx.numpy(), topk_w.numpy(), layout=layout)
        out.copy_(torch.from_numpy(y).to(torch.bfloat16))
        return out

    @staticmethod
    def ep_sources(local_out, row_off, rows=None, err=None):
        return {"out": local_out, "off": [int(o) for o in row_off]}

    @staticmethod
    def ep_combine(src, send_idx, H_, out=None):
        import torch
        T, R_ = send_idx.shape
        acc = torch.zeros(T, H_, dtype=torch.float32)
        for t in range(T):
            for d in range(R_):                          # ascending rank order
                j = int(send_idx[t, d])
                if j >= 0:
                    acc[t] += src["out"][d][src["off"][d] + j].float()
        return acc.to(torch.bfloat16)


def _worker(rank: int, world: int, port: int, share_dir: str, out_dir: str) -> None:
    import torch
    import torch.distributed as dist
    from datetime import timedelta

    sys.path.insert(0, ROOT)
    from mixture_experts_routed_non_b200 import ep as ep_mod

    class FileSharedRanks(ep_mod.ProcessGroupRanks):
        """Buffers in files mapped by both processes instead of CUDA IPC."""

        def _open_peers(self, mine, opener):
            def mapped(r, i, like):
                path = os.path.join(share_dir, f"rank{r}_buf{i}.bin")
                return torch.from_file(path, shared=True, size=like.numel(), dtype=like.dtype).view(like.shape)

            own = tuple(mapped(self.me, i, t) for i, t in enumerate(mine))
            self.recv_x, self.recv_idx, self.recv_w, self.local_out = own
            dist.barrier(group=self.group)               # every rank's files exist
            return [own if d == self.me else tuple(mapped(d, i, t) for i, t in enumerate(mine))
                    for d in range(self.R)]

    ep_mod.binding = _CpuLibrary()
    torch.cuda.synchronize = lambda *a, **k: None        # CPU buffers: nothing to wait for
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        x, idx, w, w1, w2 = _inputs(rank)
        ranks = FileSharedRanks(E_LOCAL, CAPACITY, H, K, device="cpu")
        lo, hi = rank * E_LOCAL, (rank + 1) * E_LOCAL
        out = ranks.forward(x, idx, w, w1[lo:hi], w2[lo:hi])
        cap_rows = int(ranks.recv_idx.shape[0])
        dist.barrier()
        # a capacity too small for the routing is refused before any row moves
        small = FileSharedRanks.__new__(FileSharedRanks)
        small.__dict__.update(ranks.__dict__)
        small.capacity = 1
        try:
            small.forward(x, idx, w, w1[lo:hi], w2[lo:hi])
            refused = False
        except ValueError:
            refused = True
        dist.barrier()
    finally:
        dist.destroy_process_group()
    np.save(os.path.join(out_dir, f"out{rank}.npy"), out.float().numpy())
    np.save(os.path.join(out_dir, f"flags{rank}.npy"), np.array([cap_rows, int(refused)]))


def test_process_group_ranks_two_gloo_ranks(tmp_path):
    from helpers import assert_close_ep
    import oracle

    share, outd = tmp_path / "share", tmp_path / "out"
    share.mkdir()
    outd.mkdir()
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, R, port, str(share), str(outd))) for r in range(R)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
    for p in procs:
        if p.is_alive():
            p.kill()
            p.join()
    assert [p.exitcode for p in procs] == [0, 0]
    for s in range(R):
        x, idx, w, w1, w2 = _inputs(s)
        wts = oracle.Weights(x, w1, None, w2, None)
        idx_np, w_np = idx.numpy(), w.numpy()
        ref = np.zeros((T_OF[s], H))
        mag = np.zeros((T_OF[s], H))
        for d in range(R):   # each destination's partial: the forward over its experts only
            idx_d = np.where((idx_np >= 0) & (idx_np // E_LOCAL == d), idx_np, -1).astype(np.int32)
            part = oracle.forward_rows(wts, idx_d, w_np)
            ref += part
            mag += np.abs(part)
        np.testing.assert_allclose(ref, oracle.forward_rows(wts, idx_np, w_np), rtol=1e-12, atol=1e-12)
        got = np.load(outd / f"out{s}.npy")
        assert_close_ep(got, ref, mag, f"routed_out of rank {s}")
        assert not got[2].any()                          # the token sent nowhere
        cap_rows, refused = np.load(outd / f"flags{s}.npy")
        assert cap_rows == CAPACITY and refused == 1
