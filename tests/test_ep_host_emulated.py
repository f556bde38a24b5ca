"""The host side of ``EmulatedRanks`` (R ranks in one device's memory) on CPU.

The library calls are replaced by the CPU stand-ins of test_ep_host_gloo.py
(written from the oracle's definitions), so what is tested is the
orchestration: the layouts of every source, the count matrix and block
offsets, the receive buffers (at least one row each), the per-rank local
forward over that rank's slice of the global weights, and the combine with a
rank that received nothing.  The GPU tests run the same class on the CUDA
kernels.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_close_ep
from mixture_experts_routed_non_b200 import binding
from mixture_experts_routed_non_b200 import ep as ep_mod
from test_ep_host_gloo import _CpuLibrary


class _CpuLibraryAlloc(_CpuLibrary):
    EP_MAX_RANKS = binding.EP_MAX_RANKS

    @staticmethod
    def forward(x, topk_idx, topk_w, w1, w2, b1=None, b2=None, layout=0, out=None):
        if out is None:
            out = torch.empty((x.shape[0], x.shape[1]), dtype=torch.bfloat16)
        return _CpuLibrary.forward(x, topk_idx, topk_w, w1, w2, b1, b2, layout=layout, out=out)


def _case(R, E_local, T_of, H, I, K, used_ranks, seed):
    g = torch.Generator().manual_seed(seed)
    rng = np.random.default_rng(seed)
    experts = [e for d in used_ranks for e in range(d * E_local, (d + 1) * E_local)]
    xs, idxs, ws = [], [], []
    for T in T_of:
        xs.append(torch.randn(T, H, generator=g).to(torch.bfloat16))
        idx = np.full((T, K), -1, np.int32)
        for t in range(T):
            m = int(rng.integers(0, K + 1))
            idx[t, rng.permutation(K)[:m]] = rng.choice(experts, size=m, replace=False)
        w = rng.random((T, K)).astype(np.float32)
        w[idx < 0] = np.nan
        idxs.append(torch.from_numpy(idx))
        ws.append(torch.from_numpy(w))
    E = R * E_local
    w1 = (torch.randn(E, H, 2 * I, generator=g) / np.sqrt(H)).to(torch.bfloat16)
    w2 = (torch.randn(E, I, H, generator=g) / np.sqrt(I)).to(torch.bfloat16)
    return xs, idxs, ws, w1, w2


@pytest.mark.parametrize("R,E_local,T_of,used", [
    (2, 4, (24, 17), (0, 1)),
    (3, 2, (9, 0, 13), (0, 2)),        # rank 1 holds no routed expert and has no tokens
    (1, 6, (11,), (0,)),               # one rank: dispatch and combine are the identity
])
def test_emulated_ranks_host_side(monkeypatch, R, E_local, T_of, used):
    monkeypatch.setattr(ep_mod, "binding", _CpuLibraryAlloc())
    H, I, K = 64, 64, 3
    xs, idxs, ws, w1, w2 = _case(R, E_local, T_of, H, I, K, used, seed=31 + R)
    ranks = ep_mod.EmulatedRanks(R, E_local, device="cpu")
    outs = ranks.forward(xs, idxs, ws, w1, w2)
    assert len(outs) == R
    for s in range(R):
        wts = oracle.Weights(xs[s], w1, None, w2, None)
        idx_np, w_np = idxs[s].numpy(), ws[s].numpy()
        ref = np.zeros((T_of[s], H))
        mag = np.zeros((T_of[s], H))
        for d in range(R):
            idx_d = np.where((idx_np >= 0) & (idx_np // E_local == d), idx_np, -1).astype(np.int32)
            part = oracle.forward_rows(wts, idx_d, w_np) if T_of[s] else np.zeros((0, H))
            ref += part
            mag += np.abs(part)
        assert tuple(outs[s].shape) == (T_of[s], H)
        assert_close_ep(outs[s].float().numpy(), ref, mag, f"routed_out of rank {s}")


def test_emulated_ranks_receive_counts(monkeypatch):
    """The dispatch state: counts[s, d] from the layouts, offsets in source
    order, and receive buffers cut to each rank's count."""
    monkeypatch.setattr(ep_mod, "binding", _CpuLibraryAlloc())
    from oracle import ep as oep
    R, E_local = 3, 2
    xs, idxs, ws, _, _ = _case(R, E_local, (9, 0, 13), 64, 64, 3, (0, 2), seed=5)
    st = ep_mod.EmulatedRanks(R, E_local, device="cpu").dispatch(xs, idxs, ws)
    ref = oep.ep_dispatch([x.float().numpy() for x in xs], [i.numpy() for i in idxs], [w.numpy() for w in ws],
                          R, E_local)
    assert np.array_equal(st["counts"], ref["counts"])
    assert np.array_equal(st["off"], ref["off"]) and np.array_equal(st["n_recv"], ref["n_recv"])
    for d in range(R):
        assert st["recv_x"][d].shape[0] == ref["n_recv"][d]
        assert np.array_equal(st["recv_x"][d].float().numpy(), ref["recv_x"][d])
        assert np.array_equal(st["recv_idx"][d].numpy(), ref["recv_idx"][d])
        assert np.array_equal(st["recv_w"][d].numpy(), ref["recv_w"][d])
    assert st["n_recv"][1] == 0
