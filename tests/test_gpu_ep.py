"""Expert-parallel dispatch / combine (moe_ep_layout, moe_ep_dispatch,
moe_ep_combine) on one GPU, with R ranks emulated in its memory.

The non-expand dataflow of "End-to-end DeepEP v2 non-expand + SonicMoE
integration #68": the layout and the dispatched rows, ids and weights are
compared bit-exactly with the oracle (oracle.ep); the combine within the
output tolerance of the oracle's float64 sum (and bit-exactly with the same
fp32 sum done by torch in the same order); dispatch -> local forward ->
combine within the forward tolerance of the oracle's forward over all
experts on one rank.  With R ranks in one GPU's memory, every kernel reads
and writes ordinary device pointers and none waits on another.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_close, assert_close_ep, to_np
from mixture_experts_routed_non_b200 import binding
from mixture_experts_routed_non_b200.ep import EmulatedRanks, block_offsets
from oracle import ep as oep

pytestmark = pytest.mark.gpu


def _problem(R, E_local, T, K, H, seed, p_invalid=0.1, per_rank_T=None, local_only=False):
    """Per-source-rank (x bf16, topk_idx int32 global ids, topk_w fp32) on the GPU."""
    rng = np.random.default_rng(seed)
    xs, idxs, ws = [], [], []
    for s in range(R):
        Ts = per_rank_T[s] if per_rank_T is not None else T
        if local_only:  # every token's experts on one rank (non-expand: one row per token)
            owner = rng.integers(0, R, size=Ts)
            idx = np.stack([owner[t] * E_local + rng.choice(E_local, size=K, replace=False) for t in range(Ts)])
        else:
            idx = np.stack([rng.choice(R * E_local, size=K, replace=False) for _ in range(Ts)]) if Ts else \
                np.zeros((0, K), np.int64)
        idx = idx.astype(np.int32)
        if Ts:
            idx[rng.random((Ts, K)) < p_invalid] = -1
        xs.append(torch.from_numpy(rng.standard_normal((Ts, H)).astype(np.float32)).to(torch.bfloat16).cuda())
        idxs.append(torch.from_numpy(idx).cuda())
        ws.append(torch.from_numpy(rng.random((Ts, K)).astype(np.float32)).cuda())
    return xs, idxs, ws


def _oracle_dispatch(xs, idxs, ws, R, E_local):
    return oep.ep_dispatch([x.view(torch.int16).cpu().numpy() for x in xs], [i.cpu().numpy() for i in idxs],
                           [w.cpu().numpy() for w in ws], R, E_local)


CASES = [(2, 4, 16, 3, 64), (4, 2, 257, 4, 128), (8, 4, 300, 8, 64), (3, 5, 1025, 2, 72), (1, 8, 200, 4, 64),
         (32, 1, 100, 4, 8)]


@pytest.mark.parametrize("R,E_local,T,K,H", CASES)
def test_layout_and_dispatch_bit_exact(R, E_local, T, K, H):
    xs, idxs, ws = _problem(R, E_local, T, K, H, seed=R * 100 + K)
    ref = _oracle_dispatch(xs, idxs, ws, R, E_local)
    st = EmulatedRanks(R, E_local).dispatch(xs, idxs, ws)
    torch.cuda.synchronize()
    assert np.array_equal(st["counts"], ref["counts"])
    assert np.array_equal(st["off"], ref["off"])
    for s in range(R):
        assert np.array_equal(st["send_idx"][s].cpu().numpy(), ref["send_idx"][s])
    for d in range(R):
        assert np.array_equal(st["recv_x"][d].view(torch.int16).cpu().numpy(), ref["recv_x"][d])
        assert np.array_equal(st["recv_idx"][d].cpu().numpy(), ref["recv_idx"][d])
        assert np.array_equal(st["recv_w"][d].cpu().numpy(), ref["recv_w"][d])


def test_non_expand_sends_one_row_per_rank():
    R, E_local, K = 4, 8, 4
    xs, idxs, ws = _problem(R, E_local, 200, K, 64, seed=9, p_invalid=0.0, local_only=True)
    st = EmulatedRanks(R, E_local).dispatch(xs, idxs, ws)
    assert int(st["n_recv"].sum()) == R * 200  # one row per token, although each has K experts on its rank
    for d in range(R):
        assert ((st["recv_idx"][d] >= 0).sum(dim=1) == K).all()


def test_bad_ids_are_flagged_and_not_sent():
    R, E_local = 2, 3
    xs, idxs, ws = _problem(R, E_local, 40, 2, 64, seed=4)
    idxs[0][3, 0] = R * E_local + 1
    idxs[1][7, 1] = -7
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ref = _oracle_dispatch(xs, idxs, ws, R, E_local)
    st = EmulatedRanks(R, E_local).dispatch(xs, idxs, ws, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & 0x1
    for d in range(R):
        assert np.array_equal(st["recv_idx"][d].cpu().numpy(), ref["recv_idx"][d])
        assert np.array_equal(st["recv_w"][d].cpu().numpy(), ref["recv_w"][d])


def test_ranks_with_no_tokens_and_ranks_receiving_nothing():
    R, E_local, K, H = 4, 2, 2, 64
    xs, idxs, ws = _problem(R, E_local, 0, K, H, seed=2, per_rank_T=[0, 50, 0, 13])
    idxs[1][idxs[1] >= 2 * E_local] = -1  # nothing for ranks 2 and 3 from rank 1
    idxs[3][idxs[3] >= 2 * E_local] = -1
    ref = _oracle_dispatch(xs, idxs, ws, R, E_local)
    er = EmulatedRanks(R, E_local)
    st = er.dispatch(xs, idxs, ws)
    assert list(st["n_recv"][2:]) == [0, 0]
    for d in range(R):
        assert np.array_equal(st["recv_idx"][d].cpu().numpy(), ref["recv_idx"][d])
    local = [torch.randn((int(n), H), device="cuda").to(torch.bfloat16) for n in st["n_recv"]]
    outs = er.combine(local, st, H)
    ref_out = oep.ep_combine([to_np(l).astype(np.float64) for l in local], ref["send_idx"], ref["off"])
    for s in range(R):
        assert outs[s].shape == (xs[s].shape[0], H)
        assert_close(to_np(outs[s]), ref_out[s], f"rank {s}")


@pytest.mark.parametrize("R,E_local,T,K,H", CASES)
def test_combine(R, E_local, T, K, H):
    xs, idxs, ws = _problem(R, E_local, T, K, H, seed=R * 7 + T)
    er = EmulatedRanks(R, E_local)
    st = er.dispatch(xs, idxs, ws)
    g = torch.Generator(device="cuda").manual_seed(3)
    local = [torch.randn((int(n), H), generator=g, device="cuda").to(torch.bfloat16) for n in st["n_recv"]]
    outs = er.combine(local, st, H)
    ref = oep.ep_combine([to_np(l).astype(np.float64) for l in local], [s.cpu().numpy() for s in st["send_idx"]],
                         st["off"])
    for s in range(R):
        assert_close(to_np(outs[s]), ref[s], f"combine rank {s}")
        # the same fp32 sum in ascending rank order, then one bf16 rounding
        si = st["send_idx"][s].long()
        acc = torch.zeros((T, H), dtype=torch.float32, device="cuda")
        for d in range(R):
            sel = si[:, d] >= 0
            acc[sel] += local[d][int(st["off"][d, s]) + si[sel, d]].float()
        assert torch.equal(outs[s], acc.to(torch.bfloat16))


def _weights(E, H, I, seed, bias=True):
    g = torch.Generator(device="cpu").manual_seed(seed)
    w1 = (torch.randn((E, H, 2 * I), generator=g) / H ** 0.5).to(torch.bfloat16).cuda()
    w2 = (torch.randn((E, I, H), generator=g) / I ** 0.5).to(torch.bfloat16).cuda()
    b1 = (torch.randn((E, 2 * I), generator=g) * 0.01).to(torch.bfloat16).cuda() if bias else None
    b2 = (torch.randn((E, H), generator=g) * 0.01).to(torch.bfloat16).cuda() if bias else None
    return w1, w2, b1, b2


@pytest.mark.parametrize("R,E_local,T,K,H,I,layout,bias", [
    (2, 4, 96, 2, 128, 256, 0, True),
    (4, 2, 300, 4, 128, 128, 1, False),
    (8, 4, 256, 8, 256, 128, 0, False),
])
def test_dispatch_local_forward_combine_matches_oracle(R, E_local, T, K, H, I, layout, bias):
    """routed_out of every source rank against the oracle's forward over all
    R * E_local experts on one rank."""
    xs, idxs, ws = _problem(R, E_local, T, K, H, seed=T + K)
    w1, w2, b1, b2 = _weights(R * E_local, H, I, seed=R, bias=bias)
    if layout == 1:
        w1 = torch.cat([w1[:, :, 0::2], w1[:, :, 1::2]], dim=2).contiguous()
        if b1 is not None:
            b1 = torch.cat([b1[:, 0::2], b1[:, 1::2]], dim=1).contiguous()
    outs = EmulatedRanks(R, E_local).forward(xs, idxs, ws, w1, w2, b1, b2, layout=layout)
    torch.cuda.synchronize()
    # the oracle's partials: dispatch, then every rank's forward over its experts
    d = _oracle_dispatch(xs, idxs, ws, R, E_local)
    sl = lambda t, r: None if t is None else t[r * E_local:(r + 1) * E_local].cpu()
    partial = []
    for r in range(R):
        rx = torch.from_numpy(d["recv_x"][r]).view(torch.bfloat16)
        wts = oracle.Weights(rx, sl(w1, r), sl(b1, r), sl(w2, r), sl(b2, r))
        partial.append(oracle.forward_rows(wts, d["recv_idx"][r], d["recv_w"][r], layout=layout)
                       if rx.shape[0] else np.zeros((0, H)))
    routed = oep.ep_combine(partial, d["send_idx"], d["off"])
    mag = oep.ep_combine([np.abs(p) for p in partial], d["send_idx"], d["off"])
    for s in range(R):
        # the composition equals the forward over all experts (pinned in the oracle tests)
        wts = oracle.Weights(xs[s].cpu(), w1.cpu(), None if b1 is None else b1.cpu(), w2.cpu(),
                             None if b2 is None else b2.cpu())
        ref = oracle.forward_rows(wts, idxs[s].cpu().numpy(), ws[s].cpu().numpy(), layout=layout)
        np.testing.assert_allclose(routed[s], ref, rtol=1e-9, atol=1e-9)
        assert_close_ep(to_np(outs[s]), ref, mag[s], f"routed_out rank {s}")


def test_deterministic():
    R, E_local, T, K, H, I = 4, 2, 200, 4, 128, 128
    xs, idxs, ws = _problem(R, E_local, T, K, H, seed=1)
    w1, w2, _, _ = _weights(R * E_local, H, I, seed=2, bias=False)
    a = EmulatedRanks(R, E_local).forward(xs, idxs, ws, w1, w2)
    b = EmulatedRanks(R, E_local).forward(xs, idxs, ws, w1, w2)
    for s in range(R):
        assert torch.equal(a[s], b[s])


def test_rank_local_shape_sampled():
    """The rank-local shape after 8-way dispatch (H=7168, I=2048, 32 local
    experts), scaled down to 8 emulated ranks of 4 experts and 512 tokens
    each; routed_out checked on a sample of tokens."""
    R, E_local, T, K, H, I = 8, 4, 512, 8, 7168, 2048
    xs, idxs, ws = _problem(R, E_local, T, K, H, seed=77, p_invalid=0.0)
    g = torch.Generator(device="cuda").manual_seed(5)
    w1 = (torch.randn((R * E_local, H, 2 * I), generator=g, device="cuda") / H ** 0.5).to(torch.bfloat16)
    w2 = (torch.randn((R * E_local, I, H), generator=g, device="cuda") / I ** 0.5).to(torch.bfloat16)
    outs = EmulatedRanks(R, E_local).forward(xs, idxs, ws, w1, w2)
    torch.cuda.synchronize()
    rng = np.random.default_rng(0)
    w1c, w2c = w1.cpu(), w2.cpu()
    for s in (0, 5):
        toks = np.sort(rng.choice(T, size=12, replace=False))
        # the sampled tokens' partials: each (token, rank) row of the forward over that rank's experts
        idx = idxs[s].cpu().numpy()[toks]
        w = ws[s].cpu().numpy()[toks]
        ref = np.zeros((len(toks), H))
        mag = np.zeros((len(toks), H))
        for r in range(R):
            on = (idx >= r * E_local) & (idx < (r + 1) * E_local)
            rows = np.nonzero(on.any(axis=1))[0]
            if rows.size == 0:
                continue
            sl = slice(r * E_local, (r + 1) * E_local)
            wts = oracle.Weights(xs[s][torch.from_numpy(toks[rows]).cuda()].cpu(), w1c[sl], None, w2c[sl], None)
            p = oracle.forward_rows(wts, np.where(on[rows], idx[rows] - r * E_local, -1).astype(np.int32),
                                    np.where(on[rows], w[rows], 0).astype(np.float32))
            ref[rows] += p
            mag[rows] += np.abs(p)
        assert_close_ep(to_np(outs[s][torch.from_numpy(toks).cuda()]), ref, mag, f"rank {s} sampled")


def test_argument_errors():
    R, E_local = 2, 2
    xs, idxs, ws = _problem(R, E_local, 8, 2, 64, seed=0)
    with pytest.raises(binding.MoeError):
        binding.ep_layout(idxs[0], 33, E_local)  # more ranks than the tables hold
    send_idx, _ = binding.ep_layout(idxs[0], R, E_local)
    bad = binding.ep_peers([0, 0], [0, 0], [0, 0], [0, 0], recv_rows=[1, 1])
    with pytest.raises(binding.MoeError):
        binding.ep_dispatch(xs[0], idxs[0], ws[0], send_idx, E_local, bad, R)
    assert block_offsets(np.array([[1, 2], [3, 4]]))[0].tolist() == [[0, 1], [0, 2]]


def test_process_group_ranks_single_rank():
    """The one-process-per-GPU path with a one-rank NCCL group: the count
    all-gather, barriers and buffers of ProcessGroupRanks around dispatch ->
    local forward -> combine.  With one rank the routed output must equal the
    plain forward bit for bit (same rows, same arithmetic, one partial)."""
    import socket
    from datetime import timedelta

    import torch.distributed as dist

    from mixture_experts_routed_non_b200.ep import ProcessGroupRanks
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True, timeout=timedelta(seconds=60))
    dist.init_process_group("nccl", store=store, rank=0, world_size=1, timeout=timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        E, T, K, H, I = 8, 300, 4, 128, 128
        xs, idxs, ws = _problem(1, E, T, K, H, seed=21)
        w1, w2, _, _ = _weights(E, H, I, seed=3, bias=False)
        pg = ProcessGroupRanks(E_local=E, capacity=T, H=H, K=K)
        out = pg.forward(xs[0], idxs[0], ws[0], w1, w2)
        ref = binding.forward(xs[0], idxs[0], ws[0], w1, w2)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
    finally:
        dist.destroy_process_group()


def test_duplicate_experts_and_all_slots_on_one_rank():
    """A row naming the same expert twice keeps both slots (one receive row);
    a row whose slots all live on one rank is sent to that rank only."""
    R, E_local, K, H, I = 4, 3, 4, 64, 64
    T = 40
    rng = np.random.default_rng(8)
    idx = np.stack([rng.choice(R * E_local, size=K, replace=False) for _ in range(T)]).astype(np.int32)
    idx[0] = [5, 5, 1, -1]               # expert 5 twice
    idx[1] = [6, 7, 8, 6]                # all on rank 2, expert 6 twice
    idx[2] = [-1, -1, -1, -1]            # sent nowhere
    xs = [torch.randn((T, H), device="cuda").to(torch.bfloat16) for _ in range(R)]
    idxs = [torch.from_numpy(idx).cuda() for _ in range(R)]
    ws = [torch.rand((T, K), device="cuda") for _ in range(R)]
    ref = _oracle_dispatch(xs, idxs, ws, R, E_local)
    st = EmulatedRanks(R, E_local).dispatch(xs, idxs, ws)
    for d in range(R):
        assert np.array_equal(st["recv_idx"][d].cpu().numpy(), ref["recv_idx"][d])
        assert np.array_equal(st["recv_w"][d].cpu().numpy(), ref["recv_w"][d])
    si = st["send_idx"][0].cpu().numpy()
    assert (si[1] >= 0).tolist() == [False, False, True, False]
    assert (si[2] < 0).all()
    w1, w2, b1, b2 = _weights(R * E_local, H, I, seed=9)
    outs = EmulatedRanks(R, E_local).forward(xs, idxs, ws, w1, w2, b1, b2)
    torch.cuda.synchronize()
    for s in range(R):
        wts = oracle.Weights(xs[s].cpu(), w1.cpu(), b1.cpu(), w2.cpu(), b2.cpu())
        fwd = oracle.forward_rows(wts, idx, ws[s].cpu().numpy())
        # each token here has at most two partials; the bound uses their magnitudes
        d = _oracle_dispatch(xs[s:s + 1] * R, idxs[s:s + 1] * R, ws[s:s + 1] * R, R, E_local)
        part = []
        for r in range(R):
            rx = torch.from_numpy(d["recv_x"][r]).view(torch.bfloat16)
            sl = slice(r * E_local, (r + 1) * E_local)
            wr = oracle.Weights(rx, w1[sl].cpu(), b1[sl].cpu(), w2[sl].cpu(), b2[sl].cpu())
            part.append(oracle.forward_rows(wr, d["recv_idx"][r], d["recv_w"][r]) if rx.shape[0] else
                        np.zeros((0, H)))
        mag = oep.ep_combine([np.abs(p) for p in part], d["send_idx"], d["off"])[0]
        assert_close_ep(to_np(outs[s]), fwd, mag, f"rank {s}")
        assert (to_np(outs[s])[2] == 0).all()


def test_rows_past_a_buffer_are_neither_written_nor_read():
    """A destination buffer smaller than its rows: the dispatch skips the rows
    past it and flags MOE_DEVERR_ABORTED; the combine reads no row past a
    local_out's row count, counts it 0 and flags the same bit."""
    R, E_local, T, K, H = 2, 2, 64, 2, 64
    xs, idxs, ws = _problem(R, E_local, T, K, H, seed=12, p_invalid=0.0)
    ref = _oracle_dispatch(xs, idxs, ws, R, E_local)
    n0 = int(ref["n_recv"][0])
    cap = n0 - 5
    pad = 16  # guard rows after the declared capacity, checked untouched
    rx = [torch.full((cap + pad, H), 7.0, device="cuda").to(torch.bfloat16),
          torch.empty((int(ref["n_recv"][1]), H), dtype=torch.bfloat16, device="cuda")]
    ri = [torch.full((cap + pad, K), 99, dtype=torch.int32, device="cuda"),
          torch.empty((int(ref["n_recv"][1]), K), dtype=torch.int32, device="cuda")]
    rw = [torch.full((cap + pad, K), 9.0, device="cuda"),
          torch.empty((int(ref["n_recv"][1]), K), device="cuda")]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for s in range(R):
        send_idx, _ = binding.ep_layout(idxs[s], R, E_local)
        peers = binding.ep_peers(rx, ri, rw, ref["off"][:, s], recv_rows=[cap, int(ref["n_recv"][1])], err=err)
        binding.ep_dispatch(xs[s], idxs[s], ws[s], send_idx, E_local, peers, R)
    torch.cuda.synchronize()
    assert int(err.item()) & 0x8
    assert np.array_equal(rx[0][:cap].view(torch.int16).cpu().numpy(), ref["recv_x"][0][:cap])
    assert np.array_equal(ri[0][:cap].cpu().numpy(), ref["recv_idx"][0][:cap])
    assert (rx[0][cap:].float() == 7.0).all() and (ri[0][cap:] == 99).all() and (rw[0][cap:] == 9.0).all()
    # combine of the last source (its block ends rank 0's rows) reading a local_out that
    # holds fewer rows than that block needs
    local = [torch.randn((int(n), H), device="cuda").to(torch.bfloat16) for n in ref["n_recv"]]
    err.zero_()
    last = R - 1
    send_idx_l, _ = binding.ep_layout(idxs[last], R, E_local)
    out = binding.ep_combine(binding.ep_sources(local, ref["off"][:, last], rows=[cap, int(ref["n_recv"][1])],
                                                err=err), send_idx_l, H)
    torch.cuda.synchronize()
    assert int(err.item()) & 0x8
    short = [np.where(np.arange(int(n))[:, None] < (cap if d == 0 else int(n)), to_np(l), 0.0)
             for d, (n, l) in enumerate(zip(ref["n_recv"], local))]
    exp = oep.ep_combine(short, ref["send_idx"], ref["off"])[last]
    assert_close(to_np(out), exp, "combine with a short local_out")
