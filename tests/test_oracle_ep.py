"""Pins of the expert-parallel dispatch/combine oracle (oracle.ep).

What the pages fix ("End-to-end DeepEP v2 non-expand + SonicMoE integration
#68": non-expand dispatch sends a token row once per destination rank, with
local expert ids and -1 for slots whose expert lives elsewhere; the combine
returns each token's contributions to its original row): a hand-worked
example, invariants of the slot bookkeeping, the one-rank case as the
identity, and the composition dispatch -> local forward -> combine equal to
the forward over all experts on one rank (the sum over experts is linear).
"""
import json
import os

import numpy as np
import pytest

import oracle
from oracle import ep

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng_problem(R, E_local, T, K, H, seed, p_invalid=0.1, bad=False):
    rng = np.random.default_rng(seed)
    xs, idxs, ws = [], [], []
    for s in range(R):
        idx = np.stack([rng.choice(R * E_local, size=K, replace=False) for _ in range(T)]).astype(np.int32)
        idx[rng.random((T, K)) < p_invalid] = -1
        if bad:
            idx[0, 0] = R * E_local + 3  # not an expert: not sent
        xs.append(rng.standard_normal((T, H)).astype(np.float32))
        idxs.append(idx)
        ws.append(rng.random((T, K)).astype(np.float32))
    return xs, idxs, ws


def test_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "ep_worked_example.json")))
    src = g["sources"]
    xs = [np.array(s["x"], np.float32) for s in src]
    idxs = [np.array(s["topk_idx"], np.int32) for s in src]
    ws = [np.array(s["topk_w"], np.float32) for s in src]
    d = ep.ep_dispatch(xs, idxs, ws, g["R"], g["E_local"])
    assert [si.tolist() for si in d["send_idx"]] == g["send_idx"]
    assert d["counts"].tolist() == g["counts"]
    assert d["off"].tolist() == g["off"]
    for r, exp in enumerate(g["recv"]):
        assert d["recv_x"][r].tolist() == exp["x"]
        assert d["recv_idx"][r].tolist() == exp["topk_idx"]
        assert d["recv_w"][r].tolist() == exp["topk_w"]
    outs = ep.ep_combine([np.array(o, np.float64) for o in g["local_out"]], d["send_idx"], d["off"])
    assert [o.tolist() for o in outs] == g["routed_out"]


@pytest.mark.parametrize("R,E_local,K", [(2, 4, 3), (4, 2, 4), (8, 2, 8), (3, 5, 2)])
def test_slot_bookkeeping(R, E_local, K):
    xs, idxs, ws = _rng_problem(R, E_local, T=37, K=K, H=4, seed=R * 10 + K, bad=True)
    d = ep.ep_dispatch(xs, idxs, ws, R, E_local)
    valid = sum(int(((i >= 0) & (i < R * E_local)).sum()) for i in idxs)
    # every valid slot lands exactly once, on its owner, with its weight
    assert sum(int((ri >= 0).sum()) for ri in d["recv_idx"]) == valid
    wsum = sum(float(w[(i >= 0) & (i < R * E_local)].sum(dtype=np.float64)) for w, i in zip(ws, idxs))
    assert np.isclose(sum(float(rw.sum(dtype=np.float64)) for rw in d["recv_w"]), wsum, rtol=1e-12)
    assert all(((ri >= -1) & (ri < E_local)).all() for ri in d["recv_idx"])
    # brute force: the rows of rank r are the (source, token) pairs with an expert on r,
    # in (source, token) order, each carrying its token's row
    for r in range(R):
        expect = [(s, t) for s in range(R) for t in range(idxs[s].shape[0])
                  if any(0 <= e < R * E_local and e // E_local == r for e in idxs[s][t])]
        assert d["n_recv"][r] == len(expect)
        for row, (s, t) in enumerate(expect):
            assert np.array_equal(d["recv_x"][r][row], xs[s][t])
            assert d["send_idx"][s][t, r] == row - d["off"][r, s]
            for k in range(K):
                e = idxs[s][t, k]
                on = 0 <= e < R * E_local and e // E_local == r
                assert d["recv_idx"][r][row, k] == (e - r * E_local if on else -1)
                assert d["recv_w"][r][row, k] == (ws[s][t, k] if on else 0.0)
    # counts and offsets: each destination's blocks tile its rows
    assert (d["counts"].sum(axis=0) == d["n_recv"]).all()
    assert (d["off"][:, 0] == 0).all()


def test_one_rank_is_identity():
    xs, idxs, ws = _rng_problem(1, 6, T=50, K=3, H=8, seed=3)
    d = ep.ep_dispatch(xs, idxs, ws, 1, 6)
    sent = (idxs[0] >= 0).any(axis=1)
    assert np.array_equal(d["recv_x"][0], xs[0][sent])
    assert np.array_equal(d["recv_idx"][0], idxs[0][sent])
    assert np.array_equal(d["recv_w"][0], np.where(idxs[0][sent] >= 0, ws[0][sent], 0))
    assert (d["send_idx"][0][sent, 0] == np.arange(sent.sum())).all()
    assert (d["send_idx"][0][~sent, 0] == -1).all()


@pytest.mark.parametrize("R,E_local", [(2, 3), (4, 2)])
def test_composition_equals_single_rank_forward(R, E_local):
    """dispatch -> each rank's local forward over its experts -> combine gives
    the forward over all R * E_local experts on one rank (fp64)."""
    import torch
    T, K, H, I = 24, 3, 64, 64
    rng = np.random.default_rng(11)
    xs, idxs, ws = _rng_problem(R, E_local, T, K, H, seed=5)
    xs = [torch.from_numpy(x).to(torch.bfloat16) for x in xs]
    E = R * E_local
    w1 = torch.from_numpy(rng.standard_normal((E, H, 2 * I)) / np.sqrt(H)).to(torch.bfloat16)
    w2 = torch.from_numpy(rng.standard_normal((E, I, H)) / np.sqrt(I)).to(torch.bfloat16)
    b1 = torch.from_numpy(rng.standard_normal((E, 2 * I)) * 0.1).to(torch.bfloat16)
    b2 = torch.from_numpy(rng.standard_normal((E, H)) * 0.1).to(torch.bfloat16)
    d = ep.ep_dispatch([x.view(torch.int16).numpy() for x in xs], idxs, ws, R, E_local)
    local = []
    for r in range(R):
        rx = torch.from_numpy(d["recv_x"][r]).view(torch.bfloat16)
        sl = slice(r * E_local, (r + 1) * E_local)
        wts = oracle.Weights(rx, w1[sl], b1[sl], w2[sl], b2[sl])
        local.append(oracle.forward_rows(wts, d["recv_idx"][r], d["recv_w"][r]) if rx.shape[0] else
                     np.zeros((0, H)))
    routed = ep.ep_combine(local, d["send_idx"], d["off"])
    for s in range(R):
        wts = oracle.Weights(xs[s], w1, b1, w2, b2)
        ref = oracle.forward_rows(wts, idxs[s], ws[s])
        np.testing.assert_allclose(routed[s], ref, rtol=1e-12, atol=1e-12)


def _mutant_layout(topk_idx, R, E_local):
    # plausible mistake: one row per (token, expert) instead of per (token, rank)
    T, K = topk_idx.shape
    send_idx = np.full((T, R), -1, np.int32)
    counts = np.zeros(R, np.int64)
    for t in range(T):
        for k in range(K):
            e = int(topk_idx[t, k])
            if 0 <= e < R * E_local:
                d = e // E_local
                send_idx[t, d] = counts[d]
                counts[d] += 1
    return send_idx, counts


@pytest.mark.parametrize("which", ["offsets", "layout"])
def test_pins_catch_planted_mistakes(monkeypatch, which):
    """A planted mistake in the oracle (CPU) fails the pins above."""
    if which == "offsets":
        # plausible mistake: offsets indexed [s, d] instead of [d, s]
        orig = ep.recv_offsets
        monkeypatch.setattr(ep, "recv_offsets", lambda c: (orig(c)[0].T.copy(), orig(c)[1]))
    else:
        monkeypatch.setattr(ep, "ep_layout", _mutant_layout)
    failed = 0
    for fn in (test_worked_example, lambda: test_slot_bookkeeping(4, 2, 4)):
        try:
            fn()
        except (AssertionError, IndexError, ValueError):
            failed += 1
    assert failed >= 1
