"""Pins of the CPU oracle against what the pages and the mathematics fix.

Every function of the oracle is checked here against something other than
itself: hand-worked fixtures (tests/golden), invariants of the metadata the
pages list (sonic-moe issue #68, the metadata list and question 3), brute force
over every tiny routing table, numpy's stable argsort, a float64 numpy dense MLP
for the one-expert case, and an independent torch-CPU implementation of the
sort-by-expert recipe of the qwen3_5.py commit notes (CCCL segmented-sort
pattern: sort pairs by expert, one linear per contiguous expert slice, fused
silu x up, index_add_ scatter-back).
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from mixture_experts_routed_non_b200 import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _num(v):
    return float("nan") if v == "nan" else float(v)


# ---------------------------------------------------------------------------
# metadata
# ---------------------------------------------------------------------------

def check_metadata_invariants(idx, w, E, md):
    """Properties the metadata must have whatever the routing."""
    N, K = idx.shape
    valid = (idx >= 0) & (idx < E)
    P = int(valid.sum())
    assert md["P"] == P
    freq, off = md["freq"], md["off"]
    assert freq.sum() == P
    assert off[0] == 0 and np.array_equal(np.cumsum(freq), off[1:])
    xg, ss, sr, to, sc = (md[k] for k in ("x_gather_idx", "s_scatter_idx",
                                           "s_reverse_scatter_idx", "token_offset", "scores"))
    # token offsets = prefix of valid slots per row
    assert np.array_equal(to, np.concatenate([[0], np.cumsum(valid.sum(1))]))
    # pair q -> (token, slot) in row-major order
    tok_of_q, slot_of_q = np.nonzero(valid)
    e_of_q = idx[tok_of_q, slot_of_q]
    # s_scatter and s_rev are mutually inverse permutations of range(P)
    assert np.array_equal(np.sort(ss), np.arange(P))
    assert np.array_equal(sr[ss], np.arange(P))
    assert np.array_equal(ss[sr], np.arange(P))
    # gather index is the token of the pair at each sorted position
    assert np.array_equal(xg, tok_of_q[ss])
    # segments hold their own expert, q strictly ascending inside (stability)
    for e in range(E):
        seg = ss[off[e]:off[e + 1]]
        assert np.all(e_of_q[seg] == e)
        assert np.all(np.diff(seg) > 0)
    # compact scores are the weights of the valid slots in q order
    assert np.array_equal(sc.view(np.int32), w[tok_of_q, slot_of_q].view(np.int32))


def test_metadata_worked_example():
    g = _load("metadata_worked_example.json")
    idx = np.array(g["topk_idx"], np.int32)
    w = np.array([[_num(v) for v in r] for r in g["topk_w"]], np.float32)
    md = oracle.metadata(idx, w, g["E"])
    ex = g["expected"]
    assert md["P"] == ex["P"]
    assert md["freq"].tolist() == ex["expert_frequency"]
    assert md["off"].tolist() == ex["expert_frequency_offset"]
    assert md["x_gather_idx"].tolist() == ex["x_gather_idx"]
    assert md["s_scatter_idx"].tolist() == ex["s_scatter_idx"]
    assert md["s_reverse_scatter_idx"].tolist() == ex["s_reverse_scatter_idx"]
    assert md["token_offset"].tolist() == ex["num_activated_expert_per_token_offset"]
    assert md["scores"].tolist() == ex["router_scores"]
    check_metadata_invariants(idx, w, g["E"], md)


def _brute(idx, E):
    N, K = idx.shape
    pairs = [(t, k, int(idx[t, k])) for t in range(N) for k in range(K) if 0 <= idx[t, k] < E]
    order = sorted(range(len(pairs)), key=lambda q: (pairs[q][2], q))
    freq = [sum(1 for p in pairs if p[2] == e) for e in range(E)]
    off = [0]
    for f in freq:
        off.append(off[-1] + f)
    rev = [0] * len(pairs)
    for p, q in enumerate(order):
        rev[q] = p
    to = [0]
    for t in range(N):
        to.append(to[-1] + sum(1 for k in range(K) if 0 <= idx[t, k] < E))
    return dict(freq=freq, off=off, xg=[pairs[q][0] for q in order], ss=order, sr=rev, to=to)


@pytest.mark.parametrize("N,K,E", [(1, 1, 1), (2, 2, 2), (3, 2, 3), (2, 3, 2), (3, 1, 3)])
def test_metadata_brute_force_all_tables(N, K, E):
    """Every table in {-1,0..E-1}^(N*K) against a direct Python sort."""
    vals = list(range(-1, E))
    w = np.arange(N * K, dtype=np.float32).reshape(N, K) + 0.5
    for combo in itertools.product(vals, repeat=N * K):
        idx = np.array(combo, np.int32).reshape(N, K)
        md = oracle.metadata(idx, w, E)
        b = _brute(idx, E)
        assert md["freq"].tolist() == b["freq"]
        assert md["off"].tolist() == b["off"]
        assert md["x_gather_idx"].tolist() == b["xg"]
        assert md["s_scatter_idx"].tolist() == b["ss"]
        assert md["s_reverse_scatter_idx"].tolist() == b["sr"]
        assert md["token_offset"].tolist() == b["to"]


def test_metadata_matches_numpy_stable_argsort():
    wl = synthetic.WORKLOADS["metadata"]
    idx, w = synthetic.make_routing(wl)
    md = oracle.metadata(idx, w, wl.E)
    valid = idx >= 0
    e_of_q = idx[valid]
    order = np.argsort(e_of_q, kind="stable")
    assert np.array_equal(md["s_scatter_idx"], order)
    assert np.array_equal(md["freq"], np.bincount(e_of_q, minlength=wl.E))
    check_metadata_invariants(idx, w, wl.E, md)


@pytest.mark.parametrize("name", ["tiny", "prefill", "ranklocal", "decode256"])
def test_metadata_invariants_workloads(name):
    wl = synthetic.WORKLOADS[name]
    idx, w = synthetic.make_routing(wl, invalid_value=float("nan"))
    md = oracle.metadata(idx, w, wl.E)
    check_metadata_invariants(idx, w, wl.E, md)


def test_metadata_out_of_range_ids_are_counted_and_skipped():
    idx = np.array([[0, 5], [-1, -2], [1, 0]], np.int32)
    w = np.ones((3, 2), np.float32)
    md = oracle.metadata(idx, w, 2)
    assert md["bad_ids"] == 2
    assert md["P"] == 3
    assert md["token_offset"].tolist() == [0, 1, 1, 3]
    assert md["s_scatter_idx"].tolist() == [0, 2, 1]


def test_metadata_all_invalid_and_empty():
    md = oracle.metadata(np.full((4, 3), -1, np.int32), np.zeros((4, 3), np.float32), 5)
    assert md["P"] == 0 and md["off"].tolist() == [0] * 6
    assert md["token_offset"].tolist() == [0] * 5
    md = oracle.metadata(np.zeros((0, 3), np.int32), np.zeros((0, 3), np.float32), 5)
    assert md["P"] == 0 and md["token_offset"].tolist() == [0]


# ---------------------------------------------------------------------------
# expert MLP and forward
# ---------------------------------------------------------------------------

def _bf(a):
    return torch.tensor(a, dtype=torch.float32).to(torch.bfloat16)


@pytest.mark.parametrize("layout,key", [(0, "interleaved"), (1, "concatenated")])
def test_swiglu_closed_form(layout, key):
    g = _load("swiglu_closed_form.json")
    x, w1, b1, w2, b2 = (_bf(g[k]) for k in ("x", "w1", "b1", "w2", "b2"))
    z, h, y = oracle.expert_row(x[0], w1[0], b1[0], w2[0], b2[0], layout)
    ex = g["expected_closed_form"][key]
    env = {"exp": math.exp}
    h_ex = [eval(s, env) for s in ex["h"]]
    out_ex = [eval(s, env) for s in ex["out"]]
    np.testing.assert_allclose(h, h_ex, rtol=1e-14, atol=1e-14)
    idx = np.array(g["topk_idx"], np.int32)
    w = np.array([[_num(v) for v in r] for r in g["topk_w"]], np.float32)
    wts = oracle.Weights(x, w1, b1, w2, b2)
    out = oracle.forward_rows(wts, idx, w, layout=layout)
    np.testing.assert_allclose(out[0], out_ex, rtol=1e-14, atol=1e-14)


def _dense_inputs(N, H, I, E, K, seed, bias=True, p_invalid=0.0):
    wl = synthetic.custom(N, H, I, E, K, p_invalid=p_invalid, bias=bias, seed=seed)
    return synthetic.make_inputs(wl, device="cpu", invalid_value=float("nan"))


def test_single_expert_single_slot_is_dense_mlp():
    """E=1, K=1, all slots valid, score 1: the forward is one dense SwiGLU MLP,
    computed here with float64 numpy matmuls."""
    inp = _dense_inputs(N=37, H=48, I=40, E=1, K=1, seed=11)
    idx = np.zeros((37, 1), np.int32)
    w = np.ones((37, 1), np.float32)
    wts = oracle.Weights(inp.x, inp.w1, inp.b1, inp.w2, inp.b2)
    out = oracle.forward_rows(wts, idx, w)
    x = inp.x.double().numpy()
    W1 = inp.w1[0].double().numpy()
    W2 = inp.w2[0].double().numpy()
    z = x @ W1 + inp.b1[0].double().numpy()
    g, u = z[:, 0::2], z[:, 1::2]
    ref = (g * (1.0 / (1.0 + np.exp(-g))) * u) @ W2 + inp.b2[0].double().numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-10)


def test_concatenated_equals_interleaved_after_column_permutation():
    inp = _dense_inputs(N=20, H=32, I=24, E=3, K=2, seed=12)
    wts_i = oracle.Weights(inp.x, inp.w1, inp.b1, inp.w2, inp.b2)
    # interleaved columns (g0,u0,g1,u1,...) -> concatenated (g..., u...)
    w1c = torch.cat([inp.w1[:, :, 0::2], inp.w1[:, :, 1::2]], dim=2).contiguous()
    b1c = torch.cat([inp.b1[:, 0::2], inp.b1[:, 1::2]], dim=1).contiguous()
    wts_c = oracle.Weights(inp.x, w1c, b1c, inp.w2, inp.b2)
    idx, w = inp.topk_idx.numpy(), inp.topk_w.numpy()
    a = oracle.forward_rows(wts_i, idx, w, layout=0)
    b = oracle.forward_rows(wts_c, idx, w, layout=1)
    np.testing.assert_array_equal(a, b)


def test_one_hot_scores_select_one_expert():
    inp = _dense_inputs(N=16, H=32, I=16, E=4, K=3, seed=13)
    idx = inp.topk_idx.numpy()
    wts = oracle.Weights(inp.x, inp.w1, inp.b1, inp.w2, inp.b2)
    for k in range(3):
        w = np.zeros(idx.shape, np.float32)
        w[:, k] = 1.0
        out = oracle.forward_rows(wts, idx, w)
        h, y = oracle.pair_rows(wts, np.arange(16), idx[:, k])
        np.testing.assert_allclose(out, y, rtol=1e-13, atol=1e-13)


def test_linear_in_scores_and_invariant_to_slot_order():
    inp = _dense_inputs(N=24, H=32, I=16, E=5, K=3, seed=14, p_invalid=0.2)
    idx = inp.topk_idx.numpy()
    w = np.nan_to_num(inp.topk_w.numpy())
    wts = oracle.Weights(inp.x, inp.w1, inp.b1, inp.w2, inp.b2)
    base = oracle.forward_rows(wts, idx, w)
    np.testing.assert_allclose(oracle.forward_rows(wts, idx, 0.25 * w), 0.25 * base, rtol=1e-12, atol=1e-13)
    perm = np.array([2, 0, 1])
    np.testing.assert_allclose(oracle.forward_rows(wts, idx[:, perm], w[:, perm]), base,
                               rtol=1e-12, atol=1e-13)


def test_token_without_valid_slot_is_zero_and_invalid_weights_unread():
    inp = _dense_inputs(N=6, H=16, I=8, E=2, K=2, seed=15)
    idx = inp.topk_idx.numpy().copy()
    idx[3, :] = -1
    w = inp.topk_w.numpy().copy()
    w[idx < 0] = np.nan
    wts = oracle.Weights(inp.x, inp.w1, inp.b1, inp.w2, inp.b2)
    out = oracle.forward_rows(wts, idx, w)
    assert np.all(out[3] == 0.0)
    assert np.all(np.isfinite(out))


def _recipe_torch_cpu(inp, layout=0):
    """Independent float64 torch-CPU implementation of the sort-by-expert
    recipe (qwen3_5.py commit notes, CCCL segmented-sort pattern): flatten the
    valid (token, expert) assignments, sort them by expert, run one F.linear per
    contiguous expert slice, silu x up over all pairs at once, and index_add_
    the score-weighted rows back to their tokens."""
    x = inp.x.double()
    idx = inp.topk_idx.long()
    w = inp.topk_w.double()
    N, K = idx.shape
    E, H, I2 = inp.w1.shape
    I = I2 // 2
    flat_e = idx.reshape(-1)
    flat_t = torch.arange(N).repeat_interleave(K)
    keep = flat_e >= 0
    flat_e, flat_t, flat_w = flat_e[keep], flat_t[keep], w.reshape(-1)[keep]
    order = torch.sort(flat_e, stable=True).indices
    e_s, t_s, w_s = flat_e[order], flat_t[order], flat_w[order]
    xs = x[t_s]
    z = torch.empty(xs.shape[0], I2, dtype=torch.float64)
    counts = torch.bincount(e_s, minlength=E).tolist()
    start = 0
    for e in range(E):
        n = counts[e]
        if n:
            bias = None if inp.b1 is None else inp.b1[e].double()
            z[start:start + n] = F.linear(xs[start:start + n], inp.w1[e].double().t(), bias)
        start += n
    if layout == 0:
        g, u = z[:, 0::2], z[:, 1::2]
    else:
        g, u = z[:, :I], z[:, I:]
    hs = F.silu(g) * u
    ys = torch.empty(xs.shape[0], H, dtype=torch.float64)
    start = 0
    for e in range(E):
        n = counts[e]
        if n:
            bias = None if inp.b2 is None else inp.b2[e].double()
            ys[start:start + n] = F.linear(hs[start:start + n], inp.w2[e].double().t(), bias)
        start += n
    out = torch.zeros(N, H, dtype=torch.float64)
    out.index_add_(0, t_s, ys * w_s[:, None])
    return out.numpy()


@pytest.mark.parametrize("layout", [0, 1])
def test_oracle_matches_sort_recipe_on_tiny_workload(layout):
    inp = synthetic.make_inputs("tiny", device="cpu")
    wts = oracle.Weights(inp.x, inp.w1, inp.b1, inp.w2, inp.b2)
    out = oracle.forward_rows(wts, inp.topk_idx.numpy(), inp.topk_w.numpy(), layout=layout)
    ref = _recipe_torch_cpu(inp, layout)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-11)


def check_combine_direct_sum(lib=None):
    """The combine oracle against a per-slot sum that finds each pair's sorted
    position by search (raises AssertionError on a mismatch)."""
    rng = np.random.default_rng(5)
    idx = rng.integers(-1, 4, size=(9, 3)).astype(np.int32)
    w = rng.random((9, 3)).astype(np.float32)
    md = oracle.metadata(idx, w, 4, lib_path=lib)
    ys = rng.standard_normal((md["P"], 7))
    out = oracle.combine(md["token_offset"], md["s_reverse_scatter_idx"], md["scores"], ys, lib_path=lib)
    ref = np.zeros((9, 7))
    for t in range(9):
        for k in range(3):
            e = idx[t, k]
            if e < 0:
                continue
            # position of this (t,k) pair in expert-sorted order, found by search
            q = int(np.count_nonzero(idx[:t] >= 0) + np.count_nonzero(idx[t, :k] >= 0))
            p = int(np.nonzero(md["s_scatter_idx"] == q)[0][0])
            ref[t] += float(w[t, k]) * ys[p]
    np.testing.assert_allclose(out, ref, rtol=1e-13, atol=1e-13)


def test_combine_oracle_against_direct_sum():
    check_combine_direct_sum()
