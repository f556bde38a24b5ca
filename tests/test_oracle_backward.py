"""Pins of the backward oracle (oracle.pairs_backward / oracle.backward).

The pages leave the backward open (sonic-moe issue #68 asks how the routing
scores get their gradient back to [N,K]); the oracle applies the chain rule
to the forward.  Pinned by: its forward part against the pinned forward
oracle; central finite differences of sum_t <dout_t, out_t> for every input;
torch autograd through an independent float64 implementation of the
sort-by-expert recipe (qwen3_5.py commit notes, steps 1-5).
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from mixture_experts_routed_non_b200 import synthetic

GRADS = ("dx", "dw1", "db1", "dw2", "db2", "dtopk_w")


def _small_problem(seed=0, layout=0):
    rng = np.random.default_rng(seed)
    N, H, I, E, K = 4, 8, 4, 3, 2
    wd = oracle.WeightsF64(rng.standard_normal((N, H)), rng.standard_normal((E, H, 2 * I)) * 0.4,
                           rng.standard_normal((E, 2 * I)) * 0.2, rng.standard_normal((E, I, H)) * 0.4,
                           rng.standard_normal((E, H)) * 0.2)
    idx = np.array([[0, 2], [1, -1], [2, 0], [-1, -1]], np.int32)
    tw = rng.random((N, K))
    dout = rng.standard_normal((N, H))
    return wd, idx, tw, dout


def _loss(wd, idx, tw, dout, layout, lib=None):
    """sum_t <dout_t, out_t> with out from the oracle's double forward."""
    N, K = idx.shape
    tok, slot = np.nonzero(idx >= 0)
    r = oracle.pairs_backward(wd, dout, tok, idx[tok, slot], tw[tok, slot], layout, lib_path=lib)
    out = np.zeros((N, wd.H))
    np.add.at(out, tok, tw[tok, slot][:, None] * r["y"])
    return float((out * dout).sum())


def check_finite_differences(layout, lib=None, eps=1e-6):
    wd, idx, tw, dout = _small_problem(1, layout)
    g = oracle.backward(wd, idx, tw, dout, layout, lib_path=lib)
    fields = {"dx": (wd, "x"), "dw1": (wd, "_w1"), "db1": (wd, "b1"), "dw2": (wd, "_w2"), "db2": (wd, "b2")}
    for gname, (obj, attr) in fields.items():
        arr = getattr(obj, attr)
        num = np.zeros_like(arr)
        for i in np.ndindex(arr.shape):
            keep = arr[i]
            arr[i] = keep + eps
            lp = _loss(wd, idx, tw, dout, layout, lib)
            arr[i] = keep - eps
            lm = _loss(wd, idx, tw, dout, layout, lib)
            arr[i] = keep
            num[i] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(g[gname], num, rtol=1e-6, atol=1e-7, err_msg=gname)
    num = np.zeros_like(tw)
    for i in np.ndindex(tw.shape):
        if idx[i] < 0:
            continue
        keep = tw[i]
        tw[i] = keep + eps
        lp = _loss(wd, idx, tw, dout, layout, lib)
        tw[i] = keep - eps
        lm = _loss(wd, idx, tw, dout, layout, lib)
        tw[i] = keep
        num[i] = (lp - lm) / (2 * eps)
    np.testing.assert_allclose(g["dtopk_w"], num, rtol=1e-6, atol=1e-7, err_msg="dtopk_w")


def _recipe_autograd(inp, dout, layout):
    """float64 torch autograd through the sort-by-expert recipe: flatten the
    valid assignments, stable sort by expert, F.linear per expert slice,
    silu x up, index_add_ of the score-weighted rows."""
    x = inp.x.double().requires_grad_()
    w1 = inp.w1.double().requires_grad_()
    w2 = inp.w2.double().requires_grad_()
    b1 = inp.b1.double().requires_grad_()
    b2 = inp.b2.double().requires_grad_()
    tw = inp.topk_w.double().requires_grad_()
    idx = inp.topk_idx.long()
    N, K = idx.shape
    E, H, I2 = w1.shape
    I = I2 // 2
    flat_e = idx.reshape(-1)
    flat_t = torch.arange(N).repeat_interleave(K)
    flat_s = torch.arange(N * K)
    keep = flat_e >= 0
    flat_e, flat_t, flat_s = flat_e[keep], flat_t[keep], flat_s[keep]
    order = torch.sort(flat_e, stable=True).indices
    e_s, t_s, s_s = flat_e[order], flat_t[order], flat_s[order]
    xs = x[t_s]
    zs, ys = [], []
    for e in range(E):
        sel = e_s == e
        zs.append(F.linear(xs[sel], w1[e].t(), b1[e]))
    z = torch.cat(zs)
    g, u = (z[:, 0::2], z[:, 1::2]) if layout == 0 else (z[:, :I], z[:, I:])
    hs = F.silu(g) * u
    start = 0
    for e in range(E):
        n = int((e_s == e).sum())
        ys.append(F.linear(hs[start:start + n], w2[e].t(), b2[e]))
        start += n
    y = torch.cat(ys)
    out = torch.zeros(N, H, dtype=torch.float64).index_add(0, t_s, y * tw.reshape(-1)[s_s][:, None])
    out.backward(torch.from_numpy(dout))
    return dict(dx=x.grad.numpy(), dw1=w1.grad.numpy(), db1=b1.grad.numpy(), dw2=w2.grad.numpy(),
                db2=b2.grad.numpy(), dtopk_w=tw.grad.numpy())


def check_autograd(layout, lib=None):
    inp = synthetic.make_inputs("tiny", device="cpu")
    dout = np.random.default_rng(2).standard_normal((inp.wl.N, inp.wl.H))
    wd = oracle.WeightsF64(inp.x, inp.w1, inp.b1, inp.w2, inp.b2)
    g = oracle.backward(wd, inp.topk_idx.numpy(), inp.topk_w.numpy(), dout, layout, lib_path=lib)
    ref = _recipe_autograd(inp, dout, layout)
    for k in GRADS:
        np.testing.assert_allclose(g[k], ref[k], rtol=1e-9, atol=1e-10, err_msg=k)


def test_backward_forward_part_matches_forward_oracle():
    inp = synthetic.make_inputs("tiny", device="cpu")
    wl = inp.wl
    wd = oracle.WeightsF64(inp.x, inp.w1, inp.b1, inp.w2, inp.b2)
    wts = oracle.Weights(inp.x, inp.w1, inp.b1, inp.w2, inp.b2)
    idx = inp.topk_idx.numpy()
    tok, slot = np.nonzero(idx >= 0)
    tok, slot = tok[:200], slot[:200]
    for layout in (0, 1):
        r = oracle.pairs_backward(wd, np.zeros((wl.N, wl.H)), tok, idx[tok, slot], np.ones(len(tok)), layout)
        h, y = oracle.pair_rows(wts, tok, idx[tok, slot], layout=layout)
        np.testing.assert_allclose(r["h"], h, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(r["y"], y, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("layout", [0, 1])
def test_backward_finite_differences(layout):
    check_finite_differences(layout)


@pytest.mark.parametrize("layout", [0, 1])
def test_backward_matches_torch_autograd(layout):
    check_autograd(layout)


def test_backward_experts_only_is_complete_for_those_experts():
    inp = synthetic.make_inputs("tiny", device="cpu")
    dout = np.random.default_rng(4).standard_normal((inp.wl.N, inp.wl.H))
    wd = oracle.WeightsF64(inp.x, inp.w1, inp.b1, inp.w2, inp.b2)
    idx, w = inp.topk_idx.numpy(), inp.topk_w.numpy()
    full = oracle.backward(wd, idx, w, dout)
    part = oracle.backward(wd, idx, w, dout, experts_only=[3, 5])
    for k in ("dw1", "db1", "dw2", "db2"):
        np.testing.assert_array_equal(part[k][[3, 5]], full[k][[3, 5]])


def test_backward_pairs_equals_table_backward_on_its_flattening():
    """A pair list holding a table's valid slots in row-major order is the same
    routing: every gradient matches, and each entry's score gradient is its
    slot's."""
    inp = synthetic.make_inputs("tiny", device="cpu", invalid_value=float("nan"))
    dout = np.random.default_rng(8).standard_normal((inp.wl.N, inp.wl.H))
    wd = oracle.WeightsF64(inp.x, inp.w1, inp.b1, inp.w2, inp.b2)
    idx, w = inp.topk_idx.numpy(), inp.topk_w.numpy()
    tok, exp, wt = synthetic.pair_list_from_table(idx, w)
    for layout in (0, 1):
        a = oracle.backward(wd, idx, w, dout, layout)
        b = oracle.backward_pairs(wd, tok, exp, wt, dout, layout)
        for k in ("dx", "dw1", "db1", "dw2", "db2"):
            np.testing.assert_allclose(b[k], a[k], rtol=1e-13, atol=1e-13, err_msg=k)
        np.testing.assert_allclose(b["dweights"], a["dtopk_w"][idx >= 0], rtol=1e-13, atol=1e-13)


def test_backward_pairs_dropped_entries_have_zero_gradient():
    inp = synthetic.make_inputs("tiny", device="cpu")
    dout = np.random.default_rng(9).standard_normal((inp.wl.N, inp.wl.H))
    wd = oracle.WeightsF64(inp.x, inp.w1, inp.b1, inp.w2, inp.b2)
    tok, exp, wt = synthetic.pair_list_from_table(inp.topk_idx.numpy(), inp.topk_w.numpy())
    tok, exp = tok.copy(), exp.copy()
    exp[5] = -1
    exp[9] = inp.wl.E + 2
    tok[-2:] = inp.wl.N
    g = oracle.backward_pairs(wd, tok, exp, wt, dout)
    assert g["dweights"][[5, 9, len(tok) - 2, len(tok) - 1]].tolist() == [0.0] * 4
    keep = np.ones(len(tok), bool)
    keep[[5, 9, len(tok) - 2, len(tok) - 1]] = False
    h = oracle.backward_pairs(wd, tok[keep], exp[keep], wt[keep], dout)
    for k in ("dx", "dw1", "dw2"):
        np.testing.assert_array_equal(g[k], h[k])
    np.testing.assert_array_equal(g["dweights"][keep], h["dweights"])


def _sum_pair_terms_mutant(kind):
    """A copy of the oracle's summation of the per-pair backward terms with one
    plausible mistake planted (test code; the oracle itself is untouched)."""
    def summed(wd, dout, tok, exp, sc, N, layout, lib_path):
        H, I, E = wd.H, wd.I, wd.E
        r = oracle.pairs_backward(wd, dout, tok, exp, sc, layout, lib_path=lib_path)
        g = dict(dx=np.zeros((N, H)), dw1=np.zeros((E, H, 2 * I)), db1=np.zeros((E, 2 * I)),
                 dw2=np.zeros((E, I, H)), db2=np.zeros((E, H)))
        g["pairs"] = dict(tok=tok, exp=exp, **r)
        for e in np.unique(exp):
            sel = exp == e
            te = tok[sel]
            g["dw2"][e] = r["h"][sel].T @ r["dy"][sel]
            g["db2"][e] = r["dy"][sel].sum(0)
            rows = tok[:int(sel.sum())] if kind == "dw1_rows_of_first_tokens" else te
            g["dw1"][e] = wd.x[rows].T @ r["dz"][sel]
            if kind != "db1_dropped":
                g["db1"][e] = r["dz"][sel].sum(0)
            if kind == "dx_overwritten_per_expert":
                g["dx"][te] = r["dz"][sel] @ wd.w1e(e).T
            else:
                np.add.at(g["dx"], te, r["dz"][sel] @ wd.w1e(e).T)
        return g
    return summed


@pytest.mark.parametrize("kind", ["db1_dropped", "dw1_rows_of_first_tokens", "dx_overwritten_per_expert"])
def test_finite_differences_reject_summation_mistakes(monkeypatch, kind):
    """The summation of the per-pair terms is numpy code outside the C source
    the mutation suite edits; the finite-difference pin must still catch a
    mistake planted there."""
    monkeypatch.setattr(oracle, "_sum_pair_terms", _sum_pair_terms_mutant(None))
    check_finite_differences(0)                      # the unmutated copy passes
    monkeypatch.setattr(oracle, "_sum_pair_terms", _sum_pair_terms_mutant(kind))
    with pytest.raises(AssertionError):
        check_finite_differences(0)


def test_pair_dx_rows_sum_to_the_pinned_dx():
    """oracle.pair_dx_rows gives each pair's share of dx (dz . w1[e]^T); summed
    per token they are the backward oracle's dx, which the finite differences
    above pin."""
    import torch

    from mixture_experts_routed_non_b200 import synthetic
    inp = synthetic.make_inputs("tiny", device="cpu")
    wd = oracle.WeightsF64(inp.x, inp.w1, inp.b1, inp.w2, inp.b2)
    g_ = torch.Generator().manual_seed(3)
    dout = torch.randn((inp.wl.N, inp.wl.H), generator=g_).to(torch.bfloat16)
    g = oracle.backward(wd, inp.topk_idx.numpy(), inp.topk_w.numpy(), dout, 0)
    pr = g["pairs"]
    rows = oracle.pair_dx_rows(wd, pr["dz"], pr["exp"])
    dx = np.zeros_like(g["dx"])
    np.add.at(dx, pr["tok"], rows)
    np.testing.assert_allclose(dx, g["dx"], rtol=0, atol=1e-12)
