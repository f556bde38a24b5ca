"""GPU backward (moe_nonexpand_forward_train + moe_nonexpand_backward)
against the backward oracle.

Every gradient is compared with the forward's tolerance widened by the
rounding noise of the backward's bf16 intermediates,
|gpu - ref| <= 2e-2 |ref| + 2e-2 rms(ref) + 8 * 2^-8 * rss (tests/helpers.py):
the GPU keeps z, dy, dz and the per-pair dx rows in bf16 and accumulates in
fp32, the oracle is exact double on the same bf16 inputs, and rss, the root
sum of squares of an entry's terms, is the scale of that noise.  Small cases are compared
everywhere; the prefill workload, at full size, on two experts' complete
weight gradients and on a sample of tokens.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_close, assert_close_bwd, backward_rss, tile_rows, to_np
from mixture_experts_routed_non_b200 import binding, synthetic

pytestmark = pytest.mark.gpu

GRADS = ("dx", "dw1", "dw2", "dtopk_w")


def _concat_from_interleaved(w1, b1):
    w1c = torch.cat([w1[:, :, 0::2], w1[:, :, 1::2]], dim=2).contiguous()
    b1c = None if b1 is None else torch.cat([b1[:, 0::2], b1[:, 1::2]], dim=1).contiguous()
    return w1c, b1c


def _dout(wl, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    return torch.randn((wl.N, wl.H), generator=g, device="cuda").to(torch.bfloat16)


def _run(inp, layout, dout, bias_grads=True):
    wl = inp.wl
    w1, b1 = inp.w1, inp.b1
    if layout == 1:
        w1, b1 = _concat_from_interleaved(w1, b1)
    ws = binding.alloc_train_workspace(wl.N, wl.H, wl.I, wl.E, wl.K)
    out = binding.forward_train(inp.x, inp.topk_idx, inp.topk_w, w1, inp.w2, b1, inp.b2, ws=ws, layout=layout)
    grads = binding.backward(dout, inp.x, inp.topk_idx, inp.topk_w, w1, inp.w2, ws=ws, layout=layout,
                             bias_grads=bias_grads and inp.b1 is not None)
    torch.cuda.synchronize()
    assert binding.read_error(ws) == 0
    return out, grads, w1, b1


def _check_full(inp, layout, seed=0):
    wl = inp.wl
    dout = _dout(wl, seed + 100)
    out, grads, w1, b1 = _run(inp, layout, dout)
    # the training forward computes the same output as the forward
    ref_out = binding.forward(inp.x, inp.topk_idx, inp.topk_w, w1, inp.w2, b1, inp.b2, layout=layout)
    assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16))
    wd = oracle.WeightsF64(inp.x, w1, b1, inp.w2, inp.b2)
    ref = oracle.backward(wd, inp.topk_idx.cpu().numpy(), inp.topk_w.cpu().numpy(), dout, layout)
    rss = backward_rss(ref, wd, dout)
    for k in GRADS + (("db1", "db2") if "db1" in grads else ()):
        assert_close_bwd(to_np(grads[k]), ref[k], rss[k], f"{k} ({wl.name}, layout {layout})")


@pytest.mark.parametrize("layout", [0, 1])
def test_tiny_backward_full(layout):
    inp = synthetic.make_inputs("tiny", device="cuda", invalid_value=float("nan"))
    _check_full(inp, layout)


@pytest.mark.parametrize("N,H,I,E,K,p_invalid,bias,seed", [
    (300, 256, 192, 5, 3, 0.2, True, 2),      # I % 128 == 64: partial column tiles
    (129, 192, 128, 3, 2, 0.0, False, 3),     # H % 256 == 192
    (700, 128, 64, 9, 4, 0.3, True, 4),       # I = 64
    (64, 320, 320, 2, 1, 0.5, True, 6),
    (50, 128, 128, 64, 2, 0.0, True, 7),      # most experts empty: zero weight gradients
])
@pytest.mark.parametrize("layout", [0, 1])
def test_ragged_backward_full(N, H, I, E, K, p_invalid, bias, seed, layout):
    wl = synthetic.custom(N, H, I, E, K, p_invalid=p_invalid, bias=bias, seed=seed)
    inp = synthetic.make_inputs(wl, device="cuda", invalid_value=float("nan"))
    _check_full(inp, layout, seed)


def test_backward_deterministic():
    inp = synthetic.make_inputs("tiny", device="cuda")
    dout = _dout(inp.wl, 5)
    _, g1, _, _ = _run(inp, 0, dout)
    _, g2, _, _ = _run(inp, 0, dout)
    for k in g1:
        assert torch.equal(g1[k].view(torch.uint8), g2[k].view(torch.uint8)), k


def test_prefill_backward_sampled():
    """Full-size prefill, the launch configuration the benchmark times: two
    experts' dW1/dW2 complete, and the dx / score-gradient rows of 24 tokens."""
    inp = synthetic.make_inputs("prefill", device="cuda")
    wl = inp.wl
    dout = _dout(wl, 11)
    _, grads, _, _ = _run(inp, 0, dout, bias_grads=False)
    idx, w = inp.topk_idx.cpu().numpy(), inp.topk_w.cpu().numpy()
    wd = oracle.WeightsF64(inp.x, inp.w1, None, inp.w2, None)
    experts = [7, 100]
    ref = oracle.backward(wd, idx, w, dout, 0, experts_only=experts)
    rss = backward_rss(ref, wd, dout)
    for k in ("dw1", "dw2"):
        assert_close_bwd(to_np(grads[k][experts]), ref[k][experts], rss[k][experts],
                         f"{k} (prefill, experts {experts})")
    tokens = np.sort(np.random.default_rng(3).choice(wl.N, size=24, replace=False))
    sub = np.full_like(idx, -1)
    sub[tokens] = idx[tokens]
    ref_t = oracle.backward(wd, sub, w, dout, 0)
    rss_t = backward_rss(ref_t, wd, dout)
    assert_close_bwd(to_np(grads["dx"])[tokens], ref_t["dx"][tokens], rss_t["dx"][tokens],
                     "dx (prefill, sampled tokens)")
    assert_close_bwd(to_np(grads["dtopk_w"])[tokens], ref_t["dtopk_w"][tokens], rss_t["dtopk_w"][tokens],
                     "dtopk_w (prefill, sampled tokens)")


@pytest.mark.parametrize("bits", [32, 64])
def test_pair_list_backward_equals_table_backward_bitwise(bits):
    """The pair list of a table (invalid slots dropped) is the same routing in
    the same pair order: every gradient is bit-identical, and each entry's
    score gradient is its slot's."""
    dt = {32: torch.int32, 64: torch.int64}[bits]
    inp = synthetic.make_inputs("tiny", device="cuda", invalid_value=float("nan"))
    wl = inp.wl
    dout = _dout(wl, 21)
    _, ga, _, _ = _run(inp, 0, dout)
    tok, exp, wt = synthetic.pair_list_from_table(inp.topk_idx.cpu().numpy(), inp.topk_w.cpu().numpy())
    ti, ei, wi = (torch.from_numpy(v).cuda() for v in (tok, exp, wt))
    ti, ei = ti.to(dt), ei.to(dt)
    r = binding.routing(ei, wi, token_idx=ti, N=wl.N)
    ws = torch.empty(binding.routed_train_workspace_bytes(r, wl.H, wl.I, wl.E), dtype=torch.uint8, device="cuda")
    binding.routed_forward_train(inp.x, ei, wi, inp.w1, inp.w2, inp.b1, inp.b2, ws=ws, token_idx=ti)
    gb = binding.routed_backward(dout, inp.x, ei, wi, inp.w1, inp.w2, ws=ws, token_idx=ti, bias_grads=True)
    torch.cuda.synchronize()
    assert binding.read_error(ws) == 0
    for k in ("dx", "dw1", "dw2", "db1", "db2"):
        assert torch.equal(ga[k].view(torch.int16), gb[k].view(torch.int16)), k
    valid = inp.topk_idx >= 0
    assert torch.equal(gb["dweights"].view(torch.int32), ga["dtopk_w"][valid].view(torch.int32))


@pytest.mark.parametrize("bits", [32, 64])
def test_pair_list_backward_heavy_tokens_and_dropped_entries(bits):
    """Tokens routed to all 300 experts (more pairs than one batch of the
    score-gradient kernel), tokens without pairs, dropped entries."""
    dt = {32: torch.int32, 64: torch.int64}[bits]
    wl = synthetic.custom(N=300, H=256, I=192, E=300, K=4, bias=True, seed=12, name="heavy")
    inp = synthetic.make_inputs(wl, device="cuda")
    rng = np.random.default_rng(4)
    heavy = np.array([0, 7, 150, 299])
    tok, exp, wt = synthetic.many_pair_tokens(wl.N, wl.E, heavy, wl.K, rng)
    keep = ~np.isin(tok, [30, 31, 200])
    tok, exp, wt = tok[keep], exp[keep].copy(), wt[keep]
    exp[3] = -1
    exp[100] = wl.E + 5
    ti, ei, wi = (torch.from_numpy(np.ascontiguousarray(v)).cuda() for v in (tok, exp, wt))
    ti, ei = ti.to(dt), ei.to(dt)
    r = binding.routing(ei, wi, token_idx=ti, N=wl.N)
    ws = torch.empty(binding.routed_train_workspace_bytes(r, wl.H, wl.I, wl.E), dtype=torch.uint8, device="cuda")
    binding.routed_forward_train(inp.x, ei, wi, inp.w1, inp.w2, inp.b1, inp.b2, ws=ws, token_idx=ti)
    dout = _dout(wl, 22)
    g = binding.routed_backward(dout, inp.x, ei, wi, inp.w1, inp.w2, ws=ws, token_idx=ti, bias_grads=True)
    torch.cuda.synchronize()
    assert binding.read_error(ws) == binding.DEVERR_BAD_EXPERT_ID
    wd = oracle.WeightsF64(inp.x, inp.w1, inp.b1, inp.w2, inp.b2)
    ref = oracle.backward_pairs(wd, tok, exp, wt, dout)
    rss = backward_rss(ref, wd, dout)
    for k in ("dx", "dw1", "dw2", "db1", "db2", "dweights"):
        assert_close_bwd(to_np(g[k]), ref[k], rss[k], f"{k} (pair list, heavy tokens)")
    assert g["dweights"][3].item() == 0.0 and g["dweights"][100].item() == 0.0


def test_backward_with_no_pairs_gives_zero_gradients():
    """Every slot invalid (P = 0): the weight gradients are written as zeros,
    dx and the score gradients are zero."""
    wl = synthetic.custom(50, 128, 128, 6, 2, bias=True, seed=13)
    inp = synthetic.make_inputs(wl, device="cuda")
    inp.topk_idx.fill_(-1)
    dout = _dout(wl, 31)
    _, g, _, _ = _run(inp, 0, dout)
    for k, v in g.items():
        assert torch.count_nonzero(v) == 0, k


def test_backward_int64_table_equals_int32_table_bitwise():
    inp = synthetic.make_inputs("tiny", device="cuda", invalid_value=float("nan"))
    wl = inp.wl
    dout = _dout(wl, 41)
    _, ga, _, _ = _run(inp, 1, dout)
    idx64 = inp.topk_idx.to(torch.int64)
    w1c, b1c = _concat_from_interleaved(inp.w1, inp.b1)
    r = binding.routing(idx64, inp.topk_w)
    ws = torch.empty(binding.routed_train_workspace_bytes(r, wl.H, wl.I, wl.E), dtype=torch.uint8, device="cuda")
    binding.routed_forward_train(inp.x, idx64, inp.topk_w, w1c, inp.w2, b1c, inp.b2, ws=ws, layout=1)
    gb = binding.routed_backward(dout, inp.x, idx64, inp.topk_w, w1c, inp.w2, ws=ws, layout=1, bias_grads=True)
    torch.cuda.synchronize()
    for k in ("dx", "dw1", "dw2", "db1", "db2"):
        assert torch.equal(ga[k].view(torch.int16), gb[k].view(torch.int16)), k
    assert torch.equal(ga["dtopk_w"].view(torch.int32), gb["dweights"].view(torch.int32))


def test_prefill256_backward_skewed_routing():
    """Zipf routing over 256 experts at full size: no wait may run out (the
    error word stays 0), a mid-sized and a small expert's weight gradients
    match the oracle, and experts without pairs get zero gradients."""
    inp = synthetic.make_inputs("prefill256", device="cuda")
    wl = inp.wl
    dout = _dout(wl, 51)
    _, grads, _, _ = _run(inp, 0, dout, bias_grads=False)  # asserts the error word is 0
    idx, w = inp.topk_idx.cpu().numpy(), inp.topk_w.cpu().numpy()
    freq = np.bincount(idx[idx >= 0], minlength=wl.E)
    mid = int(np.argmin(np.abs(freq - 600)))
    small = int(np.argmin(np.where(freq > 0, np.abs(freq - 40), 1 << 30)))
    experts = [mid, small]
    wd = oracle.WeightsF64(inp.x, inp.w1, None, inp.w2, None)
    ref = oracle.backward(wd, idx, w, dout, 0, experts_only=experts)
    rss = backward_rss(ref, wd, dout)
    for k in ("dw1", "dw2"):
        assert_close_bwd(to_np(grads[k][experts]), ref[k][experts], rss[k][experts],
                         f"{k} (prefill256, experts {experts} with {freq[experts].tolist()} rows)")
    empty = np.nonzero(freq == 0)[0]
    if empty.size:
        e = torch.from_numpy(empty).cuda()
        assert torch.count_nonzero(grads["dw1"][e]) == 0 and torch.count_nonzero(grads["dw2"][e]) == 0


def test_prefill256_backward_every_tile():
    """Full-size, Zipf-skewed (256 experts, segments of ~50 to ~15k rows), the
    launch configuration the bench times: DH's dz and DX's per-pair dx rows on
    the boundary rows of every (expert, 256-row m-tile), and the complete dW1
    and dW2 -- every one of their tiles -- of the most and the least popular
    expert with pairs."""
    inp = synthetic.make_inputs("prefill256", device="cuda")
    wl = inp.wl
    dout = _dout(wl, 31)
    _, grads, _, _ = _run(inp, 0, dout, bias_grads=False)
    ws_args = (wl.N, wl.H, wl.I, wl.E, wl.K)
    idx, w = inp.topk_idx.cpu().numpy(), inp.topk_w.cpu().numpy()
    meta = oracle.metadata(idx, w, wl.E)
    wd = oracle.WeightsF64(inp.x, inp.w1, None, inp.w2, None)
    # the workspace of the run above holds dz and the dx rows: recompute them in a
    # fresh training workspace so the views below belong to this call
    ws = binding.alloc_train_workspace(*ws_args)
    binding.forward_train(inp.x, inp.topk_idx, inp.topk_w, inp.w1, inp.w2, ws=ws)
    binding.backward(dout, inp.x, inp.topk_idx, inp.topk_w, inp.w1, inp.w2, ws=ws)
    torch.cuda.synchronize()
    assert binding.read_error(ws) == 0
    dz_gpu, dxr_gpu = binding.backward_intermediates_from_workspace(ws, *ws_args)
    ps = tile_rows(meta["off"])
    tok = meta["x_gather_idx"][ps]
    ex = (np.searchsorted(meta["off"], ps, side="right") - 1).astype(np.int32)
    sc = meta["scores"][meta["s_scatter_idx"][ps]]
    ref = oracle.pairs_backward(wd, dout, tok, ex, sc, 0)
    ps_t = torch.from_numpy(ps).cuda()
    assert_close(to_np(dz_gpu[ps_t]), ref["dz"], f"dz (DH) on {ps.size} tile boundary rows")
    dxr_ref = oracle.pair_dx_rows(wd, ref["dz"], ex)
    # root sum of squares of the terms of each dx-row entry: sum_c (dz_c w1[e][j, c])^2
    rss = np.zeros_like(dxr_ref)
    for e in np.unique(ex):
        sel = ex == e
        rss[sel] = (ref["dz"][sel] ** 2) @ (wd.w1e(e) ** 2).T
    assert_close_bwd(to_np(dxr_gpu[ps_t]), dxr_ref, np.sqrt(rss), f"per-pair dx rows (DX) on {ps.size} rows")
    freq = meta["freq"]
    nz = np.nonzero(freq)[0]
    experts = [int(nz[np.argmax(freq[nz])]), int(nz[np.argmin(freq[nz])])]
    refw = oracle.backward(wd, idx, w, dout, 0, experts_only=experts)
    rssw = backward_rss(refw, wd, dout)
    for k in ("dw1", "dw2"):
        assert_close_bwd(to_np(grads[k][experts]), refw[k][experts], rssw[k][experts],
                         f"{k} (prefill256, experts {experts}, M_e {[int(freq[e]) for e in experts]})")
