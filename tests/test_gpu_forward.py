"""GPU forward (moe_nonexpand_forward) against the oracle.

Small cases are compared element by element on every output; the full-size
workloads, in the launch configuration the benchmark times, are compared on a
seeded sample of tokens the oracle computes one by one.  Metadata is compared
bit-exactly in every case, and the bf16 intermediates h and y are checked
against the oracle's per-pair rows so a failure points at the stage.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_close, check_meta_equal, tile_rows, to_np, within_tolerance
from mixture_experts_routed_non_b200 import binding, synthetic

pytestmark = pytest.mark.gpu


def _concat_from_interleaved(w1, b1):
    w1c = torch.cat([w1[:, :, 0::2], w1[:, :, 1::2]], dim=2).contiguous()
    b1c = None if b1 is None else torch.cat([b1[:, 0::2], b1[:, 1::2]], dim=1).contiguous()
    return w1c, b1c


def run_case(inp, layout=0, total_pairs=-1, sample=None, check_stages=True, seed=0, every_tile=False):
    """Forward of ``inp``; metadata compared bit-exactly, the output on all
    tokens (or a seeded sample of ``sample`` tokens), and the intermediates h
    (bf16) and y (fp16 with an exponent per 32 columns) on every pair of the
    compared tokens -- plus, with ``every_tile``, on the boundary rows of every
    (expert, m-tile) of the run."""
    wl = inp.wl
    N, H, I, E, K = wl.N, wl.H, wl.I, wl.E, wl.K
    w1, b1 = inp.w1, inp.b1
    if layout == 1:
        w1, b1 = _concat_from_interleaved(w1, b1)
    ws = binding.alloc_workspace(N, H, I, E, K, total_pairs, inp.x.device)
    out = binding.forward(inp.x, inp.topk_idx, inp.topk_w, w1, inp.w2, b1, inp.b2, layout=layout,
                          total_pairs=total_pairs, ws=ws)
    err = binding.read_error(ws)
    assert err == 0, f"device error word {err:#x}"

    idx = inp.topk_idx.cpu().numpy()
    w = inp.topk_w.cpu().numpy()
    ref_meta = oracle.metadata(idx, w, E)
    check_meta_equal(binding.meta_from_workspace(ws, N, H, I, E, K, total_pairs), ref_meta)

    wts = oracle.Weights(inp.x, w1, b1, inp.w2, inp.b2)
    if sample is None:
        tokens = np.arange(N)
    else:
        tokens = np.sort(np.random.default_rng(seed).choice(N, size=min(sample, N), replace=False))
    if check_stages and ref_meta["P"] > 0:
        # intermediates: every pair of the compared tokens, and the tile boundary rows
        P = ref_meta["P"]
        h_gpu, y16, y_scale = binding.intermediates_from_workspace(ws, N, H, I, E, K, total_pairs)
        assert P <= h_gpu.shape[0]
        to = ref_meta["token_offset"]
        qs = np.concatenate([np.arange(to[t], to[t + 1]) for t in tokens] + [np.zeros(0, np.int64)])
        ps = ref_meta["s_reverse_scatter_idx"][qs].astype(np.int64)
        if every_tile:
            ps = np.union1d(ps, tile_rows(ref_meta["off"]))
        if ps.size:
            tok = ref_meta["x_gather_idx"][ps]
            ex = np.searchsorted(ref_meta["off"], ps, side="right") - 1
            h_ref, y_ref = oracle.pair_rows(wts, tok, ex, layout=layout)
            ps_t = torch.from_numpy(ps).to(h_gpu.device)
            assert_close(to_np(h_gpu[ps_t]), h_ref, f"h (up GEMM + SwiGLU, {ps.size} rows)")
            # y: fp16 times 2^e per 32-column block of each row
            yf = to_np(y16[ps_t].float()).astype(np.float64)
            e = to_np(y_scale[ps_t]).astype(np.int64)
            assert np.all((e >= -100) & (e <= 113)), "exponent out of range"
            yv = yf * np.exp2(np.repeat(e, 32, axis=1))
            assert_close(yv, y_ref, f"y (down GEMM, fp16 x 2^e, {ps.size} rows)")
            # no block's fp16 exceeds 2^15 (fp16 rounding may carry a maximum just below
            # 2^15 to 2^15 itself); the grouped GEMM puts each block's largest in
            # [2^14, 2^15] (or the block is zero, or the exponent sits at its floor); the
            # decode kernels share an exponent over up to 32 rows of one expert
            bmax = np.abs(yf).reshape(ps.size, -1, 32).max(axis=2)
            assert np.all(bmax <= 2.0 ** 15), "a block's fp16 values exceed 2^15"
            lay = binding.workspace_layout(N, H, I, E, K, total_pairs)
            if lay.p_cap > 32 * E:  # the grouped GEMM path
                ok = (bmax >= 2.0 ** 14) | (bmax == 0) | (e == -100)
                assert np.all(ok), "a block's exponent does not match its largest value"
    ref = oracle.forward_rows(wts, idx, w, tokens=tokens, layout=layout)
    got = to_np(out)[tokens]
    assert_close(got, ref, f"out ({wl.name}, layout {layout})")
    return out, ws


@pytest.mark.parametrize("layout", [0, 1])
def test_tiny_workload_full(layout):
    inp = synthetic.make_inputs("tiny", device="cuda", invalid_value=float("nan"))
    run_case(inp, layout=layout)


@pytest.mark.parametrize("layout", [0, 1])
def test_tiny_workload_with_total_pairs(layout):
    inp = synthetic.make_inputs("tiny", device="cuda")
    run_case(inp, layout=layout, total_pairs=inp.total_pairs)


@pytest.mark.parametrize("N,H,I,E,K,p_invalid,bias,seed", [
    (1, 64, 64, 1, 1, 0.0, True, 1),          # one token, one expert, smallest tile
    (300, 256, 192, 5, 3, 0.2, True, 2),      # I % 128 == 64: partial last column tile
    (129, 192, 128, 3, 2, 0.0, False, 3),     # H % 256 == 192: partial down tile
    (700, 128, 64, 9, 4, 0.3, True, 4),       # I = 64
    (1000, 512, 256, 64, 8, 0.1, False, 5),   # many small segments
    (64, 320, 320, 2, 1, 0.5, True, 6),
])
@pytest.mark.parametrize("layout", [0, 1])
def test_ragged_shapes_full(N, H, I, E, K, p_invalid, bias, seed, layout):
    wl = synthetic.custom(N, H, I, E, K, p_invalid=p_invalid, bias=bias, seed=seed,
                          routing_kind="uniform" if K <= E else "ranklocal")
    if K > E:
        pytest.skip("distinct routing needs K <= E")
    inp = synthetic.make_inputs(wl, device="cuda", invalid_value=float("nan"))
    run_case(inp, layout=layout)


def test_single_expert_single_slot_dense():
    wl = synthetic.custom(1000, 256, 256, 1, 1, bias=True, seed=7, scores_kind="uniform")
    inp = synthetic.make_inputs(wl, device="cuda")
    inp.topk_w.fill_(1.0)
    run_case(inp)


def test_duplicate_experts_and_tail_segments():
    """Long segments that are not a multiple of 128 rows, with the same expert
    twice in a row."""
    wl = synthetic.custom(2000, 128, 128, 4, 2, bias=True, seed=8)
    inp = synthetic.make_inputs(wl, device="cuda")
    idx = torch.tensor(np.random.default_rng(8).integers(0, 4, size=(2000, 2)), dtype=torch.int32)
    inp.topk_idx.copy_(idx)
    run_case(inp)


def test_all_slots_invalid_gives_zero():
    wl = synthetic.custom(50, 128, 64, 3, 2, seed=9)
    inp = synthetic.make_inputs(wl, device="cuda")
    inp.topk_idx.fill_(-1)
    inp.topk_w.fill_(float("nan"))
    ws = binding.alloc_workspace(50, 128, 64, 3, 2, -1)
    out = binding.forward(inp.x, inp.topk_idx, inp.topk_w, inp.w1, inp.w2, ws=ws)
    assert binding.read_error(ws) == 0
    assert torch.count_nonzero(out) == 0
    out = binding.forward(inp.x, inp.topk_idx, inp.topk_w, inp.w1, inp.w2, total_pairs=0)
    assert torch.count_nonzero(out) == 0


def test_forward_deterministic():
    inp = synthetic.make_inputs("tiny", device="cuda")
    ws = binding.alloc_workspace(256, 128, 256, 8, 2, -1)
    a = binding.forward(inp.x, inp.topk_idx, inp.topk_w, inp.w1, inp.w2, inp.b1, inp.b2, ws=ws).clone()
    for _ in range(3):
        b = binding.forward(inp.x, inp.topk_idx, inp.topk_w, inp.w1, inp.w2, inp.b1, inp.b2, ws=ws)
        assert torch.equal(a, b)


def test_bad_ids_flagged_forward_still_right():
    inp = synthetic.make_inputs("tiny", device="cuda")
    idx = inp.topk_idx.clone()
    idx[3, 0] = 99
    inp.topk_idx.copy_(idx)
    ws = binding.alloc_workspace(256, 128, 256, 8, 2, -1)
    out = binding.forward(inp.x, inp.topk_idx, inp.topk_w, inp.w1, inp.w2, inp.b1, inp.b2, ws=ws)
    assert binding.read_error(ws) == binding.DEVERR_BAD_EXPERT_ID
    wts = oracle.Weights(inp.x, inp.w1, inp.b1, inp.w2, inp.b2)
    ref = oracle.forward_rows(wts, inp.topk_idx.cpu().numpy(), inp.topk_w.cpu().numpy())
    assert_close(to_np(out), ref, "out with a bad id")


# ---- full-size workloads (the benchmark's launch configuration) ------------
# Every (expert, 256-row m-tile) of each run is compared on its boundary rows
# (tests/helpers.py tile_rows), and the output on a seeded 2048-token subset
# (all 128 tokens of the decode shape) with h and y on all of their pairs.

@pytest.mark.parametrize("name,sample", [("prefill", 2048), ("ranklocal", 2048), ("decode256", None),
                                         ("prefill256", 2048)])
def test_full_size_workloads_every_tile(name, sample):
    inp = synthetic.make_inputs(name, device="cuda")
    run_case(inp, sample=sample, seed=17, every_tile=True)
    del inp
    torch.cuda.empty_cache()


def test_prefill_with_total_pairs_and_concat_layout_every_tile():
    inp = synthetic.make_inputs("prefill", device="cuda")
    run_case(inp, layout=1, total_pairs=inp.total_pairs, sample=2048, seed=18, every_tile=True)
    del inp
    torch.cuda.empty_cache()


def test_full_size_properties_hold_everywhere():
    """Properties that hold at any size, over all rows: finite output, zero
    rows exactly for tokens with no valid slot, and a bitwise repeat."""
    inp = synthetic.make_inputs("ranklocal", device="cuda")
    inp.topk_idx[::97] = -1
    ws = binding.alloc_workspace(8192, 7168, 2048, 32, 8, -1)
    out = binding.forward(inp.x, inp.topk_idx, inp.topk_w, inp.w1, inp.w2, ws=ws).clone()
    assert binding.read_error(ws) == 0
    assert torch.isfinite(out.float()).all()
    empty = (inp.topk_idx < 0).all(dim=1)
    assert torch.count_nonzero(out[empty]) == 0
    assert torch.count_nonzero(out[~empty].float().abs().sum(1) == 0) == 0
    out2 = binding.forward(inp.x, inp.topk_idx, inp.topk_w, inp.w1, inp.w2, ws=ws)
    assert torch.equal(out, out2)


# ---- decode-sized segments: the swap-AB kernels (chosen when P_cap <= 32 E) ----

@pytest.mark.parametrize("N,H,I,E,K,p_invalid,bias,seed", [
    (64, 256, 192, 64, 8, 0.1, True, 21),     # I % 128 == 64: a 64-column last unit in the up GEMM
    (40, 320, 128, 32, 4, 0.0, False, 22),    # H % 128 == 64: half of the last down unit is out of range
    (128, 512, 256, 256, 8, 0.0, True, 23),   # the decode shape, smaller
    (1, 64, 64, 1, 1, 0.0, True, 24),         # one pair
    (16, 128, 64, 16, 2, 0.5, True, 25),      # many empty experts
])
@pytest.mark.parametrize("layout", [0, 1])
def test_decode_path_shapes_full(N, H, I, E, K, p_invalid, bias, seed, layout):
    assert N * K <= 32 * E  # the sizes select the decode kernels
    wl = synthetic.custom(N, H, I, E, K, p_invalid=p_invalid, bias=bias, seed=seed)
    inp = synthetic.make_inputs(wl, device="cuda", invalid_value=float("nan"))
    run_case(inp, layout=layout)
    run_case(inp, layout=layout, total_pairs=int((inp.topk_idx >= 0).sum()))


@pytest.mark.parametrize("layout", [0, 1])
def test_decode_path_long_segment_and_duplicates(layout):
    """One expert with 300 rows (three chunks of at most 128 tokens), the same
    expert twice in some rows, the rest spread thinly."""
    N, H, I, E, K = 320, 192, 128, 32, 2
    wl = synthetic.custom(N, H, I, E, K, bias=True, seed=26)
    inp = synthetic.make_inputs(wl, device="cuda")
    rng = np.random.default_rng(26)
    idx = rng.integers(0, E, size=(N, K)).astype(np.int32)
    idx[:300, 0] = 5
    idx[:40, 1] = 5
    inp.topk_idx.copy_(torch.from_numpy(idx))
    assert N * K <= 32 * E
    run_case(inp, layout=layout)


@pytest.mark.parametrize("name", ["decode256", "prefill256"])
def test_back_to_back_forwards_match_serialised_ones(name):
    """Forwards on changing routings enqueued back to back on one stream (every
    kernel after the metadata starts as a programmatic dependent of the one
    before it) give, bit for bit, the outputs of the same forwards run one at a
    time with stage events between the launches (which serialise them) and the
    host waiting after each."""
    inp = synthetic.make_inputs(name, device="cuda")
    wl = inp.wl
    routes = [synthetic.make_routing(wl, seed=wl.seed + 7 * i) for i in range(4)]
    idx = [torch.from_numpy(a).cuda() for a, _ in routes]
    wts = [torch.from_numpy(b).cuda() for _, b in routes]
    ws = binding.alloc_workspace(wl.N, wl.H, wl.I, wl.E, wl.K, -1)
    outs = [torch.empty(wl.N, wl.H, dtype=torch.bfloat16, device="cuda") for _ in routes]
    torch.cuda.synchronize()
    for i in range(len(routes)):
        binding.forward(inp.x, idx[i], wts[i], inp.w1, inp.w2, inp.b1, inp.b2, out=outs[i], ws=ws)
    torch.cuda.synchronize()
    assert binding.read_error(ws) == 0
    for i in range(len(routes)):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
        ref = binding.forward(inp.x, idx[i], wts[i], inp.w1, inp.w2, inp.b1, inp.b2, ws=ws, events=ev)
        torch.cuda.synchronize()
        assert binding.read_error(ws) == 0
        assert torch.equal(outs[i], ref), f"forward {i}"


@pytest.mark.parametrize("shift", [-100, -60, 60, 100])
@pytest.mark.parametrize("shape", ["grouped", "decode"])
def test_y_keeps_bf16_range(shift, shape):
    """w2 and b2 scaled by 2^shift (exact in bf16) scale y and the output by
    2^shift: the expert rows, stored as fp16 with a power-of-two exponent per
    32-column block, keep bf16's range at both ends, on the grouped-GEMM path
    and on the decode path, and the output stays within tolerance of the oracle
    run on the same scaled weights."""
    if shape == "grouped":
        wl = synthetic.custom(300, 256, 128, 8, 2, p_invalid=0.1, bias=True, seed=31)
    else:
        wl = synthetic.custom(48, 256, 128, 32, 4, p_invalid=0.1, bias=True, seed=32)
        assert wl.N * wl.K <= 32 * wl.E  # the sizes select the decode kernels
    inp = synthetic.make_inputs(wl, device="cuda")
    f = 2.0 ** shift
    inp.w2 = (inp.w2.float() * f).to(torch.bfloat16)
    inp.b2 = (inp.b2.float() * f).to(torch.bfloat16)
    assert torch.isfinite(inp.w2.float()).all() and (inp.w2 != 0).any()
    out, _ = run_case(inp)
    o = out.float()
    assert torch.isfinite(o).all()
    mag = o.abs()[o != 0].log2().median().item()
    assert abs(mag - shift) < 8, f"output magnitude 2^{mag:.1f} for weights scaled by 2^{shift}"
