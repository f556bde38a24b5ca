"""Router top-k (moe_router_topk) on the GPU against the oracle.

The chosen experts are an integer decision taken on the logits as given, on
both sides, so topk_idx must match bit for bit.  The weights: the kernels use
fp32 expf for the chosen logits (a few ulp), the fast exponential for the
full softmax's sum (relative error a few 1e-6 per term) and fixed-order sums
of at most 1024 positive terms, so their relative error stays near 5e-6; the
test allows RTOL = 1e-5 against the float64 oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_close, check_meta_equal, to_np
from mixture_experts_routed_non_b200 import binding, synthetic

pytestmark = pytest.mark.gpu

RTOL = 1e-5
ATOL = 1e-7
MODES = (binding.ROUTER_SOFTMAX_TOPK, binding.ROUTER_TOPK_SOFTMAX, binding.ROUTER_TOPK_SOFTMAX_RENORM)


def _check(logits, K, mode):
    idx, w = binding.router_topk(logits, K, mode)
    torch.cuda.synchronize()
    ri, rw = oracle.router_topk(logits, K, mode)
    np.testing.assert_array_equal(to_np(idx), ri)
    np.testing.assert_allclose(to_np(w), rw, rtol=RTOL, atol=ATOL, equal_nan=True)


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("N,E,K", [(16384, 128, 8), (2048, 256, 8), (777, 1024, 32), (301, 33, 1),
                                   (5, 3, 3), (64, 1000, 17), (1, 1, 1)])
def test_router_matches_oracle(N, E, K, dtype, mode):
    _check(synthetic.make_logits(N, E, seed=N + E + K, dtype=dtype, device="cuda"), K, mode)


@pytest.mark.parametrize("mode", MODES)
def test_router_ties_go_to_lower_ids(mode):
    _check(synthetic.make_logits(4096, 64, seed=3, kind="ties", device="cuda"), 8, mode)
    _check(synthetic.make_logits(100, 512, seed=4, kind="ties", dtype=torch.bfloat16, device="cuda"), 32, mode)


def test_router_nan_and_inf():
    lg = synthetic.make_logits(64, 40, seed=9, device="cuda")
    lg[0, :] = float("-inf")                        # all -inf: weights NaN, ids 0..K-1
    lg[1, 5] = float("nan")
    lg[2, :35] = float("-inf")
    lg[3, 7] = float("inf")
    lg[4, ::3] = float("nan")
    for mode in MODES:
        _check(lg, 6, mode)


def test_router_empty_and_bad_arguments():
    e = torch.empty((0, 16), device="cuda")
    idx, w = binding.router_topk(e, 4)
    assert idx.shape == (0, 4)
    lg = torch.zeros((4, 16), device="cuda")
    for K in (0, 17, 33):
        with pytest.raises(binding.MoeError):
            binding.router_topk(lg, K)
    with pytest.raises(binding.MoeError):
        binding.router_topk(lg, 2, mode=3)


def test_router_feeds_the_forward():
    """Logits -> router -> forward on the tiny workload's sizes; the oracle
    takes its own router output, so the two paths meet only at the output."""
    wl = synthetic.WORKLOADS["tiny"]
    inp = synthetic.make_inputs("tiny", device="cuda")
    logits = synthetic.make_logits(wl.N, wl.E, seed=21, device="cuda")
    idx, w = binding.router_topk(logits, wl.K, binding.ROUTER_TOPK_SOFTMAX_RENORM)
    ws = binding.alloc_workspace(wl.N, wl.H, wl.I, wl.E, wl.K)
    out = binding.forward(inp.x, idx, w, inp.w1, inp.w2, inp.b1, inp.b2, ws=ws)
    torch.cuda.synchronize()
    ri, rw = oracle.router_topk(logits, wl.K, oracle.ROUTER_TOPK_SOFTMAX_RENORM)
    np.testing.assert_array_equal(to_np(idx), ri)
    check_meta_equal(binding.meta_from_workspace(ws, wl.N, wl.H, wl.I, wl.E, wl.K),
                     oracle.metadata(ri, to_np(w), wl.E))
    wts = oracle.Weights(inp.x, inp.w1, inp.b1, inp.w2, inp.b2)
    ref = oracle.forward_rows(wts, ri, rw.astype(np.float32))
    assert_close(to_np(out), ref, "out (router -> forward)")


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("E", [32, 64, 128, 256])
@pytest.mark.parametrize("K", [1, 3, 8])
def test_router_common_shapes(E, K, dtype, mode):
    """Expert counts of the common MoE shapes with K <= 8, N not a multiple of
    the tokens a block handles."""
    _check(synthetic.make_logits(1003, E, seed=E * 10 + K, dtype=dtype, device="cuda"), K, mode)


@pytest.mark.parametrize("mode", MODES)
def test_router_ties_nan_inf_at_128_and_256(mode):
    _check(synthetic.make_logits(2051, 128, seed=5, kind="ties", device="cuda"), 8, mode)
    _check(synthetic.make_logits(515, 256, seed=6, kind="ties", dtype=torch.bfloat16, device="cuda"), 6, mode)
    lg = synthetic.make_logits(40, 128, seed=7, device="cuda")
    lg[0, :] = float("-inf")
    lg[1, 5] = float("nan")
    lg[2, :120] = float("-inf")   # fewer finite logits than K
    lg[3, 77] = float("inf")
    lg[4, ::3] = float("nan")
    lg[5, :] = 1.0                # every logit equal: ids 0..K-1
    lg[6, 96:] = 3.0              # the largest all in the last lane
    _check(lg, 8, mode)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("E", [128, 1000])
def test_router_negative_zero_ties_with_zero(E, dtype):
    """-0.0 and +0.0 are equal logits: the lower id goes first."""
    lg = torch.full((64, E), -1.0, device="cuda")
    lg[:, 3] = -0.0
    lg[:, 1] = 0.0
    lg[:, 7] = -0.0
    lg[1::2, 0] = -0.0
    for mode in MODES:
        _check(lg.to(dtype), 4, mode)


@pytest.mark.parametrize("mode", MODES)
def test_router_near_ties_in_the_low_bits(mode):
    """fp32 logits a few ulp apart, so that keys sharing their high bits
    decide the result (the exact retry)."""
    g = np.random.default_rng(11)
    base = np.float32(1.25)
    a = base + g.integers(-300, 300, size=(999, 128)).astype(np.float32) * np.spacing(base)
    _check(torch.from_numpy(a.astype(np.float32)).cuda(), 8, mode)
    _check(torch.from_numpy(a[:, :96].copy().astype(np.float32)).cuda(), 5, mode)


@pytest.mark.parametrize("mode", MODES)
def test_router_outputs_4_byte_aligned(mode):
    """Output arrays 4 bytes past an 8-byte boundary (K = 8: the kernel's paired
    stores fall back to single ones)."""
    lg = synthetic.make_logits(333, 128, seed=12, device="cuda")
    ib = torch.empty(333 * 8 + 1, dtype=torch.int32, device="cuda")
    wb = torch.empty(333 * 8 + 1, dtype=torch.float32, device="cuda")
    idx, w = ib[1:].view(333, 8), wb[1:].view(333, 8)
    assert idx.data_ptr() % 8 == 4 and w.data_ptr() % 8 == 4
    binding.router_topk(lg, 8, mode, idx, w)
    torch.cuda.synchronize()
    ri, rw = oracle.router_topk(lg, 8, mode)
    np.testing.assert_array_equal(to_np(idx), ri)
    np.testing.assert_allclose(to_np(w), rw, rtol=RTOL, atol=ATOL, equal_nan=True)


def test_router_logits_not_16_byte_aligned():
    """Logits 4 bytes past a 16-byte boundary (a slice) give the same results."""
    big = synthetic.make_logits(301 * 128 + 1, 1, seed=8, device="cuda").reshape(-1)
    lg = big[1:].view(301, 128)
    assert lg.data_ptr() % 16 == 4
    for mode in MODES:
        _check(lg, 8, mode)
