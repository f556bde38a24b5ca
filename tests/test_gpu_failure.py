"""Failure detection on the GPU without a fault: a bounded pipeline wait that
nothing completes gives up, reports MOE_DEVERR_TIMEOUT through the error word,
and leaves the context usable.  Plus: the forward is free of host syncs, so
it can be captured in a CUDA graph and replayed."""
import time

import numpy as np
import pytest
import torch

import oracle
from helpers import assert_close, to_np
from mixture_experts_routed_non_b200 import binding, synthetic

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_reports():
    ws = binding.alloc_workspace(16, 0, 0, 4, 2)
    t0 = time.perf_counter()
    binding.selftest_wait_timeout(ws, 20000)  # 20 ms
    err = binding.read_error(ws)
    dt = time.perf_counter() - t0
    assert err == binding.DEVERR_TIMEOUT
    assert 0.015 < dt < 2.0
    # the context still works: a forward afterwards matches the oracle
    inp = synthetic.make_inputs("tiny", device="cuda")
    ws2 = binding.alloc_workspace(256, 128, 256, 8, 2)
    out = binding.forward(inp.x, inp.topk_idx, inp.topk_w, inp.w1, inp.w2, inp.b1, inp.b2, ws=ws2)
    assert binding.read_error(ws2) == 0
    wts = oracle.Weights(inp.x, inp.w1, inp.b1, inp.w2, inp.b2)
    ref = oracle.forward_rows(wts, inp.topk_idx.cpu().numpy(), inp.topk_w.cpu().numpy())
    assert_close(to_np(out), ref, "forward after a timed-out wait")


def test_selftest_rejects_bad_arguments():
    ws = binding.alloc_workspace(16, 0, 0, 4, 2)
    with pytest.raises(binding.MoeError):
        binding.selftest_wait_timeout(ws, 0)
    with pytest.raises(binding.MoeError):
        binding.selftest_wait_timeout(ws, 3_000_000)


@pytest.mark.parametrize("name", ["tiny", "prefill", "decode256"])
def test_forward_captures_in_cuda_graph(name):
    inp = synthetic.make_inputs(name, device="cuda")
    wl = inp.wl
    ws = binding.alloc_workspace(wl.N, wl.H, wl.I, wl.E, wl.K, -1)
    out = torch.empty(wl.N, wl.H, dtype=torch.bfloat16, device="cuda")
    eager = binding.forward(inp.x, inp.topk_idx, inp.topk_w, inp.w1, inp.w2, inp.b1, inp.b2, ws=ws).clone()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        binding.forward(inp.x, inp.topk_idx, inp.topk_w, inp.w1, inp.w2, inp.b1, inp.b2, out=out, ws=ws, stream=s)
        with torch.cuda.graph(g, stream=s):
            binding.forward(inp.x, inp.topk_idx, inp.topk_w, inp.w1, inp.w2, inp.b1, inp.b2, out=out, ws=ws,
                            stream=s)
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, eager)
    # new routing written into the same input buffers is picked up on replay
    idx2, w2 = synthetic.make_routing(wl, seed=wl.seed + 99)
    inp.topk_idx.copy_(torch.from_numpy(idx2))
    inp.topk_w.copy_(torch.from_numpy(w2))
    g.replay()
    ref = binding.forward(inp.x, inp.topk_idx, inp.topk_w, inp.w1, inp.w2, inp.b1, inp.b2)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
