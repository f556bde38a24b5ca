"""GPU combine (moe_nonexpand_combine) against the oracle's combine."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_close, to_np
from mixture_experts_routed_non_b200 import binding

pytestmark = pytest.mark.gpu


def _case(N, K, E, H, p_invalid, seed):
    rng = np.random.default_rng(seed)
    idx = rng.integers(0, E, size=(N, K)).astype(np.int32)
    idx[rng.random((N, K)) < p_invalid] = -1
    w = rng.random((N, K)).astype(np.float32)
    ref_meta = oracle.metadata(idx, w, E)
    P = ref_meta["P"]
    y = torch.randn(max(P, 1), H, generator=torch.Generator().manual_seed(seed)).to(torch.bfloat16)
    return idx, w, ref_meta, y


@pytest.mark.parametrize("N,K,E,H,p_invalid,seed", [
    (1, 1, 1, 64, 0.0, 1), (257, 2, 8, 128, 0.1, 2), (1000, 8, 128, 2048, 0.0, 3),
    (333, 8, 32, 7168, 0.75, 4), (64, 32, 5, 192, 0.3, 5), (100, 4, 4, 64, 1.0, 6)])
def test_combine_matches_oracle(N, K, E, H, p_invalid, seed):
    idx, w, ref_meta, y = _case(N, K, E, H, p_invalid, seed)
    dev = torch.device("cuda")
    meta = binding.metadata(torch.from_numpy(idx).to(dev), torch.from_numpy(w).to(dev), E)
    yd = y.to(dev)
    out = binding.combine(yd, meta, N)
    ref = oracle.combine(ref_meta["token_offset"], ref_meta["s_reverse_scatter_idx"], ref_meta["scores"],
                         y.double().numpy()[:ref_meta["P"]])
    assert_close(to_np(out), ref, "combine")
    # tokens without a valid slot are exactly zero
    empty = np.nonzero((idx < 0).all(1))[0]
    assert np.all(to_np(out)[empty] == 0)
    # bitwise deterministic
    out2 = binding.combine(yd, meta, N)
    assert torch.equal(out, out2)
