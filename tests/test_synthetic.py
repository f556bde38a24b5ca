"""The seeded generators: reproducible and shaped like the workloads they name."""
import numpy as np
import pytest
import torch

from mixture_experts_routed_non_b200 import synthetic


@pytest.mark.parametrize("name", ["tiny", "metadata", "prefill", "ranklocal", "decode256", "prefill256"])
def test_routing_is_seeded_and_well_formed(name):
    wl = synthetic.WORKLOADS[name]
    a_idx, a_w = synthetic.make_routing(wl)
    b_idx, b_w = synthetic.make_routing(wl)
    assert np.array_equal(a_idx, b_idx) and np.array_equal(a_w, b_w)
    assert a_idx.shape == (wl.N, wl.K) and a_idx.dtype == np.int32
    assert a_w.dtype == np.float32
    assert a_idx.min() >= -1 and a_idx.max() < wl.E
    # valid experts are distinct within a row
    for row in a_idx[:512]:
        v = row[row >= 0]
        assert len(set(v.tolist())) == len(v)
    c_idx, _ = synthetic.make_routing(wl, seed=wl.seed + 100)
    assert not np.array_equal(a_idx, c_idx)


def test_invalid_fractions_and_scores():
    idx, w = synthetic.make_routing(synthetic.WORKLOADS["metadata"])
    frac = (idx < 0).mean()
    assert 0.04 < frac < 0.06
    valid = idx >= 0
    sums = np.where(valid, w, 0).sum(1)
    rows = valid.any(1)
    np.testing.assert_allclose(sums[rows], 1.0, rtol=1e-5)
    idx, w = synthetic.make_routing(synthetic.WORKLOADS["ranklocal"])
    m = (idx >= 0).sum(1)
    assert m.min() == 1 and m.max() == 4
    idx, w = synthetic.make_routing(synthetic.WORKLOADS["tiny"], invalid_value=float("nan"))
    assert np.all(np.isnan(w[idx < 0])) and np.all(np.isfinite(w[idx >= 0]))


def test_zipf_routing_is_skewed():
    idx, _ = synthetic.make_routing(synthetic.WORKLOADS["prefill256"])
    counts = np.bincount(idx[idx >= 0], minlength=256)
    assert counts.max() > 20 * np.median(counts)


def test_dense_tensors_seeded():
    a = synthetic.make_inputs("tiny", device="cpu")
    b = synthetic.make_inputs("tiny", device="cpu")
    for k in ("x", "w1", "b1", "w2", "b2"):
        assert torch.equal(getattr(a, k), getattr(b, k))
    assert a.w1.shape == (8, 128, 512) and a.w2.shape == (8, 256, 128)
    assert a.x.dtype == torch.bfloat16
    # std of w1 follows 1/sqrt(fan_in)
    assert abs(a.w1.float().std().item() - 128 ** -0.5) < 0.01
