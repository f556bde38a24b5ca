"""GPU metadata (moe_nonexpand_metadata) against the oracle: bit-exact."""
import numpy as np
import pytest
import torch

import oracle
from helpers import check_meta_equal, to_np
from mixture_experts_routed_non_b200 import binding, synthetic

pytestmark = pytest.mark.gpu


def run_meta(idx: np.ndarray, w: np.ndarray, E: int, total_pairs: int = -1):
    dev = torch.device("cuda")
    ti = torch.from_numpy(np.ascontiguousarray(idx, np.int32)).to(dev)
    tw = torch.from_numpy(np.ascontiguousarray(w, np.float32)).to(dev)
    ws = binding.alloc_workspace(idx.shape[0], 0, 0, E, idx.shape[1], total_pairs, dev)
    meta = binding.metadata(ti, tw, E, total_pairs=total_pairs, ws=ws)
    err = binding.read_error(ws)
    return meta, err, ws


@pytest.mark.parametrize("name", ["tiny", "metadata", "prefill", "ranklocal", "decode256", "prefill256"])
def test_metadata_workloads_bit_exact(name):
    wl = synthetic.WORKLOADS[name]
    idx, w = synthetic.make_routing(wl, invalid_value=float("nan"))
    ref = oracle.metadata(idx, w, wl.E)
    meta, err, _ = run_meta(idx, w, wl.E)
    assert err == 0
    check_meta_equal(meta, ref)
    # with the pair count given, as a dispatch handle would
    meta, err, _ = run_meta(idx, w, wl.E, total_pairs=ref["P"])
    assert err == 0
    check_meta_equal(meta, ref)


@pytest.mark.parametrize("N,K,E,p_invalid,seed", [
    (1, 1, 1, 0.0, 1), (3, 2, 3, 0.3, 2), (37, 3, 5, 0.2, 3), (511, 1, 7, 0.0, 4),
    (513, 8, 64, 0.1, 5), (4097, 5, 1024, 0.05, 6), (1000, 32, 40, 0.5, 7), (2500, 7, 1, 0.3, 8),
    (9999, 6, 300, 0.0, 9), (200003, 4, 17, 0.01, 10),
    # tiles of more than 4096 slots, ranked and written in several passes
    (70000, 8, 1024, 0.1, 11), (300001, 3, 513, 0.02, 12)])
def test_metadata_ragged_sizes_bit_exact(N, K, E, p_invalid, seed):
    rng = np.random.default_rng(seed)
    idx = rng.integers(0, E, size=(N, K)).astype(np.int32)   # duplicates within a row allowed
    idx[rng.random((N, K)) < p_invalid] = -1
    w = rng.random((N, K)).astype(np.float32)
    w[idx < 0] = np.nan
    ref = oracle.metadata(idx, w, E)
    meta, err, _ = run_meta(idx, w, E)
    assert err == 0
    check_meta_equal(meta, ref)


def test_metadata_all_invalid_and_empty():
    idx = np.full((300, 4), -1, np.int32)
    w = np.full((300, 4), np.nan, np.float32)
    meta, err, _ = run_meta(idx, w, 8)
    assert err == 0
    check_meta_equal(meta, oracle.metadata(idx, w, 8))
    idx = np.zeros((0, 4), np.int32)
    meta, err, _ = run_meta(idx, np.zeros((0, 4), np.float32), 8)
    assert err == 0
    assert to_np(meta["token_offset"]).tolist() == [0]
    assert to_np(meta["expert_frequency_offset"]).tolist() == [0] * 9


def test_metadata_one_expert_takes_everything():
    idx = np.zeros((5000, 3), np.int32)
    idx[:, 1] = 2
    w = np.ones((5000, 3), np.float32)
    ref = oracle.metadata(idx, w, 4)
    meta, err, _ = run_meta(idx, w, 4)
    assert err == 0
    check_meta_equal(meta, ref)


def test_metadata_bad_ids_flagged_and_skipped():
    rng = np.random.default_rng(3)
    idx = rng.integers(-1, 6, size=(700, 4)).astype(np.int32)
    idx[5, 2] = 9
    idx[600, 0] = -7
    w = rng.random((700, 4)).astype(np.float32)
    ref = oracle.metadata(idx, w, 6)
    assert ref["bad_ids"] == 2
    meta, err, _ = run_meta(idx, w, 6)
    assert err & binding.DEVERR_BAD_EXPERT_ID
    check_meta_equal(meta, ref)


def test_metadata_pair_count_mismatch_flagged():
    rng = np.random.default_rng(4)
    idx = rng.integers(-1, 6, size=(300, 4)).astype(np.int32)
    w = rng.random((300, 4)).astype(np.float32)
    P = int((idx >= 0).sum())
    # declared larger than the real count: flagged, results still right
    meta, err, _ = run_meta(idx, w, 6, total_pairs=P + 5)
    assert err == binding.DEVERR_PAIR_COUNT
    check_meta_equal(meta, oracle.metadata(idx, w, 6))
    # declared smaller: flagged and the later steps are skipped (no overflow)
    meta, err, _ = run_meta(idx, w, 6, total_pairs=P - 1)
    assert err == binding.DEVERR_PAIR_COUNT | binding.DEVERR_ABORTED


def test_error_word_is_rewritten_by_every_call():
    """A call's error bits do not outlive it: after a call with a bad id, the
    next good call on the same workspace reports 0."""
    rng = np.random.default_rng(5)
    idx = rng.integers(0, 6, size=(500, 4)).astype(np.int32)
    w = rng.random((500, 4)).astype(np.float32)
    dev = torch.device("cuda")
    ws = binding.alloc_workspace(500, 0, 0, 6, 4, -1, dev)
    bad = idx.copy()
    bad[7, 1] = 42
    binding.metadata(torch.from_numpy(bad).to(dev), torch.from_numpy(w).to(dev), 6, ws=ws)
    assert binding.read_error(ws) == binding.DEVERR_BAD_EXPERT_ID
    meta = binding.metadata(torch.from_numpy(idx).to(dev), torch.from_numpy(w).to(dev), 6, ws=ws)
    assert binding.read_error(ws) == 0
    check_meta_equal(meta, oracle.metadata(idx, w, 6))


def test_metadata_deterministic_and_workspace_reusable():
    wl = synthetic.WORKLOADS["metadata"]
    idx, w = synthetic.make_routing(wl)
    dev = torch.device("cuda")
    ti = torch.from_numpy(idx).to(dev)
    tw = torch.from_numpy(w).to(dev)
    ws = binding.alloc_workspace(wl.N, 0, 0, wl.E, wl.K, -1, dev)
    m1 = binding.metadata(ti, tw, wl.E, ws=ws)
    P = int((idx >= 0).sum())
    pair_arrays = ("x_gather_idx", "s_scatter_idx", "s_reverse_scatter_idx", "scores")
    snap = {k: (v[:P] if k in pair_arrays else v).clone() for k, v in m1.items()}
    for _ in range(3):
        m2 = binding.metadata(ti, tw, wl.E, ws=ws)
        for k in snap:
            got = m2[k][:P] if k in pair_arrays else m2[k]
            assert torch.equal(snap[k], got), k
    assert binding.read_error(ws) == 0
