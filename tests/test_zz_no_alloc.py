"""moe_nonexpand_metadata_noalloc against moe_nonexpand_metadata.

The no-allocation entry point serves callers that cannot allocate device
memory when they call in (a serving process with a memory pool frozen at
start-up, a plugin whose host framework owns every allocation), so they cannot
pass a workspace.  It must produce exactly the metadata of the workspace entry
point.  Metadata is integer and copied data, so the tolerance the other
metadata tests use applies: bit-exact.  Two calls in a row (different routing,
then the first again) show that the shared scratch's leftover contents from
the previous call do not leak into the next.

This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from mixture_experts_routed_non_b200 import binding, synthetic

pytestmark = pytest.mark.gpu

PAIR_ARRAYS = ("x_gather_idx", "s_scatter_idx", "s_reverse_scatter_idx", "scores")


def _noalloc_via_cabi(topk_idx, topk_w, E, total_pairs, meta):
    lib = binding.load()
    N, K = topk_idx.shape
    m = binding.MoeMeta(*[meta[f].data_ptr() for f, _ in binding.MoeMeta._fields_])
    stream = torch.cuda.current_stream().cuda_stream
    st = lib.moe_nonexpand_metadata_noalloc(topk_idx.data_ptr(), topk_w.data_ptr(), N, K, E, total_pairs,
                                            ctypes.byref(m), stream)
    assert st == binding.MOE_OK, binding.strerror(st)


def _compare(name, seed_offset=0, total_pairs_known=False):
    wl = synthetic.WORKLOADS[name]
    idx, w = synthetic.make_routing(wl, seed=wl.seed + seed_offset, invalid_value=float("nan"))
    dev = torch.device("cuda")
    ti = torch.from_numpy(idx).to(dev)
    tw = torch.from_numpy(w).to(dev)
    P = int((idx >= 0).sum())
    tp = P if total_pairs_known else -1
    ref = binding.metadata(ti, tw, wl.E, total_pairs=tp)            # workspace entry point
    got = binding.alloc_meta(wl.N, wl.K, wl.E, tp, dev)
    for v in got.values():
        v.fill_(-7)  # anything the call fails to write shows up
    _noalloc_via_cabi(ti, tw, wl.E, tp, got)
    torch.cuda.synchronize()
    for k in ref:
        a, b = ref[k], got[k]
        if k in PAIR_ARRAYS:
            a, b = a[:P], b[:P]
        assert torch.equal(a.view(torch.int32), b.view(torch.int32)), k


def test_noalloc_matches_workspace_entry_point_twice_in_a_row():
    _compare("metadata")                   # 65536 x 8, Zipf, 5 % invalid
    _compare("tiny", total_pairs_known=True)
    _compare("metadata", seed_offset=7)    # same sizes, new routing, after a smaller call


def test_noalloc_repeat_same_input_bitwise():
    _compare("prefill256")
    _compare("prefill256")


def test_noalloc_reports_device_errors_and_clears_them():
    """The scratch's error word: a bad expert id and a total_pairs below the
    real pair count are reported through
    moe_nonexpand_metadata_noalloc_read_error; the next good call rewrites the
    word whole, so no bit of an earlier call is reported again."""
    import oracle
    from helpers import check_meta_equal

    wl = synthetic.WORKLOADS["tiny"]
    idx, w = synthetic.make_routing(wl, seed=wl.seed, invalid_value=float("nan"))
    dev = torch.device("cuda")
    P = int((idx >= 0).sum())

    bad = idx.copy()
    bad[3, 0] = 99                     # neither a valid id nor -1: flagged and skipped like -1
    meta = binding.alloc_meta(wl.N, wl.K, wl.E, -1, dev)
    binding.metadata_noalloc(torch.from_numpy(bad).to(dev), torch.from_numpy(w).to(dev), wl.E, meta)
    assert binding.metadata_noalloc_read_error() == binding.DEVERR_BAD_EXPERT_ID
    check_meta_equal(meta, oracle.metadata(bad, w, wl.E))

    short = binding.alloc_meta(wl.N, wl.K, wl.E, P - 1, dev)
    binding.metadata_noalloc(torch.from_numpy(idx).to(dev), torch.from_numpy(w).to(dev), wl.E, short,
                             total_pairs=P - 1)
    err = binding.metadata_noalloc_read_error()
    assert err == binding.DEVERR_PAIR_COUNT | binding.DEVERR_ABORTED, hex(err)

    good = binding.alloc_meta(wl.N, wl.K, wl.E, P, dev)
    binding.metadata_noalloc(torch.from_numpy(idx).to(dev), torch.from_numpy(w).to(dev), wl.E, good,
                             total_pairs=P)
    assert binding.metadata_noalloc_read_error() == 0
    check_meta_equal(good, oracle.metadata(idx, w, wl.E))


def test_noalloc_bit_exact_against_the_oracle_at_full_size():
    import oracle
    from helpers import check_meta_equal

    wl = synthetic.WORKLOADS["metadata"]   # 65536 x 8, Zipf, 5 % invalid
    idx, w = synthetic.make_routing(wl, seed=wl.seed + 3)
    dev = torch.device("cuda")
    meta = binding.alloc_meta(wl.N, wl.K, wl.E, -1, dev)
    binding.metadata_noalloc(torch.from_numpy(idx).to(dev), torch.from_numpy(w).to(dev), wl.E, meta)
    assert binding.metadata_noalloc_read_error() == 0
    check_meta_equal(meta, oracle.metadata(idx, w, wl.E))
