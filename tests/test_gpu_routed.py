"""The routed entry points (moe_nonexpand_routed_*) on the GPU.

Routing arrives either as the non-expand table or as the compact pair list of
sonic-moe issue #68's general routing API (token_indices / expert_indices /
router_scores, ascending tokens), with int32 or int64 ids.  Metadata is
compared bit-exactly with the pair-list oracle; the forward output within the
forward tolerance with the oracle's rows, and bit-exactly with the table
entry point on the same pairs in the same order (same arithmetic).
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_close, check_meta_equal, to_np
from mixture_experts_routed_non_b200 import binding, synthetic

pytestmark = pytest.mark.gpu

DT = {32: torch.int32, 64: torch.int64}


def _dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    return (t.to(dtype) if dtype is not None else t).cuda()


def _routed_meta(tok, exp, w, N, E, bits):
    ws = torch.empty(binding.routed_workspace_bytes(
        binding.routing(_dev(exp, DT[bits]), _dev(w), token_idx=_dev(tok, DT[bits]), N=N), 0, 0, E),
        dtype=torch.uint8, device="cuda")
    meta = binding.routed_metadata(_dev(exp, DT[bits]), _dev(w), E, token_idx=_dev(tok, DT[bits]), N=N, ws=ws)
    torch.cuda.synchronize()
    return meta, binding.read_error(ws)


@pytest.mark.parametrize("bits", [32, 64])
@pytest.mark.parametrize("name", ["tiny", "metadata", "prefill"])
def test_pair_list_metadata_matches_oracle(name, bits):
    wl = synthetic.WORKLOADS[name]
    idx, w = synthetic.make_routing(wl, invalid_value=float("nan"))
    rng = np.random.default_rng(wl.seed + 5)
    empty = rng.choice(wl.N, size=max(1, wl.N // 50), replace=False)
    tok, exp, wt = synthetic.pair_list_from_table(idx, w, empty_tokens=empty)
    ref = oracle.metadata_pairs(tok, exp, wt, wl.N, wl.E)
    meta, err = _routed_meta(tok, exp, wt, wl.N, wl.E, bits)
    assert err == 0
    check_meta_equal(meta, ref)


@pytest.mark.parametrize("bits", [32, 64])
def test_pair_list_keeping_invalid_entries_and_bad_ids(bits):
    wl = synthetic.WORKLOADS["metadata"]
    idx, w = synthetic.make_routing(wl, invalid_value=float("nan"))
    tok, exp, wt = synthetic.pair_list_from_table(idx, w, keep_invalid=True)
    exp = exp.copy()
    exp[7] = wl.E + 3              # a bad expert id
    exp[1000] = -(2 ** 33) if bits == 64 else -5
    tok = tok.copy()
    tok[-3:] = wl.N + (2 ** 35 if bits == 64 else 1)   # bad tokens at the tail, still ascending
    exp[-3:] = 0
    ref = oracle.metadata_pairs(tok, exp, wt, wl.N, wl.E)
    assert ref["bad_ids"] == 2 and ref["bad_tokens"] == 3 and not ref["unsorted"]
    meta, err = _routed_meta(tok, exp, wt, wl.N, wl.E, bits)
    assert err == binding.DEVERR_BAD_EXPERT_ID | binding.DEVERR_BAD_TOKEN
    check_meta_equal(meta, ref)


def test_unsorted_pair_list_is_flagged_and_sorts_the_pairs():
    """Tokens out of order: the error bit is set; the pair arrays still follow
    the list order (token_offset is then unspecified and not compared)."""
    wl = synthetic.WORKLOADS["tiny"]
    idx, w = synthetic.make_routing(wl)
    tok, exp, wt = synthetic.pair_list_from_table(idx, w)
    tok = tok.copy()
    tok[[3, 40]] = tok[[40, 3]]
    ref = oracle.metadata_pairs(tok, exp, wt, wl.N, wl.E)
    assert ref["unsorted"]
    meta, err = _routed_meta(tok, exp, wt, wl.N, wl.E, 32)
    assert err & binding.DEVERR_BAD_TOKEN
    P = ref["P"]
    for k in ("x_gather_idx", "s_scatter_idx", "s_reverse_scatter_idx"):
        np.testing.assert_array_equal(to_np(meta[k])[:P], ref[k], err_msg=k)
    np.testing.assert_array_equal(to_np(meta["expert_frequency_offset"]), ref["off"])
    to = to_np(meta["token_offset"])
    assert to.min() >= 0 and to.max() <= P


@pytest.mark.parametrize("N", [0, 5])
def test_empty_pair_list(N):
    e = np.zeros(0, np.int64)
    meta, err = _routed_meta(e, e, np.zeros(0, np.float32), N, 4, 32)
    assert err == 0
    assert to_np(meta["token_offset"]).tolist() == [0] * (N + 1)
    assert to_np(meta["expert_frequency_offset"]).tolist() == [0] * 5


@pytest.mark.parametrize("name", ["metadata", "decode256"])
def test_int64_table_matches_int32_table(name):
    wl = synthetic.WORKLOADS[name]
    idx, w = synthetic.make_routing(wl)
    a = binding.metadata(_dev(idx), _dev(w), wl.E)
    b = binding.routed_metadata(_dev(idx, torch.int64), _dev(w), wl.E)
    torch.cuda.synchronize()
    ref = oracle.metadata(idx, w, wl.E)
    check_meta_equal(a, ref)
    check_meta_equal(b, ref)


@pytest.mark.parametrize("bits", [32, 64])
def test_pair_list_forward_equals_table_forward_bitwise(bits):
    """The pair list of a table (invalid slots dropped) gives the same pairs
    in the same order, so every stage does the same arithmetic."""
    inp = synthetic.make_inputs("tiny", device="cuda")
    idx, w = inp.topk_idx.cpu().numpy(), inp.topk_w.cpu().numpy()
    tok, exp, wt = synthetic.pair_list_from_table(idx, w)
    a = binding.forward(inp.x, inp.topk_idx, inp.topk_w, inp.w1, inp.w2, inp.b1, inp.b2)
    b = binding.routed_forward(inp.x, _dev(exp, DT[bits]), _dev(wt), inp.w1, inp.w2, inp.b1, inp.b2,
                               token_idx=_dev(tok, DT[bits]))
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def _pair_forward_ref(inp, tok, exp, wt, tokens, layout=0):
    """out rows of the given tokens (float64): each token's kept entries, in
    list order, score x expert row (oracle rows)."""
    N, E = inp.wl.N, inp.wl.E
    keep = (exp >= 0) & (exp < E) & (tok >= 0) & (tok < N)
    tok, exp, wt = tok[keep], exp[keep], wt[keep]
    sel = np.isin(tok, tokens)
    wts = oracle.Weights(inp.x, inp.w1, inp.b1, inp.w2, inp.b2)
    _, y = oracle.pair_rows(wts, tok[sel], exp[sel], layout=layout)
    out = np.zeros((len(tokens), wts.H), np.float64)
    row = {int(t): i for i, t in enumerate(tokens)}
    for q, t in enumerate(tok[sel]):
        out[row[int(t)]] += float(wt[sel][q]) * y[q]
    return out


@pytest.mark.parametrize("bits", [32, 64])
def test_pair_list_forward_with_heavy_tokens(bits):
    """Tokens routed to every expert: blocks of the combine see more pairs than
    its shared-memory staging holds; other tokens have K pairs or none."""
    wl = synthetic.custom(N=300, H=256, I=192, E=300, K=4, bias=True, seed=11, name="heavy")
    inp = synthetic.make_inputs(wl, device="cuda")
    rng = np.random.default_rng(3)
    heavy = np.array([0, 1, 2, 3, 9, 150, 151, 299])
    tok, exp, wt = synthetic.many_pair_tokens(wl.N, wl.E, heavy, wl.K, rng)
    keep = ~np.isin(tok, [20, 21, 22, 200])          # tokens without pairs
    tok, exp, wt = tok[keep], exp[keep], wt[keep]
    meta = binding.alloc_routed_meta(binding.routing(_dev(exp, DT[bits]), _dev(wt), token_idx=_dev(tok, DT[bits]),
                                                     N=wl.N), wl.E)
    out = binding.routed_forward(inp.x, _dev(exp, DT[bits]), _dev(wt), inp.w1, inp.w2, inp.b1, inp.b2,
                                 token_idx=_dev(tok, DT[bits]), meta=meta)
    torch.cuda.synchronize()
    check_meta_equal(meta, oracle.metadata_pairs(tok, exp, wt, wl.N, wl.E))
    # the bound's rms term is taken over rows of one kind: a heavy row sums 300
    # terms, so its rounding error and its size both grow by ~sqrt(300/4)
    ref = _pair_forward_ref(inp, tok, exp, wt, np.arange(wl.N))
    got = to_np(out)
    is_heavy = np.isin(np.arange(wl.N), heavy)
    assert_close(got[is_heavy], ref[is_heavy], "out (heavy rows of the pair list)")
    assert_close(got[~is_heavy], ref[~is_heavy], "out (other rows of the pair list)")


def test_pair_list_forward_prefill_sample():
    """The prefill workload as a pair list with tokens dropped, in the
    launch configuration of the table path; sampled rows against the oracle."""
    inp = synthetic.make_inputs("prefill", device="cuda")
    wl = inp.wl
    idx, w = inp.topk_idx.cpu().numpy(), inp.topk_w.cpu().numpy()
    rng = np.random.default_rng(17)
    empty = rng.choice(wl.N, size=wl.N // 20, replace=False)
    tok, exp, wt = synthetic.pair_list_from_table(idx, w, empty_tokens=empty)
    out = binding.routed_forward(inp.x, _dev(exp, torch.int64), _dev(wt), inp.w1, inp.w2, inp.b1, inp.b2,
                                 token_idx=_dev(tok, torch.int64))
    torch.cuda.synchronize()
    tokens = np.sort(np.concatenate([rng.choice(wl.N, size=48, replace=False), empty[:8]]))
    assert_close(to_np(out)[tokens], _pair_forward_ref(inp, tok, exp, wt, tokens), "out (prefill pair list)")
    assert not to_np(out)[empty].any()
