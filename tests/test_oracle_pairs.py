"""Pins of the pair-list metadata oracle (oracle.metadata_pairs).

The compact pair list is the general routing input of sonic-moe issue #68
(token_indices / expert_indices / router_scores, one entry per (token,
expert) pair, ascending tokens); the non-expand table is the same routing
with the token implied by the row.  The pins: a hand-worked fixture, the
table oracle on the row-major flattening of a table (pinned on its own by
tests/test_oracle_pins.py), a direct Python construction from the
definitions on every small list, and the error counts.
"""
import itertools

import numpy as np
import pytest

import oracle
from mixture_experts_routed_non_b200 import synthetic
from test_oracle_pins import _load, _num

KEYS = ("freq", "off", "x_gather_idx", "s_scatter_idx", "s_reverse_scatter_idx", "token_offset")


def check_pair_fixture(lib=None):
    g = _load("metadata_pair_list_example.json")
    md = oracle.metadata_pairs(np.array(g["token_idx"]), np.array(g["expert_idx"]),
                               np.array([_num(v) for v in g["weights"]], np.float32), g["N"], g["E"],
                               lib_path=lib)
    ex = g["expected"]
    assert md["P"] == ex["P"]
    assert md["bad_tokens"] == ex["bad_tokens"] and md["bad_ids"] == 0 and not md["unsorted"]
    assert md["freq"].tolist() == ex["expert_frequency"]
    assert md["off"].tolist() == ex["expert_frequency_offset"]
    assert md["x_gather_idx"].tolist() == ex["x_gather_idx"]
    assert md["s_scatter_idx"].tolist() == ex["s_scatter_idx"]
    assert md["s_reverse_scatter_idx"].tolist() == ex["s_reverse_scatter_idx"]
    assert md["token_offset"].tolist() == ex["num_activated_expert_per_token_offset"]
    assert md["scores"].tolist() == ex["router_scores"]


def table_as_pair_list(idx, w):
    """Row-major flattening of an [N,K] table: entry s = (s // K, idx, w)."""
    N, K = idx.shape
    return np.repeat(np.arange(N, dtype=np.int64), K), idx.reshape(-1).astype(np.int64), w.reshape(-1)


def check_table_equivalence(idx, w, E, lib=None):
    ti, ei, wi = table_as_pair_list(idx, w)
    a = oracle.metadata(idx, w, E)                       # the table oracle (never the mutant)
    b = oracle.metadata_pairs(ti, ei, wi, idx.shape[0], E, lib_path=lib)
    assert a["P"] == b["P"] and a["bad_ids"] == b["bad_ids"] and b["bad_tokens"] == 0
    for k in KEYS:
        assert np.array_equal(a[k], b[k]), k
    assert np.array_equal(a["scores"].view(np.int32), b["scores"].view(np.int32))


def test_pair_list_worked_example():
    check_pair_fixture()


@pytest.mark.parametrize("name", ["tiny", "metadata", "decode256"])
def test_pair_list_of_table_matches_table_oracle(name):
    wl = synthetic.WORKLOADS[name]
    idx, w = synthetic.make_routing(wl, invalid_value=float("nan"))
    check_table_equivalence(idx, w, wl.E)


def _brute_pairs(tok, exp, N, E):
    kept = [(int(t), int(e)) for t, e in zip(tok, exp) if 0 <= e < E and 0 <= t < N]
    order = sorted(range(len(kept)), key=lambda q: (kept[q][1], q))
    freq = [sum(1 for _, e in kept if e == ee) for ee in range(E)]
    off = list(itertools.accumulate([0] + freq))
    rev = [0] * len(kept)
    for p, q in enumerate(order):
        rev[q] = p
    # pairs of token t: the kept entries naming t, which are contiguous in q
    to, q = [], 0
    for t in range(N + 1):
        to.append(q)
        q += sum(1 for tt, _ in kept if tt == t)
    return dict(freq=freq, off=off, x_gather_idx=[kept[q][0] for q in order], s_scatter_idx=order,
                s_reverse_scatter_idx=rev, token_offset=to)


@pytest.mark.parametrize("N,E,L", [(1, 1, 3), (3, 2, 3), (4, 2, 4), (2, 3, 3)])
def test_pair_list_brute_force(N, E, L):
    """Every ascending token list of length L over [0,N] (N itself out of
    range) with every expert assignment in {-1,0..E-1}."""
    w = np.arange(L, dtype=np.float32) + 0.5
    for tok in itertools.combinations_with_replacement(range(N + 1), L):
        for exp in itertools.product(range(-1, E), repeat=L):
            md = oracle.metadata_pairs(np.array(tok), np.array(exp), w, N, E)
            b = _brute_pairs(tok, exp, N, E)
            for k in KEYS:
                assert md[k].tolist() == b[k], (tok, exp, k)
            assert md["bad_tokens"] == sum(1 for t, e in zip(tok, exp) if 0 <= e < E and t >= N)
            assert not md["unsorted"]


def test_pair_list_errors_and_edges():
    w = np.ones(4, np.float32)
    md = oracle.metadata_pairs(np.array([0, 2, 1, 3]), np.array([0, 0, 0, 0]), w, 4, 1)
    assert md["unsorted"]
    md = oracle.metadata_pairs(np.array([-1, 0, 0, 1]), np.array([0, 5, -1, -7]), w, 2, 2)
    assert md["bad_tokens"] == 1 and md["bad_ids"] == 2 and md["P"] == 0
    assert md["token_offset"].tolist() == [0, 0, 0]
    md = oracle.metadata_pairs(np.zeros(0), np.zeros(0), np.zeros(0, np.float32), 3, 2)
    assert md["P"] == 0 and md["token_offset"].tolist() == [0, 0, 0, 0]
    big = np.array([0, 1, 2 ** 40, 2 ** 41], np.int64)          # int64 ids past the int32 range
    md = oracle.metadata_pairs(big, np.array([1, 0, 0, 2 ** 40]), w, 3, 2)
    assert md["P"] == 2 and md["bad_tokens"] == 1 and md["bad_ids"] == 1 and not md["unsorted"]
    assert md["token_offset"].tolist() == [0, 1, 2, 2]
