"""Pins of the router top-k oracle (oracle.router_topk).

The two conventions of the sonic-moe write-up ("Three routing strategies,
selected on the command line"): TC top-K (softmax over the top-k logits) and
Qwen3-style (top-k of the softmax over all experts, optionally renormalised).
Pinned by hand-worked closed forms, torch.topk / torch.softmax in float64 on
distinct logits, a direct Python sort on every small row, and invariants.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from test_oracle_pins import _load

MODES = (oracle.ROUTER_SOFTMAX_TOPK, oracle.ROUTER_TOPK_SOFTMAX, oracle.ROUTER_TOPK_SOFTMAX_RENORM)
ENV = {"log": math.log, "exp": math.exp, "e": math.e, "inf": math.inf, "nan": math.nan}


def _ev(rows):
    return np.array([[float(eval(v, ENV)) for v in r] for r in rows], np.float64)


def check_router_fixture(lib=None):
    for case in _load("router_worked_example.json")["cases"]:
        lg = _ev(case["logits"])
        for m in MODES:
            idx, w = oracle.router_topk(lg, case["K"], m, lib_path=lib)
            assert idx.tolist() == case["topk_idx"], (case["derivation"], m)
            np.testing.assert_allclose(w, _ev(case["w"][str(m)]), rtol=1e-12, atol=1e-15)


def _torch_reference(lg, K, mode):
    t = torch.from_numpy(lg)
    vals, idx = torch.topk(t, K, dim=1, sorted=True)
    if mode == oracle.ROUTER_SOFTMAX_TOPK:
        w = torch.softmax(vals, dim=1)
    else:
        w = torch.softmax(t, dim=1).gather(1, idx)
        if mode == oracle.ROUTER_TOPK_SOFTMAX_RENORM:
            w = w / w.sum(dim=1, keepdim=True)
    return idx.numpy().astype(np.int32), w.numpy()


def check_router_against_torch(lib=None, seed=0):
    rng = np.random.default_rng(seed)
    for E, K in ((64, 8), (128, 8), (7, 3), (256, 1)):
        lg = rng.permutation(200 * E).reshape(200, E).astype(np.float64) / (7.0 * E)  # distinct
        for m in MODES:
            idx, w = oracle.router_topk(lg, K, m, lib_path=lib)
            ri, rw = _torch_reference(lg, K, m)
            assert np.array_equal(idx, ri), (E, K, m)
            np.testing.assert_allclose(w, rw, rtol=1e-12, atol=1e-15)


def test_router_worked_example():
    check_router_fixture()


def test_router_against_torch_topk_softmax():
    check_router_against_torch()


@pytest.mark.parametrize("E", [1, 2, 3, 4])
def test_router_brute_force_small_rows(E):
    """Every row over {-1, 0, 1}^E (many ties) and every K: the chosen list is
    a Python sort by (larger logit, lower id)."""
    for row in itertools.product((-1.0, 0.0, 1.0), repeat=E):
        lg = np.array([row])
        order = sorted(range(E), key=lambda e: (-row[e], e))
        for K in range(1, E + 1):
            for m in MODES:
                idx, w = oracle.router_topk(lg, K, m)
                assert idx[0].tolist() == order[:K]
                if m != oracle.ROUTER_TOPK_SOFTMAX:
                    assert abs(w.sum() - 1.0) < 1e-12
                else:
                    full = np.exp(np.array(row) - max(row))
                    np.testing.assert_allclose(w[0], full[order[:K]] / full.sum(), rtol=1e-12)


def test_router_invariants():
    rng = np.random.default_rng(5)
    lg = rng.standard_normal((100, 96))
    for m in MODES:
        idx, w = oracle.router_topk(lg, 6, m)
        idx2, w2 = oracle.router_topk(lg + 3.25, 6, m)           # shift invariance
        assert np.array_equal(idx, idx2)
        np.testing.assert_allclose(w, w2, rtol=1e-12)
        assert np.all(np.diff(w, axis=1) <= 0)                   # largest first
        assert np.all(np.take_along_axis(lg, idx.astype(np.int64), 1)[:, :1] == lg.max(1, keepdims=True))
    _, w0 = oracle.router_topk(lg, 6, oracle.ROUTER_SOFTMAX_TOPK)
    _, w2 = oracle.router_topk(lg, 6, oracle.ROUTER_TOPK_SOFTMAX_RENORM)
    np.testing.assert_allclose(w0, w2, rtol=1e-12)               # renormalised = softmax over the chosen
    _, w1 = oracle.router_topk(lg, 96, oracle.ROUTER_TOPK_SOFTMAX)
    np.testing.assert_allclose(w1.sum(1), 1.0, rtol=1e-12)       # K = E: the full softmax
