"""Seeded synthetic inputs for the local MoE expert forward on the non-expand layout.

This module only draws random numbers and arranges them into the input tensors
of the method; it holds none of the method's own arithmetic (no histogram,
scan, sort, GEMM, activation or combine).  Both the CUDA path and the CPU
oracle are fed from here, and neither of them is imported by it.

Input layout (sonic-moe issue #68, "End-to-end DeepEP v2 non-expand + SonicMoE
integration", the non-expand receive block): ``x [N,H]`` bf16, ``topk_idx
[N,K]`` int32 holding a local expert id or -1 for an invalid slot, and
``topk_w [N,K]`` fp32.  Expert weights follow the proposed API of the same
issue (``w1, b1, w2, b2``): ``w1 [E,H,2I]``, ``b1 [E,2I]``, ``w2 [E,I,H]``,
``b2 [E,H]``, all bf16.

Recipes (one per named workload):

* routing tensors and scores come from ``numpy.random.Generator(PCG64(seed))``
  on the host;
* ``x``, weights and biases come from a seeded ``torch.Generator`` on the
  requested device, drawn in fp32 and rounded to bf16.  The values therefore
  depend on the device the generator runs on; every consumer (kernel or
  oracle) is always handed the very same tensors.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch


# ----------------------------------------------------------------------------
# Named workloads.  Sizes follow the shapes the pages benchmark (sonic-moe
# write-up, "Three routing strategies" and "Interleaved by default" sections:
# E=128 / E=256 experts with top-8; issue #68: rank-local rows after an
# 8-way dispatch).
# ----------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    N: int
    H: int
    I: int
    E: int
    K: int
    routing: str            # "uniform", "zipf", "ranklocal"
    zipf_s: float = 0.0
    p_invalid: float = 0.0  # probability that a slot is set to -1
    scores: str = "softmax"  # "softmax" over valid slots, "uniform", "uniform_renorm"
    bias: bool = False
    seed: int = 0
    description: str = ""


WORKLOADS = {
    "tiny": Workload(
        "tiny", N=256, H=128, I=256, E=8, K=2, routing="uniform", p_invalid=0.10,
        scores="softmax", bias=True, seed=1,
        description="tiny correctness case: 2 distinct uniform experts per row, "
                    "10% of slots -1, softmax scores over valid slots, biases"),
    "metadata": Workload(
        "metadata", N=65536, H=0, I=0, E=128, K=8, routing="zipf", zipf_s=1.1,
        p_invalid=0.05, scores="uniform_renorm", seed=2,
        description="metadata only: Zipf(1.1) popularity over a permuted expert "
                    "order, distinct per row, 5% of slots -1, U(0,1) scores "
                    "renormalised over valid slots"),
    "prefill": Workload(
        "prefill", N=16384, H=2048, I=768, E=128, K=8, routing="uniform",
        scores="softmax", seed=3,
        description="Qwen3-MoE-like prefill: 8 distinct uniform experts of 128, "
                    "no invalid slots, softmax scores, no biases"),
    "ranklocal": Workload(
        "ranklocal", N=8192, H=7168, I=2048, E=32, K=8, routing="ranklocal",
        scores="uniform", seed=4,
        description="rank-local rows after an 8-way dispatch: each row keeps "
                    "1-4 distinct local experts in random slots, the rest -1, "
                    "U(0,1) scores"),
    "decode256": Workload(
        "decode256", N=128, H=2048, I=512, E=256, K=8, routing="zipf", zipf_s=1.2,
        scores="softmax", seed=5,
        description="256-expert Zipf(1.2) imbalance, decode-sized"),
    "profile_small": Workload(
        "profile_small", N=4096, H=2048, I=768, E=32, K=8, routing="uniform",
        scores="softmax", seed=7,
        description="profiling case: the prefill shape with 32 experts and 4096 tokens "
                    "(1024 rows per expert as in prefill, about 1 GB on the device)"),
    "prefill256": Workload(
        "prefill256", N=16384, H=2048, I=512, E=256, K=8, routing="zipf", zipf_s=1.2,
        scores="softmax", seed=6,
        description="256-expert Zipf(1.2) imbalance, prefill-sized"),
}


# ----------------------------------------------------------------------------
# Routing draws (host, numpy PCG64).
# ----------------------------------------------------------------------------

def _distinct_uniform(rng: np.random.Generator, N: int, K: int, E: int) -> np.ndarray:
    """K distinct experts per row, uniformly (argpartition of uniform keys)."""
    keys = rng.random((N, E))
    return np.argpartition(keys, K - 1, axis=1)[:, :K].astype(np.int32)


def _distinct_zipf(rng: np.random.Generator, N: int, K: int, E: int, s: float) -> np.ndarray:
    """K distinct experts per row drawn without replacement from Zipf(s)
    popularity over a seeded random expert permutation (Gumbel-top-k)."""
    perm = rng.permutation(E)
    ranks = np.empty(E, dtype=np.float64)
    ranks[perm] = np.arange(1, E + 1, dtype=np.float64)
    logp = -s * np.log(ranks)
    out = np.empty((N, K), dtype=np.int32)
    step = max(1, (1 << 22) // E)
    for r0 in range(0, N, step):
        r1 = min(N, r0 + step)
        g = rng.gumbel(size=(r1 - r0, E)) + logp[None, :]
        top = np.argpartition(-g, K - 1, axis=1)[:, :K]
        # order the K picks by key so the slot order is itself random-looking
        out[r0:r1] = top.astype(np.int32)
    return out


def _ranklocal(rng: np.random.Generator, N: int, K: int, E: int, lo: int = 1, hi: int = 4) -> np.ndarray:
    """Each row keeps m ~ U{lo..hi} distinct uniform experts placed in m random
    slot positions; the other slots are -1."""
    idx = np.full((N, K), -1, dtype=np.int32)
    m = rng.integers(lo, hi + 1, size=N)
    experts = _distinct_uniform(rng, N, hi, E)
    pos = np.argsort(rng.random((N, K)), axis=1)[:, :hi]
    for j in range(hi):
        rows = np.nonzero(m > j)[0]
        idx[rows, pos[rows, j]] = experts[rows, j]
    return idx


def routing(wl: Workload, rng: np.random.Generator) -> np.ndarray:
    if wl.routing == "uniform":
        idx = _distinct_uniform(rng, wl.N, wl.K, wl.E)
    elif wl.routing == "zipf":
        idx = _distinct_zipf(rng, wl.N, wl.K, wl.E, wl.zipf_s)
    elif wl.routing == "ranklocal":
        idx = _ranklocal(rng, wl.N, wl.K, wl.E)
    else:
        raise ValueError(wl.routing)
    if wl.p_invalid > 0:
        drop = rng.random(idx.shape) < wl.p_invalid
        idx = np.where(drop, np.int32(-1), idx).astype(np.int32)
    return np.ascontiguousarray(idx, dtype=np.int32)


def scores(wl: Workload, idx: np.ndarray, rng: np.random.Generator,
           invalid_value: float = 0.0) -> np.ndarray:
    """Router scores [N,K] fp32.  Invalid slots get ``invalid_value`` (tests
    pass NaN to prove their values are never used)."""
    valid = idx >= 0
    if wl.scores == "softmax":
        logits = rng.standard_normal(idx.shape)
        logits = np.where(valid, logits, -np.inf)
        mx = np.max(np.where(valid, logits, -1e300), axis=1, keepdims=True)
        ex = np.where(valid, np.exp(logits - mx), 0.0)
        den = ex.sum(axis=1, keepdims=True)
        w = np.divide(ex, den, out=np.zeros_like(ex), where=den > 0)
    elif wl.scores == "uniform":
        w = rng.random(idx.shape)
    elif wl.scores == "uniform_renorm":
        w = np.where(valid, rng.random(idx.shape), 0.0)
        den = w.sum(axis=1, keepdims=True)
        w = np.divide(w, den, out=np.zeros_like(w), where=den > 0)
    else:
        raise ValueError(wl.scores)
    w = np.where(valid, w, invalid_value).astype(np.float32)
    return np.ascontiguousarray(w)


# ----------------------------------------------------------------------------
# Dense tensors (torch, seeded, on a chosen device).
# ----------------------------------------------------------------------------

def _normal_bf16(shape, std: float, gen: torch.Generator, device) -> torch.Tensor:
    t = torch.empty(shape, dtype=torch.float32, device=device)
    t.normal_(mean=0.0, std=std, generator=gen)
    return t.to(torch.bfloat16)


def _normal_bf16_per_expert(E: int, shape, std: float, gen: torch.Generator, device) -> torch.Tensor:
    out = torch.empty((E,) + tuple(shape), dtype=torch.bfloat16, device=device)
    for e in range(E):
        out[e] = _normal_bf16(shape, std, gen, device)
    return out


@dataclasses.dataclass
class Inputs:
    wl: Workload
    x: Optional[torch.Tensor]        # [N,H] bf16
    topk_idx: torch.Tensor           # [N,K] int32
    topk_w: torch.Tensor             # [N,K] fp32
    w1: Optional[torch.Tensor]       # [E,H,2I] bf16
    b1: Optional[torch.Tensor]       # [E,2I] bf16 or None
    w2: Optional[torch.Tensor]       # [E,I,H] bf16
    b2: Optional[torch.Tensor]       # [E,H] bf16 or None

    @property
    def total_pairs(self) -> int:
        return int((self.topk_idx >= 0).sum().item())


def make_routing(wl: Workload, seed: Optional[int] = None, invalid_value: float = 0.0):
    rng = np.random.Generator(np.random.PCG64(wl.seed if seed is None else seed))
    idx = routing(wl, rng)
    w = scores(wl, idx, rng, invalid_value=invalid_value)
    return idx, w


def make_inputs(wl: Workload | str, device="cpu", seed: Optional[int] = None,
                invalid_value: float = 0.0, with_dense: bool = True) -> Inputs:
    """Build one workload's inputs.  ``seed`` overrides the workload's seed."""
    if isinstance(wl, str):
        wl = WORKLOADS[wl]
    s = wl.seed if seed is None else seed
    idx, w = make_routing(wl, s, invalid_value)
    topk_idx = torch.from_numpy(idx).to(device)
    topk_w = torch.from_numpy(w).to(device)
    x = w1 = b1 = w2 = b2 = None
    if with_dense and wl.H > 0:
        gen = torch.Generator(device=device)
        gen.manual_seed(1000003 * s + 17)
        x = _normal_bf16((wl.N, wl.H), 1.0, gen, device)
        w1 = _normal_bf16_per_expert(wl.E, (wl.H, 2 * wl.I), wl.H ** -0.5, gen, device)
        w2 = _normal_bf16_per_expert(wl.E, (wl.I, wl.H), wl.I ** -0.5, gen, device)
        if wl.bias:
            b1 = _normal_bf16((wl.E, 2 * wl.I), 0.01, gen, device)
            b2 = _normal_bf16((wl.E, wl.H), 0.01, gen, device)
    return Inputs(wl, x, topk_idx, topk_w, w1, b1, w2, b2)


def custom(N: int, H: int, I: int, E: int, K: int, *, routing_kind="uniform",
           zipf_s=1.2, p_invalid=0.0, scores_kind="softmax", bias=False, seed=0,
           name="custom") -> Workload:
    """A workload with arbitrary sizes (tests use it for ragged and edge cases)."""
    return Workload(name, N=N, H=H, I=I, E=E, K=K, routing=routing_kind, zipf_s=zipf_s,
                    p_invalid=p_invalid, scores=scores_kind, bias=bias, seed=seed)


def pair_list_from_table(idx: np.ndarray, w: np.ndarray, *, keep_invalid: bool = False,
                         empty_tokens: Optional[np.ndarray] = None):
    """A compact pair list (token_idx, expert_idx, weights; tokens ascending)
    holding the slots of an [N,K] routing table in row-major order.  Slots
    marked -1 are dropped unless ``keep_invalid``; tokens listed in
    ``empty_tokens`` lose all their entries (tokens without pairs)."""
    N, K = idx.shape
    tok = np.repeat(np.arange(N, dtype=np.int64), K)
    exp = idx.reshape(-1).astype(np.int64)
    wt = w.reshape(-1).astype(np.float32)
    keep = np.ones(N * K, bool) if keep_invalid else exp >= 0
    if empty_tokens is not None:
        keep &= ~np.isin(tok, empty_tokens)
    return tok[keep], exp[keep], wt[keep]


def many_pair_tokens(N: int, E: int, heavy: np.ndarray, K: int, rng: np.random.Generator):
    """A pair list where the tokens in ``heavy`` route to every expert and the
    others to K distinct experts (tokens ascending, experts in random order
    within a token); weights uniform in [0,1)."""
    toks, exps = [], []
    for t in range(N):
        k = E if t in set(heavy.tolist()) else K
        e = rng.permutation(E)[:k]
        toks.append(np.full(k, t, np.int64))
        exps.append(e.astype(np.int64))
    tok = np.concatenate(toks)
    exp = np.concatenate(exps)
    return tok, exp, rng.random(tok.shape[0]).astype(np.float32)


def make_logits(N: int, E: int, seed: int = 0, dtype=torch.float32, kind: str = "normal",
                device="cpu") -> torch.Tensor:
    """Router logits [N,E]: ``normal`` draws N(0,1) (distinct values in
    practice); ``ties`` draws integers in [-2,2] (many equal logits per row)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    if kind == "normal":
        a = rng.standard_normal((N, E)).astype(np.float32)
    elif kind == "ties":
        a = rng.integers(-2, 3, size=(N, E)).astype(np.float32)
    else:
        raise ValueError(kind)
    return torch.from_numpy(a).to(dtype).to(device)
