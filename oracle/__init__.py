"""CPU oracle for the local MoE expert forward on the non-expand layout.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may use it; the product path never does.  It is a
plain C file (``moe_oracle.c``) compiled here with gcc into ``_oracle.so`` and
called through ctypes; it shares no code with the CUDA library.

The functions follow the definitions written at the top of ``moe_oracle.c``
(sonic-moe issue #68 metadata list and question 3; qwen3_5.py commit notes,
CCCL segmented-sort recipe; sonic-moe write-up, weight-layout section).
Arithmetic is double precision on bf16 inputs, with no intermediate rounding.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_oracle.so")
_lock = threading.Lock()
_libs = {}

LAYOUT_INTERLEAVED = 0
LAYOUT_CONCATENATED = 1


def compile_source(src: str, out: str) -> str:
    """Compile a C file of the oracle's interface with gcc (OpenMP)."""
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", tmp, src, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile the oracle if the shared object is missing or stale."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    return compile_source(_SRC, _LIB_PATH)


def _load(path: str | None = None):
    """The oracle library (or, for the mutation pins, a variant compiled
    from an edited copy of its source at ``path``)."""
    with _lock:
        key = path or _LIB_PATH
        if key in _libs:
            return _libs[key]
        lib = ctypes.CDLL(build() if path is None else path)
        P = ctypes.c_void_p
        i64, i32 = ctypes.c_int64, ctypes.c_int32
        lib.oracle_metadata.restype = i64
        lib.oracle_metadata.argtypes = [i64, i32, i32, P, P, P, P, P, P, P, P, P, P]
        lib.oracle_metadata_pairs.restype = i64
        lib.oracle_metadata_pairs.argtypes = [i64, i64, i32, P, P, P, P, P, P, P, P, P, P, P, P, P]
        lib.oracle_router_topk.restype = None
        lib.oracle_router_topk.argtypes = [i64, i32, i32, i32, P, P, P]
        lib.oracle_pair_backward.restype = None
        lib.oracle_pair_backward.argtypes = [i32, i32, i32, P, P, P, P, P, P, ctypes.c_double, P, P, P, P, P, P]
        lib.oracle_pairs_backward.restype = None
        lib.oracle_pairs_backward.argtypes = [i32, i32, i32, P, P, P, P, P, P, i64, P, P, P, P, P, P, P, P, i32]
        lib.oracle_expert_row.restype = None
        lib.oracle_expert_row.argtypes = [i32, i32, i32, P, P, P, P, P, P, P, P]
        lib.oracle_forward_rows.restype = None
        lib.oracle_forward_rows.argtypes = [i64, i32, i32, i32, i32, i32, P, P, P, P, P, P, P,
                                            i64, P, P, i32]
        lib.oracle_combine.restype = None
        lib.oracle_combine.argtypes = [i64, i32, P, P, P, P, P]
        lib.oracle_pair_rows.restype = None
        lib.oracle_pair_rows.argtypes = [i32, i32, i32, P, P, P, P, P, i64, P, P, P, P, i32]
        _libs[key] = lib
        return lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _bf16_bits(t):
    """Raw bf16 bit patterns (uint16) of a torch bf16 tensor, or None."""
    if t is None:
        return None
    import torch
    assert t.dtype == torch.bfloat16
    return np.ascontiguousarray(t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def metadata(topk_idx: np.ndarray, topk_w: np.ndarray, E: int, lib_path: str | None = None) -> dict:
    """Routing metadata of a [N,K] non-expand layout.  Returns a dict with
    freq [E], off [E+1], x_gather_idx / s_scatter_idx / s_reverse_scatter_idx
    [P], token_offset [N+1], scores [P], P and bad_ids."""
    lib = _load(lib_path)
    idx = np.ascontiguousarray(topk_idx, dtype=np.int32)
    w = np.ascontiguousarray(topk_w, dtype=np.float32)
    N, K = idx.shape
    cap = max(1, N * K)
    freq = np.zeros(E, np.int32)
    off = np.zeros(E + 1, np.int32)
    xg = np.zeros(cap, np.int32)
    ss = np.zeros(cap, np.int32)
    sr = np.zeros(cap, np.int32)
    to = np.zeros(N + 1, np.int32)
    sc = np.zeros(cap, np.float32)
    bad = np.zeros(1, np.int64)
    P = lib.oracle_metadata(N, K, E, _ptr(idx), _ptr(w), _ptr(freq), _ptr(off), _ptr(xg),
                            _ptr(ss), _ptr(sr), _ptr(to), _ptr(sc), _ptr(bad))
    return dict(freq=freq, off=off, x_gather_idx=xg[:P].copy(), s_scatter_idx=ss[:P].copy(),
                s_reverse_scatter_idx=sr[:P].copy(), token_offset=to, scores=sc[:P].copy(),
                P=int(P), bad_ids=int(bad[0]))


def metadata_pairs(token_idx: np.ndarray, expert_idx: np.ndarray, weights: np.ndarray, N: int, E: int,
                   lib_path: str | None = None) -> dict:
    """Routing metadata of a compact pair list (token_idx ascending).  Returns
    the keys of ``metadata`` plus bad_tokens and unsorted."""
    lib = _load(lib_path)
    ti = np.ascontiguousarray(token_idx, dtype=np.int64).reshape(-1)
    ei = np.ascontiguousarray(expert_idx, dtype=np.int64).reshape(-1)
    w = np.ascontiguousarray(weights, dtype=np.float32).reshape(-1)
    PL = ti.shape[0]
    assert ei.shape[0] == PL and w.shape[0] == PL
    cap = max(1, PL)
    freq = np.zeros(E, np.int32)
    off = np.zeros(E + 1, np.int32)
    xg = np.zeros(cap, np.int32)
    ss = np.zeros(cap, np.int32)
    sr = np.zeros(cap, np.int32)
    to = np.zeros(N + 1, np.int32)
    sc = np.zeros(cap, np.float32)
    bad = np.zeros(1, np.int64)
    badt = np.zeros(1, np.int64)
    uns = np.zeros(1, np.int32)
    P = lib.oracle_metadata_pairs(N, PL, E, _ptr(ti), _ptr(ei), _ptr(w), _ptr(freq), _ptr(off), _ptr(xg),
                                  _ptr(ss), _ptr(sr), _ptr(to), _ptr(sc), _ptr(bad), _ptr(badt), _ptr(uns))
    return dict(freq=freq, off=off, x_gather_idx=xg[:P].copy(), s_scatter_idx=ss[:P].copy(),
                s_reverse_scatter_idx=sr[:P].copy(), token_offset=to, scores=sc[:P].copy(),
                P=int(P), bad_ids=int(bad[0]), bad_tokens=int(badt[0]), unsorted=bool(uns[0]))


ROUTER_SOFTMAX_TOPK = 0
ROUTER_TOPK_SOFTMAX = 1
ROUTER_TOPK_SOFTMAX_RENORM = 2


def router_topk(logits, K: int, mode: int = ROUTER_SOFTMAX_TOPK, lib_path: str | None = None):
    """Router top-k of logits [N,E] (a torch fp32/bf16 tensor or a numpy
    array; widened exactly to double, NaN read as -inf).  Returns
    (topk_idx [N,K] int32, topk_w [N,K] float64)."""
    lib = _load(lib_path)
    if not isinstance(logits, np.ndarray):
        import torch
        logits = logits.detach().cpu().to(torch.float64).numpy()
    lg = np.ascontiguousarray(logits, dtype=np.float64).copy()
    lg[np.isnan(lg)] = -np.inf
    N, E = lg.shape
    idx = np.zeros((N, K), np.int32)
    w = np.zeros((N, K), np.float64)
    lib.oracle_router_topk(N, E, K, mode, _ptr(lg), _ptr(idx), _ptr(w))
    return idx, w


def expert_row(x_row, w1e, b1e, w2e, b2e, layout: int = LAYOUT_INTERLEAVED, lib_path: str | None = None):
    """One expert on one token row (bf16 torch tensors in, float64 numpy out):
    returns (z [2I], h [I], y [H])."""
    lib = _load(lib_path)
    xr, a, b, c, d = (_bf16_bits(v) for v in (x_row, w1e, b1e, w2e, b2e))
    H = xr.shape[0]
    I = c.shape[0]
    z = np.zeros(2 * I, np.float64)
    h = np.zeros(I, np.float64)
    y = np.zeros(H, np.float64)
    lib.oracle_expert_row(H, I, layout, _ptr(xr), _ptr(a), _ptr(b), _ptr(c), _ptr(d),
                          _ptr(z), _ptr(h), _ptr(y))
    return z, h, y


class Weights:
    """Host bf16 bit copies of the forward's dense inputs, made once."""

    def __init__(self, x, w1, b1, w2, b2):
        self.x = _bf16_bits(x)
        self.w1 = _bf16_bits(w1)
        self.b1 = _bf16_bits(b1)
        self.w2 = _bf16_bits(w2)
        self.b2 = _bf16_bits(b2)
        self.N, self.H = self.x.shape
        self.E, _, two_i = self.w1.shape
        self.I = two_i // 2


def forward_rows(wts: Weights, topk_idx: np.ndarray, topk_w: np.ndarray, tokens=None,
                 layout: int = LAYOUT_INTERLEAVED, n_threads: int = 0, lib_path: str | None = None) -> np.ndarray:
    """Output rows [len(tokens), H] (float64) of the forward for the chosen
    tokens (all tokens when None)."""
    lib = _load(lib_path)
    idx = np.ascontiguousarray(topk_idx, dtype=np.int32)
    w = np.ascontiguousarray(topk_w, dtype=np.float32)
    N, K = idx.shape
    if tokens is None:
        tokens = np.arange(N, dtype=np.int64)
    tokens = np.ascontiguousarray(tokens, dtype=np.int64)
    out = np.zeros((tokens.shape[0], wts.H), np.float64)
    if n_threads <= 0:
        n_threads = len(os.sched_getaffinity(0))
    lib.oracle_forward_rows(N, wts.H, wts.I, wts.E, K, layout, _ptr(wts.x), _ptr(idx), _ptr(w),
                            _ptr(wts.w1), _ptr(wts.b1), _ptr(wts.w2), _ptr(wts.b2),
                            tokens.shape[0], _ptr(tokens), _ptr(out), n_threads)
    return out


def pair_rows(wts: Weights, tokens, experts, layout: int = LAYOUT_INTERLEAVED, n_threads: int = 0, lib_path: str | None = None):
    """(h [n,I], y [n,H]) float64 for the given (token, expert) pairs."""
    lib = _load(lib_path)
    tokens = np.ascontiguousarray(tokens, dtype=np.int64)
    experts = np.ascontiguousarray(experts, dtype=np.int32)
    n = tokens.shape[0]
    h = np.zeros((n, wts.I), np.float64)
    y = np.zeros((n, wts.H), np.float64)
    if n_threads <= 0:
        n_threads = len(os.sched_getaffinity(0))
    lib.oracle_pair_rows(wts.H, wts.I, layout, _ptr(wts.x), _ptr(wts.w1), _ptr(wts.b1),
                         _ptr(wts.w2), _ptr(wts.b2), n, _ptr(tokens), _ptr(experts),
                         _ptr(h), _ptr(y), n_threads)
    return h, y


def combine(token_offset: np.ndarray, s_rev: np.ndarray, scores: np.ndarray,
            ysorted: np.ndarray, lib_path: str | None = None) -> np.ndarray:
    """out [N,H] float64 = per token, sum over its pairs q (in q order) of
    scores[q] * ysorted[s_rev[q]]."""
    lib = _load(lib_path)
    to = np.ascontiguousarray(token_offset, dtype=np.int32)
    sr = np.ascontiguousarray(s_rev, dtype=np.int32)
    sc = np.ascontiguousarray(scores, dtype=np.float32)
    ys = np.ascontiguousarray(ysorted, dtype=np.float64)
    N = to.shape[0] - 1
    H = ys.shape[1]
    out = np.zeros((N, H), np.float64)
    lib.oracle_combine(N, H, _ptr(to), _ptr(sr), _ptr(sc), _ptr(ys), _ptr(out))
    return out


# ---------------------------------------------------------------------------
# Backward (chain rule of the forward above, in double)
# ---------------------------------------------------------------------------

def _f64(t):
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return np.ascontiguousarray(t, dtype=np.float64)
    import torch
    return np.ascontiguousarray(t.detach().cpu().to(torch.float64).numpy())


class WeightsF64:
    """The dense inputs for the backward oracle: x and the biases widened to
    float64 at once, each expert's weights widened exactly on demand (full
    float64 copies of large expert banks would not fit in host memory)."""

    def __init__(self, x, w1, b1, w2, b2):
        self.x, self.b1, self.b2 = _f64(x), _f64(b1), _f64(b2)
        self._w1, self._w2 = w1, w2
        self.N, self.H = self.x.shape
        self.E, _, two_i = w1.shape
        self.I = two_i // 2

    def w1e(self, e):
        return _f64(self._w1[e])

    def w2e(self, e):
        return _f64(self._w2[e])


def pairs_backward(wd: WeightsF64, dout, tokens, experts, scores, layout: int = LAYOUT_INTERLEAVED,
                   n_threads: int = 0, lib_path: str | None = None) -> dict:
    """Per pair (tokens[i], experts[i], scores[i]): h [n,I], y [n,H],
    dy [n,H], dz [n,2I] and ds [n], all float64."""
    lib = _load(lib_path)
    do = _f64(dout)
    tokens = np.ascontiguousarray(tokens, dtype=np.int64)
    experts = np.ascontiguousarray(experts, dtype=np.int32)
    scores = np.ascontiguousarray(scores, dtype=np.float64)
    n = tokens.shape[0]
    H, I = wd.H, wd.I
    out = dict(h=np.zeros((n, I)), y=np.zeros((n, H)), dy=np.zeros((n, H)), dz=np.zeros((n, 2 * I)),
               ds=np.zeros(n))
    if n_threads <= 0:
        n_threads = len(os.sched_getaffinity(0))
    for e in np.unique(experts):  # one expert's weights at a time
        sel = np.nonzero(experts == e)[0]
        m = sel.shape[0]
        w1e, w2e = wd.w1e(e), wd.w2e(e)
        b1e = None if wd.b1 is None else np.ascontiguousarray(wd.b1[e])
        b2e = None if wd.b2 is None else np.ascontiguousarray(wd.b2[e])
        part = dict(h=np.zeros((m, I)), y=np.zeros((m, H)), dy=np.zeros((m, H)), dz=np.zeros((m, 2 * I)),
                    ds=np.zeros(m))
        tk = np.ascontiguousarray(tokens[sel])
        ex = np.zeros(m, np.int32)
        sc = np.ascontiguousarray(scores[sel])
        lib.oracle_pairs_backward(H, I, layout, _ptr(wd.x), _ptr(w1e), _ptr(b1e), _ptr(w2e), _ptr(b2e), _ptr(do),
                                  m, _ptr(tk), _ptr(ex), _ptr(sc), _ptr(part["h"]), _ptr(part["y"]),
                                  _ptr(part["dy"]), _ptr(part["dz"]), _ptr(part["ds"]), n_threads)
        for k in out:
            out[k][sel] = part[k]
    return out


def pair_dx_rows(wd: WeightsF64, dz, experts) -> np.ndarray:
    """Each pair's share of dx before the per-token sum: dz[i] . w1[experts[i]]^T
    ([n, H], float64), from the per-pair dz of pairs_backward."""
    dz = np.asarray(dz, dtype=np.float64)
    experts = np.asarray(experts)
    out = np.zeros((dz.shape[0], wd.H))
    for e in np.unique(experts):
        sel = experts == e
        out[sel] = dz[sel] @ wd.w1e(e).T
    return out


def backward(wd: WeightsF64, topk_idx: np.ndarray, topk_w: np.ndarray, dout, layout: int = LAYOUT_INTERLEAVED,
             experts_only=None, lib_path: str | None = None) -> dict:
    """Gradients of sum_t <dout_t, out_t> for the [N,K] non-expand routing:
    dx [N,H], dw1 [E,H,2I], db1 [E,2I], dw2 [E,I,H], db2 [E,H], dtopk_w [N,K]
    (0 at invalid slots).  The per-pair terms come from pairs_backward; the
    sums over pairs use float64 matrix products.  With ``experts_only`` only
    those experts' pairs are computed (their weight gradients are complete;
    dx and dtopk_w then hold only those pairs' shares)."""
    idx = np.asarray(topk_idx)
    w = np.asarray(topk_w)
    N, K = idx.shape
    E = wd.E
    valid = (idx >= 0) & (idx < E)
    if experts_only is not None:
        valid &= np.isin(idx, np.asarray(experts_only))
    tok, slot = np.nonzero(valid)
    exp = idx[tok, slot].astype(np.int32)
    sc = w[tok, slot].astype(np.float64)
    g = _sum_pair_terms(wd, dout, tok, exp, sc, N, layout, lib_path)
    g["dtopk_w"] = np.zeros((N, K))
    g["dtopk_w"][tok, slot] = g["pairs"]["ds"]
    g["pairs"]["slot"] = slot
    return g


def backward_pairs(wd: WeightsF64, token_idx, expert_idx, weights, dout, layout: int = LAYOUT_INTERLEAVED,
                   lib_path: str | None = None) -> dict:
    """Gradients for a compact pair list (entries kept as in metadata_pairs:
    expert in [0,E) and token in [0,N)); dweights [P_list] holds each entry's
    score gradient, 0 for dropped entries."""
    ti = np.asarray(token_idx, dtype=np.int64).reshape(-1)
    ei = np.asarray(expert_idx, dtype=np.int64).reshape(-1)
    w = np.asarray(weights, dtype=np.float64).reshape(-1)
    N, E = wd.N, wd.E
    keep = (ei >= 0) & (ei < E) & (ti >= 0) & (ti < N)
    entry = np.nonzero(keep)[0]
    g = _sum_pair_terms(wd, dout, ti[entry], ei[entry].astype(np.int32), w[entry], N, layout, lib_path)
    g["dweights"] = np.zeros(ti.shape[0])
    g["dweights"][entry] = g["pairs"]["ds"]
    g["pairs"]["entry"] = entry
    return g


def _sum_pair_terms(wd, dout, tok, exp, sc, N, layout, lib_path):
    """Per-pair terms (pairs_backward) summed into dx, dW1, db1, dW2, db2."""
    H, I, E = wd.H, wd.I, wd.E
    r = pairs_backward(wd, dout, tok, exp, sc, layout, lib_path=lib_path)
    g = dict(dx=np.zeros((N, H)), dw1=np.zeros((E, H, 2 * I)), db1=np.zeros((E, 2 * I)),
             dw2=np.zeros((E, I, H)), db2=np.zeros((E, H)))
    g["pairs"] = dict(tok=tok, exp=exp, **r)  # the per-pair terms, for the tests' error scales
    for e in np.unique(exp):
        sel = exp == e
        te = tok[sel]
        g["dw2"][e] = r["h"][sel].T @ r["dy"][sel]
        g["db2"][e] = r["dy"][sel].sum(0)
        g["dw1"][e] = wd.x[te].T @ r["dz"][sel]
        g["db1"][e] = r["dz"][sel].sum(0)
        np.add.at(g["dx"], te, r["dz"][sel] @ wd.w1e(e).T)
    return g
