"""CPU models of two kernel designs, checked against plain definitions.

These pin the reasoning the kernels rest on, without a GPU; the GPU tests
compare the kernels themselves with the oracle.

- Router top-k for K <= 8, E <= 256 (csrc/router.cu, router_top8_kernel):
  eight threads per token, each holding the 16-byte chunks c = j, j+8, ... of
  the row; integer keys that carry the expert id in their low bits; groups of
  8 keys sorted by a 19-comparator network; a bitonic half-cleaner step and a
  12-comparator bitonic sort to merge a group (or a partner thread's list)
  into a top-8 list, keeping the largest discarded key; three shuffle rounds;
  for fp32 keys a retry with exact 64-bit keys when two keys that decide the
  result share their high bits.  The model follows those steps and must give
  the K largest logits, ties to the lower id, on random, tied, near-tied and
  -inf rows.
- The expert rows' storage (common.cuh y_block_exp): fp16 of v * 2^-e with
  e = clamp(floor(log2 m) - 14, -100, 113) for a block whose largest |v| is m.
  Every stored value stays below fp16's largest finite value over bf16's whole
  range, the decode is exact, and every element within 2^28 of m keeps fp16's
  11 significant bits.
"""
import struct

import numpy as np
import pytest

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")

NET8 = [(0, 2), (1, 3), (4, 6), (5, 7), (0, 4), (1, 5), (2, 6), (3, 7), (0, 1), (2, 3), (4, 5), (6, 7),
        (2, 4), (3, 5), (1, 4), (3, 6), (1, 2), (3, 4), (5, 6)]
SORT4 = [(0, 1), (2, 3), (0, 2), (1, 3), (1, 2)]
TPT = 8  # threads per token


def order_key(v: float) -> int:
    """Order-preserving unsigned image of an fp32 value (NaN read as -inf, -0 as +0)."""
    v = np.float32(v)
    if np.isnan(v):
        v = np.float32(-np.inf)
    v = np.float32(v + np.float32(0.0))
    u = struct.unpack("<I", struct.pack("<f", v))[0]
    return (~u) & 0xFFFFFFFF if u & 0x80000000 else u | 0x80000000


def pack(v, e, mask, wide):
    k = order_key(v)
    return (k << 32) | (0xFFFFFFFF - e) if wide else (k | mask) - e


def cx(b, i, j):
    b[i], b[j] = max(b[i], b[j]), min(b[i], b[j])


def bitonic8(a):
    for d in (4, 2, 1):
        for j in range(8):
            if j & d == 0:
                cx(a, j, j + d)


def merge_top8(a, b, rej):
    for j in range(8):
        o = b[7 - j]
        rej = max(rej, min(a[j], o))
        a[j] = max(a[j], o)
    bitonic8(a)
    return rej


def chunk_keys(x, q, m, E, mask, wide):
    e0 = 4 * (q + TPT * m)
    return [pack(x[e0 + i], e0 + i, mask, wide) if e0 < E else 0 for i in range(4)]


def top8_keys(x, E, chunks, mask, wide):
    lists = []
    for q in range(TPT):
        rej = 0
        if chunks == 1:
            a = chunk_keys(x, q, 0, E, mask, wide)
            for i, j in SORT4:
                cx(a, i, j)
            a += [0] * 4
        else:
            a = chunk_keys(x, q, 0, E, mask, wide) + chunk_keys(x, q, 1, E, mask, wide)
            for i, j in NET8:
                cx(a, i, j)
            for m in range(2, chunks, 2):
                b = chunk_keys(x, q, m, E, mask, wide) + chunk_keys(x, q, m + 1, E, mask, wide)
                for i, j in NET8:
                    cx(b, i, j)
                rej = merge_top8(a, b, rej)
        lists.append((a, rej))
    for s in (1, 2, 4):  # shuffle rounds: thread q merges with q ^ s
        merged = []
        for q in range(TPT):
            a = list(lists[q][0])
            rej = max(lists[q][1], lists[q ^ s][1])
            rej = merge_top8(a, lists[q ^ s][0], rej)
            merged.append((a, rej))
        lists = merged
    assert all(l == lists[0] for l in lists), "the eight threads end with one list"
    return lists[0]


def router_model(x, K, bf16=False):
    E = len(x)
    chunks = next(c for c in (1, 2, 4, 8) if E <= 32 * c)
    mask = 0xFFFF if bf16 else 32 * chunks - 1
    a, rej = top8_keys(x, E, chunks, mask, False)
    redo = False
    if not bf16:
        hi = lambda k: k | mask
        redo = any(hi(a[j]) == hi(a[j + 1]) for j in range(K - 1))
        nxt = a[K] if K < 8 else rej
        redo |= hi(a[K - 1]) == hi(nxt)
    if redo:
        b, _ = top8_keys(x, E, chunks, mask, True)
        return [0xFFFFFFFF - (k & 0xFFFFFFFF) for k in b][:K], True
    return [mask - (k & mask) for k in a][:K], False


def topk_by_sort(x, K):
    v = [(-np.inf if np.isnan(t) else float(t)) for t in x]
    return sorted(range(len(v)), key=lambda e: (-v[e], e))[:K]


def _rows(rng, n):
    for t in range(n):
        E = int(rng.choice([4, 8, 12, 16, 32, 36, 64, 100, 128, 200, 256]))
        K = int(rng.integers(1, min(8, E) + 1))
        kind = t % 5
        if kind == 0:
            x = rng.standard_normal(E).astype(np.float32)
        elif kind == 1:  # many exact ties
            x = np.round(rng.standard_normal(E) * 2).astype(np.float32)
        elif kind == 2:  # a few ulp apart: keys share their high bits
            base = np.float32(rng.standard_normal())
            x = (base + rng.integers(-40, 40, E).astype(np.float32) * np.spacing(base)).astype(np.float32)
        elif kind == 3:  # -inf and NaN
            x = rng.standard_normal(E).astype(np.float32)
            x[rng.integers(0, E, E // 3)] = -np.inf
            x[rng.integers(0, E, 2)] = np.nan
        else:  # signed zeros next to negative values
            x = -np.abs(rng.standard_normal(E)).astype(np.float32)
            x[rng.integers(0, E, 3)] = np.float32(-0.0)
            x[rng.integers(0, E, 3)] = np.float32(0.0)
        bf16 = t % 3 == 0
        if bf16:
            x = (np.frombuffer(x.tobytes(), np.uint32) & 0xFFFF0000).view(np.float32)
        yield x, K, bf16


def test_router_network_model_matches_a_sort():
    rng = np.random.default_rng(0)
    retried = 0
    for x, K, bf16 in _rows(rng, 600):
        got, redo = router_model(list(x), K, bf16)
        retried += redo
        assert got == topk_by_sort(list(x), K), (len(x), K, bf16, got)
    assert retried > 0  # the exact retry path was exercised


def test_router_bf16_keys_are_exact():
    """A bf16 logit widened to fp32 has zero low 16 bits: (key | 0xffff) - id
    orders exactly as (logit, -id), so bf16 rows never need the retry."""
    rng = np.random.default_rng(1)
    for x, K, bf16 in _rows(rng, 300):
        if bf16:
            assert not router_model(list(x), K, True)[1]


def test_sort8_network_sorts_every_binary_input():
    """The 0-1 principle: a comparator network that sorts all 2^8 binary inputs
    sorts every input."""
    for bits in range(256):
        a = [(bits >> i) & 1 for i in range(8)]
        for i, j in NET8:
            cx(a, i, j)
        assert a == sorted(a, reverse=True)


# ---- the expert rows: fp16 times a power of two per 32-column block ----------

def y_block_exp(m: float) -> int:
    """common.cuh y_block_exp on the fp32 bits of m >= 0."""
    be = (struct.unpack("<I", struct.pack("<f", np.float32(m)))[0] >> 23) & 0xFF
    return min(max(be - 127 - 14, -100), 113)


def encode_block(v):
    m = float(np.max(np.abs(v)))
    e = y_block_exp(m)
    return (v.astype(np.float64) * 2.0 ** -e).astype(np.float32).astype(np.float16), e


@pytest.mark.parametrize("log2_scale", [-126, -120, -100, -60, -14, 0, 14, 60, 100, 120, 126])
def test_block_exponent_keeps_bf16_range_and_11_bits(log2_scale):
    rng = np.random.default_rng(log2_scale + 200)
    for _ in range(200):
        # one block: a spread of magnitudes up to ~2^30 below its largest
        v = (rng.standard_normal(32) * np.exp2(rng.uniform(-30, 0, 32))).astype(np.float32)
        v = (v.astype(np.float64) * 2.0 ** log2_scale)
        v = np.clip(v, -3.0e38, 3.0e38).astype(np.float32)
        f16, e = encode_block(v)
        assert np.all(np.isfinite(f16)), "a stored value overflowed fp16"
        assert np.max(np.abs(f16.astype(np.float64))) <= 2.0 ** 15
        dec = f16.astype(np.float64) * 2.0 ** e
        m = float(np.max(np.abs(v)))
        if m == 0:
            continue
        big = np.abs(v) >= m * 2.0 ** -28
        big &= np.abs(v) >= 2.0 ** -126  # fp32 normals (the device's inputs are bf16/fp32)
        rel = np.abs(dec[big] - v[big]) / np.abs(v[big].astype(np.float64))
        if -100 <= np.floor(np.log2(m)) - 14 <= 113:  # exponent not clamped
            assert np.all(rel <= 2.0 ** -11), f"max rel {rel.max():.3g}"
            assert 2.0 ** 14 <= np.max(np.abs(f16.astype(np.float64))) <= 2.0 ** 15


def test_block_exponent_decode_is_exact():
    """A stored value (|fp16| <= 2^15, as the encoder makes them) times 2^e for
    e in [-100, 113] is an exact fp32, so the combine folds 2^e into the pair's
    weight without a rounding.  The one exception, 2^15 at e = 113 (2^128),
    comes only from an fp32 y within 2^-12 of fp32's largest value, which the
    bf16 output could not hold either."""
    f16 = np.arange(-32768, 32769, 7, dtype=np.float64).astype(np.float16)
    for e in (-100, -50, -14, 0, 14, 50, 100, 112, 113):
        d = f16.astype(np.float64) * 2.0 ** e
        if e == 113:
            d = d[np.abs(f16.astype(np.float64)) < 2.0 ** 15]
        assert np.array_equal(d.astype(np.float32).astype(np.float64), d)
