"""Shared helpers of the parity tests: the output tolerance and comparisons."""
import numpy as np
import torch

# Output tolerance of the bf16 forward, per element:
#   |gpu - ref| <= RTOL * |ref| + ATOL_RMS * rms(ref)
# with rms over the compared elements.  The GPU path rounds h and y to bf16
# (relative step 2^-8) and accumulates in fp32; the oracle is exact double.
RTOL = 2e-2
ATOL_RMS = 2e-2


def within_tolerance(gpu: np.ndarray, ref: np.ndarray, rtol=RTOL, atol_rms=ATOL_RMS):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    bound = rtol * np.abs(ref) + atol_rms * rms
    err = np.abs(gpu - ref)
    bad = ~(err <= bound)
    return (not bad.any()), dict(max_err=float(err.max()) if err.size else 0.0, rms=rms,
                                 n_bad=int(bad.sum()), n=int(err.size),
                                 worst=np.unravel_index(int(np.argmax(err - bound)), err.shape)
                                 if err.size else None)


def assert_close_ep(gpu, ref, mag, what=""):
    """Expert-parallel routed_out: every rank's partial (its local forward
    output) carries the forward tolerance of that partial and is rounded to
    bf16 before the combine adds the partials.  So |ref| and rms(ref) of the
    forward bound become S = sum over the partials of |partial| (``mag``) and
    rms(S); with a single partial this is the forward tolerance itself."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    mag = np.asarray(mag, dtype=np.float64)
    rms = float(np.sqrt(np.mean(mag * mag))) if mag.size else 0.0
    bound = RTOL * mag + ATOL_RMS * rms
    err = np.abs(gpu - ref)
    bad = ~(err <= bound)
    assert not bad.any(), (f"{what}: max_err {err.max():.4g}, rms(S) {rms:.4g}, n_bad {int(bad.sum())}/{err.size}, "
                           f"worst {np.unravel_index(int(np.argmax(err - bound)), err.shape)}")


def assert_close(gpu, ref, what=""):
    ok, info = within_tolerance(gpu, ref)
    assert ok, f"{what}: {info}"


def to_np(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.detach().cpu().numpy()


def check_meta_equal(gpu_meta: dict, ref: dict):
    """Bit-exact comparison of the GPU metadata with the oracle's."""
    P = ref["P"]
    pairs = ("x_gather_idx", "s_scatter_idx", "s_reverse_scatter_idx")
    np.testing.assert_array_equal(to_np(gpu_meta["expert_frequency"]), ref["freq"])
    np.testing.assert_array_equal(to_np(gpu_meta["expert_frequency_offset"]), ref["off"])
    for k in pairs:
        np.testing.assert_array_equal(to_np(gpu_meta[k])[:P], ref[k], err_msg=k)
    np.testing.assert_array_equal(to_np(gpu_meta["token_offset"]), ref["token_offset"])
    np.testing.assert_array_equal(to_np(gpu_meta["scores"])[:P].view(np.int32),
                                  ref["scores"].view(np.int32))


# Backward tolerance.  A gradient entry is a sum of products whose factors
# carry at most a few bf16 roundings on the GPU path (dz or dy, the stored dx
# rows, the output itself; z is kept in fp32 and dh is formed from bf16
# inputs in fp32), each a relative error within the bf16 unit roundoff
# u = 2^-8 of the factor it rounds and independent across terms, so the
# entry's error is of order u * rss, rss = the root sum of squares of its
# terms; over ~10^6 entries the largest reaches ~5 standard deviations.  The
# bound adds 8 u rss to the forward's bound.
BWD_ULP = 2.0 ** -8
BWD_RSS_FACTOR = 8.0


def backward_rss(g, wd, dout):
    """Root sum of squares of the terms of every gradient entry, from the
    oracle's per-pair values (oracle.backward(...)["pairs"])."""
    pr = g["pairs"]
    tok, exp = pr["tok"], pr["exp"]
    score = "dtopk_w" if "dtopk_w" in g else "dweights"
    rss = {k: np.zeros_like(g[k]) for k in ("dx", "dw1", "db1", "dw2", "db2", score)}
    x2 = wd.x ** 2
    for e in np.unique(exp):
        sel = exp == e
        h2, dy2, dz2 = pr["h"][sel] ** 2, pr["dy"][sel] ** 2, pr["dz"][sel] ** 2
        rss["dw2"][e] = h2.T @ dy2
        rss["dw1"][e] = x2[tok[sel]].T @ dz2
        rss["db2"][e] = dy2.sum(0)
        rss["db1"][e] = dz2.sum(0)
        np.add.at(rss["dx"], tok[sel], dz2 @ (wd.w1e(e) ** 2).T)
    d = dout.detach().double().cpu().numpy() if hasattr(dout, "detach") else np.asarray(dout, np.float64)
    where = (tok, pr["slot"]) if score == "dtopk_w" else pr["entry"]
    rss[score][where] = (pr["y"] ** 2 * d[tok] ** 2).sum(1)
    return {k: np.sqrt(v) for k, v in rss.items()}


def assert_close_bwd(gpu, ref, rss, what=""):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    bound = RTOL * np.abs(ref) + ATOL_RMS * rms + BWD_RSS_FACTOR * BWD_ULP * rss
    err = np.abs(gpu - ref)
    bad = ~(err <= bound)
    assert not bad.any(), (f"{what}: max_err {err.max():.4g}, rms {rms:.4g}, n_bad {int(bad.sum())}/{err.size}, "
                           f"worst {np.unravel_index(int(np.argmax(err - bound)), err.shape)}")


def tile_rows(off, tile=256):
    """Expert-sorted rows to compare for every (expert, tile-row m-tile) of a
    run, from the expert offsets [E+1]: each tile's first and last stored row
    and the rows on both sides of the CTA-pair splits (64 and 128 rows into
    the tile), so every m-tile -- tail tiles of at most 128 rows included -- and
    every segment end is checked."""
    off = np.asarray(off, dtype=np.int64)
    rows = []
    for e in range(off.shape[0] - 1):
        a, b = int(off[e]), int(off[e + 1])
        for t0 in range(a, b, tile):
            t1 = min(t0 + tile, b)
            for r in (t0, t0 + 63, t0 + 64, t0 + 127, t0 + 128, t1 - 1):
                if t0 <= r < t1:
                    rows.append(r)
    return np.unique(np.asarray(rows, dtype=np.int64))
