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
