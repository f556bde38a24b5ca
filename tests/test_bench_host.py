"""Host-side pieces of bench.py and the expert-parallel host module, on CPU:
the DRAM-traffic record file, its use only while the kernel sources hash to
it (checked on a copy of the sources), the roofline arithmetic, the clocks
record of the timed region, and the receive-block offsets against the
oracle's."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from mixture_experts_routed_non_b200.ep import block_offsets  # noqa: E402
from oracle import ep as oep  # noqa: E402


def test_traffic_record_file_parses():
    """Every record names a kernel, a workload, a 16-hex-digit source hash and
    read + write = per-launch bytes."""
    n = 0
    for line in open(os.path.join(ROOT, "profiles", "ncu_traffic.txt")):
        if line.startswith("#") or not line.strip():
            continue
        kv = dict(p.split("=", 1) for p in line.split())
        assert kv["kernel"] in ("gemm_up", "gemm_down") and kv["workload"]
        assert len(kv["sources"]) == 16 and int(kv["sources"], 16) >= 0
        assert int(kv["read"]) + int(kv["write"]) == int(kv["dram_bytes_per_launch"])
        n += 1
    assert n >= 2
    assert bench.traffic_record("gemm_up", "no-such-workload") is None


def test_traffic_record_rejects_changed_sources(tmp_path, monkeypatch):
    """A record is used only while the kernel sources hash to it: a copy of the
    sources with a record written for them finds it; one byte more, and not."""
    import hashlib
    import shutil
    root = tmp_path / "repo"
    (root / "profiles").mkdir(parents=True)
    csrc = root / "mixture_experts_routed_non_b200" / "csrc"
    csrc.mkdir(parents=True)
    h = hashlib.sha256()
    for f in ("grouped_gemm_sm100.cu", "common.cuh"):
        shutil.copy(os.path.join(ROOT, "mixture_experts_routed_non_b200", "csrc", f), csrc / f)
        h.update(open(csrc / f, "rb").read())
    with open(root / "profiles" / "ncu_traffic.txt", "w") as fh:
        fh.write(f"kernel=gemm_up workload=prefill sources={h.hexdigest()[:16]} "
                 f"dram_bytes_per_launch=300 read=200 write=100\n")
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.traffic_record("gemm_up", "prefill") == 300.0
    with open(csrc / "common.cuh", "a") as fh:
        fh.write("\n")
    assert bench.traffic_record("gemm_up", "prefill") is None


def test_gemm_flops_and_peaks():
    up, down = bench.gemm_flops(131072, 2048, 768)
    assert up == 4 * 131072 * 2048 * 768 and down == 2 * 131072 * 2048 * 768
    peaks, src = bench.load_peaks()
    assert src in ("measured", "fallback")
    assert peaks["hbm_gbs"] > 1000 and peaks["bf16_tflops_sustained"] > 100


def test_block_offsets_match_the_oracle():
    rng = np.random.default_rng(0)
    for R in (1, 2, 5, 8, 32):
        counts = rng.integers(0, 50, size=(R, R))
        off, n = block_offsets(counts)
        ref_off, ref_n = oep.recv_offsets(counts)
        assert np.array_equal(off, ref_off) and np.array_equal(n, ref_n)


def test_clock_summary_window_median_and_reasons():
    """The clocks record of the timed region: samples outside the window and
    malformed lines are dropped; the SM clock is the median of the rest, and
    every throttle reason seen active in the window is listed."""
    s = bench.ClockSampler(0)
    na = "Not Active"
    s.lines = [
        (0.5, f"1965, 1965, 300.0, 0x0, {na}, {na}, {na}, {na}"),            # before the window
        (1.0, f"1500, 1965, 990.0, 0x4, {na}, {na}, {na}, Active"),
        (1.1, f"1400, 1965, 1000.0, 0x4, {na}, {na}, {na}, Active"),
        (1.2, "garbage"),
        (1.3, f"[N/A], 1965, 1000.0, 0x4, {na}, {na}, {na}, Active"),          # unreadable clock
        (1.4, f"1300, 1965, 1000.0, 0x44, {na}, Active, {na}, Active"),
        (3.0, f"900, 1965, 1000.0, 0x8, Active, {na}, {na}, {na}"),          # after the window
    ]
    out = s.summary(0.9, 2.0)
    assert out["sm_mhz"] == 1400.0 and out["sm_max_mhz"] == 1965.0 and out["samples"] == 3
    assert out["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    assert bench.ClockSampler(0).summary(0.0, 1.0) == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [],
                                                        "samples": 0}


def test_tensor_peak_follows_the_clock_record():
    """Burst for a short timed region or one without the power cap; the
    sustained figure only for a region of seconds whose samples show the cap."""
    peaks = {"hbm_gbs": 6500.0, "bf16_tflops": 1677.6, "bf16_tflops_sustained": 1391.2}
    capped = {"reasons": ["sw_power_cap"], "sm_mhz": 1350.0, "sm_max_mhz": 1965.0, "samples": 40}
    free = {"reasons": [], "sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "samples": 40}
    assert bench.choose_tensor_peak(peaks, free, 0.023) == (1677.6, "burst")
    assert bench.choose_tensor_peak(peaks, capped, 0.023) == (1677.6, "burst")
    assert bench.choose_tensor_peak(peaks, free, 5.0) == (1677.6, "burst")
    assert bench.choose_tensor_peak(peaks, capped, 5.0) == (1391.2, "sustained")
    assert bench.choose_tensor_peak(peaks, {"reasons": [], "samples": 0}, 0.02) == (1677.6, "burst")


def test_clock_record_widens_to_the_leg_when_the_region_is_short():
    s = bench.ClockSampler(0)
    na = "Not Active"
    s.lines = [(1.00, f"1965, 1965, 500.0, 0x0, {na}, {na}, {na}, {na}"),
               (1.02, f"1950, 1965, 600.0, 0x0, {na}, {na}, {na}, {na}"),
               (1.30, f"1965, 1965, 700.0, 0x0, {na}, {na}, {na}, {na}")]
    c = bench.clocks_for(s, 1.05, 1.07, 0.9, 1.4)          # no sample inside the 20 ms region
    assert c["window"].startswith("forward leg") and c["samples"] == 3 and c["sm_mhz"] == 1965.0
    c = bench.clocks_for(s, 1.01, 1.03, 0.9, 1.4)
    assert c["window"] == "timed region" and c["samples"] == 1 and c["sm_mhz"] == 1950.0


def _bench_lines(args, timeout=300):
    import json
    import subprocess
    env = dict(os.environ)
    env.pop("WORLD_SIZE", None)
    env.pop("RANK", None)
    env.pop("LOCAL_RANK", None)
    env.setdefault("OMP_NUM_THREADS", "1")
    r = subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=timeout)
    assert r.returncode == 0, r.stderr[-3000:]
    return [json.loads(ln) for ln in r.stdout.splitlines() if ln.startswith("{")]


def test_gpus_flag_launches_that_many_ranks():
    """`bench.py --gpus 2` run without a launcher starts two ranks itself
    (torch.distributed.run, 127.0.0.1); each rank sees WORLD_SIZE 2."""
    for impl in ("ours", "reference"):
        lines = _bench_lines(["--gpus", "2", "--check-launch", "--impl", impl])
        assert sorted(d["rank"] for d in lines) == [0, 1]
        assert all(d["world"] == 2 and d["impl"] == impl for d in lines)


def test_reference_arm_reports_the_ranks_it_ran():
    lines = _bench_lines(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0",
                          "--workload", "tiny", "--ref-seconds", "0.05"])
    assert len(lines) == 1 and lines[0]["n_gpus"] == 2 and lines[0]["impl"] == "reference"


def test_both_arms_share_one_config_object():
    """The reference arm's config is built by the same function as ours, from
    the same workload, so the two lines name the same configuration."""
    import torch  # noqa: F401
    from mixture_experts_routed_non_b200 import synthetic
    wl = synthetic.WORKLOADS["tiny"]
    inp = synthetic.make_inputs(wl, device="cpu")
    P = int((inp.topk_idx >= 0).sum())
    lines = _bench_lines(["--impl", "reference", "--steps", "1", "--warmup", "0", "--workload", "tiny",
                          "--ref-seconds", "0.05"])
    assert lines[0]["config"] == bench.bench_config(wl, 0, 1, P, (inp.w1.numel() + inp.w2.numel()) * 2)
