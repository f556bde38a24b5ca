"""Benchmark of the local MoE expert forward on the non-expand routed layout.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload prefill] [--layout 0|1]

One step = one moe_nonexpand_forward (metadata, grouped GEMM up + SwiGLU,
grouped GEMM down, combine) over one batch of seeded synthetic inputs of the
named workload, inputs resident in HBM.  Prints one JSON line on rank 0.

Multi-GPU (torchrun, one process per GPU): every rank runs its own replica on
its own token batch (the path has no exchange step), so scaling is weak and
the value is all ranks' tokens divided by the slowest rank's time.

--impl reference times the CPU oracle (the only reference this method has)
on the host cores, on a bounded token sample per step, rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE fwd tokens/sec and grouped-GEMM TFLOP/s (% bf16 peak) on 1 B200"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(value: float, device, world: int) -> float:
    """The largest of every rank's `value` (a device-timed duration); every
    rank calls it at the same point, so the collective order stays the same on
    all ranks.  With one rank it returns `value` unchanged."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int, interval_ms: int = 20):
        self.device_index = device_index
        self.interval_ms = interval_ms
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.device_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", str(self.interval_ms)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)

    def summary(self, t0: float, t1: float):
        rows = []
        for ts, line in self.lines:
            if not (t0 <= ts <= t1):
                continue
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                rows.append(dict(sm=float(parts[0]), max=float(parts[1]), active=parts[3],
                                 hw=parts[4], hwt=parts[5], swt=parts[6], pcap=parts[7]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in rows),
                "sm_max_mhz": max(r["max"] for r in rows), "reasons": sorted(reasons),
                "samples": len(rows)}


# ---------------------------------------------------------------------------
# roofline bookkeeping
# ---------------------------------------------------------------------------
def gemm_flops(P: int, H: int, I: int):
    return 4.0 * P * H * I, 2.0 * P * H * I


def choose_tensor_peak(peaks, clocks, timed_s: float):
    """The bf16 peak a GEMM timed inside a region of ``timed_s`` seconds is
    held to: the burst figure (a short region runs at full clock) unless the
    region lasts seconds and its clock record shows the power cap, in which
    case the sustained figure.  Returns (TFLOP/s, label)."""
    capped = "sw_power_cap" in (clocks or {}).get("reasons", [])
    if timed_s >= 1.0 and capped:
        return peaks["bf16_tflops_sustained"], "sustained"
    return peaks["bf16_tflops"], "burst"


def clocks_for(sampler, t0: float, t1: float, leg0: float, leg1: float):
    """The clock record of the timed region [t0, t1]; when the region is
    shorter than the sampling interval and holds no sample, that of the whole
    forward leg [leg0, leg1] (warm-up, timed steps and end-to-end steps, the
    same kernels back to back), with the window named."""
    c = sampler.summary(t0, t1)
    c["window"] = "timed region"
    if c["samples"] == 0:
        c = sampler.summary(leg0, leg1)
        c["window"] = "forward leg (timed region shorter than the sampling interval)"
    c["interval_ms"] = sampler.interval_ms
    return c


def algorithmic_bytes(inp, P: int, freq):
    """x read once + the weights of experts with at least one pair + routing
    tensors + out written."""
    wl = inp.wl
    active = int((freq > 0).sum())
    per_expert = (wl.H * 2 * wl.I + wl.I * wl.H) * 2
    return wl.N * wl.H * 2 + active * per_expert + wl.N * wl.K * 8 + wl.N * wl.H * 2


def traffic_record(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` from a committed ncu summary, valid
    only while the kernel's sources are unchanged (else None)."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if not os.path.exists(path):
        return None
    srcs = ["mixture_experts_routed_non_b200/csrc/grouped_gemm_sm100.cu",
            "mixture_experts_routed_non_b200/csrc/common.cuh"]
    h = hashlib.sha256()
    for s in srcs:
        with open(os.path.join(ROOT, s), "rb") as f:
            h.update(f.read())
    digest = h.hexdigest()[:16]
    with open(path) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            kv = dict(p.split("=", 1) for p in line.split() if "=" in p)
            if (kv.get("kernel") == kernel and kv.get("workload") == workload
                    and kv.get("sources") == digest):
                return float(kv["dram_bytes_per_launch"])
    return None


# ---------------------------------------------------------------------------
# CPU oracle legs
# ---------------------------------------------------------------------------
def oracle_tokens_per_s(inp, target_s: float, rng_seed: int = 123, max_tokens=None):
    """Time the oracle on a seeded token sample sized for about target_s of
    wall time.  Returns (tokens/s, tokens, seconds, threads)."""
    import numpy as np

    import oracle
    wts = oracle.Weights(inp.x, inp.w1, inp.b1, inp.w2, inp.b2)
    idx = inp.topk_idx.cpu().numpy()
    w = inp.topk_w.cpu().numpy()
    threads = len(os.sched_getaffinity(0))
    rng = np.random.default_rng(rng_seed)
    N = inp.wl.N
    n = min(N, 8)
    oracle.forward_rows(wts, idx, w, tokens=np.arange(min(N, 2)), n_threads=threads)  # load + warm
    while True:
        toks = np.sort(rng.choice(N, size=n, replace=False))
        t0 = time.perf_counter()
        oracle.forward_rows(wts, idx, w, tokens=toks, n_threads=threads)
        dt = time.perf_counter() - t0
        if dt >= target_s * 0.5 or n >= N or (max_tokens and n >= max_tokens):
            return n / dt, n, dt, threads
        grow = max(2.0, min(16.0, target_s / max(dt, 1e-3)))
        n = min(N, int(n * grow) + 1)
        if max_tokens:
            n = min(n, max_tokens)


# ---------------------------------------------------------------------------
def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="prefill")
    ap.add_argument("--layout", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true", help="skip the other configured workloads")
    ap.add_argument("--only", choices=["forward", "train", "metadata", "router"], default=None,
                    help="profiler runs: time only the forward of --workload, only its training step "
                         "(forward_train + backward), only the metadata on the metadata workload, or "
                         "only the router top-k on the prefill sizes")
    ap.add_argument("--check-launch", action="store_true",
                    help="every rank prints its rank and world size and exits (checks the --gpus launch)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-seconds", type=float, default=6.0,
                    help="at most this much oracle work per step of --impl reference (sets its token sample)")
    ap.add_argument("--ref-budget", type=float, default=150.0,
                    help="oracle work of the whole --impl reference run, spread over its warm-up and timed steps")
    return ap.parse_args()


def metadata_only(dev, peaks, reps: int = 50):
    """moe_nonexpand_metadata alone on the metadata workload (N=65536, K=8,
    E=128, Zipf routing), L2 flushed before every rep; median device time."""
    import numpy as np
    import torch

    from mixture_experts_routed_non_b200 import binding, synthetic
    wl = synthetic.WORKLOADS["metadata"]
    idx, w = synthetic.make_routing(wl)
    ti = torch.from_numpy(idx).to(dev)
    tw = torch.from_numpy(w).to(dev)
    P = int((idx >= 0).sum())
    ws = binding.alloc_workspace(wl.N, 0, 0, wl.E, wl.K, -1, dev)
    meta = binding.alloc_meta(wl.N, wl.K, wl.E, -1, dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(3):
        binding.metadata(ti, tw, wl.E, meta=meta, ws=ws)
    times = []
    for _ in range(reps):
        flush.zero_()
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record()
        binding.metadata(ti, tw, wl.E, meta=meta, ws=ws)
        e.record()
        e.synchronize()
        times.append(s.elapsed_time(e))
    ms = float(np.median(times))
    nbytes = wl.N * wl.K * 8 + 4 * P * 4 + 4 * (wl.N + 1) + 8 * wl.E
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"workload": "metadata", "N": wl.N, "K": wl.K, "E": wl.E, "P": P, "ms": ms,
            "algorithmic_bytes": nbytes, "gbs": gbs, "frac_hbm": gbs / peaks["hbm_gbs"],
            "launches": 1, "l2": "flushed before every rep"}


def metadata_pairs_only(dev, peaks, reps: int = 50):
    """moe_nonexpand_routed_metadata on the metadata workload given as the
    compact pair list (token / expert / score per pair, tokens ascending),
    with int32 and with int64 ids; L2 flushed before every rep, median device
    time.  The pair-list read replaces the table's N*K slots by P pairs."""
    import numpy as np
    import torch

    from mixture_experts_routed_non_b200 import binding, synthetic
    wl = synthetic.WORKLOADS["metadata"]
    idx, w = synthetic.make_routing(wl)
    tok, exp, wt = synthetic.pair_list_from_table(idx, w)
    P = int(tok.shape[0])
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    res = {"workload": "metadata (pair list)", "N": wl.N, "E": wl.E, "P": P, "l2": "flushed before every rep"}
    for bits, dt in ((32, torch.int32), (64, torch.int64)):
        t_ = torch.from_numpy(tok).to(dt).to(dev)
        e_ = torch.from_numpy(exp).to(dt).to(dev)
        w_ = torch.from_numpy(wt).to(dev)
        r = binding.routing(e_, w_, token_idx=t_, N=wl.N)
        meta = binding.alloc_routed_meta(r, wl.E, dev)
        ws = torch.empty(binding.routed_workspace_bytes(r, 0, 0, wl.E), dtype=torch.uint8, device=dev)
        for _ in range(3):
            binding.routed_metadata(e_, w_, wl.E, token_idx=t_, N=wl.N, meta=meta, ws=ws)
        times = []
        for _ in range(reps):
            flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            binding.routed_metadata(e_, w_, wl.E, token_idx=t_, N=wl.N, meta=meta, ws=ws)
            b.record()
            b.synchronize()
            times.append(a.elapsed_time(b))
        ms = float(np.median(times))
        nbytes = P * (2 * (bits // 8) + 4) + 4 * P * 4 + 4 * (wl.N + 1) + 8 * wl.E
        res[f"int{bits}"] = {"ms": ms, "algorithmic_bytes": nbytes, "gbs": nbytes / (ms * 1e-3) / 1e9}
    return res


def router_only(dev, peaks, reps: int = 10, ring: int = 20):
    """moe_router_topk alone on the prefill sizes (N=16384, E=128, K=8, fp32
    logits, top-k of the softmax renormalised).  A ring of ``ring`` logits
    buffers (168 MB, more than L2) is routed by one CUDA graph of ``ring``
    launches, so every launch reads from HBM and no host call sits between
    launches; device time per launch, median over ``reps`` replays."""
    import numpy as np
    import torch

    from mixture_experts_routed_non_b200 import binding, synthetic
    N, E, K = 16384, 128, 8
    base = synthetic.make_logits(N, E, seed=1, device=dev)
    bufs = [base.clone() for _ in range(ring)]
    idx = torch.empty((N, K), dtype=torch.int32, device=dev)
    w = torch.empty((N, K), dtype=torch.float32, device=dev)
    mode = binding.ROUTER_TOPK_SOFTMAX_RENORM
    for b in bufs[:3]:
        binding.router_topk(b, K, mode, idx, w)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    cs = torch.cuda.Stream()
    cs.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cs):
        with torch.cuda.graph(g, stream=cs):
            for b in bufs:
                binding.router_topk(b, K, mode, idx, w, stream=cs)
    torch.cuda.current_stream().wait_stream(cs)
    busy = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    g.replay()
    times = []
    for _ in range(reps):
        busy.zero_()  # keeps the GPU busy while the host enqueues the replay
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record()
        g.replay()
        e.record()
        e.synchronize()
        times.append(s.elapsed_time(e) / ring)
    del g
    ms = float(np.median(times))
    nbytes = N * E * 4 + N * K * 8
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"N": N, "E": E, "K": K, "logits": "fp32", "mode": "topk(softmax)+renorm", "ms": ms,
            "algorithmic_bytes": nbytes, "gbs": gbs, "frac_hbm": gbs / peaks["hbm_gbs"], "launches": 1,
            "l2": f"ring of {ring} logits buffers ({ring * N * E * 4 / 1e6:.0f} MB) in one graph"}


def ep_emulated(dev, peaks, reps: int = 20):
    """Expert-parallel dispatch and combine with 8 ranks emulated on this GPU,
    sized like the rank-local shape after 8-way dispatch (H=7168, 32 local
    experts per rank, K=8 global slots, ~8192 receive rows per rank): 1560
    tokens per source rank.  Device time of the eight dispatch launches and
    of the eight combine launches (median over ``reps``).  Emulated ranks
    move rows HBM to HBM; across GPUs the same stores and loads cross NVLink.
    Algorithmic bytes: dispatch reads x once per source row and writes each
    receive row (x, ids, weights); combine reads each receive row and writes
    the routed rows."""
    import numpy as np
    import torch

    from mixture_experts_routed_non_b200 import binding
    from mixture_experts_routed_non_b200.ep import EmulatedRanks
    R, E_local, T, K, H = 8, 32, 1560, 8, 7168
    g = torch.Generator(device=dev).manual_seed(3)
    xs = [torch.randn((T, H), generator=g, device=dev).to(torch.bfloat16) for _ in range(R)]
    idxs = [torch.argsort(torch.rand((T, R * E_local), generator=g, device=dev), dim=1)[:, :K].to(torch.int32)
            .contiguous() for _ in range(R)]
    ws = [torch.rand((T, K), generator=g, device=dev) for _ in range(R)]
    er = EmulatedRanks(R, E_local, dev)
    st = er.dispatch(xs, idxs, ws)
    recv_x, recv_idx, recv_w = st["_bufs"]
    peers = [binding.ep_peers(recv_x, recv_idx, recv_w, st["off"][:, s]) for s in range(R)]
    local = [t.clone() for t in st["recv_x"]]
    srcs = [binding.ep_sources(local, st["off"][:, s]) for s in range(R)]
    outs = [torch.empty((T, H), dtype=torch.bfloat16, device=dev) for _ in range(R)]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def timed(fn):
        # the eight launches of a phase as one CUDA graph, so that host calls do
        # not sit between them; the L2 flush runs before each replay
        fn()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        cs = torch.cuda.Stream()
        cs.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(cs):
            with torch.cuda.graph(graph, stream=cs):
                fn()
        torch.cuda.current_stream().wait_stream(cs)
        times = []
        for i in range(reps + 3):
            flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            graph.replay()
            b.record()
            b.synchronize()
            if i >= 3:
                times.append(a.elapsed_time(b))
        del graph
        return float(np.median(times))

    def dispatch():
        for s in range(R):
            binding.ep_dispatch(xs[s], idxs[s], ws[s], st["send_idx"][s], E_local, peers[s], R)

    def combine():
        for s in range(R):
            binding.ep_combine(srcs[s], st["send_idx"][s], H, out=outs[s])

    def layout():
        for s in range(R):
            binding.ep_layout(idxs[s], R, E_local, send_idx=st["send_idx"][s])

    ms_d, ms_c, ms_l = timed(dispatch), timed(combine), timed(layout)
    rows = int(st["n_recv"].sum())
    b_d = R * T * H * 2 + rows * (H * 2 + K * 8)
    b_c = rows * H * 2 + R * T * H * 2
    return {"ranks": R, "E_local": E_local, "tokens_per_rank": T, "K": K, "H": H,
            "recv_rows_per_rank": float(rows / R), "layout_ms": ms_l,
            "dispatch_ms": ms_d, "dispatch_gbs": b_d / (ms_d * 1e-3) / 1e9,
            "combine_ms": ms_c, "combine_gbs": b_c / (ms_c * 1e-3) / 1e9,
            "frac_hbm": {"dispatch": b_d / (ms_d * 1e-3) / 1e9 / peaks["hbm_gbs"],
                         "combine": b_c / (ms_c * 1e-3) / 1e9 / peaks["hbm_gbs"]},
            "launches": {"layout": R, "dispatch": R, "combine": R},
            "note": "8 ranks emulated on one GPU (HBM to HBM); each phase's 8 launches replayed as one CUDA graph, "
                    "L2 flushed before each replay"}


def backward_leg(inp, w1, b1, layout, dev, peaks, peak_tf, peak_label, steps: int = 30, warmup: int = 3):
    """One training step, forward_train + backward, on the bench workload:
    mean device time per step with the backward's seven stages timed by
    events on the launching stream.  Inputs are larger than L2 (1.2 GB of
    expert weights and their gradients per step)."""
    import numpy as np
    import torch

    from mixture_experts_routed_non_b200 import binding
    wl = inp.wl
    N, H, I, E, K = wl.N, wl.H, wl.I, wl.E, wl.K
    ws = binding.alloc_train_workspace(N, H, I, E, K, -1, dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(77)
    dout = torch.randn((N, H), generator=gen, device=dev).to(torch.bfloat16)
    out = torch.empty(N, H, dtype=torch.bfloat16, device=dev)
    grads = None
    fev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    bev = [[torch.cuda.Event(enable_timing=True) for _ in range(8)] for _ in range(steps)]
    bias = b1 is not None
    for i in range(warmup + steps):
        j = i - warmup
        if j >= 0:
            fev[j][0].record()
        binding.forward_train(inp.x, inp.topk_idx, inp.topk_w, w1, inp.w2, b1, inp.b2, ws=ws, layout=layout,
                              out=out)
        if j >= 0:
            fev[j][1].record()
        grads = binding.backward(dout, inp.x, inp.topk_idx, inp.topk_w, w1, inp.w2, ws=ws, layout=layout,
                                 bias_grads=bias, grads=grads, events=bev[j] if j >= 0 else None)
    torch.cuda.synchronize(dev)
    if binding.read_error(ws):
        raise SystemExit("bench.py: device error in the backward")
    P = int((inp.topk_idx >= 0).sum().item())
    fwd = float(np.mean([a.elapsed_time(b) for a, b in fev]))
    st = np.mean([[e[k].elapsed_time(e[k + 1]) for k in range(7)] for e in bev], axis=0)
    names = ["prep", "dh", "dw2", "dw1", "dx", "combine", "bias"]  # dw1 includes gathering x rows
    phi = P * H * I
    flops = {"dh": 2 * phi, "dw2": 2 * phi, "dx": 4 * phi, "dw1": 4 * phi}
    tf = {k: flops[k] / (st[names.index(k)] * 1e-3) / 1e12 for k in flops}
    gemm_ms = float(sum(st[names.index(k)] for k in flops))
    bwd_ms = float(st.sum())
    dom = max(flops, key=lambda k: st[names.index(k)])
    peak = peak_tf
    prep_bytes = 2 * P * H * 2 + N * H * 2  # y read, dy written, dout read
    del ws
    return {"workload": wl.name, "steps": steps, "train_step_ms": fwd + bwd_ms,
            "tokens_per_s": N / ((fwd + bwd_ms) * 1e-3), "forward_train_ms": fwd, "backward_ms": bwd_ms,
            "stages_ms": dict(zip(names, [float(v) for v in st])),
            "gemm_tflops": {k: float(v) for k, v in tf.items()},
            "bwd_gemm_tflops": 12 * phi / (gemm_ms * 1e-3) / 1e12,
            "bwd_gemm_frac_of_peak": 12 * phi / (gemm_ms * 1e-3) / 1e12 / peak,
            "prep_gbs": prep_bytes / (st[0] * 1e-3) / 1e9,
            "dominant": {"kernel": f"backward grouped GEMM {dom}", "tflops": float(tf[dom]), "peak": peak,
                         "frac": float(tf[dom] / peak), "peak_source": f"bf16 {peak_label}"},
            "gemm_frac_of_peak": {k: float(v / peak) for k, v in tf.items()}}


def bench_config(wl, layout: int, world: int, P: int, w_bytes: int):
    """The ``config`` object of the JSON line, the same for both arms."""
    return {"workload": wl.name, "N": wl.N, "H": wl.H, "I": wl.I, "E": wl.E, "K": wl.K, "P": P,
            "layout": "interleaved" if layout == 0 else "concatenated",
            "routing": wl.description, "parallelism": f"replicas x{world} (token shards)",
            "l2": "inputs larger than L2 (expert weights %.2f GB per step)" % (w_bytes / 1e9)}


def run_reference(args, rank, world):
    """The reference arm: the CPU oracle as it stands, rank 0 only."""
    if rank != 0:
        return
    import torch  # noqa: F401
    from mixture_experts_routed_non_b200 import synthetic
    wl = synthetic.WORKLOADS[args.workload]
    inp = synthetic.make_inputs(wl, device="cpu")
    import numpy as np

    import oracle
    wts = oracle.Weights(inp.x, inp.w1, inp.b1, inp.w2, inp.b2)
    idx = inp.topk_idx.numpy()
    w = inp.topk_w.numpy()
    threads = len(os.sched_getaffinity(0))
    # sample size per step: about --ref-seconds of oracle work, less when the whole run
    # (warm-up and timed steps) would exceed --ref-budget
    per_step_s = min(args.ref_seconds, args.ref_budget / max(1, args.warmup + args.steps))
    probe = np.arange(min(wl.N, 4))
    t0 = time.perf_counter()
    oracle.forward_rows(wts, idx, w, tokens=probe, layout=args.layout, n_threads=threads)
    per_tok = (time.perf_counter() - t0) / len(probe)
    n = int(max(1, min(wl.N, per_step_s / max(per_tok, 1e-6))))
    rng = np.random.default_rng(7)
    times = []
    for step in range(args.warmup + args.steps):
        toks = np.sort(rng.choice(wl.N, size=n, replace=False))
        t0 = time.perf_counter()
        oracle.forward_rows(wts, idx, w, tokens=toks, layout=args.layout, n_threads=threads)
        dt = time.perf_counter() - t0
        if step >= args.warmup:
            times.append(dt)
    total = sum(times)
    value = n * len(times) / total
    P = int((idx >= 0).sum())
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * total / len(times), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(wl, args.layout, world, P, (inp.w1.numel() + inp.w2.numel()) * 2),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": f"{n} seeded tokens of the {wl.name} workload per step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def timed_forwards(step, steps: int, stream, dev):
    """``steps`` back-to-back forwards as a caller runs them (no events between
    the launches, so each kernel after the metadata starts as a programmatic
    dependent of the one before); returns their elapsed device ms."""
    import torch
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    start.record(stream)
    for _ in range(steps):
        step()
    end.record(stream)
    torch.cuda.synchronize(dev)
    return start.elapsed_time(end)


def stage_forwards(step, steps: int, dev):
    """``steps`` more forwards, each with its five stage events on the
    launching stream (the events sit between the launches, which then run
    one after the other); returns the mean ms of the four stages."""
    import numpy as np
    import torch
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    torch.cuda.synchronize(dev)
    for i in range(steps):
        step(ev[i])
    torch.cuda.synchronize(dev)
    stage_ms = np.zeros(4)
    for e in ev:
        for j in range(4):
            stage_ms[j] += e[j].elapsed_time(e[j + 1])
    return stage_ms / steps


def graph_forward_ms(step, steps: int, dev):
    """One forward captured in a CUDA graph and replayed ``steps`` times back
    to back: device ms per replay (the launch sequence without host calls)."""
    import torch
    g = torch.cuda.CUDAGraph()
    cs = torch.cuda.Stream(dev)
    cs.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(cs):
        step(None, cs)
        torch.cuda.synchronize(dev)
        with torch.cuda.graph(g, stream=cs):
            step(None, cs)
    torch.cuda.current_stream(dev).wait_stream(cs)
    g.replay()
    torch.cuda.synchronize(dev)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        g.replay()
    b.record()
    b.synchronize()
    ms = a.elapsed_time(b) / steps
    del g
    return ms


def forward_summary(wl, P, freq, inp, stage_ms, ms_per_step, peaks, peak_tf, peak_label):
    """Per-stage rates and roofline fractions of one workload's forward."""
    H, I, N, K, E = wl.H, wl.I, wl.N, wl.K, wl.E
    up_flops, down_flops = gemm_flops(P, H, I)
    up_tf = up_flops / (stage_ms[1] * 1e-3) / 1e12 if stage_ms[1] > 0 else 0.0
    down_tf = down_flops / (stage_ms[2] * 1e-3) / 1e12 if stage_ms[2] > 0 else 0.0
    # the combine reads each pair's fp16 row (2 bytes per element) and its
    # exponents (one byte per 32 elements), writes the bf16 output
    comb_bytes = P * H * 2 + P * (H // 32) + N * H * 2 + (N + 1) * 4 + P * 8
    meta_bytes = N * K * 8 + 4 * P * 4 + 4 * (N + 1) + 8 * E
    alg_bytes = algorithmic_bytes(inp, P, freq)
    t_tensor = (up_flops + down_flops) / (peak_tf * 1e12)
    t_hbm = alg_bytes / (peaks["hbm_gbs"] * 1e9)
    return {
        "stages_ms": {"metadata": float(stage_ms[0]), "gemm_up": float(stage_ms[1]),
                      "gemm_down": float(stage_ms[2]), "combine": float(stage_ms[3])},
        "gemm_up_tflops": up_tf, "gemm_down_tflops": down_tf,
        "gemm_up_frac": up_tf / peak_tf, "gemm_down_frac": down_tf / peak_tf,
        "gemm_up_frac_of_burst": up_tf / peaks["bf16_tflops"],
        "gemm_down_frac_of_burst": down_tf / peaks["bf16_tflops"],
        "gemm_peak": {"tflops": peak_tf, "kind": peak_label},
        "combine_gbs": comb_bytes / (stage_ms[3] * 1e-3) / 1e9,
        "combine_frac_hbm": comb_bytes / (stage_ms[3] * 1e-3) / 1e9 / peaks["hbm_gbs"],
        "metadata_gbs": meta_bytes / (stage_ms[0] * 1e-3) / 1e9,
        "algorithmic_bytes": alg_bytes, "flops": up_flops + down_flops,
        "step_roofline_ms": max(t_tensor, t_hbm) * 1e3,
        "step_bound": "tensor" if t_tensor >= t_hbm else "hbm",
        "step_frac_of_roofline": max(t_tensor, t_hbm) * 1e3 / ms_per_step,
    }


def workload_leg(name: str, dev, peaks, peak_tf, peak_label, steps: int, warmup: int):
    """One configured workload timed like the headline one (interleaved
    layout): ``steps`` back-to-back forwards after ``warmup`` untimed ones,
    stage events on the launching stream, plus the CUDA-graph time."""
    import torch

    from mixture_experts_routed_non_b200 import binding, synthetic
    wl = synthetic.WORKLOADS[name]
    inp = synthetic.make_inputs(wl, device=dev)
    ws = binding.alloc_workspace(wl.N, wl.H, wl.I, wl.E, wl.K, -1, dev)
    out = torch.empty(wl.N, wl.H, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(events=None, s=None):
        binding.forward(inp.x, inp.topk_idx, inp.topk_w, inp.w1, inp.w2, inp.b1, inp.b2, out=out, ws=ws,
                        events=events, stream=s)

    for _ in range(max(3, warmup)):
        step()
    torch.cuda.synchronize(dev)
    if binding.read_error(ws):
        raise SystemExit(f"bench.py: device error in workload {name}")
    freq = binding.meta_from_workspace(ws, wl.N, wl.H, wl.I, wl.E, wl.K)["expert_frequency"].cpu().numpy()
    P = int(freq.sum())
    elapsed = timed_forwards(step, steps, stream, dev)
    stage_ms = stage_forwards(step, steps, dev)
    ms = elapsed / steps
    g_ms = graph_forward_ms(step, steps, dev)
    res = {"N": wl.N, "H": wl.H, "I": wl.I, "E": wl.E, "K": wl.K, "P": P, "routing": wl.description,
           "steps": steps, "warmup": max(3, warmup), "ms_per_step": ms, "tokens_per_s": wl.N / (ms * 1e-3),
           "graph_ms_per_step": g_ms, "graph_tokens_per_s": wl.N / (g_ms * 1e-3),
           "active_experts": int((freq > 0).sum())}
    res.update(forward_summary(wl, P, freq, inp, stage_ms, ms, peaks, peak_tf, peak_label))
    if res["step_bound"] == "hbm":
        res["note"] = "weight-read bound: step_frac_of_roofline is the algorithmic bytes at the copy bandwidth"
    del inp, ws, out
    torch.cuda.empty_cache()
    return res


def run_ours(args, rank, world, local):
    import numpy as np
    import torch
    import torch.distributed as dist

    from mixture_experts_routed_non_b200 import binding, synthetic

    if not torch.cuda.is_available():
        raise SystemExit("bench.py: no CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    peaks, peaks_src = load_peaks()
    if args.only in ("train", "metadata", "router"):
        if rank == 0:
            if args.only == "router":
                print(json.dumps({"only": "router", "router_only": router_only(dev, peaks, reps=args.steps)}),
                      flush=True)
            elif args.only == "metadata":
                print(json.dumps({"only": "metadata", "metadata_only": metadata_only(dev, peaks, reps=args.steps)}),
                      flush=True)
            else:
                wl = synthetic.WORKLOADS[args.workload]
                inp = synthetic.make_inputs(wl, device=dev)
                print(json.dumps({"only": "train", "training": backward_leg(
                    inp, inp.w1, inp.b1, 0, dev, peaks, peaks["bf16_tflops"], "burst", steps=args.steps,
                    warmup=max(1, args.warmup))}), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.2)
    t_leg0 = time.time()

    wl = synthetic.WORKLOADS[args.workload]
    inp = synthetic.make_inputs(wl, device=dev, seed=wl.seed + 1000 * rank)
    N, H, I, E, K = wl.N, wl.H, wl.I, wl.E, wl.K
    w1, b1 = inp.w1, inp.b1
    if args.layout == 1:
        w1 = torch.cat([w1[:, :, 0::2], w1[:, :, 1::2]], dim=2).contiguous()
        b1 = None if b1 is None else torch.cat([b1[:, 0::2], b1[:, 1::2]], dim=1).contiguous()
    ws = binding.alloc_workspace(N, H, I, E, K, -1, dev)
    out = torch.empty(N, H, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(events=None, s=None):
        binding.forward(inp.x, inp.topk_idx, inp.topk_w, w1, inp.w2, b1, inp.b2, layout=args.layout,
                        out=out, ws=ws, events=events, stream=s)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    err = binding.read_error(ws)
    if err:
        raise SystemExit(f"bench.py: device error word {err:#x}")
    meta = binding.meta_from_workspace(ws, N, H, I, E, K)
    freq = meta["expert_frequency"].cpu().numpy()
    P = int(freq.sum())

    # ---- timed region: K steps as a caller runs them
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    elapsed_ms = timed_forwards(step, args.steps, stream, dev)
    t_wall1 = time.time()
    if world > 1:
        dist.barrier()
    # the per-stage split, from K more steps with events between the launches
    stage_ms = stage_forwards(step, args.steps, dev)
    max_ms = max_over_ranks(elapsed_ms, dev, world)
    ms_per_step = max_ms / args.steps
    value = N * world * args.steps / (max_ms / 1000.0)
    if args.only == "forward":
        sampler.stop()
        if world > 1:
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
                              "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms_per_step,
                              "only": "forward", "stages_ms": [float(v) for v in stage_ms],
                              "config": bench_config(wl, args.layout, world, P,
                                                     (inp.w1.numel() + inp.w2.numel()) * 2)}), flush=True)
        return

    # ---- end to end: every step copies its inputs in from pinned host memory,
    # runs the forward and copies its result back out.  Steps are pipelined
    # over three streams (copy-in, compute, copy-out) with three buffer sets,
    # the way a serving loop overlaps PCIe with compute.  A step's inputs (x,
    # topk_idx, topk_w) sit in one pinned buffer and cross PCIe as one copy.
    nx, ni = inp.x.numel() * 2, inp.topk_idx.numel() * 4
    nw = inp.topk_w.numel() * 4
    packed_h = torch.empty(nx + ni + nw, dtype=torch.uint8).pin_memory()
    packed_h[:nx].copy_(inp.x.cpu().contiguous().view(torch.uint8).reshape(-1))
    packed_h[nx:nx + ni].copy_(inp.topk_idx.cpu().contiguous().view(torch.uint8).reshape(-1))
    packed_h[nx + ni:].copy_(inp.topk_w.cpu().contiguous().view(torch.uint8).reshape(-1))
    nbuf = 3
    outs_h = [torch.empty(N, H, dtype=torch.bfloat16).pin_memory() for _ in range(nbuf)]
    packed_d = [torch.empty(nx + ni + nw, dtype=torch.uint8, device=dev) for _ in range(nbuf)]
    xs_d = [b[:nx].view(torch.bfloat16).view(N, H) for b in packed_d]
    idxs_d = [b[nx:nx + ni].view(torch.int32).view(N, K) for b in packed_d]
    ws_d = [b[nx + ni:].view(torch.float32).view(N, K) for b in packed_d]
    outs_d = [torch.empty(N, H, dtype=torch.bfloat16, device=dev) for _ in range(nbuf)]
    s_in = torch.cuda.Stream(dev)
    s_cmp = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(nbuf)]
    ev_cmp = [torch.cuda.Event() for _ in range(nbuf)]
    ev_out = [torch.cuda.Event() for _ in range(nbuf)]
    # at least 100 steps: the three-stage pipeline's fill and drain (one copy each
    # way) are amortised as in a serving loop, which runs continuously
    e2e_steps = max(100, args.steps)

    def e2e_step(i):
        b = i % nbuf
        with torch.cuda.stream(s_in):
            if i >= nbuf:
                s_in.wait_event(ev_cmp[b])          # the forward of step i-nbuf is done with its inputs
            packed_d[b].copy_(packed_h, non_blocking=True)
            ev_in[b].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(ev_in[b])
            if i >= nbuf:
                s_cmp.wait_event(ev_out[b])         # step i-nbuf's result has been read out
            binding.forward(xs_d[b], idxs_d[b], ws_d[b], w1, inp.w2, b1, inp.b2, layout=args.layout,
                            out=outs_d[b], ws=ws, stream=s_cmp)
            ev_cmp[b].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_cmp[b])
            outs_h[b].copy_(outs_d[b], non_blocking=True)
            ev_out[b].record(s_out)

    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    s2 = torch.cuda.Event(enable_timing=True)
    e2 = torch.cuda.Event(enable_timing=True)
    s2.record(s_in)
    for i in range(e2e_steps):
        e2e_step(i)
    s_out.wait_stream(s_cmp)
    e2.record(s_out)
    torch.cuda.synchronize(dev)
    t_leg1 = time.time()
    e2e_ms = max_over_ranks(s2.elapsed_time(e2), dev, world)
    e2e_value = N * world * e2e_steps / (e2e_ms / 1000.0)
    h2d = nx + ni + nw
    d2h = outs_h[0].numel() * 2
    # the device result of the last step must equal the resident-input forward
    last = (e2e_steps - 1) % nbuf
    if not torch.equal(outs_h[last], out.cpu()):
        raise SystemExit("bench.py: end-to-end result differs from the device-resident forward")
    del packed_d, outs_d, xs_d, idxs_d, ws_d

    # ---- the same forward replayed from a CUDA graph (no host calls between launches)
    graph_ms = graph_forward_ms(step, args.steps, dev)

    # ---- roofline of the headline workload, against the peak its clock record supports
    time.sleep(0.1)
    clocks = clocks_for(sampler, t_wall0, t_wall1, t_leg0, t_leg1)
    peak_tf, peak_label = choose_tensor_peak(peaks, clocks, (t_wall1 - t_wall0))
    summ = forward_summary(wl, P, freq, inp, stage_ms, ms_per_step, peaks, peak_tf, peak_label)

    # ---- every other configured workload that has a forward, same timing rules
    workloads = {}
    if rank == 0 and not args.no_workloads:
        for name in ("ranklocal", "prefill256", "decode256", "tiny"):
            if name != wl.name:
                time.sleep(0.3)  # an idle gap: each leg starts from a cooled-down power state
                t0 = time.time()
                workloads[name] = workload_leg(name, dev, peaks, peak_tf, peak_label, args.steps, args.warmup)
                # the clock record of the whole leg (warm-up, timed, staged and graph forwards)
                workloads[name]["clocks"] = sampler.summary(t0, time.time())

    meta_c2 = metadata_only(dev, peaks) if rank == 0 else None
    meta_pairs = metadata_pairs_only(dev, peaks) if rank == 0 else None
    router = router_only(dev, peaks) if rank == 0 else None
    train = backward_leg(inp, w1, b1, args.layout, dev, peaks, peak_tf, peak_label) if rank == 0 else None
    ep = ep_emulated(dev, peaks) if rank == 0 else None
    sampler.stop()

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return

    cpu = None
    if not args.no_cpu_baseline and world == 1:
        tps, n_tok, secs, threads = oracle_tokens_per_s(inp, args.cpu_seconds)
        cpu = {"value": tps, "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "sample": f"{n_tok} seeded tokens of the {wl.name} workload ({secs:.1f} s of oracle time)"}

    line = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": max(3, args.warmup),
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": bench_config(wl, args.layout, world, P, (inp.w1.numel() + inp.w2.numel()) * 2),
        "roofline": {"bound": "tensor", "kernel": "grouped GEMM up (gather + SwiGLU)",
                     "achieved": summ["gemm_up_tflops"], "peak": peak_tf, "unit": "TFLOP/s",
                     "frac": summ["gemm_up_tflops"] / peak_tf,
                     "peak_source": f"{peaks_src} bf16 {peak_label} (chosen from the clock record)",
                     "frac_of_burst": summ["gemm_up_tflops"] / peaks["bf16_tflops"],
                     "frac_of_sustained": summ["gemm_up_tflops"] / peaks["bf16_tflops_sustained"],
                     "traffic": traffic_record("gemm_up", wl.name)},
        "gemm_tflops": (summ["flops"]) / ((stage_ms[1] + stage_ms[2]) * 1e-3) / 1e12,
        "gemm_frac_of_peak": (summ["flops"]) / ((stage_ms[1] + stage_ms[2]) * 1e-3) / 1e12 / peak_tf,
        "step_frac_of_roofline": summ["step_frac_of_roofline"],
        "stages_ms": summ["stages_ms"],
        "stages": {k: summ[k] for k in ("gemm_up_tflops", "gemm_down_tflops", "gemm_up_frac", "gemm_down_frac",
                                        "combine_gbs", "combine_frac_hbm", "metadata_gbs")},
        "graph": {"ms_per_step": graph_ms, "tokens_per_s": N * world / (graph_ms * 1e-3),
                  "note": "one forward captured in a CUDA graph, replayed --steps times back to back"},
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps, "pipelining": "copy-in / compute / copy-out streams, 3 buffer sets, inputs packed in one copy"},
        "workloads": workloads,
        "metadata_only": meta_c2,
        "metadata_pairs_only": meta_pairs,
        "router_only": router,
        "training": train,
        "ep_emulated": ep,
        "gpu_launches": 5 * args.steps,  # metadata count + scatter, up, down, combine
        "clocks": clocks,
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    print(json.dumps(line), flush=True)


def relaunch(n: int) -> int:
    """Run this same command as n ranks, one process per GPU, under
    torch.distributed.run (rendezvous on 127.0.0.1, a free port); returns its
    exit code.  ``timeout -k`` bounds the whole launch."""
    import socket
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = ["timeout", "-k", "60", "3600", sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n}", "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.call(cmd)


def main():
    args = parse()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        raise SystemExit(relaunch(args.gpus))
    rank, world, local = dist_env()
    if world != args.gpus:
        raise SystemExit(f"bench.py: --gpus {args.gpus} but {world} ranks were launched (WORLD_SIZE)")
    if args.check_launch:
        print(json.dumps({"rank": rank, "world": world, "impl": args.impl}), flush=True)
        return
    if args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_ours(args, rank, world, local)


if __name__ == "__main__":
    main()
