"""The N>1 plumbing of bench.py on CPU: world_size-2 gloo ranks.

The path has no exchange step (every rank runs its own replica on its own
tokens), so the only collectives are the barriers around the timed region and
the max over ranks of the device-timed durations.  These tests check that
max over ranks with two gloo processes, and that the reference arm launched
the way a multi-GPU run launches it (torchrun, two ranks) prints exactly one
JSON line, from rank 0, while the other rank exits 0 without work.
"""
from __future__ import annotations

import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _max_worker(rank: int, world: int, port: int, values, out_dir: str) -> None:
    import torch.distributed as dist
    from datetime import timedelta

    sys.path.insert(0, ROOT)
    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        got = [bench.max_over_ranks(v, "cpu", world) for v in values[rank]]
        dist.barrier()
    finally:
        dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(got, f)


def test_max_over_ranks_gloo(tmp_path):
    """Each rank passes its own durations; every rank gets the largest, in
    the same order, whichever rank held it."""
    world = 2
    values = [[1.5, 9.25, 0.0], [4.0, 2.0, 0.0]]
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_max_worker, args=(r, world, port, values, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    for p in procs:
        if p.is_alive():
            p.kill()
            p.join()
    assert [p.exitcode for p in procs] == [0, 0]
    for r in range(world):
        with open(tmp_path / f"rank{r}.json") as f:
            assert json.load(f) == [4.0, 9.25, 0.0]


def test_max_over_ranks_single_rank():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, "cpu", 1) == 3.5


@pytest.mark.timeout(600)
def test_reference_arm_torchrun_two_ranks():
    """bench.py --impl reference under torchrun with two ranks: rank 0 alone
    times the oracle and prints one JSON line with the contract's keys."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           "bench.py", "--impl", "reference", "--gpus", "2", "--steps", "2", "--warmup", "3",
           "--workload", "tiny", "--ref-seconds", "0.05"]
    env = dict(os.environ)
    env.setdefault("OMP_NUM_THREADS", "1")
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=540)
    assert r.returncode == 0, r.stderr[-4000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["n_gpus"] == 2 and d["steps"] == 2 and d["warmup"] == 3
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == "tiny"


def _counts_worker(rank: int, world: int, port: int, counts, out_dir: str) -> None:
    import torch
    import torch.distributed as dist
    from datetime import timedelta

    sys.path.insert(0, ROOT)
    from mixture_experts_routed_non_b200 import ep

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        got = ep.exchange_counts(torch.tensor(counts[rank], dtype=torch.int32))
        off, n_recv = ep.block_offsets(got)
    finally:
        dist.destroy_process_group()
    with open(os.path.join(out_dir, f"counts{rank}.json"), "w") as f:
        json.dump({"counts": got.tolist(), "off": off.tolist(), "n_recv": n_recv.tolist()}, f)


def test_ep_count_exchange_gloo(tmp_path):
    """The expert-parallel count exchange (an all-gather of every rank's send
    counts) and the receive-block offsets derived from it agree on every rank
    with the oracle's offsets."""
    sys.path.insert(0, ROOT)
    from oracle import ep as oep
    world = 2
    counts = [[3, 5], [0, 7]]  # counts[s][d]
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_counts_worker, args=(r, world, port, counts, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    for p in procs:
        if p.is_alive():
            p.kill()
            p.join()
    assert [p.exitcode for p in procs] == [0, 0]
    ref_off, ref_n = oep.recv_offsets(np.array(counts))
    for r in range(world):
        with open(tmp_path / f"counts{r}.json") as f:
            got = json.load(f)
        assert got["counts"] == counts
        assert got["off"] == ref_off.tolist() and got["n_recv"] == ref_n.tolist()
