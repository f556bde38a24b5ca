"""The C-ABI library: it builds, loads without a GPU, exports exactly what the
header declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

from mixture_experts_routed_non_b200 import binding, build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "moe_nonexpand.h")


def declared_symbols():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load()


def test_header_declares_the_entry_points():
    assert declared_symbols() == sorted(binding.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_library_exports_nothing_else(lib):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    names = sorted(l.split()[-1] for l in out.splitlines() if l.strip())
    assert names == sorted(binding.EXPORTED)


def test_strerror(lib):
    for st in range(6):
        assert lib.moe_nonexpand_strerror(st)
    assert b"unknown" in lib.moe_nonexpand_strerror(99)


def test_workspace_bytes_rejects_bad_sizes(lib):
    f = lib.moe_nonexpand_workspace_bytes
    assert f(16, 128, 128, 4, 2, -1) > 0
    assert f(-1, 128, 128, 4, 2, -1) == 0            # N < 0
    assert f(16, 128, 128, 0, 2, -1) == 0            # E < 1
    assert f(16, 128, 128, 2000, 2, -1) == 0         # E > 1024
    assert f(16, 128, 128, 4, 0, -1) == 0            # K < 1
    assert f(16, 128, 128, 4, 33, -1) == 0           # K > 32
    assert f(16, 100, 128, 4, 2, -1) == 0            # H % 64
    assert f(16, 128, 96, 4, 2, -1) == 0             # I % 64
    assert f(16, 128, 128, 4, 2, 33) == 0            # total_pairs > N*K
    assert f(16, 0, 0, 4, 2, -1) > 0                 # metadata-only sizing


def test_workspace_layout_is_consistent(lib):
    for args in [(16384, 2048, 768, 128, 8, -1), (8192, 7168, 2048, 32, 8, 20000), (0, 64, 64, 1, 1, -1),
                 (65536, 0, 0, 128, 8, -1)]:
        lay = binding.workspace_layout(*args)
        assert lay.total == lib.moe_nonexpand_workspace_bytes(*args)
        offs = [lay.header, lay.tile_hist, lay.tile_valid, lay.tile_err, lay.gemm_tile_offset,
                lay.meta_freq, lay.meta_off, lay.meta_x_gather, lay.meta_s_scatter, lay.meta_s_rev,
                lay.meta_token_offset, lay.meta_scores]
        assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
        if args[1]:
            assert lay.h % 1024 == 0 and lay.y % 1024 == 0
            assert lay.y > lay.h if lay.p_cap > 0 else lay.y == lay.h
        assert lay.meta_tile_slots % 1024 == 0 and lay.meta_tiles <= 148
        assert lay.meta_tiles * lay.meta_tile_slots >= args[0] * args[4]


def _fwd(lib, **kw):
    a = dict(x=16, idx=16, w=16, N=4, H=128, I=128, E=2, K=2, tp=-1, w1=16, b1=None, w2=16, b2=None,
             act=0, lay=0, out=16, meta=None, ws=256, wsb=1 << 30, s=None)
    a.update(kw)
    return lib.moe_nonexpand_forward(a["x"], a["idx"], a["w"], a["N"], a["H"], a["I"], a["E"], a["K"],
                                     a["tp"], a["w1"], a["b1"], a["w2"], a["b2"], a["act"], a["lay"],
                                     a["out"], a["meta"], a["ws"], a["wsb"], a["s"])


def test_forward_argument_checks_need_no_device(lib):
    # fake, aligned, never-dereferenced addresses: every case fails in the
    # host-side checks before any CUDA call
    assert _fwd(lib, x=None) == binding.MOE_ERR_ARG
    assert _fwd(lib, N=-3) == binding.MOE_ERR_ARG
    assert _fwd(lib, K=40) == binding.MOE_ERR_ARG
    assert _fwd(lib, act=7) == binding.MOE_ERR_ARG
    assert _fwd(lib, lay=2) == binding.MOE_ERR_ARG
    assert _fwd(lib, x=18) == binding.MOE_ERR_ARG          # misaligned
    assert _fwd(lib, H=96) == binding.MOE_ERR_SHAPE
    assert _fwd(lib, I=32) == binding.MOE_ERR_SHAPE
    assert _fwd(lib, ws=None) == binding.MOE_ERR_WS
    assert _fwd(lib, wsb=100) == binding.MOE_ERR_WS
    assert _fwd(lib, ws=272) == binding.MOE_ERR_WS         # workspace not 256-byte aligned
    assert _fwd(lib, tp=100) == binding.MOE_ERR_ARG         # total_pairs > N*K


def test_no_device_is_reported_as_cuda_error(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    assert _fwd(lib) in (binding.MOE_ERR_CUDA, binding.MOE_ERR_DEVICE)


def test_calls_fail_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(binding, "_lib", None)
    monkeypatch.setattr(binding, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="CUDA library missing"):
        binding.load()
