"""Thin ctypes binding of ``libmoe_nonexpand.so`` (C ABI in include/moe_nonexpand.h).

Argument marshalling only: torch tensors are checked for dtype, shape,
device and contiguity, and their device pointers plus the current CUDA stream
are handed to the library; every step of the computation runs in the
library's CUDA kernels.  The library is required: importing works anywhere,
but any call without a built library raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_nonexpand.so")

MOE_OK = 0
MOE_ERR_ARG = 1
MOE_ERR_SHAPE = 2
MOE_ERR_WS = 3
MOE_ERR_CUDA = 4
MOE_ERR_DEVICE = 5

DEVERR_BAD_EXPERT_ID = 0x1
DEVERR_PAIR_COUNT = 0x2
DEVERR_TIMEOUT = 0x4
DEVERR_ABORTED = 0x8
DEVERR_BAD_TOKEN = 0x10

ROUTING_TOPK = 0
ROUTING_PAIRS = 1
INDEX_INT32 = 0
INDEX_INT64 = 1

ACT_SWIGLU = 0
LAYOUT_INTERLEAVED = 0
LAYOUT_CONCATENATED = 1

EXPORTED = (
    "moe_nonexpand_workspace_bytes",
    "moe_nonexpand_metadata",
    "moe_nonexpand_forward",
    "moe_nonexpand_forward_timed",
    "moe_nonexpand_combine",
    "moe_nonexpand_workspace_layout",
    "moe_nonexpand_read_error",
    "moe_nonexpand_strerror",
    "moe_nonexpand_metadata_noalloc",
    "moe_nonexpand_metadata_noalloc_read_error",
    "moe_nonexpand_selftest_wait_timeout",
    "moe_nonexpand_routed_workspace_bytes",
    "moe_nonexpand_routed_metadata",
    "moe_nonexpand_routed_forward",
    "moe_router_topk",
    "moe_nonexpand_train_workspace_bytes",
    "moe_nonexpand_forward_train",
    "moe_nonexpand_backward",
    "moe_nonexpand_backward_timed",
    "moe_nonexpand_routed_train_workspace_bytes",
    "moe_nonexpand_routed_forward_train",
    "moe_nonexpand_routed_backward",
    "moe_ep_layout",
    "moe_ep_dispatch",
    "moe_ep_combine",
)

EP_MAX_RANKS = 32

ROUTER_SOFTMAX_TOPK = 0
ROUTER_TOPK_SOFTMAX = 1
ROUTER_TOPK_SOFTMAX_RENORM = 2
DTYPE_F32 = 0
DTYPE_BF16 = 1


class MoeMeta(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "expert_frequency", "expert_frequency_offset", "x_gather_idx", "s_scatter_idx",
        "s_reverse_scatter_idx", "token_offset", "scores")]


class WsLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in (
        "total", "header", "tile_hist", "tile_valid", "tile_err", "gemm_tile_offset",
        "meta_freq", "meta_off", "meta_x_gather", "meta_s_scatter", "meta_s_rev",
        "meta_token_offset", "meta_scores", "h", "y")] + [
        ("p_cap", ctypes.c_int64), ("meta_tiles", ctypes.c_int32), ("meta_tile_slots", ctypes.c_int32),
        ("z", ctypes.c_size_t), ("dz", ctypes.c_size_t), ("dy", ctypes.c_size_t),
        ("slot_pair", ctypes.c_size_t), ("ds", ctypes.c_size_t), ("train_total", ctypes.c_size_t),
        ("y_scale", ctypes.c_size_t)]


class MoeRouting(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("index_dtype", ctypes.c_int32), ("N", ctypes.c_int64),
                ("K", ctypes.c_int32), ("pairs", ctypes.c_int64), ("expert_idx", ctypes.c_void_p),
                ("weights", ctypes.c_void_p), ("token_idx", ctypes.c_void_p)]


class MoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {strerror(status)} (status {status})")
        self.status = status


_lib = None


class MoeEpPeers(ctypes.Structure):
    """moe_ep_peers_t: every rank's receive buffers as seen from the caller."""
    _fields_ = [("recv_x", ctypes.c_void_p * EP_MAX_RANKS),
                ("recv_idx", ctypes.c_void_p * EP_MAX_RANKS),
                ("recv_w", ctypes.c_void_p * EP_MAX_RANKS),
                ("row_off", ctypes.c_int64 * EP_MAX_RANKS),
                ("recv_rows", ctypes.c_int64 * EP_MAX_RANKS),
                ("err_word", ctypes.c_void_p)]


class MoeEpSources(ctypes.Structure):
    """moe_ep_sources_t: every rank's local_out as seen from the caller."""
    _fields_ = [("local_out", ctypes.c_void_p * EP_MAX_RANKS),
                ("row_off", ctypes.c_int64 * EP_MAX_RANKS),
                ("rows", ctypes.c_int64 * EP_MAX_RANKS),
                ("err_word", ctypes.c_void_p)]


def load() -> ctypes.CDLL:
    """Load the CUDA library (fails loudly when it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"CUDA library missing: {LIB_PATH}; build it with "
                           f"`python -m mixture_experts_routed_non_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
    lib.moe_nonexpand_workspace_bytes.restype = sz
    lib.moe_nonexpand_workspace_bytes.argtypes = [i64, i32, i32, i32, i32, i64]
    lib.moe_nonexpand_metadata.restype = ctypes.c_int
    lib.moe_nonexpand_metadata.argtypes = [P, P, i64, i32, i32, i64, ctypes.POINTER(MoeMeta), P, sz, P]
    fwd = [P, P, P, i64, i32, i32, i32, i32, i64, P, P, P, P, i32, i32, P, ctypes.POINTER(MoeMeta), P, sz, P]
    lib.moe_nonexpand_forward.restype = ctypes.c_int
    lib.moe_nonexpand_forward.argtypes = fwd
    lib.moe_nonexpand_forward_timed.restype = ctypes.c_int
    lib.moe_nonexpand_forward_timed.argtypes = fwd + [P]
    lib.moe_nonexpand_combine.restype = ctypes.c_int
    lib.moe_nonexpand_combine.argtypes = [P, ctypes.POINTER(MoeMeta), i64, i32, P, P]
    lib.moe_nonexpand_workspace_layout.restype = ctypes.c_int
    lib.moe_nonexpand_workspace_layout.argtypes = [i64, i32, i32, i32, i32, i64, ctypes.POINTER(WsLayout)]
    lib.moe_nonexpand_read_error.restype = ctypes.c_int
    lib.moe_nonexpand_read_error.argtypes = [P, P, ctypes.POINTER(ctypes.c_uint32)]
    lib.moe_nonexpand_metadata_noalloc.restype = ctypes.c_int
    lib.moe_nonexpand_metadata_noalloc.argtypes = [P, P, i64, i32, i32, i64, ctypes.POINTER(MoeMeta), P]
    lib.moe_nonexpand_metadata_noalloc_read_error.restype = ctypes.c_int
    lib.moe_nonexpand_metadata_noalloc_read_error.argtypes = [P, ctypes.POINTER(ctypes.c_uint32)]
    lib.moe_nonexpand_selftest_wait_timeout.restype = ctypes.c_int
    lib.moe_nonexpand_selftest_wait_timeout.argtypes = [P, sz, ctypes.c_uint32, P]
    R = ctypes.POINTER(MoeRouting)
    lib.moe_nonexpand_routed_workspace_bytes.restype = sz
    lib.moe_nonexpand_routed_workspace_bytes.argtypes = [R, i32, i32, i32]
    lib.moe_nonexpand_routed_metadata.restype = ctypes.c_int
    lib.moe_nonexpand_routed_metadata.argtypes = [R, i32, ctypes.POINTER(MoeMeta), P, sz, P]
    lib.moe_nonexpand_routed_forward.restype = ctypes.c_int
    lib.moe_nonexpand_routed_forward.argtypes = [P, R, i32, i32, i32, P, P, P, P, i32, i32, P,
                                                 ctypes.POINTER(MoeMeta), P, sz, P]
    lib.moe_router_topk.restype = ctypes.c_int
    lib.moe_router_topk.argtypes = [P, i32, i64, i32, i32, i32, P, P, P]
    lib.moe_nonexpand_train_workspace_bytes.restype = sz
    lib.moe_nonexpand_train_workspace_bytes.argtypes = [i64, i32, i32, i32, i32, i64]
    lib.moe_nonexpand_forward_train.restype = ctypes.c_int
    lib.moe_nonexpand_forward_train.argtypes = [P, P, P, i64, i32, i32, i32, i32, i64, P, P, P, P, i32, i32, P, P,
                                                sz, P]
    bwd = [P, P, P, P, i64, i32, i32, i32, i32, i64, P, P, i32, i32, P, P, P, P, P, P, P, sz, P]
    lib.moe_nonexpand_backward.restype = ctypes.c_int
    lib.moe_nonexpand_backward.argtypes = bwd
    lib.moe_nonexpand_backward_timed.restype = ctypes.c_int
    lib.moe_nonexpand_backward_timed.argtypes = bwd + [P]
    lib.moe_nonexpand_routed_train_workspace_bytes.restype = sz
    lib.moe_nonexpand_routed_train_workspace_bytes.argtypes = [R, i32, i32, i32]
    lib.moe_nonexpand_routed_forward_train.restype = ctypes.c_int
    lib.moe_nonexpand_routed_forward_train.argtypes = [P, R, i32, i32, i32, P, P, P, P, i32, i32, P, P, sz, P]
    lib.moe_nonexpand_routed_backward.restype = ctypes.c_int
    lib.moe_nonexpand_routed_backward.argtypes = [P, P, R, i32, i32, i32, P, P, i32, i32, P, P, P, P, P, P, P, sz, P]
    lib.moe_ep_layout.restype = ctypes.c_int
    lib.moe_ep_layout.argtypes = [P, i64, i32, i32, i32, P, P, P, P]
    lib.moe_ep_dispatch.restype = ctypes.c_int
    lib.moe_ep_dispatch.argtypes = [P, P, P, P, i64, i32, i32, i32, i32, ctypes.POINTER(MoeEpPeers), P]
    lib.moe_ep_combine.restype = ctypes.c_int
    lib.moe_ep_combine.argtypes = [ctypes.POINTER(MoeEpSources), P, i64, i32, i32, P, P]
    lib.moe_nonexpand_strerror.restype = ctypes.c_char_p
    lib.moe_nonexpand_strerror.argtypes = [ctypes.c_int]
    _lib = lib
    return lib


def strerror(status: int) -> str:
    return load().moe_nonexpand_strerror(status).decode()


def _check(status: int, what: str):
    if status != MOE_OK:
        raise MoeError(status, what)


def _stream_handle(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _need(t: torch.Tensor, name: str, dtype, shape, device):
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.device != device:
        raise ValueError(f"{name}: expected device {device}, got {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")


# ---------------------------------------------------------------------------
# Sizes and workspace
# ---------------------------------------------------------------------------

def p_cap(N: int, K: int, total_pairs: int = -1) -> int:
    return total_pairs if total_pairs >= 0 else N * K


def workspace_bytes(N: int, H: int, I: int, E: int, K: int, total_pairs: int = -1) -> int:
    n = load().moe_nonexpand_workspace_bytes(N, H, I, E, K, total_pairs)
    if n == 0:
        raise MoeError(MOE_ERR_ARG, "moe_nonexpand_workspace_bytes")
    return n


def workspace_layout(N: int, H: int, I: int, E: int, K: int, total_pairs: int = -1) -> WsLayout:
    out = WsLayout()
    _check(load().moe_nonexpand_workspace_layout(N, H, I, E, K, total_pairs, ctypes.byref(out)),
           "moe_nonexpand_workspace_layout")
    return out


def alloc_workspace(N: int, H: int, I: int, E: int, K: int, total_pairs: int = -1,
                    device=None) -> torch.Tensor:
    """A workspace of the required size (its contents need no initialisation)."""
    n = workspace_bytes(N, H, I, E, K, total_pairs)
    return torch.empty(n, dtype=torch.uint8, device=device or torch.device("cuda"))


def alloc_meta(N: int, K: int, E: int, total_pairs: int = -1, device=None) -> dict:
    dev = device or torch.device("cuda")
    pc = max(1, p_cap(N, K, total_pairs))
    i32 = torch.int32
    return dict(
        expert_frequency=torch.empty(E, dtype=i32, device=dev),
        expert_frequency_offset=torch.empty(E + 1, dtype=i32, device=dev),
        x_gather_idx=torch.empty(pc, dtype=i32, device=dev),
        s_scatter_idx=torch.empty(pc, dtype=i32, device=dev),
        s_reverse_scatter_idx=torch.empty(pc, dtype=i32, device=dev),
        token_offset=torch.empty(N + 1, dtype=i32, device=dev),
        scores=torch.empty(pc, dtype=torch.float32, device=dev),
    )


def _meta_struct(meta: dict) -> MoeMeta:
    return MoeMeta(*[meta[f].data_ptr() for f, _ in MoeMeta._fields_])


def meta_from_workspace(ws: torch.Tensor, N: int, H: int, I: int, E: int, K: int,
                        total_pairs: int = -1) -> dict:
    """Views of the metadata that moe_nonexpand_forward keeps in the workspace."""
    lay = workspace_layout(N, H, I, E, K, total_pairs)
    pc = lay.p_cap

    def view(off, n, dtype):
        nbytes = n * torch.empty((), dtype=dtype).element_size()
        return ws[off:off + nbytes].view(dtype)

    return dict(
        expert_frequency=view(lay.meta_freq, E, torch.int32),
        expert_frequency_offset=view(lay.meta_off, E + 1, torch.int32),
        x_gather_idx=view(lay.meta_x_gather, pc, torch.int32),
        s_scatter_idx=view(lay.meta_s_scatter, pc, torch.int32),
        s_reverse_scatter_idx=view(lay.meta_s_rev, pc, torch.int32),
        token_offset=view(lay.meta_token_offset, N + 1, torch.int32),
        scores=view(lay.meta_scores, pc, torch.float32),
    )


def intermediates_from_workspace(ws: torch.Tensor, N: int, H: int, I: int, E: int, K: int,
                                 total_pairs: int = -1):
    """Views of the intermediates that moe_nonexpand_forward keeps in the
    workspace, expert-sorted rows: h [P_cap,I] bf16; y [P_cap,H] fp16 and
    y_scale [P_cap,H/32] int8, row p's element c being y[p,c] * 2^y_scale[p,c//32]."""
    lay = workspace_layout(N, H, I, E, K, total_pairs)
    pc = lay.p_cap
    h = ws[lay.h:lay.h + pc * I * 2].view(torch.bfloat16).view(pc, I)
    y = ws[lay.y:lay.y + pc * H * 2].view(torch.float16).view(pc, H)
    y_scale = ws[lay.y_scale:lay.y_scale + pc * (H // 32)].view(torch.int8).view(pc, H // 32)
    return h, y, y_scale


def backward_intermediates_from_workspace(ws: torch.Tensor, N: int, H: int, I: int, E: int, K: int,
                                          total_pairs: int = -1):
    """Views, after moe_nonexpand_backward on a training workspace, of dz
    [P_cap, 2I] (bf16, the SwiGLU backward in w1's column order) and of the
    per-pair dx rows [P_cap, H] (bf16, dz . w1[e]^T, before they are summed
    per token), both in expert-sorted row order."""
    lay = workspace_layout(N, H, I, E, K, total_pairs)
    pc = lay.p_cap
    dz = ws[lay.dz:lay.dz + pc * 2 * I * 2].view(torch.bfloat16).view(pc, 2 * I)
    dx_rows = ws[lay.y:lay.y + pc * H * 2].view(torch.bfloat16).view(pc, H)
    return dz, dx_rows


# ---------------------------------------------------------------------------
# Entry points
# ---------------------------------------------------------------------------

def metadata(topk_idx: torch.Tensor, topk_w: torch.Tensor, E: int, total_pairs: int = -1,
             meta: Optional[dict] = None, ws: Optional[torch.Tensor] = None,
             stream: Optional[torch.cuda.Stream] = None) -> dict:
    """Routing metadata of [N,K] (moe_nonexpand_metadata).  Returns the dict of
    device tensors (P_cap-sized pair arrays; the first P entries are valid)."""
    N, K = topk_idx.shape
    dev = topk_idx.device
    _need(topk_idx, "topk_idx", torch.int32, (N, K), dev)
    _need(topk_w, "topk_w", torch.float32, (N, K), dev)
    if meta is None:
        meta = alloc_meta(N, K, E, total_pairs, dev)
    if ws is None:
        ws = alloc_workspace(N, 0, 0, E, K, total_pairs, dev)
    m = _meta_struct(meta)
    _check(load().moe_nonexpand_metadata(topk_idx.data_ptr(), topk_w.data_ptr(), N, K, E, total_pairs,
                                         ctypes.byref(m), ws.data_ptr(), ws.numel(), _stream_handle(stream)),
           "moe_nonexpand_metadata")
    return meta


def metadata_noalloc(topk_idx: torch.Tensor, topk_w: torch.Tensor, E: int, meta: dict,
                     total_pairs: int = -1, stream: Optional[torch.cuda.Stream] = None) -> dict:
    """moe_nonexpand_metadata_noalloc: the metadata into the caller's `meta`
    buffers (see alloc_meta) using the library's own fixed device scratch, for
    callers that cannot allocate a workspace.  Calls that can overlap on the
    GPU must not be issued (they share the scratch)."""
    N, K = topk_idx.shape
    dev = topk_idx.device
    _need(topk_idx, "topk_idx", torch.int32, (N, K), dev)
    _need(topk_w, "topk_w", torch.float32, (N, K), dev)
    m = _meta_struct(meta)
    _check(load().moe_nonexpand_metadata_noalloc(topk_idx.data_ptr(), topk_w.data_ptr(), N, K, E, total_pairs,
                                                 ctypes.byref(m), _stream_handle(stream)),
           "moe_nonexpand_metadata_noalloc")
    return meta


def metadata_noalloc_read_error(stream: Optional[torch.cuda.Stream] = None) -> int:
    """The device error word of the last metadata_noalloc call on the current
    device (syncs the stream)."""
    v = ctypes.c_uint32(0)
    _check(load().moe_nonexpand_metadata_noalloc_read_error(_stream_handle(stream), ctypes.byref(v)),
           "moe_nonexpand_metadata_noalloc_read_error")
    return int(v.value)


def forward(x: torch.Tensor, topk_idx: torch.Tensor, topk_w: torch.Tensor,
            w1: torch.Tensor, w2: torch.Tensor, b1: Optional[torch.Tensor] = None,
            b2: Optional[torch.Tensor] = None, *, layout: int = LAYOUT_INTERLEAVED,
            total_pairs: int = -1, out: Optional[torch.Tensor] = None,
            ws: Optional[torch.Tensor] = None, meta: Optional[dict] = None,
            stream: Optional[torch.cuda.Stream] = None,
            events: Optional[Sequence[torch.cuda.Event]] = None) -> torch.Tensor:
    """Local expert forward on the non-expand layout (moe_nonexpand_forward).

    x [N,H] bf16, topk_idx [N,K] int32 (-1 = invalid slot), topk_w [N,K] fp32,
    w1 [E,H,2I], w2 [E,I,H], b1 [E,2I] / b2 [E,H] bf16 or None.  Returns
    out [N,H] bf16.  ``events`` (five timing-enabled CUDA events) are recorded
    before/after each stage on the launching stream."""
    N, H = x.shape
    K = topk_idx.shape[1]
    E, H1, I2 = w1.shape
    I = I2 // 2
    dev = x.device
    _need(x, "x", torch.bfloat16, (N, H), dev)
    _need(topk_idx, "topk_idx", torch.int32, (N, K), dev)
    _need(topk_w, "topk_w", torch.float32, (N, K), dev)
    _need(w1, "w1", torch.bfloat16, (E, H, 2 * I), dev)
    _need(w2, "w2", torch.bfloat16, (E, I, H), dev)
    if b1 is not None:
        _need(b1, "b1", torch.bfloat16, (E, 2 * I), dev)
    if b2 is not None:
        _need(b2, "b2", torch.bfloat16, (E, H), dev)
    if out is None:
        out = torch.empty((N, H), dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, (N, H), dev)
    if ws is None:
        ws = alloc_workspace(N, H, I, E, K, total_pairs, dev)
    m = _meta_struct(meta) if meta is not None else None
    mp = ctypes.byref(m) if m is not None else None
    args = (x.data_ptr(), topk_idx.data_ptr(), topk_w.data_ptr(), N, H, I, E, K, total_pairs,
            w1.data_ptr(), _ptr(b1), w2.data_ptr(), _ptr(b2), ACT_SWIGLU, layout,
            out.data_ptr(), mp, ws.data_ptr(), ws.numel(), _stream_handle(stream))
    lib = load()
    if events is None:
        _check(lib.moe_nonexpand_forward(*args), "moe_nonexpand_forward")
    else:
        if len(events) != 5:
            raise ValueError("events: expected 5 CUDA events")
        s = stream if stream is not None else torch.cuda.current_stream()
        for ev in events:
            if not ev.cuda_event:  # torch creates the CUDA event on its first record
                ev.record(s)
        arr = (ctypes.c_void_p * 5)(*[ev.cuda_event for ev in events])
        _check(lib.moe_nonexpand_forward_timed(*args, arr), "moe_nonexpand_forward_timed")
    return out


def combine(y: torch.Tensor, meta: dict, N: int, out: Optional[torch.Tensor] = None,
            stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """The combine step alone (moe_nonexpand_combine): y [P_cap,H] bf16 in
    expert-sorted order -> out [N,H] bf16."""
    H = y.shape[1]
    if y.dtype != torch.bfloat16 or not y.is_contiguous():
        raise TypeError("y: expected contiguous bf16")
    if out is None:
        out = torch.empty((N, H), dtype=torch.bfloat16, device=y.device)
    m = _meta_struct(meta)
    _check(load().moe_nonexpand_combine(y.data_ptr(), ctypes.byref(m), N, H, out.data_ptr(),
                                        _stream_handle(stream)), "moe_nonexpand_combine")
    return out


def selftest_wait_timeout(ws: torch.Tensor, timeout_us: int,
                          stream: Optional[torch.cuda.Stream] = None) -> None:
    """Run one bounded device wait that nothing completes (limit timeout_us);
    afterwards read_error(ws) reports DEVERR_TIMEOUT."""
    _check(load().moe_nonexpand_selftest_wait_timeout(ws.data_ptr(), ws.numel(), timeout_us,
                                                      _stream_handle(stream)),
           "moe_nonexpand_selftest_wait_timeout")


def read_error(ws: torch.Tensor, stream: Optional[torch.cuda.Stream] = None) -> int:
    """The device error word of the last call that used ``ws`` (syncs the stream)."""
    v = ctypes.c_uint32(0)
    _check(load().moe_nonexpand_read_error(ws.data_ptr(), _stream_handle(stream), ctypes.byref(v)),
           "moe_nonexpand_read_error")
    return int(v.value)


# ---------------------------------------------------------------------------
# Either routing layout, int32 or int64 ids (moe_nonexpand_routed_*)
# ---------------------------------------------------------------------------

_INDEX_DTYPES = {torch.int32: INDEX_INT32, torch.int64: INDEX_INT64}


def routing(expert_idx: torch.Tensor, weights: torch.Tensor, *, token_idx: Optional[torch.Tensor] = None,
            N: Optional[int] = None, total_pairs: int = -1) -> MoeRouting:
    """The routing descriptor.  Without ``token_idx``: the non-expand table
    (expert_idx [N,K], weights [N,K]).  With it: a compact pair list
    (token_idx / expert_idx / weights [P], tokens ascending, N tokens)."""
    dev = expert_idx.device
    if expert_idx.dtype not in _INDEX_DTYPES:
        raise TypeError(f"expert_idx: expected int32 or int64, got {expert_idx.dtype}")
    r = MoeRouting()
    r.index_dtype = _INDEX_DTYPES[expert_idx.dtype]
    if token_idx is None:
        if expert_idx.dim() != 2:
            raise ValueError("expert_idx: expected [N,K]")
        n, k = expert_idx.shape
        _need(expert_idx, "expert_idx", expert_idx.dtype, (n, k), dev)
        _need(weights, "weights", torch.float32, (n, k), dev)
        if N is not None and N != n:
            raise ValueError("N does not match expert_idx")
        r.kind, r.N, r.K, r.pairs = ROUTING_TOPK, n, k, total_pairs
        r.token_idx = None
    else:
        if N is None:
            raise ValueError("a pair list needs N")
        p = expert_idx.numel()
        _need(expert_idx, "expert_idx", expert_idx.dtype, (p,), dev)
        _need(token_idx, "token_idx", expert_idx.dtype, (p,), dev)
        _need(weights, "weights", torch.float32, (p,), dev)
        r.kind, r.N, r.K, r.pairs = ROUTING_PAIRS, N, 1, p
        r.token_idx = token_idx.data_ptr()
    r.expert_idx = expert_idx.data_ptr()
    r.weights = weights.data_ptr()
    return r


def routing_p_cap(r: MoeRouting) -> int:
    if r.kind == ROUTING_PAIRS:
        return r.pairs
    return p_cap(r.N, r.K, r.pairs)


def routed_workspace_bytes(r: MoeRouting, H: int, I: int, E: int) -> int:
    n = load().moe_nonexpand_routed_workspace_bytes(ctypes.byref(r), H, I, E)
    if n == 0:
        raise MoeError(MOE_ERR_ARG, "moe_nonexpand_routed_workspace_bytes")
    return n


def alloc_routed_meta(r: MoeRouting, E: int, device=None) -> dict:
    return alloc_meta(r.N, 1, E, routing_p_cap(r), device)


def routed_metadata(expert_idx: torch.Tensor, weights: torch.Tensor, E: int, *,
                    token_idx: Optional[torch.Tensor] = None, N: Optional[int] = None, total_pairs: int = -1,
                    meta: Optional[dict] = None, ws: Optional[torch.Tensor] = None,
                    stream: Optional[torch.cuda.Stream] = None) -> dict:
    """moe_nonexpand_routed_metadata: the metadata of either routing layout."""
    r = routing(expert_idx, weights, token_idx=token_idx, N=N, total_pairs=total_pairs)
    dev = expert_idx.device
    if meta is None:
        meta = alloc_routed_meta(r, E, dev)
    if ws is None:
        ws = torch.empty(routed_workspace_bytes(r, 0, 0, E), dtype=torch.uint8, device=dev)
    m = _meta_struct(meta)
    _check(load().moe_nonexpand_routed_metadata(ctypes.byref(r), E, ctypes.byref(m), ws.data_ptr(), ws.numel(),
                                                _stream_handle(stream)), "moe_nonexpand_routed_metadata")
    return meta


def routed_forward(x: torch.Tensor, expert_idx: torch.Tensor, weights: torch.Tensor,
                   w1: torch.Tensor, w2: torch.Tensor, b1: Optional[torch.Tensor] = None,
                   b2: Optional[torch.Tensor] = None, *, token_idx: Optional[torch.Tensor] = None,
                   layout: int = LAYOUT_INTERLEAVED, total_pairs: int = -1,
                   out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                   meta: Optional[dict] = None, stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """moe_nonexpand_routed_forward: the forward for either routing layout
    (see ``routing``); other arguments as ``forward``."""
    N, H = x.shape
    E, _, I2 = w1.shape
    I = I2 // 2
    dev = x.device
    _need(x, "x", torch.bfloat16, (N, H), dev)
    _need(w1, "w1", torch.bfloat16, (E, H, 2 * I), dev)
    _need(w2, "w2", torch.bfloat16, (E, I, H), dev)
    if b1 is not None:
        _need(b1, "b1", torch.bfloat16, (E, 2 * I), dev)
    if b2 is not None:
        _need(b2, "b2", torch.bfloat16, (E, H), dev)
    r = routing(expert_idx, weights, token_idx=token_idx, N=N, total_pairs=total_pairs)
    if out is None:
        out = torch.empty((N, H), dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, (N, H), dev)
    if ws is None:
        ws = torch.empty(routed_workspace_bytes(r, H, I, E), dtype=torch.uint8, device=dev)
    m = _meta_struct(meta) if meta is not None else None
    mp = ctypes.byref(m) if m is not None else None
    _check(load().moe_nonexpand_routed_forward(x.data_ptr(), ctypes.byref(r), H, I, E, w1.data_ptr(), _ptr(b1),
                                               w2.data_ptr(), _ptr(b2), ACT_SWIGLU, layout, out.data_ptr(), mp,
                                               ws.data_ptr(), ws.numel(), _stream_handle(stream)),
           "moe_nonexpand_routed_forward")
    return out


# ---------------------------------------------------------------------------
# Router top-k (moe_router_topk)
# ---------------------------------------------------------------------------

def router_topk(logits: torch.Tensor, K: int, mode: int = ROUTER_SOFTMAX_TOPK,
                topk_idx: Optional[torch.Tensor] = None, topk_w: Optional[torch.Tensor] = None,
                stream: Optional[torch.cuda.Stream] = None):
    """Router logits [N,E] (fp32 or bf16) -> (topk_idx [N,K] int32, topk_w [N,K] fp32)."""
    N, E = logits.shape
    dev = logits.device
    dtypes = {torch.float32: DTYPE_F32, torch.bfloat16: DTYPE_BF16}
    if logits.dtype not in dtypes:
        raise TypeError(f"logits: expected float32 or bfloat16, got {logits.dtype}")
    _need(logits, "logits", logits.dtype, (N, E), dev)
    if topk_idx is None:
        topk_idx = torch.empty((N, K), dtype=torch.int32, device=dev)
    if topk_w is None:
        topk_w = torch.empty((N, K), dtype=torch.float32, device=dev)
    _need(topk_idx, "topk_idx", torch.int32, (N, K), dev)
    _need(topk_w, "topk_w", torch.float32, (N, K), dev)
    _check(load().moe_router_topk(logits.data_ptr(), dtypes[logits.dtype], N, E, K, mode, topk_idx.data_ptr(),
                                  topk_w.data_ptr(), _stream_handle(stream)), "moe_router_topk")
    return topk_idx, topk_w


# ---------------------------------------------------------------------------
# Expert-parallel dispatch / combine (non-expand); see include/moe_nonexpand.h
# ---------------------------------------------------------------------------

def ep_layout(topk_idx: torch.Tensor, R: int, E_local: int, send_idx: Optional[torch.Tensor] = None,
              send_count: Optional[torch.Tensor] = None, err: Optional[torch.Tensor] = None,
              stream: Optional[torch.cuda.Stream] = None):
    """Source-rank layout: (send_idx [T,R] int32, send_count [R] int32)."""
    T, K = topk_idx.shape
    dev = topk_idx.device
    _need(topk_idx, "topk_idx", torch.int32, (T, K), dev)
    if send_idx is None:
        send_idx = torch.empty((T, R), dtype=torch.int32, device=dev)
    if send_count is None:
        send_count = torch.empty((R,), dtype=torch.int32, device=dev)
    _need(send_idx, "send_idx", torch.int32, (T, R), dev)
    _need(send_count, "send_count", torch.int32, (R,), dev)
    if err is not None:
        _need(err, "err", torch.int32, (1,), dev)
    _check(load().moe_ep_layout(topk_idx.data_ptr(), T, K, R, E_local, send_idx.data_ptr(), send_count.data_ptr(),
                                _ptr(err), _stream_handle(stream)), "moe_ep_layout")
    return send_idx, send_count


def _rows_of(bufs, rows, what):
    if rows is not None:
        return [int(r) for r in rows]
    if all(isinstance(b, torch.Tensor) for b in bufs):
        return [int(b.shape[0]) for b in bufs]
    raise ValueError(f"{what}: give the row counts when the buffers are raw addresses")


def ep_peers(recv_x, recv_idx, recv_w, row_off, recv_rows=None, err: Optional[torch.Tensor] = None) -> MoeEpPeers:
    """A moe_ep_peers_t from per-rank buffers (tensors, or raw addresses with
    ``recv_rows``) and the caller's block offsets on every rank.  The dispatch
    writes no row at or past a rank's row count (it flags the error in
    ``err`` instead)."""
    R = len(recv_x)
    if not (1 <= R <= EP_MAX_RANKS) or not (len(recv_idx) == len(recv_w) == len(row_off) == R):
        raise ValueError("ep_peers: one entry per rank, 1..32 ranks")
    rows = _rows_of(recv_x, recv_rows, "ep_peers")
    p = MoeEpPeers()
    addr = lambda v: v.data_ptr() if isinstance(v, torch.Tensor) else int(v)
    for d in range(R):
        p.recv_x[d], p.recv_idx[d], p.recv_w[d] = addr(recv_x[d]), addr(recv_idx[d]), addr(recv_w[d])
        p.row_off[d] = int(row_off[d])
        p.recv_rows[d] = rows[d]
    p.err_word = _ptr(err)
    return p


def ep_sources(local_out, row_off, rows=None, err: Optional[torch.Tensor] = None) -> MoeEpSources:
    """A moe_ep_sources_t from per-rank local outputs (tensors, or raw
    addresses with ``rows``); the combine reads no row at or past a rank's
    row count (it counts 0 and flags the error in ``err``)."""
    R = len(local_out)
    if not (1 <= R <= EP_MAX_RANKS) or len(row_off) != R:
        raise ValueError("ep_sources: one entry per rank, 1..32 ranks")
    nrows = _rows_of(local_out, rows, "ep_sources")
    src = MoeEpSources()
    for d in range(R):
        v = local_out[d]
        src.local_out[d] = v.data_ptr() if isinstance(v, torch.Tensor) else int(v)
        src.row_off[d] = int(row_off[d])
        src.rows[d] = nrows[d]
    src.err_word = _ptr(err)
    return src


def ep_dispatch(x: torch.Tensor, topk_idx: torch.Tensor, topk_w: torch.Tensor, send_idx: torch.Tensor,
                E_local: int, peers: MoeEpPeers, R: int, stream: Optional[torch.cuda.Stream] = None):
    """Write this source rank's rows into every destination's receive buffers."""
    T, H = x.shape
    K = topk_idx.shape[1]
    dev = x.device
    _need(x, "x", torch.bfloat16, (T, H), dev)
    _need(topk_idx, "topk_idx", torch.int32, (T, K), dev)
    _need(topk_w, "topk_w", torch.float32, (T, K), dev)
    _need(send_idx, "send_idx", torch.int32, (T, R), dev)
    _check(load().moe_ep_dispatch(x.data_ptr(), topk_idx.data_ptr(), topk_w.data_ptr(), send_idx.data_ptr(), T, H,
                                  K, R, E_local, ctypes.byref(peers), _stream_handle(stream)), "moe_ep_dispatch")


def ep_combine(src: MoeEpSources, send_idx: torch.Tensor, H: int, out: Optional[torch.Tensor] = None,
               stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """routed_out [T,H] bf16 of this source rank from every destination's local_out."""
    T, R = send_idx.shape
    dev = send_idx.device
    _need(send_idx, "send_idx", torch.int32, (T, R), dev)
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, (T, H), dev)
    _check(load().moe_ep_combine(ctypes.byref(src), send_idx.data_ptr(), T, H, R, out.data_ptr(),
                                 _stream_handle(stream)), "moe_ep_combine")
    return out


# ---------------------------------------------------------------------------
# Training: forward that keeps z, and the backward
# ---------------------------------------------------------------------------

def train_workspace_bytes(N: int, H: int, I: int, E: int, K: int, total_pairs: int = -1) -> int:
    n = load().moe_nonexpand_train_workspace_bytes(N, H, I, E, K, total_pairs)
    if n == 0:
        raise MoeError(MOE_ERR_ARG, "moe_nonexpand_train_workspace_bytes")
    return n


def alloc_train_workspace(N: int, H: int, I: int, E: int, K: int, total_pairs: int = -1,
                          device=None) -> torch.Tensor:
    n = train_workspace_bytes(N, H, I, E, K, total_pairs)
    return torch.empty(n, dtype=torch.uint8, device=device or torch.device("cuda"))


def forward_train(x: torch.Tensor, topk_idx: torch.Tensor, topk_w: torch.Tensor, w1: torch.Tensor,
                  w2: torch.Tensor, b1: Optional[torch.Tensor] = None, b2: Optional[torch.Tensor] = None, *,
                  ws: torch.Tensor, layout: int = LAYOUT_INTERLEAVED, total_pairs: int = -1,
                  out: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """moe_nonexpand_forward_train: the forward, keeping metadata, h, y and z
    in ``ws`` (see alloc_train_workspace) for ``backward``."""
    N, H = x.shape
    K = topk_idx.shape[1]
    E, _, I2 = w1.shape
    I = I2 // 2
    dev = x.device
    _need(x, "x", torch.bfloat16, (N, H), dev)
    _need(topk_idx, "topk_idx", torch.int32, (N, K), dev)
    _need(topk_w, "topk_w", torch.float32, (N, K), dev)
    _need(w1, "w1", torch.bfloat16, (E, H, 2 * I), dev)
    _need(w2, "w2", torch.bfloat16, (E, I, H), dev)
    if b1 is not None:
        _need(b1, "b1", torch.bfloat16, (E, 2 * I), dev)
    if b2 is not None:
        _need(b2, "b2", torch.bfloat16, (E, H), dev)
    if out is None:
        out = torch.empty((N, H), dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, (N, H), dev)
    _check(load().moe_nonexpand_forward_train(x.data_ptr(), topk_idx.data_ptr(), topk_w.data_ptr(), N, H, I, E, K,
                                              total_pairs, w1.data_ptr(), _ptr(b1), w2.data_ptr(), _ptr(b2),
                                              ACT_SWIGLU, layout, out.data_ptr(), ws.data_ptr(), ws.numel(),
                                              _stream_handle(stream)), "moe_nonexpand_forward_train")
    return out


def backward(dout: torch.Tensor, x: torch.Tensor, topk_idx: torch.Tensor, topk_w: torch.Tensor,
             w1: torch.Tensor, w2: torch.Tensor, *, ws: torch.Tensor, layout: int = LAYOUT_INTERLEAVED,
             total_pairs: int = -1, bias_grads: bool = False, stream: Optional[torch.cuda.Stream] = None,
             events: Optional[Sequence[torch.cuda.Event]] = None, grads: Optional[dict] = None) -> dict:
    """moe_nonexpand_backward after forward_train on the same ``ws``.  Returns
    dict(dx, dw1, dw2, dtopk_w[, db1, db2]).  ``events`` (eight timing
    events) bracket its seven steps."""
    N, H = x.shape
    K = topk_idx.shape[1]
    E, _, I2 = w1.shape
    I = I2 // 2
    dev = x.device
    _need(dout, "dout", torch.bfloat16, (N, H), dev)
    if grads is None:
        grads = dict(dx=torch.empty((N, H), dtype=torch.bfloat16, device=dev),
                     dw1=torch.empty((E, H, 2 * I), dtype=torch.bfloat16, device=dev),
                     dw2=torch.empty((E, I, H), dtype=torch.bfloat16, device=dev),
                     dtopk_w=torch.empty((N, K), dtype=torch.float32, device=dev))
        if bias_grads:
            grads["db1"] = torch.empty((E, 2 * I), dtype=torch.bfloat16, device=dev)
            grads["db2"] = torch.empty((E, H), dtype=torch.bfloat16, device=dev)
    args = (dout.data_ptr(), x.data_ptr(), topk_idx.data_ptr(), topk_w.data_ptr(), N, H, I, E, K, total_pairs,
            w1.data_ptr(), w2.data_ptr(), ACT_SWIGLU, layout, grads["dx"].data_ptr(), grads["dw1"].data_ptr(),
            _ptr(grads.get("db1")), grads["dw2"].data_ptr(), _ptr(grads.get("db2")), grads["dtopk_w"].data_ptr(),
            ws.data_ptr(), ws.numel(), _stream_handle(stream))
    lib = load()
    if events is None:
        _check(lib.moe_nonexpand_backward(*args), "moe_nonexpand_backward")
    else:
        if len(events) != 8:
            raise ValueError("events: expected 8 CUDA events")
        s = stream if stream is not None else torch.cuda.current_stream()
        for ev in events:
            if not ev.cuda_event:
                ev.record(s)
        arr = (ctypes.c_void_p * 8)(*[ev.cuda_event for ev in events])
        _check(lib.moe_nonexpand_backward_timed(*args, arr), "moe_nonexpand_backward_timed")
    return grads


def routed_train_workspace_bytes(r: MoeRouting, H: int, I: int, E: int) -> int:
    n = load().moe_nonexpand_routed_train_workspace_bytes(ctypes.byref(r), H, I, E)
    if n == 0:
        raise MoeError(MOE_ERR_ARG, "moe_nonexpand_routed_train_workspace_bytes")
    return n


def routed_forward_train(x: torch.Tensor, expert_idx: torch.Tensor, weights: torch.Tensor, w1: torch.Tensor,
                         w2: torch.Tensor, b1: Optional[torch.Tensor] = None, b2: Optional[torch.Tensor] = None, *,
                         ws: torch.Tensor, token_idx: Optional[torch.Tensor] = None,
                         layout: int = LAYOUT_INTERLEAVED, total_pairs: int = -1,
                         out: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None):
    """moe_nonexpand_routed_forward_train for either routing layout."""
    N, H = x.shape
    E, _, I2 = w1.shape
    I = I2 // 2
    dev = x.device
    r = routing(expert_idx, weights, token_idx=token_idx, N=N, total_pairs=total_pairs)
    if out is None:
        out = torch.empty((N, H), dtype=torch.bfloat16, device=dev)
    _check(load().moe_nonexpand_routed_forward_train(x.data_ptr(), ctypes.byref(r), H, I, E, w1.data_ptr(),
                                                     _ptr(b1), w2.data_ptr(), _ptr(b2), ACT_SWIGLU, layout,
                                                     out.data_ptr(), ws.data_ptr(), ws.numel(),
                                                     _stream_handle(stream)), "moe_nonexpand_routed_forward_train")
    return out


def routed_backward(dout: torch.Tensor, x: torch.Tensor, expert_idx: torch.Tensor, weights: torch.Tensor,
                    w1: torch.Tensor, w2: torch.Tensor, *, ws: torch.Tensor, token_idx: Optional[torch.Tensor] = None,
                    layout: int = LAYOUT_INTERLEAVED, total_pairs: int = -1, bias_grads: bool = False,
                    stream: Optional[torch.cuda.Stream] = None) -> dict:
    """moe_nonexpand_routed_backward: dict(dx, dw1, dw2, dweights[, db1, db2]);
    dweights has the shape of ``weights``."""
    N, H = x.shape
    E, _, I2 = w1.shape
    I = I2 // 2
    dev = x.device
    r = routing(expert_idx, weights, token_idx=token_idx, N=N, total_pairs=total_pairs)
    g = dict(dx=torch.empty((N, H), dtype=torch.bfloat16, device=dev),
             dw1=torch.empty((E, H, 2 * I), dtype=torch.bfloat16, device=dev),
             dw2=torch.empty((E, I, H), dtype=torch.bfloat16, device=dev),
             dweights=torch.empty(weights.shape, dtype=torch.float32, device=dev))
    if bias_grads:
        g["db1"] = torch.empty((E, 2 * I), dtype=torch.bfloat16, device=dev)
        g["db2"] = torch.empty((E, H), dtype=torch.bfloat16, device=dev)
    _check(load().moe_nonexpand_routed_backward(dout.data_ptr(), x.data_ptr(), ctypes.byref(r), H, I, E,
                                                w1.data_ptr(), w2.data_ptr(), ACT_SWIGLU, layout, g["dx"].data_ptr(),
                                                g["dw1"].data_ptr(), _ptr(g.get("db1")), g["dw2"].data_ptr(),
                                                _ptr(g.get("db2")), g["dweights"].data_ptr(), ws.data_ptr(),
                                                ws.numel(), _stream_handle(stream)), "moe_nonexpand_routed_backward")
    return g
