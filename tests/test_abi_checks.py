"""Host-side argument checks of every C entry point, called through the C ABI
with fake, never-dereferenced addresses: each bad argument must be rejected
before the library touches a device, so these run without a GPU.  A call with
good arguments reaches the device query, which reports the missing device
here (checked only where no device is present: the fake addresses must never
reach a kernel)."""
import ctypes

import pytest

from mixture_experts_routed_non_b200 import binding

A = 1 << 20        # an aligned fake address
A2 = A + 2         # aligned to 2 only
A4 = A + 4         # aligned to 4 only
A8 = A + 8         # aligned to 8 only


@pytest.fixture(scope="module")
def lib():
    return binding.load()


def _no_device():
    import torch
    return not torch.cuda.is_available()


NO_DEVICE = (binding.MOE_ERR_CUDA, binding.MOE_ERR_DEVICE)


# ---------------------------------------------------------------------------
# routing descriptors (moe_routing_t): rejected ones size to 0 bytes
# ---------------------------------------------------------------------------
def _routing(kind=binding.ROUTING_TOPK, dt=binding.INDEX_INT32, N=64, K=4, pairs=-1, e=A, w=A, t=None):
    r = binding.MoeRouting()
    r.kind, r.index_dtype, r.N, r.K, r.pairs = kind, dt, N, K, pairs
    r.expert_idx, r.weights, r.token_idx = e, w, t
    return r


def _bytes(lib, r, E=8, H=0, I=0):
    return lib.moe_nonexpand_routed_workspace_bytes(ctypes.byref(r) if r is not None else None, H, I, E)


def test_routing_descriptors_accepted(lib):
    assert _bytes(lib, _routing()) > 0
    assert _bytes(lib, _routing(dt=binding.INDEX_INT64, e=A8)) > 0
    assert _bytes(lib, _routing(kind=binding.ROUTING_PAIRS, N=64, K=1, pairs=100, t=A)) > 0
    assert _bytes(lib, _routing(kind=binding.ROUTING_PAIRS, dt=binding.INDEX_INT64, pairs=100, e=A8, t=A8)) > 0
    # the empty pair list needs no arrays
    assert _bytes(lib, _routing(kind=binding.ROUTING_PAIRS, pairs=0, e=None, w=None, t=None)) > 0


@pytest.mark.parametrize("case", [
    "null", "kind", "index_dtype", "N", "E0", "E_big", "K0", "K_big", "topk_token_idx", "topk_pairs_over_NK",
    "pairs_negative", "pairs_no_token_idx", "pairs_token_misaligned", "null_experts", "null_weights",
    "int64_experts_misaligned", "weights_misaligned",
])
def test_routing_descriptors_rejected(lib, case):
    E, r = 8, _routing()
    if case == "null":
        r = None
    elif case == "kind":
        r.kind = 7
    elif case == "index_dtype":
        r.index_dtype = 3
    elif case == "N":
        r.N = -1
    elif case == "E0":
        E = 0
    elif case == "E_big":
        E = 1025
    elif case == "K0":
        r.K = 0
    elif case == "K_big":
        r.K = 33
    elif case == "topk_token_idx":
        r.token_idx = A          # a table takes its tokens from slot / K
    elif case == "topk_pairs_over_NK":
        r.pairs = 64 * 4 + 1
    elif case == "pairs_negative":
        r = _routing(kind=binding.ROUTING_PAIRS, pairs=-1, t=A)
    elif case == "pairs_no_token_idx":
        r = _routing(kind=binding.ROUTING_PAIRS, pairs=10, t=None)
    elif case == "pairs_token_misaligned":
        r = _routing(kind=binding.ROUTING_PAIRS, dt=binding.INDEX_INT64, pairs=10, e=A8, t=A4)
    elif case == "null_experts":
        r.expert_idx = None
    elif case == "null_weights":
        r.weights = None
    elif case == "int64_experts_misaligned":
        r = _routing(dt=binding.INDEX_INT64, e=A4)
    elif case == "weights_misaligned":
        r.weights = A2
    assert _bytes(lib, r, E=E) == 0


def test_routed_metadata_rejects_before_the_device(lib):
    meta = binding.MoeMeta(*([A] * 7))
    bad = _routing(kind=9)
    assert lib.moe_nonexpand_routed_metadata(ctypes.byref(bad), 8, ctypes.byref(meta), A, 1 << 30, None) \
        == binding.MOE_ERR_ARG
    good = _routing()
    incomplete = binding.MoeMeta(*([A] * 6 + [None]))          # scores missing
    assert lib.moe_nonexpand_routed_metadata(ctypes.byref(good), 8, ctypes.byref(incomplete), A, 1 << 30, None) \
        == binding.MOE_ERR_ARG
    assert lib.moe_nonexpand_routed_metadata(ctypes.byref(good), 8, ctypes.byref(meta), A, 16, None) \
        == binding.MOE_ERR_WS
    assert lib.moe_nonexpand_routed_metadata(ctypes.byref(good), 8, ctypes.byref(meta), A + 16, 1 << 30, None) \
        == binding.MOE_ERR_WS


# ---------------------------------------------------------------------------
# metadata and combine
# ---------------------------------------------------------------------------
def _meta_call(lib, idx=A, w=A, N=64, K=4, E=8, tp=-1, meta="full", ws=A, wsb=1 << 30):
    m = {"full": binding.MoeMeta(*([A] * 7)), "none": None,
         "no_scores": binding.MoeMeta(*([A] * 6 + [None]))}[meta]
    return lib.moe_nonexpand_metadata(idx, w, N, K, E, tp, ctypes.byref(m) if m is not None else None,
                                      ws, wsb, None)


def test_metadata_argument_checks(lib):
    assert _meta_call(lib, N=-1) == binding.MOE_ERR_ARG
    assert _meta_call(lib, K=0) == binding.MOE_ERR_ARG
    assert _meta_call(lib, K=33) == binding.MOE_ERR_ARG
    assert _meta_call(lib, E=0) == binding.MOE_ERR_ARG
    assert _meta_call(lib, E=1025) == binding.MOE_ERR_ARG
    assert _meta_call(lib, tp=64 * 4 + 1) == binding.MOE_ERR_ARG
    assert _meta_call(lib, idx=None) == binding.MOE_ERR_ARG
    assert _meta_call(lib, w=None) == binding.MOE_ERR_ARG
    assert _meta_call(lib, meta="none") == binding.MOE_ERR_ARG
    assert _meta_call(lib, meta="no_scores") == binding.MOE_ERR_ARG
    assert _meta_call(lib, idx=A2) == binding.MOE_ERR_ARG
    assert _meta_call(lib, ws=None) == binding.MOE_ERR_WS
    assert _meta_call(lib, wsb=16) == binding.MOE_ERR_WS
    if _no_device():
        assert _meta_call(lib) in NO_DEVICE


def _noalloc_call(lib, idx=A, w=A, N=64, K=4, E=8, tp=-1, meta="full"):
    m = {"full": binding.MoeMeta(*([A] * 7)), "none": None,
         "no_scores": binding.MoeMeta(*([A] * 6 + [None]))}[meta]
    return lib.moe_nonexpand_metadata_noalloc(idx, w, N, K, E, tp, ctypes.byref(m) if m is not None else None,
                                              None)


def test_metadata_noalloc_argument_checks(lib):
    """The no-allocation metadata rejects what the workspace entry point
    rejects -- sizes, null and misaligned pointers -- before any CUDA call, so
    a misaligned id or weight pointer never reaches a kernel."""
    assert _noalloc_call(lib, N=-1) == binding.MOE_ERR_ARG
    assert _noalloc_call(lib, K=0) == binding.MOE_ERR_ARG
    assert _noalloc_call(lib, K=33) == binding.MOE_ERR_ARG
    assert _noalloc_call(lib, E=0) == binding.MOE_ERR_ARG
    assert _noalloc_call(lib, E=1025) == binding.MOE_ERR_ARG
    assert _noalloc_call(lib, N=1 << 28, K=8) == binding.MOE_ERR_ARG   # N*K beyond 2^31
    assert _noalloc_call(lib, tp=64 * 4 + 1) == binding.MOE_ERR_ARG
    assert _noalloc_call(lib, tp=-2) == binding.MOE_ERR_ARG
    assert _noalloc_call(lib, idx=None) == binding.MOE_ERR_ARG
    assert _noalloc_call(lib, w=None) == binding.MOE_ERR_ARG
    assert _noalloc_call(lib, meta="none") == binding.MOE_ERR_ARG
    assert _noalloc_call(lib, meta="no_scores") == binding.MOE_ERR_ARG
    assert _noalloc_call(lib, idx=A + 1) == binding.MOE_ERR_ARG
    assert _noalloc_call(lib, idx=A2) == binding.MOE_ERR_ARG
    assert _noalloc_call(lib, w=A + 3) == binding.MOE_ERR_ARG
    assert _noalloc_call(lib, w=A2) == binding.MOE_ERR_ARG
    err = ctypes.c_uint32(0)
    assert lib.moe_nonexpand_metadata_noalloc_read_error(None, None) == binding.MOE_ERR_ARG
    if _no_device():
        assert _noalloc_call(lib) in NO_DEVICE
        assert lib.moe_nonexpand_metadata_noalloc_read_error(None, ctypes.byref(err)) in NO_DEVICE


def test_combine_argument_checks(lib):
    meta = binding.MoeMeta(*([A] * 7))
    no_rev = binding.MoeMeta(A, A, A, A, None, A, A)

    def call(y=A, m=meta, N=64, H=128, out=A):
        return lib.moe_nonexpand_combine(y, ctypes.byref(m), N, H, out, None)

    assert call(y=None) == binding.MOE_ERR_ARG
    assert call(out=None) == binding.MOE_ERR_ARG
    assert call(m=no_rev) == binding.MOE_ERR_ARG
    assert call(N=-1) == binding.MOE_ERR_ARG
    assert call(H=96) == binding.MOE_ERR_SHAPE
    assert call(H=0) == binding.MOE_ERR_SHAPE
    assert call(y=A8) == binding.MOE_ERR_ARG
    assert call(out=A8) == binding.MOE_ERR_ARG
    if _no_device():
        assert call() in NO_DEVICE


# ---------------------------------------------------------------------------
# router
# ---------------------------------------------------------------------------
def _router(lib, logits=A, dt=binding.DTYPE_F32, N=16, E=64, K=8, mode=binding.ROUTER_SOFTMAX_TOPK, idx=A, w=A):
    return lib.moe_router_topk(logits, dt, N, E, K, mode, idx, w, None)


def test_router_argument_checks(lib):
    assert _router(lib, N=-1) == binding.MOE_ERR_ARG
    assert _router(lib, E=0) == binding.MOE_ERR_ARG
    assert _router(lib, E=1025) == binding.MOE_ERR_ARG
    assert _router(lib, K=0) == binding.MOE_ERR_ARG
    assert _router(lib, K=33, E=64) == binding.MOE_ERR_ARG
    assert _router(lib, K=9, E=8) == binding.MOE_ERR_ARG           # K > E
    assert _router(lib, dt=5) == binding.MOE_ERR_ARG
    assert _router(lib, mode=3) == binding.MOE_ERR_ARG
    assert _router(lib, logits=None) == binding.MOE_ERR_ARG
    assert _router(lib, idx=None) == binding.MOE_ERR_ARG
    assert _router(lib, w=None) == binding.MOE_ERR_ARG
    assert _router(lib, logits=A2) == binding.MOE_ERR_ARG           # fp32 logits need 4-byte alignment
    assert _router(lib, idx=A2) == binding.MOE_ERR_ARG
    assert _router(lib, N=1 << 34, E=64) == binding.MOE_ERR_ARG     # N*E past 2^40
    if _no_device():
        assert _router(lib, logits=A2, dt=binding.DTYPE_BF16) in NO_DEVICE   # bf16 needs 2 only
        assert _router(lib, N=0, logits=None, idx=None, w=None) in NO_DEVICE


# ---------------------------------------------------------------------------
# expert-parallel dispatch / combine
# ---------------------------------------------------------------------------
def _layout(lib, idx=A, T=64, K=8, R=4, E_local=8, send_idx=A, send_count=A, err=A):
    return lib.moe_ep_layout(idx, T, K, R, E_local, send_idx, send_count, err, None)


def test_ep_layout_argument_checks(lib):
    assert _layout(lib, T=-1) == binding.MOE_ERR_ARG
    assert _layout(lib, K=0) == binding.MOE_ERR_ARG
    assert _layout(lib, K=33) == binding.MOE_ERR_ARG
    assert _layout(lib, R=0) == binding.MOE_ERR_ARG
    assert _layout(lib, R=binding.EP_MAX_RANKS + 1) == binding.MOE_ERR_ARG
    assert _layout(lib, E_local=0) == binding.MOE_ERR_ARG
    assert _layout(lib, R=32, E_local=1 << 26) == binding.MOE_ERR_ARG   # R*E_local past 2^31
    assert _layout(lib, send_count=None) == binding.MOE_ERR_ARG
    assert _layout(lib, idx=None) == binding.MOE_ERR_ARG
    assert _layout(lib, send_idx=None) == binding.MOE_ERR_ARG
    assert _layout(lib, send_idx=A2) == binding.MOE_ERR_ARG
    assert _layout(lib, err=A2) == binding.MOE_ERR_ARG
    if _no_device():
        assert _layout(lib) in NO_DEVICE


def _peers(R=4, **bad):
    p = binding.MoeEpPeers()
    for d in range(min(R, binding.EP_MAX_RANKS)):
        p.recv_x[d], p.recv_idx[d], p.recv_w[d] = A, A, A
        p.row_off[d], p.recv_rows[d] = 0, 100
    p.err_word = A
    for k, (d, v) in bad.items():
        getattr(p, k)[d] = v
    return p


def _dispatch(lib, x=A, idx=A, w=A, send_idx=A, T=64, H=256, K=8, R=4, E_local=8, peers="ok", **bad):
    p = _peers(R, **bad) if peers == "ok" else None
    return lib.moe_ep_dispatch(x, idx, w, send_idx, T, H, K, R, E_local,
                               ctypes.byref(p) if p is not None else None, None)


def test_ep_dispatch_argument_checks(lib):
    assert _dispatch(lib, peers=None) == binding.MOE_ERR_ARG
    assert _dispatch(lib, T=-1) == binding.MOE_ERR_ARG
    assert _dispatch(lib, H=4) == binding.MOE_ERR_ARG
    assert _dispatch(lib, H=260) == binding.MOE_ERR_ARG              # rows move in 16-byte pieces
    assert _dispatch(lib, R=0) == binding.MOE_ERR_ARG
    assert _dispatch(lib, R=binding.EP_MAX_RANKS + 1) == binding.MOE_ERR_ARG
    assert _dispatch(lib, E_local=0) == binding.MOE_ERR_ARG
    assert _dispatch(lib, x=None) == binding.MOE_ERR_ARG
    assert _dispatch(lib, x=A8) == binding.MOE_ERR_ARG
    assert _dispatch(lib, send_idx=None) == binding.MOE_ERR_ARG
    assert _dispatch(lib, recv_x=(3, None)) == binding.MOE_ERR_ARG    # a rank below R without a buffer
    assert _dispatch(lib, recv_x=(1, A8)) == binding.MOE_ERR_ARG
    assert _dispatch(lib, recv_idx=(0, A2)) == binding.MOE_ERR_ARG
    assert _dispatch(lib, row_off=(2, -1)) == binding.MOE_ERR_ARG
    assert _dispatch(lib, recv_rows=(2, -5)) == binding.MOE_ERR_ARG
    if _no_device():
        # ranks at or past R are never looked at
        assert _dispatch(lib, R=2, recv_x=(3, None)) in NO_DEVICE


def _sources(R=4, **bad):
    s = binding.MoeEpSources()
    for d in range(min(R, binding.EP_MAX_RANKS)):
        s.local_out[d], s.row_off[d], s.rows[d] = A, 0, 100
    s.err_word = A
    for k, (d, v) in bad.items():
        getattr(s, k)[d] = v
    return s


def _ep_combine(lib, src="ok", send_idx=A, T=64, H=256, R=4, out=A, **bad):
    s = _sources(R, **bad) if src == "ok" else None
    return lib.moe_ep_combine(ctypes.byref(s) if s is not None else None, send_idx, T, H, R, out, None)


def test_ep_combine_argument_checks(lib):
    assert _ep_combine(lib, src=None) == binding.MOE_ERR_ARG
    assert _ep_combine(lib, T=-1) == binding.MOE_ERR_ARG
    assert _ep_combine(lib, H=12) == binding.MOE_ERR_ARG
    assert _ep_combine(lib, R=binding.EP_MAX_RANKS + 1) == binding.MOE_ERR_ARG
    assert _ep_combine(lib, out=None) == binding.MOE_ERR_ARG
    assert _ep_combine(lib, out=A8) == binding.MOE_ERR_ARG
    assert _ep_combine(lib, send_idx=None) == binding.MOE_ERR_ARG
    assert _ep_combine(lib, local_out=(2, None)) == binding.MOE_ERR_ARG
    assert _ep_combine(lib, local_out=(0, A8)) == binding.MOE_ERR_ARG
    assert _ep_combine(lib, row_off=(1, -1)) == binding.MOE_ERR_ARG
    assert _ep_combine(lib, rows=(3, -1)) == binding.MOE_ERR_ARG
    if _no_device():
        assert _ep_combine(lib) in NO_DEVICE


# ---------------------------------------------------------------------------
# training pair
# ---------------------------------------------------------------------------
def test_train_workspace_bytes(lib):
    n = lib.moe_nonexpand_train_workspace_bytes(64, 128, 128, 8, 4, -1)
    assert n > lib.moe_nonexpand_workspace_bytes(64, 128, 128, 8, 4, -1) > 0
    assert lib.moe_nonexpand_train_workspace_bytes(64, 0, 128, 8, 4, -1) == 0     # H needed
    assert lib.moe_nonexpand_train_workspace_bytes(64, 128, 96, 8, 4, -1) == 0    # I % 64
    assert lib.moe_nonexpand_train_workspace_bytes(64, 128, 128, 8, 0, -1) == 0
    r = _routing()
    assert lib.moe_nonexpand_routed_train_workspace_bytes(ctypes.byref(r), 128, 128, 8) == n
    bad = _routing(kind=7)
    assert lib.moe_nonexpand_routed_train_workspace_bytes(ctypes.byref(bad), 128, 128, 8) == 0


def _fwd_train(lib, x=A, idx=A, w=A, N=64, H=128, I=128, E=8, K=4, tp=-1, w1=A, b1=None, w2=A, b2=None,
               act=binding.ACT_SWIGLU, lay=binding.LAYOUT_INTERLEAVED, out=A, ws=A, wsb=1 << 30):
    return lib.moe_nonexpand_forward_train(x, idx, w, N, H, I, E, K, tp, w1, b1, w2, b2, act, lay, out, ws, wsb,
                                           None)


def test_forward_train_argument_checks(lib):
    total = lib.moe_nonexpand_workspace_bytes(64, 128, 128, 8, 4, -1)
    assert _fwd_train(lib, K=0) == binding.MOE_ERR_ARG
    assert _fwd_train(lib, idx=A2) == binding.MOE_ERR_ARG
    assert _fwd_train(lib, x=None) == binding.MOE_ERR_ARG
    assert _fwd_train(lib, w2=None) == binding.MOE_ERR_ARG
    assert _fwd_train(lib, act=3) == binding.MOE_ERR_ARG
    assert _fwd_train(lib, lay=5) == binding.MOE_ERR_ARG
    assert _fwd_train(lib, b1=A8) == binding.MOE_ERR_ARG
    assert _fwd_train(lib, H=100) == binding.MOE_ERR_SHAPE
    assert _fwd_train(lib, wsb=total) == binding.MOE_ERR_WS     # the inference size is too small
    if _no_device():
        assert _fwd_train(lib) in NO_DEVICE


def _bwd(lib, fn="moe_nonexpand_backward", dout=A, x=A, idx=A, w=A, N=64, H=128, I=128, E=8, K=4, tp=-1,
         w1=A, w2=A, act=binding.ACT_SWIGLU, lay=binding.LAYOUT_INTERLEAVED, dx=A, dw1=A, db1=None, dw2=A,
         db2=None, dw=A, ws=A, wsb=1 << 30, events="none"):
    args = [dout, x, idx, w, N, H, I, E, K, tp, w1, w2, act, lay, dx, dw1, db1, dw2, db2, dw, ws, wsb, None]
    if fn == "moe_nonexpand_backward_timed":
        args.append(None if events == "none" else events)
    return getattr(lib, fn)(*args)


def test_backward_argument_checks(lib):
    train_total = lib.moe_nonexpand_train_workspace_bytes(64, 128, 128, 8, 4, -1)
    assert _bwd(lib, N=-1) == binding.MOE_ERR_ARG
    assert _bwd(lib, idx=None) == binding.MOE_ERR_ARG
    assert _bwd(lib, dout=None) == binding.MOE_ERR_ARG
    assert _bwd(lib, dx=None) == binding.MOE_ERR_ARG
    assert _bwd(lib, dw=None) == binding.MOE_ERR_ARG           # the score gradient is always produced
    assert _bwd(lib, dw1=None) == binding.MOE_ERR_ARG
    assert _bwd(lib, act=1) == binding.MOE_ERR_ARG
    assert _bwd(lib, lay=2) == binding.MOE_ERR_ARG
    assert _bwd(lib, dx=A8) == binding.MOE_ERR_ARG
    assert _bwd(lib, db2=A8) == binding.MOE_ERR_ARG
    assert _bwd(lib, dw=A2) == binding.MOE_ERR_ARG
    assert _bwd(lib, I=32) == binding.MOE_ERR_SHAPE
    assert _bwd(lib, wsb=train_total - 1) == binding.MOE_ERR_WS
    assert _bwd(lib, ws=A + 64) == binding.MOE_ERR_WS
    assert _bwd(lib, fn="moe_nonexpand_backward_timed") == binding.MOE_ERR_ARG   # events required
    if _no_device():
        assert _bwd(lib) in NO_DEVICE


def test_routed_training_rejects_bad_descriptors(lib):
    bad = _routing(kind=binding.ROUTING_PAIRS, pairs=10, t=None)
    assert lib.moe_nonexpand_routed_forward_train(A, ctypes.byref(bad), 128, 128, 8, A, None, A, None,
                                                  binding.ACT_SWIGLU, binding.LAYOUT_INTERLEAVED, A, A, 1 << 30,
                                                  None) == binding.MOE_ERR_ARG
    assert lib.moe_nonexpand_routed_backward(A, A, ctypes.byref(bad), 128, 128, 8, A, A, binding.ACT_SWIGLU,
                                             binding.LAYOUT_INTERLEAVED, A, A, None, A, None, A, A, 1 << 30,
                                             None) == binding.MOE_ERR_ARG
    good = _routing()
    assert lib.moe_nonexpand_routed_backward(A, A, ctypes.byref(good), 128, 128, 8, A, A, binding.ACT_SWIGLU,
                                             binding.LAYOUT_INTERLEAVED, A, A, None, A, None, None, A, 1 << 30,
                                             None) == binding.MOE_ERR_ARG   # no score-gradient buffer
