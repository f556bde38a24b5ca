"""The Python binding's host-side marshalling, on CPU tensors: routing
descriptors, workspace sizes through the C ABI's host-only size queries, the
tensor checks, and the expert-parallel pointer tables.  Nothing here launches
device work."""
import ctypes

import pytest
import torch

from mixture_experts_routed_non_b200 import binding


def test_table_descriptor_and_sizes():
    idx = torch.zeros(64, 4, dtype=torch.int32)
    w = torch.zeros(64, 4, dtype=torch.float32)
    r = binding.routing(idx, w)
    assert (r.kind, r.index_dtype, r.N, r.K, r.pairs) == (binding.ROUTING_TOPK, binding.INDEX_INT32, 64, 4, -1)
    assert r.expert_idx == idx.data_ptr() and r.weights == w.data_ptr() and not r.token_idx
    assert binding.routing_p_cap(r) == 256
    # the table descriptor sizes its workspace exactly like the [N,K] entry points
    assert binding.routed_workspace_bytes(r, 128, 128, 8) == binding.workspace_bytes(64, 128, 128, 8, 4)
    assert binding.routed_workspace_bytes(r, 0, 0, 8) == binding.workspace_bytes(64, 0, 0, 8, 4)
    r2 = binding.routing(idx, w, total_pairs=100)
    assert binding.routing_p_cap(r2) == 100
    assert binding.routed_workspace_bytes(r2, 128, 128, 8) == binding.workspace_bytes(64, 128, 128, 8, 4, 100)
    assert binding.routed_workspace_bytes(r2, 128, 128, 8) < binding.routed_workspace_bytes(r, 128, 128, 8)


@pytest.mark.parametrize("dt,kind", [(torch.int32, binding.INDEX_INT32), (torch.int64, binding.INDEX_INT64)])
def test_pair_list_descriptor(dt, kind):
    P, N = 300, 80
    e = torch.zeros(P, dtype=dt)
    t = torch.zeros(P, dtype=dt)
    w = torch.zeros(P, dtype=torch.float32)
    r = binding.routing(e, w, token_idx=t, N=N)
    assert (r.kind, r.index_dtype, r.N, r.K, r.pairs) == (binding.ROUTING_PAIRS, kind, N, 1, P)
    assert r.token_idx == t.data_ptr()
    assert binding.routing_p_cap(r) == P
    n = binding.routed_workspace_bytes(r, 128, 128, 8)
    assert n > 0
    # a list of P pairs needs at most the room of a table with the same P slots
    assert n <= binding.workspace_bytes(P, 128, 128, 8, 1)


def test_routing_rejects_bad_tensors():
    idx = torch.zeros(8, 2, dtype=torch.int32)
    w = torch.zeros(8, 2, dtype=torch.float32)
    with pytest.raises(TypeError):
        binding.routing(idx.float(), w)
    with pytest.raises(TypeError):
        binding.routing(idx, w.double())
    with pytest.raises(ValueError):
        binding.routing(idx, w[:, :1].contiguous())
    with pytest.raises(ValueError):
        binding.routing(idx, w, N=9)
    with pytest.raises(ValueError):
        binding.routing(idx.reshape(-1), w.reshape(-1))          # a table must be [N,K]
    with pytest.raises(ValueError):
        binding.routing(idx.t(), w.t())                          # not contiguous
    e = torch.zeros(16, dtype=torch.int64)
    with pytest.raises(ValueError):
        binding.routing(e, torch.zeros(16), token_idx=e)         # a pair list needs N
    with pytest.raises(TypeError):
        binding.routing(e, torch.zeros(16), token_idx=e.int(), N=4)   # tokens and experts share a dtype
    with pytest.raises(ValueError):
        binding.routing(e, torch.zeros(16), token_idx=torch.zeros(15, dtype=torch.int64), N=4)


def test_routed_workspace_rejects_bad_descriptor():
    r = binding.routing(torch.zeros(8, 2, dtype=torch.int32), torch.zeros(8, 2))
    with pytest.raises(binding.MoeError):
        binding.routed_workspace_bytes(r, 128, 128, 0)           # no experts
    with pytest.raises(binding.MoeError):
        binding.routed_workspace_bytes(r, 96, 128, 8)            # H not a multiple of 64
    with pytest.raises(binding.MoeError):
        binding.workspace_bytes(8, 128, 128, 8, 33)              # K above 32


def test_ep_pointer_tables():
    R = 3
    xs = [torch.zeros(5 + d, 16, dtype=torch.bfloat16) for d in range(R)]
    ids = [torch.zeros(5 + d, 4, dtype=torch.int32) for d in range(R)]
    ws = [torch.zeros(5 + d, 4, dtype=torch.float32) for d in range(R)]
    err = torch.zeros(1, dtype=torch.int32)
    p = binding.ep_peers(xs, ids, ws, [0, 2, 4], err=err)
    for d in range(R):
        assert p.recv_x[d] == xs[d].data_ptr() and p.recv_idx[d] == ids[d].data_ptr()
        assert p.recv_w[d] == ws[d].data_ptr()
        assert p.row_off[d] == 2 * d and p.recv_rows[d] == 5 + d
    assert not p.recv_x[R] and p.err_word == err.data_ptr()
    # raw addresses need explicit row counts
    with pytest.raises(ValueError):
        binding.ep_peers([1 << 20] * R, [1 << 20] * R, [1 << 20] * R, [0] * R)
    p2 = binding.ep_peers([1 << 20] * R, [1 << 21] * R, [1 << 22] * R, [0] * R, recv_rows=[7, 8, 9])
    assert list(p2.recv_rows)[:R] == [7, 8, 9] and p2.recv_x[0] == 1 << 20
    with pytest.raises(ValueError):
        binding.ep_peers(xs, ids[:2], ws, [0, 0, 0])              # one entry per rank
    with pytest.raises(ValueError):
        binding.ep_peers([xs[0]] * 33, [ids[0]] * 33, [ws[0]] * 33, [0] * 33)
    s = binding.ep_sources(xs, [1, 2, 3])
    assert [s.local_out[d] for d in range(R)] == [x.data_ptr() for x in xs]
    assert list(s.rows)[:R] == [5, 6, 7] and list(s.row_off)[:R] == [1, 2, 3] and not s.err_word
    with pytest.raises(ValueError):
        binding.ep_sources(xs, [0, 0])
    # the tables are what the C ABI receives
    assert ctypes.sizeof(p) == binding.EP_MAX_RANKS * (3 * 8 + 2 * 8) + 8
    assert ctypes.sizeof(s) == binding.EP_MAX_RANKS * (8 + 8 + 8) + 8


def test_tensor_checks():
    t = torch.zeros(4, 8, dtype=torch.float32)
    binding._need(t, "t", torch.float32, (4, 8), t.device)
    with pytest.raises(TypeError):
        binding._need(t, "t", torch.bfloat16, (4, 8), t.device)
    with pytest.raises(ValueError):
        binding._need(t, "t", torch.float32, (8, 4), t.device)
    with pytest.raises(ValueError):
        binding._need(t.t(), "t", torch.float32, (8, 4), t.device)
    with pytest.raises(ValueError):
        binding._need(t, "t", torch.float32, (4, 8), torch.device("meta"))
    assert binding.p_cap(10, 3) == 30 and binding.p_cap(10, 3, 7) == 7
