"""CPU oracle of expert-parallel dispatch and combine around the local path.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
legs of ``bench.py`` may use it; the product path never does.  Plain Python
loops over tokens, slots and ranks (small cases only); it shares no code with
the CUDA library.

What it computes follows "End-to-end DeepEP v2 non-expand + SonicMoE
integration #68": a dispatch in non-expand mode hands each rank
``recv_x [N_recv, H]``, ``recv_topk_idx [N_recv, K]`` (local expert ids, -1 for
a slot whose expert lives elsewhere) and ``recv_topk_weights``; the local
expert compute turns them into ``local_out [N_recv, H]``; the combine returns
``routed_out [T, H]`` in the source's token order.  Non-expand means a token
row travels once to each destination rank that owns at least one of its
experts, not once per expert.  The Neuron unpermute-a2av page describes the
same combine as a scatter-add of every destination's contribution back to the
token's original row.

Readings where the pages leave the layout open (used identically by the
CUDA path, which is checked against this):

- expert ``e`` (global id) lives on rank ``e // E_local`` as local expert
  ``e % E_local``; an id outside ``[0, R * E_local)`` other than -1 is not
  sent (and the layout step flags it);
- a destination's receive rows are blocks by source rank in rank order, and
  inside a block the source's tokens in ascending order;
- the combine adds the destinations' rows in ascending rank order.
"""
from __future__ import annotations

import numpy as np


def ep_layout(topk_idx: np.ndarray, R: int, E_local: int):
    """Per source rank: ``send_idx [T, R]`` (the token's row inside its block
    for destination d, or -1 when d owns none of its experts) and
    ``counts [R]`` (rows sent to each destination)."""
    T, K = topk_idx.shape
    send_idx = np.full((T, R), -1, np.int32)
    counts = np.zeros(R, np.int64)
    for t in range(T):
        dests = set()
        for k in range(K):
            e = int(topk_idx[t, k])
            if 0 <= e < R * E_local:
                dests.add(e // E_local)
        for d in sorted(dests):
            send_idx[t, d] = counts[d]
            counts[d] += 1
    return send_idx, counts


def recv_offsets(count_matrix: np.ndarray):
    """``count_matrix[s, d]`` rows from source s to destination d ->
    ``off[d, s]`` (first receive row of source s's block on d) and
    ``n_recv[d]``."""
    R = count_matrix.shape[0]
    off = np.zeros((R, R), np.int64)
    n_recv = np.zeros(R, np.int64)
    for d in range(R):
        acc = 0
        for s in range(R):
            off[d, s] = acc
            acc += int(count_matrix[s, d])
        n_recv[d] = acc
    return off, n_recv


def ep_dispatch(xs, idxs, ws, R: int, E_local: int) -> dict:
    """Dispatch of R source ranks' (x [T_s, H], topk_idx [T_s, K] global ids,
    topk_w [T_s, K]).  Rows of x are copied exactly (any dtype)."""
    layouts = [ep_layout(np.asarray(idxs[s]), R, E_local) for s in range(R)]
    C = np.stack([c for _, c in layouts])
    off, n_recv = recv_offsets(C)
    K = np.asarray(idxs[0]).shape[1]
    H = np.asarray(xs[0]).shape[1]
    recv_x = [np.zeros((int(n_recv[d]), H), np.asarray(xs[0]).dtype) for d in range(R)]
    recv_idx = [np.full((int(n_recv[d]), K), -1, np.int32) for d in range(R)]
    recv_w = [np.zeros((int(n_recv[d]), K), np.float32) for d in range(R)]
    for s in range(R):
        x, idx, w = np.asarray(xs[s]), np.asarray(idxs[s]), np.asarray(ws[s])
        send_idx = layouts[s][0]
        for t in range(idx.shape[0]):
            for d in range(R):
                j = int(send_idx[t, d])
                if j < 0:
                    continue
                row = int(off[d, s]) + j
                recv_x[d][row] = x[t]
                for k in range(K):
                    e = int(idx[t, k])
                    if 0 <= e < R * E_local and e // E_local == d:
                        recv_idx[d][row, k] = e - d * E_local
                        recv_w[d][row, k] = w[t, k]
    return {"recv_x": recv_x, "recv_idx": recv_idx, "recv_w": recv_w, "send_idx": [l[0] for l in layouts],
            "counts": C, "off": off, "n_recv": n_recv}


def ep_combine(local_outs, send_idxs, off: np.ndarray):
    """``routed_out`` of every source rank (float64): for token t of source s,
    the sum over destinations d (ascending) with ``send_idx[t, d] >= 0`` of
    ``local_outs[d][off[d, s] + send_idx[t, d]]``; a token sent nowhere is 0."""
    R = len(local_outs)
    outs = []
    for s in range(R):
        si = np.asarray(send_idxs[s])
        T = si.shape[0]
        H = np.asarray(local_outs[0]).shape[1]
        out = np.zeros((T, H), np.float64)
        for t in range(T):
            for d in range(R):
                j = int(si[t, d])
                if j >= 0:
                    out[t] += np.asarray(local_outs[d][int(off[d, s]) + j], np.float64)
        outs.append(out)
    return outs
