// Expert-parallel dispatch and combine around the local path, non-expand
// ("End-to-end DeepEP v2 non-expand + SonicMoE integration #68": dispatch ->
// recv_x / recv_topk_idx (local ids, -1 for slots whose expert lives on
// another rank) / recv_topk_weights -> local expert compute -> local_out ->
// combine -> routed_out).  A token row travels once to each rank owning one
// of its experts.
//
//   layout    one CTA walks the source's tokens in chunks (ids read and rows
//             written through shared memory, coalesced): each thread
//             forms its token's destination mask, warp ballots per destination
//             give the token's rank inside its warp, a shuffle scan over the
//             warps (one warp per destination) and a running base give its
//             row inside each destination's block (stable: tokens ascending).
//   dispatch  one CTA per token (grid-stride): each thread loads 16-byte chunks
//             of x[t] once and stores them to every destination's receive
//             rows; stores to another GPU's buffers go over NVLink as plain
//             peer stores (no TMA, no multicast).
//   combine   one CTA per token: each thread sums its chunk of the
//             destinations' local_out rows in ascending rank order in fp32
//             (peer loads) and writes one bf16 rounding.
//
// The phases are ordered across ranks by the caller (a barrier between
// dispatch and the local forward, and between the forward and the combine);
// no kernel here waits on another rank.
#include "common.cuh"
#include "ep.cuh"

namespace moe {

namespace {

constexpr int kLayoutThreads = 1024;
constexpr int kLayoutWarps = kLayoutThreads / 32;
constexpr int kEpThreads = 256;

constexpr int kLayoutStage = 8192;  // ints staged per chunk (32 KB): ids in, then rows out

__global__ void __launch_bounds__(kLayoutThreads, 1) ep_layout_kernel(const int32_t *__restrict__ topk_idx,
                                                                     int64_t T, int K, int R, int E_local,
                                                                     int32_t *__restrict__ send_idx,
                                                                     int32_t *__restrict__ send_count,
                                                                     uint32_t *err) {
    __shared__ int stage[kLayoutStage];                            // a chunk's ids, then its send_idx rows
    __shared__ int warp_base[kLayoutWarps][MOE_EP_MAX_RANKS + 1];  // per warp and destination
    __shared__ int run[MOE_EP_MAX_RANKS];                          // rows given out so far
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const unsigned lt = (1u << lane) - 1u;
    const int64_t n_exp = (int64_t)R * E_local;
    // tokens per chunk: both the chunk's [C,K] ids and its [C,R] rows fit the stage
    const int C = min(kLayoutThreads, kLayoutStage / max(K, R));
    if (tid < MOE_EP_MAX_RANKS) run[tid] = 0;
    bool bad = false;
    for (int64_t t0 = 0; t0 < T; t0 += C) {
        const int nt = (int)min((int64_t)C, T - t0);
        __syncthreads();  // the stage's previous rows have been written out
        for (int i = tid; i < nt * K; i += kLayoutThreads) stage[i] = __ldg(topk_idx + t0 * K + i);  // coalesced
        __syncthreads();
        uint32_t mask = 0;
        if (tid < nt) {
            for (int k = 0; k < K; ++k) {
                const int e = stage[tid * K + k];
                if (e >= 0 && e < n_exp) mask |= 1u << (e / E_local);
                else if (e != -1) bad = true;
            }
        }
        int pre[MOE_EP_MAX_RANKS];  // this token's rank among its warp's tokens bound for d
#pragma unroll
        for (int d = 0; d < MOE_EP_MAX_RANKS; ++d) {
            if (d < R) {
                const unsigned b = __ballot_sync(0xffffffffu, (mask >> d) & 1u);
                pre[d] = __popc(b & lt);
                if (lane == 0) warp_base[warp][d] = __popc(b);
            }
        }
        __syncthreads();  // counts in; every thread has read its ids from the stage
        if (warp < R) {  // warp d: exclusive scan over the 32 warps' counts for destination d
            const int d = warp;
            const int c = warp_base[lane][d];
            int v = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += u;
            }
            const int base = run[d];
            warp_base[lane][d] = base + v - c;
            __syncwarp();
            if (lane == 31) run[d] = base + v;
        }
        __syncthreads();
        if (tid < nt) {
#pragma unroll
            for (int d = 0; d < MOE_EP_MAX_RANKS; ++d)
                if (d < R) stage[tid * R + d] = ((mask >> d) & 1u) ? warp_base[warp][d] + pre[d] : -1;
        }
        __syncthreads();
        for (int i = tid; i < nt * R; i += kLayoutThreads) send_idx[t0 * R + i] = stage[i];  // coalesced
    }
    __syncthreads();
    if (tid < R) send_count[tid] = run[tid];
    if (bad && err) atomicOr(err, MOE_DEVERR_BAD_EXPERT_ID);
}

__global__ void __launch_bounds__(kEpThreads) ep_dispatch_kernel(const uint4 *__restrict__ x,
                                                                const int32_t *__restrict__ topk_idx,
                                                                const float *__restrict__ topk_w,
                                                                const int32_t *__restrict__ send_idx, int64_t T,
                                                                int H, int K, int R, int E_local,
                                                                const moe_ep_peers_t peers) {
    __shared__ int64_t row[MOE_EP_MAX_RANKS];  // destination row of this token, or -1
    const int chunks = H >> 3;
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        if (threadIdx.x < R) {
            const int j = __ldg(send_idx + t * R + threadIdx.x);
            int64_t r = j >= 0 ? peers.row_off[threadIdx.x] + j : -1;
            if (r >= peers.recv_rows[threadIdx.x]) {  // past the destination's buffer: not written
                if (peers.err_word) atomicOr(peers.err_word, MOE_DEVERR_ABORTED);
                r = -1;
            }
            row[threadIdx.x] = r;
        }
        __syncthreads();
        const uint4 *src = x + t * chunks;
        for (int c = threadIdx.x; c < chunks; c += kEpThreads) {
            const uint4 v = __ldg(src + c);
            for (int d = 0; d < R; ++d)
                if (row[d] >= 0) reinterpret_cast<uint4 *>(peers.recv_x[d])[row[d] * chunks + c] = v;
        }
        if (threadIdx.x < K) {
            const int k = threadIdx.x;
            const int e = __ldg(topk_idx + t * K + k);
            const float w = __ldg(topk_w + t * K + k);
            for (int d = 0; d < R; ++d) {
                if (row[d] < 0) continue;
                const bool on = e >= 0 && e / E_local == d && e < R * E_local;
                peers.recv_idx[d][row[d] * K + k] = on ? e - d * E_local : -1;
                peers.recv_w[d][row[d] * K + k] = on ? w : 0.f;
            }
        }
        __syncthreads();  // row[] is rewritten by the next token
    }
}

__global__ void __launch_bounds__(kEpThreads) ep_combine_kernel(const moe_ep_sources_t src,
                                                               const int32_t *__restrict__ send_idx, int64_t T,
                                                               int H, int R, uint4 *__restrict__ out) {
    // the token's destinations in ascending rank order, compacted: their row pointers
    __shared__ const uint4 *vrow[MOE_EP_MAX_RANKS];
    __shared__ int nv;
    const int chunks = H >> 3;
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        if (threadIdx.x < 32) {
            const int lane = threadIdx.x;
            int j = lane < R ? __ldg(send_idx + t * R + lane) : -1;
            if (j >= 0 && src.row_off[lane] + j >= src.rows[lane]) {  // past the buffer: not read
                if (src.err_word) atomicOr(src.err_word, MOE_DEVERR_ABORTED);
                j = -1;
            }
            const unsigned b = __ballot_sync(0xffffffffu, j >= 0);
            if (j >= 0)
                vrow[__popc(b & ((1u << lane) - 1u))] =
                    reinterpret_cast<const uint4 *>(src.local_out[lane]) + (src.row_off[lane] + j) * chunks;
            if (lane == 0) nv = __popc(b);
        }
        __syncthreads();
        const int n = nv;
        for (int c = threadIdx.x; c < chunks; c += kEpThreads) {
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            for (int i0 = 0; i0 < n; i0 += 4) {  // four rows in flight, added in ascending rank order
                uint4 v[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) v[u] = i0 + u < n ? vrow[i0 + u][c] : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    if (i0 + u >= n) break;
                    const uint32_t q[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        acc[2 * i] += bf16lo(q[i]);
                        acc[2 * i + 1] += bf16hi(q[i]);
                    }
                }
            }
            out[t * chunks + c] = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                                             pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
        }
        __syncthreads();
    }
}

int64_t grid_for(int64_t T, int num_sms) {
    int64_t blocks = T;
    const int64_t cap = (int64_t)num_sms * 8;
    if (blocks > cap) blocks = cap;
    return blocks < 1 ? 1 : blocks;
}

}  // namespace

cudaError_t launch_ep_layout(const int32_t *topk_idx, int64_t T, int K, int R, int E_local, int32_t *send_idx,
                             int32_t *send_count, uint32_t *err, cudaStream_t s) {
    ep_layout_kernel<<<1, kLayoutThreads, 0, s>>>(topk_idx, T, K, R, E_local, send_idx, send_count, err);
    return cudaGetLastError();
}

cudaError_t launch_ep_dispatch(const void *x, const int32_t *topk_idx, const float *topk_w, const int32_t *send_idx,
                               int64_t T, int H, int K, int R, int E_local, const moe_ep_peers_t &peers,
                               int num_sms, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    ep_dispatch_kernel<<<(unsigned)grid_for(T, num_sms), kEpThreads, 0, s>>>(
        static_cast<const uint4 *>(x), topk_idx, topk_w, send_idx, T, H, K, R, E_local, peers);
    return cudaGetLastError();
}

cudaError_t launch_ep_combine(const moe_ep_sources_t &src, const int32_t *send_idx, int64_t T, int H, int R, void *out,
                              int num_sms, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    ep_combine_kernel<<<(unsigned)grid_for(T, num_sms), kEpThreads, 0, s>>>(src, send_idx, T, H, R,
                                                                            static_cast<uint4 *>(out));
    return cudaGetLastError();
}

}  // namespace moe
