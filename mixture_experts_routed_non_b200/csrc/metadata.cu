// Routing metadata of the non-expand layout, built straight from [N,K]
// (sonic-moe issue #68, "End-to-end DeepEP v2 non-expand + SonicMoE
// integration": the metadata list -- expert_frequency,
// expert_frequency_offset, x_gather_idx, s_scatter_idx,
// s_reverse_scatter_idx, num_activated_expert_per_token_offset, compact
// router_scores -- and question 3: pairs are numbered in ascending token
// order).  The sort by expert is a stable counting sort (the segmented-sort
// recipe of the qwen3_5.py commit notes, steps 1-2), done in two kernels:
//
//   meta_count_kernel   one CTA per tile of slots: expert histogram in shared
//                       memory (match_any aggregation), per-tile valid count.
//                       The last CTA to finish (atomic ticket, no waiting)
//                       scans: totals, offsets, per-(tile,expert) bases,
//                       per-tile pair bases and the GEMM tile table.
//   meta_scatter_kernel one CTA per tile again: each warp owns a contiguous
//                       slice of the tile; per-warp counts give each warp its
//                       base per expert, and inside a 32-slot step the rank of
//                       a slot among equal experts is popc(peers & lanes
//                       below).  Every result is a pure function of the input
//                       (no atomics decide an order), so the output is
//                       bit-exact and deterministic.
#include "common.cuh"

namespace moe {

namespace {

constexpr unsigned kFull = 0xffffffffu;

// Exclusive scan of n ints from `in` into `out` (either may be shared or
// global; in == out allowed) by the whole block; returns the total.
__device__ int block_exclusive_scan(const int *in, int *out, int n, bool in_global) {
    __shared__ int warp_tot[kMetaWarps];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int carry = 0;
    for (int base = 0; base < n; base += 2 * kMetaThreads) {
        const int i0 = base + 2 * threadIdx.x, i1 = i0 + 1;
        int v0 = 0, v1 = 0;
        if (in_global) {
            if (i0 < n) v0 = __ldcg(in + i0);
            if (i1 < n) v1 = __ldcg(in + i1);
        } else {
            if (i0 < n) v0 = in[i0];
            if (i1 < n) v1 = in[i1];
        }
        const int s = v0 + v1;
        int x = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(kFull, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) warp_tot[warp] = x;
        __syncthreads();
        if (warp == 0) {
            int w = lane < kMetaWarps ? warp_tot[lane] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(kFull, w, o);
                if (lane >= o) w += y;
            }
            if (lane < kMetaWarps) warp_tot[lane] = w;  // inclusive
        }
        __syncthreads();
        const int excl = carry + (warp ? warp_tot[warp - 1] : 0) + x - s;
        if (i0 < n) out[i0] = excl;
        if (i1 < n) out[i1] = excl + v0;
        carry += warp_tot[kMetaWarps - 1];
        __syncthreads();
    }
    return carry;
}

// Shared memory of the count kernel / last-block scan (ints).
constexpr int kScanPart = kMaxExperts;          // part[G*E] (G*E <= max(E, kMetaThreads))
constexpr int kCountSmemInts = kScanPart + 3 * (kMaxExperts + 1) + 8;

__device__ void last_block_scan(const MetaArgs &a, int *sm) {
    const int E = a.E, T = a.tiles;
    int *part = sm;                             // [G][E]
    int *freq = sm + kScanPart;                 // [E]
    int *off = freq + (kMaxExperts + 1);        // [E+1]
    int *gtile = off + (kMaxExperts + 1);       // [E+1]
    __shared__ unsigned s_err;

    int G = E <= kMetaThreads ? kMetaThreads / E : 1;
    if (G > T) G = T;
    const int chunk = (T + G - 1) / G;

    // 1. per-group partial column sums of the tile histograms
    for (int i = threadIdx.x; i < G * E; i += kMetaThreads) {
        const int g = i / E, e = i - g * E;
        const int t0 = g * chunk, t1 = min(T, t0 + chunk);
        int sum = 0;
        int t = t0;
        for (; t + 4 <= t1; t += 4) {
            const int v0 = __ldcg(a.tile_hist + (size_t)(t + 0) * E + e);
            const int v1 = __ldcg(a.tile_hist + (size_t)(t + 1) * E + e);
            const int v2 = __ldcg(a.tile_hist + (size_t)(t + 2) * E + e);
            const int v3 = __ldcg(a.tile_hist + (size_t)(t + 3) * E + e);
            sum += v0 + v1 + v2 + v3;
        }
        for (; t < t1; ++t) sum += __ldcg(a.tile_hist + (size_t)t * E + e);
        part[i] = sum;
    }
    if (threadIdx.x == 0) s_err = 0;
    __syncthreads();
    // 2. per expert: exclusive prefix over groups, total = frequency
    for (int e = threadIdx.x; e < E; e += kMetaThreads) {
        int run = 0;
        for (int g = 0; g < G; ++g) {
            const int v = part[g * E + e];
            part[g * E + e] = run;
            run += v;
        }
        freq[e] = run;
        gtile[e] = (run + kBM - 1) / kBM;
    }
    __syncthreads();
    // 3. offsets and GEMM tile table
    const int P = block_exclusive_scan(freq, off, E, false);
    const int GT = block_exclusive_scan(gtile, gtile, E, false);
    for (int e = threadIdx.x; e < E; e += kMetaThreads) {
        a.meta.expert_frequency[e] = freq[e];
        a.meta.expert_frequency_offset[e] = off[e];
        a.gemm_tile_off[e] = gtile[e];
    }
    if (threadIdx.x == 0) {
        off[E] = P;
        a.meta.expert_frequency_offset[E] = P;
        a.gemm_tile_off[E] = GT;
    }
    __syncthreads();
    // 4. per-(tile, expert) global bases, written over the histograms
    for (int i = threadIdx.x; i < G * E; i += kMetaThreads) {
        const int g = i / E, e = i - g * E;
        const int t0 = g * chunk, t1 = min(T, t0 + chunk);
        int base = off[e] + part[i];
        for (int t = t0; t < t1; ++t) {
            int *cell = a.tile_hist + (size_t)t * E + e;
            const int v = __ldcg(cell);
            *cell = base;
            base += v;
        }
    }
    // 5. per-tile pair bases
    block_exclusive_scan(a.tile_valid, a.tile_pbase, T, true);
    // 6. errors of this call, pair-count check, abort decision
    unsigned err = 0;
    for (int t = threadIdx.x; t < T; t += kMetaThreads) err |= (unsigned)__ldcg(a.tile_err + t);
    if (err) atomicOr(&s_err, err);
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned e = s_err;
        unsigned abort = 0;
        if (a.total_pairs >= 0 && (int64_t)P != a.total_pairs) e |= MOE_DEVERR_PAIR_COUNT;
        if ((int64_t)P > a.p_cap) {
            e |= MOE_DEVERR_PAIR_COUNT | MOE_DEVERR_ABORTED;
            abort = 1;
        }
        a.meta.token_offset[a.N] = P;
        a.hdr->P = P;
        a.hdr->err = e;
        a.hdr->abort = abort;
        __threadfence();
        a.hdr->ticket = 0;  // ready for the next call
    }
}

__global__ void __launch_bounds__(kMetaThreads) meta_count_kernel(const MetaArgs a) {
    extern __shared__ int sm[];
    __shared__ int s_valid;
    __shared__ unsigned s_err;
    __shared__ int s_last;
    int *hist = sm;
    const int E = a.E;
    const int lane = threadIdx.x & 31;
    for (int e = threadIdx.x; e < E; e += kMetaThreads) hist[e] = 0;
    if (threadIdx.x == 0) {
        s_valid = 0;
        s_err = 0;
    }
    __syncthreads();

    const int tile = blockIdx.x;
    const int s0 = tile * a.tile_slots;
    const int s1 = (int)min((int64_t)s0 + a.tile_slots, a.NK);
    int my_valid = 0;
    unsigned my_err = 0;
    for (int base = s0; base < s1; base += kMetaThreads) {  // same trip count in every thread
        const int s = base + threadIdx.x;
        const int e = s < s1 ? __ldg(a.topk_idx + s) : -1;
        const bool valid = (e >= 0) && (e < E);
        if (!valid && e != -1) my_err = MOE_DEVERR_BAD_EXPERT_ID;
        const unsigned peers = __match_any_sync(kFull, valid ? e : -1);
        if (valid && lane == __ffs(peers) - 1) atomicAdd(&hist[e], __popc(peers));
        const unsigned vb = __ballot_sync(kFull, valid);
        my_valid += __popc(vb);
    }
    if (lane == 0 && my_valid) atomicAdd(&s_valid, my_valid);
    if (my_err) atomicOr(&s_err, my_err);
    __syncthreads();
    int *th = a.tile_hist + (size_t)tile * E;
    for (int e = threadIdx.x; e < E; e += kMetaThreads) th[e] = hist[e];
    if (threadIdx.x == 0) {
        a.tile_valid[tile] = s_valid;
        a.tile_err[tile] = (int)s_err;
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned t = atomicAdd(&a.hdr->ticket, 1u);
        s_last = (t == (unsigned)(a.tiles - 1));
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    last_block_scan(a, sm);
}

__global__ void __launch_bounds__(kMetaThreads) meta_scatter_kernel(const MetaArgs a) {
    extern __shared__ int cnt[];  // [kMetaWarps][E]: per-warp running base of each expert
    __shared__ int wq[kMetaWarps];
    if (*(volatile uint32_t *)&a.hdr->abort) return;
    const int E = a.E, K = a.K;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t lt = lanemask_lt();
    const int tile = blockIdx.x;
    for (int i = threadIdx.x; i < kMetaWarps * E; i += kMetaThreads) cnt[i] = 0;
    __syncthreads();

    const int s0 = tile * a.tile_slots;
    const int s1 = (int)min((int64_t)s0 + a.tile_slots, a.NK);
    const int sub = a.tile_slots / kMetaWarps;
    const int w0 = s0 + warp * sub;
    const int w1 = min(w0 + sub, s1);
    int *mycnt = cnt + warp * E;

    // pass 1: per-warp counts of each expert and of valid slots
    int nvalid = 0;
    for (int base = w0; base < w1; base += 32) {
        const int s = base + lane;
        const int e = s < w1 ? __ldg(a.topk_idx + s) : -1;
        const bool valid = (e >= 0) && (e < E);
        const unsigned peers = __match_any_sync(kFull, valid ? e : -1);
        if (valid && lane == __ffs(peers) - 1) mycnt[e] += __popc(peers);
        nvalid += __popc(__ballot_sync(kFull, valid));
        __syncwarp();
    }
    if (lane == 0) wq[warp] = nvalid;
    __syncthreads();

    // bases: the tile's global base per expert (from the scan) plus the
    // counts of the warps before this one
    for (int e = threadIdx.x; e < E; e += kMetaThreads) {
        int run = __ldcg(a.tile_hist + (size_t)tile * E + e);
        for (int w = 0; w < kMetaWarps; ++w) {
            const int c = cnt[w * E + e];
            cnt[w * E + e] = run;
            run += c;
        }
    }
    if (threadIdx.x == 0) {
        int run = __ldcg(a.tile_pbase + tile);
        for (int w = 0; w < kMetaWarps; ++w) {
            const int c = wq[w];
            wq[w] = run;
            run += c;
        }
    }
    __syncthreads();

    // pass 2: positions, in slot order
    int q_run = wq[warp];
    for (int base = w0; base < w1; base += 32) {
        const int s = base + lane;
        const bool in = s < w1;
        const int e = in ? __ldg(a.topk_idx + s) : -1;
        const bool valid = (e >= 0) && (e < E);
        const unsigned peers = __match_any_sync(kFull, valid ? e : -1);
        const int pbase = valid ? mycnt[e] : 0;
        __syncwarp();
        if (valid && lane == __ffs(peers) - 1) mycnt[e] = pbase + __popc(peers);
        const unsigned vb = __ballot_sync(kFull, valid);
        const int q = q_run + __popc(vb & lt);
        if (valid) {
            const int p = pbase + __popc(peers & lt);
            const int t = s / K;
            a.meta.x_gather_idx[p] = t;
            a.meta.s_scatter_idx[p] = q;
            a.meta.s_reverse_scatter_idx[q] = p;
            a.meta.scores[q] = __ldg(a.topk_w + s);
        }
        if (in && (s % K) == 0) a.meta.token_offset[s / K] = q;
        q_run += __popc(vb);
        __syncwarp();
    }
}

}  // namespace

cudaError_t launch_meta(const MetaArgs &a, cudaStream_t s) {
    static_assert(kCountSmemInts * 4 <= 48 * 1024, "count kernel shared memory");
    meta_count_kernel<<<a.tiles, kMetaThreads, kCountSmemInts * sizeof(int), s>>>(a);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    const size_t scatter_smem = (size_t)kMetaWarps * a.E * sizeof(int);
    if (scatter_smem > 48 * 1024) {
        err = cudaFuncSetAttribute(meta_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)(kMetaWarps * kMaxExperts * sizeof(int)));
        if (err != cudaSuccess) return err;
    }
    meta_scatter_kernel<<<a.tiles, kMetaThreads, scatter_smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace moe
