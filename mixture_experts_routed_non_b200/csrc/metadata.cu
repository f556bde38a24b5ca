// Routing metadata of the non-expand layout, built straight from [N,K]
// (sonic-moe issue #68, "End-to-end DeepEP v2 non-expand + SonicMoE
// integration": the metadata list -- expert_frequency,
// expert_frequency_offset, x_gather_idx, s_scatter_idx,
// s_reverse_scatter_idx, num_activated_expert_per_token_offset, compact
// router_scores -- and question 3: pairs are numbered in ascending token
// order).  The sort by expert is a stable counting sort (the segmented-sort
// recipe of the qwen3_5.py commit notes, steps 1-2) done by one cooperative
// kernel over T tiles of consecutive slots (T <= number of SMs, one CTA each):
//
//   phase A  each warp of a tile owns a contiguous slice of its slots and
//            counts the experts in it (shared-memory increments into a row of
//            its own: integer counts, so their order does not matter); the
//            tile's histogram, valid count and error bits go to the workspace.
//   barrier  all T CTAs (co-resident by the cooperative launch) meet at a
//            bounded grid barrier whose counter the host clears per call.
//   phase B  every CTA reads the whole (small) [T,E] histogram table and
//            derives the global offsets, its tile's base per expert and its
//            pair base; its warps' bases follow from the per-warp counts of
//            phase A; then each warp ranks its slice (match_any finds the
//            lanes with the same expert, popc(peers & lanes below) orders
//            them inside each 32-slot step) and writes the outputs.  CTA 0
//            also writes the histogram, offsets, the GEMM tile table and the
//            call's error word.
//
// Every result is a pure function of the input (no atomic decides an order;
// the grid barrier is a GPU-scope release add polled with acquire loads),
// so the output is bit-exact and deterministic.  Each lane keeps kV slots in
// flight; the first kWarpChunk slots of every warp, and their weights, stay in
// registers from phase A to phase B.
#include "common.cuh"

namespace moe {

namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kV = 8;                     // slots per lane per step
constexpr int kWarpChunk = 32 * kV;       // slots per warp step
constexpr unsigned long long kGridBarrierTimeoutNs = 1000000000ull;
static_assert(kMetaMaxTiles < kMetaThreads, "phase B reads one tile's counts per thread");

// The grid barrier's arrival: a GPU-scope release add (the block's earlier
// writes, ordered before it by __syncthreads, become visible with it) and an
// acquire load for the polling.
__device__ __forceinline__ void red_add_release_gpu(uint32_t *p, uint32_t v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Exclusive scan of n ints in shared memory (in place allowed) by the whole
// block; returns the total.
__device__ int block_exclusive_scan(const int *in, int *out, int n) {
    __shared__ int warp_tot[kMetaWarps];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int carry = 0;
    for (int base = 0; base < n; base += 2 * kMetaThreads) {
        const int i0 = base + 2 * threadIdx.x, i1 = i0 + 1;
        const int v0 = i0 < n ? in[i0] : 0;
        const int v1 = i1 < n ? in[i1] : 0;
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

// Sum over the block of one int per thread.
__device__ int block_sum(int v) {
    __shared__ int part[kMetaWarps];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    if (lane == 0) part[warp] = v;
    __syncthreads();
    int t = 0;
#pragma unroll
    for (int w = 0; w < kMetaWarps; ++w) t += part[w];
    __syncthreads();
    return t;
}

// An id read as int: int64 values are clamped to the int range, which keeps
// their order and keeps every out-of-range id out of range (and off -1).
template <bool kIdx64>
__device__ __forceinline__ int load_id(const void *ids, int s) {
    if (kIdx64) {
        const long long v = __ldg(static_cast<const long long *>(ids) + s);
        return (int)max(min(v, 0x7fffffffLL), -0x80000000LL);
    }
    return __ldg(static_cast<const int *>(ids) + s);
}

// An id at its own width (for the order check of a pair list's tokens).
template <bool kIdx64>
__device__ __forceinline__ long long load_id_wide(const void *ids, int s) {
    return kIdx64 ? __ldg(static_cast<const long long *>(ids) + s) : (long long)__ldg(static_cast<const int *>(ids) + s);
}

template <bool kIdx64>
__device__ __forceinline__ void load_chunk(const void *ids, int base, int end, int lane, int (&e)[kV]) {
#pragma unroll
    for (int v = 0; v < kV; ++v) {
        const int s = base + 32 * v + lane;
        e[v] = s < end ? load_id<kIdx64>(ids, s) : -1;
    }
}

// Token of slot s: s / K for the [N,K] table, token_idx[s] for a pair list.
template <bool kPairs, bool kIdx64>
__device__ __forceinline__ int slot_token(const MetaArgs &a, int s) {
    return kPairs ? load_id<kIdx64>(a.token_idx, s) : s / a.K;
}

// A slot becomes a pair when its expert id is in [0,E) and (pair list) its
// token id is in [0,N).  Sets *bad for ids that are neither valid nor -1.
template <bool kPairs>
__device__ __forceinline__ bool slot_valid(const MetaArgs &a, int e, int t, unsigned *bad) {
    const bool e_ok = (e >= 0) && (e < a.E);
    if (!e_ok && e != -1) *bad |= MOE_DEVERR_BAD_EXPERT_ID;
    if (kPairs && e_ok && (t < 0 || (int64_t)t >= a.N)) {
        *bad |= MOE_DEVERR_BAD_TOKEN;
        return false;
    }
    return e_ok;
}

// Shared memory (ints): cnt[kMetaWarps][E] | part_all[kPartInts] | part_before[kPartInts]
//                       | off[kMaxExperts+1] | gt[kMaxExperts+1]
constexpr int kPartInts = kMaxExperts;   // G*E <= max(kMetaThreads, E) <= kMaxExperts

template <bool kPairs, bool kIdx64>
__global__ void __launch_bounds__(kMetaThreads, 1) meta_kernel(const MetaArgs a) {
    extern __shared__ int sm[];
    const int E = a.E, K = a.K, T = a.tiles;
    int *cnt = sm;
    int *part_all = cnt + kMetaWarps * E;
    int *part_before = part_all + kPartInts;
    int *off = part_before + kPartInts;
    int *gt = off + (kMaxExperts + 1);
    __shared__ int wq[kMetaWarps];
    __shared__ unsigned s_err;
    __shared__ int s_bar_ok;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t lt = lanemask_lt();
    const int tile = blockIdx.x;

    // this warp's contiguous slice of the tile
    const int s0 = tile * a.tile_slots;
    const int s1 = (int)min((int64_t)s0 + a.tile_slots, a.NK);
    const int sub = a.tile_slots / kMetaWarps;
    const int w0 = s0 + warp * sub;
    const int w1 = min(w0 + sub, s1);
    int ev0[kV], tv0[kV];
    float wv0[kV];  // kept for phase B; an invalid slot's weight is never written
    load_chunk<kIdx64>(a.topk_idx, w0, w1, lane, ev0);
#pragma unroll
    for (int v = 0; v < kV; ++v) {
        const int s = w0 + 32 * v + lane;
        wv0[v] = s < w1 ? __ldg(a.topk_w + s) : 0.f;
        tv0[v] = (kPairs && s < w1) ? slot_token<kPairs, kIdx64>(a, s) : 0;
    }
    for (int i = threadIdx.x; i < kMetaWarps * E; i += kMetaThreads) cnt[i] = 0;
    if (threadIdx.x == 0) s_err = 0;
    __syncthreads();

    // ---- phase A: per-warp expert counts of the slice
    int *mycnt = cnt + warp * E;
    int nvalid = 0;
    unsigned my_err = 0;
    for (int base = w0; base < w1; base += kWarpChunk) {
        int ev[kV], tv[kV];
        if (base == w0) {
#pragma unroll
            for (int v = 0; v < kV; ++v) {
                ev[v] = ev0[v];
                tv[v] = tv0[v];
            }
        } else {
            load_chunk<kIdx64>(a.topk_idx, base, w1, lane, ev);
#pragma unroll
            for (int v = 0; v < kV; ++v) {
                const int s = base + 32 * v + lane;
                tv[v] = (kPairs && s < w1) ? slot_token<kPairs, kIdx64>(a, s) : 0;
            }
        }
#pragma unroll
        for (int v = 0; v < kV; ++v) {
            const int e = ev[v];
            const bool valid = slot_valid<kPairs>(a, e, tv[v], &my_err);
            if (kPairs) {  // a pair list must be in ascending token order
                const int s = base + 32 * v + lane;
                if (s > 0 && s < w1 &&
                    load_id_wide<kIdx64>(a.token_idx, s - 1) > load_id_wide<kIdx64>(a.token_idx, s))
                    my_err |= MOE_DEVERR_BAD_TOKEN;
            }
            if (valid) {  // integer counts: the order of the atomics does not matter
                atomicAdd(&mycnt[e], 1);
                ++nvalid;
            }
        }
    }
    nvalid = (int)__reduce_add_sync(kFull, (unsigned)nvalid);
    if (lane == 0) wq[warp] = nvalid;
    if (my_err) atomicOr(&s_err, my_err);
    __syncthreads();
    // tile histogram = sum of the warps' rows
    int *th = a.tile_hist + (size_t)tile * E;
    for (int e = threadIdx.x; e < E; e += kMetaThreads) {
        int sum = 0;
        for (int w = 0; w < kMetaWarps; ++w) sum += cnt[w * E + e];
        th[e] = sum;
    }
    if (threadIdx.x == 0) {
        int v = 0;
        for (int w = 0; w < kMetaWarps; ++w) v += wq[w];
        a.tile_valid[tile] = v;
        a.tile_err[tile] = (int)s_err;
    }

    // ---- grid barrier (bounded)
    __syncthreads();
    if (threadIdx.x == 0) {
        red_add_release_gpu(&a.hdr->grid_arrive, 1u);
        const uint64_t t0 = globaltimer_ns();
        int ok = 1;
        while (ld_acquire_gpu(&a.hdr->grid_arrive) < (uint32_t)T) {
            if (globaltimer_ns() - t0 > kGridBarrierTimeoutNs) {
                ok = 0;
                break;
            }
        }
        s_bar_ok = ok;
    }
    __syncthreads();
    if (!s_bar_ok) {
        if (threadIdx.x == 0) {
            atomicOr(&a.hdr->err, MOE_DEVERR_TIMEOUT);
            a.hdr->abort = 1u;
        }
        return;
    }

    // ---- phase B.1: global column sums and this tile's column prefix.  T is at
    // most kMetaMaxTiles < kMetaThreads, so one thread reads each tile's valid
    // count and error bits; they are issued before the histogram table loads.
    const int tq = threadIdx.x;
    const int tv_before = (tq < T && tq < tile) ? __ldcg(a.tile_valid + tq) : 0;
    const unsigned terr = (tile == 0 && tq < T) ? (unsigned)__ldcg(a.tile_err + tq) : 0u;
    int G = E <= kMetaThreads ? kMetaThreads / E : 1;
    if (G > T) G = T;
    for (int i = threadIdx.x; i < G * E; i += kMetaThreads) {
        const int g = i / E, e = i - g * E;
        int all = 0, before = 0;
        for (int t0 = g; t0 < T; t0 += 8 * G) {
            int v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int t = t0 + u * G;
                v[u] = t < T ? __ldcg(a.tile_hist + (size_t)t * E + e) : 0;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                all += v[u];
                if (t0 + u * G < tile) before += v[u];
            }
        }
        part_all[i] = all;
        part_before[i] = before;
    }
    if (threadIdx.x == 0) s_err = 0;
    __syncthreads();
    if (terr) atomicOr(&s_err, terr);
    for (int e = threadIdx.x; e < E; e += kMetaThreads) {
        int all = 0, before = 0;
        for (int g = 0; g < G; ++g) {
            all += part_all[g * E + e];
            before += part_before[g * E + e];
        }
        off[e] = all;             // scanned below
        part_before[e] = before;  // this tile's prefix per expert (rows g > 0 no longer needed)
        gt[e] = (all + kTileRows - 1) / kTileRows;
    }
    __syncthreads();
    const int P = block_exclusive_scan(off, off, E);
    const int pbase = block_sum(tv_before);
    const bool abort = (int64_t)P > a.p_cap;

    if (tile == 0) {
        const int GT = block_exclusive_scan(gt, gt, E);
        for (int e = threadIdx.x; e < E; e += kMetaThreads) {
            a.meta.expert_frequency[e] = (e + 1 < E ? off[e + 1] : P) - off[e];
            a.meta.expert_frequency_offset[e] = off[e];
            a.gemm_tile_off[e] = gt[e];
        }
        if (threadIdx.x == 0) {
            unsigned err = s_err;
            if (a.total_pairs >= 0 && (int64_t)P != a.total_pairs) err |= MOE_DEVERR_PAIR_COUNT;
            if (abort) err |= MOE_DEVERR_PAIR_COUNT | MOE_DEVERR_ABORTED;
            a.meta.expert_frequency_offset[E] = P;
            a.gemm_tile_off[E] = GT;
            a.meta.token_offset[a.N] = P;
            a.hdr->P = P;
            a.hdr->err = err;
            a.hdr->abort = abort ? 1u : 0u;
        }
        if (kPairs) {
            // tokens after the last listed token (all tokens if the list is empty)
            int last = a.NK > 0 ? slot_token<kPairs, kIdx64>(a, (int)a.NK - 1) : -1;
            if (last < -1) last = -1;
            for (int64_t tt = (int64_t)last + 1 + threadIdx.x; tt < a.N; tt += kMetaThreads)
                a.meta.token_offset[tt] = P;
        }
    }
    if (abort) return;  // the pair arrays are too small for the pairs seen

    // ---- phase B.2: bases: global offset + earlier tiles + earlier warps
    for (int e = threadIdx.x; e < E; e += kMetaThreads) {
        int run = off[e] + part_before[e];
        for (int w = 0; w < kMetaWarps; ++w) {
            const int c = cnt[w * E + e];
            cnt[w * E + e] = run;
            run += c;
        }
    }
    if (threadIdx.x == 0) {
        int run = pbase;
        for (int w = 0; w < kMetaWarps; ++w) {
            const int c = wq[w];
            wq[w] = run;
            run += c;
        }
    }
    __syncthreads();

    // ---- phase B.3: positions, in slot order
    int q_run = wq[warp];
    for (int base = w0; base < w1; base += kWarpChunk) {
        int ev[kV], tv[kV];
        float wv[kV];
        if (base == w0) {
#pragma unroll
            for (int v = 0; v < kV; ++v) {
                ev[v] = ev0[v];
                tv[v] = tv0[v];
                wv[v] = wv0[v];
            }
        } else {
            load_chunk<kIdx64>(a.topk_idx, base, w1, lane, ev);
#pragma unroll
            for (int v = 0; v < kV; ++v) {
                const int s = base + 32 * v + lane;
                wv[v] = s < w1 ? __ldg(a.topk_w + s) : 0.f;
                tv[v] = (kPairs && s < w1) ? slot_token<kPairs, kIdx64>(a, s) : 0;
            }
        }
#pragma unroll
        for (int v = 0; v < kV; ++v) {
            const int s = base + 32 * v + lane;
            const int e = ev[v];
            unsigned ignore = 0;
            const bool valid = slot_valid<kPairs>(a, e, tv[v], &ignore);
            const unsigned peers = __match_any_sync(kFull, valid ? e : -1);
            const int pb = valid ? mycnt[e] : 0;
            __syncwarp();
            if (valid && lane == __ffs(peers) - 1) mycnt[e] = pb + __popc(peers);
            const unsigned vb = __ballot_sync(kFull, valid);
            const int q = q_run + __popc(vb & lt);
            if (valid) {
                const int p = pb + __popc(peers & lt);
                a.meta.x_gather_idx[p] = kPairs ? tv[v] : s / K;
                a.meta.s_scatter_idx[p] = q;
                a.meta.s_reverse_scatter_idx[q] = p;
                a.meta.scores[q] = wv[v];
            }
            if (s < w1) {
                if (a.slot_pair) a.slot_pair[s] = valid ? q : -1;  // training: slot -> pair
                if (!kPairs) {
                    if ((s % K) == 0) a.meta.token_offset[s / K] = q;
                } else {
                    // tokens (previous slot's token, this slot's token] start at q
                    // (an order violation was flagged in phase A; offsets then unspecified)
                    const int t = tv[v];
                    const int tprev = s > 0 ? slot_token<kPairs, kIdx64>(a, s - 1) : -1;
                    const int64_t lo = max((int64_t)tprev + 1, (int64_t)0);
                    const int64_t hi = min((int64_t)t, a.N - 1);
                    for (int64_t tt = lo; tt <= hi; ++tt) a.meta.token_offset[tt] = q;
                }
            }
            q_run += __popc(vb);
            __syncwarp();
        }
    }
}

}  // namespace

size_t meta_smem_bytes(int E) {
    return ((size_t)kMetaWarps * E + 2 * kPartInts + 2 * (kMaxExperts + 1)) * sizeof(int);
}

template <bool kPairs, bool kIdx64>
cudaError_t launch_meta_as(const MetaArgs &a, cudaStream_t s, int dev) {
    static bool configured[64] = {};
    if (dev < 64 && !configured[dev]) {
        const cudaError_t err = cudaFuncSetAttribute(meta_kernel<kPairs, kIdx64>,
                                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                     (int)meta_smem_bytes(kMaxExperts));
        if (err != cudaSuccess) return err;
        configured[dev] = true;
    }
    MetaArgs args = a;
    void *params[] = {&args};
    // cooperative: all T CTAs are resident at once, so the grid barrier ends
    return cudaLaunchCooperativeKernel((const void *)meta_kernel<kPairs, kIdx64>, dim3(a.tiles),
                                       dim3(kMetaThreads), params, meta_smem_bytes(a.E), s);
}

cudaError_t launch_meta(const MetaArgs &a, cudaStream_t s) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    // the grid barrier's arrival counter starts from zero in every call
    err = cudaMemsetAsync(&a.hdr->grid_arrive, 0, sizeof(a.hdr->grid_arrive), s);
    if (err != cudaSuccess) return err;
    if (a.pair_list) return a.idx64 ? launch_meta_as<true, true>(a, s, dev) : launch_meta_as<true, false>(a, s, dev);
    return a.idx64 ? launch_meta_as<false, true>(a, s, dev) : launch_meta_as<false, false>(a, s, dev);
}

}  // namespace moe
