// Routing metadata of the non-expand layout, built straight from [N,K]
// (sonic-moe issue #68, "End-to-end DeepEP v2 non-expand + SonicMoE
// integration": the metadata list -- expert_frequency,
// expert_frequency_offset, x_gather_idx, s_scatter_idx,
// s_reverse_scatter_idx, num_activated_expert_per_token_offset, compact
// router_scores -- and question 3: pairs are numbered in ascending token
// order).  The sort by expert is a stable counting sort (the segmented-sort
// recipe of the qwen3_5.py commit notes, steps 1-2) over T tiles of
// consecutive slots, in two kernels on the caller's stream:
//
//   count    one CTA per tile counts the experts of its slots (shared-memory
//            increments: integer counts, so their order does not matter) and
//            stores the tile's histogram row, valid count and error bits.
//            Its first instruction lets the scatter kernel start.
//   scatter  launched as a programmatic dependent of the count kernel, so
//            its CTAs start while the counts are still running.  Before it
//            waits for them, each CTA loads its tile's ids and weights and
//            ranks every valid slot stably inside the tile: each warp owns a
//            contiguous slice, ballots over the bits of the expert id group
//            the lanes of one expert in a 32-slot step, popc(peers & lanes
//            below) orders them, and a
//            per-warp row of counts in shared memory carries the rank across
//            steps; a scan over the warps then gives every pair its position
//            in the tile's expert-sorted order, where its token and pair
//            index are staged in shared memory.  After the wait (the count
//            kernel has finished and its stores are visible) the CTA reads
//            the whole [T,E] histogram table once, derives the global
//            offsets and its tile's base per expert, and writes: the sorted
//            arrays as contiguous runs per expert from the staged copy, and
//            the pair-order arrays and token offsets in slot order.  CTA 0
//            also writes the histogram, offsets, GEMM tile table and the
//            call's error word.
//
// Every result is a pure function of the input (no atomic decides an order),
// so the output is bit-exact and deterministic.  Nothing waits on a flag: the
// only dependency between CTAs is the kernel boundary, so no counter has to be
// cleared between calls and no wait can hang.
#include <mutex>

#include "common.cuh"

namespace moe {

namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kCountThreads = 256;
constexpr int kCountUnroll = 8;                         // ids in flight per thread of the count kernel
constexpr int kChunk = 4096;                            // slots staged per pass of the scatter kernel
constexpr int kStepMax = kChunk / (32 * kMetaWarps);    // 32-slot steps per warp and pass (8)
constexpr int kPartInts = 2 * 4 * kMetaThreads;         // table partial sums: 2 x G x hist_ld, G*hist_ld <= 4*512
static_assert(kPartInts % 4 == 0, "the arrays after the partial sums start 16-byte aligned");
static_assert(kMetaMaxTiles <= kMetaThreads, "one thread of CTA 0 reads each tile's error bits");


__device__ __forceinline__ int4 ld_cg_int4(const int *p) {
    int4 v;
    asm volatile("ld.global.cg.v4.s32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Exclusive scan of n ints in shared memory (in place allowed) by the whole
// 512-thread block; returns the total.
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

// Sum over the 512-thread block of one int per thread.
__device__ int block_sum(int v) {
    __shared__ int part[kMetaWarps];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v = (int)__reduce_add_sync(kFull, (unsigned)v);
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

// ---------------------------------------------------------------------------
// count: tile histogram, valid count and error bits
// ---------------------------------------------------------------------------
template <bool kPairs, bool kIdx64>
__global__ void __launch_bounds__(kCountThreads) meta_count_kernel(const MetaArgs a) {
    pdl_launch_dependents();
    extern __shared__ int hist[];  // [hist_ld]
    __shared__ unsigned s_err;
    __shared__ int s_valid;
    for (int e = threadIdx.x; e < a.hist_ld; e += kCountThreads) hist[e] = 0;
    if (threadIdx.x == 0) {
        s_err = 0;
        s_valid = 0;
    }
    __syncthreads();
    const int s0 = blockIdx.x * a.tile_slots;
    const int s1 = (int)min((int64_t)s0 + a.tile_slots, a.NK);
    unsigned err = 0;
    int nvalid = 0;
    for (int base = s0; base < s1; base += kCountUnroll * kCountThreads) {
        int e[kCountUnroll], t[kCountUnroll];
#pragma unroll
        for (int u = 0; u < kCountUnroll; ++u) {
            const int s = base + u * kCountThreads + threadIdx.x;
            e[u] = s < s1 ? load_id<kIdx64>(a.topk_idx, s) : -1;
            t[u] = (kPairs && s < s1) ? load_id<kIdx64>(a.token_idx, s) : 0;
        }
#pragma unroll
        for (int u = 0; u < kCountUnroll; ++u) {
            const int s = base + u * kCountThreads + threadIdx.x;
            if (kPairs && s > 0 && s < s1 &&
                load_id_wide<kIdx64>(a.token_idx, s - 1) > load_id_wide<kIdx64>(a.token_idx, s))
                err |= MOE_DEVERR_BAD_TOKEN;  // a pair list must be in ascending token order
            if (slot_valid<kPairs>(a, e[u], t[u], &err)) {
                atomicAdd(&hist[e[u]], 1);
                ++nvalid;
            }
        }
    }
    nvalid = (int)__reduce_add_sync(kFull, (unsigned)nvalid);
    err = __reduce_or_sync(kFull, err);
    if ((threadIdx.x & 31) == 0) {
        if (nvalid) atomicAdd(&s_valid, nvalid);
        if (err) atomicOr(&s_err, err);
    }
    __syncthreads();
    int *row = a.tile_hist + (size_t)blockIdx.x * a.hist_ld;
    for (int e = threadIdx.x; e < a.hist_ld; e += kCountThreads) row[e] = hist[e];
    if (threadIdx.x == 0) {
        a.tile_valid[blockIdx.x] = s_valid;
        a.tile_err[blockIdx.x] = (int)s_err;
    }
}

// ---------------------------------------------------------------------------
// scatter: stable positions and every output array
// ---------------------------------------------------------------------------

// One pass's slots in registers: lane `lane` of warp `warp` holds slot
// c0 + warp * slice + 32 v + lane for step v.
struct PassRegs {
    int e[kStepMax];    // expert, -1 for a slot that is no pair (or past the end)
    int tok[kStepMax];  // token of the slot
    float w[kStepMax];  // weight of the slot
    int pos[kStepMax];  // rank among the warp's earlier pairs of its expert, then position in the pass's sorted order
    int qv[kStepMax];   // valid slots before this one in the pass (its pair index within the pass if valid)
};

// Shared memory of the scatter kernel (ints), from a 16-byte aligned base:
//   part [kPartInts]       column sums of the histogram table (all tiles / earlier tiles),
//                          stored as int4: first, so that every row stays 16-byte aligned
//   wrow [kMetaWarps][E]   per-warp expert counts, then the warps' bases inside the pass
//   coff [E+1]             the pass's expert offsets (exclusive scan of its counts); [E] = its pairs
//   gbase[E]               global position of each expert's next pair of this tile
//   dlt  [E]               gbase - coff for the pass being written
//   stok, sq, se [kChunk]  token, pair index in the pass and expert by position in the pass
struct ScatterSmem {
    int *wrow, *coff, *gbase, *dlt, *stok, *sq, *se, *part;
};

__host__ __device__ inline size_t scatter_smem_ints(int E) {
    return (size_t)kMetaWarps * E + (E + 1) + 2 * E + 3 * kChunk + kPartInts;
}

__device__ __forceinline__ ScatterSmem scatter_smem(int *sm, int E) {
    ScatterSmem m;
    m.part = sm;
    m.wrow = m.part + kPartInts;
    m.coff = m.wrow + kMetaWarps * E;
    m.gbase = m.coff + (E + 1);
    m.dlt = m.gbase + E;
    m.stok = m.dlt + E;
    m.sq = m.stok + kChunk;
    m.se = m.sq + kChunk;
    return m;
}

// Slice of each warp in a pass of L slots: a multiple of 32, at most 32 * kStepMax.
__device__ __forceinline__ int pass_slice(int L) {
    return ((L + 32 * kMetaWarps - 1) / (32 * kMetaWarps)) * 32;
}

// Lanes of the warp whose key equals this lane's key (keys < 2^nbits): one
// ballot per key bit, each lane keeping the lanes that agree with it on that
// bit -- the mask match_any gives, in nbits ballots (measured faster here
// than match_any on the 32-slot steps).
__device__ __forceinline__ unsigned peers_of(unsigned key, int nbits) {
    unsigned peers = kFull;
    for (int b = 0; b < nbits; ++b) {
        const unsigned bb = __ballot_sync(kFull, (key >> b) & 1u);
        peers &= ((key >> b) & 1u) ? bb : ~bb;
    }
    return peers;
}

// Loads the slots [c0, c1) and gives every pair its position inside the
// pass's expert-sorted order; stages (token, pair index in the pass, expert)
// at that position.  Inputs only: runs before the wait on the count kernel.
// Returns the pass's pair count (all threads).
template <bool kPairs, bool kIdx64>
__device__ int rank_pass(const MetaArgs &a, const ScatterSmem &m, int c0, int c1, PassRegs &r) {
    __shared__ int s_wv[kMetaWarps];
    const int E = a.E;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t lt = lanemask_lt();
    const int slice = pass_slice(c1 - c0);
    const int w0 = c0 + warp * slice;
    const int w1 = min(w0 + slice, c1);
    int *myrow = m.wrow + warp * E;
    const int nbits = 32 - __clz(E);  // keys 0..E; E marks a slot that is no pair
#pragma unroll
    for (int v = 0; v < kStepMax; ++v) {
        const int s = w0 + 32 * v + lane;
        const bool in = s < w1;
        r.e[v] = in ? load_id<kIdx64>(a.topk_idx, s) : -1;
        r.w[v] = in ? __ldg(a.topk_w + s) : 0.f;
        r.tok[v] = in ? slot_token<kPairs, kIdx64>(a, s) : 0;
    }
    for (int e = lane; e < E; e += 32) myrow[e] = 0;
    __syncwarp();
    int q_run = 0;
#pragma unroll
    for (int v = 0; v < kStepMax; ++v) {
        if (32 * v >= slice) break;  // uniform over the block
        unsigned ignore = 0;
        const bool valid = slot_valid<kPairs>(a, r.e[v], r.tok[v], &ignore);
        if (!valid) r.e[v] = -1;
        const unsigned peers = peers_of(valid ? (unsigned)r.e[v] : (unsigned)E, nbits);
        const int before = valid ? myrow[r.e[v]] : 0;
        __syncwarp();
        if (valid && lane == __ffs(peers) - 1) myrow[r.e[v]] = before + __popc(peers);
        __syncwarp();
        r.pos[v] = before + __popc(peers & lt);
        const unsigned vb = __ballot_sync(kFull, valid);
        r.qv[v] = q_run + __popc(vb & lt);
        q_run += __popc(vb);
    }
    if (lane == 0) s_wv[warp] = q_run;
    __syncthreads();
    // per expert: the warps' bases inside the pass, and the pass's count
    for (int e = threadIdx.x; e < E; e += kMetaThreads) {
        int run = 0;
#pragma unroll
        for (int w = 0; w < kMetaWarps; ++w) {
            const int c = m.wrow[w * E + e];
            m.wrow[w * E + e] = run;
            run += c;
        }
        m.coff[e] = run;
    }
    if (warp == 0) {  // the warps' pair bases inside the pass
        int x = lane < kMetaWarps ? s_wv[lane] : 0;
        const int own = x;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(kFull, x, o);
            if (lane >= o) x += y;
        }
        if (lane < kMetaWarps) s_wv[lane] = x - own;
    }
    __syncthreads();  // the counts in coff are complete before the scan reads them
    const int npairs = block_exclusive_scan(m.coff, m.coff, E);
    if (threadIdx.x == 0) m.coff[E] = npairs;
    const int qw = s_wv[warp];
#pragma unroll
    for (int v = 0; v < kStepMax; ++v) {
        if (32 * v >= slice) break;
        r.qv[v] += qw;
        const int e = r.e[v];
        if (e >= 0) {
            const int p = m.coff[e] + m.wrow[warp * E + e] + r.pos[v];
            r.pos[v] = p;
            m.stok[p] = r.tok[v];
            m.sq[p] = r.qv[v];
            m.se[p] = e;
        }
    }
    __syncthreads();
    return npairs;
}

// Writes one pass's outputs: qbase = pairs before the pass, m.gbase = the
// global position of each expert's first pair in the pass (advanced here to
// the next pass).
template <bool kPairs, bool kIdx64>
__device__ void write_pass(const MetaArgs &a, const ScatterSmem &m, int c0, int c1, int qbase, int npairs,
                           const PassRegs &r) {
    const int E = a.E, K = a.K;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int e = threadIdx.x; e < E; e += kMetaThreads) {
        const int gb = m.gbase[e], cf = m.coff[e];
        m.dlt[e] = gb - cf;
        m.gbase[e] = gb + (m.coff[e + 1] - cf);
    }
    __syncthreads();
    // sorted order: runs of consecutive positions per expert
    for (int j = threadIdx.x; j < npairs; j += kMetaThreads) {
        const int p = j + m.dlt[m.se[j]];
        a.meta.x_gather_idx[p] = m.stok[j];
        a.meta.s_scatter_idx[p] = qbase + m.sq[j];
    }
    // pair order and token offsets, in slot order
    const int slice = pass_slice(c1 - c0);
    const int w0 = c0 + warp * slice;
    const int w1 = min(w0 + slice, c1);
#pragma unroll
    for (int v = 0; v < kStepMax; ++v) {
        if (32 * v >= slice) break;
        const int s = w0 + 32 * v + lane;
        if (s >= w1) continue;
        const int q = qbase + r.qv[v];
        const int e = r.e[v];
        if (e >= 0) {
            a.meta.s_reverse_scatter_idx[q] = r.pos[v] + m.dlt[e];
            a.meta.scores[q] = r.w[v];
        }
        if (a.slot_pair) a.slot_pair[s] = e >= 0 ? q : -1;  // training: slot -> pair
        if (!kPairs) {
            if (s - r.tok[v] * K == 0) a.meta.token_offset[r.tok[v]] = q;
        } else {
            // tokens (previous slot's token, this slot's token] start at q
            // (an order violation is flagged by the count kernel; offsets then unspecified)
            const int t = r.tok[v];
            const int tprev = s > 0 ? slot_token<kPairs, kIdx64>(a, s - 1) : -1;
            const int64_t lo = max((int64_t)tprev + 1, (int64_t)0);
            const int64_t hi = min((int64_t)t, a.N - 1);
            for (int64_t tt = lo; tt <= hi; ++tt) a.meta.token_offset[tt] = q;
        }
    }
}

template <bool kPairs, bool kIdx64>
__global__ void __launch_bounds__(kMetaThreads, 1) meta_scatter_kernel(const MetaArgs a) {
    extern __shared__ __align__(16) int sm[];
    __shared__ unsigned s_err;
    // a programmatic dependent (the decode up GEMM) may start its set-up now;
    // it waits for this grid to finish before it reads the metadata
    pdl_launch_dependents();
    const int E = a.E, T = a.tiles, tile = blockIdx.x, ld = a.hist_ld;
    const ScatterSmem m = scatter_smem(sm, E);
    const int t0 = tile * a.tile_slots;
    const int t1 = (int)min((int64_t)t0 + a.tile_slots, a.NK);
    if (threadIdx.x == 0) s_err = 0;

    // ---- first pass: inputs only, overlapping the count kernel
    PassRegs r;
    int c0 = t0;
    int c1 = min(c0 + kChunk, t1);
    int npairs = rank_pass<kPairs, kIdx64>(a, m, c0, c1, r);

    // ---- the count kernel has finished: read its table once
    pdl_wait();
    const int ld4 = ld >> 2;
    const int G = min(kMetaThreads / ld4 > 0 ? kMetaThreads / ld4 : 1, T);
    int *part_all = m.part;
    int *part_before = m.part + G * ld;
    const int tid = threadIdx.x;
    const unsigned terr = (tile == 0 && tid < T) ? (unsigned)__ldcg(a.tile_err + tid) : 0u;
    if (tid < G * ld4) {
        const int g = tid / ld4, c4 = tid - (tid / ld4) * ld4;
        int4 all = make_int4(0, 0, 0, 0), bef = make_int4(0, 0, 0, 0);
        for (int tb = g; tb < T; tb += 8 * G) {
            int4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int t = tb + u * G;
                v[u] = t < T ? ld_cg_int4(a.tile_hist + (size_t)t * ld + 4 * c4) : make_int4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                all.x += v[u].x; all.y += v[u].y; all.z += v[u].z; all.w += v[u].w;
                if (tb + u * G < tile) {
                    bef.x += v[u].x; bef.y += v[u].y; bef.z += v[u].z; bef.w += v[u].w;
                }
            }
        }
        *reinterpret_cast<int4 *>(part_all + g * ld + 4 * c4) = all;
        *reinterpret_cast<int4 *>(part_before + g * ld + 4 * c4) = bef;
    }
    if (terr) atomicOr(&s_err, terr);
    __syncthreads();
    int before_sum = 0;
    for (int e = tid; e < E; e += kMetaThreads) {
        int all = 0, before = 0;
        for (int g = 0; g < G; ++g) {
            all += part_all[g * ld + e];
            before += part_before[g * ld + e];
        }
        m.gbase[e] = all;          // scanned below
        m.dlt[e] = before;         // this tile's pairs before it, per expert
        before_sum += before;
    }
    __syncthreads();
    const int P = block_exclusive_scan(m.gbase, m.gbase, E);
    int qbase = block_sum(before_sum);  // pairs of the earlier tiles
    const bool abort = (int64_t)P > a.p_cap;

    if (tile == 0) {
        // histogram, offsets and the GEMM tile table: freq is the step of the offsets
        int *gt = part_all;  // the partial sums are no longer needed
        for (int e = tid; e < E; e += kMetaThreads) {
            const int f = (e + 1 < E ? m.gbase[e + 1] : P) - m.gbase[e];
            a.meta.expert_frequency[e] = f;
            a.meta.expert_frequency_offset[e] = m.gbase[e];
            gt[e] = (f + kTileRows - 1) / kTileRows;
        }
        __syncthreads();
        const int GT = block_exclusive_scan(gt, gt, E);
        for (int e = tid; e < E; e += kMetaThreads) a.gemm_tile_off[e] = gt[e];
        if (tid == 0) {
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
            for (int64_t tt = (int64_t)last + 1 + tid; tt < a.N; tt += kMetaThreads) a.meta.token_offset[tt] = P;
        }
    }
    if (abort) return;  // the pair arrays are too small for the pairs seen
    for (int e = tid; e < E; e += kMetaThreads) m.gbase[e] += m.dlt[e];
    __syncthreads();

    // ---- write the passes
    for (;;) {
        write_pass<kPairs, kIdx64>(a, m, c0, c1, qbase, npairs, r);
        qbase += npairs;
        c0 = c1;
        if (c0 >= t1) break;
        c1 = min(c0 + kChunk, t1);
        __syncthreads();  // the staged copy is read before the next pass overwrites it
        npairs = rank_pass<kPairs, kIdx64>(a, m, c0, c1, r);
    }
}

}  // namespace

size_t meta_smem_bytes(int E) { return scatter_smem_ints(E) * sizeof(int); }

template <bool kPairs, bool kIdx64>
cudaError_t launch_meta_as(const MetaArgs &a, cudaStream_t s) {
    int unused = 0;
    cudaError_t err = launch_setup_once(
        (const void *)meta_scatter_kernel<kPairs, kIdx64>, &unused, [](int, int *v) -> cudaError_t {
            *v = 1;
            return cudaFuncSetAttribute(meta_scatter_kernel<kPairs, kIdx64>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)meta_smem_bytes(kMaxExperts));
        });
    if (err != cudaSuccess) return err;
    meta_count_kernel<kPairs, kIdx64><<<a.tiles, kCountThreads, (size_t)a.hist_ld * sizeof(int), s>>>(a);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)a.tiles);
    cfg.blockDim = dim3(kMetaThreads);
    cfg.dynamicSmemBytes = meta_smem_bytes(a.E);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, meta_scatter_kernel<kPairs, kIdx64>, a);
}

cudaError_t launch_meta(const MetaArgs &a, cudaStream_t s) {
    if (a.pair_list) return a.idx64 ? launch_meta_as<true, true>(a, s) : launch_meta_as<true, false>(a, s);
    return a.idx64 ? launch_meta_as<false, true>(a, s) : launch_meta_as<false, false>(a, s);
}

}  // namespace moe
