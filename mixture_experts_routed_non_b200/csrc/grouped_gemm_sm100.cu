// Grouped GEMMs over the expert-sorted pair segments on sm_100a: tcgen05 MMAs
// with TMEM accumulators, issued for a CTA pair (cta_group::2), fed by TMA and
// cp.async.  The grouped GEMM is the compute core of the layer (sonic-moe
// write-up, "CuTeDSL, Triton and QuACK grouped GEMM kernels"; issue #68: the
// grouped GEMM consumes the metadata unchanged).
//
//   up   (kUp = true):  acc = x[x_gather_idx[p], :] . w1[e] (+ b1[e]),
//                       h[p, j] = silu(gate_j) * up_j   (bf16 [P_cap, I])
//        The A rows are gathered from x by four producer warps with 16-byte
//        cp.async copies written straight into the 128-byte-swizzled stage
//        (one TMA tile::gather4 per four rows proved too slow: a stage needed
//        32 of them and the TMA unit became the bottleneck), so no permuted
//        copy of x is ever written.  The SwiGLU ("silu times up", qwen3_5.py
//        commit notes, recipe step 4) runs in the epilogue on the fp32
//        accumulator.  Interleaved w1 columns (g0,u0,g1,u1,...) give gate/up in
//        adjacent accumulator columns; with concatenated w1 (all gates, then
//        all ups; sonic-moe write-up, "Interleaved by default, concatenated if
//        your model is HuggingFace") the even CTA loads 128 gate columns and
//        the odd CTA the matching 128 up columns, so gate and up land in
//        accumulator columns c and c+128.
//   down (kUp = false): y[p, :] = h[p, :] . w2[e] (+ b2[e]), stored as fp16
//        scaled by a power of two per 32-column block of each row ([P_cap, H]
//        fp16 bits and the int8 exponents y_scale [P_cap, H/32]): the rows the
//        combine sums carry 11 significant bits instead of bf16's 8, at bf16's
//        range and 1/32 byte per element more than bf16 rows.
//
// Tiles: a cluster of two CTAs owns a tile of 256 rows of one expert's
// segment x 256 accumulator columns.  CTA r holds A rows [128r, 128r+128) and
// B columns [128r, 128r+128) of each stage (16 KB + 16 KB), and its TMEM holds
// the fp32 accumulator of its 128 rows.  The even CTA issues the pair MMA
// (M=256, N=256, K=16) for both; commits are multicast to both CTAs' barriers.
// Clusters walk a static round-robin list of tiles, row-tile major so that
// consecutive clusters share the gathered A rows in L2.
//
// Warp roles per CTA: warp 0 = TMA producer (B; A for the down GEMM), warp 1 =
// TMEM allocator, and the MMA issuer (even CTA) or, in the up GEMM, the relay
// that tells the even CTA when the odd CTA's gathered rows have landed (odd
// CTA); warps 2-5 = epilogue (TMEM lane quarter warp%4); warps 6-9 (up only)
// = A-row gather.  The even CTA's gather threads arrive with cp.async straight
// on the stage barrier, so the MMA thread checks a single barrier per stage:
// its per-stage work is on the tensor pipe's critical path.  Three
// shared-memory stages of 128 K (64 KB per CTA); two TMEM accumulators so the
// epilogue of one tile overlaps the MMAs of the next.  A segment's last tile
// with at most 128 rows runs the pair MMA at M=128 (64 rows per CTA).  Rows
// past the end of an expert's segment are computed (stale stage rows) but
// never stored.  In training the up GEMM also writes the SwiGLU backward's
// factors (u silu'(g), silu(g)) in bf16, by TMA through the store buffer.
//
// Every wait is bounded (common.cuh); on a timeout a CTA raises its abort
// flag, records MOE_DEVERR_TIMEOUT, drains what it has in flight and returns
// through the final cluster barrier with its TMEM freed.
#include "common.cuh"

namespace moe {

namespace {

constexpr int kPairM = 256;                     // rows per tile (two CTAs x kBM)
#ifndef MOE_STAGE_K
#define MOE_STAGE_K 128
#endif
constexpr int kStageK = MOE_STAGE_K;            // K per pipeline stage: 64 or 128
constexpr int kAtoms = kStageK / 64;            // 128-byte-swizzle atoms along K per stage
constexpr int kPairStages = kStageK == 128 ? 3 : 6;
constexpr int kGatherWarps = 4;
constexpr int kGatherThreads = 32 * kGatherWarps;
constexpr uint32_t kAtomA = kBM * 64 * 2;       // 16 KB: 128 rows x 64 K (one swizzle atom column)
constexpr uint32_t kStageA = kAtomA * kAtoms;   // this CTA's 128 rows x kStageK
constexpr uint32_t kChunkB = kStageK * 64 * 2;  // 64 columns x kStageK rows of K
constexpr uint32_t kStageB = 2 * kChunkB;       // this CTA's 128 columns x kStageK
constexpr uint32_t kStageBytes = kStageA + kStageB;
constexpr uint32_t kTmemCols = 2 * kBN;         // two accumulators
constexpr uint32_t kNumBars = 3 * kPairStages + 5;
constexpr uint32_t kIdesc = idesc_bf16_f32(kPairM, kBN, /*b_mn_major=*/true);
// A segment's last tile with at most 128 rows runs the pair MMA at M=128: each
// CTA holds 64 rows of A, and its TMEM accumulator holds those 64 rows with
// columns [0,128) in lanes 0-63 and columns [128,256) in lanes 64-127.
constexpr uint32_t kIdescTail = idesc_bf16_f32(kBM, kBN, /*b_mn_major=*/true);
constexpr int kTailRows = kBM / 2;  // rows per CTA of a tail tile
constexpr unsigned long long kAbortSettleNs = 2000000ull;

constexpr uint32_t kStoreBuf = 32 * 128;        // 4 KB per epilogue warp: 32 rows x 64 bf16
constexpr size_t kSmemStoreOff = (size_t)kPairStages * kStageBytes;
constexpr size_t kSmemBarOff = kSmemStoreOff + 4 * kStoreBuf;
constexpr size_t kSmemMiscOff = kSmemBarOff + 8 * kNumBars;
constexpr size_t kSmemTableOff = kSmemMiscOff + 16;
constexpr size_t kSmemBytes = 1024 /*alignment slack*/ + kSmemTableOff + 2 * (kMaxExperts + 1) * 4;
static_assert(kSmemBytes <= 232448, "shared memory of one CTA (227 KB)");

__host__ __device__ constexpr int threads_of(bool up) { return up ? 192 + kGatherThreads : 192; }

struct Tile {
    int e, m0, m_end, nt;
};

__device__ __forceinline__ Tile decode_tile(int tile, int n_tiles, int E, const int *tile_off,
                                            const int *off) {
    Tile t;
    const int mt = tile / n_tiles;
    t.nt = tile - mt * n_tiles;
    int lo = 0, hi = E - 1;  // largest e with tile_off[e] <= mt
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tile_off[mid] <= mt) lo = mid;
        else hi = mid - 1;
    }
    t.e = lo;
    t.m0 = off[lo] + (mt - tile_off[lo]) * kPairM;
    t.m_end = off[lo + 1];
    return t;
}

// silu(g) * u; for very negative g the quotient underflows to 0 as silu does.
__device__ __forceinline__ float silu_mul(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

// Training: h = silu(g) u (bit for bit what silu_mul gives) and the two
// factors of the SwiGLU backward the forward keeps for the backward, so that
// dg = dh * fa and du = dh * fb there, all from one exponential:
//   fa = u silu'(g) = u s (1 + g (1 - s)),  fb = silu(g) = g s,  s = sigmoid(g).
// Each factor is rounded once to bf16 when stored; g itself is never rounded
// (near silu's minimum, g ~ -1.28, silu'(g) of a rounded g would lose its
// accuracy).
__device__ __forceinline__ float swiglu_train(float g, float u, float &fa, float &fb) {
    const float d = 1.0f + __expf(-g);
    const float sg = __fdividef(1.0f, d);  // 0 once exp(-g) overflows, as the limit
    fb = g * sg;
    fa = u * sg * (1.0f + g * (1.0f - sg));
    return __fdividef(g, d) * u;  // silu_mul(g, u), the same expression
}

// r[i] (fp32 bits) += bias[i] for 32 consecutive columns; nothing when bias is null.
__device__ __forceinline__ void add_bias32(uint32_t (&r)[32], const __nv_bfloat16 *b) {
    if (!b) return;
    const uint4 *p = reinterpret_cast<const uint4 *>(b);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint4 w = __ldg(p + i);
        const uint32_t q[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            r[8 * i + 2 * j] = __float_as_uint(__uint_as_float(r[8 * i + 2 * j]) + bf16lo(q[j]));
            r[8 * i + 2 * j + 1] = __float_as_uint(__uint_as_float(r[8 * i + 2 * j + 1]) + bf16hi(q[j]));
        }
    }
}



// 64 bf16 columns (32 packed pairs) of one row per lane: a warp whose 32 rows
// are all stored stages the 32 x 64 block in its store buffer (128-byte
// swizzle) and writes it with one TMA store; otherwise each valid lane stores
// its row's 128 bytes.
__device__ __forceinline__ void store_block64(const CUtensorMap *map, uint32_t store_buf, int lane, bool warp_full,
                                              bool valid, int wrow0, __nv_bfloat16 *row, int col0,
                                              const uint32_t (&v)[32]) {
    if (warp_full) {
        if (lane == 0) bulk_wait_read0();  // the buffer's previous store has been read
        __syncwarp();
#pragma unroll
        for (int c = 0; c < 8; ++c)
            st_shared_v4(store_buf + lane * 128 + ((c ^ (lane & 7)) << 4), v[4 * c], v[4 * c + 1], v[4 * c + 2],
                         v[4 * c + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            tma_store_2d(map, store_buf, col0, wrow0);
            bulk_commit();
        }
    } else if (valid) {
        uint4 *dst = reinterpret_cast<uint4 *>(row + col0);
#pragma unroll
        for (int c = 0; c < 8; ++c) dst[c] = make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
    }
}

__device__ __forceinline__ void settle_after_abort() {
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < kAbortSettleNs) {
    }
}

// kTrain (up only): also store the SwiGLU backward's factors (a.z_out); a
// separate instantiation keeps the inference kernel free of that code.
template <bool kUp, bool kTrain = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(threads_of(kUp), 1)
    grouped_gemm_kernel(const __grid_constant__ GemmArgs a) {
    constexpr int kThreads = threads_of(kUp);
    extern __shared__ uint8_t smem_raw[];
    // uniform for both CTAs of the pair: they return together
    if (*(volatile uint32_t *)&a.hdr->abort) return;

    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *base_ptr = smem_raw + (base - raw);
    const uint32_t sA = base;
    const uint32_t sB = base + kPairStages * kStageA;
    const uint32_t bars = base + (uint32_t)kSmemBarOff;
    auto full_bar = [&](int s) { return bars + 8u * s; };
    auto empty_bar = [&](int s) { return bars + 8u * (kPairStages + s); };
    auto gfull_bar = [&](int s) { return bars + 8u * (2 * kPairStages + s); };
    auto tfull_bar = [&](int b) { return bars + 8u * (3 * kPairStages + b); };
    auto tempty_bar = [&](int b) { return bars + 8u * (3 * kPairStages + 2 + b); };
    const uint32_t drain_bar = bars + 8u * (3 * kPairStages + 4);
    uint32_t *misc = reinterpret_cast<uint32_t *>(base_ptr + kSmemMiscOff);
    int *tile_off_s = reinterpret_cast<int *>(base_ptr + kSmemTableOff);
    int *off_s = tile_off_s + (kMaxExperts + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int E = a.E;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPairStages; ++s) {
            // even CTA: producer's arrive (+ both CTAs' TMA bytes); in the up GEMM
            // also its own gather threads' cp.async arrivals and the odd CTA's relay
            mbar_init(full_bar(s), 1 + (kUp ? 1 + kGatherThreads : 0));
            mbar_init(empty_bar(s), 1);
            mbar_init(gfull_bar(s), kGatherThreads);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull_bar(b), 1);
            mbar_init(tempty_bar(b), 8);  // 4 epilogue warps x 2 CTAs
        }
        mbar_init(drain_bar, 1);
        misc[1] = 0;
        fence_barrier_init();
    }
    if (threadIdx.x == 32) {
        if (!kUp) tma_prefetch_desc(&a.tmap_a);
        tma_prefetch_desc(&a.tmap_b);
    }
    for (int i = threadIdx.x; i <= E; i += kThreads) {
        tile_off_s[i] = __ldg(a.tile_off + i);
        off_s[i] = __ldg(a.expert_off + i);
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(&misc[0]), kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();  // barriers of both CTAs initialised before any remote arrive
    tc_fence_after();

    const uint32_t tmem_base = misc[0];
    volatile uint32_t *abort = &misc[1];
    const int n_tiles = a.n_tiles;
    const int total_tiles = tile_off_s[E] * n_tiles;
    const int nk = (a.k_dim + kStageK - 1) / kStageK;   // K % kStageK is 0 or 64
    const int last_mmas = (a.k_dim % kStageK) ? (a.k_dim % kStageK) / kUmmaK : kStageK / kUmmaK;
    const int cluster = blockIdx.x >> 1;
    const int n_clusters = gridDim.x >> 1;
    const int row0 = (int)rank * kBM;  // this CTA's first row inside a full tile
    // a tail tile (at most 128 rows; the concatenated up GEMM keeps full tiles, its
    // gate and up halves sit in different CTAs) and this CTA's first row and rows in it
    auto is_tail = [&](const Tile &tt) {
        return tt.m_end - tt.m0 <= kBM && (!kUp || a.layout != MOE_LAYOUT_CONCATENATED);
    };
    auto rbase = [&](const Tile &tt) { return is_tail(tt) ? (int)rank * kTailRows : row0; };
    auto rspan = [&](const Tile &tt) { return is_tail(tt) ? kTailRows : kBM; };

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        // A rows of one CTA in the down GEMM: a full 128-row box, or, for a short
        // segment, only its 16-row groups (rows past the segment end are never
        // stored, so they need no data)
        auto a_groups = [&](const Tile &tt, int r) {
            const bool tl = is_tail(tt);
            const int span = tl ? kTailRows : kBM;
            const int v = min(max(tt.m_end - (tt.m0 + r * span), 0), span);
            const int g = (v + 15) / 16;
            return (!tl && g >= 6) ? 8 : g;  // 8 = one full box
        };
        auto a_bytes = [&](int groups) { return (uint32_t)groups * 16 * 128 * kAtoms; };
        int stage = 0;
        uint32_t phase = 0;
        uint32_t issued = 0, issued_parity = 0;
        if (lane == 0) {
            for (int tile = cluster; tile < total_tiles; tile += n_clusters) {
                const Tile t = decode_tile(tile, n_tiles, E, tile_off_s, off_s);
                const int brow0 = t.e * a.k_dim;
                const int ga0 = kUp ? 0 : a_groups(t, 0), ga1 = kUp ? 0 : a_groups(t, 1);
                const int ga_mine = rank == 0 ? ga0 : ga1;
                bool ok = true;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, abort)) {
                        ok = false;
                        break;
                    }
                    // both CTAs' TMA bytes land on the even CTA's barrier
                    if (rank == 0)
                        mbar_arrive_expect_tx(full_bar(stage),
                                              2 * kStageB + (kUp ? 0u : a_bytes(ga0) + a_bytes(ga1)));
                    const uint32_t fb = mapa_shared(full_bar(stage), 0);
                    const int k0 = kb * kStageK;
                    const uint32_t b_dst = sB + stage * kStageB;
                    if (!kUp) {
                        const uint32_t a_dst = sA + stage * kStageA;
                        if (ga_mine == 8) {
                            tma_load_3d_pair(a_dst, &a.tmap_a, fb, 0, t.m0 + row0, k0 / 64);
                        } else {
                            for (int g = 0; g < ga_mine; ++g)
#pragma unroll
                                for (int at = 0; at < kAtoms; ++at)
                                    tma_load_3d_pair(a_dst + at * kAtomA + g * 16 * 128, &a.tmap_a16, fb, 0,
                                                     t.m0 + rbase(t) + 16 * g, k0 / 64 + at);
                        }
                    }
                    if (kUp && a.layout == MOE_LAYOUT_CONCATENATED)
                        tma_load_4d_pair(b_dst, &a.tmap_b, fb, 0, brow0 + k0, t.nt * 2, (int)rank);
                    else
                        tma_load_3d_pair(b_dst, &a.tmap_b, fb, 0, brow0 + k0, t.nt * 4 + 2 * (int)rank);
                    issued |= 1u << stage;
                    issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == kPairStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
            }
            // the even CTA's full barriers count both CTAs' bytes: wait for every
            // phase this CTA issued before the CTA may exit
            if (rank == 0)
                for (int s = 0; s < kPairStages; ++s)
                    if ((issued & (1u << s)) && !mbar_wait_timed(full_bar(s), (issued_parity >> s) & 1u))
                        atomicOr(&a.hdr->err, MOE_DEVERR_TIMEOUT);  // a drain that ran out is an error too
        }
        __syncwarp();
    } else if (warp == 1) {
        if (rank == 0) {
            // ---------------------------------------------------- MMA issuer
            if (lane == 0) {
                int stage = 0;
                uint32_t phase = 0;
                int tcount = 0;
                bool ok = true;
                int e_cur = 0;  // tiles come in increasing order: the expert only moves forward
                for (int tile = cluster; ok && tile < total_tiles; tile += n_clusters, ++tcount) {
                    const int mt = tile / n_tiles;
                    while (tile_off_s[e_cur + 1] <= mt) ++e_cur;
                    Tile tt;
                    tt.m0 = off_s[e_cur] + (mt - tile_off_s[e_cur]) * kPairM;
                    tt.m_end = off_s[e_cur + 1];
                    const bool tail = is_tail(tt);
                    const int acc = tcount & 1;
                    const uint32_t acc_phase = (tcount >> 1) & 1;
                    if (!mbar_wait_bounded(tempty_bar(acc), acc_phase ^ 1u, abort)) break;
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + acc * kBN;
                    for (int kb = 0; kb < nk; ++kb) {
                        // one barrier per stage: every wait here is on the MMA's critical path
                        if (!mbar_wait_bounded(full_bar(stage), phase, abort)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t a_addr = sA + stage * kStageA;
                        const uint32_t b_addr = sB + stage * kStageB;
#pragma unroll
                        for (int kk = 0; kk < kStageK / kUmmaK; ++kk) {
                            if (kb == nk - 1 && kk >= last_mmas) break;  // K tail of 64
                            // A: K-major, 128-byte rows, 8-row atoms 1024 B apart, 64-wide K
                            // atoms 16 KB apart; K step 32 B inside an atom.
                            const uint64_t adesc = smem_desc_sw128(
                                a_addr + (kk >> 2) * kAtomA + (kk & 3) * (kUmmaK * 2), 16, 1024);
                            // B: N-major, 64-column chunks 8 KB apart (LBO), 8-row K atoms
                            // 1024 B apart (SBO); K step = 16 rows = 2 KB.
                            const uint64_t bdesc =
                                smem_desc_sw128(b_addr + kk * (kUmmaK * 128), kChunkB, 1024);
                            umma_f16_pair(d_tmem, adesc, bdesc, tail ? kIdescTail : kIdesc, (kb | kk) != 0 ? 1u : 0u);
                        }
                        umma_commit_pair_mc(empty_bar(stage), 0x3);
                        if (++stage == kPairStages) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                    if (!ok) break;
                    umma_commit_pair_mc(tfull_bar(acc), 0x3);
                }
                // all pair MMAs issued here complete before TMEM is freed
                umma_commit_pair(drain_bar);
                if (!mbar_wait_timed(drain_bar, 0)) atomicOr(&a.hdr->err, MOE_DEVERR_TIMEOUT);
            }
        } else if (kUp && lane == 0) {
            // ------------------------------------------- relay (odd CTA, up)
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = cluster; ok && tile < total_tiles; tile += n_clusters) {
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait_bounded(gfull_bar(stage), phase, abort)) {
                        ok = false;
                        break;
                    }
                    fence_proxy_async_smem();
                    mbar_arrive_cluster(mapa_shared(full_bar(stage), 0));
                    if (++stage == kPairStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp < 6) {
        // ------------------------------------------------------------ epilogue
        const int quarter = warp & 3;
        const uint32_t store_buf = base + (uint32_t)kSmemStoreOff + (uint32_t)(warp - 2) * kStoreBuf;
        int tcount = 0;
        for (int tile = cluster; tile < total_tiles; tile += n_clusters, ++tcount) {
            const Tile t = decode_tile(tile, n_tiles, E, tile_off_s, off_s);
            const int acc = tcount & 1;
            const uint32_t acc_phase = (tcount >> 1) & 1;
            bool w = true;
            if (lane == 0) w = mbar_wait_bounded(tfull_bar(acc), acc_phase, abort);
            w = __shfl_sync(0xffffffffu, w, 0);
            if (!w) break;
            tc_fence_after();
            // full tile: this warp's 32 rows (TMEM lanes) hold all 256 accumulator
            // columns.  Tail tile: the CTA holds 64 rows; lanes 0-63 hold columns
            // [0,128) of them and lanes 64-127 columns [128,256), at TMEM columns [0,128)
            const bool tail = is_tail(t);
            const int chalf = tail ? (quarter >> 1) : 0;  // which 128 logical columns (tail)
            const int wrow0 = t.m0 + (tail ? rbase(t) + (quarter & 1) * 32 : row0 + quarter * 32);
            const int p = wrow0 + lane;
            const bool valid = p < t.m_end;
            // whole warp inside the segment: stage in shared memory, one TMA store
            // per 32 x 64 block; otherwise masked per-row stores
            const bool warp_full = wrow0 + 31 < t.m_end;
            const uint32_t tbase = tmem_base + acc * kBN + ((uint32_t)(quarter * 32) << 16);
            __nv_bfloat16 *orow = a.out + (size_t)(valid ? p : 0) * a.out_cols;
            const __nv_bfloat16 *brow = a.bias ? a.bias + (size_t)t.e * a.n_dim : nullptr;

            auto store64 = [&](int col0, const uint32_t (&v)[32]) {
                store_block64(&a.tmap_out, store_buf, lane, warp_full, valid, wrow0, orow, col0, v);
            };
            // training: the SwiGLU backward's factors, in w1's column order
            __nv_bfloat16 *zrow = kTrain ? a.z_out + (size_t)(valid ? p : 0) * (2 * a.I) : nullptr;

            if (kUp && a.layout == MOE_LAYOUT_CONCATENATED) {
                // gate = accumulator columns [0,128), up = [128,256)
#pragma unroll 1
                for (int gi = 0; gi < 2; ++gi) {
                    const int col0 = t.nt * (kBN / 2) + gi * 64;  // output column = gate column
                    if (col0 >= a.I) break;
                    uint32_t packed[32];
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        const int c = 2 * gi + hf;
                        uint32_t g[32], u[32];
                        tmem_ld_32x32b_x32(tbase + c * 32, g);
                        tmem_ld_32x32b_x32(tbase + 128 + c * 32, u);
                        tmem_ld_wait();
                        if (brow) {
                            add_bias32(g, brow + col0 + hf * 32);
                            add_bias32(u, brow + a.I + col0 + hf * 32);
                        }
                        // h, and in training u silu'(g) at the gate columns and silu(g) at the up
                        // columns (each thread its own row, 16 bytes to each half per 8 columns),
                        // one pair of columns at a time so that g and u die as they are used
                        uint4 *za = kTrain ? reinterpret_cast<uint4 *>(zrow + col0 + hf * 32) : nullptr;
                        uint4 *zb = kTrain ? reinterpret_cast<uint4 *>(zrow + a.I + col0 + hf * 32) : nullptr;
                        uint32_t wa[4], wb[4];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const float g0 = __uint_as_float(g[2 * i]), g1 = __uint_as_float(g[2 * i + 1]);
                            const float u0 = __uint_as_float(u[2 * i]), u1 = __uint_as_float(u[2 * i + 1]);
                            if (kTrain) {
                                float a0, b0, a1, b1;
                                const float h0 = swiglu_train(g0, u0, a0, b0);
                                const float h1 = swiglu_train(g1, u1, a1, b1);
                                packed[16 * hf + i] = pack_bf16x2(h0, h1);
                                wa[i & 3] = pack_bf16x2(a0, a1);
                                wb[i & 3] = pack_bf16x2(b0, b1);
                                if ((i & 3) == 3 && valid) {
                                    za[i >> 2] = make_uint4(wa[0], wa[1], wa[2], wa[3]);
                                    zb[i >> 2] = make_uint4(wb[0], wb[1], wb[2], wb[3]);
                                }
                            } else {
                                packed[16 * hf + i] = pack_bf16x2(silu_mul(g0, u0), silu_mul(g1, u1));
                            }
                        }
                    }
                    store64(col0, packed);
                }
            } else if (kUp) {
                // interleaved: accumulator columns (2j, 2j+1) = (gate_j, up_j)
#pragma unroll 1
                for (int gi = 0; gi < (tail ? 1 : 2); ++gi) {
                    const int col0 = t.nt * (kBN / 2) + (tail ? chalf : gi) * 64;  // output column
                    if (col0 >= a.out_cols) break;
                    uint32_t packed[32];
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        const int c = 4 * gi + 2 * hf;  // first of two 32-column accumulator chunks
                        uint32_t r0[32], r1[32];
                        tmem_ld_32x32b_x32(tbase + c * 32, r0);
                        tmem_ld_32x32b_x32(tbase + (c + 1) * 32, r1);
                        tmem_ld_wait();
                        const int acol = t.nt * kBN + chalf * (kBN / 2) + c * 32;  // logical column
                        if (brow) {
                            add_bias32(r0, brow + acol);
                            add_bias32(r1, brow + acol + 32);
                        }
                        if (kTrain) {
                            // training: (u silu'(g), silu(g)) in place of (g, u), 64 columns of
                            // w1's order, written 16 bytes at a time as they are computed (the
                            // register budget of ten warps leaves no room for the whole row)
                            if (warp_full) {
                                if (lane == 0) bulk_wait_read0();  // the buffer's previous store has been read
                                __syncwarp();
                            }
                            // four (gate, up) pairs per 16 bytes of factors; their h in the same pass
                            auto train_group = [&](const uint32_t(&rr)[32], int qq, uint32_t &h01, uint32_t &h23,
                                                   uint32_t (&w4)[4]) {
                                float hv[4];
#pragma unroll
                                for (int k = 0; k < 4; ++k) {
                                    float fa, fb;
                                    const int j = 8 * qq + 2 * k;
                                    hv[k] = swiglu_train(__uint_as_float(rr[j]), __uint_as_float(rr[j + 1]), fa, fb);
                                    w4[k] = pack_bf16x2(fa, fb);
                                }
                                h01 = pack_bf16x2(hv[0], hv[1]);
                                h23 = pack_bf16x2(hv[2], hv[3]);
                            };
#pragma unroll
                            for (int q = 0; q < 8; ++q) {
                                uint32_t w4[4];
                                if (q < 4) train_group(r0, q, packed[16 * hf + 2 * q], packed[16 * hf + 2 * q + 1], w4);
                                else train_group(r1, q - 4, packed[16 * hf + 8 + 2 * (q - 4)],
                                                 packed[16 * hf + 8 + 2 * (q - 4) + 1], w4);
                                if (warp_full)
                                    st_shared_v4(store_buf + lane * 128 + ((q ^ (lane & 7)) << 4), w4[0], w4[1], w4[2],
                                                 w4[3]);
                                else if (valid)
                                    reinterpret_cast<uint4 *>(zrow + acol)[q] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                            }
                            if (warp_full) {
                                fence_proxy_async_smem();
                                __syncwarp();
                                if (lane == 0) {
                                    tma_store_2d(&a.tmap_z, store_buf, acol, wrow0);
                                    bulk_commit();
                                }
                            }
                        } else {
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                packed[16 * hf + i] =
                                    pack_bf16x2(silu_mul(__uint_as_float(r0[4 * i]), __uint_as_float(r0[4 * i + 1])),
                                                silu_mul(__uint_as_float(r0[4 * i + 2]), __uint_as_float(r0[4 * i + 3])));
                                packed[16 * hf + 8 + i] =
                                    pack_bf16x2(silu_mul(__uint_as_float(r1[4 * i]), __uint_as_float(r1[4 * i + 1])),
                                                silu_mul(__uint_as_float(r1[4 * i + 2]), __uint_as_float(r1[4 * i + 3])));
                            }
                        }
                    }
                    store64(col0, packed);
                }
            } else {
                // y as fp16 scaled per 32-column block (its exponents in y_scale), 64
                // columns at a time: each thread holds its row's values, so a block's
                // largest |value| needs no exchange
#pragma unroll 1
                for (int gi = 0; gi < (tail ? 2 : 4); ++gi) {
                    const int col0 = t.nt * kBN + chalf * (kBN / 2) + gi * 64;
                    if (col0 >= a.n_dim) break;
                    uint32_t r0[32], r1[32];
                    tmem_ld_32x32b_x32(tbase + gi * 64, r0);
                    tmem_ld_32x32b_x32(tbase + gi * 64 + 32, r1);
                    tmem_ld_wait();
                    if (brow) {
                        add_bias32(r0, brow + col0);
                        add_bias32(r1, brow + col0 + 32);
                    }
                    float m0 = 0.f, m1 = 0.f;  // fmaxf drops NaN
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        m0 = fmaxf(m0, fabsf(__uint_as_float(r0[i])));
                        m1 = fmaxf(m1, fabsf(__uint_as_float(r1[i])));
                    }
                    const int e0 = y_block_exp(m0), e1 = y_block_exp(m1);
                    const float s0 = exp2i(-e0), s1 = exp2i(-e1);
                    uint32_t packed[32];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        packed[i] = pack_f16x2(__uint_as_float(r0[2 * i]) * s0, __uint_as_float(r0[2 * i + 1]) * s0);
                        packed[16 + i] =
                            pack_f16x2(__uint_as_float(r1[2 * i]) * s1, __uint_as_float(r1[2 * i + 1]) * s1);
                    }
                    if (valid)  // the two blocks' exponents (col0 is a multiple of 64: 2-byte aligned)
                        *reinterpret_cast<uint16_t *>(a.out_scale + (size_t)p * (a.n_dim / kYBlock) + col0 / kYBlock) =
                            (uint16_t)((uint32_t)(uint8_t)e0 | ((uint32_t)(uint8_t)e1 << 8));
                    store64(col0, packed);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (rank == 0) mbar_arrive(tempty_bar(acc));
                else mbar_arrive_cluster(mapa_shared(tempty_bar(acc), 0));
            }
        }
        if (lane == 0) bulk_wait0();  // this warp's stores have landed
    } else if (kUp) {
        // ------------------------------------------------------- A-row gather
        // thread g: 16-byte chunk (g & 7) of rows (g >> 3) + 16 i, i = 0..7 of
        // this CTA's 128 rows, stored at row * 128 + ((chunk ^ (row & 7)) << 4):
        // the 128-byte swizzle the MMA descriptors expect.
        const int g = threadIdx.x - 192;
        const int chunk = g & 7;
        const int r0 = g >> 3;
        const int gl = g & 31;
        int stage = 0;
        uint32_t phase = 0;
        const char *xb = reinterpret_cast<const char *>(a.x);
        const size_t ld = (size_t)a.k_dim * 2;
        // x rows are read by every pair of their token, at different times (one
        // expert after another) while the weights stream through L2: keep them
        const uint64_t x_policy = l2_policy_evict_last();
        int tile = cluster;
        Tile t{};
        const char *src[8];
        auto load_rows = [&](const Tile &tt, const char *(&pp)[8]) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int pr = min(tt.m0 + rbase(tt) + r0 + 16 * i, tt.m_end - 1);
                pp[i] = xb + (size_t)__ldg(a.x_gather_idx + pr) * ld + chunk * 16;
            }
        };
        if (tile < total_tiles) {
            t = decode_tile(tile, n_tiles, E, tile_off_s, off_s);
            load_rows(t, src);
        }
        bool ok = true;
        for (; ok && tile < total_tiles; tile += n_clusters) {
            const int next = tile + n_clusters;
            Tile tn = t;
            const char *nsrc[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) nsrc[i] = src[i];
            if (next < total_tiles) {
                tn = decode_tile(next, n_tiles, E, tile_off_s, off_s);
                if (tn.m0 != t.m0) load_rows(tn, nsrc);
            }
            for (int kb = 0; kb < nk; ++kb) {
                bool w = true;
                if (gl == 0) w = mbar_wait_bounded(empty_bar(stage), phase ^ 1u, abort);
                w = __shfl_sync(0xffffffffu, w, 0);
                if (!w) {
                    ok = false;
                    break;
                }
                const uint32_t a_dst = sA + stage * kStageA;
                const int rb = rbase(t), rs = rspan(t);  // a tail tile: 64 rows per CTA
#pragma unroll
                for (int at = 0; at < kAtoms; ++at) {
                    const int k0 = kb * kStageK + at * 64;
                    if (k0 >= a.k_dim) break;  // K tail of 64: that atom is not multiplied
                    const size_t koff = (size_t)k0 * 2;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int rr = r0 + 16 * i;
                        // rows past the segment end are never stored: skip their copies
                        // (the stage keeps stale data there, which only feeds those rows)
                        if (rr < rs && t.m0 + rb + rr < t.m_end)
                            cp_async_16_hint(a_dst + at * kAtomA + rr * 128 + ((chunk ^ (rr & 7)) << 4),
                                             src[i] + koff, x_policy);
                    }
                }
                // even CTA: straight onto the stage barrier the MMA waits on; odd
                // CTA: onto gfull, which its relay forwards to the even CTA
                cp_async_arrive_noinc(rank == 0 ? full_bar(stage) : gfull_bar(stage));
                if (++stage == kPairStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            t = tn;
#pragma unroll
            for (int i = 0; i < 8; ++i) src[i] = nsrc[i];
        }
        cp_async_wait_all();
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (*abort) {
        if (threadIdx.x == 0) atomicOr(&a.hdr->err, MOE_DEVERR_TIMEOUT);
        settle_after_abort();  // let copies issued by the peer CTA land
    }
    cluster_sync_all();  // no CTA leaves while its peer may still touch it
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, kTmemCols);
    }
}

template <bool kUp, bool kTrain>
cudaError_t launch(const GemmArgs &a, int max_clusters, cudaStream_t s) {
    // once per device: the shared-memory limit, and how many clusters fit at once
    int fit = 1;
    cudaError_t err = launch_setup_once(
        (const void *)grouped_gemm_kernel<kUp, kTrain>, &fit, [](int dev, int *v) -> cudaError_t {
            cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<kUp, kTrain>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
            if (e != cudaSuccess) return e;
            int sms = 0;
            e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            if (e != cudaSuccess) return e;
            // the kernel's cluster shape (2,1,1) is compiled in (__cluster_dims__)
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3((unsigned)(sms & ~1));
            cfg.blockDim = dim3(threads_of(kUp));
            cfg.dynamicSmemBytes = kSmemBytes;
            int n = 0;
            e = cudaOccupancyMaxActiveClusters(&n, grouped_gemm_kernel<kUp, kTrain>, &cfg);
            if (e != cudaSuccess) return e;
            *v = n > 0 ? n : 1;
            return cudaSuccess;
        });
    if (err != cudaSuccess) return err;
    int clusters = fit < max_clusters ? fit : max_clusters;
    if (clusters < 1) clusters = 1;
    grouped_gemm_kernel<kUp, kTrain><<<2 * clusters, threads_of(kUp), kSmemBytes, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

size_t gemm_smem_bytes() { return kSmemBytes; }

cudaError_t launch_gemm_up(const GemmArgs &a, int max_clusters, cudaStream_t s) {
    return a.z_out ? launch<true, true>(a, max_clusters, s) : launch<true, false>(a, max_clusters, s);
}
cudaError_t launch_gemm_down(const GemmArgs &a, int max_clusters, cudaStream_t s) {
    return launch<false, false>(a, max_clusters, s);
}

}  // namespace moe
