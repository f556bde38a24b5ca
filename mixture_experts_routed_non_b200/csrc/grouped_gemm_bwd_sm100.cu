// Grouped GEMMs of the backward on sm_100a: tcgen05 MMAs issued for a CTA pair
// (cta_group::2, M=256 x N=256 x K=16) with TMEM accumulators, operands staged
// in shared memory by TMA and cp.async.  The pages leave the backward open
// (sonic-moe issue #68 asks how the scores' gradient returns to [N,K]; the
// write-up names the layer a training layer); these are the chain rule of the
// forward, over the same expert-sorted segments:
//
//   DH  dh = s_p (dout[x_gather_idx[p],:] . W2[e]^T)  (K = H, N = I; the
//       A rows are gathered from dout and the score applied in fp32, so dh
//       sees no rounded operand), then the SwiGLU backward in the epilogue:
//       with the factors the training forward saved,
//       dg = dh u silu'(g), du = dh silu(g), written as bf16 dz at the
//       gate/up columns of the layout (so dz keeps W1's column order); the
//       training forward saved u silu'(g) and silu(g) (bf16) for this.
//   DX  dxs[p,:] = dz[p,:] . W1[e]^T  (K = 2I, N = H).
//   DW  out[e] = sum over the rows p of segment e of A[p,:]^T B[p,:]:
//       dW2[e] = h^T dy (A = h, B = dy) and dW1[e] = x[x_gather_idx]^T dz
//       (A = x rows gathered by token, B = dz).  K is the segment length; the
//       rows past its end are zero-filled in both operands.
//
// A cluster of two CTAs owns a 256 x 256 tile: CTA r holds rows [128r, 128r+128)
// of A and columns [128r, 128r+128) of B per stage, and its TMEM the fp32
// accumulator of its 128 rows; the even CTA issues the pair MMAs and the
// commits reach both CTAs.  DH and DX tile the segments in 256-row tiles (the
// metadata's GEMM tile table); DW tiles each expert's [M,N] output.
// Operands: K-major (rows of 64 contiguous K values, 128-byte swizzle) for
// the row operands of DH/DX and for the weights read as [N][K]; MN-major
// (rows = K, 64-element MN atoms, 128-byte swizzle) for both DW operands.
// Warp roles: warp 0 = TMEM allocator and MMA issuer (even CTA) or the relay
// that forwards the odd CTA's copy completions to the even CTA; four epilogue
// warps (TMEM lane quarter warp % 4), which write full 32 x 64 output blocks
// through shared memory with TMA stores (DH also reads z through shared memory
// by TMA); one TMA producer warp (whole-stage boxes of every operand that needs
// no gather); four cp.async producer warps (the gathered dout rows of DH, and
// the zero-filled last stage of a DW segment).  In a stage with no copies the
// even CTA's TMA thread arrives for the copy warps and the relay, which keeps
// them off that stage's critical path.  Shared-memory stages of 32 KB per CTA
// (six; five for DH, whose z staging takes the room of one), two TMEM
// accumulators.  Every wait is bounded; on a timeout the CTA raises its abort
// flag, records MOE_DEVERR_TIMEOUT, drains its MMAs and copies and frees its TMEM.
#include "common.cuh"

namespace moe {

namespace {

constexpr int kM = 128;                      // rows per CTA (TMEM lanes)
constexpr int kPairM = 2 * kM;               // rows per tile (UMMA M of the pair)
constexpr int kN = 256;                      // tile columns (UMMA N)
constexpr int kNh = kN / 2;                  // B columns per CTA
constexpr int kSK = 64;                      // K per stage: one 128-byte swizzle atom of bf16
constexpr int kProducerThreads = 128;
constexpr uint32_t kStageA = kM * kSK * 2;   // 16 KB
constexpr uint32_t kStageB = kNh * kSK * 2;  // 16 KB
constexpr uint32_t kStageBytes = kStageA + kStageB;
constexpr uint32_t kMnAtom = kSK * 128;      // MN-major: one 64-element column of a stage (8 KB)
constexpr uint32_t kTmemCols = 2 * kN;
constexpr uint32_t kStoreBuf = 32 * 128;     // 4 KB per epilogue warp: 32 rows x 64 bf16 (TMA stores)
constexpr uint32_t kZBox = 32 * 128;         // DH: 32 rows x 64 bf16 of the saved factors (one TMA box)
constexpr uint32_t kZBuf = 2 * kZBox;        // DH: two boxes in flight per epilogue warp (32 dh columns each)
// Four epilogue warps, one per TMEM lane quarter.  DH also stages z per
// epilogue warp, which costs it one pipeline stage.
template <int kMode>
struct Roles {
    static constexpr int kEpiWarps = 4;
    static constexpr int kParts = 1;
    static constexpr int kTmaWarp = 1 + kEpiWarps;
    static constexpr int kCopyThread0 = 32 * (kTmaWarp + 1);
    static constexpr int kThreads = kCopyThread0 + kProducerThreads;  // MMA, epilogue, TMA, cp.async
    static constexpr int kStages = kMode == kBwdDH ? 5 : 6;
    static constexpr uint32_t kNumBars = 4 * kStages + 5 + 2 * kEpiWarps;  // + two z barriers per epilogue warp
    static constexpr size_t kStoreOff = (size_t)kStages * kStageBytes;
    static constexpr size_t kZOff = kStoreOff + (size_t)kEpiWarps * kStoreBuf;
    static constexpr size_t kBarOff = kZOff + (kMode == kBwdDH ? (size_t)kEpiWarps * kZBuf : 0);
    static constexpr size_t kMiscOff = kBarOff + 8 * kNumBars;
    static constexpr size_t kTableOff = kMiscOff + 16;
    static constexpr size_t kSmemBytes = 1024 + kTableOff + 2 * (kMaxExperts + 1) * 4;
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};
constexpr unsigned long long kAbortSettleNs = 2000000ull;

// Instruction descriptor, kind::f16: fp32 accumulate, bf16 A and B, M x N,
// each operand K-major or MN-major.
__host__ __device__ constexpr uint32_t idesc(bool a_mn, bool b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
           ((uint32_t)(kN >> 3) << 17) | ((uint32_t)(kPairM >> 4) << 24);
}

struct BTile {
    int e, m0, m_end, n0, nk;   // DW: m0 = output row, m_end = M_dim; segment rows via kp0/kp1
    int kp0, kp1;               // DW: segment rows [kp0, kp1)
};

// DH/DX: tile -> (expert, 256-row tile of its segment, 256-column tile)
__device__ __forceinline__ BTile decode_rows(int tile, int n_tiles, int E, const int *tile_off, const int *off,
                                             int K_dim) {
    BTile t;
    const int mt = tile / n_tiles;
    const int nt = tile - mt * n_tiles;
    int lo = 0, hi = E - 1;  // largest e with tile_off[e] <= mt
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tile_off[mid] <= mt) lo = mid;
        else hi = mid - 1;
    }
    t.e = lo;
    t.m0 = off[lo] + (mt - tile_off[lo]) * kPairM;
    t.m_end = off[lo + 1];
    t.n0 = nt * kN;
    t.nk = K_dim / kSK;
    t.kp0 = t.kp1 = 0;
    return t;
}

// DW: tile -> (expert, 256-row tile of its [M,N] output, 256-column tile).
// Experts are taken kDwGroup at a time, the expert index varying fastest, so
// the clusters running at once read the rows of a few experts, each expert's
// A columns and B columns shared by several tiles, and the rows stay in L2
// while its other tiles run.  Four experts (a working set of ~28 MB on
// prefill) measured best: sixteen thrashed L2 (DRAM reads twice the operand
// bytes), one or two left too few tiles per group for short segments.
constexpr int kDwGroup = 4;

__device__ __forceinline__ BTile decode_weights(int tile, int m_tiles, int n_tiles, int E, const int *off) {
    BTile t;
    const int per = m_tiles * n_tiles;
    const int g = tile / (kDwGroup * per);
    const int e0 = g * kDwGroup;
    const int ng = min(kDwGroup, E - e0);
    const int r = tile - g * (kDwGroup * per);
    t.e = e0 + r % ng;
    const int tn = r / ng;
    const int mt = tn / n_tiles;
    t.m0 = mt * kPairM;
    t.n0 = (tn - mt * n_tiles) * kN;
    t.kp0 = off[t.e];
    t.kp1 = off[t.e + 1];
    t.nk = (t.kp1 - t.kp0 + kSK - 1) / kSK;
    t.m_end = 0;
    return t;
}

// `count` arrivals on a barrier of this CTA at once
__device__ __forceinline__ void mbar_arrive_n(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

__device__ __forceinline__ void settle_after_abort() {
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < kAbortSettleNs) {
    }
}

__device__ __forceinline__ void prefetch_l2(const void *p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}


template <int kMode>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Roles<kMode>::kThreads, 1)
    bwd_gemm_kernel(const __grid_constant__ BwdGemmArgs a) {
    using R = Roles<kMode>;
    constexpr int kThreads = R::kThreads;
    constexpr int kBwdStages = R::kStages;
    constexpr bool kMN = kMode == kBwdDW;  // both operands MN-major, K = segment rows
    constexpr uint32_t kIdesc = idesc(kMN, kMN);
    extern __shared__ uint8_t smem_raw[];
    if (*(volatile uint32_t *)&a.hdr->abort) return;  // an earlier step of this call gave up

    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *base_ptr = smem_raw + (base - raw);
    auto a_stage = [&](int s) { return base + (uint32_t)s * kStageBytes; };
    auto b_stage = [&](int s) { return base + (uint32_t)s * kStageBytes + kStageA; };
    const uint32_t bars = base + (uint32_t)R::kBarOff;
    auto full_bar = [&](int s) { return bars + 8u * s; };                       // even CTA: stage ready
    auto empty_bar = [&](int s) { return bars + 8u * (kBwdStages + s); };
    auto gfull_bar = [&](int s) { return bars + 8u * (2 * kBwdStages + s); };   // odd CTA: its copies
    auto tail_bar = [&](int s) { return bars + 8u * (3 * kBwdStages + s); };    // DW: a tail stage's TMA
    auto tfull_bar = [&](int b) { return bars + 8u * (4 * kBwdStages + b); };
    auto tempty_bar = [&](int b) { return bars + 8u * (4 * kBwdStages + 2 + b); };
    const uint32_t drain_bar = bars + 8u * (4 * kBwdStages + 4);
    auto z_bar = [&](int w) { return bars + 8u * (4 * kBwdStages + 5 + w); };  // DH: z buffer w (two per warp)
    uint32_t *misc = reinterpret_cast<uint32_t *>(base_ptr + R::kMiscOff);
    int *tile_off_s = reinterpret_cast<int *>(base_ptr + R::kTableOff);
    int *off_s = tile_off_s + (kMaxExperts + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int row0 = (int)rank * kM;   // this CTA's first row inside a tile
    const int col0b = (int)rank * kNh; // this CTA's first B column inside a tile
    const int E = a.E;
    for (int i = threadIdx.x; i <= E; i += kThreads) {
        off_s[i] = __ldg(a.expert_off + i);
        if (!kMN) tile_off_s[i] = __ldg(a.tile_off + i);
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < kBwdStages; ++s) {
            // even CTA: its TMA thread + its copy threads + the odd CTA's relay
            mbar_init(full_bar(s), 1 + kProducerThreads + 1);
            mbar_init(empty_bar(s), 1);
            mbar_init(gfull_bar(s), kProducerThreads);
            mbar_init(tail_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull_bar(b), 1);
            mbar_init(tempty_bar(b), 2 * R::kEpiWarps);  // both CTAs' epilogue warps
        }
        mbar_init(drain_bar, 1);
        for (int w = 0; w < 2 * R::kEpiWarps; ++w) mbar_init(z_bar(w), 1);
        misc[1] = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (warp == 0) {
        tmem_alloc_pair(smem_u32(&misc[0]), kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();  // both CTAs' barriers initialised before any remote arrive
    tc_fence_after();

    const uint32_t tmem_base = misc[0];
    volatile uint32_t *abort = &misc[1];
    const int n_tiles = (a.N_dim + kN - 1) / kN;
    const int m_tiles = kMN ? (a.M_dim + kPairM - 1) / kPairM : 0;
    const int cluster = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;
    const int total = kMN ? E * m_tiles * n_tiles : tile_off_s[E] * n_tiles;
    auto decode = [&](int tile) {
        return kMN ? decode_weights(tile, m_tiles, n_tiles, E, off_s)
                   : decode_rows(tile, n_tiles, E, tile_off_s, off_s, a.K_dim);
    };
    // whether the copy warps (and, for the odd CTA, the relay) take part in
    // this stage: an operand comes by cp.async, or a DW segment's last stage
    // has rows past the segment end to zero.  In the other stages the even
    // CTA's TMA thread makes their arrivals on the stage barrier itself, which
    // keeps the copy warps and the relay off the stage's critical path.
    auto stage_copies = [&](const BTile &tt, int kb) {
        if (!a.a_tma || !a.b_tma) return true;
        return kMN && tt.kp0 + (kb + 1) * kSK > tt.kp1;
    };

    if (warp == 0) {
        if (rank == 0) {
            // ---------------------------------------------------- MMA issuer (even CTA)
            if (lane == 0) {
                int stage = 0;
                uint32_t phase = 0;
                int tcount = 0;
                bool ok = true;
                for (int tile = cluster; ok && tile < total; tile += n_clusters, ++tcount) {
                    const BTile t = decode(tile);
                    const int acc = tcount & 1;
                    const uint32_t acc_phase = (tcount >> 1) & 1;
                    if (!mbar_wait_bounded(tempty_bar(acc), acc_phase ^ 1u, abort)) break;
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + acc * kN;
                    for (int kb = 0; kb < t.nk; ++kb) {
                        // one barrier per stage: both CTAs' TMA bytes, this CTA's copies
                        // and the relayed copies of the odd CTA
                        if (!mbar_wait_bounded(full_bar(stage), phase, abort)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        fence_proxy_async_smem();  // copies and zeroed rows (generic proxy) -> tensor cores
                        const uint32_t sa = a_stage(stage), sb = b_stage(stage);
#pragma unroll
                        for (int kk = 0; kk < kSK / kUmmaK; ++kk) {
                            uint64_t ad, bd;
                            if (kMN) {
                                // rows = K (128 B each, 8-row groups 1024 B apart), 64-element
                                // MN columns kMnAtom apart; K step = 16 rows
                                ad = smem_desc_sw128(sa + kk * (kUmmaK * 128), kMnAtom, 1024);
                                bd = smem_desc_sw128(sb + kk * (kUmmaK * 128), kMnAtom, 1024);
                            } else {
                                // rows = M or N (128 B of K each, 8-row groups 1024 B apart);
                                // K step = 32 B inside the swizzle atom
                                ad = smem_desc_sw128(sa + kk * (kUmmaK * 2), 16, 1024);
                                bd = smem_desc_sw128(sb + kk * (kUmmaK * 2), 16, 1024);
                            }
                            umma_f16_pair(d_tmem, ad, bd, kIdesc, (kb | kk) != 0 ? 1u : 0u);
                        }
                        umma_commit_pair_mc(empty_bar(stage), 0x3);
                        if (++stage == kBwdStages) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                    if (!ok) break;
                    umma_commit_pair_mc(tfull_bar(acc), 0x3);  // with no MMA (empty segment) at once
                }
                umma_commit_pair(drain_bar);  // every MMA issued here completes before TMEM is freed
                if (!mbar_wait_timed(drain_bar, 0)) atomicOr(&a.hdr->err, MOE_DEVERR_TIMEOUT);
            }
        } else if (lane == 0) {
            // ------------------------------------------------------- relay (odd CTA)
            // forwards the completion of this CTA's copy threads to the even CTA
            int stage = 0;
            uint32_t gpar = 0;  // parity of each stage's next gfull phase (stages with copies only)
            bool ok = true;
            for (int tile = cluster; ok && tile < total; tile += n_clusters) {
                const BTile t = decode(tile);
                for (int kb = 0; kb < t.nk; ++kb) {
                    if (stage_copies(t, kb)) {
                        if (!mbar_wait_bounded(gfull_bar(stage), (gpar >> stage) & 1u, abort)) {
                            ok = false;
                            break;
                        }
                        gpar ^= 1u << stage;
                        fence_proxy_async_smem();
                        mbar_arrive_cluster(mapa_shared(full_bar(stage), 0));
                    }
                    if (++stage == kBwdStages) stage = 0;
                }
            }
        }
        __syncwarp();
    } else if (warp < R::kTmaWarp) {
        // ------------------------------------------------------------ epilogue
        const int quarter = warp & 3;
        const int rl = quarter * 32 + lane;  // this thread's tile row (TMEM lane)
        const int part = (warp - 1) >> 2;    // this warp's part of the tile's columns
        const uint32_t store_buf = base + (uint32_t)R::kStoreOff + (uint32_t)(warp - 1) * kStoreBuf;
        const uint32_t zbuf = base + (uint32_t)R::kZOff + (uint32_t)(warp - 1) * kZBuf;  // DH
        // DH: the saved factors (u silu'(g), silu(g)) of 32 dh columns [i0, i0+32) of this
        // warp's 32 rows, one TMA box of 64 bf16 per row, in buffer b of two: two boxes
        // in flight, so a chunk's DRAM latency hides behind the chunk before it
        uint32_t zphase = 0;    // bit b: the phase buffer b's barrier completes next
        uint32_t zpending = 0;  // bit b: a load into buffer b is in flight
        auto load_z = [&](int i0, int wrow0, int b) {
            if (lane == 0) {
                mbar_arrive_expect_tx(z_bar(2 * (warp - 1) + b), kZBox);
                tma_load_2d(zbuf + b * kZBox, &a.tmap_z, z_bar(2 * (warp - 1) + b), 2 * i0, wrow0);
            }
            zpending |= 1u << b;
        };
        bool ok = true;
        int tcount = 0;
        for (int tile = cluster; ok && tile < total; tile += n_clusters, ++tcount) {
            const BTile t = decode(tile);
            const int acc = tcount & 1;
            const uint32_t acc_phase = (tcount >> 1) & 1;
            const int wrow0 = t.m0 + row0 + quarter * 32;  // this warp's first tile row
            // DH, interleaved gate/up, all 32 rows of the warp in the segment: the factors
            // come in and dz goes out by TMA through shared memory, in coalesced boxes;
            // otherwise each thread reads and writes its own row
            const bool dh_tma = kMode == kBwdDH && a.layout == MOE_LAYOUT_INTERLEAVED && wrow0 + 31 < t.m_end;
            const int cfirst = part * (kN / 32 / R::kParts), clast = (part + 1) * (kN / 32 / R::kParts);
            if (dh_tma) {
                fence_proxy_async_smem();  // the buffers' last reads come before these writes
                for (int b = 0; b < 2; ++b)
                    if (cfirst + b < clast && t.n0 + 32 * (cfirst + b) < a.I) load_z(t.n0 + 32 * (cfirst + b), wrow0, b);
            }
            if (kMode == kBwdDH) {
                // bring this row's factors of the tile into L2 while the MMAs run
                const int p = t.m0 + row0 + rl;
                if (p < t.m_end) {
                    const int c0 = t.n0 + part * (kN / R::kParts);  // this warp's first I column
                    const int ncols = min(kN / R::kParts, a.I - c0);
                    const __nv_bfloat16 *zr = a.z + (size_t)p * (2 * a.I);
                    if (a.layout == MOE_LAYOUT_INTERLEAVED) {
                        for (int b = 0; b < 2 * ncols * 2; b += 128) prefetch_l2((const char *)(zr + 2 * c0) + b);
                    } else {
                        for (int b = 0; b < ncols * 2; b += 128) {
                            prefetch_l2((const char *)(zr + c0) + b);
                            prefetch_l2((const char *)(zr + a.I + c0) + b);
                        }
                    }
                }
            }
            bool w = true;
            if (lane == 0) w = mbar_wait_bounded(tfull_bar(acc), acc_phase, abort);
            w = __shfl_sync(0xffffffffu, w, 0);
            if (!w) break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + acc * kN + ((uint32_t)(quarter * 32) << 16);
            if (kMode == kBwdDH) {
                const int p = t.m0 + row0 + rl;
                const bool valid = p < t.m_end;
                const size_t zoff = (size_t)(valid ? p : 0) * (2 * a.I);
                const __nv_bfloat16 *zrow = a.z + zoff;
                __nv_bfloat16 *dzrow = a.dz + zoff;
                // the pair's score: dh = s (dout . W2^T)
                const float sc = valid ? __ldg(a.row_scale + __ldg(a.row_pair + p)) : 0.f;
#pragma unroll 1
                for (int c = cfirst; c < clast; ++c) {
                    const int i0 = t.n0 + 32 * c;
                    if (i0 >= a.I) break;
                    uint32_t dh[32];
                    tmem_ld_32x32b_x32(tbase + c * 32, dh);
                    if (dh_tma) {
                        const int b = (c - cfirst) & 1;
                        bool zw = true;
                        if (lane == 0) zw = mbar_wait_bounded(z_bar(2 * (warp - 1) + b), (zphase >> b) & 1u, abort);
                        zw = __shfl_sync(0xffffffffu, zw, 0);
                        if (!zw) {  // the load stays pending: the exit path waits for it
                            tmem_ld_wait();
                            ok = false;
                            break;
                        }
                        zphase ^= 1u << b;
                        zpending &= ~(1u << b);
                        // this row's 32 (a_j, b_j) factor pairs of columns i0 + j
                        uint32_t zr[32];
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const uint4 v = ld_shared_v4(zbuf + b * kZBox + lane * 128 + ((q ^ (lane & 7)) << 4));
                            zr[4 * q] = v.x;
                            zr[4 * q + 1] = v.y;
                            zr[4 * q + 2] = v.z;
                            zr[4 * q + 3] = v.w;
                        }
                        __syncwarp();  // every lane has read the buffer: the chunk two ahead may land
                        if (c + 2 < clast && i0 + 64 < a.I) {
                            fence_proxy_async_smem();
                            load_z(i0 + 64, wrow0, b);
                        }
                        tmem_ld_wait();
                        uint32_t o[32];  // (dg_j, du_j) packed: dz columns 2 i0 .. 2 i0 + 63
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const float d = sc * __uint_as_float(dh[j]);
                            o[j] = pack_bf16x2(d * bf16lo(zr[j]), d * bf16hi(zr[j]));
                        }
                        if (lane == 0) bulk_wait_read0();  // the buffer's previous store has been read
                        __syncwarp();
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            st_shared_v4(store_buf + lane * 128 + ((q ^ (lane & 7)) << 4), o[4 * q], o[4 * q + 1],
                                         o[4 * q + 2], o[4 * q + 3]);
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&a.tmap_out, store_buf, 2 * i0, wrow0);
                            bulk_commit();
                        }
                        continue;
                    }
                    tmem_ld_wait();
                    if (!valid) continue;
                    if (a.layout == MOE_LAYOUT_INTERLEAVED) {
                        // (a_i, b_i) adjacent: 32 pairs = 64 bf16 in, 64 bf16 out
                        const uint4 *zp = reinterpret_cast<const uint4 *>(zrow + 2 * i0);
                        uint4 *dp = reinterpret_cast<uint4 *>(dzrow + 2 * i0);
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const uint4 zv = zp[q];
                            const uint32_t zw4[4] = {zv.x, zv.y, zv.z, zv.w};
                            uint32_t o[4];
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const float d = sc * __uint_as_float(dh[4 * q + j]);
                                o[j] = pack_bf16x2(d * bf16lo(zw4[j]), d * bf16hi(zw4[j]));
                            }
                            dp[q] = make_uint4(o[0], o[1], o[2], o[3]);
                        }
                    } else {
                        // u silu'(g) at [i0, i0+32), silu(g) at [I+i0, I+i0+32)
                        const uint4 *ap = reinterpret_cast<const uint4 *>(zrow + i0);
                        const uint4 *bp = reinterpret_cast<const uint4 *>(zrow + a.I + i0);
                        uint4 *dg_out = reinterpret_cast<uint4 *>(dzrow + i0);
                        uint4 *du_out = reinterpret_cast<uint4 *>(dzrow + a.I + i0);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const uint4 av = ap[q], bv = bp[q];
                            const uint32_t aw[4] = {av.x, av.y, av.z, av.w};
                            const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
                            uint32_t og[4], ou[4];
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const float d0 = sc * __uint_as_float(dh[8 * q + 2 * j]);
                                const float d1 = sc * __uint_as_float(dh[8 * q + 2 * j + 1]);
                                og[j] = pack_bf16x2(d0 * bf16lo(aw[j]), d1 * bf16hi(aw[j]));
                                ou[j] = pack_bf16x2(d0 * bf16lo(bw[j]), d1 * bf16hi(bw[j]));
                            }
                            dg_out[q] = make_uint4(og[0], og[1], og[2], og[3]);
                            du_out[q] = make_uint4(ou[0], ou[1], ou[2], ou[3]);
                        }
                    }
                }
            } else {
                // DX: row p of dxs; DW: row m of expert e's [M,N] output.  A warp whose
                // 32 rows are all stored stages each 32 x 64 block in shared memory
                // (128-byte swizzle) and writes it with one TMA store; a DX warp that
                // straddles a segment end stores its valid rows one by one.
                const int r = wrow0 + lane;
                const bool valid = kMode == kBwdDX ? r < t.m_end : r < a.M_dim;
                const bool warp_full = kMode == kBwdDX ? wrow0 + 31 < t.m_end : wrow0 + 31 < a.M_dim;
                const int out_row0 = kMode == kBwdDX ? wrow0 : t.e * a.M_dim + wrow0;  // row in tmap_out
                const size_t row_off = kMode == kBwdDX
                                           ? (size_t)(valid ? r : 0) * a.out_ld
                                           : ((size_t)t.e * a.M_dim + (valid ? r : 0)) * a.out_ld;
                __nv_bfloat16 *orow = a.out + row_off;
                const bool zero = kMode == kBwdDW && t.nk == 0;  // empty segment: the gradient is 0
#pragma unroll 1
                for (int g = part * (kN / 64 / R::kParts); g < (part + 1) * (kN / 64 / R::kParts); ++g) {
                    const int col0 = t.n0 + 64 * g;
                    if (col0 >= a.N_dim) break;
                    uint32_t r0[32], r1[32];
                    if (!zero) {
                        tmem_ld_32x32b_x32(tbase + g * 64, r0);
                        tmem_ld_32x32b_x32(tbase + g * 64 + 32, r1);
                        tmem_ld_wait();
                    }
                    uint32_t o[32];  // 64 bf16 of this thread's row
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        o[j] = zero ? 0u : pack_bf16x2(__uint_as_float(r0[2 * j]), __uint_as_float(r0[2 * j + 1]));
                        o[16 + j] =
                            zero ? 0u : pack_bf16x2(__uint_as_float(r1[2 * j]), __uint_as_float(r1[2 * j + 1]));
                    }
                    if (warp_full) {
                        if (lane == 0) bulk_wait_read0();  // the buffer's previous store has been read
                        __syncwarp();
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            st_shared_v4(store_buf + lane * 128 + ((c ^ (lane & 7)) << 4), o[4 * c], o[4 * c + 1],
                                         o[4 * c + 2], o[4 * c + 3]);
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&a.tmap_out, store_buf, col0, out_row0);
                            bulk_commit();
                        }
                    } else if (valid) {
                        uint4 *dst = reinterpret_cast<uint4 *>(orow + col0);
#pragma unroll
                        for (int c = 0; c < 8; ++c) dst[c] = make_uint4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (rank == 0) mbar_arrive(tempty_bar(acc));
                else mbar_arrive_cluster(mapa_shared(tempty_bar(acc), 0));
            }
        }
        for (int b = 0; b < 2; ++b)  // a z load still in flight: wait for it
            if (kMode == kBwdDH && ((zpending >> b) & 1u) && lane == 0 &&
                !mbar_wait_timed(z_bar(2 * (warp - 1) + b), (zphase >> b) & 1u))
                atomicOr(&a.hdr->err, MOE_DEVERR_TIMEOUT);
        if (lane == 0) bulk_wait0();                    // this warp's TMA stores have landed
    } else if (warp == R::kTmaWarp) {
        // ---------------------------------------------------------- TMA producer
        // whole-stage boxes of the operands that need no gather: 128-byte-swizzled
        // [atom][row][128 B] boxes of a (64, rows, cols/64) view of each matrix.
        // Both CTAs' boxes complete on the even CTA's stage barrier; a DW
        // segment's last stage instead lands on each CTA's own tail barrier.
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued = 0, issued_parity = 0;
            uint32_t tissued = 0, tissued_parity = 0, tphase = 0;  // tail-stage TMAs (DW)
            bool ok = true;
            for (int tile = cluster; ok && tile < total; tile += n_clusters) {
                const BTile t = decode(tile);
                for (int kb = 0; kb < t.nk; ++kb) {
                    if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, abort)) {
                        ok = false;
                        break;
                    }
                    const int kbase = t.kp0 + kb * kSK;
                    const bool tail = kMN && kbase + kSK > t.kp1;
                    const bool ta = a.a_tma != 0, tb = a.b_tma != 0;
                    const uint32_t bytes = (ta ? kStageA : 0u) + (tb ? kStageB : 0u);
                    if (tail && bytes) {
                        // this CTA's boxes, on its own barrier; the copy warps zero the
                        // rows past the segment end, then release the stage
                        const uint32_t tb_bar = tail_bar(stage);
                        mbar_arrive_expect_tx(tb_bar, bytes);
                        if (ta) tma_load_3d(a_stage(stage), &a.tmap_a, tb_bar, 0, kbase, (t.m0 + row0) / 64);
                        if (tb) tma_load_3d(b_stage(stage), &a.tmap_b, tb_bar, 0, kbase, (t.n0 + col0b) / 64);
                        const uint32_t par = (tphase >> stage) & 1u;
                        tissued |= 1u << stage;
                        tissued_parity = (tissued_parity & ~(1u << stage)) | (par << stage);
                        tphase ^= 1u << stage;
                        if (rank == 0) mbar_arrive(full_bar(stage));
                    } else if (bytes) {
                        // both CTAs' bytes are expected by the even CTA's barrier; with
                        // no copies in this stage its TMA thread also arrives for the
                        // copy threads and the odd CTA's relay
                        if (rank == 0) {
                            mbar_arrive_expect_tx(full_bar(stage), 2 * bytes);
                            if (!stage_copies(t, kb)) mbar_arrive_n(full_bar(stage), kProducerThreads + 1);
                        }
                        const uint32_t fb = mapa_shared(full_bar(stage), 0);
                        if (kMN) {
                            if (ta) tma_load_3d_pair(a_stage(stage), &a.tmap_a, fb, 0, kbase, (t.m0 + row0) / 64);
                            if (tb)
                                tma_load_3d_pair(b_stage(stage), &a.tmap_b, fb, 0, kbase, (t.n0 + col0b) / 64);
                        } else {
                            if (ta) tma_load_3d_pair(a_stage(stage), &a.tmap_a, fb, 0, t.m0 + row0, kb);
                            if (tb)
                                tma_load_3d_pair(b_stage(stage), &a.tmap_b, fb, 0,
                                                 t.e * a.b_rows_per_expert + t.n0 + col0b, kb);
                        }
                    } else if (rank == 0) {
                        mbar_arrive(full_bar(stage));
                    }
                    // the last use of each stage, whatever filled it: its full phase
                    // completes only after every earlier phase (and its bytes)
                    issued |= 1u << stage;
                    issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == kBwdStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // the CTA may not exit while a TMA it issued can still write its memory:
            // the even CTA's stage barriers count both CTAs' boxes (the odd CTA is
            // held by the final cluster barrier until this drain ends)
            for (int st = 0; st < kBwdStages; ++st) {
                bool drained = true;
                if (rank == 0 && (issued & (1u << st)))
                    drained &= mbar_wait_timed(full_bar(st), (issued_parity >> st) & 1u);
                if (tissued & (1u << st)) drained &= mbar_wait_timed(tail_bar(st), (tissued_parity >> st) & 1u);
                if (!drained) atomicOr(&a.hdr->err, MOE_DEVERR_TIMEOUT);  // a drain that ran out is an error too
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ cp.async producers
        // the gathered operand (dout rows in DH, x rows in dW1) and, in DW, the
        // segment's last stage of both operands with the rows past its end zeroed
        const int pt = threadIdx.x - R::kCopyThread0;
        int stage = 0;
        uint32_t phase = 0;
        uint32_t tpar = 0;  // parity of each stage's next tail_bar phase
        bool ok = true;
        const int gl = pt & 31;
        for (int tile = cluster; ok && tile < total; tile += n_clusters) {
            const BTile t = decode(tile);
            // K-major gathered rows (DH): this thread's 8 row pointers, once per tile
            // (null past the segment end: those rows feed unstored outputs only)
            const __nv_bfloat16 *arow[kM / 16];
            if (!kMN && !a.a_tma) {
#pragma unroll
                for (int i = 0; i < kM / 16; ++i) {
                    const int p = t.m0 + row0 + (pt >> 3) + 16 * i;
                    arow[i] = p < t.m_end ? a.a + (size_t)(a.a_rows ? __ldg(a.a_rows + p) : p) * a.a_ld : nullptr;
                }
            }
            // MN-major gathered rows (dW1): the next stage's row indices are loaded
            // while this stage's copies are in flight
            int nrow[kSK / 8];
            auto load_rows = [&](int kb) {
                const int kbase = t.kp0 + kb * kSK;
#pragma unroll
                for (int i = 0; i < kSK / 8; ++i) {
                    const int p = kbase + (pt >> 4) + 8 * i;
                    nrow[i] = p < t.kp1 ? (a.a_rows ? __ldg(a.a_rows + p) : p) : -1;
                }
            };
            if (kMN && t.nk > 0) load_rows(0);
            for (int kb = 0; kb < t.nk; ++kb) {
                if (!stage_copies(t, kb)) {  // the TMA thread arrived for this stage
                    if (++stage == kBwdStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                    continue;
                }
                int crow[kSK / 8];
#pragma unroll
                for (int i = 0; i < kSK / 8; ++i) crow[i] = nrow[i];
                if (kMN && kb + 1 < t.nk) load_rows(kb + 1);
                // The stage is free once the MMAs of its previous use completed.  That
                // wait is only meaningful when these warps take part in every use of
                // every stage: a parity wait cannot tell a phase from the one two
                // phases earlier.  When they only zero the TMA-loaded last stage of a
                // DW segment, the tail barrier below orders them instead (its TMA is
                // issued after the producer's own wait for the free stage).
                bool w = true;
                if (gl == 0 && (!a.a_tma || !a.b_tma)) w = mbar_wait_bounded(empty_bar(stage), phase ^ 1u, abort);
                w = __shfl_sync(0xffffffffu, w, 0);
                if (!w) {
                    ok = false;
                    break;
                }
                const uint32_t sa = a_stage(stage), sb = b_stage(stage);
                if (!kMN) {
                    // K-major rows: 8 chunks of 16 B per 128-byte row, swizzled by row & 7
                    const int c = pt & 7, r0 = pt >> 3;
                    const int k0 = kb * kSK + 8 * c;
                    if (!a.a_tma) {
#pragma unroll
                        for (int i = 0; i < kM / 16; ++i) {
                            const int r = r0 + 16 * i;
                            if (arow[i]) cp_async_16(sa + r * 128 + ((c ^ (r & 7)) << 4), arow[i] + k0);
                        }
                    }
                    if (!a.b_tma) {
                        const __nv_bfloat16 *bw = a.b + (size_t)t.e * a.b_rows_per_expert * a.b_ld;
#pragma unroll
                        for (int i = 0; i < kNh / 16; ++i) {
                            const int r = r0 + 16 * i;
                            const int n = t.n0 + col0b + r;  // columns past N_dim are never stored
                            if (n < a.N_dim)
                                cp_async_16(sb + r * 128 + ((c ^ (r & 7)) << 4), bw + (size_t)n * a.b_ld + k0);
                        }
                    }
                } else {
                    // MN-major: row kr of the stage = segment row p
                    const int kbase = t.kp0 + kb * kSK;
                    const bool tail = kbase + kSK > t.kp1;
                    if (tail && (a.a_tma || a.b_tma)) {
                        // the TMA brought whole boxes: zero the rows past the segment
                        // end (they hold the next expert's rows, or unwritten memory)
                        bool tw = true;
                        if (gl == 0) tw = mbar_wait_bounded(tail_bar(stage), (tpar >> stage) & 1u, abort);
                        tw = __shfl_sync(0xffffffffu, tw, 0);
                        tpar ^= 1u << stage;
                        if (!tw) {
                            ok = false;
                            break;
                        }
                        const int rv = t.kp1 - kbase;  // rows of the segment in this stage
                        const int atoms = (a.a_tma ? 2 : 0) + (a.b_tma ? 2 : 0);
                        // 16 rows of 8 chunks per pass of the 128 threads; whole 128-byte rows
                        // are zeroed, so the swizzle does not matter
                        const int zc = pt & 7, zr = pt >> 3;
                        for (int at = 0; at < atoms; ++at) {
                            const uint32_t base_at = (a.a_tma && at < 2) ? sa + at * kMnAtom
                                                                         : sb + (at - (a.a_tma ? 2 : 0)) * kMnAtom;
                            for (int row = rv + zr; row < kSK; row += kProducerThreads / 8)
                                st_shared_v4(base_at + row * 128 + zc * 16, 0u, 0u, 0u, 0u);
                        }
                        fence_proxy_async_smem();  // the zeros are read by the tensor cores
                    }
                    if (!a.a_tma) {
                        const int c = pt & 15, kr0 = pt >> 4;  // 16 chunks per 128-element A row
                        const int m = t.m0 + row0 + 8 * c;
#pragma unroll
                        for (int i = 0; i < kSK / 8; ++i) {
                            const int kr = kr0 + 8 * i;
                            const bool in = crow[i] >= 0;  // rows past the segment end are zero
                            const uint32_t dst = sa + (c >> 3) * kMnAtom + kr * 128 + (((c & 7) ^ (kr & 7)) << 4);
                            if (m < a.M_dim)
                                cp_async_16_zfill(dst, a.a + (size_t)(in ? crow[i] : 0) * a.a_ld + m, in ? 16u : 0u);
                        }
                    }
                    if (!a.b_tma) {
                        const int c = pt & 15, kr0 = pt >> 4;  // 16 chunks per 128-element B row
                        const int n = t.n0 + col0b + 8 * c;
#pragma unroll
                        for (int i = 0; i < kSK / 8; ++i) {
                            const int kr = kr0 + 8 * i;
                            const int p = kbase + kr;
                            const bool in = p < t.kp1;
                            const uint32_t dst = sb + (c >> 3) * kMnAtom + kr * 128 + (((c & 7) ^ (kr & 7)) << 4);
                            if (n < a.N_dim)
                                cp_async_16_zfill(dst, a.b + (size_t)(in ? p : 0) * a.b_ld + n, in ? 16u : 0u);
                        }
                    }
                }
                // even CTA: straight onto the stage barrier; odd CTA: onto gfull,
                // which its relay forwards to the even CTA
                cp_async_arrive_noinc(rank == 0 ? full_bar(stage) : gfull_bar(stage));
                if (++stage == kBwdStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
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
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, kTmemCols);
    }
}

template <int kMode>
cudaError_t launch_mode(const BwdGemmArgs &a, int max_ctas, cudaStream_t s) {
    // once per device: the shared-memory limit, and how many clusters can be
    // resident at once (one CTA per SM: the shared memory allows no second)
    int fit = 1;
    cudaError_t err = launch_setup_once(
        (const void *)bwd_gemm_kernel<kMode>, &fit, [max_ctas](int, int *v) -> cudaError_t {
            cudaError_t e = cudaFuncSetAttribute(bwd_gemm_kernel<kMode>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)Roles<kMode>::kSmemBytes);
            if (e != cudaSuccess) return e;
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3((unsigned)(max_ctas & ~1));
            cfg.blockDim = dim3(Roles<kMode>::kThreads);
            cfg.dynamicSmemBytes = Roles<kMode>::kSmemBytes;
            int n = 0;
            e = cudaOccupancyMaxActiveClusters(&n, bwd_gemm_kernel<kMode>, &cfg);
            if (e != cudaSuccess) return e;
            *v = n > 0 ? n : 1;
            return cudaSuccess;
        });
    if (err != cudaSuccess) return err;
    int clusters = max_ctas / 2;
    if (clusters > fit) clusters = fit;
    if (kMode == kBwdDW) {
        const int total = a.E * ((a.M_dim + kPairM - 1) / kPairM) * ((a.N_dim + kN - 1) / kN);
        if (total < clusters) clusters = total;
    }
    if (clusters < 1) clusters = 1;
    // the kernel's cluster shape (2,1,1) is compiled in (__cluster_dims__)
    bwd_gemm_kernel<kMode><<<2 * clusters, Roles<kMode>::kThreads, Roles<kMode>::kSmemBytes, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_bwd(int mode, const BwdGemmArgs &a, int max_ctas, cudaStream_t s) {
    if (mode == kBwdDH) return launch_mode<kBwdDH>(a, max_ctas, s);
    if (mode == kBwdDX) return launch_mode<kBwdDX>(a, max_ctas, s);
    return launch_mode<kBwdDW>(a, max_ctas, s);
}

}  // namespace moe
