// Grouped GEMMs over the expert-sorted pair segments, tcgen05 + TMEM + TMA,
// for sm_100a.  One persistent CTA per SM walks a static round-robin list of
// output tiles; a tile is (expert e, 128 rows of e's segment, 256 accumulator
// columns).  The grouped GEMM is the compute core of the layer (sonic-moe
// write-up, "CuTeDSL, Triton and QuACK grouped GEMM kernels"; issue #68: the
// grouped GEMM consumes the metadata unchanged).
//
//   up   (kUp = true):  acc = x[x_gather_idx[p], :] . w1[e] (+ b1[e]),
//                       h[p, j] = silu(gate_j) * up_j   (bf16 [P_cap, I])
//        The A rows are gathered from x by four producer warps with 16-byte
//        cp.async copies written straight into the 128-byte-swizzled stage
//        (one TMA instruction per four rows proved too slow: a stage needed 32
//        of them), so no permuted copy of x is ever written.  The SwiGLU ("silu
//        times up", qwen3_5.py commit notes, recipe step 4) runs in the
//        epilogue on the fp32 accumulator.  Interleaved w1 columns
//        (g0,u0,g1,u1,...) give gate/up in adjacent accumulator columns;
//        concatenated w1 (all gates, then all ups; sonic-moe write-up,
//        "Interleaved by default, concatenated if your model is
//        HuggingFace") is loaded as 128 gate columns + the matching 128 up
//        columns, so gate and up land in columns c and c+128.
//   down (kUp = false): y[p, :] = h[p, :] . w2[e] (+ b2[e])  (bf16 [P_cap, H])
//
// Warp roles: warp 0 = TMA producer (B; and A for the down GEMM), warp 1 =
// TMEM allocator and single-thread MMA issuer, warps 2-5 = epilogue (TMEM lane
// quarter warp%4), warps 6-9 (up only) = A-row gather.  Each B stage (64 K-rows
// x 256 columns) is one TMA box of a 3-D / 4-D view of the weights.
// Pipeline: kStages shared-memory stages (A 128x64 + B 64x256 bf16, 128-byte
// swizzle), two TMEM accumulators of 128x256 fp32 so the epilogue of one tile
// overlaps the MMAs of the next.  Rows past the end of an expert's segment are
// computed (clamped gather / neighbouring rows) but never stored.
//
// Every wait is bounded (common.cuh); on a timeout the CTA raises a shared
// abort flag, records MOE_DEVERR_TIMEOUT, drains its in-flight copies and
// MMAs, frees its TMEM and returns.
#include "common.cuh"

namespace moe {

namespace {

constexpr int kGatherWarps = 4;
constexpr int kGatherThreads = 32 * kGatherWarps;
__host__ __device__ constexpr int threads_of(bool up) { return up ? 192 + kGatherThreads : 192; }
constexpr uint32_t kStageA = kBM * kBK * 2;   // 16 KB
constexpr uint32_t kStageB = kBK * kBN * 2;   // 32 KB: 4 chunks of 64 K-rows x 64 N-columns
constexpr uint32_t kChunkB = kBK * 64 * 2;    // 8 KB
constexpr uint32_t kStageBytes = kStageA + kStageB;
constexpr uint32_t kTmemCols = 2 * kBN;       // two accumulators
constexpr uint32_t kNumBars = 2 * kStages + 5;
constexpr uint32_t kIdesc = idesc_bf16_f32(kBM, kBN, /*b_mn_major=*/true);

constexpr size_t kSmemBarOff = (size_t)kStages * kStageBytes;
constexpr size_t kSmemMiscOff = kSmemBarOff + 8 * kNumBars;
constexpr size_t kSmemTableOff = kSmemMiscOff + 16;
constexpr size_t kSmemBytes = 1024 /*alignment slack*/ + kSmemTableOff + 2 * (kMaxExperts + 1) * 4;

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
    t.m0 = off[lo] + (mt - tile_off[lo]) * kBM;
    t.m_end = off[lo + 1];
    return t;
}

__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.0f + __expf(-g)) * u; }

__device__ __forceinline__ void load_bias32(const __nv_bfloat16 *b, float (&v)[32]) {
    const uint4 *p = reinterpret_cast<const uint4 *>(b);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint4 w = __ldg(p + i);
        v[8 * i + 0] = bf16lo(w.x);
        v[8 * i + 1] = bf16hi(w.x);
        v[8 * i + 2] = bf16lo(w.y);
        v[8 * i + 3] = bf16hi(w.y);
        v[8 * i + 4] = bf16lo(w.z);
        v[8 * i + 5] = bf16hi(w.z);
        v[8 * i + 6] = bf16lo(w.w);
        v[8 * i + 7] = bf16hi(w.w);
    }
}

template <bool kUp>
__global__ void __launch_bounds__(threads_of(kUp), 1) grouped_gemm_kernel(const __grid_constant__ GemmArgs a) {
    constexpr int kThreads = threads_of(kUp);
    extern __shared__ uint8_t smem_raw[];
    if (*(volatile uint32_t *)&a.hdr->abort) return;

    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *base_ptr = smem_raw + (base - raw);
    const uint32_t sA = base;
    const uint32_t sB = base + kStages * kStageA;
    const uint32_t bars = base + (uint32_t)kSmemBarOff;
    auto full_bar = [&](int s) { return bars + 8u * s; };
    auto empty_bar = [&](int s) { return bars + 8u * (kStages + s); };
    auto tfull_bar = [&](int b) { return bars + 8u * (2 * kStages + b); };
    auto tempty_bar = [&](int b) { return bars + 8u * (2 * kStages + 2 + b); };
    const uint32_t drain_bar = bars + 8u * (2 * kStages + 4);
    uint32_t *misc = reinterpret_cast<uint32_t *>(base_ptr + kSmemMiscOff);
    int *tile_off_s = reinterpret_cast<int *>(base_ptr + kSmemTableOff);
    int *off_s = tile_off_s + (kMaxExperts + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = a.E;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            // TMA producer's arrive (+ transaction bytes), plus one cp.async
            // arrival per gather thread in the up GEMM
            mbar_init(full_bar(s), 1 + (kUp ? kGatherThreads : 0));
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull_bar(b), 1);
            mbar_init(tempty_bar(b), 4);
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
        tmem_alloc(smem_u32(&misc[0]), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem_base = misc[0];
    volatile uint32_t *abort = &misc[1];
    const int n_tiles = a.n_tiles;
    const int total_tiles = tile_off_s[E] * n_tiles;
    const int nk = a.k_dim / kBK;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        constexpr uint32_t kTxBytes = kUp ? kStageB : kStageBytes;
        int stage = 0;
        uint32_t phase = 0;
        uint32_t issued = 0, issued_parity = 0;
        if (lane == 0) {
            for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
                const Tile t = decode_tile(tile, n_tiles, E, tile_off_s, off_s);
                const int brow0 = t.e * a.k_dim;
                bool ok = true;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, abort)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(full_bar(stage), kTxBytes);
                    const int k0 = kb * kBK;
                    const uint32_t b_dst = sB + stage * kStageB;
                    if (!kUp) tma_load_2d(sA + stage * kStageA, &a.tmap_a, full_bar(stage), k0, t.m0);
                    if (kUp && a.layout == MOE_LAYOUT_CONCATENATED)
                        tma_load_4d(b_dst, &a.tmap_b, full_bar(stage), 0, brow0 + k0, t.nt * 2, 0);
                    else
                        tma_load_3d(b_dst, &a.tmap_b, full_bar(stage), 0, brow0 + k0, t.nt * 4);
                    issued |= 1u << stage;
                    issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
            }
            // every copy this CTA issued must land before the CTA may exit
            for (int s = 0; s < kStages; ++s)
                if (issued & (1u << s)) mbar_wait_timed(full_bar(s), (issued_parity >> s) & 1u);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int tcount = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x, ++tcount) {
                const int acc = tcount & 1;
                const uint32_t acc_phase = (tcount >> 1) & 1;
                if (!mbar_wait_bounded(tempty_bar(acc), acc_phase ^ 1u, abort)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * kBN;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait_bounded(full_bar(stage), phase, abort)) {
                        ok = false;
                        break;
                    }
                    if (kUp) fence_proxy_async_smem();
                    tc_fence_after();
                    const uint32_t a_addr = sA + stage * kStageA;
                    const uint32_t b_addr = sB + stage * kStageB;
#pragma unroll
                    for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
                        // A: K-major, 128-byte rows, 8-row atoms 1024 B apart; K step = 32 B.
                        const uint64_t adesc = smem_desc_sw128(a_addr + kk * (kUmmaK * 2), 16, 1024);
                        // B: N-major, 64-column chunks 8 KB apart (LBO), 8-row K atoms
                        // 1024 B apart (SBO); K step = 16 rows = 2 KB.
                        const uint64_t bdesc = smem_desc_sw128(b_addr + kk * (kUmmaK * 128), kChunkB, 1024);
                        umma_f16(d_tmem, adesc, bdesc, kIdesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    umma_commit(empty_bar(stage));
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit(tfull_bar(acc));
            }
            // all MMAs issued by this thread complete before TMEM is freed
            umma_commit(drain_bar);
            mbar_wait_timed(drain_bar, 0);
        }
        __syncwarp();
    } else if (warp < 6) {
        // ------------------------------------------------------------ epilogue
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        int tcount = 0;
        for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++tcount) {
            const Tile t = decode_tile(tile, n_tiles, E, tile_off_s, off_s);
            const int acc = tcount & 1;
            const uint32_t acc_phase = (tcount >> 1) & 1;
            bool w = true;
            if (lane == 0) w = mbar_wait_bounded(tfull_bar(acc), acc_phase, abort);
            w = __shfl_sync(0xffffffffu, w, 0);
            if (!w) break;
            tc_fence_after();
            const int p = t.m0 + row;
            const bool valid = p < t.m_end;
            const uint32_t tbase = tmem_base + acc * kBN + ((uint32_t)(quarter * 32) << 16);
            __nv_bfloat16 *orow = a.out + (size_t)(valid ? p : 0) * a.out_cols;
            const __nv_bfloat16 *brow = a.bias ? a.bias + (size_t)t.e * a.n_dim : nullptr;

            if (kUp && a.layout == MOE_LAYOUT_CONCATENATED) {
                // gate = accumulator columns [0,128), up = [128,256)
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    const int col = t.nt * (kBN / 2) + c * 32;  // output column = gate column
                    if (col >= a.I) break;
                    uint32_t g[32], u[32];
                    tmem_ld_32x32b_x32(tbase + c * 32, g);
                    tmem_ld_32x32b_x32(tbase + 128 + c * 32, u);
                    tmem_ld_wait();
                    float bg[32], bu[32];
                    if (brow) {
                        load_bias32(brow + col, bg);
                        load_bias32(brow + a.I + col, bu);
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) bg[i] = bu[i] = 0.f;
                    }
                    uint32_t packed[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float h0 = silu_mul(__uint_as_float(g[2 * i]) + bg[2 * i],
                                                  __uint_as_float(u[2 * i]) + bu[2 * i]);
                        const float h1 = silu_mul(__uint_as_float(g[2 * i + 1]) + bg[2 * i + 1],
                                                  __uint_as_float(u[2 * i + 1]) + bu[2 * i + 1]);
                        packed[i] = pack_bf16x2(h0, h1);
                    }
                    if (valid) {
                        uint4 *dst = reinterpret_cast<uint4 *>(orow + col);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2],
                                                packed[4 * i + 3]);
                    }
                }
            } else if (kUp) {
                // interleaved: accumulator columns (2j, 2j+1) = (gate_j, up_j)
#pragma unroll 1
                for (int c = 0; c < 8; ++c) {
                    const int acol = t.nt * kBN + c * 32;  // column of w1
                    if (acol >= a.n_dim) break;
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(tbase + c * 32, r);
                    tmem_ld_wait();
                    float b[32];
                    if (brow) {
                        load_bias32(brow + acol, b);
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) b[i] = 0.f;
                    }
                    uint32_t packed[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float h0 = silu_mul(__uint_as_float(r[4 * i + 0]) + b[4 * i + 0],
                                                  __uint_as_float(r[4 * i + 1]) + b[4 * i + 1]);
                        const float h1 = silu_mul(__uint_as_float(r[4 * i + 2]) + b[4 * i + 2],
                                                  __uint_as_float(r[4 * i + 3]) + b[4 * i + 3]);
                        packed[i] = pack_bf16x2(h0, h1);
                    }
                    if (valid) {
                        uint4 *dst = reinterpret_cast<uint4 *>(orow + acol / 2);
                        dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
                        dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
                    }
                }
            } else {
#pragma unroll 1
                for (int c = 0; c < 8; ++c) {
                    const int col = t.nt * kBN + c * 32;
                    if (col >= a.n_dim) break;
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(tbase + c * 32, r);
                    tmem_ld_wait();
                    float b[32];
                    if (brow) {
                        load_bias32(brow + col, b);
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) b[i] = 0.f;
                    }
                    uint32_t packed[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        packed[i] = pack_bf16x2(__uint_as_float(r[2 * i]) + b[2 * i],
                                                __uint_as_float(r[2 * i + 1]) + b[2 * i + 1]);
                    if (valid) {
                        uint4 *dst = reinterpret_cast<uint4 *>(orow + col);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2],
                                                packed[4 * i + 3]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty_bar(acc));
        }
    }

    if (kUp && warp >= 6) {
        // ------------------------------------------------------- A-row gather
        // thread g: 16-byte chunk (g & 7) of rows (g >> 3) + 16 i, i = 0..7,
        // stored at row * 128 + ((chunk ^ (row & 7)) << 4): the 128-byte
        // swizzle the MMA descriptors expect.
        const int g = threadIdx.x - 192;
        const int chunk = g & 7;
        const int r0 = g >> 3;
        const int gl = g & 31;
        int stage = 0;
        uint32_t phase = 0;
        const char *xb = reinterpret_cast<const char *>(a.x);
        const size_t ld = (size_t)a.k_dim * 2;
        int tile = blockIdx.x;
        Tile t{};
        const char *src[8];
        auto load_rows = [&](const Tile &tt, const char *(&p)[8]) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int pr = min(tt.m0 + r0 + 16 * i, tt.m_end - 1);
                p[i] = xb + (size_t)__ldg(a.x_gather_idx + pr) * ld + chunk * 16;
            }
        };
        if (tile < total_tiles) {
            t = decode_tile(tile, n_tiles, E, tile_off_s, off_s);
            load_rows(t, src);
        }
        bool ok = true;
        for (; ok && tile < total_tiles; tile += gridDim.x) {
            const int next = tile + gridDim.x;
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
                const size_t koff = (size_t)kb * kBK * 2;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int row = r0 + 16 * i;
                    cp_async_16(a_dst + row * 128 + ((chunk ^ (row & 7)) << 4), src[i] + koff);
                }
                cp_async_arrive_noinc(full_bar(stage));
                if (++stage == kStages) {
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

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
    if (threadIdx.x == 0 && *abort) atomicOr(&a.hdr->err, MOE_DEVERR_TIMEOUT);
}

template <bool kUp>
cudaError_t launch(const GemmArgs &a, int grid, cudaStream_t s) {
    static bool configured[64] = {};
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 64 && !configured[dev]) {
        err = cudaFuncSetAttribute(grouped_gemm_kernel<kUp>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)kSmemBytes);
        if (err != cudaSuccess) return err;
        configured[dev] = true;
    }
    grouped_gemm_kernel<kUp><<<grid, threads_of(kUp), kSmemBytes, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

size_t gemm_smem_bytes() { return kSmemBytes; }

cudaError_t launch_gemm_up(const GemmArgs &a, int grid, cudaStream_t s) { return launch<true>(a, grid, s); }
cudaError_t launch_gemm_down(const GemmArgs &a, int grid, cudaStream_t s) { return launch<false>(a, grid, s); }

}  // namespace moe
