// Decode-shaped grouped GEMMs on sm_100a: swap-AB tcgen05 tiles for expert
// segments of a few rows (the 256-expert top-8 decode case of the qwen3_5.py
// commit notes; sonic-moe write-up, "Three routing strategies, selected on the
// command line", 256 experts).  With a handful of tokens per expert the layer
// is bound by reading the active experts' weights, so the weights take the
// MMA's M side and the tokens its N side:
//
//   up   (kUp = true):  Z^T[c, n] = sum_k w1[e][k][c] * x[x_gather_idx[off_e + n]][k]
//                       h[off_e + n][j] = silu(gate_j) * up_j      (bf16 [P_cap, I])
//   down (kUp = false): Y^T[c, n] = sum_k w2[e][k][c] * h[off_e + n][k]
//                       y[off_e + n][c] (fp16 with an exponent per 32 columns in y_scale)
//
// A work unit is (expert e with pairs, 128 output columns mt), dealt
// round-robin over the CTAs from a list of the active experts that each CTA
// builds first; its segment's rows are
// taken in chunks of at most 128 tokens (one chunk for a decode-sized
// segment, so each expert's weights are read once; longer segments re-read
// the unit's weight slice from L2 per chunk).  The MMA is
// tcgen05.mma.cta_group::1.kind::f16 with M = 128 (A = the weights, MN-major:
// a 64 x 64 TMA box per 64-column chunk lands in the 128-byte swizzle) and
// N = the chunk's rows rounded up to 16 (B = the token rows, K-major).  Each
// stage holds 64 K of both operands (16 KB + 16 KB) and six stages are in
// flight, so about 96 KB of weights stream into every SM at once.  The fp32
// accumulator (128 lanes = output columns x N columns = tokens) is
// double-buffered in TMEM.
//
// Warp roles (one CTA per SM, units round-robin over the CTAs): warp 0 = TMA
// producer (weights; in the down GEMM also the h rows), warp 1 = TMEM
// allocator and MMA issuer, warps 2-5 = epilogue (TMEM lane quarter warp%4),
// warps 6-7 (up only) = token-row gather with cp.async straight into the
// swizzled stage.  Every wait is bounded (common.cuh); on a timeout the CTA
// raises its abort flag, records MOE_DEVERR_TIMEOUT, drains and returns.
#include "common.cuh"

namespace moe {

namespace {

constexpr int kDM = 128;                      // output columns per unit (MMA M)
#ifndef MOE_DECODE_N
#define MOE_DECODE_N 128
#endif
#ifndef MOE_DECODE_STAGES
#define MOE_DECODE_STAGES 6
#endif
constexpr int kDN = MOE_DECODE_N;             // rows (tokens) per chunk at most (MMA N)
constexpr int kDK = 64;                       // K per stage: one 128-byte swizzle atom of bf16
constexpr int kDStages = MOE_DECODE_STAGES;
constexpr uint32_t kDChunkA = kDK * 64 * 2;   // 8 KB: 64 output columns x 64 K (MN-major)
constexpr uint32_t kDStageA = 2 * kDChunkA;   // 128 output columns
constexpr uint32_t kDStageB = kDN * kDK * 2;  // 16 KB: 128 rows x 64 K (K-major)
constexpr uint32_t kDStage = kDStageA + kDStageB;
constexpr uint32_t kDTmemCols = 2 * kDN;      // two accumulators
constexpr int kDGatherWarps = 2;
constexpr int kDGatherThreads = 32 * kDGatherWarps;
constexpr uint32_t kDNumBars = 2 * kDStages + 5;
constexpr size_t kDXchgOff = (size_t)kDStages * kDStage;          // concatenated up: 64 x 32 fp32 up values
constexpr size_t kDBarOff = kDXchgOff + 64 * 32 * 4;
constexpr size_t kDMiscOff = kDBarOff + 8 * kDNumBars;
constexpr size_t kDOffTableOff = kDMiscOff + 16;
constexpr size_t kDActOff = kDOffTableOff + (kMaxExperts + 1) * 4;   // experts with at least one pair
constexpr size_t kDSmemBytes = 1024 + kDActOff + kMaxExperts * 4;
static_assert(kDSmemBytes <= 232448, "shared memory of one CTA (227 KB)");
static_assert(kDN % 32 == 0 && kDN <= 128, "chunks of whole 32-column TMEM loads, at most the 128 of one MMA tile here");

__host__ __device__ constexpr int decode_threads(bool up) { return up ? 192 + kDGatherThreads : 192; }

__device__ __forceinline__ float silu_mul_d(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

// Named barrier of the four epilogue warps (id 1; 0 is __syncthreads).
__device__ __forceinline__ void epilogue_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ void settle() {
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 2000000ull) {
    }
}

template <bool kUp>
__global__ void __launch_bounds__(decode_threads(kUp), 1) decode_gemm_kernel(const __grid_constant__ DecodeArgs a) {
    constexpr int kThreads = decode_threads(kUp);
    extern __shared__ uint8_t smem_raw[];

    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *base_ptr = smem_raw + (base - raw);
    const uint32_t bars = base + (uint32_t)kDBarOff;
    auto full_bar = [&](int s) { return bars + 8u * s; };
    auto empty_bar = [&](int s) { return bars + 8u * (kDStages + s); };
    auto tfull_bar = [&](int b) { return bars + 8u * (2 * kDStages + b); };
    auto tempty_bar = [&](int b) { return bars + 8u * (2 * kDStages + 2 + b); };
    const uint32_t drain_bar = bars + 8u * (2 * kDStages + 4);
    uint32_t *misc = reinterpret_cast<uint32_t *>(base_ptr + kDMiscOff);
    int *off_s = reinterpret_cast<int *>(base_ptr + kDOffTableOff);
    int *act_s = reinterpret_cast<int *>(base_ptr + kDActOff);
    float *xchg = reinterpret_cast<float *>(base_ptr + kDXchgOff);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = a.E;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kDStages; ++s) {
            mbar_init(full_bar(s), 1 + (kUp ? kDGatherThreads : 0));
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
        tma_prefetch_desc(&a.tmap_w);
        if (!kUp) tma_prefetch_desc(&a.tmap_h);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&misc[0]), kDTmemCols);
        tmem_relinquish();
    }
    // Launched as a programmatic dependent, the up GEMM starts while the
    // metadata kernel runs: it waits for it here, and only then lets the
    // down GEMM start, so a running down GEMM implies finished metadata.
    // The down GEMM starts while the up GEMM runs: it reads the metadata (in
    // L2, written before the up GEMM got past its wait) at once, and its
    // producer waits for the up GEMM before the first load of h.
    if (kUp) pdl_wait();
    pdl_launch_dependents();
    for (int i = threadIdx.x; i <= E; i += kThreads) off_s[i] = __ldcg(a.expert_off + i);
    __syncthreads();
    if (warp == 0) {
        // the experts that have pairs, in order: work is dealt over these only, so
        // empty experts (many, at random, in a skewed decode batch) unbalance no CTA
        int n = 0;
        for (int e0 = 0; e0 < E; e0 += 32) {
            const int e = e0 + lane;
            const bool has = e < E && off_s[e + 1] > off_s[e];
            const unsigned m = __ballot_sync(0xffffffffu, has);
            if (has) act_s[n + __popc(m & lanemask_lt())] = e;
            n += __popc(m);
        }
        // nothing to do when the metadata found more pairs than the arrays hold
        if (lane == 0) misc[3] = __ldcg(&a.hdr->abort) ? 0u : (uint32_t)n;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem_base = misc[0];
    volatile uint32_t *abort = &misc[1];
    const bool concat = kUp && a.layout == MOE_LAYOUT_CONCATENATED;
    // units: (expert, 128 output columns); concatenated up: 64 gate + 64 up columns
    const int n_mt = concat ? a.I / 64 : (a.n_out + kDM - 1) / kDM;
    const int units = (int)misc[3] * n_mt;  // (active expert, 128 output columns)
    const int nk = a.k_dim / kDK;
    const uint32_t sA0 = base;  // stage s: weights at sA0 + s * kDStage, token rows kDStageA after them

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            auto load_w = [&](uint32_t sa, uint32_t fb, int e, int mt, int kb) {
                const int krow = e * a.k_dim + kb * kDK;
                if (concat) {
                    tma_load_4d(sa, &a.tmap_w, fb, 0, krow, mt, 0);             // gate columns
                    tma_load_4d(sa + kDChunkA, &a.tmap_w, fb, 0, krow, mt, 1);  // up columns
                } else {
                    tma_load_3d(sa, &a.tmap_w, fb, 0, krow, 2 * mt);
                }
            };
            // down: the weights of the first stages need nothing from the up
            // GEMM; they are requested before waiting for it
            int npre = 0;
            if (!kUp) {
                for (int u = blockIdx.x; npre < kDStages && u < units; u += gridDim.x) {
                    const int e = act_s[u / n_mt], mt = u - (u / n_mt) * n_mt;
                    const int Me = off_s[e + 1] - off_s[e];
                    for (int c0 = 0; npre < kDStages && c0 < Me; c0 += kDN)
                        for (int kb = 0; npre < kDStages && kb < nk; ++kb, ++npre) {
                            const uint32_t fb = full_bar(npre);  // a fresh stage: nothing to wait for
                            mbar_arrive_expect_tx(fb, kDStageA + kDStageB);
                            load_w(sA0 + npre * kDStage, fb, e, mt, kb);
                        }
                }
                pdl_wait();
            }
            int stage = 0, issued = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int u = blockIdx.x; ok && u < units; u += gridDim.x) {
                const int e = act_s[u / n_mt], mt = u - (u / n_mt) * n_mt;
                const int m0 = off_s[e], Me = off_s[e + 1] - m0;
                for (int c0 = 0; ok && c0 < Me; c0 += kDN) {
                    for (int kb = 0; kb < nk; ++kb, ++issued) {
                        const uint32_t fb = full_bar(stage);
                        const uint32_t sa = sA0 + stage * kDStage;
                        if (issued >= npre) {
                            if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, abort)) {
                                ok = false;
                                break;
                            }
                            mbar_arrive_expect_tx(fb, kDStageA + (kUp ? 0u : kDStageB));
                            load_w(sa, fb, e, mt, kb);
                        }
                        if (!kUp) tma_load_3d(sa + kDStageA, &a.tmap_h, fb, 0, m0 + c0, kb);
                        if (++stage == kDStages) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int tcount = 0;
            bool ok = true;
            for (int u = blockIdx.x; ok && u < units; u += gridDim.x) {
                const int e = act_s[u / n_mt];
                const int Me = off_s[e + 1] - off_s[e];
                for (int c0 = 0; ok && c0 < Me; c0 += kDN, ++tcount) {
                    const int nv = min(kDN, Me - c0);
                    const uint32_t idesc = idesc_bf16_f32(kDM, (nv + 15) & ~15, /*b_mn_major=*/false,
                                                          /*a_mn_major=*/true);
                    const int acc = tcount & 1;
                    if (!mbar_wait_bounded(tempty_bar(acc), ((tcount >> 1) & 1) ^ 1u, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + acc * kDN;
                    for (int kb = 0; kb < nk; ++kb) {
                        if (!mbar_wait_bounded(full_bar(stage), phase, abort)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t sa = sA0 + stage * kDStage, sb = sA0 + stage * kDStage + kDStageA;
#pragma unroll
                        for (int kk = 0; kk < kDK / kUmmaK; ++kk) {
                            // A: MN-major, 64-column chunks 8 KB apart (LBO), 8-row K groups
                            // 1024 B apart (SBO); K step of 16 rows = 2 KB
                            const uint64_t ad = smem_desc_sw128(sa + kk * (kUmmaK * 128), kDChunkA, 1024);
                            // B: K-major token rows of 128 B, 8-row atoms 1024 B apart; K step 32 B
                            const uint64_t bd = smem_desc_sw128(sb + kk * (kUmmaK * 2), 16, 1024);
                            umma_f16(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
                        }
                        umma_commit(empty_bar(stage));
                        if (++stage == kDStages) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                    if (!ok) break;
                    umma_commit(tfull_bar(acc));
                }
            }
            umma_commit(drain_bar);  // every MMA issued here completes before TMEM is freed
            if (!mbar_wait_timed(drain_bar, 0)) atomicOr(&a.hdr->err, MOE_DEVERR_TIMEOUT);
        }
        __syncwarp();
    } else if (warp < 6) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;          // TMEM lanes 32q .. 32q+31 = output rows of the unit
        volatile uint32_t *s_go = &misc[2];  // concatenated layout: the waiting warp's verdict
        const int r = 32 * q + lane;     // this thread's output row
        int tcount = 0;
        bool ok = true;
        for (int u = blockIdx.x; ok && u < units; u += gridDim.x) {
            const int e = act_s[u / n_mt], mt = u - (u / n_mt) * n_mt;
            const int m0 = off_s[e], Me = off_s[e + 1] - m0;
            for (int c0 = 0; c0 < Me; c0 += kDN, ++tcount) {
                const int nv = min(kDN, Me - c0);
                const int acc = tcount & 1;
                bool w = true;
                if (concat) {
                    // the four warps meet at named barriers below: one of them waits and
                    // all take its verdict, so they pass the same barriers or leave together
                    if (warp == 2 && lane == 0) *s_go = mbar_wait_bounded(tfull_bar(acc), (tcount >> 1) & 1, abort);
                    epilogue_bar();
                    w = *s_go != 0;
                } else {
                    if (lane == 0) w = mbar_wait_bounded(tfull_bar(acc), (tcount >> 1) & 1, abort);
                    w = __shfl_sync(0xffffffffu, w, 0);
                }
                if (!w) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t tb = tmem_base + ((uint32_t)(32 * q) << 16) + acc * kDN;
                for (int n0 = 0; n0 < nv; n0 += 32) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(tb + n0, v);
                    tmem_ld_wait();
                    if (n0 + 32 >= nv) {
                        // the accumulator's last load has landed in registers: hand it back to
                        // the MMA before this group's arithmetic and stores
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(tempty_bar(acc));
                    }
                    const int p0 = m0 + c0 + n0;  // segment row (sorted position) of column n0
                    const int nn = min(32, nv - n0);
                    if (!kUp) {
                        // y[p][c] as fp16 scaled per 32-column block.  The warp's lanes hold
                        // the 32 consecutive columns of one block (H and the warp's first
                        // column are multiples of 32: a whole warp is inside or past H) for
                        // this group of up to 32 tokens; one exponent for the group, from
                        // its largest |y| (one warp reduction), serves every token's block
                        const int c = mt * kDM + r;
                        if (c < a.n_out) {
                            const float b = a.bias ? __bfloat162float(a.bias[(size_t)e * a.n_out + c]) : 0.f;
                            float yv[32], am[16];
#pragma unroll
                            for (int n = 0; n < 32; ++n) yv[n] = __uint_as_float(v[n]) + b;
                            // the group's largest |y| over its nn tokens (columns past them are
                            // never stored): a pairwise tree, fmaxf dropping NaN
#pragma unroll
                            for (int n = 0; n < 16; ++n)
                                am[n] = fmaxf(2 * n < nn ? fabsf(yv[2 * n]) : 0.f,
                                              2 * n + 1 < nn ? fabsf(yv[2 * n + 1]) : 0.f);
#pragma unroll
                            for (int w = 8; w > 0; w >>= 1)
#pragma unroll
                                for (int n = 0; n < w; ++n) am[n] = fmaxf(am[n], am[n + w]);
                            const float tmax = am[0];
                            // |y| bits order like |y|
                            const int ex = y_block_exp(
                                __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(tmax))));
                            const float sc = exp2i(-ex);
                            uint16_t *yo = reinterpret_cast<uint16_t *>(a.out);
#pragma unroll
                            for (int n = 0; n < 32; ++n) {
                                if (n < nn) {
                                    yo[(size_t)(p0 + n) * a.out_cols + c] = __half_as_ushort(__float2half_rn(yv[n] * sc));
                                    if (lane == n)
                                        a.out_scale[(size_t)(p0 + n) * (a.out_cols / kYBlock) + c / kYBlock] =
                                            (int8_t)ex;
                                }
                            }
                        }
                    } else if (!concat) {
                        // interleaved: rows 2j / 2j+1 = gate_j / up_j, in adjacent lanes
                        const int c = mt * kDM + r;
                        const float b = a.bias ? __bfloat162float(a.bias[(size_t)e * a.n_out + c]) : 0.f;
                        float mine[32], other[32];
#pragma unroll
                        for (int n = 0; n < 32; ++n) mine[n] = __uint_as_float(v[n]) + b;
#pragma unroll
                        for (int n = 0; n < 32; ++n) other[n] = __shfl_xor_sync(0xffffffffu, mine[n], 1);
                        const int j = c >> 1;
                        // the gate lane writes tokens 0-15 of the 32, the up lane 16-31
                        if ((r & 1) == 0) {
#pragma unroll
                            for (int n = 0; n < 16; ++n)
                                if (n < nn)
                                    a.out[(size_t)(p0 + n) * a.out_cols + j] =
                                        __float2bfloat16_rn(silu_mul_d(mine[n], other[n]));
                        } else {
#pragma unroll
                            for (int n = 16; n < 32; ++n)
                                if (n < nn)
                                    a.out[(size_t)(p0 + n) * a.out_cols + j] =
                                        __float2bfloat16_rn(silu_mul_d(other[n], mine[n]));
                        }
                    } else {
                        // concatenated: rows 0-63 gate columns, 64-127 the matching up columns;
                        // the up warps pass their values through shared memory
                        const int jj = r & 63;
                        const int j = mt * 64 + jj;
                        const float b = a.bias ? __bfloat162float(a.bias[(size_t)e * a.n_out + (r < 64 ? j : a.I + j)])
                                               : 0.f;
                        if (r >= 64) {
#pragma unroll
                            for (int n = 0; n < 32; ++n) xchg[jj * 32 + ((n + jj) & 31)] = __uint_as_float(v[n]) + b;
                        }
                        epilogue_bar();
                        if (r < 64) {
#pragma unroll
                            for (int n = 0; n < 32; ++n) {
                                if (n < nn) {
                                    const float g = __uint_as_float(v[n]) + b;
                                    const float up = xchg[jj * 32 + ((n + jj) & 31)];
                                    a.out[(size_t)(p0 + n) * a.out_cols + j] = __float2bfloat16_rn(silu_mul_d(g, up));
                                }
                            }
                        }
                        epilogue_bar();
                    }
                }
            }
        }
    } else if (kUp) {
        // ------------------------------------------------------- token-row gather
        // thread g: 16-byte chunk (g & 7) of rows (g >> 3) + 8 i, i < kDN / 8,
        // stored at row * 128 + ((chunk ^ (row & 7)) << 4) (the 128-byte swizzle)
        const int g = threadIdx.x - 192;
        const int chunk = g & 7, r0 = g >> 3;
        const int gl = g & 31;
        const char *xb = reinterpret_cast<const char *>(a.x);
        const size_t ld = (size_t)a.k_dim * 2;
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int u = blockIdx.x; ok && u < units; u += gridDim.x) {
            const int e = act_s[u / n_mt];
            const int m0 = off_s[e], Me = off_s[e + 1] - m0;
            for (int c0 = 0; ok && c0 < Me; c0 += kDN) {
                const int nv = min(kDN, Me - c0);
                const char *src[kDN / 8];
#pragma unroll
                for (int i = 0; i < kDN / 8; ++i) {
                    const int rr = r0 + 8 * i;
                    src[i] = rr < nv ? xb + (size_t)__ldg(a.x_gather_idx + m0 + c0 + rr) * ld + chunk * 16 : xb;
                }
                for (int kb = 0; kb < nk; ++kb) {
                    bool w = true;
                    if (gl == 0) w = mbar_wait_bounded(empty_bar(stage), phase ^ 1u, abort);
                    w = __shfl_sync(0xffffffffu, w, 0);
                    if (!w) {
                        ok = false;
                        break;
                    }
                    const uint32_t sb = sA0 + stage * kDStage + kDStageA;
                    const size_t koff = (size_t)kb * kDK * 2;
#pragma unroll
                    for (int i = 0; i < kDN / 8; ++i) {
                        const int rr = r0 + 8 * i;
                        // rows past the chunk's end feed only accumulator columns that are never stored
                        if (rr < nv) cp_async_16(sb + rr * 128 + ((chunk ^ (rr & 7)) << 4), src[i] + koff);
                    }
                    cp_async_arrive_noinc(full_bar(stage));
                    if (++stage == kDStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
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
        settle();  // let copies already issued land
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kDTmemCols);
    }
}

template <bool kUp>
cudaError_t launch_decode(const DecodeArgs &a, int max_ctas, cudaStream_t s, bool pdl) {
    int unused = 0;
    cudaError_t err = launch_setup_once((const void *)decode_gemm_kernel<kUp>, &unused, [](int, int *v) -> cudaError_t {
        *v = 1;
        return cudaFuncSetAttribute(decode_gemm_kernel<kUp>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)kDSmemBytes);
    });
    if (err != cudaSuccess) return err;
    const int n_mt = (kUp && a.layout == MOE_LAYOUT_CONCATENATED) ? a.I / 64 : (a.n_out + kDM - 1) / kDM;
    int ctas = a.E * n_mt;
    if (ctas > max_ctas) ctas = max_ctas;
    if (ctas < 1) ctas = 1;
    return launch_maybe_pdl(decode_gemm_kernel<kUp>, dim3(ctas), dim3(decode_threads(kUp)), kDSmemBytes, s, pdl, a);
}

}  // namespace

cudaError_t launch_decode_up(const DecodeArgs &a, int max_ctas, cudaStream_t s, bool pdl) {
    return launch_decode<true>(a, max_ctas, s, pdl);
}
cudaError_t launch_decode_down(const DecodeArgs &a, int max_ctas, cudaStream_t s, bool pdl) {
    return launch_decode<false>(a, max_ctas, s, pdl);
}

}  // namespace moe
