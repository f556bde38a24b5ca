// Shared definitions of the CUDA library: workspace header, launch-side
// structs and the sm_100a inline-PTX primitives the kernels use (mbarrier,
// TMA bulk-tensor loads, tcgen05 MMA / TMEM).  Only this library includes it.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <functional>
#include <utility>

#include "moe_nonexpand.h"

namespace moe {

// ---------------------------------------------------------------------------
// Workspace header (first 256 bytes of the workspace).
// ---------------------------------------------------------------------------
struct WsHeader {
    uint32_t reserved0;
    uint32_t err;      // MOE_DEVERR_* bits of the current call (stored whole by the metadata)
    int32_t P;         // pairs counted on the device
    uint32_t abort;    // nonzero: later kernels of this call skip their work
    uint32_t pad[60];
};
static_assert(sizeof(WsHeader) == 256, "header size");

// Tile sizes of the grouped GEMMs.
constexpr int kBM = 128;        // rows (pairs) per CTA of a tile
constexpr int kTileRows = 256;  // rows per GEMM tile (a CTA pair); the metadata's tile table counts these
constexpr int kBN = 256;        // accumulator columns per tile = UMMA N
constexpr int kBK = 64;         // K of one 128-byte swizzle atom of bf16
#ifndef MOE_STAGE_K
#define MOE_STAGE_K 128
#endif
constexpr int kGemmStageK = MOE_STAGE_K;  // K per GEMM pipeline stage (64 or 128)
constexpr int kUmmaK = 16;      // K of one tcgen05.mma kind::f16
constexpr int kStages = 4;      // shared-memory pipeline depth (4 x 48 KB)

// Metadata kernels: tiles of kMetaTileUnit * c slots, at most kMetaMaxTiles tiles,
// and a histogram table [T, hist_ld] of at most kMetaTableInts entries (every
// CTA of the scatter kernel reads all of it).
#ifndef MOE_META_TILE_UNIT
#define MOE_META_TILE_UNIT 1024
#endif
constexpr int kMetaTileUnit = MOE_META_TILE_UNIT;
constexpr int kMetaMaxTiles = 148;
constexpr int kMetaTableInts = 32768;
constexpr int kMetaThreads = 512;
constexpr int kMetaWarps = kMetaThreads / 32;
constexpr int kMaxExperts = 1024;

// Row stride of the per-tile histogram table: E rounded up to 4 (16-byte rows).
inline int meta_hist_ld(int E) { return (E + 3) & ~3; }

// Metadata tiling of NK routing slots over E experts: tiles of kMetaTileUnit * c
// slots, as few c as keep T <= min(kMetaMaxTiles, kMetaTableInts / hist_ld).
inline void meta_tiling(int64_t NK, int E, int32_t *tile_slots, int32_t *tiles) {
    int64_t tmax = kMetaTableInts / meta_hist_ld(E);
    if (tmax > kMetaMaxTiles) tmax = kMetaMaxTiles;
    if (tmax < 1) tmax = 1;
    const int64_t per = (int64_t)kMetaTileUnit * tmax;
    int64_t c = (NK + per - 1) / per;
    if (c < 1) c = 1;
    const int64_t S = (int64_t)kMetaTileUnit * c;
    int64_t T = (NK + S - 1) / S;
    if (T < 1) T = 1;
    *tile_slots = (int32_t)S;
    *tiles = (int32_t)T;
}

// Timeout of every pipeline wait (ns of %globaltimer).
constexpr unsigned long long kWaitTimeoutNs = 4000000000ull;

// ---------------------------------------------------------------------------
// Host-side launch descriptions (filled by capi.cu).
// ---------------------------------------------------------------------------
struct MetaArgs {
    const void *topk_idx;     // expert id per slot: [N,K] non-expand table, or [P] pair list
    const float *topk_w;      // weight per slot
    const void *token_idx;    // pair list: token of each slot ([P], ascending)
    int32_t pair_list;        // 1: compact pair list (token from token_idx); 0: table (slot s is token s/K)
    int32_t idx64;            // ids are int64 (else int32)
    int64_t NK;               // slots
    int32_t K;
    int32_t E;
    int64_t total_pairs;  // -1: unknown
    int64_t p_cap;
    int32_t tiles;        // T
    int32_t tile_slots;   // slots per tile
    int32_t hist_ld;      // row stride of tile_hist (meta_hist_ld(E))
    WsHeader *hdr;
    int32_t *tile_hist;   // [T,hist_ld]
    int32_t *tile_valid;  // [T]
    int32_t *tile_err;    // [T]
    int32_t *gemm_tile_off;  // [E+1] prefix of ceil(freq / kTileRows)
    moe_meta_t meta;
    int64_t N;
    int32_t *slot_pair;   // training: [NK] pair index q of each slot, -1 where the slot is no pair (or null)
};

struct GemmArgs {
    CUtensorMap tmap_a;       // down: h [P_cap,I] as (64, rows, I/64), box = one CTA's A stage (up: unused)
    CUtensorMap tmap_b;       // w1 / w2 viewed as (64 columns, K rows, column chunk[, half]):
                              // one box = this CTA's 64 x 128 half of a B stage
    CUtensorMap tmap_out;     // h [P_cap,I] / y [P_cap,H], box 64 columns x 32 rows (stores)
    CUtensorMap tmap_a16;     // down: h as (64, rows, I/64), box 64 x 16 rows x 1 (short segments)
    const __nv_bfloat16 *x;   // up: x [N,H], rows gathered with cp.async
    const int32_t *x_gather_idx;
    const int32_t *expert_off;    // [E+1]
    const int32_t *tile_off;      // [E+1]
    const __nv_bfloat16 *bias;    // b1 [E,2I] / b2 [E,H] or null
    __nv_bfloat16 *out;           // h [P_cap,I] bf16 / y [P_cap,H] (down: fp16 bits, scaled per 32 columns)
    int8_t *out_scale;            // down: y_scale [P_cap, H/32], the exponent of each row's 32-column block
    __nv_bfloat16 *z_out;         // up, training: [P_cap,2I] bf16, w1 column order: u silu'(g) at the gate
                                  // columns, silu(g) at the up columns (of z with bias), or null
    CUtensorMap tmap_z;           // up, training: z_out as [P_cap][2I], box 64 columns x 32 rows (stores)
    WsHeader *hdr;
    int32_t E;
    int32_t k_dim;        // H (up) / I (down)
    int32_t n_dim;        // 2I (up) / H (down): accumulator columns of one expert
    int32_t n_tiles;      // ceil(n_dim / kBN)
    int32_t out_cols;     // I (up) / H (down)
    int32_t I;            // intermediate size (up, concatenated layout)
    int32_t layout;       // MOE_LAYOUT_*
};

// Decode-shaped grouped GEMMs (swap-AB): 128 weight columns on the MMA's M,
// a segment's tokens (at most 128 per chunk) on its N.
struct DecodeArgs {
    CUtensorMap tmap_w;       // weights: up w1 as (64 cols, E*H rows, 2I/64 chunks) [interleaved] or
                              // (64, E*H, I/64, 2) [concatenated]; down w2 as (64, E*I, H/64); box 64 x 64 K rows
    CUtensorMap tmap_h;       // down: h [P_cap, I] as (64, rows, I/64), box 64 x (chunk rows) x 1
    const __nv_bfloat16 *x;   // up: x [N,H], rows gathered through x_gather_idx
    const int32_t *x_gather_idx;
    const int32_t *expert_off;    // [E+1]
    const __nv_bfloat16 *bias;    // b1 [E,2I] / b2 [E,H] or null
    __nv_bfloat16 *out;           // h [P_cap, I] bf16 / y [P_cap, H] (down: fp16 bits, scaled per 32 columns)
    int8_t *out_scale;            // down: y_scale [P_cap, H/32]
    WsHeader *hdr;
    int32_t E;
    int32_t k_dim;        // H (up) / I (down)
    int32_t n_out;        // output columns of one expert: 2I (up, in w1 order) / H (down)
    int32_t out_cols;     // I (up) / H (down): row length of out
    int32_t I;
    int32_t layout;       // up: MOE_LAYOUT_*
};

// Backward grouped GEMMs (one CTA per tile, M=128 x N=256, cp.async operands).
enum BwdMode : int32_t {
    kBwdDH = 0,  // dz = SwiGLU'(z) applied to s * (dout[x_gather_idx[p]] . W2[e]^T)
    kBwdDX = 1,  // dxs[P,H] = dz[P,2I] . W1[e]^T
    kBwdDW = 2,  // out[e] [M,N] = sum over the segment's rows p of A[p,:]^T B[p,:]
};

struct BwdGemmArgs {
    CUtensorMap tmap_a;        // (64, rows, cols/64) view of `a` when a_tma
    CUtensorMap tmap_b;        // (64, rows, cols/64) view of `b` when b_tma
    CUtensorMap tmap_out;      // DX/DW: `out` as [rows][N]; DH: dz [P_cap, 2I]; box 64 columns x 32 rows (stores)
    CUtensorMap tmap_z;        // DH: the saved SwiGLU factors [P_cap, 2I] bf16, box 64 columns x 32 rows
    int32_t a_tma, b_tma;      // load that operand's whole stages with TMA
    int32_t b_rows_per_expert; // DH/DX: rows of `b` per expert (N of the weights)
    const __nv_bfloat16 *a;    // DH: dout [N,H]; DX: dz [P_cap,2I]; DW: rows of length M_dim
    const int32_t *a_rows;     // DH/DW: row of `a` for segment row p (null: p itself)
    int64_t a_ld;              // elements per row of `a`
    const __nv_bfloat16 *b;    // DH/DX: weights [E][N][K] (K contiguous); DW: [P_cap, N_dim] rows p
    int64_t b_ld;              // elements per row of `b`
    const int32_t *expert_off; // [E+1] segment offsets
    const int32_t *tile_off;   // DH/DX: [E+1] prefix of ceil(freq / 256) (the metadata's GEMM tile table)
    __nv_bfloat16 *out;        // DX: [P_cap, N]; DW: [E][M][N]; DH: unused (writes z)
    int64_t out_ld;
    const __nv_bfloat16 *z;    // DH: [P_cap, 2I] bf16 (u silu'(g), silu(g)) saved by the training forward
    __nv_bfloat16 *dz;         // DH: dz [P_cap, 2I] out
    const float *row_scale;    // DH: scores in pair order, read at s_scatter_idx[p]
    const int32_t *row_pair;   // DH: s_scatter_idx (sorted position -> pair)
    WsHeader *hdr;
    int32_t E;
    int32_t M_dim;             // DW: rows of each expert's output
    int32_t N_dim;             // columns of the output (DH: I)
    int32_t K_dim;             // DH/DX: reduction length (multiple of 64)
    int32_t I;                 // DH: intermediate size
    int32_t layout;            // DH: MOE_LAYOUT_*
};

// One-time launch set-up per (kernel, device), safe to call from several host
// threads: the first call for the current device runs `setup` (which may set
// function attributes and returns an integer, e.g. an occupancy figure) under
// a lock and caches the integer; later calls return the cached value.
cudaError_t launch_setup_once(const void *kernel, int *value, const std::function<cudaError_t(int dev, int *value)> &setup);

#if defined(__CUDACC__)
// Launches kernel<<<grid, block, smem, s>>>(args...), as a programmatic
// dependent of the launch before it on s when pdl is set: the kernel may
// start before that one has finished and must call pdl_wait() before it
// reads what that one writes.
template <typename... KArgs, typename... Args>
cudaError_t launch_maybe_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl,
                             Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}
#endif

// Host-side argument checks shared by the entry points (capi.cu).
int check_routing_sizes(int64_t N, int32_t E, int32_t K, int64_t total_pairs);
bool ptr_aligned(const void *p, size_t a);

// Launchers (each defined next to its kernel).
cudaError_t launch_meta(const MetaArgs &a, cudaStream_t s);
cudaError_t launch_gemm_up(const GemmArgs &a, int max_clusters, cudaStream_t s);
cudaError_t launch_gemm_down(const GemmArgs &a, int max_clusters, cudaStream_t s);
// pdl: launched as a programmatic dependent of the previous launch on s (the
// metadata's scatter kernel before the up GEMM, the up GEMM before the down).
cudaError_t launch_decode_up(const DecodeArgs &a, int max_ctas, cudaStream_t s, bool pdl);
cudaError_t launch_decode_down(const DecodeArgs &a, int max_ctas, cudaStream_t s, bool pdl);
// y_scale null: y holds bf16 rows; else fp16 rows, y_scale [rows, H/32] their exponents.
cudaError_t launch_combine(const void *y, const int8_t *y_scale, const int32_t *token_offset, const int32_t *s_rev,
                           const float *scores, int64_t N, int32_t H, __nv_bfloat16 *out,
                           const WsHeader *hdr, int num_sms, cudaStream_t s, bool pdl);
cudaError_t launch_router(const void *logits, bool bf16, int64_t N, int E, int K, int mode, int32_t *idx, float *w,
                          int num_sms, cudaStream_t s);
size_t gemm_smem_bytes();
cudaError_t launch_gemm_bwd(int mode, const BwdGemmArgs &a, int max_ctas, cudaStream_t s);
cudaError_t launch_bwd_prep(const __nv_bfloat16 *dout, const void *y, const int8_t *y_scale, const moe_meta_t &meta, int64_t N,
                            int32_t H, __nv_bfloat16 *dy, float *ds, const int32_t *slot_pair, int64_t NK,
                            float *dweights, const WsHeader *hdr, int num_sms, cudaStream_t s);
cudaError_t launch_gather_rows(const __nv_bfloat16 *src, const int32_t *idx, const int32_t *p_total, int32_t cols,
                               __nv_bfloat16 *dst, const WsHeader *hdr, int num_sms, cudaStream_t s);
cudaError_t launch_bias_grad(const __nv_bfloat16 *src, int32_t cols, const int32_t *expert_off, int32_t E,
                             __nv_bfloat16 *db, const WsHeader *hdr, cudaStream_t s);

// ---------------------------------------------------------------------------
// Device primitives.
// ---------------------------------------------------------------------------
#if defined(__CUDACC__)

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Programmatic dependent launch (sm_90+): the primary lets its dependent
// start; the dependent waits until the primary grid has completed and its
// memory operations are visible.  Both are no-ops in a kernel launched
// without the programmatic-serialization attribute.
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %lanemask_lt;" : "=r"(m));
    return m;
}

// --- mbarrier ---------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase of `parity` to complete.  Gives up (returns false) when
// another role of the CTA raised *abort or after kWaitTimeoutNs, in which case
// it raises *abort itself.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  volatile uint32_t *abort,
                                                  unsigned long long timeout_ns = kWaitTimeoutNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 31u) == 0) {
            if (*abort) return false;
            if (globaltimer_ns() - t0 > timeout_ns) {
                *abort = 1u;
                return false;
            }
        }
    }
}

// Same, ignoring the abort flag: used only to drain copies already in flight.
__device__ __forceinline__ bool mbar_wait_timed(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer_ns() - t0 > kWaitTimeoutNs) return false;
    }
}

// --- TMA (tensor bulk copies, CTA-local destination, no multicast) ----------
__device__ __forceinline__ void tma_prefetch_desc(const void *tmap) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void *tmap, uint32_t bar, int32_t c0,
                                            int32_t c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar), "r"(c0), "r"(c1)
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void *tmap, uint32_t bar, int32_t c0,
                                            int32_t c1, int32_t c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

// Four rows (r0..r3) of a 2-D tensor, columns [c0, c0 + box), into four
// consecutive 128-byte rows of shared memory.  The tensor map's box is one row
// high.
__device__ __forceinline__ void tma_gather4(uint32_t dst, const void *tmap, uint32_t bar, int32_t c0,
                                            int32_t r0, int32_t r1, int32_t r2, int32_t r3) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar), "r"(c0), "r"(r0), "r"(r1), "r"(r2), "r"(r3)
        : "memory");
}

// --- cp.async (16-byte, L2 only) feeding shared memory ----------------------
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
// 16-byte copy that reads src_bytes (0 or 16) and zero-fills the rest.
__device__ __forceinline__ void cp_async_16_zfill(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
                 : "memory");
}
// An L2 cache policy that marks the lines an access brings in as evicted last.
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
// cp_async_16 with an L2 cache policy.
__device__ __forceinline__ void cp_async_16_hint(uint32_t dst, const void *src, uint64_t pol) {
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "l"(pol)
                 : "memory");
}
// Arrive on `bar` once every cp.async this thread issued so far has landed
// (the arrival is one of the barrier's expected arrivals).
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// TMA store of a shared-memory box to global memory (bulk-group completion).
__device__ __forceinline__ void tma_store_2d(const void *tmap, uint32_t src, int32_t c0, int32_t c1) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(tmap)),
                 "r"(src), "r"(c0), "r"(c1)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// The shared-memory sources of this thread's committed stores have been read.
__device__ __forceinline__ void bulk_wait_read0() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// This thread's committed stores are complete.
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const void *tmap, uint32_t bar, int32_t c0,
                                            int32_t c1, int32_t c2, int32_t c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

// --- clusters (CTA pairs) -----------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
// Arrive on an mbarrier given by its cluster address (possibly in the peer
// CTA), with the default (CTA-scope release) semantics: a cluster-scope
// release made every arrive cost about three stages' worth of MMA time.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// Whole-cluster barrier, called by every thread of both CTAs.
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// TMA loads into this CTA's shared memory whose completion is signalled on an
// mbarrier of either CTA of the pair (cluster address).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const void *tmap, uint32_t bar_cluster,
                                                 int32_t c0, int32_t c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar_cluster), "r"(c0), "r"(c1)
        : "memory");
}
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const void *tmap, uint32_t bar_cluster,
                                                 int32_t c0, int32_t c1, int32_t c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}
__device__ __forceinline__ void tma_load_4d_pair(uint32_t dst, const void *tmap, uint32_t bar_cluster,
                                                 int32_t c0, int32_t c1, int32_t c2, int32_t c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

// --- tcgen05 / TMEM ---------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc], kind::f16 (bf16 in, fp32 accumulate).
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on `bar` when all previously issued tcgen05 async ops of this
// thread have completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// CTA-pair forms (cta_group::2): one MMA instruction, issued by the even CTA,
// multiplies A rows held by both CTAs with B columns split between them.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void umma_f16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                              uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive once on the mbarrier at offset `bar` in every CTA of `cta_mask` when
// the pair MMAs issued so far by this thread have completed.
__device__ __forceinline__ void umma_commit_pair_mc(uint32_t bar, uint16_t cta_mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            bar),
        "h"(cta_mask)
        : "memory");
}
__device__ __forceinline__ void umma_commit_pair(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i gets lane (base_lane + i).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor (tcgen05), 128-byte swizzle.
//   bits  0-13 start address >> 4; 16-29 leading byte offset >> 4;
//   32-45 stride byte offset >> 4; 46-47 version (1 on sm_100);
//   49-51 base offset (0: atoms 1024-byte aligned); 61-63 layout (2 = 128B swizzle).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr, uint32_t lbo_bytes,
                                                    uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((addr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= 1ull << 46;
    d |= 2ull << 61;
    return d;
}

// Instruction descriptor, kind::f16: fp32 accumulate, bf16 A and B, A
// K-major (or MN-major: M contiguous), B MN-major (N contiguous) or K-major,
// shape M x N.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool b_mn_major, bool a_mn_major = false) {
    return (1u << 4)                              // D format: f32
           | (1u << 7)                            // A format: bf16
           | (1u << 10)                           // B format: bf16
           | ((a_mn_major ? 1u : 0u) << 15)       // A major
           | ((b_mn_major ? 1u : 0u) << 16)       // B major
           | ((static_cast<uint32_t>(N) >> 3) << 17)
           | ((static_cast<uint32_t>(M) >> 4) << 24);
}

// The expert rows y are stored as fp16 scaled by a power of two per row and
// 32-column block: value = fp16 * 2^e, e an int8 in y_scale[p][c / 32].  fp16
// keeps 11 significant bits (the combine sums rows that may cancel); the
// exponent keeps bf16's range.  y_block_exp(m) puts m in [2^14, 2^15) (fp16
// holds up to 65504), clamped to [-100, 113] so that 2^e and 2^-e are normal
// floats.  The grouped GEMM takes m = the block's largest |value|; the decode
// GEMM the largest over the block and up to 31 other tokens of its chunk.
// Either way every element within 2^28 of m is a normal fp16, rounded once.
constexpr int kYBlock = 32;
__device__ __forceinline__ int y_block_exp(float amax) {  // amax >= 0 (inf and NaN: the top of the range)
    const int biased = (int)((__float_as_uint(amax) >> 23) & 0xffu);
    return min(max(biased - 127 - 14, -100), 113);
}
__device__ __forceinline__ float exp2i(int e) { return __uint_as_float((uint32_t)(e + 127) << 23); }  // e in [-126,127]
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    const __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}
__device__ __forceinline__ float2 f16x2_to_f32(uint32_t v) {
    __half2 h2;
    memcpy(&h2, &v, sizeof v);
    return __half22float2(h2);
}

__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

#endif  // __CUDACC__

}  // namespace moe
