// Host side of the C ABI declared in include/moe_nonexpand.h: argument
// checks, workspace layout, tensor-map encoding and the launch sequence
//   metadata (count, scan + scatter) -> grouped GEMM up (+b1,
//   SwiGLU) -> grouped GEMM down (+b2) -> combine
// all on the caller's stream, with no host synchronisation (the proposed
// entry point of sonic-moe issue #68 takes a stream and is meant to be
// sync-free when the pair count comes from the caller).
#include <mutex>
#include <stdio.h>
#include <string.h>

#include "common.cuh"
#include "ep.cuh"


namespace moe {

int check_routing_sizes(int64_t N, int32_t E, int32_t K, int64_t total_pairs) {
    if (N < 0 || K < 1 || K > 32 || E < 1 || E > kMaxExperts) return MOE_ERR_ARG;
    if (N * (int64_t)K >= (int64_t)(1u << 31) - (1 << 20)) return MOE_ERR_ARG;
    if (total_pairs < -1 || total_pairs > N * K) return MOE_ERR_ARG;
    return MOE_OK;
}

bool ptr_aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

cudaError_t launch_setup_once(const void *kernel, int *value,
                              const std::function<cudaError_t(int dev, int *value)> &setup) {
    struct Entry {
        const void *kernel;
        int dev;
        int value;
    };
    static std::mutex mu;
    static Entry done[1024];  // (kernel, device) pairs already set up
    static int n_done = 0;
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    std::lock_guard<std::mutex> g(mu);
    for (int i = 0; i < n_done; ++i) {
        if (done[i].kernel == kernel && done[i].dev == dev) {
            *value = done[i].value;
            return cudaSuccess;
        }
    }
    int v = 0;
    err = setup(dev, &v);
    if (err != cudaSuccess) return err;
    if (n_done < 1024) done[n_done++] = Entry{kernel, dev, v};
    *value = v;
    return cudaSuccess;
}

namespace {

constexpr size_t kAlign = 256;
constexpr int64_t kDecodeRowsPerExpert = 32;  // decode GEMMs when P_cap <= 32 E
#ifndef MOE_DECODE_N
#define MOE_DECODE_N 128
#endif
constexpr uint32_t kDecodeChunkRows = MOE_DECODE_N;  // rows of one decode chunk (its h box)

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool aligned_to(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct Layout {
    moe_ws_layout_t l;
};

int check_sizes(int64_t N, int32_t E, int32_t K, int64_t total_pairs) { return check_routing_sizes(N, E, K, total_pairs); }

int check_dense(int64_t p_cap, int32_t H, int32_t I, int32_t E) {
    if (H <= 0 || I <= 0 || (H % 64) != 0 || (I % 64) != 0) return MOE_ERR_SHAPE;
    const int64_t big = (int64_t)1 << 31;
    if ((int64_t)E * H >= big || (int64_t)E * I >= big) return MOE_ERR_SHAPE;
    if (p_cap * (int64_t)H >= big * 8 || p_cap * (int64_t)I >= big * 8) return MOE_ERR_SHAPE;
    return MOE_OK;
}

// Workspace layout for N tokens, NK routing slots and room for p_cap pairs.
moe_ws_layout_t compute_layout_nk(int64_t N, int32_t H, int32_t I, int32_t E, int64_t NK, int64_t pc) {
    moe_ws_layout_t l;
    memset(&l, 0, sizeof l);
    l.p_cap = pc;
    meta_tiling(NK, E, &l.meta_tile_slots, &l.meta_tiles);
    const size_t T = (size_t)l.meta_tiles;
    size_t o = 0;
    l.header = o;
    o = align_up(o + sizeof(WsHeader), kAlign);
    l.tile_hist = o;
    o = align_up(o + T * meta_hist_ld(E) * 4, kAlign);
    l.tile_valid = o;
    o = align_up(o + T * 4, kAlign);
    l.tile_err = o;
    o = align_up(o + T * 4, kAlign);
    l.gemm_tile_offset = o;
    o = align_up(o + (size_t)(E + 1) * 4, kAlign);
    l.meta_freq = o;
    o = align_up(o + (size_t)E * 4, kAlign);
    l.meta_off = o;
    o = align_up(o + (size_t)(E + 1) * 4, kAlign);
    l.meta_x_gather = o;
    o = align_up(o + (size_t)pc * 4, kAlign);
    l.meta_s_scatter = o;
    o = align_up(o + (size_t)pc * 4, kAlign);
    l.meta_s_rev = o;
    o = align_up(o + (size_t)pc * 4, kAlign);
    l.meta_token_offset = o;
    o = align_up(o + (size_t)(N + 1) * 4, kAlign);
    l.meta_scores = o;
    o = align_up(o + (size_t)pc * 4, kAlign);
    if (H > 0 && I > 0) {
        o = align_up(o, 1024);
        l.h = o;
        o = align_up(o + (size_t)pc * I * 2, 1024);
        l.y = o;
        o = align_up(o + (size_t)pc * H * 2, 1024);
        l.y_scale = o;
        o = align_up(o + (size_t)pc * (H / kYBlock), 1024);
    }
    l.total = o;
    if (H > 0 && I > 0) {  // training: z (bf16 factors), dz and dy after the inference workspace
        l.z = o;  // bf16: u silu'(g) at gate columns, silu(g) at up columns
        o = align_up(o + (size_t)pc * 2 * I * 2, 1024);
        l.dz = o;
        o = align_up(o + (size_t)pc * 2 * I * 2, 1024);
        l.dy = o;
        o = align_up(o + (size_t)pc * H * 2, 1024);
        l.slot_pair = o;
        o = align_up(o + (size_t)NK * 4, kAlign);
        l.ds = o;
        o = align_up(o + (size_t)pc * 4, kAlign);
    }
    l.train_total = o;
    return l;
}

moe_ws_layout_t compute_layout(int64_t N, int32_t H, int32_t I, int32_t E, int32_t K, int64_t total_pairs) {
    return compute_layout_nk(N, H, I, E, N * K, total_pairs >= 0 ? total_pairs : N * K);
}

// ---------------------------------------------------------------------------
// Routing input, either layout (checked).
// ---------------------------------------------------------------------------
struct Routing {
    bool pairs;               // compact pair list (else the non-expand [N,K] table)
    int idx64;
    int64_t N;
    int32_t K;                // [N,K] table: slots per token; pair list: 1
    int64_t NK;               // slots
    int64_t total_pairs;      // -1: unknown
    int64_t p_cap;
    const void *expert_idx;
    const float *weights;
    const void *token_idx;
};

Routing routing_topk32(const int32_t *topk_idx, const float *topk_w, int64_t N, int32_t K, int64_t total_pairs) {
    Routing r;
    r.pairs = false;
    r.idx64 = 0;
    r.N = N;
    r.K = K;
    r.NK = N * K;
    r.total_pairs = total_pairs;
    r.p_cap = total_pairs >= 0 ? total_pairs : N * K;
    r.expert_idx = topk_idx;
    r.weights = topk_w;
    r.token_idx = nullptr;
    return r;
}

int routing_from_desc(const moe_routing_t *d, int32_t E, Routing *r) {
    if (!d || E < 1 || E > kMaxExperts) return MOE_ERR_ARG;
    if (d->index_dtype != MOE_INDEX_INT32 && d->index_dtype != MOE_INDEX_INT64) return MOE_ERR_ARG;
    const size_t isz = d->index_dtype == MOE_INDEX_INT64 ? 8 : 4;
    if (d->N < 0) return MOE_ERR_ARG;
    r->idx64 = d->index_dtype == MOE_INDEX_INT64;
    r->N = d->N;
    r->expert_idx = d->expert_idx;
    r->weights = d->weights;
    if (d->kind == MOE_ROUTING_TOPK) {
        if (check_sizes(d->N, E, d->K, d->pairs)) return MOE_ERR_ARG;
        r->pairs = false;
        r->K = d->K;
        r->NK = d->N * d->K;
        r->total_pairs = d->pairs;
        r->p_cap = d->pairs >= 0 ? d->pairs : r->NK;
        r->token_idx = nullptr;
        if (d->token_idx) return MOE_ERR_ARG;
    } else if (d->kind == MOE_ROUTING_PAIRS) {
        if (d->pairs < 0 || d->pairs >= (int64_t)(1u << 31) - (1 << 20)) return MOE_ERR_ARG;
        if (d->N >= (int64_t)(1u << 31) - (1 << 20)) return MOE_ERR_ARG;
        r->pairs = true;
        r->K = 1;
        r->NK = d->pairs;
        r->total_pairs = -1;      // the list's own length bounds the pairs
        r->p_cap = d->pairs;
        r->token_idx = d->token_idx;
        if (r->NK > 0 && !r->token_idx) return MOE_ERR_ARG;
        if (r->token_idx && !aligned_to(r->token_idx, isz)) return MOE_ERR_ARG;
    } else {
        return MOE_ERR_ARG;
    }
    if (r->NK > 0 && (!r->expert_idx || !r->weights)) return MOE_ERR_ARG;
    if (!aligned_to(r->expert_idx, isz) || !aligned_to(r->weights, 4)) return MOE_ERR_ARG;
    return MOE_OK;
}

// ---------------------------------------------------------------------------
// Per-device facts.
// ---------------------------------------------------------------------------
struct DeviceInfo {
    bool ok = false;
    int sms = 0;
    int status = MOE_ERR_DEVICE;
};

int device_info(DeviceInfo *out) {
    static std::mutex mu;
    static DeviceInfo cache[64];
    static bool have[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> g(mu);
    if (dev < 0 || dev >= 64) return MOE_ERR_DEVICE;
    if (!have[dev]) {
        DeviceInfo d;
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return MOE_ERR_CUDA;
        d.sms = sms;
        d.ok = (major == 10 && minor == 0);
        d.status = d.ok ? MOE_OK : MOE_ERR_DEVICE;
        cache[dev] = d;
        have[dev] = true;
    }
    *out = cache[dev];
    return out->status;
}

// ---------------------------------------------------------------------------
// Tensor maps through the driver entry point (no link against libcuda).
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

bool make_map_2d(CUtensorMap *m, const void *ptr, uint64_t inner, uint64_t outer, uint32_t box_inner,
                 uint32_t box_outer) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {inner * 2};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A row-major weight [rows][ncols] (ncols % 64 == 0) viewed as
// (64 columns, rows, ncols/64 column chunks): one box of 64 x stage-K x 2 lands in
// shared memory as two 64-column chunks of stage-K rows each -- the
// N-major operand layout of one CTA's 128-column half of a 256-column stage.
bool make_map_b_chunks(CUtensorMap *m, const void *ptr, uint64_t ncols, uint64_t rows) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[3] = {64, rows, ncols / 64};
    cuuint64_t strides[2] = {ncols * 2, 128};
    cuuint32_t box[3] = {64, (cuuint32_t)kGemmStageK, (cuuint32_t)(kBN / 128)};
    cuuint32_t estr[3] = {1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A row-major weight [rows][ncols] viewed as (64 columns, rows, ncols/64
// chunks) with a box of 64 x box_rows x 2: 128 columns of box_rows K rows
// (the decode GEMMs' MN-major weight operand).
bool make_map_w_chunks(CUtensorMap *m, const void *ptr, uint64_t ncols, uint64_t rows, uint32_t box_rows) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[3] = {64, rows, ncols / 64};
    cuuint64_t strides[2] = {ncols * 2, 128};
    cuuint32_t box[3] = {64, box_rows, 2};
    cuuint32_t estr[3] = {1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// w1 in the concatenated layout [rows][2][I] viewed as (64 columns, rows, I/64
// chunks, gate/up half) with a box of 64 x box_rows x 1 x 1: one 64-column
// chunk of the gate or of the up half (the decode up GEMM loads one of each).
bool make_map_w1_concat_rows(CUtensorMap *m, const void *ptr, uint64_t I, uint64_t rows, uint32_t box_rows) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[4] = {64, rows, I / 64, 2};
    cuuint64_t strides[3] = {I * 4, 128, I * 2};
    cuuint32_t box[4] = {64, box_rows, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// h [rows][I] viewed as (64 columns, rows, I/64 column chunks): a box of
// 64 x 128 rows x (stage K / 64) is one CTA's A stage (64-wide K atoms 16 KB
// apart); a box of 64 x 16 rows x 1 is one 16-row group of one atom.
bool make_map_a_chunks(CUtensorMap *m, const void *ptr, uint64_t ncols, uint64_t rows, uint32_t box_rows,
                       uint32_t box_atoms) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[3] = {64, rows, ncols / 64};
    cuuint64_t strides[2] = {ncols * 2, 128};
    cuuint32_t box[3] = {64, box_rows, box_atoms};
    cuuint32_t estr[3] = {1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// w1 in the concatenated layout [rows][2][I] viewed as (64 columns, rows,
// I/64 chunks, gate/up half): one box of 64 x stage-K x 2 x 1 is two 64-column
// chunks of the gate half (even CTA) or of the up half (odd CTA), 8 KB apart.
bool make_map_w1_concat(CUtensorMap *m, const void *ptr, uint64_t I, uint64_t rows) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[4] = {64, rows, I / 64, 2};
    cuuint64_t strides[3] = {I * 4, 128, I * 2};
    cuuint32_t box[4] = {64, (cuuint32_t)kGemmStageK, 2, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

MetaArgs meta_args(const Routing &r, int32_t E, const moe_ws_layout_t &l, uint8_t *ws, const moe_meta_t &meta) {
    MetaArgs a;
    a.topk_idx = r.expert_idx;
    a.topk_w = r.weights;
    a.token_idx = r.token_idx;
    a.pair_list = r.pairs ? 1 : 0;
    a.idx64 = r.idx64;
    a.NK = r.NK;
    a.K = r.K;
    a.E = E;
    a.total_pairs = r.total_pairs;
    a.p_cap = l.p_cap;
    a.tiles = l.meta_tiles;
    a.tile_slots = l.meta_tile_slots;
    a.hist_ld = meta_hist_ld(E);
    a.hdr = reinterpret_cast<WsHeader *>(ws + l.header);
    a.tile_hist = reinterpret_cast<int32_t *>(ws + l.tile_hist);
    a.tile_valid = reinterpret_cast<int32_t *>(ws + l.tile_valid);
    a.tile_err = reinterpret_cast<int32_t *>(ws + l.tile_err);
    a.gemm_tile_off = reinterpret_cast<int32_t *>(ws + l.gemm_tile_offset);
    a.meta = meta;
    a.N = r.N;
    a.slot_pair = nullptr;
    return a;
}

moe_meta_t ws_meta(const moe_ws_layout_t &l, uint8_t *ws) {
    moe_meta_t m;
    m.expert_frequency = reinterpret_cast<int32_t *>(ws + l.meta_freq);
    m.expert_frequency_offset = reinterpret_cast<int32_t *>(ws + l.meta_off);
    m.x_gather_idx = reinterpret_cast<int32_t *>(ws + l.meta_x_gather);
    m.s_scatter_idx = reinterpret_cast<int32_t *>(ws + l.meta_s_scatter);
    m.s_reverse_scatter_idx = reinterpret_cast<int32_t *>(ws + l.meta_s_rev);
    m.token_offset = reinterpret_cast<int32_t *>(ws + l.meta_token_offset);
    m.scores = reinterpret_cast<float *>(ws + l.meta_scores);
    return m;
}

bool meta_complete(const moe_meta_t *m) {
    return m && m->expert_frequency && m->expert_frequency_offset && m->x_gather_idx && m->s_scatter_idx &&
           m->s_reverse_scatter_idx && m->token_offset && m->scores;
}

int record(const moe_event_t *ev, int i, cudaStream_t s) {
    if (!ev) return MOE_OK;
    return cudaEventRecord(reinterpret_cast<cudaEvent_t>(ev[i]), s) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int forward_impl(const void *x, const Routing &r, int32_t H, int32_t I, int32_t E, const void *w1,
                 const void *b1, const void *w2, const void *b2, int32_t activation, int32_t layout_kind,
                 void *out, const moe_meta_t *meta_out, void *ws, size_t ws_bytes, cudaStream_t s,
                 const moe_event_t *ev, bool train = false) {
    const int64_t N = r.N;
    int st = MOE_OK;
    // with N == 0 the token-sized buffers may be empty (null)
    if ((N > 0 && (!x || !out)) || (r.NK > 0 && (!r.expert_idx || !r.weights)) || !w1 || !w2)
        return MOE_ERR_ARG;
    if (activation != MOE_ACT_SWIGLU) return MOE_ERR_ARG;
    if (layout_kind != MOE_LAYOUT_INTERLEAVED && layout_kind != MOE_LAYOUT_CONCATENATED) return MOE_ERR_ARG;
    if (meta_out && !meta_complete(meta_out)) return MOE_ERR_ARG;
    if (!aligned(x, 16) || !aligned(w1, 16) || !aligned(w2, 16) || !aligned(out, 16) ||
        (b1 && !aligned(b1, 16)) || (b2 && !aligned(b2, 16)))
        return MOE_ERR_ARG;
    const moe_ws_layout_t l = compute_layout_nk(N, H, I, E, r.NK, r.p_cap);
    st = check_dense(l.p_cap, H, I, E);
    if (st) return st;
    if (!ws || !aligned(ws, kAlign) || ws_bytes < (train ? l.train_total : l.total)) return MOE_ERR_WS;
    DeviceInfo dev;
    st = device_info(&dev);
    if (st) return st;

    uint8_t *w = static_cast<uint8_t *>(ws);
    const moe_meta_t meta = meta_out ? *meta_out : ws_meta(l, w);
    MetaArgs ma = meta_args(r, E, l, w, meta);
    if (train) ma.slot_pair = reinterpret_cast<int32_t *>(w + l.slot_pair);  // for the backward's score gradients
    WsHeader *hdr = ma.hdr;

    if ((st = record(ev, 0, s))) return st;
    if (launch_meta(ma, s) != cudaSuccess) return MOE_ERR_CUDA;
    if ((st = record(ev, 1, s))) return st;

    __nv_bfloat16 *hbuf = reinterpret_cast<__nv_bfloat16 *>(w + l.h);
    __nv_bfloat16 *ybuf = reinterpret_cast<__nv_bfloat16 *>(w + l.y);
    int8_t *yscale = reinterpret_cast<int8_t *>(w + l.y_scale);
    // Segments of a few rows on average (decode): swap-AB kernels that stream
    // each active expert's weights once.  Chosen per call from the sizes alone
    // (no host sync); they handle segments of any length.
    const bool decode = !train && l.p_cap > 0 && l.p_cap <= (int64_t)kDecodeRowsPerExpert * E;
    // Kernels after the metadata start as programmatic dependents of the one
    // before (their set-up and, in the decode down GEMM, the first weight
    // loads overlap it), unless stage events sit between the launches.
    const bool pdl = ev == nullptr;
    if (decode) {
        DecodeArgs up;
        memset(&up, 0, sizeof up);
        if (layout_kind == MOE_LAYOUT_CONCATENATED) {
            if (!make_map_w1_concat_rows(&up.tmap_w, w1, (uint64_t)I, (uint64_t)E * H, 64)) return MOE_ERR_CUDA;
        } else {
            if (!make_map_w_chunks(&up.tmap_w, w1, (uint64_t)2 * I, (uint64_t)E * H, 64)) return MOE_ERR_CUDA;
        }
        up.x = static_cast<const __nv_bfloat16 *>(x);
        up.x_gather_idx = meta.x_gather_idx;
        up.expert_off = meta.expert_frequency_offset;
        up.bias = static_cast<const __nv_bfloat16 *>(b1);
        up.out = hbuf;
        up.hdr = hdr;
        up.E = E;
        up.k_dim = H;
        up.n_out = 2 * I;
        up.out_cols = I;
        up.I = I;
        up.layout = layout_kind;
        if (launch_decode_up(up, dev.sms, s, pdl) != cudaSuccess) return MOE_ERR_CUDA;
        if ((st = record(ev, 2, s))) return st;
        DecodeArgs dn;
        memset(&dn, 0, sizeof dn);
        if (!make_map_w_chunks(&dn.tmap_w, w2, (uint64_t)H, (uint64_t)E * I, 64) ||
            !make_map_a_chunks(&dn.tmap_h, hbuf, (uint64_t)I, (uint64_t)l.p_cap, kDecodeChunkRows, 1))
            return MOE_ERR_CUDA;
        dn.expert_off = meta.expert_frequency_offset;
        dn.bias = static_cast<const __nv_bfloat16 *>(b2);
        dn.out = ybuf;
        dn.out_scale = yscale;
        dn.hdr = hdr;
        dn.E = E;
        dn.k_dim = I;
        dn.n_out = H;
        dn.out_cols = H;
        dn.I = I;
        dn.layout = MOE_LAYOUT_INTERLEAVED;
        if (launch_decode_down(dn, dev.sms, s, pdl) != cudaSuccess) return MOE_ERR_CUDA;
        if ((st = record(ev, 3, s))) return st;
    } else if (l.p_cap > 0) {
        const int64_t cap_mtiles = (l.p_cap + kTileRows - 1) / kTileRows + E;
        // ---- up: x gathered rows . w1 -> h
        GemmArgs up;
        memset(&up, 0, sizeof up);
        if (layout_kind == MOE_LAYOUT_CONCATENATED) {
            if (!make_map_w1_concat(&up.tmap_b, w1, (uint64_t)I, (uint64_t)E * H)) return MOE_ERR_CUDA;
        } else {
            if (!make_map_b_chunks(&up.tmap_b, w1, (uint64_t)2 * I, (uint64_t)E * H)) return MOE_ERR_CUDA;
        }
        up.x = static_cast<const __nv_bfloat16 *>(x);
        if (!make_map_2d(&up.tmap_out, hbuf, (uint64_t)I, (uint64_t)l.p_cap, 64, 32)) return MOE_ERR_CUDA;
        up.x_gather_idx = meta.x_gather_idx;
        up.expert_off = meta.expert_frequency_offset;
        up.tile_off = ma.gemm_tile_off;
        up.bias = static_cast<const __nv_bfloat16 *>(b1);
        up.out = hbuf;
        up.z_out = train ? reinterpret_cast<__nv_bfloat16 *>(w + l.z) : nullptr;
        if (train && !make_map_2d(&up.tmap_z, up.z_out, (uint64_t)2 * I, (uint64_t)l.p_cap, 64, 32))
            return MOE_ERR_CUDA;
        up.hdr = hdr;
        up.E = E;
        up.k_dim = H;
        up.n_dim = 2 * I;
        up.n_tiles = (2 * I + kBN - 1) / kBN;
        up.out_cols = I;
        up.I = I;
        up.layout = layout_kind;
        int64_t clusters = cap_mtiles * up.n_tiles;
        if (clusters > dev.sms / 2) clusters = dev.sms / 2;
        if (launch_gemm_up(up, (int)clusters, s) != cudaSuccess) return MOE_ERR_CUDA;
        if ((st = record(ev, 2, s))) return st;

        // ---- down: h . w2 -> y
        GemmArgs dn;
        memset(&dn, 0, sizeof dn);
        if (!make_map_a_chunks(&dn.tmap_a, hbuf, (uint64_t)I, (uint64_t)l.p_cap, kBM, kGemmStageK / 64))
            return MOE_ERR_CUDA;
        if (!make_map_a_chunks(&dn.tmap_a16, hbuf, (uint64_t)I, (uint64_t)l.p_cap, 16, 1)) return MOE_ERR_CUDA;
        if (!make_map_b_chunks(&dn.tmap_b, w2, (uint64_t)H, (uint64_t)E * I)) return MOE_ERR_CUDA;
        if (!make_map_2d(&dn.tmap_out, ybuf, (uint64_t)H, (uint64_t)l.p_cap, 64, 32)) return MOE_ERR_CUDA;
        dn.out_scale = yscale;
        dn.expert_off = meta.expert_frequency_offset;
        dn.tile_off = ma.gemm_tile_off;
        dn.bias = static_cast<const __nv_bfloat16 *>(b2);
        dn.out = ybuf;
        dn.hdr = hdr;
        dn.E = E;
        dn.k_dim = I;
        dn.n_dim = H;
        dn.n_tiles = (H + kBN - 1) / kBN;
        dn.out_cols = H;
        dn.I = I;
        dn.layout = MOE_LAYOUT_INTERLEAVED;
        clusters = cap_mtiles * dn.n_tiles;
        if (clusters > dev.sms / 2) clusters = dev.sms / 2;
        if (launch_gemm_down(dn, (int)clusters, s) != cudaSuccess) return MOE_ERR_CUDA;
        if ((st = record(ev, 3, s))) return st;
    } else {
        if ((st = record(ev, 2, s))) return st;
        if ((st = record(ev, 3, s))) return st;
    }
    if (launch_combine(ybuf, yscale, meta.token_offset, meta.s_reverse_scatter_idx, meta.scores, N, H,
                       static_cast<__nv_bfloat16 *>(out), hdr, dev.sms, s, pdl) != cudaSuccess)
        return MOE_ERR_CUDA;
    if ((st = record(ev, 4, s))) return st;
    return MOE_OK;
}

int backward_impl(const void *dout, const void *x, const Routing &r, int32_t H, int32_t I, int32_t E,
                  const void *w1, const void *w2, int32_t activation, int32_t layout_kind, void *dx, void *dw1,
                  void *db1, void *dw2, void *db2, float *dweights, void *ws, size_t ws_bytes, cudaStream_t s,
                  const moe_event_t *ev) {
    const int64_t N = r.N;
    int st = MOE_OK;
    if ((N > 0 && (!dout || !x || !dx)) || (r.NK > 0 && !dweights) || !w1 || !w2 || !dw1 || !dw2)
        return MOE_ERR_ARG;
    if (activation != MOE_ACT_SWIGLU) return MOE_ERR_ARG;
    if (layout_kind != MOE_LAYOUT_INTERLEAVED && layout_kind != MOE_LAYOUT_CONCATENATED) return MOE_ERR_ARG;
    if (!aligned(dout, 16) || !aligned(x, 16) || !aligned(w1, 16) || !aligned(w2, 16) || !aligned(dx, 16) ||
        !aligned(dw1, 16) || !aligned(dw2, 16) || (db1 && !aligned(db1, 16)) || (db2 && !aligned(db2, 16)) ||
        !aligned(dweights, 4))
        return MOE_ERR_ARG;
    const moe_ws_layout_t l = compute_layout_nk(N, H, I, E, r.NK, r.p_cap);
    st = check_dense(l.p_cap, H, I, E);
    if (st) return st;
    if (!ws || !aligned(ws, kAlign) || ws_bytes < l.train_total) return MOE_ERR_WS;
    DeviceInfo dev;
    st = device_info(&dev);
    if (st) return st;

    uint8_t *w = static_cast<uint8_t *>(ws);
    const moe_meta_t meta = ws_meta(l, w);
    WsHeader *hdr = reinterpret_cast<WsHeader *>(w + l.header);
    auto bf = [&](size_t off) { return reinterpret_cast<__nv_bfloat16 *>(w + off); };
    __nv_bfloat16 *hbuf = bf(l.h), *ybuf = bf(l.y), *dzbuf = bf(l.dz), *dybuf = bf(l.dy);
    const __nv_bfloat16 *zbuf = reinterpret_cast<const __nv_bfloat16 *>(w + l.z);
    const __nv_bfloat16 *w1b = static_cast<const __nv_bfloat16 *>(w1);
    const __nv_bfloat16 *w2b = static_cast<const __nv_bfloat16 *>(w2);

    if ((st = record(ev, 0, s))) return st;
    // score gradients (to the [N,K] slots) and dy = s dout per pair
    if (launch_bwd_prep(static_cast<const __nv_bfloat16 *>(dout), ybuf, reinterpret_cast<const int8_t *>(w + l.y_scale),
                        meta, N, H, dybuf,
                        reinterpret_cast<float *>(w + l.ds), reinterpret_cast<const int32_t *>(w + l.slot_pair),
                        r.NK, dweights, hdr, dev.sms, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    if ((st = record(ev, 1, s))) return st;

    const uint64_t prow = (uint64_t)(l.p_cap > 0 ? l.p_cap : 1);
    BwdGemmArgs g;
    memset(&g, 0, sizeof g);
    g.expert_off = meta.expert_frequency_offset;
    g.tile_off = reinterpret_cast<const int32_t *>(w + l.gemm_tile_offset);
    g.hdr = hdr;
    g.E = E;
    g.I = I;
    g.layout = layout_kind;
    // dh = s (dout[x_gather_idx] . W2[e]^T), SwiGLU backward: z -> dz
    {
        BwdGemmArgs a = g;
        a.a = static_cast<const __nv_bfloat16 *>(dout);
        a.a_rows = meta.x_gather_idx;
        a.a_ld = H;
        a.b = w2b;
        a.b_ld = H;
        a.b_rows_per_expert = I;
        if (!make_map_a_chunks(&a.tmap_b, w2b, (uint64_t)H, (uint64_t)E * I, 128, 1)) return MOE_ERR_CUDA;
        a.b_tma = 1;
        if (!make_map_2d(&a.tmap_z, zbuf, (uint64_t)2 * I, prow, 64, 32) ||
            !make_map_2d(&a.tmap_out, dzbuf, (uint64_t)2 * I, prow, 64, 32))
            return MOE_ERR_CUDA;
        a.z = zbuf;
        a.dz = dzbuf;
        a.row_scale = meta.scores;
        a.row_pair = meta.s_scatter_idx;
        a.N_dim = I;
        a.K_dim = H;
        if (launch_gemm_bwd(kBwdDH, a, dev.sms, s) != cudaSuccess) return MOE_ERR_CUDA;
    }
    if ((st = record(ev, 2, s))) return st;
    // dW2[e] = h^T dy
    {
        BwdGemmArgs a = g;
        a.a = hbuf;
        a.a_ld = I;
        a.b = dybuf;
        a.b_ld = H;
        if (!make_map_a_chunks(&a.tmap_a, hbuf, (uint64_t)I, prow, 64, 2) ||
            !make_map_a_chunks(&a.tmap_b, dybuf, (uint64_t)H, prow, 64, 2))
            return MOE_ERR_CUDA;
        a.a_tma = a.b_tma = 1;
        if (!make_map_2d(&a.tmap_out, dw2, (uint64_t)H, (uint64_t)E * I, 64, 32)) return MOE_ERR_CUDA;
        a.out = static_cast<__nv_bfloat16 *>(dw2);
        a.out_ld = H;
        a.M_dim = I;
        a.N_dim = H;
        if (launch_gemm_bwd(kBwdDW, a, dev.sms, s) != cudaSuccess) return MOE_ERR_CUDA;
    }
    if ((st = record(ev, 3, s))) return st;
    // dW1[e] = xs^T dz with xs = x[x_gather_idx] gathered into the (no longer
    // needed) y region, so both operands load by TMA
    if (launch_gather_rows(static_cast<const __nv_bfloat16 *>(x), meta.x_gather_idx, meta.expert_frequency_offset + E,
                           H, ybuf, hdr, dev.sms, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    {
        BwdGemmArgs a = g;
        a.a = ybuf;
        a.a_ld = H;
        a.b = dzbuf;
        a.b_ld = 2 * I;
        if (!make_map_a_chunks(&a.tmap_a, ybuf, (uint64_t)H, prow, 64, 2) ||
            !make_map_a_chunks(&a.tmap_b, dzbuf, (uint64_t)2 * I, prow, 64, 2))
            return MOE_ERR_CUDA;
        a.a_tma = a.b_tma = 1;
        if (!make_map_2d(&a.tmap_out, dw1, (uint64_t)2 * I, (uint64_t)E * H, 64, 32)) return MOE_ERR_CUDA;
        a.out = static_cast<__nv_bfloat16 *>(dw1);
        a.out_ld = 2 * I;
        a.M_dim = H;
        a.N_dim = 2 * I;
        if (launch_gemm_bwd(kBwdDW, a, dev.sms, s) != cudaSuccess) return MOE_ERR_CUDA;
    }
    if ((st = record(ev, 4, s))) return st;
    // dx rows = dz . W1[e]^T, into the y region (xs is no longer needed)
    {
        BwdGemmArgs a = g;
        a.a = dzbuf;
        a.a_ld = 2 * I;
        a.b = w1b;
        a.b_ld = 2 * I;
        a.b_rows_per_expert = H;
        if (!make_map_a_chunks(&a.tmap_a, dzbuf, (uint64_t)2 * I, prow, 128, 1) ||
            !make_map_a_chunks(&a.tmap_b, w1b, (uint64_t)2 * I, (uint64_t)E * H, 128, 1))
            return MOE_ERR_CUDA;
        a.a_tma = a.b_tma = 1;
        if (!make_map_2d(&a.tmap_out, ybuf, (uint64_t)H, prow, 64, 32)) return MOE_ERR_CUDA;
        a.out = ybuf;
        a.out_ld = H;
        a.N_dim = H;
        a.K_dim = 2 * I;
        if (launch_gemm_bwd(kBwdDX, a, dev.sms, s) != cudaSuccess) return MOE_ERR_CUDA;
    }
    if ((st = record(ev, 5, s))) return st;
    // dx[t] = sum of its pairs' dx rows (weight 1)
    if (launch_combine(ybuf, nullptr, meta.token_offset, meta.s_reverse_scatter_idx, nullptr, N, H,
                       static_cast<__nv_bfloat16 *>(dx), hdr, dev.sms, s, false) != cudaSuccess)
        return MOE_ERR_CUDA;
    if ((st = record(ev, 6, s))) return st;
    if (db2 && launch_bias_grad(dybuf, H, meta.expert_frequency_offset, E, static_cast<__nv_bfloat16 *>(db2), hdr,
                                s) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (db1 && launch_bias_grad(dzbuf, 2 * I, meta.expert_frequency_offset, E, static_cast<__nv_bfloat16 *>(db1),
                                hdr, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    if ((st = record(ev, 7, s))) return st;
    return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" MOE_API size_t moe_nonexpand_train_workspace_bytes(int64_t N, int32_t H, int32_t I, int32_t E, int32_t K,
                                                              int64_t total_pairs) {
    if (check_sizes(N, E, K, total_pairs)) return 0;
    if (H <= 0 || I <= 0) return 0;
    const moe_ws_layout_t l = compute_layout(N, H, I, E, K, total_pairs);
    if (check_dense(l.p_cap, H, I, E)) return 0;
    return l.train_total;
}

extern "C" MOE_API int moe_nonexpand_forward_train(const void *x, const int32_t *topk_idx, const float *topk_w,
                                                   int64_t N, int32_t H, int32_t I, int32_t E, int32_t K,
                                                   int64_t total_pairs, const void *w1, const void *b1,
                                                   const void *w2, const void *b2, int32_t activation,
                                                   int32_t gate_up_layout, void *out, void *ws, size_t ws_bytes,
                                                   moe_stream_t stream) {
    int st = check_sizes(N, E, K, total_pairs);
    if (st) return st;
    if (!aligned(topk_idx, 4) || !aligned(topk_w, 4)) return MOE_ERR_ARG;
    return forward_impl(x, routing_topk32(topk_idx, topk_w, N, K, total_pairs), H, I, E, w1, b1, w2, b2,
                        activation, gate_up_layout, out, nullptr, ws, ws_bytes,
                        reinterpret_cast<cudaStream_t>(stream), nullptr, true);
}

extern "C" MOE_API int moe_nonexpand_backward(const void *dout, const void *x, const int32_t *topk_idx,
                                              const float *topk_w, int64_t N, int32_t H, int32_t I, int32_t E,
                                              int32_t K, int64_t total_pairs, const void *w1, const void *w2,
                                              int32_t activation, int32_t gate_up_layout, void *dx, void *dw1,
                                              void *db1, void *dw2, void *db2, float *dtopk_w, void *ws,
                                              size_t ws_bytes, moe_stream_t stream) {
    int st = check_sizes(N, E, K, total_pairs);
    if (st) return st;
    if ((N > 0 && (!topk_idx || !topk_w)) || !aligned(topk_idx, 4) || !aligned(topk_w, 4)) return MOE_ERR_ARG;
    return backward_impl(dout, x, routing_topk32(topk_idx, topk_w, N, K, total_pairs), H, I, E, w1, w2, activation,
                         gate_up_layout, dx, dw1, db1, dw2, db2, dtopk_w, ws, ws_bytes,
                         reinterpret_cast<cudaStream_t>(stream), nullptr);
}

extern "C" MOE_API int moe_nonexpand_backward_timed(const void *dout, const void *x, const int32_t *topk_idx,
                                                    const float *topk_w, int64_t N, int32_t H, int32_t I,
                                                    int32_t E, int32_t K, int64_t total_pairs, const void *w1,
                                                    const void *w2, int32_t activation, int32_t gate_up_layout,
                                                    void *dx, void *dw1, void *db1, void *dw2, void *db2,
                                                    float *dtopk_w, void *ws, size_t ws_bytes, moe_stream_t stream,
                                                    const moe_event_t *stage_events) {
    if (!stage_events) return MOE_ERR_ARG;
    int st = check_sizes(N, E, K, total_pairs);
    if (st) return st;
    if ((N > 0 && (!topk_idx || !topk_w)) || !aligned(topk_idx, 4) || !aligned(topk_w, 4)) return MOE_ERR_ARG;
    return backward_impl(dout, x, routing_topk32(topk_idx, topk_w, N, K, total_pairs), H, I, E, w1, w2, activation,
                         gate_up_layout, dx, dw1, db1, dw2, db2, dtopk_w, ws, ws_bytes,
                         reinterpret_cast<cudaStream_t>(stream), stage_events);
}

extern "C" MOE_API size_t moe_nonexpand_routed_train_workspace_bytes(const moe_routing_t *routing, int32_t H,
                                                                     int32_t I, int32_t E) {
    Routing r;
    if (routing_from_desc(routing, E, &r)) return 0;
    if (H <= 0 || I <= 0) return 0;
    const moe_ws_layout_t l = compute_layout_nk(r.N, H, I, E, r.NK, r.p_cap);
    if (check_dense(l.p_cap, H, I, E)) return 0;
    return l.train_total;
}

extern "C" MOE_API int moe_nonexpand_routed_forward_train(const void *x, const moe_routing_t *routing, int32_t H,
                                                          int32_t I, int32_t E, const void *w1, const void *b1,
                                                          const void *w2, const void *b2, int32_t activation,
                                                          int32_t gate_up_layout, void *out, void *ws,
                                                          size_t ws_bytes, moe_stream_t stream) {
    Routing r;
    const int st = routing_from_desc(routing, E, &r);
    if (st) return st;
    return forward_impl(x, r, H, I, E, w1, b1, w2, b2, activation, gate_up_layout, out, nullptr, ws, ws_bytes,
                        reinterpret_cast<cudaStream_t>(stream), nullptr, true);
}

extern "C" MOE_API int moe_nonexpand_routed_backward(const void *dout, const void *x, const moe_routing_t *routing,
                                                     int32_t H, int32_t I, int32_t E, const void *w1,
                                                     const void *w2, int32_t activation, int32_t gate_up_layout,
                                                     void *dx, void *dw1, void *db1, void *dw2, void *db2,
                                                     float *dweights, void *ws, size_t ws_bytes,
                                                     moe_stream_t stream) {
    Routing r;
    const int st = routing_from_desc(routing, E, &r);
    if (st) return st;
    return backward_impl(dout, x, r, H, I, E, w1, w2, activation, gate_up_layout, dx, dw1, db1, dw2, db2, dweights,
                         ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream), nullptr);
}

extern "C" MOE_API size_t moe_nonexpand_workspace_bytes(int64_t N, int32_t H, int32_t I, int32_t E, int32_t K,
                                             int64_t total_pairs) {
    if (check_sizes(N, E, K, total_pairs)) return 0;
    if (H < 0 || I < 0) return 0;
    const moe_ws_layout_t l = compute_layout(N, H, I, E, K, total_pairs);
    if (H > 0 || I > 0) {
        if (check_dense(l.p_cap, H, I, E)) return 0;
    }
    return l.total;
}

extern "C" MOE_API int moe_nonexpand_workspace_layout(int64_t N, int32_t H, int32_t I, int32_t E, int32_t K,
                                           int64_t total_pairs, moe_ws_layout_t *layout_out) {
    if (!layout_out) return MOE_ERR_ARG;
    int st = check_sizes(N, E, K, total_pairs);
    if (st) return st;
    if (H < 0 || I < 0) return MOE_ERR_SHAPE;
    *layout_out = compute_layout(N, H, I, E, K, total_pairs);
    return MOE_OK;
}

extern "C" MOE_API int moe_nonexpand_metadata(const int32_t *topk_idx, const float *topk_w, int64_t N, int32_t K,
                                   int32_t E, int64_t total_pairs, const moe_meta_t *meta, void *ws,
                                   size_t ws_bytes, moe_stream_t stream) {
    int st = check_sizes(N, E, K, total_pairs);
    if (st) return st;
    if ((N > 0 && (!topk_idx || !topk_w)) || !meta || !meta->token_offset || !meta->expert_frequency ||
        !meta->expert_frequency_offset)
        return MOE_ERR_ARG;
    if (N > 0 && !meta_complete(meta)) return MOE_ERR_ARG;
    if (!aligned(topk_idx, 4) || !aligned(topk_w, 4)) return MOE_ERR_ARG;
    const moe_ws_layout_t l = compute_layout(N, 0, 0, E, K, total_pairs);
    if (!ws || !aligned(ws, kAlign) || ws_bytes < l.total) return MOE_ERR_WS;
    DeviceInfo dev;
    st = device_info(&dev);
    if (st) return st;
    const MetaArgs ma =
        meta_args(routing_topk32(topk_idx, topk_w, N, K, total_pairs), E, l, static_cast<uint8_t *>(ws), *meta);
    return launch_meta(ma, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" MOE_API size_t moe_nonexpand_routed_workspace_bytes(const moe_routing_t *routing, int32_t H, int32_t I,
                                                               int32_t E) {
    Routing r;
    if (routing_from_desc(routing, E, &r)) return 0;
    if (H < 0 || I < 0) return 0;
    const moe_ws_layout_t l = compute_layout_nk(r.N, H, I, E, r.NK, r.p_cap);
    if ((H > 0 || I > 0) && check_dense(l.p_cap, H, I, E)) return 0;
    return l.total;
}

extern "C" MOE_API int moe_nonexpand_routed_metadata(const moe_routing_t *routing, int32_t E,
                                                     const moe_meta_t *meta, void *ws, size_t ws_bytes,
                                                     moe_stream_t stream) {
    Routing r;
    int st = routing_from_desc(routing, E, &r);
    if (st) return st;
    if (!meta || !meta->token_offset || !meta->expert_frequency || !meta->expert_frequency_offset)
        return MOE_ERR_ARG;
    if (r.NK > 0 && !meta_complete(meta)) return MOE_ERR_ARG;
    const moe_ws_layout_t l = compute_layout_nk(r.N, 0, 0, E, r.NK, r.p_cap);
    if (!ws || !aligned(ws, kAlign) || ws_bytes < l.total) return MOE_ERR_WS;
    DeviceInfo dev;
    st = device_info(&dev);
    if (st) return st;
    const MetaArgs ma = meta_args(r, E, l, static_cast<uint8_t *>(ws), *meta);
    return launch_meta(ma, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" MOE_API int moe_nonexpand_routed_forward(const void *x, const moe_routing_t *routing, int32_t H,
                                                    int32_t I, int32_t E, const void *w1, const void *b1,
                                                    const void *w2, const void *b2, int32_t activation,
                                                    int32_t gate_up_layout, void *out, const moe_meta_t *meta_out,
                                                    void *ws, size_t ws_bytes, moe_stream_t stream) {
    Routing r;
    const int st = routing_from_desc(routing, E, &r);
    if (st) return st;
    return forward_impl(x, r, H, I, E, w1, b1, w2, b2, activation, gate_up_layout, out, meta_out, ws, ws_bytes,
                        reinterpret_cast<cudaStream_t>(stream), nullptr);
}

extern "C" MOE_API int moe_nonexpand_forward(const void *x, const int32_t *topk_idx, const float *topk_w, int64_t N,
                                  int32_t H, int32_t I, int32_t E, int32_t K, int64_t total_pairs,
                                  const void *w1, const void *b1, const void *w2, const void *b2,
                                  int32_t activation, int32_t gate_up_layout, void *out,
                                  const moe_meta_t *meta_out, void *ws, size_t ws_bytes, moe_stream_t stream) {
    int st = check_sizes(N, E, K, total_pairs);
    if (st) return st;
    if (!aligned(topk_idx, 4) || !aligned(topk_w, 4)) return MOE_ERR_ARG;
    return forward_impl(x, routing_topk32(topk_idx, topk_w, N, K, total_pairs), H, I, E, w1, b1, w2, b2,
                        activation, gate_up_layout, out, meta_out, ws, ws_bytes,
                        reinterpret_cast<cudaStream_t>(stream), nullptr);
}

extern "C" MOE_API int moe_nonexpand_forward_timed(const void *x, const int32_t *topk_idx, const float *topk_w, int64_t N,
                                        int32_t H, int32_t I, int32_t E, int32_t K, int64_t total_pairs,
                                        const void *w1, const void *b1, const void *w2, const void *b2,
                                        int32_t activation, int32_t gate_up_layout, void *out,
                                        const moe_meta_t *meta_out, void *ws, size_t ws_bytes,
                                        moe_stream_t stream, const moe_event_t *stage_events) {
    if (!stage_events) return MOE_ERR_ARG;
    for (int i = 0; i < 5; ++i)
        if (!stage_events[i]) return MOE_ERR_ARG;
    int st = check_sizes(N, E, K, total_pairs);
    if (st) return st;
    if (!aligned(topk_idx, 4) || !aligned(topk_w, 4)) return MOE_ERR_ARG;
    return forward_impl(x, routing_topk32(topk_idx, topk_w, N, K, total_pairs), H, I, E, w1, b1, w2, b2,
                        activation, gate_up_layout, out, meta_out, ws, ws_bytes,
                        reinterpret_cast<cudaStream_t>(stream), stage_events);
}

extern "C" MOE_API int moe_nonexpand_combine(const void *y, const moe_meta_t *meta, int64_t N, int32_t H, void *out,
                                  moe_stream_t stream) {
    if (!y || !meta || !meta->token_offset || !meta->s_reverse_scatter_idx || !meta->scores || !out)
        return MOE_ERR_ARG;
    if (N < 0) return MOE_ERR_ARG;
    if (H <= 0 || (H % 64) != 0) return MOE_ERR_SHAPE;
    if (!aligned(y, 16) || !aligned(out, 16)) return MOE_ERR_ARG;
    DeviceInfo dev;
    int st = device_info(&dev);
    if (st) return st;
    return launch_combine(static_cast<const __nv_bfloat16 *>(y), nullptr, meta->token_offset, meta->s_reverse_scatter_idx,
                          meta->scores, N, H, static_cast<__nv_bfloat16 *>(out), nullptr, dev.sms,
                          reinterpret_cast<cudaStream_t>(stream), false) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

extern "C" MOE_API int moe_router_topk(const void *logits, int32_t logits_dtype, int64_t N, int32_t E, int32_t K,
                                       int32_t mode, int32_t *topk_idx, float *topk_w, moe_stream_t stream) {
    if (N < 0 || E < 1 || E > kMaxExperts || K < 1 || K > 32 || K > E) return MOE_ERR_ARG;
    if (N * (int64_t)E >= ((int64_t)1 << 40)) return MOE_ERR_ARG;
    if (logits_dtype != MOE_DTYPE_F32 && logits_dtype != MOE_DTYPE_BF16) return MOE_ERR_ARG;
    if (mode != MOE_ROUTER_SOFTMAX_TOPK && mode != MOE_ROUTER_TOPK_SOFTMAX && mode != MOE_ROUTER_TOPK_SOFTMAX_RENORM)
        return MOE_ERR_ARG;
    if (N > 0 && (!logits || !topk_idx || !topk_w)) return MOE_ERR_ARG;
    if (!aligned(logits, logits_dtype == MOE_DTYPE_F32 ? 4 : 2) || !aligned(topk_idx, 4) || !aligned(topk_w, 4))
        return MOE_ERR_ARG;
    DeviceInfo dev;
    const int st = device_info(&dev);
    if (st) return st;
    return launch_router(logits, logits_dtype == MOE_DTYPE_BF16, N, E, K, mode, topk_idx, topk_w, dev.sms,
                         reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

// ---- expert-parallel dispatch / combine (non-expand) ----------------------
extern "C" MOE_API int moe_ep_layout(const int32_t *topk_idx, int64_t T, int32_t K, int32_t R, int32_t E_local,
                                     int32_t *send_idx, int32_t *send_count, uint32_t *err_word,
                                     moe_stream_t stream) {
    if (T < 0 || K < 1 || K > 32 || R < 1 || R > MOE_EP_MAX_RANKS || E_local < 1) return MOE_ERR_ARG;
    if ((int64_t)R * E_local >= ((int64_t)1 << 31) || T * (int64_t)R >= ((int64_t)1 << 31) ||
        T * (int64_t)K >= ((int64_t)1 << 40))
        return MOE_ERR_ARG;
    if (!send_count || (T > 0 && (!topk_idx || !send_idx))) return MOE_ERR_ARG;
    if (!aligned(topk_idx, 4) || !aligned(send_idx, 4) || !aligned(send_count, 4) || !aligned(err_word, 4))
        return MOE_ERR_ARG;
    DeviceInfo dev;
    const int st = device_info(&dev);
    if (st) return st;
    return launch_ep_layout(topk_idx, T, K, R, E_local, send_idx, send_count, err_word,
                            reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

extern "C" MOE_API int moe_ep_dispatch(const void *x, const int32_t *topk_idx, const float *topk_w,
                                       const int32_t *send_idx, int64_t T, int32_t H, int32_t K, int32_t R,
                                       int32_t E_local, const moe_ep_peers_t *peers, moe_stream_t stream) {
    if (T < 0 || H < 8 || H % 8 != 0 || K < 1 || K > 32 || R < 1 || R > MOE_EP_MAX_RANKS || E_local < 1 || !peers)
        return MOE_ERR_ARG;
    if ((int64_t)R * E_local >= ((int64_t)1 << 31) || T * (int64_t)R >= ((int64_t)1 << 31)) return MOE_ERR_ARG;
    if (T > 0 && (!x || !topk_idx || !topk_w || !send_idx)) return MOE_ERR_ARG;
    if (!aligned(x, 16) || !aligned(topk_idx, 4) || !aligned(topk_w, 4) || !aligned(send_idx, 4)) return MOE_ERR_ARG;
    if (!aligned(peers->err_word, 4)) return MOE_ERR_ARG;
    for (int d = 0; d < R; ++d) {
        if (!peers->recv_x[d] || !peers->recv_idx[d] || !peers->recv_w[d] || peers->row_off[d] < 0 ||
            peers->recv_rows[d] < 0)
            return MOE_ERR_ARG;
        if (!aligned(peers->recv_x[d], 16) || !aligned(peers->recv_idx[d], 4) || !aligned(peers->recv_w[d], 4))
            return MOE_ERR_ARG;
    }
    DeviceInfo dev;
    const int st = device_info(&dev);
    if (st) return st;
    return launch_ep_dispatch(x, topk_idx, topk_w, send_idx, T, H, K, R, E_local, *peers, dev.sms,
                              reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

extern "C" MOE_API int moe_ep_combine(const moe_ep_sources_t *src, const int32_t *send_idx, int64_t T, int32_t H,
                                      int32_t R, void *out, moe_stream_t stream) {
    if (T < 0 || H < 8 || H % 8 != 0 || R < 1 || R > MOE_EP_MAX_RANKS || !src) return MOE_ERR_ARG;
    if (T * (int64_t)R >= ((int64_t)1 << 31)) return MOE_ERR_ARG;
    if (T > 0 && (!send_idx || !out)) return MOE_ERR_ARG;
    if (!aligned(send_idx, 4) || !aligned(out, 16)) return MOE_ERR_ARG;
    for (int d = 0; d < R; ++d)
        if (!src->local_out[d] || !aligned(src->local_out[d], 16) || src->row_off[d] < 0 || src->rows[d] < 0)
            return MOE_ERR_ARG;
    if (!aligned(src->err_word, 4)) return MOE_ERR_ARG;
    DeviceInfo dev;
    const int st = device_info(&dev);
    if (st) return st;
    return launch_ep_combine(*src, send_idx, T, H, R, out, dev.sms, reinterpret_cast<cudaStream_t>(stream)) ==
                   cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

extern "C" MOE_API int moe_nonexpand_read_error(const void *ws, moe_stream_t stream, uint32_t *err_word) {
    if (!ws || !err_word) return MOE_ERR_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const WsHeader *hdr = static_cast<const WsHeader *>(ws);
    uint32_t v = 0;
    if (cudaMemcpyAsync(&v, &hdr->err, sizeof v, cudaMemcpyDeviceToHost, s) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
    *err_word = v;
    return MOE_OK;
}

extern "C" MOE_API const char *moe_nonexpand_strerror(int status) {
    switch (status) {
        case MOE_OK: return "ok";
        case MOE_ERR_ARG: return "invalid argument";
        case MOE_ERR_SHAPE: return "unsupported shape (H and I must be multiples of 64)";
        case MOE_ERR_WS: return "workspace missing, misaligned or too small";
        case MOE_ERR_CUDA: return "CUDA runtime or launch failure";
        case MOE_ERR_DEVICE: return "current device is not an sm_100 (B200-class) GPU";
        default: return "unknown status";
    }
}
