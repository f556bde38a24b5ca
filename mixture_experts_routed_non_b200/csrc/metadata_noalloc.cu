// moe_nonexpand_metadata_noalloc: the routing metadata for callers that
// cannot hand the library any device memory beyond their inputs and outputs.
//
// The metadata kernels need a little scratch (a 256-byte header, the per-tile
// histogram table [T,E], per-tile valid counts and error bits, and the GEMM
// tile table [E+1]).  moe_nonexpand_metadata takes it from a caller workspace;
// this entry point instead uses one fixed array in device memory that belongs
// to the library, so it calls no allocator at all.
#include <stddef.h>

#include <mutex>

#include "common.cuh"

namespace moe {
namespace {

// Largest scratch any supported size needs: the histogram table holds at most
// kMetaTableInts entries (131,072 bytes), plus the per-tile tables of at most
// 148 tiles, the tile table of E <= 1024 experts and the header, rounded up.
constexpr size_t kNoAllocScratchBytes = 160 * 1024;

// The scratch.  Every GPU that loads the library holds it until the process
// exits.  All calls share it and it keeps the last call's contents; the
// kernels write every byte of it they read, so nothing has to start at zero.
static __device__ __align__(256) unsigned char g_meta_scratch[kNoAllocScratchBytes];

size_t up256(size_t v) { return (v + 255) / 256 * 256; }

struct ScratchLayout {
    size_t header, hist, valid, err, gemm_tiles, total;
    int32_t tiles, tile_slots;
};

// The same tiling as the workspace path (meta_tiling).
ScratchLayout scratch_layout(int64_t NK, int32_t E) {
    ScratchLayout l;
    meta_tiling(NK, E, &l.tile_slots, &l.tiles);
    const size_t T = (size_t)l.tiles;
    size_t o = 0;
    l.header = o;
    o = up256(o + sizeof(WsHeader));
    l.hist = o;
    o = up256(o + T * meta_hist_ld(E) * 4);
    l.valid = o;
    o = up256(o + T * 4);
    l.err = o;
    o = up256(o + T * 4);
    l.gemm_tiles = o;
    o = up256(o + (size_t)(E + 1) * 4);
    l.total = o;
    return l;
}

// Device address of the scratch on the current device, looked up once per
// device (cudaGetSymbolAddress; the host-side name is only a stand-in).
int scratch_address(unsigned char **out) {
    static std::mutex mu;
    static unsigned char *addr[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    if (dev < 0 || dev >= 64) return MOE_ERR_DEVICE;
    std::lock_guard<std::mutex> g(mu);
    if (!addr[dev]) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return MOE_ERR_CUDA;
        if (major != 10 || minor != 0) return MOE_ERR_DEVICE;
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_meta_scratch) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
        addr[dev] = static_cast<unsigned char *>(p);
    }
    *out = addr[dev];
    return MOE_OK;
}

bool meta_fields_set(const moe_meta_t *m) {
    return m && m->expert_frequency && m->expert_frequency_offset && m->x_gather_idx && m->s_scatter_idx &&
           m->s_reverse_scatter_idx && m->token_offset && m->scores;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" MOE_API int moe_nonexpand_metadata_noalloc(const int32_t *topk_idx, const float *topk_w, int64_t N,
                                                      int32_t K, int32_t E, int64_t total_pairs,
                                                      const moe_meta_t *meta, moe_stream_t stream) {
    // the same argument checks as moe_nonexpand_metadata, before any CUDA call
    int st = check_routing_sizes(N, E, K, total_pairs);
    if (st != MOE_OK) return st;
    if (N > 0 && (!topk_idx || !topk_w || !meta_fields_set(meta))) return MOE_ERR_ARG;
    if (!meta || !meta->token_offset || !meta->expert_frequency || !meta->expert_frequency_offset)
        return MOE_ERR_ARG;
    if (!ptr_aligned(topk_idx, 4) || !ptr_aligned(topk_w, 4)) return MOE_ERR_ARG;
    const ScratchLayout l = scratch_layout(N * K, E);
    if (l.total > kNoAllocScratchBytes) return MOE_ERR_WS;  // beyond the fixed scratch
    unsigned char *s = nullptr;
    st = scratch_address(&s);
    if (st != MOE_OK) return st;
    MetaArgs a;
    a.topk_idx = topk_idx;
    a.topk_w = topk_w;
    a.token_idx = nullptr;
    a.pair_list = 0;
    a.idx64 = 0;
    a.NK = N * K;
    a.K = K;
    a.E = E;
    a.total_pairs = total_pairs;
    a.p_cap = total_pairs >= 0 ? total_pairs : N * K;
    a.tiles = l.tiles;
    a.tile_slots = l.tile_slots;
    a.hist_ld = meta_hist_ld(E);
    a.hdr = reinterpret_cast<WsHeader *>(s + l.header);
    a.tile_hist = reinterpret_cast<int32_t *>(s + l.hist);
    a.tile_valid = reinterpret_cast<int32_t *>(s + l.valid);
    a.tile_err = reinterpret_cast<int32_t *>(s + l.err);
    a.gemm_tile_off = reinterpret_cast<int32_t *>(s + l.gemm_tiles);
    a.meta = *meta;
    a.N = N;
    a.slot_pair = nullptr;
    return launch_meta(a, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" MOE_API int moe_nonexpand_metadata_noalloc_read_error(moe_stream_t stream, uint32_t *err_word) {
    if (!err_word) return MOE_ERR_ARG;
    unsigned char *s = nullptr;
    const int st = scratch_address(&s);  // also checks the device, like the first metadata call
    if (st != MOE_OK) return st;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    uint32_t v = 0;
    if (cudaMemcpyFromSymbolAsync(&v, g_meta_scratch, sizeof v, offsetof(WsHeader, err), cudaMemcpyDeviceToHost,
                                  cs) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(cs) != cudaSuccess) return MOE_ERR_CUDA;
    *err_word = v;
    return MOE_OK;
}
