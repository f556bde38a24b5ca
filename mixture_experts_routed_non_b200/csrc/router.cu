// Router top-k on the device: router logits [N,E] -> topk_idx [N,K] and
// topk_w [N,K], the non-expand routing table the rest of the library takes.
//
// The sonic-moe write-up ("Three routing strategies, selected on the command
// line") names two conventions: TC top-K routing, softmax over the K largest
// logits, and Qwen3-style routing, the K largest of the softmax over all
// experts, optionally renormalised over the K chosen.  Softmax is strictly
// increasing, so both pick the same experts: the K largest logits.  The
// choice is made on the logits as given (fp32, or bf16 widened exactly), ties
// going to the lower expert id, and slot k holds the k-th largest.
//
// One warp owns a token.  Lane j holds the logits of experts j, j+32, ...
// (coalesced loads) in registers, as order-preserving integer keys.  K rounds
// of a warp arg-max pick the experts: each lane offers its best still-unchosen
// expert, two warp reductions (redux.sync) find the largest key and the lowest
// id holding it, and the owner marks it chosen.  With up to 8 keys a lane
// sorts them once, so its offer is its list's head and taking it is a shift.  The weights follow from
// expf of differences to the largest logit and warp sums (a fixed butterfly,
// so the result does not depend on the launch shape).  Reads N*E logits once
// and writes N*K pairs: an HBM-bound kernel.
#include "common.cuh"

namespace moe {

namespace {

constexpr int kRouterThreads = 256;
constexpr int kRouterWarps = kRouterThreads / 32;
constexpr unsigned kFull = 0xffffffffu;
constexpr int kNoExpert = 0x7fffffff;

template <bool kBf16>
__device__ __forceinline__ float load_logit(const void *p, size_t i) {
    float v;
    if (kBf16) {
        const unsigned short b = __ldg(static_cast<const unsigned short *>(p) + i);
        v = __uint_as_float((unsigned)b << 16);
    } else {
        v = __ldg(static_cast<const float *>(p) + i);
    }
    return v != v ? -INFINITY : v;  // NaN is read as -inf
}

// An order-preserving unsigned key of a float (larger float, larger key; NaN
// never reaches it).  Key 0 lies below every float's key.
__device__ __forceinline__ unsigned order_key(float v) {
    const unsigned u = __float_as_uint(v);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_value(unsigned k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    return v;
}

template <int kPer, bool kBf16>
__global__ void __launch_bounds__(kRouterThreads, 2) router_kernel(const void *__restrict__ logits, int64_t N, int E,
                                                                int K, int mode, int32_t *__restrict__ topk_idx,
                                                                float *__restrict__ topk_w) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * kRouterWarps;
    for (int64_t t = (int64_t)blockIdx.x * kRouterWarps + (threadIdx.x >> 5); t < N; t += warps) {
        const size_t row = (size_t)t * E;
        unsigned key[kPer];
        unsigned avail = 0;
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int e = lane + 32 * i;
            key[i] = e < E ? order_key(load_logit<kBf16>(logits, row + e)) : 0u;
            if (e < E) avail |= 1u << i;
        }
        const unsigned present = avail;
        unsigned kz[kPer];  // the keys as loaded, for the full softmax's sum
#pragma unroll
        for (int i = 0; i < kPer; ++i) kz[i] = key[i];
        unsigned sel_k = 0;  // lane r < K: the key and id of the r-th chosen expert
        int sel_e = 0;
        unsigned top_k = 0;
        if constexpr (kPer <= 8) {
            // sort the lane's keys, largest first (odd-even transposition: only
            // neighbours swap, on a strictly larger key, so equal keys keep
            // ascending ids); a round then reads each lane's head and the
            // owner of the winner shifts its list by one
            int id[kPer];
#pragma unroll
            for (int i = 0; i < kPer; ++i) id[i] = lane + 32 * i;
#pragma unroll
            for (int pass = 0; pass < kPer; ++pass)
#pragma unroll
                for (int i = pass & 1; i + 1 < kPer; i += 2)
                    if (key[i + 1] > key[i]) {
                        const unsigned tk = key[i];
                        key[i] = key[i + 1];
                        key[i + 1] = tk;
                        const int ti = id[i];
                        id[i] = id[i + 1];
                        id[i + 1] = ti;
                    }
            for (int r = 0; r < K; ++r) {
                const unsigned mk = __reduce_max_sync(kFull, key[0]);
                const int we = (int)__reduce_min_sync(kFull, key[0] == mk ? (unsigned)id[0] : 0xffffffffu);
                if (id[0] == we) {  // pop the head (padding enters as key 0)
#pragma unroll
                    for (int i = 0; i + 1 < kPer; ++i) {
                        key[i] = key[i + 1];
                        id[i] = id[i + 1];
                    }
                    key[kPer - 1] = 0u;
                }
                if (lane == r) {
                    sel_k = mk;
                    sel_e = we;
                }
                if (r == 0) top_k = mk;
            }
        } else {
            // many keys per lane: each round scans the lane's unchosen keys
            unsigned avail = present;
            for (int r = 0; r < K; ++r) {
                unsigned bk = 0;
                int be = kNoExpert;
#pragma unroll
                for (int i = 0; i < kPer; ++i)
                    if (((avail >> i) & 1u) && (be == kNoExpert || key[i] > bk)) {
                        bk = key[i];
                        be = lane + 32 * i;
                    }
                // the largest key, and the lowest id holding it
                const unsigned mk = __reduce_max_sync(kFull, be == kNoExpert ? 0u : bk);
                const int we =
                    (int)__reduce_min_sync(kFull, (be != kNoExpert && bk == mk) ? (unsigned)be : 0xffffffffu);
                if ((we & 31) == lane) avail &= ~(1u << (we >> 5));
                if (lane == r) {
                    sel_k = mk;
                    sel_e = we;
                }
                if (r == 0) top_k = mk;
            }
        }
        const float sel_v = key_value(sel_k);
        const float vmax = key_value(top_k);
        float w;
        if (mode == MOE_ROUTER_SOFTMAX_TOPK) {
            const float ex = lane < K ? expf(sel_v - vmax) : 0.f;
            w = ex / warp_sum(ex);
        } else {
            float z = 0.f;
#pragma unroll
            for (int i = 0; i < kPer; ++i)
                if ((present >> i) & 1u) z += expf(key_value(kz[i]) - vmax);
            const float p = expf(sel_v - vmax) / warp_sum(z);
            w = mode == MOE_ROUTER_TOPK_SOFTMAX_RENORM ? p / warp_sum(lane < K ? p : 0.f) : p;
        }
        if (lane < K) {
            topk_idx[(size_t)t * K + lane] = sel_e;
            topk_w[(size_t)t * K + lane] = w;
        }
    }
}

template <int kPer>
cudaError_t launch_router_per(const void *logits, bool bf16, int64_t N, int E, int K, int mode, int32_t *idx,
                              float *w, int num_sms, cudaStream_t s) {
    int64_t blocks = (N + kRouterWarps - 1) / kRouterWarps;
    const int64_t cap = (int64_t)num_sms * 8;
    if (blocks > cap) blocks = cap;
    if (bf16)
        router_kernel<kPer, true><<<(unsigned)blocks, kRouterThreads, 0, s>>>(logits, N, E, K, mode, idx, w);
    else
        router_kernel<kPer, false><<<(unsigned)blocks, kRouterThreads, 0, s>>>(logits, N, E, K, mode, idx, w);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_router(const void *logits, bool bf16, int64_t N, int E, int K, int mode, int32_t *idx, float *w,
                          int num_sms, cudaStream_t s) {
    if (N == 0) return cudaSuccess;
    const int per = (E + 31) / 32;
    if (per <= 1) return launch_router_per<1>(logits, bf16, N, E, K, mode, idx, w, num_sms, s);
    if (per <= 2) return launch_router_per<2>(logits, bf16, N, E, K, mode, idx, w, num_sms, s);
    if (per <= 4) return launch_router_per<4>(logits, bf16, N, E, K, mode, idx, w, num_sms, s);
    if (per <= 8) return launch_router_per<8>(logits, bf16, N, E, K, mode, idx, w, num_sms, s);
    if (per <= 16) return launch_router_per<16>(logits, bf16, N, E, K, mode, idx, w, num_sms, s);
    return launch_router_per<32>(logits, bf16, N, E, K, mode, idx, w, num_sms, s);
}

}  // namespace moe
