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
// Two kernels, one launch either way:
//
// router_top8_kernel (K <= 8, E <= 256, E % 4 == 0, aligned rows): eight
// threads own a token, each holding an eighth of its logits (16-byte chunks,
// chunk c to thread c % 8).  A logit becomes an integer key whose order is
// the logits' order with ties to the lower id: the order-preserving image of
// the float with its low bits replaced by (mask - id).  For bf16 the float's
// low 16 bits are zero, so the key is exact; for fp32 the id takes the low 5
// to 8 bits.  Each thread sorts its keys in groups of 8 (19
// compare-exchanges) and keeps the 8 largest: a group joins the list by one
// bitonic half-cleaner step and a re-sort of the list (12
// compare-exchanges), the discarded keys' maximum kept.  Three shuffle rounds
// merge the eight lists the same way, and thread j writes slot j.  An fp32
// result can differ from the exact one only where two keys that decide it
// share their high bits (adjacent chosen keys, or the K-th chosen and the
// best key left out); then the warp redoes its four tokens with exact 64-bit
// keys (the float's key above the id).
//
// router_kernel (every other shape): one warp owns a token.  Lane j holds the
// logits of experts j, j+32, ... as order-preserving keys; K rounds of a warp
// arg-max (two redux.sync) pick the experts, each lane's keys sorted once
// when it has at most 8.
//
// The weights follow from exponentials of differences to the largest logit
// and fixed-order sums (independent of the launch shape).  Both kernels read
// N*E logits once and write N*K pairs.
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
    return (v != v ? -INFINITY : v) + 0.f;  // NaN is read as -inf, -0 as +0
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

// ---- eight threads per token -----------------------------------------------

constexpr int kTopThreads = 128;  // 8 blocks per SM at <= 64 registers (E <= 128): 16384 tokens in one wave
constexpr int kTpt = 8;           // threads per token

__device__ __forceinline__ unsigned kmax(unsigned a, unsigned b) { return max(a, b); }
__device__ __forceinline__ unsigned kmin(unsigned a, unsigned b) { return min(a, b); }
__device__ __forceinline__ unsigned long long kmax(unsigned long long a, unsigned long long b) { return max(a, b); }
__device__ __forceinline__ unsigned long long kmin(unsigned long long a, unsigned long long b) { return min(a, b); }

// larger key to a, smaller to b
template <typename KT>
__device__ __forceinline__ void cx(KT &a, KT &b) {
    const KT hi = kmax(a, b), lo = kmin(a, b);
    a = hi;
    b = lo;
}

// Sorts 8 keys, largest first (19 compare-exchanges in 6 layers).
template <typename KT>
__device__ __forceinline__ void sort8(KT (&b)[8]) {
    cx(b[0], b[2]); cx(b[1], b[3]); cx(b[4], b[6]); cx(b[5], b[7]);
    cx(b[0], b[4]); cx(b[1], b[5]); cx(b[2], b[6]); cx(b[3], b[7]);
    cx(b[0], b[1]); cx(b[2], b[3]); cx(b[4], b[5]); cx(b[6], b[7]);
    cx(b[2], b[4]); cx(b[3], b[5]);
    cx(b[1], b[4]); cx(b[3], b[6]);
    cx(b[1], b[2]); cx(b[3], b[4]); cx(b[5], b[6]);
}

// Sorts 4 keys, largest first.
template <typename KT>
__device__ __forceinline__ void sort4(KT *b) {
    cx(b[0], b[1]); cx(b[2], b[3]); cx(b[0], b[2]); cx(b[1], b[3]); cx(b[1], b[2]);
}

// Sorts a bitonic sequence of 8 keys, largest first.
template <typename KT>
__device__ __forceinline__ void bitonic8(KT (&a)[8]) {
#pragma unroll
    for (int d = 4; d > 0; d >>= 1)
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if ((j & d) == 0) cx(a[j], a[j + d]);
}

// a (sorted, largest first) <- the 8 largest of a and b (sorted), sorted;
// rej <- the largest key seen that is not among them.
template <typename KT>
__device__ __forceinline__ void merge_top8(KT (&a)[8], const KT (&b)[8], KT &rej) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const KT o = b[7 - j];
        rej = kmax(rej, kmin(a[j], o));
        a[j] = kmax(a[j], o);
    }
    bitonic8(a);
}

template <typename KT>
__device__ __forceinline__ KT shfl_key(KT v, int m) {
    if constexpr (sizeof(KT) == 8) {
        const unsigned lo = __shfl_xor_sync(kFull, (unsigned)v, m);
        const unsigned hi = __shfl_xor_sync(kFull, (unsigned)(v >> 32), m);
        return ((KT)hi << 32) | lo;
    } else {
        return __shfl_xor_sync(kFull, v, m);
    }
}

// The key of logit v of expert e: 32-bit keys put (kMask - e) in the low bits
// (exact for bf16, kMask = 0xffff; the top bits of the float's key for fp32);
// 64-bit keys put the float's whole key above (0xffffffff - e).
template <typename KT, unsigned kMask>
__device__ __forceinline__ KT pack_key(float v, int e) {
    const unsigned k = order_key(v);
    if constexpr (sizeof(KT) == 8)
        return ((KT)k << 32) | (KT)(0xffffffffu - (unsigned)e);
    else
        return (k | kMask) - (unsigned)e;
}

template <typename KT, unsigned kMask>
__device__ __forceinline__ int key_expert(KT k) {
    if constexpr (sizeof(KT) == 8)
        return (int)(0xffffffffu - (unsigned)k);
    else
        return (int)(kMask - ((unsigned)k & kMask));
}

// The keys of chunk m (4 logits) of thread q; key 0 (below every logit's key)
// past the last expert.
template <typename KT, unsigned kMask>
__device__ __forceinline__ void chunk_keys(const float *x, int q, int m, int E, KT *b) {
    const int e0 = 4 * (q + kTpt * m);
#pragma unroll
    for (int i = 0; i < 4; ++i) b[i] = e0 < E ? pack_key<KT, kMask>(x[4 * m + i], e0 + i) : (KT)0;
}

// The top-8 keys of a token over its eight threads (all eight end with the
// same list, largest first), and the largest key left out.
template <typename KT, unsigned kMask, int kChunks>
__device__ __forceinline__ void top8_keys(const float (&x)[4 * kChunks], int q, int E, KT (&a)[8], KT &rej) {
    rej = 0;
    if constexpr (kChunks == 1) {
        chunk_keys<KT, kMask>(x, q, 0, E, a);
        sort4(a);
#pragma unroll
        for (int j = 4; j < 8; ++j) a[j] = 0;
    } else {
        chunk_keys<KT, kMask>(x, q, 0, E, a);
        chunk_keys<KT, kMask>(x, q, 1, E, a + 4);
        sort8(a);
#pragma unroll
        for (int m = 2; m < kChunks; m += 2) {
            KT b[8];
            chunk_keys<KT, kMask>(x, q, m, E, b);
            chunk_keys<KT, kMask>(x, q, m + 1, E, b + 4);
            sort8(b);
            merge_top8(a, b, rej);
        }
    }
#pragma unroll
    for (int s = 1; s < kTpt; s <<= 1) {
        KT o[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) o[j] = shfl_key(a[j], s);
        rej = kmax(rej, shfl_key(rej, s));
        merge_top8(a, o, rej);
    }
}

template <bool kBf16>
__device__ __forceinline__ void load_chunk(const void *logits, size_t i, float *v) {
    if (kBf16) {
        const uint2 r = __ldg(reinterpret_cast<const uint2 *>(static_cast<const unsigned short *>(logits) + i));
        v[0] = __uint_as_float(r.x << 16);
        v[1] = __uint_as_float(r.x & 0xffff0000u);
        v[2] = __uint_as_float(r.y << 16);
        v[3] = __uint_as_float(r.y & 0xffff0000u);
    } else {
        const float4 r = __ldg(reinterpret_cast<const float4 *>(static_cast<const float *>(logits) + i));
        v[0] = r.x;
        v[1] = r.y;
        v[2] = r.z;
        v[3] = r.w;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = fmaxf(v[i], -INFINITY) + 0.f;  // NaN is read as -inf, -0 as +0
}

template <int kChunks, bool kBf16>
__global__ void __launch_bounds__(kTopThreads, kChunks >= 8 ? 5 : 8) router_top8_kernel(const void *__restrict__ logits, int64_t N, int E,
                                                                 int K, int mode, int32_t *__restrict__ topk_idx,
                                                                 float *__restrict__ topk_w) {
    constexpr unsigned kMask = kBf16 ? 0xffffu : (unsigned)(4 * kTpt * kChunks - 1);
    const int q = threadIdx.x & (kTpt - 1);
    const int64_t groups = (int64_t)gridDim.x * (kTopThreads / kTpt);
    // the loop test is the warp's first token, so whole warps iterate alike
    for (int64_t t = ((int64_t)blockIdx.x * kTopThreads + threadIdx.x) / kTpt;
         t - ((threadIdx.x & 31) / kTpt) < N; t += groups) {
        const bool live = t < N;
        const size_t row = (size_t)(live ? t : 0) * E;
        float x[4 * kChunks];
#pragma unroll
        for (int m = 0; m < kChunks; ++m) {
            const int e0 = 4 * (q + kTpt * m);
            if (live && e0 < E) {
                load_chunk<kBf16>(logits, row + e0, &x[4 * m]);
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) x[4 * m + i] = -INFINITY;
            }
        }
        int id[8];
        {
            unsigned a[8], rej;
            top8_keys<unsigned, kMask, kChunks>(x, q, E, a, rej);
            bool redo = false;
            if constexpr (!kBf16) {
                // the fp32 keys decide alike with the exact ones unless two keys
                // that matter share their high bits
                unsigned last = a[7], next = rej;
#pragma unroll
                for (int j = 0; j < 7; ++j) {
                    if (j + 1 < K) redo |= (a[j] | kMask) == (a[j + 1] | kMask);
                    if (j + 1 == K) {
                        last = a[j];
                        next = a[j + 1];
                    }
                }
                redo |= (last | kMask) == (next | kMask);
            }
            if (__any_sync(kFull, redo)) {
                unsigned long long b[8], rb;
                top8_keys<unsigned long long, kMask, kChunks>(x, q, E, b, rb);
#pragma unroll
                for (int j = 0; j < 8; ++j) id[j] = key_expert<unsigned long long, kMask>(b[j]);
            } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) id[j] = key_expert<unsigned, kMask>(a[j]);
            }
        }
        // slot q of the token is this thread's (a select tree on q's bits)
        const bool b0 = q & 1, b1 = q & 2, b2 = q & 4;
        const int s01 = b0 ? id[1] : id[0], s23 = b0 ? id[3] : id[2];
        const int s45 = b0 ? id[5] : id[4], s67 = b0 ? id[7] : id[6];
        const int my = b2 ? (b1 ? s67 : s45) : (b1 ? s23 : s01);
        float vmax = -INFINITY, v = -INFINITY;
        if (live) {
            vmax = load_logit<kBf16>(logits, row + id[0]);
            if (q < K) v = load_logit<kBf16>(logits, row + my);
        }
        const float ex = q < K ? expf(v - vmax) : 0.f;
        float den;
        if (mode == MOE_ROUTER_TOPK_SOFTMAX) {
            // the full softmax's sum: fast exponentials of the differences to
            // the largest logit (non-positive), relative error a few 1e-6 each
            den = 0.f;
#pragma unroll
            for (int m = 0; m < kChunks; ++m)
                if (4 * (q + kTpt * m) < E) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) den += __expf(x[4 * m + i] - vmax);
                }
        } else {
            // softmax over the K chosen; renormalised top-k of the softmax is
            // the same ratio (the full sum cancels)
            den = ex;
        }
#pragma unroll
        for (int s = 1; s < kTpt; s <<= 1) den += __shfl_xor_sync(kFull, den, s);
        if (live && q < K) {
            topk_idx[(size_t)t * K + q] = my;
            topk_w[(size_t)t * K + q] = ex / den;
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

template <int kChunks>
cudaError_t launch_router_top8(const void *logits, bool bf16, int64_t N, int E, int K, int mode, int32_t *idx,
                               float *w, int num_sms, cudaStream_t s) {
    int64_t blocks = (N * kTpt + kTopThreads - 1) / kTopThreads;
    const int64_t cap = (int64_t)num_sms * 32;
    if (blocks > cap) blocks = cap;
    if (bf16)
        router_top8_kernel<kChunks, true><<<(unsigned)blocks, kTopThreads, 0, s>>>(logits, N, E, K, mode, idx, w);
    else
        router_top8_kernel<kChunks, false><<<(unsigned)blocks, kTopThreads, 0, s>>>(logits, N, E, K, mode, idx, w);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_router(const void *logits, bool bf16, int64_t N, int E, int K, int mode, int32_t *idx, float *w,
                          int num_sms, cudaStream_t s) {
    if (N == 0) return cudaSuccess;
    // eight threads per token: 16-byte fp32 (8-byte bf16) chunks need E % 4 == 0 and an aligned base
    const bool chunks_ok = E % 4 == 0 && reinterpret_cast<uintptr_t>(logits) % (bf16 ? 8 : 16) == 0;
    if (K <= 8 && E <= 256 && chunks_ok) {
        if (E <= 32) return launch_router_top8<1>(logits, bf16, N, E, K, mode, idx, w, num_sms, s);
        if (E <= 64) return launch_router_top8<2>(logits, bf16, N, E, K, mode, idx, w, num_sms, s);
        if (E <= 128) return launch_router_top8<4>(logits, bf16, N, E, K, mode, idx, w, num_sms, s);
        return launch_router_top8<8>(logits, bf16, N, E, K, mode, idx, w, num_sms, s);
    }
    const int per = (E + 31) / 32;
    if (per <= 1) return launch_router_per<1>(logits, bf16, N, E, K, mode, idx, w, num_sms, s);
    if (per <= 2) return launch_router_per<2>(logits, bf16, N, E, K, mode, idx, w, num_sms, s);
    if (per <= 4) return launch_router_per<4>(logits, bf16, N, E, K, mode, idx, w, num_sms, s);
    if (per <= 8) return launch_router_per<8>(logits, bf16, N, E, K, mode, idx, w, num_sms, s);
    if (per <= 16) return launch_router_per<16>(logits, bf16, N, E, K, mode, idx, w, num_sms, s);
    return launch_router_per<32>(logits, bf16, N, E, K, mode, idx, w, num_sms, s);
}

}  // namespace moe
