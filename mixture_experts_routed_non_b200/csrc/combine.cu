// Score-weighted combine back to token order (with null scores every weight
// is 1: the backward sums a token's dx rows the same way) (sonic-moe issue #68 dataflow:
// the local expert compute ends in local_out [N,H]; the qwen3_5.py commit
// notes, recipe step 5, scatter the expert rows back to their tokens).
//
// Instead of a scatter-add (index_add_, atomics, order not fixed), every
// output element is a gather: token t reads its pairs q in
// [token_offset[t], token_offset[t+1]) in q order (= slot order), fetches the
// expert row y[s_reverse_scatter_idx[q]] and accumulates scores[q] * row in
// fp32; the sum is rounded once to bf16.  The result is deterministic and
// independent of the launch shape.  With a residual array y_lo (the down
// GEMM's e5m2 rounding residuals) each row element is y + y_lo, exact in fp32.
//
// A block owns up to kTokPerBlock consecutive tokens.  Their token offsets and
// the row index and score of every one of their pairs (a contiguous q range)
// are loaded into shared memory once, with coalesced loads (a block whose
// tokens have more pairs than the staging arrays hold -- possible for a pair
// list, which bounds no token's pair count -- reads them from global memory
// instead); then each thread
// owns 16-byte column chunks and walks the block's pairs in batches of eight
// rows whose loads are all issued before any is accumulated -- across token
// boundaries, so the loads in flight do not depend on how many pairs each
// token has -- and no per-element index chain remains.
#include "common.cuh"

namespace moe {

namespace {

constexpr int kCombineThreads = 256;
constexpr int kTokPerBlock = 8;
constexpr int kStagedPairs = kTokPerBlock * 32;  // pair indices staged in shared memory per block

__device__ __forceinline__ uint4 ld_stream_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint2 ld_stream_v2(const void *p) {
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}

// acc += w * (bf16 row + e5m2 residual), eight columns
__device__ __forceinline__ void fma8_lo(float (&acc)[8], float w, const uint4 &v, const uint2 &r) {
    const float2 r0 = e5m2x2_to_f32(r.x, 0x1404u), r1 = e5m2x2_to_f32(r.x, 0x3424u);
    const float2 r2 = e5m2x2_to_f32(r.y, 0x1404u), r3 = e5m2x2_to_f32(r.y, 0x3424u);
    acc[0] = fmaf(w, bf16lo(v.x) + r0.x, acc[0]);
    acc[1] = fmaf(w, bf16hi(v.x) + r0.y, acc[1]);
    acc[2] = fmaf(w, bf16lo(v.y) + r1.x, acc[2]);
    acc[3] = fmaf(w, bf16hi(v.y) + r1.y, acc[3]);
    acc[4] = fmaf(w, bf16lo(v.z) + r2.x, acc[4]);
    acc[5] = fmaf(w, bf16hi(v.z) + r2.y, acc[5]);
    acc[6] = fmaf(w, bf16lo(v.w) + r3.x, acc[6]);
    acc[7] = fmaf(w, bf16hi(v.w) + r3.y, acc[7]);
}

__device__ __forceinline__ void fma8(float (&acc)[8], float w, const uint4 &v) {
    acc[0] = fmaf(w, bf16lo(v.x), acc[0]);
    acc[1] = fmaf(w, bf16hi(v.x), acc[1]);
    acc[2] = fmaf(w, bf16lo(v.y), acc[2]);
    acc[3] = fmaf(w, bf16hi(v.y), acc[3]);
    acc[4] = fmaf(w, bf16lo(v.z), acc[4]);
    acc[5] = fmaf(w, bf16hi(v.z), acc[5]);
    acc[6] = fmaf(w, bf16lo(v.w), acc[6]);
    acc[7] = fmaf(w, bf16hi(v.w), acc[7]);
}

__device__ __forceinline__ uint4 pack8(const float (&acc)[8]) {
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    return o;
}

// One block's tokens [t0, t0+nt): their pairs are q in [qa, qa+np) with
// token-local ends s_off[j+1]-qa.  pidx/pw are the pairs' row indices and
// scores: in shared memory when staged, else read from global memory.
template <bool kStaged, bool kLo>
__device__ __forceinline__ void combine_tokens(const __nv_bfloat16 *__restrict__ y, const uint8_t *__restrict__ y_lo,
                                               const int *pidx, const float *pw, const int *s_off, int qa, int np,
                                               int nt, int32_t H, __nv_bfloat16 *__restrict__ out_t0) {
    const int chunks = H >> 3;
    for (int c = threadIdx.x; c < chunks; c += kCombineThreads) {
        const __nv_bfloat16 *ycol = y + (size_t)c * 8;
        const uint8_t *lcol = kLo ? y_lo + (size_t)c * 8 : nullptr;
        __nv_bfloat16 *ocol = out_t0 + (size_t)c * 8;
        // walk the block's pairs in batches of 8 rows in flight, across token
        // boundaries; each token's pairs are still summed in q order
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        int j = 0;                       // current token (block-local)
        int tok_end = s_off[1] - qa;     // its pairs end here
        for (int base = 0; base < np; base += 8) {
            uint4 v[8];
            uint2 r[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int q = base + u;
                const int row = q < np ? (kStaged ? pidx[q] : __ldg(pidx + q)) : 0;
                v[u] = q < np ? ld_stream_v4(ycol + (size_t)row * H) : make_uint4(0, 0, 0, 0);
                if (kLo) r[u] = q < np ? ld_stream_v2(lcol + (size_t)row * H) : make_uint2(0, 0);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int q = base + u;
                if (q >= np) break;
                while (q >= tok_end) {  // finish token j (and any token without pairs)
                    *reinterpret_cast<uint4 *>(ocol + (size_t)j * H) = pack8(acc);
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
                    ++j;
                    tok_end = s_off[j + 1] - qa;
                }
                const float wq = kStaged ? pw[q] : (pw ? __ldg(pw + q) : 1.f);
                if (kLo) fma8_lo(acc, wq, v[u], r[u]);
                else fma8(acc, wq, v[u]);
            }
        }
        for (; j < nt; ++j) {  // the last token with pairs, then trailing tokens without
            *reinterpret_cast<uint4 *>(ocol + (size_t)j * H) = pack8(acc);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = 0.f;
        }
    }
}

// Blocks per SM: 4, or 3 with the residual rows (their registers; 8 rows of
// 24 bytes in flight per thread still cover the memory latency).
template <bool kLo>
__global__ void __launch_bounds__(kCombineThreads, kLo ? 3 : 4) combine_kernel(
    const __nv_bfloat16 *__restrict__ y, const uint8_t *__restrict__ y_lo, const int32_t *__restrict__ token_offset,
    const int32_t *__restrict__ s_rev, const float *__restrict__ scores, int64_t N, int32_t H,
    __nv_bfloat16 *__restrict__ out, const WsHeader *hdr, int tok_per_block) {
    __shared__ int s_off[kTokPerBlock + 1];
    __shared__ int s_p[kStagedPairs];
    __shared__ float s_w[kStagedPairs];
    pdl_wait();  // launched as a programmatic dependent: y is the kernel before's
    if (hdr && *(volatile const uint32_t *)&hdr->abort) return;
    const int64_t n_groups = (N + tok_per_block - 1) / tok_per_block;
    for (int64_t grp = blockIdx.x; grp < n_groups; grp += gridDim.x) {
        const int64_t t0 = grp * tok_per_block;
        const int nt = (int)min((int64_t)tok_per_block, N - t0);
        if (threadIdx.x <= nt) s_off[threadIdx.x] = __ldg(token_offset + t0 + threadIdx.x);
        __syncthreads();
        const int qa = s_off[0];
        const int np = s_off[nt] - qa;  // pairs of the block's tokens, a contiguous q range
        __nv_bfloat16 *out_t0 = out + (size_t)t0 * H;
        if (np <= kStagedPairs) {
            for (int i = threadIdx.x; i < np; i += kCombineThreads) {
                s_p[i] = __ldg(s_rev + qa + i);
                s_w[i] = scores ? __ldg(scores + qa + i) : 1.f;
            }
            __syncthreads();
            combine_tokens<true, kLo>(y, y_lo, s_p, s_w, s_off, qa, np, nt, H, out_t0);
        } else {  // more pairs than the staging arrays hold (a pair list may give a token any number)
            combine_tokens<false, kLo>(y, y_lo, s_rev + qa, scores ? scores + qa : nullptr, s_off, qa, np, nt, H,
                                       out_t0);
        }
        __syncthreads();  // shared indices are reused by the next group
    }
}

}  // namespace

cudaError_t launch_combine(const __nv_bfloat16 *y, const uint8_t *y_lo, const int32_t *token_offset, const int32_t *s_rev,
                           const float *scores, int64_t N, int32_t H, __nv_bfloat16 *out,
                           const WsHeader *hdr, int num_sms, cudaStream_t s, bool pdl) {
    if (N == 0) return cudaSuccess;
    // tokens per block: up to kTokPerBlock, fewer when that would leave SMs idle
    const int64_t chunks = H / 8;
    const int per_sm = y_lo ? 3 : 4;
    int64_t tpb = (N * chunks) / ((int64_t)num_sms * per_sm * kCombineThreads);
    if (tpb < 1) tpb = 1;
    if (tpb > kTokPerBlock) tpb = kTokPerBlock;
    const int64_t groups = (N + tpb - 1) / tpb;
    int64_t blocks = groups;
    const int64_t cap = (int64_t)num_sms * 16;
    if (blocks > cap) blocks = cap;
    const uint8_t *no_lo = nullptr;
    if (y_lo)
        return launch_maybe_pdl(combine_kernel<true>, dim3((unsigned)blocks), dim3(kCombineThreads), 0, s, pdl, y,
                                y_lo, token_offset, s_rev, scores, N, H, out, hdr, (int)tpb);
    return launch_maybe_pdl(combine_kernel<false>, dim3((unsigned)blocks), dim3(kCombineThreads), 0, s, pdl, y, no_lo,
                            token_offset, s_rev, scores, N, H, out, hdr, (int)tpb);
}

}  // namespace moe
