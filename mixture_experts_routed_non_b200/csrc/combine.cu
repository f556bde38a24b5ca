// Score-weighted combine back to token order (sonic-moe issue #68 dataflow:
// the local expert compute ends in local_out [N,H]; the qwen3_5.py commit
// notes, recipe step 5, scatter the expert rows back to their tokens).
//
// Instead of a scatter-add (index_add_, atomics, order not fixed), every
// output element is a gather: token t reads its pairs q in
// [token_offset[t], token_offset[t+1]) in q order (= slot order), fetches the
// expert row y[s_reverse_scatter_idx[q]] and accumulates scores[q] * row in
// fp32; the sum is rounded once to bf16.  The result is deterministic and
// independent of the launch shape.
//
// One thread owns 8 consecutive columns (one 16-byte vector) of one token;
// the K row reads of a token are issued four at a time before accumulating,
// to keep several HBM requests in flight per thread.
#include "common.cuh"

namespace moe {

namespace {

constexpr int kCombineThreads = 256;

__device__ __forceinline__ uint4 ld_stream_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
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

__global__ void __launch_bounds__(kCombineThreads) combine_kernel(
    const __nv_bfloat16 *__restrict__ y, const int32_t *__restrict__ token_offset,
    const int32_t *__restrict__ s_rev, const float *__restrict__ scores, int64_t N, int32_t H,
    __nv_bfloat16 *__restrict__ out, const WsHeader *hdr) {
    if (hdr && *(volatile const uint32_t *)&hdr->abort) return;
    const int chunks = H >> 3;
    const int64_t total = N * chunks;
    for (int64_t i = (int64_t)blockIdx.x * kCombineThreads + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * kCombineThreads) {
        const int64_t t = i / chunks;
        const int c = (int)(i - t * chunks);
        const int q0 = __ldg(token_offset + t);
        const int q1 = __ldg(token_offset + t + 1);
        const __nv_bfloat16 *ycol = y + (size_t)c * 8;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        int q = q0;
        for (; q + 4 <= q1; q += 4) {
            int p[4];
            float w[4];
            uint4 v[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                p[j] = __ldg(s_rev + q + j);
                w[j] = __ldg(scores + q + j);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) v[j] = ld_stream_v4(ycol + (size_t)p[j] * H);
#pragma unroll
            for (int j = 0; j < 4; ++j) fma8(acc, w[j], v[j]);
        }
        for (; q < q1; ++q) {
            const int p = __ldg(s_rev + q);
            const float w = __ldg(scores + q);
            fma8(acc, w, ld_stream_v4(ycol + (size_t)p * H));
        }
        uint4 o;
        o.x = pack_bf16x2(acc[0], acc[1]);
        o.y = pack_bf16x2(acc[2], acc[3]);
        o.z = pack_bf16x2(acc[4], acc[5]);
        o.w = pack_bf16x2(acc[6], acc[7]);
        *reinterpret_cast<uint4 *>(out + (size_t)t * H + (size_t)c * 8) = o;
    }
}

}  // namespace

cudaError_t launch_combine(const __nv_bfloat16 *y, const int32_t *token_offset, const int32_t *s_rev,
                           const float *scores, int64_t N, int32_t H, __nv_bfloat16 *out,
                           const WsHeader *hdr, int num_sms, cudaStream_t s) {
    const int64_t total = N * (H / 8);
    if (total == 0) return cudaSuccess;
    int64_t blocks = (total + kCombineThreads - 1) / kCombineThreads;
    const int64_t cap = (int64_t)num_sms * 8;
    if (blocks > cap) blocks = cap;
    combine_kernel<<<(unsigned)blocks, kCombineThreads, 0, s>>>(y, token_offset, s_rev, scores, N, H, out,
                                                                 hdr);
    return cudaGetLastError();
}

}  // namespace moe
