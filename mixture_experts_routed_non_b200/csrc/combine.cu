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
// independent of the launch shape.  The forward's rows are fp16 with a
// power-of-two exponent per 32-column block (the down GEMM's y and y_scale):
// each row element is fp16 * 2^e, exact in fp32, and the exponent folds into
// the pair's weight.  The backward's dx rows and the public combine's rows are
// plain bf16.
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
constexpr int kTokPerBlock = 32;
constexpr int kStagedPairs = 256;  // pair indices staged in shared memory per block (28 tokens of 8 pairs fit)

__device__ __forceinline__ uint4 ld_stream_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// acc += w * fp16 row, eight columns (w carries the block's 2^e)
__device__ __forceinline__ void fma8_f16(float (&acc)[8], float w, const uint4 &v) {
    const float2 a = f16x2_to_f32(v.x), b = f16x2_to_f32(v.y), c = f16x2_to_f32(v.z), d = f16x2_to_f32(v.w);
    acc[0] = fmaf(w, a.x, acc[0]);
    acc[1] = fmaf(w, a.y, acc[1]);
    acc[2] = fmaf(w, b.x, acc[2]);
    acc[3] = fmaf(w, b.y, acc[3]);
    acc[4] = fmaf(w, c.x, acc[4]);
    acc[5] = fmaf(w, c.y, acc[5]);
    acc[6] = fmaf(w, d.x, acc[6]);
    acc[7] = fmaf(w, d.y, acc[7]);
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
template <bool kStaged, bool kScaled>
__device__ __forceinline__ void combine_tokens(const uint16_t *__restrict__ y, const int8_t *__restrict__ y_scale,
                                               const int *pidx, const float *pw, const int *s_off, int qa, int np,
                                               int nt, int32_t H, __nv_bfloat16 *__restrict__ out_t0) {
    const int chunks = H >> 3;
    const int sld = H / kYBlock;  // exponents per row
    for (int c = threadIdx.x; c < chunks; c += kCombineThreads) {
        const uint16_t *ycol = y + (size_t)c * 8;
        const int8_t *scol = kScaled ? y_scale + (c >> 2) : nullptr;  // the chunk's 32-column block
        __nv_bfloat16 *ocol = out_t0 + (size_t)c * 8;
        // walk the block's pairs in batches of 8 rows in flight, across token
        // boundaries; each token's pairs are still summed in q order
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        int j = 0;                       // current token (block-local)
        int tok_end = s_off[1] - qa;     // its pairs end here
        for (int base = 0; base < np; base += 8) {
            uint4 v[8];
            int ex[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int q = base + u;
                const int row = q < np ? (kStaged ? pidx[q] : __ldg(pidx + q)) : 0;
                v[u] = q < np ? ld_stream_v4(ycol + (size_t)row * H) : make_uint4(0, 0, 0, 0);
                if (kScaled) ex[u] = q < np ? (int)__ldg(scol + (size_t)row * sld) : 0;
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
                if (kScaled) fma8_f16(acc, wq * exp2i(ex[u]), v[u]);
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

// Four blocks per SM; eight 16-byte row chunks in flight per thread.
template <bool kScaled>
__global__ void __launch_bounds__(kCombineThreads, 4) combine_kernel(
    const uint16_t *__restrict__ y, const int8_t *__restrict__ y_scale, const int32_t *__restrict__ token_offset,
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
            combine_tokens<true, kScaled>(y, y_scale, s_p, s_w, s_off, qa, np, nt, H, out_t0);
        } else {  // more pairs than the staging arrays hold (a pair list may give a token any number)
            combine_tokens<false, kScaled>(y, y_scale, s_rev + qa, scores ? scores + qa : nullptr, s_off, qa, np, nt,
                                           H, out_t0);
        }
        __syncthreads();  // shared indices are reused by the next group
    }
}

}  // namespace

cudaError_t launch_combine(const void *y, const int8_t *y_scale, const int32_t *token_offset, const int32_t *s_rev,
                           const float *scores, int64_t N, int32_t H, __nv_bfloat16 *out,
                           const WsHeader *hdr, int num_sms, cudaStream_t s, bool pdl) {
    if (N == 0) return cudaSuccess;
    // tokens per block: as many as fill every SM's four resident blocks once (one
    // wave, no partial last wave), at most kTokPerBlock
    const int64_t resident = (int64_t)num_sms * 4;
    int64_t tpb = (N + resident - 1) / resident;
    if (tpb < 1) tpb = 1;
    if (tpb > kTokPerBlock) tpb = kTokPerBlock;
    const int64_t groups = (N + tpb - 1) / tpb;
    int64_t blocks = groups;
    const int64_t cap = (int64_t)num_sms * 16;
    if (blocks > cap) blocks = cap;
    const uint16_t *rows = static_cast<const uint16_t *>(y);
    if (y_scale)
        return launch_maybe_pdl(combine_kernel<true>, dim3((unsigned)blocks), dim3(kCombineThreads), 0, s, pdl, rows,
                                y_scale, token_offset, s_rev, scores, N, H, out, hdr, (int)tpb);
    const int8_t *no_scale = nullptr;
    return launch_maybe_pdl(combine_kernel<false>, dim3((unsigned)blocks), dim3(kCombineThreads), 0, s, pdl, rows,
                            no_scale, token_offset, s_rev, scores, N, H, out, hdr, (int)tpb);
}

}  // namespace moe
