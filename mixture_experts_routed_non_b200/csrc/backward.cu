// Memory-bound steps of the backward (the GEMMs are in
// grouped_gemm_bwd_sm100.cu; the pages leave the backward open, so these are
// the chain rule of the forward):
//
//   prep      per token t and each of its pairs q (sorted position p):
//             ds_q = <dout_t, y_p>, the score's gradient (y_p as the forward
//             stored it, fp16 times 2^e per 32 columns; fp32, summed in a
//             fixed order), and dy_p = s_q dout_t (bf16 [P_cap,H]); ds is then
//             scattered to the routing slot each pair came from through the
//             slot -> pair index the training forward's metadata recorded (0 at
//             slots that are no pair) -- sonic-moe issue #68 asks for the
//             scores' gradient back in the routing layout.
//   bias      db[e,c] = sum of the segment's rows of dy (db2) or dz (db1), in
//             row order, fp32, rounded once to bf16.
//   gather    xs[p,:] = x[x_gather_idx[p],:], so the dW1 GEMM reads its A
//             operand with whole-stage TMA boxes instead of per-row copies.
#include "common.cuh"

namespace moe {

namespace {

constexpr int kPrepThreads = 256;
constexpr int kPrepWarps = kPrepThreads / 32;
constexpr int kMaxSlots = 32;

// eight bf16 dout values . eight fp16 y values (the row's 2^e applied by the caller)
__device__ __forceinline__ float dot8_f16(const uint4 &d, const uint4 &v) {
    const float2 a = f16x2_to_f32(v.x), b = f16x2_to_f32(v.y), c = f16x2_to_f32(v.z), e = f16x2_to_f32(v.w);
    return bf16lo(d.x) * a.x + bf16hi(d.x) * a.y + bf16lo(d.y) * b.x + bf16hi(d.y) * b.y + bf16lo(d.z) * c.x +
           bf16hi(d.z) * c.y + bf16lo(d.w) * e.x + bf16hi(d.w) * e.y;
}

__device__ __forceinline__ uint4 scale8(const uint4 &v, float s) {
    return make_uint4(pack_bf16x2(s * bf16lo(v.x), s * bf16hi(v.x)), pack_bf16x2(s * bf16lo(v.y), s * bf16hi(v.y)),
                      pack_bf16x2(s * bf16lo(v.z), s * bf16hi(v.z)), pack_bf16x2(s * bf16lo(v.w), s * bf16hi(v.w)));
}

// One block per token (grid-stride).  Each thread owns 16-byte column chunks
// of the row; for up to 32 pairs at a time it accumulates its share of each
// dot product, then the block reduces those partials at once (warp
// butterfly, then warps in order).  A pair list may give a token any number
// of pairs, hence the batches of 32.
__global__ void __launch_bounds__(kPrepThreads, 4) bwd_prep_kernel(
    const __nv_bfloat16 *__restrict__ dout, const uint16_t *__restrict__ y, const int8_t *__restrict__ y_scale,
    const int32_t *__restrict__ token_offset, const int32_t *__restrict__ s_rev, const float *__restrict__ scores,
    int64_t N, int32_t H, __nv_bfloat16 *__restrict__ dy, float *__restrict__ ds, const WsHeader *hdr) {
    __shared__ float part[kPrepWarps][kMaxSlots];
    if (hdr && *(volatile const uint32_t *)&hdr->abort) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int chunks = H >> 3;
    for (int64_t t = blockIdx.x; t < N; t += gridDim.x) {
        const int q0 = __ldg(token_offset + t), q1 = __ldg(token_offset + t + 1);
        const __nv_bfloat16 *drow = dout + (size_t)t * H;
        for (int qb = q0; qb < q1; qb += kMaxSlots) {
            const int np = min(kMaxSlots, q1 - qb);
            float acc[kMaxSlots];
#pragma unroll
            for (int j = 0; j < kMaxSlots; ++j) acc[j] = 0.f;
            for (int c = threadIdx.x; c < chunks; c += kPrepThreads) {
                const uint4 d = __ldg(reinterpret_cast<const uint4 *>(drow) + c);
#pragma unroll
                for (int j = 0; j < kMaxSlots; ++j) {
                    if (j >= np) break;
                    const int p = __ldg(s_rev + qb + j);
                    const uint4 v = __ldg(reinterpret_cast<const uint4 *>(y + (size_t)p * H) + c);
                    acc[j] += dot8_f16(d, v) * exp2i(__ldg(y_scale + (size_t)p * (H / kYBlock) + (c >> 2)));
                    reinterpret_cast<uint4 *>(dy + (size_t)p * H)[c] = scale8(d, __ldg(scores + qb + j));
                }
            }
#pragma unroll
            for (int j = 0; j < kMaxSlots; ++j) {
                if (j >= np) break;
                float v = acc[j];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (lane == 0) part[warp][j] = v;
            }
            __syncthreads();
            if (threadIdx.x < np) {
                float v = 0.f;
#pragma unroll
                for (int w = 0; w < kPrepWarps; ++w) v += part[w][threadIdx.x];
                ds[qb + threadIdx.x] = v;  // pair order; scattered to the slots afterwards
            }
            __syncthreads();  // part is reused by the next batch
        }
    }
}

// dweights[s] = ds[slot_pair[s]] where slot s is a pair, else 0.
__global__ void __launch_bounds__(256) scatter_slots_kernel(const int32_t *__restrict__ slot_pair,
                                                            const float *__restrict__ ds, int64_t NK,
                                                            float *__restrict__ dweights, const WsHeader *hdr) {
    if (hdr && *(volatile const uint32_t *)&hdr->abort) return;
    for (int64_t s = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; s < NK; s += (int64_t)gridDim.x * blockDim.x) {
        const int q = __ldg(slot_pair + s);
        dweights[s] = q >= 0 ? __ldg(ds + q) : 0.f;
    }
}

// db[e, c] = sum over rows p in [off[e], off[e+1]) of src[p, c]; one thread per
// column pair, rows in order.
__global__ void __launch_bounds__(256) bias_grad_kernel(const __nv_bfloat16 *__restrict__ src, int32_t cols,
                                                        const int32_t *__restrict__ expert_off,
                                                        __nv_bfloat16 *__restrict__ db, const WsHeader *hdr) {
    if (hdr && *(volatile const uint32_t *)&hdr->abort) return;
    const int e = blockIdx.y;
    const int c2 = blockIdx.x * blockDim.x + threadIdx.x;  // column pair
    if (2 * c2 >= cols) return;
    const int p0 = __ldg(expert_off + e), p1 = __ldg(expert_off + e + 1);
    float s0 = 0.f, s1 = 0.f;
    const uint32_t *base = reinterpret_cast<const uint32_t *>(src) + c2;
    const int ld = cols >> 1;
    int p = p0;
    for (; p + 4 <= p1; p += 4) {
        uint32_t v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = __ldg(base + (size_t)(p + u) * ld);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            s0 += bf16lo(v[u]);
            s1 += bf16hi(v[u]);
        }
    }
    for (; p < p1; ++p) {
        const uint32_t v = __ldg(base + (size_t)p * ld);
        s0 += bf16lo(v);
        s1 += bf16hi(v);
    }
    reinterpret_cast<uint32_t *>(db + (size_t)e * cols)[c2] = pack_bf16x2(s0, s1);
}

// dst[p, :] = src[idx[p], :] for p < P = expert_off[E] (16-byte chunks): four
// rows per block iteration (grid-stride over rows, their loads in flight
// together), the block's threads over the chunks, so no per-chunk division
// is needed.
__global__ void __launch_bounds__(256) gather_rows_kernel(const __nv_bfloat16 *__restrict__ src,
                                                          const int32_t *__restrict__ idx,
                                                          const int32_t *__restrict__ p_total, int32_t cols,
                                                          __nv_bfloat16 *__restrict__ dst, const WsHeader *hdr) {
    if (hdr && *(volatile const uint32_t *)&hdr->abort) return;
    const int P = __ldg(p_total);
    const int chunks = cols >> 3;
    constexpr int kRows = 4;  // rows in flight per block iteration
    for (int p0 = blockIdx.x * kRows; p0 < P; p0 += gridDim.x * kRows) {
        const uint4 *s[kRows];
#pragma unroll
        for (int u = 0; u < kRows; ++u)
            s[u] = reinterpret_cast<const uint4 *>(src + (size_t)__ldg(idx + min(p0 + u, P - 1)) * cols);
        for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
            uint4 v[kRows];
#pragma unroll
            for (int u = 0; u < kRows; ++u) v[u] = __ldg(s[u] + c);
#pragma unroll
            for (int u = 0; u < kRows; ++u)
                if (p0 + u < P) reinterpret_cast<uint4 *>(dst + (size_t)(p0 + u) * cols)[c] = v[u];
        }
    }
}

}  // namespace

cudaError_t launch_gather_rows(const __nv_bfloat16 *src, const int32_t *idx, const int32_t *p_total, int32_t cols,
                               __nv_bfloat16 *dst, const WsHeader *hdr, int num_sms, cudaStream_t s) {
    gather_rows_kernel<<<(unsigned)(num_sms * 8), 256, 0, s>>>(src, idx, p_total, cols, dst, hdr);
    return cudaGetLastError();
}

cudaError_t launch_bwd_prep(const __nv_bfloat16 *dout, const void *y, const int8_t *y_scale, const moe_meta_t &meta, int64_t N,
                            int32_t H, __nv_bfloat16 *dy, float *ds, const int32_t *slot_pair, int64_t NK,
                            float *dweights, const WsHeader *hdr, int num_sms, cudaStream_t s) {
    if (N > 0) {
        int64_t blocks = N;
        const int64_t cap = (int64_t)num_sms * 8;
        if (blocks > cap) blocks = cap;
        bwd_prep_kernel<<<(unsigned)blocks, kPrepThreads, 0, s>>>(dout, static_cast<const uint16_t *>(y), y_scale,
                                                                  meta.token_offset,
                                                                  meta.s_reverse_scatter_idx, meta.scores, N, H,
                                                                  dy, ds, hdr);
        const cudaError_t err = cudaGetLastError();
        if (err != cudaSuccess) return err;
    }
    if (NK > 0) {
        int64_t blocks = (NK + 255) / 256;
        const int64_t cap = (int64_t)num_sms * 8;
        if (blocks > cap) blocks = cap;
        scatter_slots_kernel<<<(unsigned)blocks, 256, 0, s>>>(slot_pair, ds, NK, dweights, hdr);
    }
    return cudaGetLastError();
}

cudaError_t launch_bias_grad(const __nv_bfloat16 *src, int32_t cols, const int32_t *expert_off, int32_t E,
                             __nv_bfloat16 *db, const WsHeader *hdr, cudaStream_t s) {
    const dim3 grid((unsigned)((cols / 2 + 255) / 256), (unsigned)E);
    bias_grad_kernel<<<grid, 256, 0, s>>>(src, cols, expert_off, db, hdr);
    return cudaGetLastError();
}

}  // namespace moe
