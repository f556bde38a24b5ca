// Self-test of the failure path every pipeline wait of the GEMM kernels
// takes: a bounded mbarrier wait that nothing will ever complete must give up
// after its limit, record MOE_DEVERR_TIMEOUT in the workspace's error word and
// let the kernel return normally, leaving the context usable.  No fault, trap
// or endless loop is involved.
#include "common.cuh"

namespace moe {
namespace {

__global__ void wait_timeout_selftest_kernel(WsHeader *hdr, unsigned long long timeout_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // nothing arrives on the barrier: its first phase never completes
        const bool ok = mbar_wait_bounded(smem_u32(&bar), 0, &abort_flag, timeout_ns);
        if (!ok && abort_flag) atomicOr(&hdr->err, MOE_DEVERR_TIMEOUT);
    }
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" MOE_API int moe_nonexpand_selftest_wait_timeout(void *ws, size_t ws_bytes, uint32_t timeout_us,
                                                          moe_stream_t stream) {
    if (!ws || ws_bytes < sizeof(WsHeader) || (reinterpret_cast<uintptr_t>(ws) % 256) != 0) return MOE_ERR_WS;
    if (timeout_us < 1 || timeout_us > 2000000) return MOE_ERR_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    WsHeader *hdr = static_cast<WsHeader *>(ws);
    if (cudaMemsetAsync(&hdr->err, 0, sizeof(hdr->err), s) != cudaSuccess) return MOE_ERR_CUDA;
    wait_timeout_selftest_kernel<<<1, 32, 0, s>>>(hdr, (unsigned long long)timeout_us * 1000ull);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
