// Launchers of the expert-parallel dispatch / combine kernels (ep.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_nonexpand.h"

namespace moe {

cudaError_t launch_ep_layout(const int32_t *topk_idx, int64_t T, int K, int R, int E_local, int32_t *send_idx,
                             int32_t *send_count, uint32_t *err, cudaStream_t s);
cudaError_t launch_ep_dispatch(const void *x, const int32_t *topk_idx, const float *topk_w, const int32_t *send_idx,
                               int64_t T, int H, int K, int R, int E_local, const moe_ep_peers_t &peers,
                               int num_sms, cudaStream_t s);
cudaError_t launch_ep_combine(const moe_ep_sources_t &src, const int32_t *send_idx, int64_t T, int H, int R, void *out,
                              int num_sms, cudaStream_t s);

}  // namespace moe
