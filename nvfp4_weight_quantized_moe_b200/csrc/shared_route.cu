// The shared expert as extra routing slots.
//
// metrale_model_layers/layers/ops/nvfp4_moe_grouped.rs, docs of the gate+up and
// down launchers: the shared expert runs in the same launches as the routed
// experts, one row per token, with grid rows of its own after the routed ones.
// Here every token gets one more slot, k, naming table entry
// num_experts + t / shared_rows; the caller's tables hold the shared weights
// at those entries.  Grouping by expert then places the shared rows after all
// routed rows, in token order, in blocks of shared_rows tokens, and the
// unchanged projection kernels give each block its own CTAs.

#include "common.cuh"
#include "kernels.h"

namespace nvm {

namespace {
constexpr int kAppendThreads = 256;
}

__global__ void __launch_bounds__(kAppendThreads)
    append_shared_kernel(const int32_t* __restrict__ ids, const float* __restrict__ w,
                         const float* __restrict__ shared_w, int32_t* __restrict__ ids_out,
                         float* __restrict__ w_out, uint32_t num_tokens, uint32_t topk,
                         uint32_t num_experts, uint32_t shared_rows) {
  griddep_wait();  // the previous kernel on the stream may still read ids_out / w_out
  griddep_launch_dependents();
  const uint32_t k1 = topk + 1;
  const uint64_t total = (uint64_t)num_tokens * k1;
  const uint64_t stride = (uint64_t)gridDim.x * kAppendThreads;
  for (uint64_t i = (uint64_t)blockIdx.x * kAppendThreads + threadIdx.x; i < total; i += stride) {
    const uint32_t t = (uint32_t)(i / k1);
    const uint32_t s = (uint32_t)(i - (uint64_t)t * k1);
    if (s < topk) {
      const uint64_t src = (uint64_t)t * topk + s;
      ids_out[i] = ids[src];
      w_out[i] = w[src];
    } else {
      ids_out[i] = (int32_t)(num_experts + t / shared_rows);
      w_out[i] = shared_w != nullptr ? shared_w[t] : 1.0f;
    }
  }
}

cudaError_t launch_append_shared(const int32_t* ids, const float* w, const float* shared_w,
                                 int32_t* ids_out, float* w_out, uint32_t num_tokens,
                                 uint32_t topk, uint32_t num_experts, uint32_t shared_rows,
                                 cudaStream_t stream) {
  const uint64_t total = (uint64_t)num_tokens * (topk + 1);
  uint64_t blocks = (total + kAppendThreads - 1) / kAppendThreads;
  if (blocks > 148 * 8) blocks = 148 * 8;
  return launch_pdl(append_shared_kernel, dim3((unsigned)blocks), dim3(kAppendThreads), 0, stream,
                    ids, w, shared_w, ids_out, w_out, num_tokens, topk, num_experts, shared_rows);
}

}  // namespace nvm
