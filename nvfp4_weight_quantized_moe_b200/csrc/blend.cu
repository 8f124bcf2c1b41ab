// Step 4 of the expert forward: the router-weighted blend back into token
// order (`moe_weighted_sum_blend_fp8_grouped`, named in the module doc of
// metrale_model_layers/layers/ops/nvfp4_moe_grouped.rs).
//
// out[t, j] = sum over s = 0..k-1, in that order, of w[t, s] * y[pair_pos[t*k+s], j]
// as an FP32 fused multiply-add chain: a gather, no atomics, so the result is
// the same on every run.  Each thread owns 4 consecutive columns (16-byte loads
// of y, 16-byte stores of out); an optional BF16 copy is rounded to nearest even.

#include "common.cuh"
#include "kernels.h"

namespace nvm {

namespace {
constexpr int kBlendThreads = 256;
}

__global__ void __launch_bounds__(kBlendThreads)
    blend_kernel(const float* __restrict__ y, const float* __restrict__ w,
                 const int32_t* __restrict__ pair_pos, float* __restrict__ out,
                 uint16_t* __restrict__ out_bf16, int k, int H) {
  griddep_wait();  // y of the down projection is complete
  griddep_launch_dependents();
  const int t = blockIdx.y;
  const int col = (blockIdx.x * kBlendThreads + threadIdx.x) * 4;
  if (col >= H) return;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s = 0; s < k; ++s) {
    const int pos = __ldg(pair_pos + (size_t)t * k + s);
    if (pos < 0) continue;
    const float ws = __ldg(w + (size_t)t * k + s);
    const float4 v = __ldg(reinterpret_cast<const float4*>(y + (size_t)pos * H + col));
    acc.x = fmaf(ws, v.x, acc.x);
    acc.y = fmaf(ws, v.y, acc.y);
    acc.z = fmaf(ws, v.z, acc.z);
    acc.w = fmaf(ws, v.w, acc.w);
  }
  *reinterpret_cast<float4*>(out + (size_t)t * H + col) = acc;
  if (out_bf16 != nullptr) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
    __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
    uint2 packed;
    packed.x = *reinterpret_cast<uint32_t*>(&lo);
    packed.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(out_bf16 + (size_t)t * H + col) = packed;
  }
}

cudaError_t launch_blend(const float* y, const float* topk_weights, const int32_t* pair_pos,
                         float* out_f32, uint16_t* out_bf16, uint32_t num_tokens, uint32_t topk,
                         uint32_t hidden, cudaStream_t stream) {
  const dim3 grid((hidden / 4 + kBlendThreads - 1) / kBlendThreads, num_tokens);
  return launch_pdl(blend_kernel, grid, dim3(kBlendThreads), 0, stream, y, topk_weights, pair_pos,
                    out_f32, out_bf16, (int)topk, (int)hidden);
}

}  // namespace nvm
