// Load-time validation of the E4M3 block scales of one projection.
//
// metrale_model_layers/layers/ops/nvfp4_moe_grouped.rs, `nvfp4_tc_lean_repack`:
// a negative or NaN block scale leaves a matrix unusable, and the load-time
// pass reports it in a device word the caller has zeroed.  Here the report is a
// count per expert of scale codes whose value is NaN (0x7F, 0xFF) or below zero
// (sign bit with a non-zero magnitude: 0x81..0xFE); 0x80 is -0 and passes.
//
// A byte scan bound by HBM: 16-byte streaming loads, four in flight per thread,
// four bytes per SIMD compare, one atomic add per warp.

#include "common.cuh"
#include "kernels.h"

namespace nvm {

namespace {
constexpr int kCheckThreads = 256;
constexpr int kCheckUnroll = 4;
constexpr uint64_t kVecsPerCta = (uint64_t)kCheckThreads * kCheckUnroll;

// Invalid codes among the four bytes of w.
__device__ __forceinline__ uint32_t bad_codes4(uint32_t w) {
  const uint32_t m = __vcmpgeu4(w, 0x81818181u) | __vcmpeq4(w, 0x7F7F7F7Fu);
  return (uint32_t)__popc(m) >> 3;
}
}  // namespace

__global__ void __launch_bounds__(kCheckThreads)
    check_scales_kernel(const void* const* __restrict__ packed_ptrs,
                        const void* const* __restrict__ scale_ptrs, uint64_t vecs_per_expert,
                        uint32_t* __restrict__ bad) {
  griddep_wait();
  griddep_launch_dependents();
  const uint32_t e = blockIdx.y;
  const uint4* p = reinterpret_cast<const uint4*>(scale_ptrs[e]);
  uint32_t cnt = 0;
  if (p != nullptr && packed_ptrs[e] != nullptr) {  // a NULL expert is not checked
    for (uint64_t base = (uint64_t)blockIdx.x * kVecsPerCta; base < vecs_per_expert;
         base += (uint64_t)gridDim.x * kVecsPerCta) {
      uint4 v[kCheckUnroll];
#pragma unroll
      for (int j = 0; j < kCheckUnroll; ++j) {
        const uint64_t i = base + (uint64_t)j * kCheckThreads + threadIdx.x;
        v[j] = i < vecs_per_expert ? __ldcs(p + i) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int j = 0; j < kCheckUnroll; ++j)
        cnt += bad_codes4(v[j].x) + bad_codes4(v[j].y) + bad_codes4(v[j].z) + bad_codes4(v[j].w);
    }
  }
  cnt = __reduce_add_sync(0xffffffffu, cnt);
  if ((threadIdx.x & 31) == 0 && cnt != 0) atomicAdd(bad + e, cnt);
}

cudaError_t launch_check_scales(const void* const* packed_ptrs, const void* const* scale_ptrs,
                                uint32_t num_experts, uint64_t bytes_per_expert, uint32_t* bad,
                                cudaStream_t stream) {
  const uint64_t vecs = bytes_per_expert / 16;
  uint64_t gx = (vecs + kVecsPerCta - 1) / kVecsPerCta;
  if (gx > 65535) gx = 65535;
  return launch_pdl(check_scales_kernel, dim3((unsigned)gx, num_experts), dim3(kCheckThreads), 0,
                    stream, packed_ptrs, scale_ptrs, vecs, bad);
}

}  // namespace nvm
