// Internal launch interface between the C ABI (abi.cu) and the kernels.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace nvm {

// Projection modes: gate+up with the fused SiLU product; down; the up
// projection of a non-gated expert followed by an activation.
enum { kModeGateUp = 0, kModeDown = 1, kModeUpAct = 2 };
// Activations of a non-gated expert (the values of nvfp4_moe_activation).
enum { kActRelu2 = 1, kActSilu = 2 };

// Limits shared by every entry point: expert table entries and routed pairs
// per call.
constexpr uint32_t kMaxExperts = 1024;
constexpr uint64_t kMaxPairs = 1ull << 24;

// Token rows per pass of the tcgen05 kernels, from the host-known sizes:
//   * more than 16 rows per expert on average: the CTA-pair kernel at 256-row
//     passes for gate+up and up+activation (A operand in shared memory), 192
//     for down (A in tensor memory);
//   * batches of at most 16 tokens (no expert can have more rows), or 5..16
//     rows per expert on average: 16 (one-CTA kernel, one pass per expert);
//   * more than 16 tokens spread at most 4 per expert on average, where a
//     skewed router gives a few experts more than 16 rows: 32 (CTA-pair
//     kernel), so those experts still take one pass.
// Measured on B200: 32-row pair passes 12 % faster than 16-row passes on the
// skewed decode M=32 workload (2 rows per expert on average), 13 % slower on
// decode M=256 (8 per expert, uniform).  `tiles` > 0 (a launch option) forces
// tiles * 8: 2 -> 16, 16 -> 128 (one-CTA kernel), 4 -> 32, 24 -> 192 and (not
// for down) 32 -> 256 (pair kernel).
constexpr int kTcPairRows = 192;
constexpr int kTcPairRowsSmall = 32;
constexpr int kTcPairRowsWide = 256;
inline int plan_tc_rows(uint64_t tokens, uint64_t pairs, uint32_t num_experts, int tiles, int mode) {
  if (tiles > 0) return tiles * 8;
  const uint64_t mean = (pairs + num_experts - 1) / num_experts;
  if (mean > 16) return mode == kModeDown ? kTcPairRows : kTcPairRowsWide;
  if (tokens > 16 && mean <= 4) return kTcPairRowsSmall;
  return 16;
}

// Arguments of the grouped projection kernels.  Mode gate+up reads BF16 x
// [M, K] and two weight tables (gate, up) with the same [N, K]; mode down
// reads FP32 act [P, K] and one table; mode up+activation reads BF16 x and
// one table.  `out` is [P, N] FP32 by sorted position.
struct GroupedArgs {
  const void* src;
  const void* const* packed0;
  const void* const* scale0;
  const float* s2_0;
  const void* const* packed1;
  const void* const* scale1;
  const float* s2_1;
  float* out;
  const int32_t* offsets;
  const int32_t* sorted_pair_ids;
  const int32_t* active_experts;
  const int32_t* active_count;
  uint32_t N, K, topk;
  uint32_t num_experts;
  int activation;  // mode up+activation: kActRelu2 or kActSilu
};

// Launch shape of the decode path (grouped_mma.cu):
//   split  warps of a CTA that split K over the same rows (1, 2 or 4)
//   tiles  8-token tiles held per pass over an expert (1, 2 or 4)
//   depth  weight chunks in flight per warp (2 or 3)
struct DecodePlan {
  int split;
  int tiles;
  int depth;
  int xres;  // 1: each pass stages every K chunk of its token rows up front
};

cudaError_t launch_grouped(int mode, const DecodePlan& plan, const GroupedArgs& a, uint32_t cap,
                           cudaStream_t stream);
bool grouped_plan_supported(int mode, const DecodePlan& plan);
int grouped_rows_per_cta(int mode, int split);
// Dynamic shared memory of whole-K staging for this plan and K.
int grouped_xres_smem(int mode, const DecodePlan& plan, uint32_t k);
// Largest dynamic shared memory a decode launch takes; automatic plans stage
// whole K only up to kDecodeXresAuto (three CTAs per SM).
constexpr int kDecodeSmemMax = 200 * 1024;
constexpr int kDecodeXresAuto = 72 * 1024;

// tcgen05 path (grouped_tc.cu): activation packing and per-expert weight
// tensor maps into `workspace` (256-byte aligned), then the projection kernel
// with NT token rows per pass (16 or 128).
size_t tc_workspace_bytes(uint64_t tokens, uint64_t topk, uint64_t hidden, uint64_t inter);
// Leading part of that workspace the gate+up step uses (sorted f16 rows, their
// scales and the per-expert weight tensor maps).
size_t tc_gate_up_workspace_bytes(uint64_t pairs, uint64_t hidden);
cudaError_t launch_tc(int mode, int nt, const GroupedArgs& a, void* workspace, uint32_t tokens,
                      uint32_t hidden, uint32_t inter, uint32_t cap, cudaStream_t stream);
cudaError_t read_device_error(int* value, bool clear);
// One bounded barrier wait on the device (self-test of the timeout path).
cudaError_t launch_wait_selftest(uint32_t cycle_limit, int arrive, cudaStream_t stream);

cudaError_t launch_route_sort(const int32_t* topk_ids, uint32_t num_pairs, uint32_t num_experts,
                              int32_t* expert_offsets, int32_t* sorted_pair_ids, int32_t* pair_pos,
                              int32_t* active_experts, int32_t* active_count, int32_t* status,
                              cudaStream_t stream);

cudaError_t launch_blend(const float* y, const float* topk_weights, const int32_t* pair_pos,
                         float* out_f32, uint16_t* out_bf16, uint32_t num_tokens, uint32_t topk,
                         uint32_t hidden, cudaStream_t stream);

cudaError_t launch_append_shared(const int32_t* ids, const float* w, const float* shared_w,
                                 int32_t* ids_out, float* w_out, uint32_t num_tokens,
                                 uint32_t topk, uint32_t num_experts, uint32_t shared_rows,
                                 cudaStream_t stream);

cudaError_t launch_check_scales(const void* const* packed_ptrs, const void* const* scale_ptrs,
                                uint32_t num_experts, uint64_t bytes_per_expert, uint32_t* bad,
                                cudaStream_t stream);

cudaError_t launch_shard_copy(const uint8_t* src, uint8_t* dst, uint64_t mats, uint32_t rows_src,
                              uint32_t cols_src, uint32_t rows_out, uint32_t cols_out,
                              uint32_t row_off, uint32_t col_off, cudaStream_t stream);

cudaError_t launch_transpose_u8(const uint8_t* src, uint8_t* dst, uint32_t rows, uint32_t cols,
                                cudaStream_t stream);
// Transpose [rows, cols] into columns dst_col_off .. of a [cols, dst_pitch] output.
cudaError_t launch_transpose_u8_pitched(const uint8_t* src, uint8_t* dst, uint32_t rows,
                                        uint32_t cols, uint64_t dst_pitch, uint64_t dst_col_off,
                                        cudaStream_t stream);
cudaError_t launch_zero_cols(uint8_t* dst, uint64_t rows, uint64_t pitch, uint64_t col_lo,
                             cudaStream_t stream);

// Raise a kernel's dynamic shared-memory limit once per (kernel, device).
cudaError_t ensure_dynamic_smem(const void* kernel, int bytes);

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel on the stream is still running; every kernel of this
// library calls griddep_wait() before it touches data an earlier kernel writes.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace nvm
