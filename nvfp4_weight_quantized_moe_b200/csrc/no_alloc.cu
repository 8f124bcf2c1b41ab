// Allocation-free form of the tcgen05 gate+up call.
//
// nvfp4_moe_gate_up_silu_ws needs a caller-provided device workspace for the
// packed f16 token rows.  Some callers cannot provide one: code that runs
// inside a host whose device memory is owned by someone else (a framework's
// caching allocator, a fixed memory budget handed out up front) and code that
// must not make a call that can block on the whole device or fail midway, which
// cudaMalloc can do.  For them, nvfp4_moe_gate_up_silu_noalloc uses a fixed
// scratch array that lives in this library's own device image instead.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library holds it until the process exits; its size is kept modest for that
// reason (kStaticScratchBytes).  Host code cannot use the variable's name as a
// device address, so the address is looked up with cudaGetSymbolAddress, once
// per device, on that device's first call.  The cached address belongs to the
// device's context at that time: after cudaDeviceReset the library must not be
// called again on that device in this process.

#include <mutex>

#include "../../include/nvfp4_moe.h"
#include "kernels.h"

namespace nvm {

// Packed token rows (f16) and their power-of-two scales for one call.
constexpr size_t kStaticScratchBytes = size_t(8) << 20;  // 8 MiB per device
static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

namespace {

// Device address of g_static_scratch on the current device (set up once per
// device, with that device current).
cudaError_t static_scratch_address(void** out) {
  constexpr int kMaxDevices = 64;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_static_scratch);
    if (err != cudaSuccess) return err;
    addr[dev] = p;
  }
  *out = addr[dev];
  return cudaSuccess;
}

// Bytes of scratch the gate+up call reads and writes: the leading gate+up part
// of the workspace layout of the _ws calls (packed rows by sorted position
// [P, k_hidden] f16, one f32 scale per row, the per-expert weight tensor maps).
size_t gate_up_scratch_bytes(uint64_t pairs, uint64_t hidden) { return tc_gate_up_workspace_bytes(pairs, hidden); }

}  // namespace
}  // namespace nvm

using namespace nvm;

extern "C" int nvfp4_moe_gate_up_silu_noalloc(
    const uint16_t* x, nvfp4_expert_tables gate, nvfp4_expert_tables up, float* act,
    const int32_t* expert_offsets, const int32_t* sorted_pair_ids, const int32_t* active_experts,
    const int32_t* active_count, uint32_t n_inter, uint32_t k_hidden, uint32_t cap,
    uint32_t num_tokens, uint32_t topk, uint32_t num_experts, cudaStream_t stream) {
  if (n_inter == 0 || n_inter % 128 != 0 || k_hidden == 0 || k_hidden % 256 != 0 || topk == 0 ||
      cap > 65535 || num_experts == 0 || num_experts > kMaxExperts)
    return NVFP4_MOE_ESHAPE;
  const uint64_t pairs = (uint64_t)num_tokens * topk;
  if (pairs > kMaxPairs) return NVFP4_MOE_ESHAPE;
  // Requests whose packed rows do not fit the fixed scratch are refused.
  if (gate_up_scratch_bytes(pairs, k_hidden) > kStaticScratchBytes) return NVFP4_MOE_ESHAPE;
  if (pairs == 0 || cap == 0) return NVFP4_MOE_OK;
  if (x == nullptr || act == nullptr || expert_offsets == nullptr || sorted_pair_ids == nullptr ||
      active_experts == nullptr || active_count == nullptr || gate.packed_ptrs == nullptr ||
      gate.scale_ptrs == nullptr || gate.scale2 == nullptr || up.packed_ptrs == nullptr ||
      up.scale_ptrs == nullptr || up.scale2 == nullptr)
    return NVFP4_MOE_EINVAL;
  void* scratch = nullptr;
  if (static_scratch_address(&scratch) != cudaSuccess) return NVFP4_MOE_ECUDA;
  // Nothing in the scratch has to start at zero: the pack kernel writes every
  // packed row and scale before the projection kernel reads them.
  const int nt = plan_tc_rows(num_tokens, pairs, num_experts, 0, kModeGateUp);  // the _ws call's rule
  GroupedArgs a{};
  a.src = x;
  a.packed0 = gate.packed_ptrs;
  a.scale0 = gate.scale_ptrs;
  a.s2_0 = gate.scale2;
  a.packed1 = up.packed_ptrs;
  a.scale1 = up.scale_ptrs;
  a.s2_1 = up.scale2;
  a.out = act;
  a.offsets = expert_offsets;
  a.sorted_pair_ids = sorted_pair_ids;
  a.active_experts = active_experts;
  a.active_count = active_count;
  a.N = n_inter;
  a.K = k_hidden;
  a.topk = topk;
  a.num_experts = num_experts;
  const cudaError_t err = launch_tc(kModeGateUp, nt, a, scratch, num_tokens, k_hidden, n_inter, cap, stream);
  return err == cudaSuccess ? NVFP4_MOE_OK : NVFP4_MOE_ECUDA;
}
