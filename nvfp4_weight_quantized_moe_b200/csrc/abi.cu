// C ABI of the grouped NVFP4 MoE expert forward: argument checks on the host,
// path choice, launches.  Declarations and argument contracts: include/nvfp4_moe.h.

#include <map>
#include <mutex>
#include <utility>

#include "../../include/nvfp4_moe.h"
#include "kernels.h"

namespace nvm {

cudaError_t ensure_dynamic_smem(const void* kernel, int bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> done;
  std::lock_guard<std::mutex> lock(mu);
  auto key = std::make_pair(kernel, dev);
  auto it = done.find(key);
  if (it != done.end() && it->second >= bytes) return cudaSuccess;
  err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (err == cudaSuccess) done[key] = bytes;
  return err;
}

namespace {

bool tables_ok(const nvfp4_expert_tables& t) {
  return t.packed_ptrs != nullptr && t.scale_ptrs != nullptr && t.scale2 != nullptr;
}

int status_of(cudaError_t err) { return err == cudaSuccess ? NVFP4_MOE_OK : NVFP4_MOE_ECUDA; }

constexpr int kSmsEstimate = 148;

// Decode-path launch shape from the host-known sizes.  Rows per expert are at
// most min(tokens, pairs) (a token picks an expert once), so small batches hold
// every row of an expert in one pass; larger ones size the pass for twice the
// mean.  With one tile, the CTA's warps split K when the grid would otherwise
// leave SMs short of weight streams.
DecodePlan plan_decode(int mode, uint64_t tokens, uint64_t pairs, uint32_t num_experts,
                       uint32_t cap, uint32_t n, uint32_t k, const nvfp4_moe_launch_opts* o) {
  DecodePlan p{};
  const uint64_t max_rows = tokens < pairs ? tokens : pairs;
  const uint64_t mean = (pairs + num_experts - 1) / num_experts;
  if (max_rows <= 16) {
    p.tiles = (int)((max_rows + 7) / 8);
  } else {
    p.tiles = (int)((2 * mean + 7) / 8);
    if (p.tiles < 2) p.tiles = 2;
  }
  if (p.tiles < 1) p.tiles = 1;
  if (p.tiles == 3 || p.tiles > 4) p.tiles = 4;
  if (mode != kModeGateUp && p.tiles > 2) p.tiles = 2;
  if (o && o->tiles) p.tiles = o->tiles;
  const uint64_t active = cap < pairs ? cap : pairs;
  auto ctas = [&](int split) {
    const uint64_t rpc = (uint64_t)grouped_rows_per_cta(mode, split);
    return ((n + rpc - 1) / rpc) * active;
  };
  p.split = 1;
  if (p.tiles == 1 && ctas(1) < 2 * kSmsEstimate) p.split = ctas(2) < kSmsEstimate ? 4 : 2;
  if (o && o->split) p.split = o->split;
  p.depth = 2;
  if (o && o->depth) p.depth = o->depth;
  // Whole-K staging when the token rows of a pass fit in shared memory next to
  // three CTAs per SM; the ring otherwise.
  p.xres = grouped_xres_smem(mode, p, k) <= kDecodeXresAuto ? 1 : 0;
  if (o && o->staging) p.xres = o->staging == 1 ? 1 : o->staging == 2 ? 0 : -1;
  return p;
}

// A plan the decode kernels have an instance for and whose staging fits.
bool plan_ok(int mode, const DecodePlan& p, uint32_t k) {
  if (p.xres < 0 || !grouped_plan_supported(mode, p)) return false;
  return !p.xres || grouped_xres_smem(mode, p, k) <= kDecodeSmemMax;
}

}  // namespace
}  // namespace nvm

using namespace nvm;

extern "C" {

uint32_t nvfp4_moe_active_cap(uint32_t num_experts, uint32_t num_pairs) {
  return num_experts < num_pairs ? num_experts : num_pairs;
}

const char* nvfp4_moe_status_string(int status) {
  switch (status) {
    case NVFP4_MOE_OK: return "ok";
    case NVFP4_MOE_EINVAL: return "invalid argument (NULL pointer or bad value)";
    case NVFP4_MOE_ESHAPE: return "unsupported shape";
    case NVFP4_MOE_ECUDA: return "CUDA launch or runtime error";
    default: return "unknown status";
  }
}

int nvfp4_moe_route_sort(const int32_t* topk_ids, uint32_t num_tokens, uint32_t topk,
                         uint32_t num_experts, int32_t* expert_offsets,
                         int32_t* sorted_pair_ids, int32_t* pair_pos,
                         int32_t* active_experts, int32_t* active_count,
                         int32_t* status, cudaStream_t stream) {
  if (expert_offsets == nullptr || active_experts == nullptr || active_count == nullptr)
    return NVFP4_MOE_EINVAL;
  if (num_experts == 0 || num_experts > kMaxExperts || topk == 0 || topk > num_experts)
    return NVFP4_MOE_ESHAPE;
  const uint64_t pairs = (uint64_t)num_tokens * topk;
  if (pairs > kMaxPairs) return NVFP4_MOE_ESHAPE;
  if (pairs > 0 && (topk_ids == nullptr || sorted_pair_ids == nullptr || pair_pos == nullptr))
    return NVFP4_MOE_EINVAL;
  return status_of(launch_route_sort(topk_ids, (uint32_t)pairs, num_experts, expert_offsets,
                                     sorted_pair_ids, pair_pos, active_experts, active_count,
                                     status, stream));
}

int nvfp4_moe_gate_up_silu_ex(const uint16_t* x, nvfp4_expert_tables gate,
                              nvfp4_expert_tables up, float* act,
                              const int32_t* expert_offsets, const int32_t* sorted_pair_ids,
                              const int32_t* active_experts, const int32_t* active_count,
                              uint32_t n_inter, uint32_t k_hidden, uint32_t cap,
                              uint32_t num_tokens, uint32_t topk,
                              const nvfp4_moe_launch_opts* opts, cudaStream_t stream) {
  if (n_inter == 0 || n_inter % 64 != 0 || k_hidden == 0 || k_hidden % 256 != 0 || topk == 0 ||
      cap > 65535)
    return NVFP4_MOE_ESHAPE;
  const uint64_t pairs = (uint64_t)num_tokens * topk;
  if (pairs > kMaxPairs) return NVFP4_MOE_ESHAPE;
  if (pairs == 0 || cap == 0) return NVFP4_MOE_OK;
  if (x == nullptr || act == nullptr || expert_offsets == nullptr || sorted_pair_ids == nullptr ||
      active_experts == nullptr || active_count == nullptr || !tables_ok(gate) || !tables_ok(up))
    return NVFP4_MOE_EINVAL;
  const int path = opts ? opts->path : 0;
  if (path != 0 && path != 1) return NVFP4_MOE_EINVAL;
  const DecodePlan plan =
      plan_decode(kModeGateUp, num_tokens, pairs, cap, cap, n_inter, k_hidden, opts);
  if (!plan_ok(kModeGateUp, plan, k_hidden)) return NVFP4_MOE_EINVAL;
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
  a.num_experts = 0;
  return status_of(launch_grouped(kModeGateUp, plan, a, cap, stream));
}

int nvfp4_moe_gate_up_silu(const uint16_t* x, nvfp4_expert_tables gate,
                           nvfp4_expert_tables up, float* act,
                           const int32_t* expert_offsets, const int32_t* sorted_pair_ids,
                           const int32_t* active_experts, const int32_t* active_count,
                           uint32_t n_inter, uint32_t k_hidden, uint32_t cap,
                           uint32_t num_tokens, uint32_t topk, cudaStream_t stream) {
  return nvfp4_moe_gate_up_silu_ex(x, gate, up, act, expert_offsets, sorted_pair_ids,
                                   active_experts, active_count, n_inter, k_hidden, cap,
                                   num_tokens, topk, nullptr, stream);
}

int nvfp4_moe_down_ex(const float* act, nvfp4_expert_tables down, float* y,
                      const int32_t* expert_offsets, const int32_t* active_experts,
                      const int32_t* active_count, uint32_t n_hidden, uint32_t k_inter,
                      uint32_t cap, uint32_t num_tokens, uint32_t topk,
                      const nvfp4_moe_launch_opts* opts, cudaStream_t stream) {
  if (n_hidden == 0 || n_hidden % 128 != 0 || k_inter == 0 || k_inter % 256 != 0 || topk == 0 ||
      cap > 65535)
    return NVFP4_MOE_ESHAPE;
  const uint64_t pairs = (uint64_t)num_tokens * topk;
  if (pairs > kMaxPairs) return NVFP4_MOE_ESHAPE;
  if (pairs == 0 || cap == 0) return NVFP4_MOE_OK;
  if (act == nullptr || y == nullptr || expert_offsets == nullptr || active_experts == nullptr ||
      active_count == nullptr || !tables_ok(down))
    return NVFP4_MOE_EINVAL;
  const int path = opts ? opts->path : 0;
  if (path != 0 && path != 1) return NVFP4_MOE_EINVAL;
  const DecodePlan plan =
      plan_decode(kModeDown, num_tokens, pairs, cap, cap, n_hidden, k_inter, opts);
  if (!plan_ok(kModeDown, plan, k_inter)) return NVFP4_MOE_EINVAL;
  GroupedArgs a{};
  a.src = act;
  a.packed0 = down.packed_ptrs;
  a.scale0 = down.scale_ptrs;
  a.s2_0 = down.scale2;
  a.out = y;
  a.offsets = expert_offsets;
  a.active_experts = active_experts;
  a.active_count = active_count;
  a.N = n_hidden;
  a.K = k_inter;
  a.topk = topk;
  return status_of(launch_grouped(kModeDown, plan, a, cap, stream));
}

int nvfp4_moe_down(const float* act, nvfp4_expert_tables down, float* y,
                   const int32_t* expert_offsets, const int32_t* active_experts,
                   const int32_t* active_count, uint32_t n_hidden, uint32_t k_inter,
                   uint32_t cap, uint32_t num_tokens, uint32_t topk, cudaStream_t stream) {
  return nvfp4_moe_down_ex(act, down, y, expert_offsets, active_experts, active_count, n_hidden,
                           k_inter, cap, num_tokens, topk, nullptr, stream);
}

size_t nvfp4_moe_workspace_bytes(uint32_t num_tokens, uint32_t topk, uint32_t hidden,
                                 uint32_t inter) {
  return tc_workspace_bytes(num_tokens, topk, hidden, inter);
}

int nvfp4_moe_device_error(int clear) {
  int v = 0;
  if (read_device_error(&v, clear != 0) != cudaSuccess) return -1;
  return v;
}

int nvfp4_moe_wait_selftest(uint32_t cycle_limit, int arrive, cudaStream_t stream) {
  if (cycle_limit == 0) return NVFP4_MOE_EINVAL;
  return status_of(launch_wait_selftest(cycle_limit, arrive != 0, stream));
}

namespace {

// The tcgen05 kernel covers 128 (gate+up) or 256 (down) output rows per CTA.
// Chosen automatically from 2 routed rows per expert on average: below that
// the register-fed decode kernel, which splits K over more CTAs, keeps more
// weight bytes in flight (measured on B200: decode kernel 2x faster at 0.06
// rows per expert; tcgen05 7% faster at 2 and 28% at 8).
bool use_tc(uint32_t n, uint32_t rows_per_cta, uint64_t pairs, uint32_t num_experts,
            const nvfp4_moe_launch_opts* o) {
  const int path = o ? o->path : 0;
  if (path == 1 || n % rows_per_cta != 0) return false;
  if (path == 2) return true;
  return pairs >= 2ull * num_experts;
}

}  // namespace

int nvfp4_moe_gate_up_silu_ws(const uint16_t* x, nvfp4_expert_tables gate, nvfp4_expert_tables up,
                              float* act, const int32_t* expert_offsets,
                              const int32_t* sorted_pair_ids, const int32_t* active_experts,
                              const int32_t* active_count, uint32_t n_inter, uint32_t k_hidden,
                              uint32_t cap, uint32_t num_tokens, uint32_t topk,
                              uint32_t num_experts, const nvfp4_moe_launch_opts* opts,
                              void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  const int path = opts ? opts->path : 0;
  if (path < 0 || path > 2) return NVFP4_MOE_EINVAL;
  if (!use_tc(n_inter, 128, (uint64_t)num_tokens * topk, num_experts, opts)) {
    if (path == 2) return NVFP4_MOE_ESHAPE;
    return nvfp4_moe_gate_up_silu_ex(x, gate, up, act, expert_offsets, sorted_pair_ids,
                                     active_experts, active_count, n_inter, k_hidden, cap,
                                     num_tokens, topk, opts, stream);
  }
  if (k_hidden == 0 || k_hidden % 256 != 0 || topk == 0 || cap > 65535 || num_experts == 0 ||
      num_experts > kMaxExperts)
    return NVFP4_MOE_ESHAPE;
  const uint64_t pairs = (uint64_t)num_tokens * topk;
  if (pairs > kMaxPairs) return NVFP4_MOE_ESHAPE;
  if (pairs == 0 || cap == 0) return NVFP4_MOE_OK;
  if (x == nullptr || act == nullptr || expert_offsets == nullptr || sorted_pair_ids == nullptr ||
      active_experts == nullptr || active_count == nullptr || !tables_ok(gate) || !tables_ok(up) ||
      workspace == nullptr)
    return NVFP4_MOE_EINVAL;
  if (workspace_bytes < tc_workspace_bytes(num_tokens, topk, k_hidden, n_inter)) return NVFP4_MOE_EINVAL;
  if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return NVFP4_MOE_EINVAL;
  const int nt = plan_tc_rows(num_tokens, pairs, num_experts, opts ? opts->tiles : 0, kModeGateUp);
  if (nt != 16 && nt != 128 && nt != kTcPairRows && nt != kTcPairRowsSmall && nt != kTcPairRowsWide) return NVFP4_MOE_EINVAL;
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
  return status_of(launch_tc(kModeGateUp, nt, a, workspace, num_tokens, k_hidden, n_inter, cap, stream));
}

int nvfp4_moe_down_ws(const float* act, nvfp4_expert_tables down, float* y,
                      const int32_t* expert_offsets, const int32_t* active_experts,
                      const int32_t* active_count, uint32_t n_hidden, uint32_t k_inter,
                      uint32_t cap, uint32_t num_tokens, uint32_t topk, uint32_t num_experts,
                      const nvfp4_moe_launch_opts* opts, void* workspace, size_t workspace_bytes,
                      cudaStream_t stream) {
  const int path = opts ? opts->path : 0;
  if (path < 0 || path > 2) return NVFP4_MOE_EINVAL;
  if (!use_tc(n_hidden, 256, (uint64_t)num_tokens * topk, num_experts, opts)) {
    if (path == 2) return NVFP4_MOE_ESHAPE;
    return nvfp4_moe_down_ex(act, down, y, expert_offsets, active_experts, active_count, n_hidden,
                             k_inter, cap, num_tokens, topk, opts, stream);
  }
  if (k_inter == 0 || k_inter % 256 != 0 || topk == 0 || cap > 65535 || num_experts == 0 ||
      num_experts > kMaxExperts)
    return NVFP4_MOE_ESHAPE;
  const uint64_t pairs = (uint64_t)num_tokens * topk;
  if (pairs > kMaxPairs) return NVFP4_MOE_ESHAPE;
  if (pairs == 0 || cap == 0) return NVFP4_MOE_OK;
  if (act == nullptr || y == nullptr || expert_offsets == nullptr || active_experts == nullptr ||
      active_count == nullptr || !tables_ok(down) || workspace == nullptr)
    return NVFP4_MOE_EINVAL;
  if (workspace_bytes < tc_workspace_bytes(num_tokens, topk, n_hidden, k_inter)) return NVFP4_MOE_EINVAL;
  if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return NVFP4_MOE_EINVAL;
  int nt = plan_tc_rows(num_tokens, pairs, num_experts, opts ? opts->tiles : 0, kModeDown);
  if (nt == kTcPairRowsWide) nt = kTcPairRows;  // down's widest pair pass (A in tensor memory)
  if (nt != 16 && nt != 128 && nt != kTcPairRows && nt != kTcPairRowsSmall) return NVFP4_MOE_EINVAL;
  GroupedArgs a{};
  a.src = act;
  a.packed0 = down.packed_ptrs;
  a.scale0 = down.scale_ptrs;
  a.s2_0 = down.scale2;
  a.out = y;
  a.offsets = expert_offsets;
  a.active_experts = active_experts;
  a.active_count = active_count;
  a.N = n_hidden;
  a.K = k_inter;
  a.topk = topk;
  a.num_experts = num_experts;
  return status_of(launch_tc(kModeDown, nt, a, workspace, num_tokens, n_hidden, k_inter, cap, stream));
}

int nvfp4_moe_up_act(const uint16_t* x, nvfp4_expert_tables up, float* act,
                     const int32_t* expert_offsets, const int32_t* sorted_pair_ids,
                     const int32_t* active_experts, const int32_t* active_count,
                     uint32_t n_inter, uint32_t k_hidden, uint32_t cap, uint32_t num_tokens,
                     uint32_t topk, int activation, const nvfp4_moe_launch_opts* opts,
                     cudaStream_t stream) {
  if (activation != NVFP4_MOE_ACT_RELU2 && activation != NVFP4_MOE_ACT_SILU) return NVFP4_MOE_EINVAL;
  if (n_inter == 0 || n_inter % 128 != 0 || k_hidden == 0 || k_hidden % 256 != 0 || topk == 0 ||
      cap > 65535)
    return NVFP4_MOE_ESHAPE;
  const uint64_t pairs = (uint64_t)num_tokens * topk;
  if (pairs > kMaxPairs) return NVFP4_MOE_ESHAPE;
  if (pairs == 0 || cap == 0) return NVFP4_MOE_OK;
  if (x == nullptr || act == nullptr || expert_offsets == nullptr || sorted_pair_ids == nullptr ||
      active_experts == nullptr || active_count == nullptr || !tables_ok(up))
    return NVFP4_MOE_EINVAL;
  const int path = opts ? opts->path : 0;
  if (path != 0 && path != 1) return NVFP4_MOE_EINVAL;
  const DecodePlan plan =
      plan_decode(kModeUpAct, num_tokens, pairs, cap, cap, n_inter, k_hidden, opts);
  if (!plan_ok(kModeUpAct, plan, k_hidden)) return NVFP4_MOE_EINVAL;
  GroupedArgs a{};
  a.src = x;
  a.packed0 = up.packed_ptrs;
  a.scale0 = up.scale_ptrs;
  a.s2_0 = up.scale2;
  a.out = act;
  a.offsets = expert_offsets;
  a.sorted_pair_ids = sorted_pair_ids;
  a.active_experts = active_experts;
  a.active_count = active_count;
  a.N = n_inter;
  a.K = k_hidden;
  a.topk = topk;
  a.activation = activation;
  return status_of(launch_grouped(kModeUpAct, plan, a, cap, stream));
}

int nvfp4_moe_up_act_ws(const uint16_t* x, nvfp4_expert_tables up, float* act,
                        const int32_t* expert_offsets, const int32_t* sorted_pair_ids,
                        const int32_t* active_experts, const int32_t* active_count,
                        uint32_t n_inter, uint32_t k_hidden, uint32_t cap, uint32_t num_tokens,
                        uint32_t topk, uint32_t num_experts, int activation,
                        const nvfp4_moe_launch_opts* opts, void* workspace, size_t workspace_bytes,
                        cudaStream_t stream) {
  const int path = opts ? opts->path : 0;
  if (path < 0 || path > 2) return NVFP4_MOE_EINVAL;
  if (activation != NVFP4_MOE_ACT_RELU2 && activation != NVFP4_MOE_ACT_SILU) return NVFP4_MOE_EINVAL;
  if (!use_tc(n_inter, 256, (uint64_t)num_tokens * topk, num_experts, opts)) {
    if (path == 2) return NVFP4_MOE_ESHAPE;
    return nvfp4_moe_up_act(x, up, act, expert_offsets, sorted_pair_ids, active_experts, active_count,
                            n_inter, k_hidden, cap, num_tokens, topk, activation, opts, stream);
  }
  if (k_hidden == 0 || k_hidden % 256 != 0 || topk == 0 || cap > 65535 || num_experts == 0 ||
      num_experts > kMaxExperts)
    return NVFP4_MOE_ESHAPE;
  const uint64_t pairs = (uint64_t)num_tokens * topk;
  if (pairs > kMaxPairs) return NVFP4_MOE_ESHAPE;
  if (pairs == 0 || cap == 0) return NVFP4_MOE_OK;
  if (x == nullptr || act == nullptr || expert_offsets == nullptr || sorted_pair_ids == nullptr ||
      active_experts == nullptr || active_count == nullptr || !tables_ok(up) || workspace == nullptr)
    return NVFP4_MOE_EINVAL;
  if (workspace_bytes < tc_workspace_bytes(num_tokens, topk, k_hidden, n_inter)) return NVFP4_MOE_EINVAL;
  if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return NVFP4_MOE_EINVAL;
  const int nt = plan_tc_rows(num_tokens, pairs, num_experts, opts ? opts->tiles : 0, kModeUpAct);
  if (nt != 16 && nt != 128 && nt != kTcPairRows && nt != kTcPairRowsSmall && nt != kTcPairRowsWide) return NVFP4_MOE_EINVAL;
  GroupedArgs a{};
  a.src = x;
  a.packed0 = up.packed_ptrs;
  a.scale0 = up.scale_ptrs;
  a.s2_0 = up.scale2;
  a.out = act;
  a.offsets = expert_offsets;
  a.sorted_pair_ids = sorted_pair_ids;
  a.active_experts = active_experts;
  a.active_count = active_count;
  a.N = n_inter;
  a.K = k_hidden;
  a.topk = topk;
  a.num_experts = num_experts;
  a.activation = activation;
  return status_of(launch_tc(kModeUpAct, nt, a, workspace, num_tokens, k_hidden, n_inter, cap, stream));
}

int nvfp4_moe_blend(const float* y, const float* topk_weights, const int32_t* pair_pos,
                    float* out_f32, uint16_t* out_bf16, uint32_t num_tokens, uint32_t topk,
                    uint32_t hidden, cudaStream_t stream) {
  // One grid row per token: at most 65535 tokens per call.
  if (hidden == 0 || hidden % 4 != 0 || topk == 0 || num_tokens > 65535 ||
      (uint64_t)num_tokens * topk > kMaxPairs)
    return NVFP4_MOE_ESHAPE;
  if (num_tokens == 0) return NVFP4_MOE_OK;
  if (y == nullptr || topk_weights == nullptr || pair_pos == nullptr || out_f32 == nullptr)
    return NVFP4_MOE_EINVAL;
  return status_of(launch_blend(y, topk_weights, pair_pos, out_f32, out_bf16, num_tokens, topk,
                                hidden, stream));
}

int nvfp4_moe_forward(const uint16_t* x, const int32_t* topk_ids, const float* topk_weights,
                      nvfp4_expert_tables gate, nvfp4_expert_tables up, nvfp4_expert_tables down,
                      const nvfp4_moe_buffers* b, uint32_t num_tokens, uint32_t topk,
                      uint32_t num_experts, uint32_t hidden, uint32_t inter,
                      const nvfp4_moe_launch_opts* opts, void* workspace, size_t workspace_bytes,
                      cudaStream_t stream) {
  if (b == nullptr) return NVFP4_MOE_EINVAL;
  const uint64_t pairs = (uint64_t)num_tokens * topk;
  if (pairs > kMaxPairs) return NVFP4_MOE_ESHAPE;
  const uint32_t cap = nvfp4_moe_active_cap(num_experts, (uint32_t)pairs);
  int st = nvfp4_moe_route_sort(topk_ids, num_tokens, topk, num_experts, b->expert_offsets,
                                b->sorted_pair_ids, b->pair_pos, b->active_experts, b->active_count,
                                b->status, stream);
  if (st != NVFP4_MOE_OK) return st;
  if (workspace != nullptr) {
    st = nvfp4_moe_gate_up_silu_ws(x, gate, up, b->act, b->expert_offsets, b->sorted_pair_ids,
                                   b->active_experts, b->active_count, inter, hidden, cap, num_tokens,
                                   topk, num_experts, opts, workspace, workspace_bytes, stream);
    if (st != NVFP4_MOE_OK) return st;
    st = nvfp4_moe_down_ws(b->act, down, b->y, b->expert_offsets, b->active_experts, b->active_count,
                           hidden, inter, cap, num_tokens, topk, num_experts, opts, workspace,
                           workspace_bytes, stream);
  } else {
    st = nvfp4_moe_gate_up_silu_ex(x, gate, up, b->act, b->expert_offsets, b->sorted_pair_ids,
                                   b->active_experts, b->active_count, inter, hidden, cap, num_tokens,
                                   topk, opts, stream);
    if (st != NVFP4_MOE_OK) return st;
    st = nvfp4_moe_down_ex(b->act, down, b->y, b->expert_offsets, b->active_experts, b->active_count,
                           hidden, inter, cap, num_tokens, topk, opts, stream);
  }
  if (st != NVFP4_MOE_OK) return st;
  return nvfp4_moe_blend(b->y, topk_weights, b->pair_pos, b->out_f32, b->out_bf16, num_tokens, topk,
                         hidden, stream);
}

int nvfp4_moe_forward_nongated(const uint16_t* x, const int32_t* topk_ids,
                               const float* topk_weights, nvfp4_expert_tables up,
                               nvfp4_expert_tables down, const nvfp4_moe_buffers* b,
                               uint32_t num_tokens, uint32_t topk, uint32_t num_experts,
                               uint32_t hidden, uint32_t inter, int activation,
                               const nvfp4_moe_launch_opts* opts, void* workspace,
                               size_t workspace_bytes, cudaStream_t stream) {
  if (b == nullptr) return NVFP4_MOE_EINVAL;
  if (activation != NVFP4_MOE_ACT_RELU2 && activation != NVFP4_MOE_ACT_SILU) return NVFP4_MOE_EINVAL;
  const uint64_t pairs = (uint64_t)num_tokens * topk;
  if (pairs > kMaxPairs) return NVFP4_MOE_ESHAPE;
  const uint32_t cap = nvfp4_moe_active_cap(num_experts, (uint32_t)pairs);
  int st = nvfp4_moe_route_sort(topk_ids, num_tokens, topk, num_experts, b->expert_offsets,
                                b->sorted_pair_ids, b->pair_pos, b->active_experts, b->active_count,
                                b->status, stream);
  if (st != NVFP4_MOE_OK) return st;
  if (workspace != nullptr) {
    st = nvfp4_moe_up_act_ws(x, up, b->act, b->expert_offsets, b->sorted_pair_ids, b->active_experts,
                             b->active_count, inter, hidden, cap, num_tokens, topk, num_experts,
                             activation, opts, workspace, workspace_bytes, stream);
    if (st != NVFP4_MOE_OK) return st;
    st = nvfp4_moe_down_ws(b->act, down, b->y, b->expert_offsets, b->active_experts, b->active_count,
                           hidden, inter, cap, num_tokens, topk, num_experts, opts, workspace,
                           workspace_bytes, stream);
  } else {
    st = nvfp4_moe_up_act(x, up, b->act, b->expert_offsets, b->sorted_pair_ids, b->active_experts,
                          b->active_count, inter, hidden, cap, num_tokens, topk, activation, opts,
                          stream);
    if (st != NVFP4_MOE_OK) return st;
    st = nvfp4_moe_down_ex(b->act, down, b->y, b->expert_offsets, b->active_experts, b->active_count,
                           hidden, inter, cap, num_tokens, topk, opts, stream);
  }
  if (st != NVFP4_MOE_OK) return st;
  return nvfp4_moe_blend(b->y, topk_weights, b->pair_pos, b->out_f32, b->out_bf16, num_tokens, topk,
                         hidden, stream);
}

int nvfp4_moe_transpose_concat(const uint8_t* const* packed_parts,
                               const uint8_t* const* scale_parts, const uint32_t* part_rows,
                               uint32_t num_parts, uint32_t k, uint32_t group_size,
                               uint32_t stride, uint8_t* packed_out, uint8_t* scale_out,
                               cudaStream_t stream) {
  if (num_parts == 0 || packed_parts == nullptr || scale_parts == nullptr || part_rows == nullptr)
    return NVFP4_MOE_EINVAL;
  if (k == 0 || k % 2 != 0 || group_size == 0 || k % group_size != 0) return NVFP4_MOE_ESHAPE;
  uint64_t n_total = 0;
  for (uint32_t p = 0; p < num_parts; ++p) {
    if (part_rows[p] > 65535u * 32u) return NVFP4_MOE_ESHAPE;
    if (part_rows[p] > 0 && (packed_parts[p] == nullptr || scale_parts[p] == nullptr))
      return NVFP4_MOE_EINVAL;
    n_total += part_rows[p];
  }
  if (stride < n_total) return NVFP4_MOE_ESHAPE;
  if (stride == 0) return NVFP4_MOE_OK;
  if (packed_out == nullptr || scale_out == nullptr) return NVFP4_MOE_EINVAL;
  const uint32_t half_k = k / 2, groups = k / group_size;
  cudaError_t err = cudaSuccess;
  uint64_t off = 0;
  for (uint32_t p = 0; p < num_parts && err == cudaSuccess; ++p) {
    err = launch_transpose_u8_pitched(packed_parts[p], packed_out, part_rows[p], half_k, stride,
                                      off, stream);
    if (err == cudaSuccess)
      err = launch_transpose_u8_pitched(scale_parts[p], scale_out, part_rows[p], groups, stride,
                                        off, stream);
    off += part_rows[p];
  }
  if (err == cudaSuccess && stride > n_total) {
    err = launch_zero_cols(packed_out, half_k, stride, n_total, stream);
    if (err == cudaSuccess) err = launch_zero_cols(scale_out, groups, stride, n_total, stream);
  }
  return status_of(err);
}

uint32_t nvfp4_moe_shared_slots(uint32_t num_tokens, uint32_t shared_rows) {
  if (shared_rows == 0) return 0;
  return (uint32_t)(((uint64_t)num_tokens + shared_rows - 1) / shared_rows);
}

int nvfp4_moe_append_shared(const int32_t* topk_ids, const float* topk_weights,
                            const float* shared_weights, uint32_t num_tokens, uint32_t topk,
                            uint32_t num_experts, uint32_t shared_rows, int32_t* ids_out,
                            float* weights_out, cudaStream_t stream) {
  if (shared_rows == 0) return NVFP4_MOE_EINVAL;
  if (topk == 0 || num_experts == 0 ||
      (uint64_t)num_experts + nvfp4_moe_shared_slots(num_tokens, shared_rows) > kMaxExperts ||
      (uint64_t)num_tokens * (topk + 1) > kMaxPairs)
    return NVFP4_MOE_ESHAPE;
  if (num_tokens == 0) return NVFP4_MOE_OK;
  if (topk_ids == nullptr || topk_weights == nullptr || ids_out == nullptr ||
      weights_out == nullptr)
    return NVFP4_MOE_EINVAL;
  return status_of(launch_append_shared(topk_ids, topk_weights, shared_weights, ids_out,
                                        weights_out, num_tokens, topk, num_experts, shared_rows,
                                        stream));
}

int nvfp4_moe_check_scales(nvfp4_expert_tables t, uint32_t num_experts, uint32_t n, uint32_t k,
                           uint32_t* bad, cudaStream_t stream) {
  if (num_experts == 0 || num_experts > kMaxExperts || n == 0 || k == 0 || k % 256 != 0 ||
      (uint64_t)n * (k / 16) > 0xFFFFFFFFull)
    return NVFP4_MOE_ESHAPE;
  if (t.packed_ptrs == nullptr || t.scale_ptrs == nullptr || bad == nullptr)
    return NVFP4_MOE_EINVAL;
  return status_of(launch_check_scales(t.packed_ptrs, t.scale_ptrs, num_experts,
                                       (uint64_t)n * (k / 16), bad, stream));
}

int nvfp4_moe_shard_nvfp4(const uint8_t* packed, const uint8_t* scale, uint32_t num_matrices,
                          uint32_t n, uint32_t k, int kind, uint32_t rank, uint32_t tp,
                          uint8_t* packed_out, uint8_t* scale_out, cudaStream_t stream) {
  if (kind != NVFP4_MOE_SHARD_COLUMN && kind != NVFP4_MOE_SHARD_ROW) return NVFP4_MOE_EINVAL;
  if (tp == 0 || rank >= tp) return NVFP4_MOE_EINVAL;
  if (k % 16 != 0) return NVFP4_MOE_ESHAPE;
  const uint32_t half_k = k / 2, groups = k / 16;
  if (kind == NVFP4_MOE_SHARD_COLUMN && n % tp != 0) return NVFP4_MOE_ESHAPE;
  if (kind == NVFP4_MOE_SHARD_ROW && (k % tp != 0 || half_k % tp != 0 || groups % tp != 0))
    return NVFP4_MOE_ESHAPE;
  if (num_matrices == 0 || n == 0 || k == 0) return NVFP4_MOE_OK;
  if (packed == nullptr || scale == nullptr || packed_out == nullptr || scale_out == nullptr)
    return NVFP4_MOE_EINVAL;
  const uint64_t mats = num_matrices;
  auto overlaps = [](const void* a, uint64_t na, const void* b, uint64_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
  };
  const uint64_t pin = mats * n * half_k, sin = mats * n * groups;
  const uint64_t pout = pin / tp, sout = sin / tp;
  if (overlaps(packed, pin, packed_out, pout) || overlaps(scale, sin, scale_out, sout) ||
      overlaps(packed, pin, scale_out, sout) || overlaps(scale, sin, packed_out, pout))
    return NVFP4_MOE_EINVAL;
  cudaError_t err;
  if (kind == NVFP4_MOE_SHARD_COLUMN) {
    const uint32_t rows = n / tp;
    err = launch_shard_copy(packed, packed_out, mats, n, half_k, rows, half_k, rank * rows, 0, stream);
    if (err == cudaSuccess)
      err = launch_shard_copy(scale, scale_out, mats, n, groups, rows, groups, rank * rows, 0, stream);
  } else {
    const uint32_t wb = half_k / tp, sb = groups / tp;
    err = launch_shard_copy(packed, packed_out, mats, n, half_k, n, wb, 0, rank * wb, stream);
    if (err == cudaSuccess)
      err = launch_shard_copy(scale, scale_out, mats, n, groups, n, sb, 0, rank * sb, stream);
  }
  return status_of(err);
}

int nvfp4_moe_transpose_u8(const uint8_t* src, uint8_t* dst, uint32_t rows, uint32_t cols,
                           cudaStream_t stream) {
  if (rows == 0 || cols == 0) return NVFP4_MOE_OK;
  if (src == nullptr || dst == nullptr) return NVFP4_MOE_EINVAL;
  if (rows > 65535u * 32u || cols > 2147483647u / 2) return NVFP4_MOE_ESHAPE;
  const uint64_t bytes = (uint64_t)rows * cols;
  const uintptr_t s = reinterpret_cast<uintptr_t>(src), d = reinterpret_cast<uintptr_t>(dst);
  if (s < d + bytes && d < s + bytes) return NVFP4_MOE_EINVAL;  // overlapping buffers
  return status_of(launch_transpose_u8(src, dst, rows, cols, stream));
}

}  // extern "C"
