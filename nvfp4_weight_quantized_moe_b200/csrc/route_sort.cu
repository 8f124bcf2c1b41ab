// Step 1 of the expert forward: group the routed (token, expert) pairs by
// expert and list the active experts (the grouping `moe_fp8_grouped_sort`
// provides, per the module doc of metrale_model_layers/layers/ops/
// nvfp4_moe_grouped.rs).
//
// One CTA of 1024 threads does a stable counting sort in shared memory:
//   1. per-expert counts (shared-memory atomics; counts are order-free);
//   2. one block-wide exclusive scan gives expert_offsets and, over the
//      "count > 0" flags, the ascending list of active experts;
//   3. the pairs are placed in passes of 1024 in pair order.  Inside a warp,
//      __match_any_sync finds the lanes with the same expert and the rank of a
//      lane among them; per-warp counts per expert (stored [expert][warp], so
//      one warp scans an expert's 32 counts with shuffles) give each warp's
//      base, so a pair's position is cursor[e] + warp base + lane rank:
//      ascending pair id within an expert, the same result on every run.  The
//      next pass's ids are loaded while the current pass is placed.
// Out-of-range ids are dropped (pair_pos = -1) and flagged in `status`.
//
// Up to 32 pairs (decode batches of a few tokens) take route_sort_small_kernel
// instead: one warp sorts the keys (expert, pair id) in registers with a
// bitonic network of shuffles (the keys are distinct, so the order is the
// same stable order), lists the active experts with ballots, and the CTA fills
// expert_offsets by binary search over the 32 sorted keys.  Same outputs, bit
// for bit, in about a third of the barrier steps.

#include <climits>

#include "common.cuh"
#include "kernels.h"

namespace nvm {

namespace {

constexpr int kSortThreads = 1024;

// Block-wide exclusive scan of one int per thread (1024 threads).
NVM_DEV int block_exclusive_scan(int v, int* warp_tmp, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) warp_tmp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int w = warp_tmp[lane];
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += t;
    }
    warp_tmp[lane] = wi - w;  // exclusive warp base
    if (lane == 31) warp_tmp[32] = wi;
  }
  __syncthreads();
  const int ex = incl - v + warp_tmp[warp];
  total = warp_tmp[32];
  __syncthreads();
  return ex;
}

}  // namespace

__global__ void __launch_bounds__(kSortThreads)
    route_sort_kernel(const int32_t* __restrict__ ids, int P, int E, int32_t* __restrict__ offsets,
                      int32_t* __restrict__ sorted, int32_t* __restrict__ pair_pos,
                      int32_t* __restrict__ active, int32_t* __restrict__ active_count,
                      int32_t* __restrict__ status) {
  extern __shared__ int sm[];
  int* cnt = sm;                                            // [E]
  int* cursor = sm + E;                                     // [E]
  uint16_t* wc = reinterpret_cast<uint16_t*>(sm + 2 * E);   // [E][32]
  __shared__ int tmp[33];
  __shared__ int bad;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  griddep_wait();  // the previous kernel on the stream (e.g. the last blend) is done
  griddep_launch_dependents();
  for (int i = tid; i < E; i += kSortThreads) cnt[i] = 0;
  for (int i = tid; i < 32 * E; i += kSortThreads) wc[i] = 0;
  if (tid == 0) bad = 0;
  __syncthreads();
  for (int p = tid; p < P; p += kSortThreads) {
    const int v = ids[p];
    if ((unsigned)v < (unsigned)E) atomicAdd(&cnt[v], 1);
    else bad = 1;
  }
  __syncthreads();

  const int c = tid < E ? cnt[tid] : 0;
  int kept = 0, nactive = 0;
  const int off = block_exclusive_scan(c, tmp, kept);
  const int arank = block_exclusive_scan(c > 0 ? 1 : 0, tmp, nactive);
  if (tid < E) {
    offsets[tid] = off;
    cursor[tid] = off;
    if (c > 0) active[arank] = tid;
  }
  if (tid == 0) {
    offsets[E] = kept;
    *active_count = nactive;
    if (status != nullptr) *status = bad;
  }
  for (int i = nactive + tid; i < E; i += kSortThreads) active[i] = -1;
  for (int i = kept + tid; i < P; i += kSortThreads) sorted[i] = -1;

  int v_next = tid < P ? ids[tid] : -1;
  for (int base = 0; base < P; base += kSortThreads) {
    const int p = base + tid;
    const int v = p < P ? v_next : -1;
    if (base + kSortThreads + tid < P) v_next = ids[base + kSortThreads + tid];
    const bool valid = (unsigned)v < (unsigned)E;
    const unsigned peers = __match_any_sync(0xffffffffu, valid ? v : -1);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    if (valid && rank == 0) wc[v * 32 + warp] = (uint16_t)__popc(peers);
    __syncthreads();
    // Exclusive scan of each expert's 32 per-warp counts, one warp per expert.
    for (int e = warp; e < E; e += 32) {
      const int c = wc[e * 32 + lane];
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      wc[e * 32 + lane] = (uint16_t)(incl - c);
      if (lane == 31) cnt[e] = incl;
    }
    __syncthreads();
    if (valid) {
      const int pos = cursor[v] + wc[v * 32 + warp] + rank;
      sorted[pos] = p;
      pair_pos[p] = pos;
    } else if (p < P) {
      pair_pos[p] = -1;
    }
    __syncthreads();
    // The same warp clears its experts' counts and advances their cursors.
    for (int e = warp; e < E; e += 32) {
      wc[e * 32 + lane] = 0;
      if (lane == 0) cursor[e] += cnt[e];
    }
    __syncthreads();
  }
}

namespace {
constexpr int kSmallThreads = 256;
constexpr int kSmallMax = 32;
}  // namespace

__global__ void __launch_bounds__(kSmallThreads)
    route_sort_small_kernel(const int32_t* __restrict__ ids, int P, int E, int32_t* __restrict__ offsets,
                            int32_t* __restrict__ sorted, int32_t* __restrict__ pair_pos,
                            int32_t* __restrict__ active, int32_t* __restrict__ active_count,
                            int32_t* __restrict__ status) {
  __shared__ int skey[kSmallMax];
  __shared__ int s_kept, s_nact;
  const int tid = threadIdx.x, lane = tid & 31;
  griddep_wait();
  griddep_launch_dependents();
  if (tid < 32) {
    // key = expert * 32 + pair id; dropped pairs sort after every valid one
    // (expert E), lanes without a pair after those.
    int key = INT_MAX;
    bool valid = false;
    if (lane < P) {
      const int v = ids[lane];
      valid = (unsigned)v < (unsigned)E;
      key = ((valid ? v : E) << 5) | lane;
    }
#pragma unroll
    for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
      for (int j = k >> 1; j > 0; j >>= 1) {
        const int other = __shfl_xor_sync(0xffffffffu, key, j);
        const bool ascending = (lane & k) == 0, lower = (lane & j) == 0;
        key = (lower == ascending) ? min(key, other) : max(key, other);
      }
    }
    const int kept = __popc(__ballot_sync(0xffffffffu, valid));
    skey[lane] = key;
    // Sorted position = lane.
    if (lane < P) {
      const int p = key & 31;
      if (lane < kept) {
        sorted[lane] = p;
        pair_pos[p] = lane;
      } else {
        sorted[lane] = -1;
        pair_pos[p] = -1;
      }
    }
    const int prev = __shfl_up_sync(0xffffffffu, key, 1);
    const bool head = lane < kept && (lane == 0 || (prev >> 5) != (key >> 5));
    const unsigned heads = __ballot_sync(0xffffffffu, head);
    if (head) active[__popc(heads & ((1u << lane) - 1u))] = key >> 5;
    if (lane == 0) {
      const int nact = __popc(heads);
      *active_count = nact;
      offsets[E] = kept;
      if (status != nullptr) *status = kept < P ? 1 : 0;
      s_kept = kept;
      s_nact = nact;
    }
  }
  __syncthreads();
  const int kept = s_kept, nact = s_nact;
  for (int e = tid; e < E; e += kSmallThreads) {
    // offsets[e] = number of kept keys with expert < e (keys are ascending).
    int lo = 0, hi = kept;
    const int bound = e << 5;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (skey[mid] < bound) lo = mid + 1;
      else hi = mid;
    }
    offsets[e] = lo;
  }
  for (int i = nact + tid; i < E; i += kSmallThreads) active[i] = -1;
}

cudaError_t launch_route_sort(const int32_t* topk_ids, uint32_t num_pairs, uint32_t num_experts,
                              int32_t* expert_offsets, int32_t* sorted_pair_ids, int32_t* pair_pos,
                              int32_t* active_experts, int32_t* active_count, int32_t* status,
                              cudaStream_t stream) {
  if (num_pairs <= (uint32_t)kSmallMax)
    return launch_pdl(route_sort_small_kernel, dim3(1), dim3(kSmallThreads), 0, stream, topk_ids,
                      (int)num_pairs, (int)num_experts, expert_offsets, sorted_pair_ids, pair_pos,
                      active_experts, active_count, status);
  const int smem = (int)num_experts * (2 * 4 + 32 * 2);
  cudaError_t err = ensure_dynamic_smem(reinterpret_cast<const void*>(route_sort_kernel), smem);
  if (err != cudaSuccess) return err;
  return launch_pdl(route_sort_kernel, dim3(1), dim3(kSortThreads), smem, stream, topk_ids,
                    (int)num_pairs, (int)num_experts, expert_offsets, sorted_pair_ids, pair_pos,
                    active_experts, active_count, status);
}

}  // namespace nvm
