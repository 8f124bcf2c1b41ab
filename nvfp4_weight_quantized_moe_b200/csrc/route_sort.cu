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
//      lane among them; per-warp counts per expert, scanned over the 32 warps in
//      warp order, give each warp's base, so a pair's position is
//      cursor[e] + warp base + lane rank: ascending pair id within an expert,
//      the same result on every run.
// Out-of-range ids are dropped (pair_pos = -1) and flagged in `status`.
//
// Large batches (more than 4096 pairs, prefill) take route_sort_cluster_kernel:
// a cluster of 8 CTAs, CTA r owning the r-th contiguous eighth of the pairs.
// Each CTA counts its slice; after a cluster barrier every CTA reads the 8
// count arrays through distributed shared memory, so it knows the expert
// offsets and, per expert, how many pairs of the lower slices precede its own;
// then it places its slice with the same passes as above.  Slices are in pair
// order, so the result is the same stable order, bit for bit.
//
// Up to 32 pairs (decode batches of a few tokens) take route_sort_small_kernel
// instead: one warp sorts the keys (expert, pair id) in registers with a
// bitonic network of shuffles (the keys are distinct, so the order is the
// same stable order), lists the active experts with ballots, and the CTA fills
// expert_offsets by binary search over the 32 sorted keys.  Same outputs, bit
// for bit, in about a third of the barrier steps.

#include <climits>

#include <cooperative_groups.h>

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

// Place pairs [lo, hi) in passes of 1024 in pair order: a pair's position is
// cursor[e] + (pairs of expert e in earlier warps of the pass) + (its rank among
// its warp's lanes with expert e); cursor advances by the pass's count.  cnt
// and wc are scratch; the caller has set cursor and synchronised.
NVM_DEV void place_pairs(const int32_t* __restrict__ ids, int lo, int hi, int E, int* cnt, int* cursor,
                         uint16_t* wc, int32_t* __restrict__ sorted, int32_t* __restrict__ pair_pos) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int base = lo; base < hi; base += kSortThreads) {
    for (int i = tid; i < 32 * E; i += kSortThreads) wc[i] = 0;
    const int p = base + tid;
    const int v = p < hi ? ids[p] : -1;
    const bool valid = (unsigned)v < (unsigned)E;
    const unsigned peers = __match_any_sync(0xffffffffu, valid ? v : -1);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    __syncthreads();
    if (valid && rank == 0) wc[warp * E + v] = (uint16_t)__popc(peers);
    __syncthreads();
    if (tid < E) {
      int run = 0;
      for (int w = 0; w < 32; ++w) {
        const int t = wc[w * E + tid];
        wc[w * E + tid] = (uint16_t)run;
        run += t;
      }
      cnt[tid] = run;
    }
    __syncthreads();
    if (valid) {
      const int pos = cursor[v] + wc[warp * E + v] + rank;
      sorted[pos] = p;
      pair_pos[p] = pos;
    } else if (p < hi) {
      pair_pos[p] = -1;
    }
    __syncthreads();
    if (tid < E) cursor[tid] += cnt[tid];
    __syncthreads();
  }
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
  uint16_t* wc = reinterpret_cast<uint16_t*>(sm + 2 * E);   // [32][E]
  __shared__ int tmp[33];
  __shared__ int bad;

  const int tid = threadIdx.x;
  griddep_wait();  // the previous kernel on the stream (e.g. the last blend) is done
  griddep_launch_dependents();
  for (int i = tid; i < E; i += kSortThreads) cnt[i] = 0;
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

  place_pairs(ids, 0, P, E, cnt, cursor, wc, sorted, pair_pos);
}

namespace {
constexpr int kClusterCtas = 8;
constexpr uint32_t kClusterMinPairs = 4097;
}  // namespace

__global__ void __cluster_dims__(kClusterCtas, 1, 1) __launch_bounds__(kSortThreads)
    route_sort_cluster_kernel(const int32_t* __restrict__ ids, int P, int E, int32_t* __restrict__ offsets,
                              int32_t* __restrict__ sorted, int32_t* __restrict__ pair_pos,
                              int32_t* __restrict__ active, int32_t* __restrict__ active_count,
                              int32_t* __restrict__ status) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ int sm[];
  int* cnt = sm;                                            // [E] this slice's counts, then scratch
  int* cursor = sm + E;                                     // [E]
  uint16_t* wc = reinterpret_cast<uint16_t*>(sm + 2 * E);   // [32][E]
  __shared__ int tmp[33];
  __shared__ int bad;

  const int tid = threadIdx.x;
  const int r = (int)cluster.block_rank();
  const int lo = (int)((int64_t)P * r / kClusterCtas), hi = (int)((int64_t)P * (r + 1) / kClusterCtas);
  griddep_wait();
  griddep_launch_dependents();
  for (int i = tid; i < E; i += kSortThreads) cnt[i] = 0;
  if (tid == 0) bad = 0;
  __syncthreads();
  for (int p = lo + tid; p < hi; p += kSortThreads) {
    const int v = ids[p];
    if ((unsigned)v < (unsigned)E) atomicAdd(&cnt[v], 1);
    else bad = 1;
  }
  cluster.sync();  // every slice's counts are complete

  // Expert e: pairs in all slices (total) and in the slices before this one.
  int total = 0, before = 0, any_bad = 0;
  if (tid < E) {
    for (int q = 0; q < kClusterCtas; ++q) {
      const int c = *cluster.map_shared_rank(cnt + tid, q);
      total += c;
      if (q < r) before += c;
    }
  }
  if (tid == 0)
    for (int q = 0; q < kClusterCtas; ++q) any_bad |= *cluster.map_shared_rank(&bad, q);
  cluster.sync();  // no CTA reuses cnt or bad before all have read them

  int kept = 0, nactive = 0;
  const int off = block_exclusive_scan(total, tmp, kept);
  const int arank = block_exclusive_scan(total > 0 ? 1 : 0, tmp, nactive);
  if (tid < E) cursor[tid] = off + before;
  if (r == 0) {
    if (tid < E) {
      offsets[tid] = off;
      if (total > 0) active[arank] = tid;
    }
    if (tid == 0) {
      offsets[E] = kept;
      *active_count = nactive;
      if (status != nullptr) *status = any_bad;
    }
    for (int i = nactive + tid; i < E; i += kSortThreads) active[i] = -1;
  }
  // Positions past the kept pairs hold -1 (split over the CTAs).
  for (int i = kept + (int)(r * kSortThreads) + tid; i < P; i += kClusterCtas * kSortThreads) sorted[i] = -1;
  __syncthreads();
  place_pairs(ids, lo, hi, E, cnt, cursor, wc, sorted, pair_pos);
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
  if (num_pairs >= kClusterMinPairs) {
    cudaError_t err = ensure_dynamic_smem(reinterpret_cast<const void*>(route_sort_cluster_kernel), smem);
    if (err != cudaSuccess) return err;
    return launch_pdl(route_sort_cluster_kernel, dim3(kClusterCtas), dim3(kSortThreads), smem, stream,
                      topk_ids, (int)num_pairs, (int)num_experts, expert_offsets, sorted_pair_ids, pair_pos,
                      active_experts, active_count, status);
  }
  cudaError_t err = ensure_dynamic_smem(reinterpret_cast<const void*>(route_sort_kernel), smem);
  if (err != cudaSuccess) return err;
  return launch_pdl(route_sort_kernel, dim3(1), dim3(kSortThreads), smem, stream, topk_ids,
                    (int)num_pairs, (int)num_experts, expert_offsets, sorted_pair_ids, pair_pos,
                    active_experts, active_count, status);
}

}  // namespace nvm
