// Grouped NVFP4 expert projections on the sm_100a tensor cores (tcgen05),
// gate+up with the fused FP32 SiLU product and down, for any rows per expert.
//
// Operation: metrale_model_layers/layers/ops/nvfp4_moe_grouped.rs,
// `moe_expert_gate_up_act_nvfp4_grouped` and `moe_expert_down_act_nvfp4_grouped`
// (grid y = slot in the device list of active experts, bounded by `cap`; output
// rows are sorted positions).
//
// Design.  A CTA owns 128 weight rows of one expert (for gate+up: 128 gate rows
// and the same 128 up rows) and a group of up to NT of the expert's token rows.
//   * Producer warps 0..7: one weight row per thread.  Each thread streams its
//     row's packed nibbles and block scales with 16-byte loads, DEPTH stages of
//     64 k ahead in registers, decodes them exactly to f16 (hardware
//     E2M1 -> f16x2 and E4M3 -> f16x2 conversions, one f16 multiply), and
//     writes them to its own TMEM lane with tcgen05.st: TMEM is the MMA's A
//     operand, so decoded weights never pass through shared memory.  The same
//     threads gather the group's activation rows (f16, prepared once per call
//     by the pack kernels below) into a K-major shared-memory ring with
//     cp.async.
//   * Warp 8: one thread issues tcgen05.mma.kind::f16 (A = 128 x 16 from TMEM,
//     B = NT x 16 from shared memory, D = FP32 accumulators in TMEM) and
//     tcgen05.commit to the ring's "empty" mbarriers.
//   * Epilogue (warps 0..7): tcgen05.ld of the accumulators; weight_scale_2 and
//     the activation row's power-of-two scale applied in FP32; SiLU(gate)*up in
//     FP32 for gate+up; coalesced FP32 stores by sorted position.
// Every mbarrier wait is bounded: on timeout the kernel sets the device error
// word, skips its remaining work and still frees its TMEM.
//
// Activations.  x is BF16 and act FP32; the MMA takes f16.  pack_x_kernel turns
// each token row into f16 after scaling it by 2^-e (e from the row's max |x|,
// so the row fits the f16 range; the epilogue multiplies by 2^e).
// pack_act_kernel turns each FP32 act row into an f16 hi + lo pair with the same
// row scaling, and down runs two MMAs (hi, lo) into one accumulator, keeping
// about 22 bits of the FP32 product.

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace nvm {

namespace {

constexpr int kStageK = 64;     // k per pipeline stage (4 MMAs of K = 16)
constexpr int kStages = 3;      // ring depth in shared memory / TMEM
constexpr int kProdWarps = 8;
constexpr int kProdThreads = 32 * kProdWarps;
constexpr int kThreads = kProdThreads + 32;  // + MMA warp

constexpr uint32_t pow2_at_least(uint32_t v) {
  uint32_t p = 32;
  while (p < v) p <<= 1;
  return p;
}

// Two A matrices per CTA, 128 rows each, always 64 k (32 TMEM columns) per
// stage: gate+up = (gate rows, up rows) of the same 128 outputs; down = the
// two 128-row halves of 256 outputs, which then share every token tile.
template <int MODE, int NT>
struct TcCfg {
  static constexpr int PLANES = MODE == kModeGateUp ? 1 : 2;  // down: f16 hi + lo
  static constexpr int ROWS_PER_CTA = MODE == kModeGateUp ? 128 : 256;
  static constexpr int B_PLANE_BYTES = NT * kStageK * 2;       // NT rows x 64 k, f16
  static constexpr int B_SLOT_BYTES = PLANES * B_PLANE_BYTES;
  static constexpr int A_COLS = 64;                             // TMEM columns per stage
  static constexpr int D_COLS = 2 * NT;
  static constexpr uint32_t TMEM_COLS = pow2_at_least(D_COLS + kStages * A_COLS);
  static constexpr int DEPTH = 4;                               // weight stages in flight
  static constexpr int OFF_BAR = kStages * B_SLOT_BYTES;        // full[3], empty[3], done
  static constexpr int OFF_TMEM = OFF_BAR + 8 * (2 * kStages + 1);
  static constexpr int OFF_ROWSRC = OFF_TMEM + 16;
  static constexpr int OFF_ABORT = OFF_ROWSRC + NT * 4;
  static constexpr int SMEM_USED = OFF_ABORT + 16;
  // A CTA that takes all 512 TMEM columns also asks for more than half of the
  // SM's shared memory, so a second one is never resident waiting in alloc.
  static constexpr int SMEM = TMEM_COLS == 512 && SMEM_USED < 120 * 1024 ? 120 * 1024 : SMEM_USED;
  static_assert(TMEM_COLS <= 512, "TMEM budget");
};

// Shared-memory layout of one B plane of a stage: no-swizzle K-major core
// matrices (8 rows x 16 B).  Per MMA k-step s (16 k) a [NT/8][2][8][16 B]
// block: LBO (between the two 8-k halves) = 128 B, SBO (between 8-row groups)
// = 256 B.  Unit u (16 bytes, u = 0 .. NT*8-1, in shared-memory order) holds
// k = 16 s + 8 h .. +7 of token row t; consecutive threads take consecutive
// units, so the 16-byte stores hit consecutive banks.
template <int NT>
NVM_DEV void b_unit(int u, int& t, int& piece) {
  const int s = u / (NT * 2);        // NT*32 bytes per k-step = NT*2 units
  const int rem = u % (NT * 2);
  const int grp = rem >> 4, h = (rem >> 3) & 1, r = rem & 7;
  t = grp * 8 + r;
  piece = 2 * s + h;
}

NVM_DEV void cp_async_16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
NVM_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
NVM_DEV void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
NVM_DEV void cp_async_wait_one() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

NVM_DEV uint32_t pack_f16x2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

}  // namespace

// ---------------------------------------------------------------------------
// Activation packing (once per call)
// ---------------------------------------------------------------------------

// One warp per token row: xs[t] = f16(x[t] * 2^-e_t), xexp[t] = 2^e_t.
__global__ void __launch_bounds__(256) pack_x_kernel(const uint16_t* __restrict__ x, int M, int K,
                                                     uint16_t* __restrict__ xs, float* __restrict__ xexp) {
  griddep_wait();
  griddep_launch_dependents();
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= M) return;
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)row * K);
  float m = 0.0f;
  for (int i = lane; i < K / 8; i += 32) {
    const uint4 v = src[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      m = fmaxf(m, fabsf(bf16_bits_to_f32(w[j] & 0xFFFFu)));
      m = fmaxf(m, fabsf(bf16_bits_to_f32(w[j] >> 16)));
    }
  }
  const int e = f16_range_exponent(warp_max(m));
  const float mul = exp2i(-e);
  uint4* dst = reinterpret_cast<uint4*>(xs + (size_t)row * K);
  for (int i = lane; i < K / 8; i += 32) {
    const uint4 v = src[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint4 o;
    uint32_t* op = &o.x;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      op[j] = pack_f16x2(bf16_bits_to_f32(w[j] & 0xFFFFu) * mul, bf16_bits_to_f32(w[j] >> 16) * mul);
    dst[i] = o;
  }
  if (lane == 0) xexp[row] = exp2i(e);
}

// One warp per sorted row r < offsets[E]: hi/lo f16 planes of act[r] * 2^-e_r.
__global__ void __launch_bounds__(256) pack_act_kernel(const float* __restrict__ act, int P, int K,
                                                       const int32_t* __restrict__ kept_rows,
                                                       uint16_t* __restrict__ hi, uint16_t* __restrict__ lo,
                                                       float* __restrict__ aexp) {
  griddep_wait();
  griddep_launch_dependents();
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= P || row >= *kept_rows) return;
  const float4* src = reinterpret_cast<const float4*>(act + (size_t)row * K);
  float m = 0.0f;
  for (int i = lane; i < K / 4; i += 32) {
    const float4 v = src[i];
    m = fmaxf(fmaxf(fmaxf(m, fabsf(v.x)), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
  }
  const int e = f16_range_exponent(warp_max(m));
  const float mul = exp2i(-e);
  uint2* dh = reinterpret_cast<uint2*>(hi + (size_t)row * K);
  uint2* dl = reinterpret_cast<uint2*>(lo + (size_t)row * K);
  for (int i = lane; i < K / 4; i += 32) {
    const float4 v = src[i];
    const float s[4] = {v.x * mul, v.y * mul, v.z * mul, v.w * mul};
    float h[4], l[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      h[j] = __half2float(__float2half_rn(s[j]));
      l[j] = s[j] - h[j];
    }
    dh[i] = make_uint2(pack_f16x2(h[0], h[1]), pack_f16x2(h[2], h[3]));
    dl[i] = make_uint2(pack_f16x2(l[0], l[1]), pack_f16x2(l[2], l[3]));
  }
  if (lane == 0) aexp[row] = exp2i(e);
}

// ---------------------------------------------------------------------------
// The projection kernel
// ---------------------------------------------------------------------------

struct TcArgs {
  const uint16_t* b0;      // gate+up: packed x [M, K]; down: act hi plane [P, K]
  const uint16_t* b1;      // down: act lo plane [P, K]
  const float* bexp;       // gate+up: per token 2^e; down: per sorted row 2^e
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
};

template <int MODE, int NT>
__global__ void __launch_bounds__(kThreads, NT <= 16 ? 2 : 1) grouped_tc_kernel(TcArgs a) {
  using C = TcCfg<MODE, NT>;
  constexpr int DEPTH = C::DEPTH;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t s_base = smem_u32(smem);
  const uint32_t bar_full = s_base + C::OFF_BAR;                 // + 8 * slot
  const uint32_t bar_empty = bar_full + 8 * kStages;             // + 8 * slot
  const uint32_t bar_done = bar_empty + 8 * kStages;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM);
  int* rowsrc = reinterpret_cast<int*>(smem + C::OFF_ROWSRC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_ABORT);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  griddep_wait();
  griddep_launch_dependents();
  const int slot_idx = blockIdx.y;
  if (slot_idx >= *a.active_count) return;
  const int e = a.active_experts[slot_idx];
  const int row_lo = a.offsets[e], row_hi = a.offsets[e + 1];
  const int N = (int)a.N, K = (int)a.K;
  const int n0 = blockIdx.x * C::ROWS_PER_CTA;

  const uint8_t* P0 = static_cast<const uint8_t*>(a.packed0[e]);
  const uint8_t* S0 = static_cast<const uint8_t*>(a.scale0[e]);
  const uint8_t* P1 = P0;
  const uint8_t* S1 = S0;
  if (MODE == kModeGateUp) {
    P1 = static_cast<const uint8_t*>(a.packed1[e]);
    S1 = static_cast<const uint8_t*>(a.scale1[e]);
  }
  if (P0 == nullptr || P1 == nullptr) {  // NULL expert: its rows are zero
    for (int i = tid; i < (row_hi - row_lo) * C::ROWS_PER_CTA; i += kThreads)
      a.out[(size_t)(row_lo + i / C::ROWS_PER_CTA) * N + n0 + i % C::ROWS_PER_CTA] = 0.0f;
    return;
  }
  const float s2a = a.s2_0[e];
  const float s2b = MODE == kModeGateUp ? a.s2_1[e] : s2a;

  // ---- set-up: barriers and TMEM ----
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar_full + 8 * s, kProdWarps);
      mbar_init(bar_empty + 8 * s, 1);
    }
    mbar_init(bar_done, 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == kProdWarps) {
    tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t tmem_d = tmem;                  // D: two NT-column regions
  const uint32_t tmem_a = tmem + C::D_COLS;      // A ring after D

  const int nst = K / kStageK;
  // Producer identity: one weight row per thread.  Warps 0-3 hold matrix 0
  // (gate / rows n0 .. n0+127), warps 4-7 matrix 1 (up / rows n0+128 ..).
  const int prow = (warp & 3) * 32 + lane;   // row within the 128 of its matrix (= TMEM lane)
  const int pmat = warp >> 2;
  const uint8_t* wrow = nullptr;
  const uint8_t* srow = nullptr;
  if (warp < kProdWarps) {
    const uint8_t* pb = (MODE == kModeGateUp && pmat == 1) ? P1 : P0;
    const uint8_t* sb = (MODE == kModeGateUp && pmat == 1) ? S1 : S0;
    const int wn = n0 + (MODE == kModeDown ? 128 * pmat : 0) + prow;
    wrow = pb + (size_t)wn * (K >> 1);
    srow = sb + (size_t)wn * (K >> 4);
  }
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;

  uint32_t it = 0;      // ring iteration, continues across groups
  uint32_t groups = 0;  // groups done (parity of the done barrier)
  for (int g0 = row_lo; g0 < row_hi; g0 += NT) {
    const int nrows = min(NT, row_hi - g0);
    if (tid < NT) {
      int src = -1;
      if (tid < nrows) src = MODE == kModeGateUp ? a.sorted_pair_ids[g0 + tid] / (int)a.topk : g0 + tid;
      rowsrc[tid] = src;
    }
    __syncthreads();

    if (warp < kProdWarps) {
      // ================= producers =================
      uint4 wb[DEPTH][2];
      uint32_t sb[DEPTH];
      // 32 bytes of nibbles (64 k) and 4 scale bytes of the row per stage.
      // L1-allocating loads: the two 16-byte halves share one 32-byte sector and
      // one scale sector serves eight stages.
      auto load = [&](int st, uint4 (&w)[2], uint32_t& sc) {
        const uint8_t* p = wrow + (size_t)st * 32;
        w[0] = __ldg(reinterpret_cast<const uint4*>(p));
        w[1] = __ldg(reinterpret_cast<const uint4*>(p + 16));
        sc = __ldg(reinterpret_cast<const uint32_t*>(srow + (size_t)st * 4));
      };
#pragma unroll
      for (int d = 0; d < DEPTH; ++d)
        if (d < nst) load(d, wb[d], sb[d]);

      // B (this group's token rows, 64 k of stage st) into ring slot `slot`,
      // after the MMAs that last read the slot have completed.
      auto issue_b = [&](int st) {
        const uint32_t slot = (it + st) % kStages;
        const uint32_t round = (it + st) / kStages;
        if (round > 0 && !*abort_flag) {
          if (!mbar_wait(bar_empty + 8 * slot, (round - 1) & 1)) *abort_flag = 1;
        }
        const uint32_t bslot = s_base + slot * C::B_SLOT_BYTES;
        for (int u = tid; u < NT * 8; u += kProdThreads) {
          int t, piece;
          b_unit<NT>(u, t, piece);
          const int off = u * 16;
          if (t < nrows) {
            const size_t eoff = (size_t)rowsrc[t] * K + (size_t)st * kStageK + piece * 8;
            cp_async_16(bslot + off, a.b0 + eoff);
            if constexpr (MODE == kModeDown) cp_async_16(bslot + C::B_PLANE_BYTES + off, a.b1 + eoff);
          } else {
            *reinterpret_cast<uint4*>(smem + slot * C::B_SLOT_BYTES + off) = make_uint4(0, 0, 0, 0);
            if constexpr (MODE == kModeDown)
              *reinterpret_cast<uint4*>(smem + slot * C::B_SLOT_BYTES + C::B_PLANE_BYTES + off) =
                  make_uint4(0, 0, 0, 0);
          }
        }
      };
      issue_b(0);
      cp_async_commit();

      for (int base = 0; base < nst; base += DEPTH) {
#pragma unroll
        for (int d = 0; d < DEPTH; ++d) {
          const int st = base + d;
          if (st < nst) {
            const uint32_t slot = (it + st) % kStages;
            // The next stage's B goes in flight before this stage is decoded;
            // its slot's "empty" wait also frees that slot's A columns.
            if (st + 1 < nst) issue_b(st + 1);
            cp_async_commit();
            // A: decode this thread's row for the stage and write it to TMEM.
            uint32_t sc0, sc1;  // f16x2 (blk0, blk1), (blk2, blk3)
            e4m3x4_to_f16x2x2(sb[d], sc0, sc1);
            uint32_t v[32];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const uint32_t wv[4] = {wb[d][q].x, wb[d][q].y, wb[d][q].z, wb[d][q].w};
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int blk = q * 2 + (i >> 1);  // 8 bytes (16 k) per block
                const uint32_t scl = blk == 0 ? bcast_lo(sc0) : blk == 1 ? bcast_hi(sc0)
                                     : blk == 2 ? bcast_lo(sc1) : bcast_hi(sc1);
                uint32_t dec[4];
                e2m1x8_to_f16x2x4(wv[i], dec);
#pragma unroll
                for (int j = 0; j < 4; ++j) v[q * 16 + i * 4 + j] = hmul2_u32(dec[j], scl);
              }
            }
            tmem_st32(tmem_a + lane_off + slot * C::A_COLS + pmat * 32, v);
            // Refill this register slot DEPTH stages ahead.
            if (st + DEPTH < nst) load(st + DEPTH, wb[d], sb[d]);
            cp_async_wait_one();  // this stage's B has landed (the next one may be in flight)
            fence_proxy_async_smem();
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_full + 8 * slot);
          }
        }
      }
      cp_async_wait_all();
    } else if (lane == 0) {
      // ================= MMA issuer =================
      constexpr uint32_t idesc = idesc_f16_f32(128, NT);
      for (int st = 0; st < nst && !*abort_flag; ++st) {
        const uint32_t slot = (it + st) % kStages;
        const uint32_t round = (it + st) / kStages;
        if (!mbar_wait(bar_full + 8 * slot, round & 1)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t bslot = s_base + slot * C::B_SLOT_BYTES;
        const uint32_t aslot = tmem_a + slot * C::A_COLS;
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const uint32_t acc = (st > 0 || s > 0) ? 1u : 0u;
          const uint64_t bdesc = smem_desc_noswizzle(bslot + s * NT * 32, 128, 256);
          tc_mma_f16_ts(tmem_d, aslot + s * 8, bdesc, idesc, acc);
          tc_mma_f16_ts(tmem_d + NT, aslot + 32 + s * 8, bdesc, idesc, acc);
          if constexpr (MODE == kModeDown) {
            const uint64_t bdesc_lo = smem_desc_noswizzle(bslot + C::B_PLANE_BYTES + s * NT * 32, 128, 256);
            tc_mma_f16_ts(tmem_d, aslot + s * 8, bdesc_lo, idesc, 1u);
            tc_mma_f16_ts(tmem_d + NT, aslot + 32 + s * 8, bdesc_lo, idesc, 1u);
          }
        }
        tc_commit(bar_empty + 8 * slot);
      }
      tc_commit(bar_done);
    }
    it += nst;

    // ================= epilogue =================
    if (warp < kProdWarps) {
      bool ok = !*abort_flag && mbar_wait(bar_done, groups & 1);
      if (!ok) *abort_flag = 1;
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
      // Warps 0-3 take tokens [0, NT/2), warps 4-7 [NT/2, NT), each lane its row.
      const int n = n0 + prow;
      constexpr int HALF = NT / 2;
#pragma unroll 1
      for (int t0 = pmat * HALF; t0 < (pmat + 1) * HALF; t0 += 8) {
        uint32_t d0[8], d1[8];
        tmem_ld8(tmem_d + lane_off + t0, d0);
        tmem_ld8(tmem_d + lane_off + NT + t0, d1);
        tmem_wait_ld();
        if (ok) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int t = t0 + j;
            if (t < nrows) {
              const float xm = a.bexp[MODE == kModeGateUp ? rowsrc[t] : g0 + t];
              float* dst = a.out + (size_t)(g0 + t) * N + n;
              if (MODE == kModeGateUp) {
                const float gv = __uint_as_float(d0[j]) * xm * s2a;
                const float uv = __uint_as_float(d1[j]) * xm * s2b;
                *dst = silu_f32(gv) * uv;
              } else {
                dst[0] = __uint_as_float(d0[j]) * xm * s2a;
                dst[128] = __uint_as_float(d1[j]) * xm * s2a;
              }
            }
          }
        }
      }
      tc_fence_before();
    }
    ++groups;
    __syncthreads();  // accumulators and rowsrc are free for the next group
    tc_fence_after();
  }

  __syncthreads();
  if (warp == kProdWarps) tmem_dealloc(tmem, C::TMEM_COLS);
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

template <int MODE, int NT>
cudaError_t launch_tc_impl(const TcArgs& a, uint32_t cap, cudaStream_t stream) {
  using C = TcCfg<MODE, NT>;
  auto kern = grouped_tc_kernel<MODE, NT>;
  cudaError_t err = ensure_dynamic_smem(reinterpret_cast<const void*>(kern), C::SMEM);
  if (err != cudaSuccess) return err;
  const dim3 grid(a.N / C::ROWS_PER_CTA, cap);
  return launch_pdl(kern, grid, dim3(kThreads), C::SMEM, stream, a);
}

size_t tc_workspace_bytes(uint64_t tokens, uint64_t topk, uint64_t hidden, uint64_t inter) {
  const uint64_t pairs = tokens * topk;
  auto al = [](uint64_t v) { return (v + 255) & ~uint64_t(255); };
  return al(tokens * hidden * 2) + al(tokens * 4) + 2 * al(pairs * inter * 2) + al(pairs * 4);
}

namespace {
struct WsLayout {
  uint16_t* xs;
  float* xexp;
  uint16_t* act_hi;
  uint16_t* act_lo;
  float* aexp;
};
WsLayout ws_layout(void* ws, uint64_t tokens, uint64_t topk, uint64_t hidden, uint64_t inter) {
  const uint64_t pairs = tokens * topk;
  auto al = [](uint64_t v) { return (v + 255) & ~uint64_t(255); };
  uint8_t* p = static_cast<uint8_t*>(ws);
  WsLayout l;
  l.xs = reinterpret_cast<uint16_t*>(p);
  p += al(tokens * hidden * 2);
  l.xexp = reinterpret_cast<float*>(p);
  p += al(tokens * 4);
  l.act_hi = reinterpret_cast<uint16_t*>(p);
  p += al(pairs * inter * 2);
  l.act_lo = reinterpret_cast<uint16_t*>(p);
  p += al(pairs * inter * 2);
  l.aexp = reinterpret_cast<float*>(p);
  return l;
}
}  // namespace

cudaError_t launch_tc(int mode, int nt, const GroupedArgs& g, void* workspace, uint32_t tokens,
                      uint32_t hidden, uint32_t inter, uint32_t cap, cudaStream_t stream) {
  const WsLayout w = ws_layout(workspace, tokens, g.topk, hidden, inter);
  const uint32_t pairs = tokens * g.topk;
  TcArgs a{};
  a.packed0 = g.packed0;
  a.scale0 = g.scale0;
  a.s2_0 = g.s2_0;
  a.packed1 = g.packed1;
  a.scale1 = g.scale1;
  a.s2_1 = g.s2_1;
  a.out = g.out;
  a.offsets = g.offsets;
  a.sorted_pair_ids = g.sorted_pair_ids;
  a.active_experts = g.active_experts;
  a.active_count = g.active_count;
  a.N = g.N;
  a.K = g.K;
  a.topk = g.topk;
  cudaError_t err;
  if (mode == kModeGateUp) {
    err = launch_pdl(pack_x_kernel, dim3((tokens + 7) / 8), dim3(256), 0, stream,
                     static_cast<const uint16_t*>(g.src), (int)tokens, (int)g.K, w.xs, w.xexp);
    if (err != cudaSuccess) return err;
    a.b0 = w.xs;
    a.b1 = w.xs;
    a.bexp = w.xexp;
    if (nt == 16) return launch_tc_impl<kModeGateUp, 16>(a, cap, stream);
    if (nt == 128) return launch_tc_impl<kModeGateUp, 128>(a, cap, stream);
  } else {
    // Rows past offsets[E] (dropped pairs) are not packed: offsets[E] bounds the grid's work.
    err = launch_pdl(pack_act_kernel, dim3((pairs + 7) / 8), dim3(256), 0, stream,
                     static_cast<const float*>(g.src), (int)pairs, (int)g.K, g.offsets + g.num_experts,
                     w.act_hi, w.act_lo, w.aexp);
    if (err != cudaSuccess) return err;
    a.b0 = w.act_hi;
    a.b1 = w.act_lo;
    a.bexp = w.aexp;
    if (nt == 16) return launch_tc_impl<kModeDown, 16>(a, cap, stream);
    if (nt == 128) return launch_tc_impl<kModeDown, 128>(a, cap, stream);
  }
  return cudaErrorInvalidValue;
}

cudaError_t read_device_error(int* value, bool clear) {
  cudaError_t err = cudaMemcpyFromSymbol(value, g_device_error, sizeof(int));
  if (err != cudaSuccess || !clear) return err;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
}

}  // namespace nvm
