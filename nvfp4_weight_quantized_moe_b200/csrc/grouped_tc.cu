// Grouped NVFP4 expert projections on the sm_100a tensor cores (tcgen05),
// gate+up with the fused FP32 SiLU product, down, and the up projection of a
// non-gated expert with its activation, for any rows per expert.
//
// Operation: metrale_model_layers/layers/ops/nvfp4_moe_grouped.rs,
// `moe_expert_gate_up_act_nvfp4_grouped` and `moe_expert_down_act_nvfp4_grouped`
// (grid y = slot in the device list of active experts, bounded by `cap`; output
// rows are sorted positions).
//
// Design.  A CTA owns 128 weight rows of one expert (for gate+up: 128 gate rows
// and the same 128 up rows; for down and up+activation: 256 rows of the one
// matrix as two halves) and walks the
// expert's sorted token rows in groups of NT.  Every operand moves by TMA:
//   * Warp 9 (one thread) loads weight tiles: per 256 k, for each of the two
//     128-row matrices, 128 rows x 128 bytes of packed nibbles (128-byte
//     swizzle) and 128 rows x 16 scale bytes, into a ring of WS slots.  The
//     tensor maps of each expert's matrices are built on the device from the
//     pointer tables (build_weight_maps_kernel).
//   * Warp 10 (one thread) loads token tiles: per 64 k, NT rows x 128 bytes of
//     f16 activations (128-byte swizzle, the canonical K-major layout of the
//     MMA's B operand), into a ring of SB slots.
//   * Warps 0..7 decode: thread (warp w, lane l) owns weight row
//     32 (w % 4) + l of matrix w / 4.  Per 64 k it reads its row's 32 nibble
//     bytes and 4 scale bytes from shared memory (conflict-free: the swizzle
//     spreads eight consecutive rows over all banks), converts them exactly
//     to f16 (hardware E2M1 -> f16x2 and E4M3 -> f16x2 conversions, one f16
//     multiply) and writes them to its own TMEM lane with tcgen05.st: TMEM is
//     the MMA's A operand, in a ring of SA stages.
//   * Warp 8 (one thread) issues tcgen05.mma.kind::f16 (A = 128 x 16 from
//     TMEM, B = NT x 16 from shared memory, D = FP32 accumulators in TMEM) and
//     one tcgen05.commit per stage to a completion ring that frees both the
//     stage's token slot and its A slot.
//   * Epilogue (warps 0..7, per group): once the next group's first A stages
//     are in TMEM, tcgen05.ld of the accumulators; weight_scale_2 and the
//     activation row's power-of-two scale applied in FP32; for gate+up,
//     SiLU(gate)*up in FP32 into registers and the accumulators handed back to
//     the MMA before the stores; coalesced FP32 stores by sorted position.  The
//     loaders run ahead into the next group meanwhile.
// The roles synchronise through mbarriers only.  Every wait is bounded: on
// timeout the kernel sets the device error word, skips its remaining waits,
// lets its TMA loads in flight land and still frees its TMEM.
//
// Activations.  x is BF16 and act FP32; the MMA takes f16.  The pack kernels
// write one f16 row per sorted position (gate+up gathers the token rows, so a
// group's B rows are contiguous for TMA), each scaled by 2^-e (e from the row's
// max |value|, so the row fits the f16 range; the epilogue multiplies by 2^e).
// act becomes an f16 hi + lo pair with the same row scaling, and down runs two
// MMAs (hi, lo) into one accumulator, keeping about 22 bits of the FP32 value.

#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace nvm {

namespace {

constexpr int kStageK = 64;                     // k per MMA stage (4 MMAs of K = 16)
constexpr int kTileK = 256;                     // k per weight tile load (4 stages)
constexpr int kProdWarps = 8;
constexpr int kMmaWarp = kProdWarps;            // warp 8
constexpr int kWLoadWarp = kProdWarps + 1;      // warp 9
constexpr int kBLoadWarp = kProdWarps + 2;      // warp 10
constexpr int kThreads = 32 * (kProdWarps + 3);
constexpr int kMapsPerExpert = 4;               // packed0, scale0, packed1, scale1
constexpr size_t kMapBytes = (size_t)kMaxExperts * kMapsPerExpert * sizeof(CUtensorMap);

// One weight tile: two matrices x (128 rows x 128 nibble bytes + 128 rows x 16
// scale bytes), every part 1024-byte aligned.
constexpr int kWNibBytes = 128 * 128;
constexpr int kWScaleBytes = 128 * 16;
constexpr int kWSlotBytes = 2 * kWNibBytes + 2 * kWScaleBytes;

constexpr int kSmemPerSM = 228 * 1024;  // shared memory of one SM
constexpr int kSmemReservedPerCta = 1024;

constexpr uint32_t pow2_at_least(uint32_t v) {
  uint32_t p = 32;
  while (p < v) p <<= 1;
  return p;
}

// Rings: weight tiles WS slots (shared memory), token tiles SB slots (shared
// memory), decoded weights SA stages (TMEM).  D takes 2 NT TMEM columns (gate
// and up, or the two row halves of down).
template <int MODE, int NT>
struct TcCfg {
  static constexpr int PLANES = MODE == kModeDown ? 2 : 1;  // down: f16 hi + lo
  static constexpr int ROWS_PER_CTA = MODE == kModeGateUp ? 128 : 256;
  static constexpr int B_PLANE_BYTES = NT * kStageK * 2;       // NT rows x 64 k, f16
  static constexpr int B_SLOT_BYTES = PLANES * B_PLANE_BYTES;
  static constexpr int A_COLS = 64;                             // TMEM columns per stage
  static constexpr int D_COLS = 2 * NT;
  static constexpr int SA = NT <= 16 ? 3 : 4;
  static constexpr int WS = 2;
  static constexpr int SB = (MODE == kModeDown && NT > 16) ? 4 : 8;
  static constexpr uint32_t TMEM_COLS = pow2_at_least(D_COLS + SA * A_COLS);
  static constexpr int OFF_W = 0;
  static constexpr int OFF_B = WS * kWSlotBytes;
  static constexpr int OFF_BAR = OFF_B + SB * B_SLOT_BYTES;
  // MMA completion is committed once per CG stages.  Any tcgen05.commit in the
  // MMA stream costs tensor-pipe time (measured: 64 -> 77 cycles per
  // 128x128x16 MMA), but that cost does not grow with the commit rate, and a
  // commit per stage frees ring slots sooner: measured 2-3 % faster than one
  // per two stages at both tile sizes.  mma_done has SB / CG entries.
  static constexpr int CG = 1;
  static constexpr int NMD = SB / CG;
  // full_w[WS], empty_w[WS], full_b[SB], mma_done[NMD], full_a[SA], done, d_free
  static constexpr int NBAR = 2 * WS + SB + NMD + SA + 2;
  static constexpr int OFF_TMEM = OFF_BAR + 8 * NBAR;
  static constexpr int OFF_ABORT = OFF_TMEM + 16;
  static constexpr int SMEM = OFF_ABORT + 16 + 1024;  // + room to align the base to 1024 B
  static constexpr int CTAS_PER_SM = kSmemPerSM / (SMEM + kSmemReservedPerCta);
  static_assert(B_PLANE_BYTES % 1024 == 0 && kWSlotBytes % 1024 == 0, "TMA tiles stay 1024-byte aligned");
  static_assert(TMEM_COLS <= 512, "TMEM budget");
  static_assert(SB % CG == 0 && (kTileK / kStageK) % CG == 0, "commit groups tile the stages");
  static_assert(SB >= SA, "mma_done also tracks the A ring");
  // Every CTA that shared memory lets share an SM must find its TMEM columns
  // free, or a CTA would wait in tcgen05.alloc.
  static_assert(CTAS_PER_SM >= 1 && CTAS_PER_SM * TMEM_COLS <= 512, "TMEM per SM");
};

NVM_DEV uint32_t pack_f16x2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

}  // namespace

// ---------------------------------------------------------------------------
// Activation packing (once per call)
// ---------------------------------------------------------------------------

// 16-byte loads each lane of the x pack kernels keeps in flight.
constexpr int kPackLoads = 4;

// One warp per token t < M: texp[t] = e, the power of two that brings the
// token's row of x into the f16 range (f16_range_exponent of its max |value|).
// A token's row is packed once per routed slot, so its exponent is found once.
__global__ void __launch_bounds__(256)
    token_exp_kernel(const uint16_t* __restrict__ x, int M, int K, int32_t* __restrict__ texp) {
  griddep_wait();
  griddep_launch_dependents();
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (t >= M) return;
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * K);
  const int n = K / 8;
  float m = 0.0f;
  // kPackLoads 16-byte pieces per lane in flight before any is used.
  for (int i0 = lane; i0 < n; i0 += 32 * kPackLoads) {
    uint4 v[kPackLoads];
#pragma unroll
    for (int u = 0; u < kPackLoads; ++u) {
      const int i = i0 + 32 * u;
      v[u] = i < n ? src[i] : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kPackLoads; ++u) {
      const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        m = fmaxf(m, fabsf(bf16_bits_to_f32(w[j] & 0xFFFFu)));
        m = fmaxf(m, fabsf(bf16_bits_to_f32(w[j] >> 16)));
      }
    }
  }
  const int e = f16_range_exponent(warp_max(m));
  if (lane == 0) texp[t] = e;
}

// One warp per sorted row r < offsets[E]: xs[r] = f16(x[t] * 2^-e), t the
// row's token and e = texp[t]; xexp[r] = 2^e.
__global__ void __launch_bounds__(256)
    pack_x_sorted_kernel(const uint16_t* __restrict__ x, int P, int K, int topk,
                         const int32_t* __restrict__ sorted_pair_ids, const int32_t* __restrict__ kept_rows,
                         const int32_t* __restrict__ texp, uint16_t* __restrict__ xs, float* __restrict__ xexp) {
  griddep_wait();
  griddep_launch_dependents();
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= P || row >= *kept_rows) return;
  const int t = sorted_pair_ids[row] / topk;
  const int e = texp[t];
  const float mul = exp2i(-e);
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * K);
  uint4* dst = reinterpret_cast<uint4*>(xs + (size_t)row * K);
  const int n = K / 8;
  for (int i0 = lane; i0 < n; i0 += 32 * kPackLoads) {
    uint4 v[kPackLoads];
#pragma unroll
    for (int u = 0; u < kPackLoads; ++u) {
      const int i = i0 + 32 * u;
      if (i < n) v[u] = src[i];
    }
#pragma unroll
    for (int u = 0; u < kPackLoads; ++u) {
      const int i = i0 + 32 * u;
      if (i >= n) continue;
      const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
      uint4 o;
      uint32_t* op = &o.x;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        op[j] = pack_f16x2(bf16_bits_to_f32(w[j] & 0xFFFFu) * mul, bf16_bits_to_f32(w[j] >> 16) * mul);
      dst[i] = o;
    }
  }
  if (lane == 0) xexp[row] = exp2i(e);
}

// Single-pass form of pack_act for rows that fit in registers (NV 16-byte
// pieces per lane): the row is read once, its max taken, then converted from
// registers.  (For x the register form needs so many registers at K = 4096
// that it runs one CTA per SM and is slower than the two-pass kernel.)
template <int NV>
__global__ void __launch_bounds__(256)
    pack_act_reg_kernel(const float* __restrict__ act, int P, int K, const int32_t* __restrict__ kept_rows,
                        uint16_t* __restrict__ hi, uint16_t* __restrict__ lo, float* __restrict__ aexp) {
  griddep_wait();
  griddep_launch_dependents();
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= P || row >= *kept_rows) return;
  const float4* src = reinterpret_cast<const float4*>(act + (size_t)row * K);
  const int n16 = K / 4;
  float4 r[NV];
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int idx = lane + 32 * i;
    r[i] = idx < n16 ? src[idx] : make_float4(0.f, 0.f, 0.f, 0.f);
    m = fmaxf(fmaxf(fmaxf(m, fabsf(r[i].x)), fabsf(r[i].y)), fmaxf(fabsf(r[i].z), fabsf(r[i].w)));
  }
  const int e = f16_range_exponent(warp_max(m));
  const float mul = exp2i(-e);
  uint2* dh = reinterpret_cast<uint2*>(hi + (size_t)row * K);
  uint2* dl = reinterpret_cast<uint2*>(lo + (size_t)row * K);
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int idx = lane + 32 * i;
    if (idx < n16) {
      const float sv[4] = {r[i].x * mul, r[i].y * mul, r[i].z * mul, r[i].w * mul};
      float h[4], l[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        h[j] = __half2float(__float2half_rn(sv[j]));
        l[j] = sv[j] - h[j];
      }
      dh[idx] = make_uint2(pack_f16x2(h[0], h[1]), pack_f16x2(h[2], h[3]));
      dl[idx] = make_uint2(pack_f16x2(l[0], l[1]), pack_f16x2(l[2], l[3]));
    }
  }
  if (lane == 0) aexp[row] = exp2i(e);
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
// Per-expert weight tensor maps (once per call)
// ---------------------------------------------------------------------------

// Block e, warp j < nmaps: out[4 e + j] = the template map (nibbles for even
// j, scales for odd j) with its global address replaced by expert e's matrix
// j / 2 (packed0/scale0, packed1/scale1).  A NULL expert gets no maps: the
// projection kernel never reads them.  The map is edited in shared memory and
// copied out with a release fence of the tensor-map proxy; the projection
// kernel acquires it before its first TMA load.
__global__ void __launch_bounds__(128)
    build_weight_maps_kernel(const __grid_constant__ CUtensorMap tmpl_nib,
                             const __grid_constant__ CUtensorMap tmpl_scale,
                             const void* const* __restrict__ p0, const void* const* __restrict__ s0,
                             const void* const* __restrict__ p1, const void* const* __restrict__ s1,
                             int nmaps, CUtensorMap* __restrict__ out) {
  __shared__ alignas(128) CUtensorMap tmp[kMapsPerExpert];
  griddep_wait();  // the kernel that last read `out` has completed
  griddep_launch_dependents();
  const int e = blockIdx.x, w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (w >= nmaps) return;
  if (p0[e] == nullptr || (nmaps == 4 && p1[e] == nullptr)) return;
  const void* src = w == 0 ? p0[e] : w == 1 ? s0[e] : w == 2 ? p1[e] : s1[e];
  const CUtensorMap* t = (w & 1) ? &tmpl_scale : &tmpl_nib;
  if (lane < (int)(sizeof(CUtensorMap) / 16))
    reinterpret_cast<uint4*>(&tmp[w])[lane] = reinterpret_cast<const uint4*>(t)[lane];
  __syncwarp();
  if (lane == 0)
    asm volatile("tensormap.replace.tile.global_address.shared::cta.b1024.b64 [%0], %1;" ::"r"(smem_u32(&tmp[w])),
                 "l"(src)
                 : "memory");
  __syncwarp();
  asm volatile(
      "tensormap.cp_fenceproxy.global.shared::cta.tensormap::generic.release.gpu.sync.aligned [%0], [%1], 128;" ::"l"(
          out + (size_t)e * kMapsPerExpert + w),
      "r"(smem_u32(&tmp[w]))
      : "memory");
}

// ---------------------------------------------------------------------------
// The projection kernel
// ---------------------------------------------------------------------------

struct TcArgs {
  const float* bexp;          // per sorted row: 2^e of its packed activation row
  const CUtensorMap* wmaps;   // [E][4] weight tensor maps
  const void* const* packed0; // NULL-expert test only
  const void* const* packed1;
  const float* s2_0;
  const float* s2_1;
  float* out;
  const int32_t* offsets;
  const int32_t* active_experts;
  const int32_t* active_count;
  uint32_t N, K;
  int activation;             // up+activation: kActRelu2 or kActSilu
  uint32_t cap;               // pair kernel: active slots it may read
};

// Registers: 128-token tiles run one CTA per SM, 16-token tiles two.  The
// register file is handed out to warps in groups of four, so the 11 warps
// count as 12: at most 168 registers per thread for one CTA, 80 for two.
template <int MODE, int NT>
__global__ void __launch_bounds__(kThreads) __maxnreg__(NT <= 16 ? 80 : 168)
    grouped_tc_kernel(const TcArgs a, const __grid_constant__ CUtensorMap tm_b0,
                      const __grid_constant__ CUtensorMap tm_b1) {
  using C = TcCfg<MODE, NT>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t s_base = (raw_base + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (s_base - raw_base);
  const uint32_t full_w = s_base + C::OFF_BAR;     // TMA weight tile landed (+ 8 * slot)
  const uint32_t empty_w = full_w + 8 * C::WS;     // decoders done with the tile
  const uint32_t full_b = empty_w + 8 * C::WS;     // TMA token tile landed
  // mma_done[(ga / CG) % NMD]: the MMAs of stages up to CG (ga / CG) + CG - 1
  // have completed.  It frees B slot ga % SB and A slot ga % SA.
  const uint32_t mma_done = full_b + 8 * C::SB;
  const uint32_t full_a = mma_done + 8 * C::NMD;   // decoded A stage in TMEM
  const uint32_t bar_done = full_a + 8 * C::SA;    // a group's accumulators are final
  const uint32_t bar_dfree = bar_done + 8;         // the epilogue has read them
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM);
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
  if (a.packed0[e] == nullptr || (MODE == kModeGateUp && a.packed1[e] == nullptr)) {
    // NULL expert: its rows are zero
    for (int i = tid; i < (row_hi - row_lo) * C::ROWS_PER_CTA; i += kThreads)
      a.out[(size_t)(row_lo + i / C::ROWS_PER_CTA) * N + n0 + i % C::ROWS_PER_CTA] = 0.0f;
    return;
  }
  const int ngroups = (row_hi - row_lo + NT - 1) / NT;
  if (ngroups <= 0) return;
  const int nst = K / kStageK;   // MMA stages per group
  const int ntile = K / kTileK;  // weight tiles per group

  // ---- set-up: barriers and TMEM ----
  if (tid == 0) {
    for (int s = 0; s < C::WS; ++s) {
      mbar_init(full_w + 8 * s, 1);
      mbar_init(empty_w + 8 * s, kProdWarps);
    }
    for (int s = 0; s < C::SB; ++s) mbar_init(full_b + 8 * s, 1);
    for (int s = 0; s < C::NMD; ++s) mbar_init(mma_done + 8 * s, 1);
    for (int s = 0; s < C::SA; ++s) mbar_init(full_a + 8 * s, kProdWarps);
    mbar_init(bar_done, 1);
    mbar_init(bar_dfree, kProdWarps);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t tmem_d = tmem;              // D: two NT-column regions
  const uint32_t tmem_a = tmem + C::D_COLS;  // A ring after D

  // A wait that gives up (and flags the CTA) once any role has timed out.
  auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
    if (*abort_flag) return false;
    if (mbar_wait(bar, parity)) return true;
    *abort_flag = 1;
    return false;
  };
  // Wait until the MMAs of stage x (and the rest of its commit group) are done.
  auto wait_mma = [&](uint32_t x) -> bool {
    const uint32_t grp = x / C::CG;
    return wait(mma_done + 8 * (grp % C::NMD), (grp / C::NMD) & 1);
  };

  if (warp == kWLoadWarp) {
    // ================= weight tile loader =================
    if (lane == 0) {
      const CUtensorMap* m = a.wmaps + (size_t)e * kMapsPerExpert;
      const CUtensorMap* nib0 = m;
      const CUtensorMap* sc0 = m + 1;
      const CUtensorMap* nib1 = MODE == kModeGateUp ? m + 2 : m;
      const CUtensorMap* sc1 = MODE == kModeGateUp ? m + 3 : m + 1;
      tmap_acquire(nib0);
      tmap_acquire(sc0);
      if (MODE == kModeGateUp) {
        tmap_acquire(nib1);
        tmap_acquire(sc1);
      }
      const int y1 = MODE == kModeGateUp ? n0 : n0 + 128;
      uint32_t issued = 0;
      for (int g = 0; g < ngroups && !*abort_flag; ++g) {
        for (int kt = 0; kt < ntile; ++kt) {
          const uint32_t slot = issued % C::WS, round = issued / C::WS;
          if (round > 0 && !wait(empty_w + 8 * slot, (round - 1) & 1)) break;
          const uint32_t dst = s_base + C::OFF_W + slot * kWSlotBytes;
          const uint32_t bar = full_w + 8 * slot;
          mbar_arrive_expect_tx(bar, kWSlotBytes);
          tma_load_2d(dst, nib0, kt * (kTileK / 2), n0, bar);
          tma_load_2d(dst + kWNibBytes, nib1, kt * (kTileK / 2), y1, bar);
          tma_load_2d(dst + 2 * kWNibBytes, sc0, kt * (kTileK / 16), n0, bar);
          tma_load_2d(dst + 2 * kWNibBytes + kWScaleBytes, sc1, kt * (kTileK / 16), y1, bar);
          ++issued;
        }
      }
      // Let the last tiles land before the CTA can exit (they already have,
      // unless a wait timed out).
      for (uint32_t i = issued > (uint32_t)C::WS ? issued - C::WS : 0; i < issued; ++i)
        mbar_wait(full_w + 8 * (i % C::WS), (i / C::WS) & 1);
    }
  } else if (warp == kBLoadWarp) {
    // ================= token tile loader =================
    if (lane == 0) {
      uint32_t issued = 0;
      for (int g = 0; g < ngroups && !*abort_flag; ++g) {
        const int g0 = row_lo + g * NT;
        for (int st = 0; st < nst; ++st) {
          const uint32_t slot = issued % C::SB, round = issued / C::SB;
          if (round > 0 && !wait_mma(issued - C::SB)) break;
          const uint32_t dst = s_base + C::OFF_B + slot * C::B_SLOT_BYTES;
          const uint32_t bar = full_b + 8 * slot;
          mbar_arrive_expect_tx(bar, C::B_SLOT_BYTES);
          tma_load_2d(dst, &tm_b0, st * kStageK, g0, bar);
          if constexpr (MODE == kModeDown) tma_load_2d(dst + C::B_PLANE_BYTES, &tm_b1, st * kStageK, g0, bar);
          ++issued;
        }
      }
      for (uint32_t i = issued > (uint32_t)C::SB ? issued - C::SB : 0; i < issued; ++i)
        mbar_wait(full_b + 8 * (i % C::SB), (i / C::SB) & 1);
    }
  } else if (warp == kMmaWarp) {
    // ================= MMA issuer =================
    if (lane == 0) {
      for (int g = 0; g < ngroups; ++g) {
        if (g > 0) {
          wait(bar_dfree, (g - 1) & 1);  // the epilogue has read the previous group's D
          tc_fence_after();
        }
        // A group short of NT rows (an expert's last) runs its MMAs with N =
        // its rows rounded up to 16: MMA time scales with N.
        const int rows_g = min(NT, row_hi - (row_lo + g * NT));
        const uint32_t idesc = idesc_f16_f32(128, NT > 16 ? (rows_g + 15) & ~15 : NT);
        for (int st = 0; st < nst; ++st) {
          const uint32_t ga = (uint32_t)(g * nst + st);
          const uint32_t aslot = ga % C::SA, bslot = ga % C::SB;
          if (!wait(full_a + 8 * aslot, (ga / C::SA) & 1)) break;
          if (!wait(full_b + 8 * bslot, (ga / C::SB) & 1)) break;
          tc_fence_after();
          const uint32_t bbase = s_base + C::OFF_B + bslot * C::B_SLOT_BYTES;
          const uint32_t abase = tmem_a + aslot * C::A_COLS;
#pragma unroll
          for (int s = 0; s < 4; ++s) {
            const uint32_t acc = (st > 0 || s > 0) ? 1u : 0u;
            const uint64_t bdesc = smem_desc_sw128(bbase + s * 32);
            tc_mma_f16_ts(tmem_d, abase + s * 8, bdesc, idesc, acc);
            tc_mma_f16_ts(tmem_d + NT, abase + 32 + s * 8, bdesc, idesc, acc);
            if constexpr (MODE == kModeDown) {
              const uint64_t bdesc_lo = smem_desc_sw128(bbase + C::B_PLANE_BYTES + s * 32);
              tc_mma_f16_ts(tmem_d, abase + s * 8, bdesc_lo, idesc, 1u);
              tc_mma_f16_ts(tmem_d + NT, abase + 32 + s * 8, bdesc_lo, idesc, 1u);
            }
          }
          if (ga % C::CG == C::CG - 1) tc_commit(mma_done + 8 * ((ga / C::CG) % C::NMD));
        }
        tc_commit(bar_done);  // also after a timeout, so nothing waits on MMAs in flight
      }
      // No MMA may still run when TMEM is freed.
      mbar_wait(bar_done, (ngroups - 1) & 1);
    }
  } else {
    // ================= decoders (warps 0..7) =================
    const int prow = (warp & 3) * 32 + lane;   // row within the 128 of its matrix (= TMEM lane)
    const int pmat = warp >> 2;                // gate / up, or the two halves of down
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const int swz = prow & 7;
    const float s2a = a.s2_0[e];
    const float s2b = a.s2_1[e];

    // Epilogue.  Warps 0-3 take tokens [0, NT/2), warps 4-7 [NT/2, NT), each
    // lane its output row n0 + prow.
    constexpr int HALF = NT / 2;
    constexpr int CHUNK = HALF < 32 ? HALF : 32;  // tokens per scale load
    constexpr int TL = HALF < 16 ? HALF : 16;     // tokens per TMEM load
    const int tbase = pmat * HALF;
    const int n = n0 + prow;

    // Down (and up+activation): read D and store it directly (through the
    // activation for up+activation), then hand D back to the MMA.
    auto epilogue_down = [&](int g) {
      const int g0 = row_lo + g * NT;
      const int nrows = min(NT, row_hi - g0);
      bool ok = wait(bar_done, g & 1);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
#pragma unroll 1
      for (int c0 = 0; c0 < HALF; c0 += CHUNK) {
        // lane l holds the scale of token tbase + c0 + l
        const int tl = tbase + c0 + lane;
        const float xm_l = (lane < CHUNK && tl < nrows) ? a.bexp[g0 + tl] : 0.0f;
#pragma unroll 1
        for (int tt = 0; tt < CHUNK; tt += TL) {
          uint32_t d0[TL], d1[TL];
#pragma unroll
          for (int h = 0; h < TL; h += 8) {
            tmem_ld8(tmem_d + lane_off + tbase + c0 + tt + h, *reinterpret_cast<uint32_t(*)[8]>(d0 + h));
            tmem_ld8(tmem_d + lane_off + NT + tbase + c0 + tt + h, *reinterpret_cast<uint32_t(*)[8]>(d1 + h));
          }
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < TL; ++j) {
            const int t = tbase + c0 + tt + j;
            const float xm = __shfl_sync(0xffffffffu, xm_l, tt + j);
            if (ok && t < nrows) {
              float* dst = a.out + (size_t)(g0 + t) * N + n;
              const float v0 = __uint_as_float(d0[j]) * xm * s2a;
              const float v1 = __uint_as_float(d1[j]) * xm * s2a;
              if constexpr (MODE == kModeUpAct) {
                dst[0] = activation_f32(a.activation, v0);
                dst[128] = activation_f32(a.activation, v1);
              } else {
                dst[0] = v0;
                dst[128] = v1;
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_dfree);
    };

    // Gate+up: SiLU(gate) * up of every token of this thread goes to registers
    // first and D is handed back at once; the stores follow while the MMA
    // already runs the next group's first stages.
    float res[MODE == kModeGateUp ? HALF : 1];
    int res_g0 = 0, res_nrows = 0;
    bool res_ok = false;
    // Row scales of the group being decoded (xm_cur) and of the one before
    // (xm_prev), loaded when a group starts: lane l holds token tbase + 32 c + l.
    constexpr int NXC = HALF / CHUNK;
    float xm_cur[NXC], xm_prev[NXC];
    auto load_scales = [&](int g) {
      const int g0 = row_lo + g * NT;
      const int nrows = min(NT, row_hi - g0);
#pragma unroll
      for (int c = 0; c < NXC; ++c) {
        xm_prev[c] = xm_cur[c];
        const int tl = tbase + c * CHUNK + lane;
        xm_cur[c] = (lane < CHUNK && tl < nrows) ? a.bexp[g0 + tl] : 0.0f;
      }
    };
    auto epilogue_gate_up = [&](int g, const float (&xm_g)[NXC]) {
      res_g0 = row_lo + g * NT;
      res_nrows = min(NT, row_hi - res_g0);
      bool ok = wait(bar_done, g & 1);
      res_ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
#pragma unroll
      for (int c0 = 0; c0 < HALF; c0 += CHUNK) {
        const float xm_l = xm_g[c0 / CHUNK];
#pragma unroll
        for (int tt = 0; tt < CHUNK; tt += 8) {
          uint32_t d0[8], d1[8];
          tmem_ld8(tmem_d + lane_off + tbase + c0 + tt, d0);
          tmem_ld8(tmem_d + lane_off + NT + tbase + c0 + tt, d1);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float xm = __shfl_sync(0xffffffffu, xm_l, tt + j);
            const float gv = __uint_as_float(d0[j]) * xm * s2a;
            const float uv = __uint_as_float(d1[j]) * xm * s2b;
            res[c0 + tt + j] = silu_f32(gv) * uv;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_dfree);
#pragma unroll
      for (int j = 0; j < HALF; ++j) {
        const int t = tbase + j;
        if (res_ok && t < res_nrows) a.out[(size_t)(res_g0 + t) * N + n] = res[j];
      }
    };

    for (int g = 0; g < ngroups; ++g) {
      if constexpr (MODE == kModeGateUp) load_scales(g);
      for (int kt = 0; kt < ntile; ++kt) {
        const uint32_t gw = (uint32_t)(g * ntile + kt);
        const uint32_t wslot = gw % C::WS;
        wait(full_w + 8 * wslot, (gw / C::WS) & 1);
        const uint8_t* wtile = smem + C::OFF_W + wslot * kWSlotBytes;
        const uint8_t* nrow = wtile + pmat * kWNibBytes + prow * 128;
        const uint4 sc4 = *reinterpret_cast<const uint4*>(wtile + 2 * kWNibBytes + pmat * kWScaleBytes + prow * 16);
        const uint32_t scw[4] = {sc4.x, sc4.y, sc4.z, sc4.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t ga = gw * 4 + j;
          const uint32_t aslot = ga % C::SA, around = ga / C::SA;
          // 32 nibble bytes (64 k) of this row: 16-byte chunks 2j, 2j+1, swizzled.
          const uint4 q0 = *reinterpret_cast<const uint4*>(nrow + (((2 * j) ^ swz) << 4));
          const uint4 q1 = *reinterpret_cast<const uint4*>(nrow + (((2 * j + 1) ^ swz) << 4));
          uint32_t sc0, sc1;  // f16x2 (blk0, blk1), (blk2, blk3)
          e4m3x4_to_f16x2x2(scw[j], sc0, sc1);
          // 32 k per half (16 TMEM columns).  The first half is decoded before
          // waiting for the A slot, so a freed slot mostly waits for stores.
          auto decode_half = [&](int q, uint32_t (&v)[16]) {
            const uint4 qq = q == 0 ? q0 : q1;
            const uint32_t wv[4] = {qq.x, qq.y, qq.z, qq.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int blk = q * 2 + (i >> 1);  // 8 bytes (16 k) per block
              const uint32_t scl = blk == 0 ? bcast_lo(sc0) : blk == 1 ? bcast_hi(sc0)
                                   : blk == 2 ? bcast_lo(sc1) : bcast_hi(sc1);
              uint32_t dec[4];
              e2m1x8_to_f16x2x4(wv[i], dec);
#pragma unroll
              for (int jj = 0; jj < 4; ++jj) v[i * 4 + jj] = hmul2_u32(dec[jj], scl);
            }
          };
          uint32_t v[16];
          decode_half(0, v);
          if (j == 3) {  // the weight tile is consumed: hand the slot back to the loader
            __syncwarp();
            if (lane == 0) mbar_arrive(empty_w + 8 * wslot);
          }
          // The A stage is free once the MMAs of stage ga - SA are done.
          if (around > 0) wait_mma(ga - C::SA);
          tc_fence_after();
          tmem_st16(tmem_a + lane_off + aslot * C::A_COLS + pmat * 32, v);
          decode_half(1, v);
          tmem_st16(tmem_a + lane_off + aslot * C::A_COLS + pmat * 32 + 16, v);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(full_a + 8 * aslot);
          // Once the first SA stages of this group are in TMEM (all the A ring
          // holds before the MMA may start on them), drain the previous group,
          // so the MMA finds its next stages ready the moment D is free.
          if (g > 0 && kt * 4 + j == C::SA - 1) {
            if constexpr (MODE == kModeGateUp) epilogue_gate_up(g - 1, xm_prev);
            else epilogue_down(g - 1);
          }
        }
      }
    }
    if constexpr (MODE == kModeGateUp) {
      epilogue_gate_up(ngroups - 1, xm_cur);
    } else {
      epilogue_down(ngroups - 1);
    }
  }

  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

#include "grouped_tc_pair.cuh"

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

namespace {

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime.
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Row-major 2-D tensor [rows, cols] of `elem`-byte elements at `base`; box
// [box_rows, box_cols]; out-of-range rows read as zero.
cudaError_t make_map_2d(CUtensorMap* map, const void* base, CUtensorMapDataType type, uint32_t elem,
                        uint64_t rows, uint64_t cols, uint32_t box_rows, uint32_t box_cols,
                        CUtensorMapSwizzle swizzle) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
  if (fn == nullptr) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * elem};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estride[2] = {1, 1};
  const CUresult r = fn(map, type, 2, const_cast<void*>(base), dims, strides, box, estride,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int MODE, int NT>
cudaError_t launch_tc_impl(const TcArgs& a, const CUtensorMap& b0, const CUtensorMap& b1, uint32_t cap,
                           cudaStream_t stream) {
  using C = TcCfg<MODE, NT>;
  auto kern = grouped_tc_kernel<MODE, NT>;
  cudaError_t err = ensure_dynamic_smem(reinterpret_cast<const void*>(kern), C::SMEM);
  if (err != cudaSuccess) return err;
  const dim3 grid(a.N / C::ROWS_PER_CTA, cap);
  return launch_pdl(kern, grid, dim3(kThreads), C::SMEM, stream, a, b0, b1);
}

uint64_t al256(uint64_t v) { return (v + 255) & ~uint64_t(255); }

// Workspace regions, in this order: gate+up [xs | xexp | texp | weight maps],
// then down [act hi | act lo | aexp | weight maps].  texp holds one exponent
// per token; it is sized by the pairs (tokens <= pairs), which is all the
// gate+up part's size may depend on.
struct WsLayout {
  uint16_t* xs;
  float* xexp;
  int32_t* texp;
  CUtensorMap* maps_gu;
  uint16_t* act_hi;
  uint16_t* act_lo;
  float* aexp;
  CUtensorMap* maps_down;
};
WsLayout ws_layout(void* ws, uint64_t pairs, uint64_t hidden, uint64_t inter) {
  uint8_t* p = static_cast<uint8_t*>(ws);
  WsLayout l;
  l.xs = reinterpret_cast<uint16_t*>(p);
  p += al256(pairs * hidden * 2);
  l.xexp = reinterpret_cast<float*>(p);
  p += al256(pairs * 4);
  l.texp = reinterpret_cast<int32_t*>(p);
  p += al256(pairs * 4);
  l.maps_gu = reinterpret_cast<CUtensorMap*>(p);
  p += kMapBytes;
  l.act_hi = reinterpret_cast<uint16_t*>(p);
  p += al256(pairs * inter * 2);
  l.act_lo = reinterpret_cast<uint16_t*>(p);
  p += al256(pairs * inter * 2);
  l.aexp = reinterpret_cast<float*>(p);
  p += al256(pairs * 4);
  l.maps_down = reinterpret_cast<CUtensorMap*>(p);
  return l;
}

}  // namespace

size_t tc_gate_up_workspace_bytes(uint64_t pairs, uint64_t hidden) {
  return al256(pairs * hidden * 2) + 2 * al256(pairs * 4) + kMapBytes;
}

size_t tc_workspace_bytes(uint64_t tokens, uint64_t topk, uint64_t hidden, uint64_t inter) {
  const uint64_t pairs = tokens * topk;
  return tc_gate_up_workspace_bytes(pairs, hidden) + 2 * al256(pairs * inter * 2) + al256(pairs * 4) +
         kMapBytes;
}

cudaError_t launch_tc(int mode, int nt, const GroupedArgs& g, void* workspace, uint32_t tokens,
                      uint32_t hidden, uint32_t inter, uint32_t cap, cudaStream_t stream) {
  const uint64_t pairs = (uint64_t)tokens * g.topk;
  const WsLayout w = ws_layout(workspace, pairs, hidden, inter);
  if (g.num_experts == 0 || g.num_experts > kMaxExperts ||
      (nt != 16 && nt != 128 && nt != kTcPairRows && nt != kTcPairRowsSmall && nt != kTcPairRowsWide) ||
      (nt == kTcPairRowsWide && mode == kModeDown))
    return cudaErrorInvalidValue;
  // Pair passes (256, 192 or 32 rows) run the CTA-pair kernel: 64-row weight
  // boxes, token boxes of half a pass.
  const bool pair = nt == kTcPairRows || nt == kTcPairRowsSmall || nt == kTcPairRowsWide;
  TcArgs a{};
  a.packed0 = g.packed0;
  a.packed1 = g.packed1 != nullptr ? g.packed1 : g.packed0;
  a.s2_0 = g.s2_0;
  a.s2_1 = g.s2_1 != nullptr ? g.s2_1 : g.s2_0;
  a.out = g.out;
  a.offsets = g.offsets;
  a.active_experts = g.active_experts;
  a.active_count = g.active_count;
  a.N = g.N;
  a.K = g.K;
  a.activation = g.activation;

  // Templates of the weight maps (address replaced per expert on the device):
  // nibbles [N, K/2] u8 in 128 x 128-byte boxes with 128-byte swizzle, scales
  // [N, K/16] u8 in 128 x 16-byte boxes.
  CUtensorMap t_nib, t_scale, b0, b1;
  const uint32_t w_rows = pair ? kPairWBoxRows : 128;
  cudaError_t err = make_map_2d(&t_nib, workspace, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, g.N, g.K / 2, w_rows,
                                kTileK / 2, CU_TENSOR_MAP_SWIZZLE_128B);
  if (err != cudaSuccess) return err;
  err = make_map_2d(&t_scale, workspace, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, g.N, g.K / 16, w_rows, kTileK / 16,
                    CU_TENSOR_MAP_SWIZZLE_NONE);
  if (err != cudaSuccess) return err;
  const uint32_t box_rows = pair ? (uint32_t)nt / 2 : (uint32_t)nt;

  if (mode == kModeGateUp) {
    err = launch_pdl(token_exp_kernel, dim3((unsigned)((tokens + 7) / 8)), dim3(256), 0, stream,
                     static_cast<const uint16_t*>(g.src), (int)tokens, (int)g.K, w.texp);
    if (err != cudaSuccess) return err;
    err = launch_pdl(pack_x_sorted_kernel, dim3((unsigned)((pairs + 7) / 8)), dim3(256), 0, stream,
                     static_cast<const uint16_t*>(g.src), (int)pairs, (int)g.K, (int)g.topk, g.sorted_pair_ids,
                     g.offsets + g.num_experts, w.texp, w.xs, w.xexp);
    if (err != cudaSuccess) return err;
    err = launch_pdl(build_weight_maps_kernel, dim3(g.num_experts), dim3(128), 0, stream, t_nib, t_scale,
                     g.packed0, g.scale0, g.packed1, g.scale1, 4, w.maps_gu);
    if (err != cudaSuccess) return err;
    err = make_map_2d(&b0, w.xs, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, pairs, g.K, box_rows, kStageK,
                      CU_TENSOR_MAP_SWIZZLE_128B);
    if (err != cudaSuccess) return err;
    b1 = b0;
    a.bexp = w.xexp;
    a.wmaps = w.maps_gu;
    if (nt == kTcPairRowsWide) return launch_tc_pair_impl<kModeGateUp, kTcPairRowsWide>(a, b0, b1, cap, stream);
    if (nt == kTcPairRows) return launch_tc_pair_impl<kModeGateUp, kTcPairRows>(a, b0, b1, cap, stream);
    if (nt == kTcPairRowsSmall) return launch_tc_pair_impl<kModeGateUp, kTcPairRowsSmall>(a, b0, b1, cap, stream);
    if (nt == 16) return launch_tc_impl<kModeGateUp, 16>(a, b0, b1, cap, stream);
    return launch_tc_impl<kModeGateUp, 128>(a, b0, b1, cap, stream);
  }
  if (mode == kModeUpAct) {
    // x packed as for gate+up; one weight table, two row halves per CTA.
    err = launch_pdl(token_exp_kernel, dim3((unsigned)((tokens + 7) / 8)), dim3(256), 0, stream,
                     static_cast<const uint16_t*>(g.src), (int)tokens, (int)g.K, w.texp);
    if (err != cudaSuccess) return err;
    err = launch_pdl(pack_x_sorted_kernel, dim3((unsigned)((pairs + 7) / 8)), dim3(256), 0, stream,
                     static_cast<const uint16_t*>(g.src), (int)pairs, (int)g.K, (int)g.topk, g.sorted_pair_ids,
                     g.offsets + g.num_experts, w.texp, w.xs, w.xexp);
    if (err != cudaSuccess) return err;
    err = launch_pdl(build_weight_maps_kernel, dim3(g.num_experts), dim3(128), 0, stream, t_nib, t_scale,
                     g.packed0, g.scale0, g.packed0, g.scale0, 2, w.maps_gu);
    if (err != cudaSuccess) return err;
    err = make_map_2d(&b0, w.xs, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, pairs, g.K, box_rows, kStageK,
                      CU_TENSOR_MAP_SWIZZLE_128B);
    if (err != cudaSuccess) return err;
    b1 = b0;
    a.bexp = w.xexp;
    a.wmaps = w.maps_gu;
    if (nt == kTcPairRowsWide) return launch_tc_pair_impl<kModeUpAct, kTcPairRowsWide>(a, b0, b1, cap, stream);
    if (nt == kTcPairRows) return launch_tc_pair_impl<kModeUpAct, kTcPairRows>(a, b0, b1, cap, stream);
    if (nt == kTcPairRowsSmall) return launch_tc_pair_impl<kModeUpAct, kTcPairRowsSmall>(a, b0, b1, cap, stream);
    if (nt == 16) return launch_tc_impl<kModeUpAct, 16>(a, b0, b1, cap, stream);
    return launch_tc_impl<kModeUpAct, 128>(a, b0, b1, cap, stream);
  }
  // Rows past offsets[E] (dropped pairs) are not packed: offsets[E] bounds the grid's work.
  {
    // Rows of up to 2048 floats go through registers in one pass.
    const uint32_t pieces = (g.K / 4 + 31) / 32;
    auto kern = pieces <= 8 ? pack_act_reg_kernel<8>
                : pieces <= 16 ? pack_act_reg_kernel<16> : pack_act_kernel;
    err = launch_pdl(kern, dim3((unsigned)((pairs + 7) / 8)), dim3(256), 0, stream,
                     static_cast<const float*>(g.src), (int)pairs, (int)g.K, g.offsets + g.num_experts,
                     w.act_hi, w.act_lo, w.aexp);
  }
  if (err != cudaSuccess) return err;
  err = launch_pdl(build_weight_maps_kernel, dim3(g.num_experts), dim3(128), 0, stream, t_nib, t_scale,
                   g.packed0, g.scale0, g.packed0, g.scale0, 2, w.maps_down);
  if (err != cudaSuccess) return err;
  err = make_map_2d(&b0, w.act_hi, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, pairs, g.K, box_rows, kStageK,
                    CU_TENSOR_MAP_SWIZZLE_128B);
  if (err != cudaSuccess) return err;
  err = make_map_2d(&b1, w.act_lo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, pairs, g.K, box_rows, kStageK,
                    CU_TENSOR_MAP_SWIZZLE_128B);
  if (err != cudaSuccess) return err;
  a.bexp = w.aexp;
  a.wmaps = w.maps_down;
  if (nt == kTcPairRows) return launch_tc_pair_impl<kModeDown, kTcPairRows>(a, b0, b1, cap, stream);
  if (nt == kTcPairRowsSmall) return launch_tc_pair_impl<kModeDown, kTcPairRowsSmall>(a, b0, b1, cap, stream);
  if (nt == 16) return launch_tc_impl<kModeDown, 16>(a, b0, b1, cap, stream);
  return launch_tc_impl<kModeDown, 128>(a, b0, b1, cap, stream);
}

// One thread initialises an mbarrier that expects one arrival, arrives on it
// only if `arrive` is set, and waits for its phase with a limit of
// `cycle_limit` SM clock cycles: the library's bounded wait, which on timeout
// sets the device error word and returns.
__global__ void wait_selftest_kernel(uint32_t cycle_limit, int arrive) {
  __shared__ alignas(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  const uint32_t b = smem_u32(&bar);
  mbar_init(b, 1);
  mbar_init_fence();
  if (arrive) mbar_arrive(b);
  mbar_wait(b, 0, (long long)cycle_limit);
}

cudaError_t launch_wait_selftest(uint32_t cycle_limit, int arrive, cudaStream_t stream) {
  wait_selftest_kernel<<<1, 32, 0, stream>>>(cycle_limit, arrive);
  return cudaGetLastError();
}

cudaError_t read_device_error(int* value, bool clear) {
  cudaError_t err = cudaMemcpyFromSymbol(value, g_device_error, sizeof(int));
  if (err != cudaSuccess || !clear) return err;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
}

}  // namespace nvm
