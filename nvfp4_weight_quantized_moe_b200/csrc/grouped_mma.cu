// Grouped NVFP4 expert projections for decode-shaped batches (few rows per
// expert): gate+up with the fused FP32 SiLU product, down, and the up
// projection of a non-gated expert with its activation.
//
// Operation: metrale_model_layers/layers/ops/nvfp4_moe_grouped.rs,
// `moe_expert_gate_up_act_nvfp4_grouped` and `moe_expert_down_act_nvfp4_grouped`:
// one launch covers every active expert (grid y = slot in the device list of
// active experts, bounded by `cap`), output rows are sorted positions.  The
// non-gated mode serves experts with only up and down projections
// (metrale_model_arch/nemotron_moe/prefill_weights.rs, `prepare_prefill_weights`).
//
// Design (sm_100a).  The weights are the bytes that matter.  Every expert
// weight byte is streamed from HBM once per pass with 16-byte
// ld.global.nc.L1::no_allocate loads, DEPTH chunks ahead of use in registers,
// and decoded in registers with the hardware E2M1 -> f16x2 and E4M3 -> f16x2
// conversions; E2M1 * E4M3 is exact in f16, and weight_scale_2 is applied to
// the FP32 sums.  The decoded weights feed warp-level tensor-core MMAs
// (m16n8k16, f16 in, f32 accumulate) straight from registers, weight rows on the
// MMA's M side and the expert's token rows on its N side (8 per tile, TILES
// tiles in registers), so one pass over an expert's weights serves all its
// rows.  Decoding into shared memory for tcgen05 instead would push four bytes
// of f16 through shared memory per weight byte; at HBM rate that is most of an
// SM's shared-memory bandwidth, which the register path does not spend.
//
// K permutation.  A dot product does not depend on the order of k, so each
// lane's 16-byte loads map onto MMA k-slots directly: in a 256-wide chunk, quad
// lane c owns k in [64c, 64c+64); at MMA step j (0..15) its A k-slots
// {2c, 2c+1} hold k = 64c+4j+{0,1} (one packed byte) and {2c+8, 2c+9} hold
// k = 64c+4j+{2,3} (the next byte).  The activation operand is staged in shared
// memory with the same permutation, so the B fragment of step j is one 8-byte
// load per lane (slot = lane ^ j, conflict-free).
//
// Activation range.  The B operand is f16.  Each (row, 256-k chunk) of x (BF16)
// or act (FP32) is scaled by a power of two 2^-e chosen from its max |value| so
// it fits the f16 range; the chunk's partial sums are multiplied back by 2^e in
// FP32.  act is split into f16 hi + lo (two MMAs) so the down projection keeps
// about 22 bits of the FP32 SiLU product.
//
// Pipeline.  A CTA (4 warps) owns 64 (gate+up) or 128 (down, up+activation) output rows of one
// expert over all of K; with S > 1 its warps split K S ways over 64/S or 128/S
// rows and add their sums through shared memory at the end (one row per
// expert needs that parallelism).  The weights run DEPTH chunks ahead in
// registers.  The activation rows of a group are staged in one of two ways
// (same arithmetic, same result):
//   * whole K, when every 256-k chunk of the group fits in shared memory (K/256
//     x 4 KB per 8-row tile, twice that for down's hi and lo planes): the warps
//     load all (chunk, row) pieces at once, convert them into the MMA layout,
//     meet at one CTA barrier, and then each warp runs over its own chunks
//     with nothing to wait for but its weight loads;
//   * a ring otherwise: per 256-k chunk the rows are copied raw with cp.async
//     two chunks ahead into a ring that only the copying lane reads back,
//     converted one chunk ahead into the MMA layout, and consumed after one
//     CTA barrier per chunk.
// No load is waited on in the same iteration that issues it.

#include "common.cuh"
#include "kernels.h"

namespace nvm {

namespace {

constexpr int kTileChunkBytes = 16 * 32 * 8;  // 16 k-steps x 32 lanes x 8 B

template <int MODE, int S, int TILES>
struct Cfg {
  static constexpr int WARPS = 4;
  static constexpr int THREADS = 32 * WARPS;
  static constexpr int NQ = WARPS / S;
  static constexpr int ROWS_PER_WARP = MODE == kModeGateUp ? 16 : 32;
  static constexpr int ROWS_PER_CTA = NQ * ROWS_PER_WARP;
  static constexpr int PLANES = MODE == kModeDown ? 2 : 1;
  static constexpr int GROUP = 8 * TILES;
  static constexpr int BPE = MODE == kModeDown ? 4 : 2;           // bytes per activation element
  static constexpr int ITEMS = S * GROUP;                           // row-chunks per iteration
  static constexpr int FRAG_BYTES = PLANES * S * TILES * kTileChunkBytes;  // one buffer
  static constexpr int RAW_BYTES = ITEMS * 256 * BPE;                        // one stage
  static constexpr int RED_FLOATS = 2 * TILES * 4;                           // per thread
  static constexpr int RED_BYTES = S > 1 ? THREADS * RED_FLOATS * 4 : 0;
  static constexpr int OFF_RAW = 2 * FRAG_BYTES;
  static constexpr int OFF_XMUL = OFF_RAW + 2 * RAW_BYTES;
  static constexpr int OFF_ROWSRC = OFF_XMUL + 2 * ITEMS * 4;
  static constexpr int OFF_RED = OFF_ROWSRC + GROUP * 4;
  static constexpr int SMEM = OFF_RED + RED_BYTES;
  // Whole-K staging: every 256-k chunk of the group's rows in MMA layout.
  static constexpr int XCH_BYTES = PLANES * TILES * kTileChunkBytes;  // one chunk
};

// Shared-memory layout of whole-K staging for K / 256 = nch chunks: fragments,
// per-(chunk, row) scale factors, row sources, split-K sums.
struct XresLayout {
  int xmul, rowsrc, red, total;
};
NVM_HD XresLayout xres_layout(int planes, int split, int tiles, int nch) {
  XresLayout l;
  l.xmul = nch * planes * tiles * kTileChunkBytes;
  l.rowsrc = l.xmul + nch * 8 * tiles * 4;
  l.red = (l.rowsrc + 8 * tiles * 4 + 15) & ~15;
  l.total = l.red + (split > 1 ? 128 * 2 * tiles * 4 * 4 : 0);
  return l;
}

// Byte offset of the 8-byte unit holding k = 64c + 4j .. +3 of token `r` (0..7)
// inside one token tile's chunk (u = 16c + j).
NVM_DEV int unit_offset(int r, int u) {
  const int c = u >> 4, j = u & 15;
  const int lane = r * 4 + c;
  return j * 256 + ((lane ^ j) << 3);
}

NVM_DEV uint32_t pack_f16x2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

NVM_DEV void cp_async_16(void* smem_dst, const void* gmem_src) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gmem_src) : "memory");
}
NVM_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
NVM_DEV void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// One (row, 256-k chunk) of the activation operand, as the warp holds it (lane
// l: bytes [16 l, 16 l + 16) of each 512-byte half), scaled by 2^-e into the
// f16 range and stored in the MMA layout: `dst` is the row's token tile in the
// chunk, `lo_off` the offset of the lo plane (down), `xm` the row's 2^e slot.
template <int MODE>
NVM_DEV void stage_piece(const uint4 (&v)[MODE == kModeDown ? 2 : 1], uint8_t* dst, int lo_off,
                         int r, float* xm, int lane) {
  float f[8];
  int u0[2];  // first 4-k unit of each 16-byte piece
  if (MODE != kModeDown) {
    const uint32_t wv[4] = {v[0].x, v[0].y, v[0].z, v[0].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = bf16_bits_to_f32(wv[i] & 0xFFFFu);
      f[2 * i + 1] = bf16_bits_to_f32(wv[i] >> 16);
    }
    u0[0] = 2 * lane;  // 8 bf16 = units 2 lane, 2 lane + 1
    u0[1] = 2 * lane + 1;
  } else {
    f[0] = __uint_as_float(v[0].x); f[1] = __uint_as_float(v[0].y);
    f[2] = __uint_as_float(v[0].z); f[3] = __uint_as_float(v[0].w);
    f[4] = __uint_as_float(v[1].x); f[5] = __uint_as_float(v[1].y);
    f[6] = __uint_as_float(v[1].z); f[7] = __uint_as_float(v[1].w);
    u0[0] = lane;
    u0[1] = 32 + lane;
  }
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(f[i]));
  const int ex = f16_range_exponent(warp_max(m));
  const float mul = exp2i(-ex);
  if (MODE != kModeDown) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint2 o;
      o.x = pack_f16x2(f[4 * h] * mul, f[4 * h + 1] * mul);
      o.y = pack_f16x2(f[4 * h + 2] * mul, f[4 * h + 3] * mul);
      *reinterpret_cast<uint2*>(dst + unit_offset(r & 7, u0[h])) = o;
    }
  } else {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float hv[4], lv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float sv = f[4 * h + i] * mul;
        hv[i] = __half2float(__float2half_rn(sv));
        lv[i] = sv - hv[i];
      }
      uint2 oh, ol;
      oh.x = pack_f16x2(hv[0], hv[1]);
      oh.y = pack_f16x2(hv[2], hv[3]);
      ol.x = pack_f16x2(lv[0], lv[1]);
      ol.y = pack_f16x2(lv[2], lv[3]);
      const int off = unit_offset(r & 7, u0[h]);
      *reinterpret_cast<uint2*>(dst + off) = oh;
      *reinterpret_cast<uint2*>(dst + lo_off + off) = ol;
    }
  }
  if (lane == 0) *xm = exp2i(ex);
}

}  // namespace

// One-tile, depth-2 instances (one token row per expert: many CTAs, all of
// which should be resident at once) are held to three CTAs per SM, 168
// registers; the whole-K form would otherwise take more for its longer-lived
// weight buffers.
template <int MODE, int S, int TILES, int DEPTH, bool XR>
__global__ void __launch_bounds__(128, (TILES == 1 && DEPTH == 2) ? 3 : 1)
    grouped_mma_kernel(GroupedArgs a) {
  using C = Cfg<MODE, S, TILES>;
  extern __shared__ __align__(16) uint8_t smem[];
  const int nch = (int)a.K >> 8;
  const XresLayout xl = xres_layout(C::PLANES, S, TILES, nch);
  static_assert(C::XCH_BYTES == C::PLANES * TILES * kTileChunkBytes &&
                    C::RED_BYTES == (S > 1 ? 128 * 2 * TILES * 4 * 4 : 0),
                "whole-K staging layout");
  uint8_t* frag = smem;
  uint8_t* raw = smem + C::OFF_RAW;
  float* xmul = reinterpret_cast<float*>(smem + (XR ? xl.xmul : C::OFF_XMUL));
  int* rowsrc = reinterpret_cast<int*>(smem + (XR ? xl.rowsrc : C::OFF_ROWSRC));
  float* red = reinterpret_cast<float*>(smem + (XR ? xl.red : C::OFF_RED));

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int s = warp % S, q = warp / S;
  const int g = lane >> 2, c = lane & 3;

  // Gate+up (and up+activation) reads the route sort's outputs at once, so it
  // waits for the previous kernel first.  Down starts before gate+up has
  // finished: the route sort's outputs are complete by the time it launches
  // (gate+up lets it launch only after its own wait), and the weights are never
  // written, so down looks up its expert and starts fetching its weights before
  // it waits for act.
  if (MODE != kModeDown) {
    griddep_wait();
    griddep_launch_dependents();
  }
  // The active count and this slot's expert id are read together (the list is
  // padded with -1 past the count), then the expert's offsets and pointers.
  const int slot = blockIdx.y;
  const int count = ld_cg_i32(a.active_count);
  const int e_raw = ld_cg_i32(a.active_experts + slot);
  const int e = (slot < count && e_raw >= 0) ? e_raw : 0;
  const int row_lo = slot < count ? ld_cg_i32(a.offsets + e) : 0;
  const int row_hi = slot < count ? ld_cg_i32(a.offsets + e + 1) : 0;
  const int N = (int)a.N, K = (int)a.K;
  const int n_cta = blockIdx.x * C::ROWS_PER_CTA;
  const int nw = n_cta + q * C::ROWS_PER_WARP;
  const bool warp_on = nw < N;

  const uint8_t* P0 = nullptr;
  const uint8_t* S0 = nullptr;
  if (slot < count) {
    P0 = static_cast<const uint8_t*>(ld_cg_ptr(a.packed0 + e));
    S0 = static_cast<const uint8_t*>(ld_cg_ptr(a.scale0 + e));
  }
  const uint8_t* P1 = P0;
  const uint8_t* S1 = S0;
  if (MODE == kModeGateUp && slot < count) {
    P1 = static_cast<const uint8_t*>(ld_cg_ptr(a.packed1 + e));
    S1 = static_cast<const uint8_t*>(ld_cg_ptr(a.scale1 + e));
  }
  // Down, whose weights do not depend on act, asks L2 for its whole (small)
  // weight slice before it waits for gate+up, so the slice streams from HBM
  // meanwhile.  Gate+up does not: its bulk prefetch queued ahead of the token-row
  // and row-index loads on its critical path (measured: decode M=1 gate+up
  // 15.8 -> 14.3 us without it).
  if (MODE == kModeDown && slot < count && P0 != nullptr && P1 != nullptr && tid < 4) {
    const uint32_t rows = (uint32_t)min(C::ROWS_PER_CTA, N - n_cta);
    const uint32_t nib = rows * (uint32_t)(K >> 1), scl = rows * (uint32_t)(K >> 4);
    if ((MODE == kModeGateUp ? 2u : 1u) * (nib + scl) <= 160u * 1024u) {
      const uint8_t* base = (tid & 2) ? ((tid & 1) ? S1 : S0) : ((tid & 1) ? P1 : P0);
      const uint32_t bytes = (tid & 2) ? scl : nib;
      const size_t row_bytes = (tid & 2) ? (size_t)(K >> 4) : (size_t)(K >> 1);
      if ((tid & 1) == 0) prefetch_l2_bulk(base + (size_t)n_cta * row_bytes, bytes);
    }
  }
  if (MODE == kModeDown) {
    griddep_wait();  // act is complete
    griddep_launch_dependents();
  }
  if (slot >= count) return;
  if (P0 == nullptr || P1 == nullptr) {
    // NULL expert: its rows are zero.
    const int rows = row_hi - row_lo;
    for (int i = tid; i < rows * C::ROWS_PER_CTA; i += C::THREADS) {
      const int n = n_cta + i % C::ROWS_PER_CTA;
      if (n < N) a.out[(size_t)(row_lo + i / C::ROWS_PER_CTA) * N + n] = 0.0f;
    }
    return;
  }
  const float s2a = a.s2_0[e];
  const float s2b = MODE == kModeGateUp ? a.s2_1[e] : s2a;

  const int my_ch0 = s * nch / S;
  const int my_nch = (s + 1) * nch / S - my_ch0;
  const int iters = (nch + S - 1) / S;

  // Per-thread weight row pointers (at this warp's first chunk): tile t, rows g, g + 8.
  const uint8_t* wp[2][2];
  const uint8_t* sp[2][2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int n = nw + (MODE != kModeGateUp ? 16 * t : 0) + g + 8 * r;
      const uint8_t* pb = (MODE == kModeGateUp && t == 1) ? P1 : P0;
      const uint8_t* sb = (MODE == kModeGateUp && t == 1) ? S1 : S0;
      wp[t][r] = pb + (size_t)n * (K >> 1) + (size_t)my_ch0 * 128 + c * 32;
      sp[t][r] = sb + (size_t)n * (K >> 4) + (size_t)my_ch0 * 16 + c * 4;
    }
  }

  uint4 wbuf[DEPTH][2][2][2];
  uint32_t sbuf[DEPTH][2][2];

  auto load_chunk = [&](int cl, uint4 (&w)[2][2][2], uint32_t (&sc)[2][2]) {
#pragma unroll
    for (int t = 0; t < 2; ++t) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const uint8_t* p = wp[t][r] + (size_t)cl * 128;
        w[t][r][0] = ld_stream_v4(p);
        w[t][r][1] = ld_stream_v4(p + 16);
        sc[t][r] = ld_stream_u32(sp[t][r] + (size_t)cl * 16);
      }
    }
  };

  for (int g0 = row_lo; g0 < row_hi; g0 += C::GROUP) {
    const int nrows = min(C::GROUP, row_hi - g0);
    const int ntiles = (nrows + 7) >> 3;
    // Split-K CTAs (short K slices) and whole-K staging put their first DEPTH
    // weight chunks in flight before the token rows are looked up; full-K ring
    // CTAs do it after, which keeps those registers free during the look-up.
    if ((S > 1 || XR) && warp_on) {
#pragma unroll
      for (int d = 0; d < DEPTH; ++d)
        if (d < my_nch) load_chunk(d, wbuf[d], sbuf[d]);
    }
    __syncthreads();  // the previous group is done with shared memory
    if (tid < C::GROUP) {
      int src = -1;
      if (tid < nrows) src = MODE != kModeDown ? a.sorted_pair_ids[g0 + tid] / (int)a.topk : g0 + tid;
      rowsrc[tid] = src;
    }
    __syncthreads();

    // Item i (row-chunk of the iteration) = split i / GROUP, row i % GROUP; warp
    // w copies and converts items w, w + 4, ... of every iteration, so each lane
    // reads back only the raw bytes it copied.
    auto copy_raw = [&](int it, int stage) {
      for (int item = warp; item < C::ITEMS; item += C::WARPS) {
        const int ss = item / C::GROUP, r = item % C::GROUP;
        const int cnt = (ss + 1) * nch / S - ss * nch / S;
        if (r >= nrows || it >= cnt) continue;
        const int kc = (ss * nch / S + it) << 8;
        uint8_t* dst = raw + stage * C::RAW_BYTES + item * 256 * C::BPE;
        const uint8_t* src = static_cast<const uint8_t*>(a.src) + ((size_t)rowsrc[r] * K + kc) * C::BPE;
#pragma unroll
        for (int h = 0; h < C::BPE / 2; ++h) cp_async_16(dst + h * 512 + lane * 16, src + h * 512 + lane * 16);
      }
    };
    auto convert = [&](int it, int stage, int buf) {
      for (int item = warp; item < C::ITEMS; item += C::WARPS) {
        const int ss = item / C::GROUP, r = item % C::GROUP;
        const int cnt = (ss + 1) * nch / S - ss * nch / S;
        if (r >= nrows || it >= cnt) continue;
        const uint8_t* rp = raw + stage * C::RAW_BYTES + item * 256 * C::BPE + lane * 16;
        uint4 v[C::PLANES];
#pragma unroll
        for (int h = 0; h < C::PLANES; ++h) v[h] = *reinterpret_cast<const uint4*>(rp + h * 512);
        stage_piece<MODE>(v, frag + buf * C::FRAG_BYTES + (ss * TILES + (r >> 3)) * kTileChunkBytes,
                          S * TILES * kTileChunkBytes, r, xmul + buf * C::ITEMS + item, lane);
      }
    };

    if (XR) {
      // ---- whole-K staging: every (chunk, row) of the group is loaded (XU per
      // warp in flight at once) and converted, then one barrier; the main loop
      // below then waits on nothing but its own weight loads ----
      constexpr int XU = MODE == kModeDown ? 2 : 4;
      const int nitems = nch * nrows;
      for (int i0 = warp; i0 < nitems; i0 += C::WARPS * XU) {
        uint4 v[XU][C::PLANES];
#pragma unroll
        for (int u = 0; u < XU; ++u) {
          const int item = i0 + u * C::WARPS;
          if (item < nitems) {
            const int ch = item / nrows, r = item - ch * nrows;
            const uint8_t* src = static_cast<const uint8_t*>(a.src) +
                                 ((size_t)rowsrc[r] * K + ((size_t)ch << 8)) * C::BPE + lane * 16;
#pragma unroll
            for (int h = 0; h < C::PLANES; ++h) v[u][h] = ld_stream_v4(src + h * 512);
          }
        }
#pragma unroll
        for (int u = 0; u < XU; ++u) {
          const int item = i0 + u * C::WARPS;
          if (item < nitems) {
            const int ch = item / nrows, r = item - ch * nrows;
            stage_piece<MODE>(v[u], frag + (size_t)ch * C::XCH_BYTES + (r >> 3) * kTileChunkBytes,
                              TILES * kTileChunkBytes, r, xmul + ch * C::GROUP + r, lane);
          }
        }
      }
      __syncthreads();
    } else {
      // ---- prologue: raw chunks 0 and 1 and weights 0..DEPTH-1 in flight ----
      copy_raw(0, 0);
      cp_async_commit();
      if (S == 1 && warp_on) {
#pragma unroll
        for (int d = 0; d < DEPTH; ++d)
          if (d < my_nch) load_chunk(d, wbuf[d], sbuf[d]);
      }
      copy_raw(1, 1);
      cp_async_commit();
      cp_async_wait<1>();
      convert(0, 0, 0);
      __syncthreads();
    }

    float acc[2][TILES][4];
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int u = 0; u < TILES; ++u)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[t][u][i] = 0.0f;

    // Whole-K staging has no CTA-wide step per chunk, so each warp runs over
    // its own chunks only.
    const int nloop = XR ? (warp_on ? my_nch : 0) : iters;
#pragma unroll 1
    for (int base = 0; base < nloop; base += DEPTH) {
#pragma unroll
      for (int d = 0; d < DEPTH; ++d) {
        const int it = base + d;
        if (it < nloop) {
          const int buf = it & 1;
          if (!XR) {
            // Raw chunk it + 2 reuses the stage of chunk it (converted last iteration).
            copy_raw(it + 2, it & 1);
            cp_async_commit();
          }
          if (warp_on && it < my_nch) {
            float pacc[2][TILES][4];
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
              for (int u = 0; u < TILES; ++u)
#pragma unroll
                for (int i = 0; i < 4; ++i) pacc[t][u][i] = 0.0f;

            // Block scales as f16x2 pairs: scl[t][r][0] = (blk0, blk1), [1] = (blk2, blk3).
            uint32_t scl[2][2][2];
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
              for (int r = 0; r < 2; ++r) e4m3x4_to_f16x2x2(sbuf[d][t][r], scl[t][r][0], scl[t][r][1]);

            const uint8_t* xb = XR ? frag + (size_t)(my_ch0 + it) * C::XCH_BYTES
                                   : frag + buf * C::FRAG_BYTES + s * TILES * kTileChunkBytes;
            constexpr int kLoOff = (XR ? 1 : S) * TILES * kTileChunkBytes;
#pragma unroll
            for (int m = 0; m < 8; ++m) {  // word m of each row's 32 bytes: steps j = 2m, 2m+1
              uint32_t dec[2][2][4];
#pragma unroll
              for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                  const uint4 v = wbuf[d][t][r][m >> 2];
                  const uint32_t word = (m & 3) == 0 ? v.x : (m & 3) == 1 ? v.y : (m & 3) == 2 ? v.z : v.w;
                  e2m1x8_to_f16x2x4(word, dec[t][r]);
                }
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int j = 2 * m + h;
                const int blk = j >> 2;  // 16-k block inside the lane's 64 k
                uint32_t A[2][4];
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                  const uint32_t sg = (blk & 1) ? bcast_hi(scl[t][0][blk >> 1]) : bcast_lo(scl[t][0][blk >> 1]);
                  const uint32_t s8 = (blk & 1) ? bcast_hi(scl[t][1][blk >> 1]) : bcast_lo(scl[t][1][blk >> 1]);
                  A[t][0] = hmul2_u32(dec[t][0][2 * h], sg);
                  A[t][1] = hmul2_u32(dec[t][1][2 * h], s8);
                  A[t][2] = hmul2_u32(dec[t][0][2 * h + 1], sg);
                  A[t][3] = hmul2_u32(dec[t][1][2 * h + 1], s8);
                }
                const int boff = j * 256 + ((lane ^ j) << 3);
#pragma unroll
                for (int u = 0; u < TILES; ++u) {
                  if (u < ntiles) {
                    const uint8_t* xt = xb + u * kTileChunkBytes;
                    const uint2 b = *reinterpret_cast<const uint2*>(xt + boff);
                    mma_f16_16816(pacc[0][u], A[0], b.x, b.y);
                    mma_f16_16816(pacc[1][u], A[1], b.x, b.y);
                    if (MODE == kModeDown) {
                      const uint2 bl =
                          *reinterpret_cast<const uint2*>(xt + kLoOff + boff);
                      mma_f16_16816(pacc[0][u], A[0], bl.x, bl.y);
                      mma_f16_16816(pacc[1][u], A[1], bl.x, bl.y);
                    }
                  }
                }
              }
            }
            // The registers of slot d are free again: refill them DEPTH chunks ahead.
            if (it + DEPTH < my_nch) load_chunk(it + DEPTH, wbuf[d], sbuf[d]);
            // Undo the chunk's activation scaling (columns 2c, 2c+1 of each tile).
            const float* xm = XR ? xmul + (my_ch0 + it) * C::GROUP : xmul + buf * C::ITEMS + s * C::GROUP;
#pragma unroll
            for (int u = 0; u < TILES; ++u) {
              if (u < ntiles) {
                const float m0 = xm[u * 8 + 2 * c], m1 = xm[u * 8 + 2 * c + 1];
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                  acc[t][u][0] = fmaf(pacc[t][u][0], m0, acc[t][u][0]);
                  acc[t][u][1] = fmaf(pacc[t][u][1], m1, acc[t][u][1]);
                  acc[t][u][2] = fmaf(pacc[t][u][2], m0, acc[t][u][2]);
                  acc[t][u][3] = fmaf(pacc[t][u][3], m1, acc[t][u][3]);
                }
              }
            }
          }
          if (!XR) {
            // Chunk it + 1: its raw copy was issued two iterations ago.
            cp_async_wait<1>();
            if (it + 1 < iters) convert(it + 1, (it + 1) & 1, buf ^ 1);
            __syncthreads();
          }
        }
      }
    }
    if (!XR) cp_async_wait<0>();

    if (S > 1) {
      // Split-K: warps with s > 0 publish their sums, s == 0 adds them in split order.
      float* mine = red + (size_t)tid * C::RED_FLOATS;
      if (s > 0) {
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int u = 0; u < TILES; ++u)
#pragma unroll
            for (int i = 0; i < 4; ++i) mine[(t * TILES + u) * 4 + i] = acc[t][u][i];
      }
      __syncthreads();
      if (s == 0) {
        for (int ss = 1; ss < S; ++ss) {
          const float* other = red + (size_t)(tid + 32 * ss) * C::RED_FLOATS;
#pragma unroll
          for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int u = 0; u < TILES; ++u)
#pragma unroll
              for (int i = 0; i < 4; ++i) acc[t][u][i] += other[(t * TILES + u) * 4 + i];
        }
      }
    }

    if (s == 0 && warp_on) {
#pragma unroll
      for (int u = 0; u < TILES; ++u) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = u * 8 + 2 * c + (i & 1);
          if (r < nrows) {
            float* orow = a.out + (size_t)(g0 + r) * N;
            const int n = nw + g + 8 * (i >> 1);
            if (MODE == kModeGateUp) {
              const float gv = acc[0][u][i] * s2a;
              const float uv = acc[1][u][i] * s2b;
              orow[n] = silu_f32(gv) * uv;
            } else if (MODE == kModeUpAct) {
              orow[n] = activation_f32(a.activation, acc[0][u][i] * s2a);
              orow[n + 16] = activation_f32(a.activation, acc[1][u][i] * s2a);
            } else {
              orow[n] = acc[0][u][i] * s2a;
              orow[n + 16] = acc[1][u][i] * s2a;
            }
          }
        }
      }
    }
  }
}

template <int MODE, int S, int TILES, int DEPTH, bool XR>
cudaError_t launch_grouped_impl(const GroupedArgs& a, uint32_t cap, cudaStream_t stream) {
  using C = Cfg<MODE, S, TILES>;
  auto kern = grouped_mma_kernel<MODE, S, TILES, DEPTH, XR>;
  const int smem = XR ? xres_layout(C::PLANES, S, TILES, (int)(a.K >> 8)).total : C::SMEM;
  if (smem > kDecodeSmemMax) return cudaErrorInvalidValue;
  cudaError_t err = ensure_dynamic_smem(reinterpret_cast<const void*>(kern), smem);
  if (err != cudaSuccess) return err;
  const dim3 grid((a.N + C::ROWS_PER_CTA - 1) / C::ROWS_PER_CTA, cap);
  return launch_pdl(kern, grid, dim3(C::THREADS), smem, stream, a);
}

cudaError_t launch_grouped(int mode, const DecodePlan& p, const GroupedArgs& a, uint32_t cap,
                           cudaStream_t stream) {
#define NVM_CASE(M, SS, T, D)                                                       \
  if (mode == M && p.split == SS && p.tiles == T && p.depth == D)                   \
    return p.xres ? launch_grouped_impl<M, SS, T, D, true>(a, cap, stream)          \
                  : launch_grouped_impl<M, SS, T, D, false>(a, cap, stream);
  // One row per expert: K split over the CTA's warps.
  NVM_CASE(kModeGateUp, 4, 1, 2)
  NVM_CASE(kModeGateUp, 2, 1, 2)
  NVM_CASE(kModeDown, 4, 1, 2)
  NVM_CASE(kModeDown, 2, 1, 2)
  // Several rows per expert: each warp streams all of K for its rows.
  NVM_CASE(kModeGateUp, 1, 1, 2)
  NVM_CASE(kModeGateUp, 1, 2, 2)
  NVM_CASE(kModeGateUp, 1, 4, 2)
  NVM_CASE(kModeGateUp, 1, 1, 3)
  NVM_CASE(kModeGateUp, 1, 2, 3)
  NVM_CASE(kModeDown, 1, 1, 2)
  NVM_CASE(kModeDown, 1, 2, 2)
  NVM_CASE(kModeDown, 1, 1, 3)
  NVM_CASE(kModeDown, 1, 2, 3)
  // Up+activation: the down kernel's row layout over BF16 token rows.
  NVM_CASE(kModeUpAct, 4, 1, 2)
  NVM_CASE(kModeUpAct, 2, 1, 2)
  NVM_CASE(kModeUpAct, 1, 1, 2)
  NVM_CASE(kModeUpAct, 1, 2, 2)
  NVM_CASE(kModeUpAct, 1, 1, 3)
  NVM_CASE(kModeUpAct, 1, 2, 3)
#undef NVM_CASE
  return cudaErrorInvalidValue;
}

bool grouped_plan_supported(int mode, const DecodePlan& p) {
  if (p.split > 1) return p.tiles == 1 && p.depth == 2 && (p.split == 2 || p.split == 4);
  if (p.split != 1) return false;
  if (p.depth == 2) return p.tiles == 1 || p.tiles == 2 || (mode == kModeGateUp && p.tiles == 4);
  if (p.depth == 3) return p.tiles == 1 || p.tiles == 2;
  return false;
}

int grouped_rows_per_cta(int mode, int split) {
  return (4 / split) * (mode == kModeGateUp ? 16 : 32);
}

int grouped_xres_smem(int mode, const DecodePlan& p, uint32_t k) {
  return xres_layout(mode == kModeDown ? 2 : 1, p.split, p.tiles, (int)(k >> 8)).total;
}

}  // namespace nvm
