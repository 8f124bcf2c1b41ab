// Grouped NVFP4 expert projections for decode-shaped batches (few rows per
// expert): gate+up with the fused FP32 SiLU product, and down.
//
// Operation: metrale_model_layers/layers/ops/nvfp4_moe_grouped.rs,
// `moe_expert_gate_up_act_nvfp4_grouped` and `moe_expert_down_act_nvfp4_grouped`:
// one launch covers every active expert (grid y = slot in the device list of
// active experts, bounded by `cap`), output rows are sorted positions.
//
// Design (sm_100a).  The weights are the bytes that matter: every expert
// weight byte is streamed from HBM once per pass with 16-byte
// ld.global.nc.L1::no_allocate loads and decoded in registers with the
// hardware E2M1 -> f16x2 and E4M3 -> f16x2 conversions; the product
// E2M1 * E4M3 is exact in f16, and weight_scale_2 is applied to the FP32 sums.
// The decoded weights feed warp-level tensor-core MMAs (m16n8k16, f16 in,
// f32 accumulate) directly from registers, weight rows on the MMA's M side and
// the expert's token rows on its N side (8 per tile, up to TILES tiles held in
// registers), so one pass over an expert's weights serves all its rows.
// Decoding into shared memory for tcgen05 would write four bytes of f16 per
// weight byte through shared memory; at HBM rate that is most of the SM's
// shared-memory bandwidth, which the register path does not spend.
//
// K permutation.  A dot product does not depend on the order of k, so each
// lane's 16-byte loads are mapped onto MMA k-slots directly: in a 256-wide
// chunk, quad lane c owns k in [64c, 64c+64); at MMA step j (0..15) its A
// k-slots {2c, 2c+1} hold k = 64c+4j+{0,1} (one packed byte) and
// {2c+8, 2c+9} hold k = 64c+4j+{2,3} (the next byte).  The activation operand
// is staged in shared memory with the same permutation, so the B fragment of
// step j is one 8-byte load per lane (slot = lane ^ j, conflict-free).
//
// Activation range.  The B operand is f16.  Each (row, 256-k chunk) of x (BF16)
// or act (FP32) is scaled by a power of two 2^-e chosen from its max |value| so
// it fits the f16 range; the chunk's partial sums are multiplied back by 2^e in
// FP32.  act is split into f16 hi + lo (two MMAs) so the down projection keeps
// about 22 bits of the FP32 SiLU product.
//
// Split-K.  With S > 1 the four warps of a CTA split K S ways over the same
// output rows and add their partial sums through shared memory before the
// epilogue (decode batches with one row per expert need the extra warps).

#include "common.cuh"
#include "kernels.h"

namespace nvm {

namespace {

template <int MODE, int S, int TILES>
struct Cfg {
  static constexpr int WARPS = 4;
  static constexpr int THREADS = 32 * WARPS;
  static constexpr int NQ = WARPS / S;
  static constexpr int ROWS_PER_WARP = MODE == kModeGateUp ? 16 : 32;
  static constexpr int ROWS_PER_CTA = NQ * ROWS_PER_WARP;
  static constexpr int PLANES = MODE == kModeGateUp ? 1 : 2;
  static constexpr int GROUP = 8 * TILES;
  static constexpr int TILE_CHUNK_BYTES = 16 * 32 * 8;  // 16 k-steps x 32 lanes x 8 B
  static constexpr int BUF_BYTES = PLANES * S * TILES * TILE_CHUNK_BYTES;
  static constexpr int XS_BYTES = 2 * BUF_BYTES;
  static constexpr int RED_BYTES = S > 1 ? WARPS * 32 * 2 * TILES * 4 * 4 : 0;
  static constexpr int XS_REGION = XS_BYTES > RED_BYTES ? XS_BYTES : RED_BYTES;
  static constexpr int XMUL_FLOATS = 2 * S * GROUP;
  static constexpr int SMEM = XS_REGION + XMUL_FLOATS * 4 + GROUP * 4;
};

// Byte offset of the 8-byte unit holding k = 64c + 4j .. +3 of token `r` (0..7)
// inside one token tile's chunk.
NVM_DEV int unit_offset(int r, int u) {
  const int c = u >> 4, j = u & 15;
  const int lane = r * 4 + c;
  return j * 256 + ((lane ^ j) << 3);
}

NVM_DEV uint32_t pack_f16x2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

}  // namespace

template <int MODE, int S, int TILES>
__global__ void __launch_bounds__(128) grouped_mma_kernel(GroupedArgs a) {
  using C = Cfg<MODE, S, TILES>;
  extern __shared__ __align__(16) uint8_t smem[];
  uint8_t* xs = smem;
  float* red = reinterpret_cast<float*>(smem);
  float* xmul = reinterpret_cast<float*>(smem + C::XS_REGION);
  int* rowsrc = reinterpret_cast<int*>(xmul + C::XMUL_FLOATS);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int s = warp % S, q = warp / S;
  const int g = lane >> 2, c = lane & 3;

  const int slot = blockIdx.y;
  if (slot >= *a.active_count) return;
  const int e = a.active_experts[slot];
  const int row_lo = a.offsets[e], row_hi = a.offsets[e + 1];
  const int N = (int)a.N, K = (int)a.K;
  const int n_cta = blockIdx.x * C::ROWS_PER_CTA;
  const int nw = n_cta + q * C::ROWS_PER_WARP;
  const bool warp_on = nw < N;

  const uint8_t* P0 = static_cast<const uint8_t*>(a.packed0[e]);
  const uint8_t* S0 = static_cast<const uint8_t*>(a.scale0[e]);
  const uint8_t* P1 = P0;
  const uint8_t* S1 = S0;
  if (MODE == kModeGateUp) {
    P1 = static_cast<const uint8_t*>(a.packed1[e]);
    S1 = static_cast<const uint8_t*>(a.scale1[e]);
  }
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

  const int nch = K >> 8;
  const int my_ch0 = s * nch / S;
  const int my_cnt = (s + 1) * nch / S - my_ch0;
  const int iters = (nch + S - 1) / S;

  // Per-thread weight row pointers: tile t in {0, 1}, rows g and g + 8.
  const uint8_t* wp[2][2];
  const uint8_t* sp[2][2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int n = nw + (MODE == kModeDown ? 16 * t : 0) + g + 8 * r;
      const uint8_t* pb = (MODE == kModeGateUp && t == 1) ? P1 : P0;
      const uint8_t* sb = (MODE == kModeGateUp && t == 1) ? S1 : S0;
      wp[t][r] = pb + (size_t)n * (K >> 1) + c * 32;
      sp[t][r] = sb + (size_t)n * (K >> 4) + c * 4;
    }
  }

  auto load_weights = [&](int chunk, uint4 (&w)[2][2][2], uint32_t (&sc)[2][2]) {
#pragma unroll
    for (int t = 0; t < 2; ++t) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const uint8_t* p = wp[t][r] + (size_t)chunk * 128;
        w[t][r][0] = ld_stream_v4(p);
        w[t][r][1] = ld_stream_v4(p + 16);
        sc[t][r] = ld_stream_u32(sp[t][r] + (size_t)chunk * 16);
      }
    }
  };

  // Stage iteration `it` of every split into buffer `buf`.
  auto stage = [&](int it, int buf, int nrows) {
    for (int item = warp; item < S * C::GROUP; item += C::WARPS) {
      const int ss = item / C::GROUP, r = item % C::GROUP;
      const int ch0 = ss * nch / S, cnt = (ss + 1) * nch / S - ch0;
      if (it >= cnt || r >= nrows) continue;  // warp-uniform
      const int kc = (ch0 + it) << 8;
      const int src = rowsrc[r];
      const int tt = r >> 3, rr = r & 7;
      uint8_t* dst = xs + buf * C::BUF_BYTES + (ss * TILES + tt) * C::TILE_CHUNK_BYTES;
      if (MODE == kModeGateUp) {
        const uint16_t* xrow = static_cast<const uint16_t*>(a.src) + (size_t)src * K + kc;
        const uint4 v = *reinterpret_cast<const uint4*>(xrow + 8 * lane);
        float f[8];
        const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          f[2 * i] = bf16_bits_to_f32(wv[i] & 0xFFFFu);
          f[2 * i + 1] = bf16_bits_to_f32(wv[i] >> 16);
        }
        float m = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(f[i]));
        const int ex = f16_range_exponent(warp_max(m));
        const float mul = exp2i(-ex);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint2 o;
          o.x = pack_f16x2(f[4 * h] * mul, f[4 * h + 1] * mul);
          o.y = pack_f16x2(f[4 * h + 2] * mul, f[4 * h + 3] * mul);
          *reinterpret_cast<uint2*>(dst + unit_offset(rr, 2 * lane + h)) = o;
        }
        if (lane == 0) xmul[(buf * S + ss) * C::GROUP + r] = exp2i(ex);
      } else {
        const float* arow = static_cast<const float*>(a.src) + (size_t)src * K + kc;
        const float4 v0 = *reinterpret_cast<const float4*>(arow + 4 * lane);
        const float4 v1 = *reinterpret_cast<const float4*>(arow + 128 + 4 * lane);
        const float f[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        float m = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(f[i]));
        const int ex = f16_range_exponent(warp_max(m));
        const float mul = exp2i(-ex);
        uint8_t* dst_lo = dst + S * TILES * C::TILE_CHUNK_BYTES;  // second plane
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
          const int off = unit_offset(rr, lane + 32 * h);
          *reinterpret_cast<uint2*>(dst + off) = oh;
          *reinterpret_cast<uint2*>(dst_lo + off) = ol;
        }
        if (lane == 0) xmul[(buf * S + ss) * C::GROUP + r] = exp2i(ex);
      }
    }
  };

  for (int g0 = row_lo; g0 < row_hi; g0 += C::GROUP) {
    const int nrows = min(C::GROUP, row_hi - g0);
    const int ntiles = (nrows + 7) >> 3;
    __syncthreads();  // the previous group is done with shared memory
    if (tid < C::GROUP) {
      int src = -1;
      if (tid < nrows) src = MODE == kModeGateUp ? a.sorted_pair_ids[g0 + tid] / (int)a.topk : g0 + tid;
      rowsrc[tid] = src;
    }
    __syncthreads();

    float acc[2][TILES][4];
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int u = 0; u < TILES; ++u)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[t][u][i] = 0.0f;

    uint4 wcur[2][2][2], wnxt[2][2][2];
    uint32_t scur[2][2], snxt[2][2];
    if (warp_on && my_cnt > 0) load_weights(my_ch0, wnxt, snxt);
    stage(0, 0, nrows);
    __syncthreads();

    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          wcur[t][r][0] = wnxt[t][r][0];
          wcur[t][r][1] = wnxt[t][r][1];
          scur[t][r] = snxt[t][r];
        }
      if (warp_on && it + 1 < my_cnt) load_weights(my_ch0 + it + 1, wnxt, snxt);
      if (it + 1 < iters) stage(it + 1, (it + 1) & 1, nrows);

      if (warp_on && it < my_cnt) {
        const int buf = it & 1;
        const uint8_t* xb = xs + buf * C::BUF_BYTES + s * TILES * C::TILE_CHUNK_BYTES;
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
          for (int r = 0; r < 2; ++r) e4m3x4_to_f16x2x2(scur[t][r], scl[t][r][0], scl[t][r][1]);

#pragma unroll
        for (int m = 0; m < 8; ++m) {  // word m of each row's 32 bytes: steps j = 2m, 2m+1
          uint32_t dec[2][2][4];
#pragma unroll
          for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int r = 0; r < 2; ++r) {
              const uint4 v = wcur[t][r][m >> 2];
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
                const uint2 b = *reinterpret_cast<const uint2*>(xb + u * C::TILE_CHUNK_BYTES + boff);
                mma_f16_16816(pacc[0][u], A[0], b.x, b.y);
                mma_f16_16816(pacc[1][u], A[1], b.x, b.y);
                if (MODE == kModeDown) {
                  const uint2 bl = *reinterpret_cast<const uint2*>(
                      xb + S * TILES * C::TILE_CHUNK_BYTES + u * C::TILE_CHUNK_BYTES + boff);
                  mma_f16_16816(pacc[0][u], A[0], bl.x, bl.y);
                  mma_f16_16816(pacc[1][u], A[1], bl.x, bl.y);
                }
              }
            }
          }
        }
        // Undo the chunk's activation scaling (columns 2c, 2c+1 of each tile).
        const float* xm = xmul + (buf * S + s) * C::GROUP;
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
      __syncthreads();
    }

    if (S > 1) {
      // Split-K: warps with s > 0 publish their sums, s == 0 adds them in split order.
      float* mine = red + (size_t)(warp * 32 + lane) * (2 * TILES * 4);
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
          const float* other = red + (size_t)((warp + ss) * 32 + lane) * (2 * TILES * 4);
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

template <int MODE, int S, int TILES>
cudaError_t launch_grouped_impl(const GroupedArgs& a, uint32_t cap, cudaStream_t stream) {
  using C = Cfg<MODE, S, TILES>;
  auto kern = grouped_mma_kernel<MODE, S, TILES>;
  cudaError_t err = ensure_dynamic_smem(reinterpret_cast<const void*>(kern), C::SMEM);
  if (err != cudaSuccess) return err;
  const dim3 grid((a.N + C::ROWS_PER_CTA - 1) / C::ROWS_PER_CTA, cap);
  kern<<<grid, C::THREADS, C::SMEM, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_grouped(int mode, int split, int tiles, const GroupedArgs& a, uint32_t cap,
                           cudaStream_t stream) {
#define NVM_CASE(M, SS, T)                                     \
  if (mode == M && split == SS && tiles == T)                  \
    return launch_grouped_impl<M, SS, T>(a, cap, stream);
  NVM_CASE(kModeGateUp, 4, 1)
  NVM_CASE(kModeGateUp, 2, 2)
  NVM_CASE(kModeGateUp, 1, 4)
  NVM_CASE(kModeDown, 4, 1)
  NVM_CASE(kModeDown, 2, 2)
  NVM_CASE(kModeDown, 1, 4)
#undef NVM_CASE
  return cudaErrorInvalidValue;
}

int grouped_rows_per_cta(int mode, int split) {
  return (4 / split) * (mode == kModeGateUp ? 16 : 32);
}

}  // namespace nvm
