// Device helpers shared by the sm_100a kernels of the NVFP4 MoE library.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>

#define NVM_DEV __device__ __forceinline__
#define NVM_HD __host__ __device__ __forceinline__

namespace nvm {

// ---------------------------------------------------------------------------
// Global loads
// ---------------------------------------------------------------------------

// 16-byte read-only streaming load: the weight bytes are read once per pass,
// so they bypass L1.
NVM_DEV uint4 ld_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

NVM_DEV uint32_t ld_stream_u32(const void* p) {
  uint32_t r;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}

// ---------------------------------------------------------------------------
// NVFP4 element decode (hardware conversions of sm_100a)
// ---------------------------------------------------------------------------

// Four bytes of packed E2M1 pairs -> four f16x2.  Byte i of `w` becomes out[i];
// its low nibble lands in the low half (the even k), its high nibble in the
// high half (the odd k).  Every E2M1 value is exact in f16.
NVM_DEV void e2m1x8_to_f16x2x4(uint32_t w, uint32_t out[4]) {
  asm("{\n\t"
      ".reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t"
      "}"
      : "=r"(out[0]), "=r"(out[1]), "=r"(out[2]), "=r"(out[3])
      : "r"(w));
}

// Four E4M3 codes -> two f16x2: lo = (byte0, byte1), hi = (byte2, byte3).
// Every finite E4M3 value is exact in f16.
NVM_DEV void e4m3x4_to_f16x2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t"
      ".reg .b16 l, h;\n\t"
      "mov.b32 {l, h}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, l;\n\t"
      "cvt.rn.f16x2.e4m3x2 %1, h;\n\t"
      "}"
      : "=r"(lo), "=r"(hi)
      : "r"(w));
}

// Broadcast the low / high f16 of a f16x2 to both halves.
NVM_DEV uint32_t bcast_lo(uint32_t v) { return __byte_perm(v, 0, 0x1010); }
NVM_DEV uint32_t bcast_hi(uint32_t v) { return __byte_perm(v, 0, 0x3232); }

NVM_DEV uint32_t hmul2_u32(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// ---------------------------------------------------------------------------
// Warp-level tensor-core MMA: D(16x8, f32) += A(16x16, f16, row) * B(16x8, f16, col)
// ---------------------------------------------------------------------------
NVM_DEV void mma_f16_16816(float d[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------------------
// Small numeric helpers
// ---------------------------------------------------------------------------

NVM_DEV float bf16_bits_to_f32(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

// Power-of-two exponent e such that m * 2^-e lies in [2^14, 2^15) for a finite
// m > 0, clamped to [-110, 110].  Returns 0 for m == 0.  Used to bring a run of
// values into the f16 range without changing their relative precision.
NVM_DEV int f16_range_exponent(float m) {
  if (!(m > 0.0f)) return 0;
  int e = (int)((__float_as_uint(m) >> 23) & 0xFF) - 127 - 14;
  e = e < -110 ? -110 : e;
  e = e > 110 ? 110 : e;
  return e;
}

NVM_DEV float exp2i(int e) { return __uint_as_float((uint32_t)(127 + e) << 23); }

NVM_DEV float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// SiLU(z) = z / (1 + exp(-z)) in FP32 with the hardware exponential and the
// fast divide (relative error ~1e-5 over the range; the IEEE-rounded divide or
// reciprocal takes a slow path whenever exp(-z) overflows, which is common for
// large negative gate values).  For z < -87 the denominator is >= 2^126 and the
// fast divide returns 0, the limit of SiLU there.
NVM_DEV float silu_f32(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

// Activation of a non-gated expert: 1 = squared ReLU, 2 = SiLU (the values of
// nvfp4_moe_activation).
NVM_DEV float activation_f32(int act, float z) {
  if (act == 1) return z > 0.0f ? z * z : 0.0f;
  return silu_f32(z);
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch and L2 prefetch
// ---------------------------------------------------------------------------
// Block until the grids this one depends on have completed and their memory
// is visible (a no-op for a kernel launched without the programmatic
// serialization attribute).
NVM_DEV void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Let the dependent grid start launching (it still waits for this grid's
// completion before it reads what this grid writes).
NVM_DEV void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Ask L2 to fetch `bytes` (multiple of 16) starting at a 16-byte aligned global
// address; nothing is returned to the SM.
NVM_DEV void prefetch_l2_bulk(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Load that is never served from a stale L1 line (cached in L2 only).
NVM_DEV int ld_cg_i32(const int32_t* p) {
  int v;
  asm volatile("ld.global.cg.s32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}
NVM_DEV const void* ld_cg_ptr(const void* const* p) {
  uint64_t v;
  asm volatile("ld.global.cg.u64 %0, [%1];" : "=l"(v) : "l"(p));
  return reinterpret_cast<const void*>(v);
}

}  // namespace nvm
