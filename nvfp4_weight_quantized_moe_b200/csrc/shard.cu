// Tensor-parallel shard of NVFP4 weights (load time).
//
// metrale_model_arch/tp_shard/quant_shard.rs, `shard_quantized_nvfp4`:
// column-parallel keeps rank's N/tp rows of the packed [N, K/2] and scale
// [N, K/16] tensors; row-parallel keeps, in every row, the rank's K/2/tp packed
// bytes and K/16/tp scale bytes.  Both are one strided 2-D byte copy per
// tensor, here over a stack of matrices in one launch: 16-, 4- or 1-byte
// vectors, whichever the offsets, widths and pointers allow.

#include "common.cuh"
#include "kernels.h"

namespace nvm {

namespace {
constexpr int kShardThreads = 256;

template <int V>
struct Vec;
template <>
struct Vec<16> { using T = uint4; };
template <>
struct Vec<4> { using T = uint32_t; };
template <>
struct Vec<1> { using T = uint8_t; };
}  // namespace

// dst[m][r][c] = src[m][r + row_off][c + col_off]; rows_out x cols_out bytes per
// matrix out of rows_src x cols_src.
template <int V>
__global__ void __launch_bounds__(kShardThreads)
    shard_copy_kernel(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst, uint64_t mats,
                      uint32_t rows_src, uint32_t cols_src, uint32_t rows_out, uint32_t cols_out,
                      uint32_t row_off, uint32_t col_off) {
  using T = typename Vec<V>::T;
  griddep_wait();
  griddep_launch_dependents();
  const uint32_t vpr = cols_out / V;
  const uint64_t total = mats * rows_out * vpr;
  const uint64_t stride = (uint64_t)gridDim.x * kShardThreads;
  for (uint64_t i = (uint64_t)blockIdx.x * kShardThreads + threadIdx.x; i < total; i += stride) {
    const uint64_t orow = i / vpr;
    const uint32_t c = (uint32_t)(i - orow * vpr) * V;
    const uint64_t m = orow / rows_out;
    const uint32_t r = (uint32_t)(orow - m * rows_out);
    const uint8_t* s = src + (m * rows_src + r + row_off) * cols_src + col_off + c;
    *reinterpret_cast<T*>(dst + orow * cols_out + c) = *reinterpret_cast<const T*>(s);
  }
}

cudaError_t launch_shard_copy(const uint8_t* src, uint8_t* dst, uint64_t mats, uint32_t rows_src,
                              uint32_t cols_src, uint32_t rows_out, uint32_t cols_out,
                              uint32_t row_off, uint32_t col_off, cudaStream_t stream) {
  const uintptr_t align = reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst) |
                          cols_src | cols_out | col_off;
  const int v = align % 16 == 0 ? 16 : align % 4 == 0 ? 4 : 1;
  const uint64_t total = mats * rows_out * (cols_out / v);
  if (total == 0) return cudaSuccess;
  uint64_t blocks = (total + kShardThreads - 1) / kShardThreads;
  if (blocks > 148 * 16) blocks = 148 * 16;
  const dim3 grid((unsigned)blocks);
  if (v == 16)
    return launch_pdl(shard_copy_kernel<16>, grid, dim3(kShardThreads), 0, stream, src, dst, mats,
                      rows_src, cols_src, rows_out, cols_out, row_off, col_off);
  if (v == 4)
    return launch_pdl(shard_copy_kernel<4>, grid, dim3(kShardThreads), 0, stream, src, dst, mats,
                      rows_src, cols_src, rows_out, cols_out, row_off, col_off);
  return launch_pdl(shard_copy_kernel<1>, grid, dim3(kShardThreads), 0, stream, src, dst, mats,
                    rows_src, cols_src, rows_out, cols_out, row_off, col_off);
}

}  // namespace nvm
