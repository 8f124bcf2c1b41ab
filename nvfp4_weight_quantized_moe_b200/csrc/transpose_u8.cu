// Load-time twin builder: byte transpose [rows, cols] -> [cols, rows].
//
// metrale_model_layers/weight_map/quantized/transpose.rs, `transpose_for_gemm_gs`:
// the packed weight [N, K/2] becomes [K/2, N] and the scales [N, K/16] become
// [K/16, N]; the host fallback loop t[j*rows + i] = b[i*cols + j] defines the
// result.  A 32x32 byte tile passes through shared memory (padded row, no bank
// conflicts on the transposed read) so both global sides are row-contiguous.
//
// The same kernel writes into a column window of a wider output (row pitch,
// column offset): transpose_concat_for_gemm_gs / _padded in transpose.rs place
// several parts' twins side by side along N in a [K/2, stride] buffer whose
// columns past the last part are zero.

#include "common.cuh"
#include "kernels.h"

namespace nvm {

__global__ void __launch_bounds__(256)
    transpose_u8_kernel(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst, int rows,
                        int cols, uint64_t dst_pitch, uint64_t dst_col_off) {
  __shared__ uint8_t tile[32][33];
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;
  for (int i = ty; i < 32; i += 8) {
    const int r = r0 + i, cc = c0 + tx;
    if (r < rows && cc < cols) tile[i][tx] = src[(size_t)r * cols + cc];
  }
  __syncthreads();
  for (int i = ty; i < 32; i += 8) {
    const int orow = c0 + i, ocol = r0 + tx;
    if (orow < cols && ocol < rows) dst[(size_t)orow * dst_pitch + dst_col_off + ocol] = tile[tx][i];
  }
}

// Zero columns [col_lo, pitch) of every one of `rows` rows.
__global__ void __launch_bounds__(256)
    zero_cols_kernel(uint8_t* __restrict__ dst, uint64_t rows, uint64_t pitch, uint64_t col_lo) {
  const uint64_t w = pitch - col_lo;
  const uint64_t total = rows * w;
  for (uint64_t i = (uint64_t)blockIdx.x * 256 + threadIdx.x; i < total;
       i += (uint64_t)gridDim.x * 256) {
    const uint64_t r = i / w;
    dst[r * pitch + col_lo + (i - r * w)] = 0;
  }
}

cudaError_t launch_transpose_u8_pitched(const uint8_t* src, uint8_t* dst, uint32_t rows,
                                        uint32_t cols, uint64_t dst_pitch, uint64_t dst_col_off,
                                        cudaStream_t stream) {
  if (rows == 0 || cols == 0) return cudaSuccess;
  const dim3 grid((cols + 31) / 32, (rows + 31) / 32);
  transpose_u8_kernel<<<grid, dim3(32, 8), 0, stream>>>(src, dst, (int)rows, (int)cols, dst_pitch,
                                                        dst_col_off);
  return cudaGetLastError();
}

cudaError_t launch_transpose_u8(const uint8_t* src, uint8_t* dst, uint32_t rows, uint32_t cols,
                                cudaStream_t stream) {
  return launch_transpose_u8_pitched(src, dst, rows, cols, rows, 0, stream);
}

cudaError_t launch_zero_cols(uint8_t* dst, uint64_t rows, uint64_t pitch, uint64_t col_lo,
                             cudaStream_t stream) {
  const uint64_t total = rows * (pitch - col_lo);
  if (total == 0) return cudaSuccess;
  uint64_t blocks = (total + 255) / 256;
  if (blocks > 148 * 8) blocks = 148 * 8;
  zero_cols_kernel<<<(unsigned)blocks, 256, 0, stream>>>(dst, rows, pitch, col_lo);
  return cudaGetLastError();
}

}  // namespace nvm
