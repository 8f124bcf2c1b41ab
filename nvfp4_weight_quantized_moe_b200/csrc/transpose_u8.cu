// Load-time twin builder: byte transpose [rows, cols] -> [cols, rows].
//
// metrale_model_layers/weight_map/quantized/transpose.rs, `transpose_for_gemm_gs`:
// the packed weight [N, K/2] becomes [K/2, N] and the scales [N, K/16] become
// [K/16, N]; the host fallback loop t[j*rows + i] = b[i*cols + j] defines the
// result.  A 32x32 byte tile passes through shared memory (padded row, no bank
// conflicts on the transposed read) so both global sides are row-contiguous.

#include "common.cuh"
#include "kernels.h"

namespace nvm {

__global__ void __launch_bounds__(256)
    transpose_u8_kernel(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst, int rows,
                        int cols) {
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
    if (orow < cols && ocol < rows) dst[(size_t)orow * rows + ocol] = tile[tx][i];
  }
}

cudaError_t launch_transpose_u8(const uint8_t* src, uint8_t* dst, uint32_t rows, uint32_t cols,
                                cudaStream_t stream) {
  const dim3 grid((cols + 31) / 32, (rows + 31) / 32);
  transpose_u8_kernel<<<grid, dim3(32, 8), 0, stream>>>(src, dst, (int)rows, (int)cols);
  return cudaGetLastError();
}

}  // namespace nvm
