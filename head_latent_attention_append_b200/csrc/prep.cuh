// Weight preparation: per-head transpose of W_UK so that the absorption
// q~_h = W_UK,h^T q_C,h runs as an "NT" GEMM with K = d_h contiguous.
#pragma once
#include "common.cuh"

namespace mla {

// in [n_h][rows][cols] -> out [n_h][cols][rows], 32x32 tiles through smem.
template <typename T>
__global__ void transpose_heads_kernel(const T* __restrict__ in, T* __restrict__ out, int rows, int cols) {
  __shared__ T tile[32][33];
  const long long hoff = (long long)blockIdx.z * rows * cols;
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    int r = r0 + i, c = c0 + threadIdx.x;
    if (r < rows && c < cols) tile[i][threadIdx.x] = in[hoff + (long long)r * cols + c];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    int c = c0 + i, r = r0 + threadIdx.x;
    if (r < rows && c < cols) out[hoff + (long long)c * rows + r] = tile[threadIdx.x][i];
  }
}

}  // namespace mla
