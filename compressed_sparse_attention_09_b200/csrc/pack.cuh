// Weight packing: the page's [in, out] matrices become K-major [out, in] rows
// of one concatenated operand per projection GEMM, and the position biases are
// widened to fp32.  Runs once per set of weights.
#pragma once
#include "common.cuh"

namespace csa {

// dst[c][r] = src[r][c] for src [R, Cc]; dst row stride ld_dst.
template <typename T>
__global__ void transpose_kernel(const T* __restrict__ src, int R, int Cc, T* __restrict__ dst,
                                 long long ld_dst) {
  __shared__ T tile[32][33];
  const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int r = r0 + i, c = c0 + threadIdx.x;
    if (r < R && c < Cc) tile[i][threadIdx.x] = src[(long long)r * Cc + c];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int c = c0 + i, r = r0 + threadIdx.x;
    if (r < R && c < Cc) dst[(long long)c * ld_dst + r] = tile[threadIdx.x][i];
  }
}

template <typename T>
__global__ void widen_kernel(const T* __restrict__ src, float* __restrict__ dst, long long n) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x)
    dst[i] = to_f32(src[i]);
}

}  // namespace csa
