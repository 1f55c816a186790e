// CUDA-core projection GEMM  D[M, N] = A[M, K] . B[N, K]^T  with fp32
// accumulation, used for the fp32 configuration (the tensor cores have no
// fp32 operand type) and for shapes below the tensor-core tile.  The bf16
// prefill projections run on the tcgen05 kernel in gemm_tcgen05.cuh.
//
// Both operands are K-major: A rows are tokens (H or c^Q), B rows are output
// columns of the packed, transposed weights.  Output columns are routed to
// up to kMaxSeg destination segments (e.g. the bf16 C/Z/c^Q block and the
// fp32 w^I block of the H-side projection).
#pragma once
#include "common.cuh"

namespace csa {

constexpr int kMaxSeg = 4;

struct OutSeg {
  int col0, ncols;     // columns [col0, col0 + ncols) of D
  void* ptr;           // destination of column col0
  long long ld;        // destination row stride (elements)
  int f32;             // 1: store fp32, 0: store the GEMM's element type
};

struct GemmOut {
  OutSeg seg[kMaxSeg];
  int nseg;
};

template <typename T>
__device__ __forceinline__ void store_out(const GemmOut& o, long long row, int col, float v) {
#pragma unroll
  for (int s = 0; s < kMaxSeg; ++s) {
    if (s < o.nseg && col >= o.seg[s].col0 && col < o.seg[s].col0 + o.seg[s].ncols) {
      const long long off = row * o.seg[s].ld + (col - o.seg[s].col0);
      if (o.seg[s].f32) static_cast<float*>(o.seg[s].ptr)[off] = v;
      else static_cast<T*>(o.seg[s].ptr)[off] = from_f32<T>(v);
    }
  }
}

struct SimtGemmArgs {
  const void* A; long long lda;
  const void* B; long long ldb;
  int M, N, K;
  GemmOut out;
};

// 128x128 output tile per CTA, 8x8 per thread, K staged 8 at a time.
template <typename T>
__global__ void __launch_bounds__(256) gemm_simt_kernel(SimtGemmArgs g) {
  constexpr int BM = 128, BN = 128, BK = 8;
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const T* A = static_cast<const T*>(g.A);
  const T* B = static_cast<const T*>(g.B);
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  // each thread stages 4 elements of A and 4 of B per K step
  const int lr = tid / 2, lk = (tid % 2) * 4;
  for (int k0 = 0; k0 < g.K; k0 += BK) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int k = k0 + lk + q;
      const int ma = m0 + lr, nb = n0 + lr;
      As[lk + q][lr] = (ma < g.M && k < g.K) ? to_f32(A[(long long)ma * g.lda + k]) : 0.f;
      Bs[lk + q][lr] = (nb < g.N && k < g.K) ? to_f32(B[(long long)nb * g.ldb + k]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[8], b[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = As[kk][ty * 4 + i];
        a[4 + i] = As[kk][64 + ty * 4 + i];
        b[i] = Bs[kk][tx * 4 + i];
        b[4 + i] = Bs[kk][64 + tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int row = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
    if (row >= g.M) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int col = n0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + (j - 4));
      if (col < g.N) store_out<T>(g.out, row, col, acc[i][j]);
    }
  }
}

}  // namespace csa
