// Lightning indexer (eq. 8) + top-k (eq. 9) of "Compressed Sparse Attention"
// (cnblogs), CUDA-core version: one CTA per query row.  The row's scores
// I_{t,s} = sum_h w_{t,h} ReLU(q^I_{t,h} . K^IComp_s), s < floor(t/m), are
// computed into shared memory (one thread per block s, its key row in
// registers, the row's queries broadcast from shared memory) and the exact
// top-k is selected there, so no score reaches global memory.  Used for the
// fp32 configuration; the bf16 path runs the tcgen05 indexer.
#pragma once
#include "common.cuh"
#include "topk.cuh"

namespace csa {

struct IndexerArgs {
  const void* qI; long long ld_qI;   // [rows, nhI*cI]
  const float* wI; long long ld_wI;  // [rows, nhI]
  const void* KI;                    // entries [*, cI]
  int* idx;                          // [rows, topk]
  int topk, nhI;
  int sc_cap;                        // capacity of the shared score array
  RowMap rm;
};

template <typename T, int CI>
__global__ void __launch_bounds__(256, 1) indexer_topk_simt_kernel(IndexerArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* q_s = reinterpret_cast<float*>(smem_raw);            // [nhI*CI]
  float* w_s = q_s + a.nhI * CI;                             // [nhI]
  unsigned* hist = reinterpret_cast<unsigned*>(w_s + a.nhI); // [256]
  int* ws = reinterpret_cast<int*>(hist + 256);              // [40]
  float* sc = reinterpret_cast<float*>(ws + 40);             // [sc_cap]

  const int row = blockIdx.x;
  long long base;
  int avail;
  row_entries(a.rm, row, base, avail);
  int* out = a.idx + (long long)row * a.topk;
  if (avail > a.sc_cap) {
    if (threadIdx.x == 0) flag_status(kStatusMetadata);
    avail = a.sc_cap;
  }
  if (avail <= a.topk) {  // every visible block is kept
    for (int j = threadIdx.x; j < a.topk; j += blockDim.x) out[j] = j < avail ? j : -1;
    return;
  }
  const T* q = static_cast<const T*>(a.qI) + (long long)row * a.ld_qI;
  for (int j = threadIdx.x; j < a.nhI * CI; j += blockDim.x) q_s[j] = to_f32(q[j]);
  for (int j = threadIdx.x; j < a.nhI; j += blockDim.x) w_s[j] = a.wI[(long long)row * a.ld_wI + j];
  __syncthreads();

  const T* K = static_cast<const T*>(a.KI) + base * CI;
  constexpr int V = Vec16<T>::V;
  for (int s = threadIdx.x; s < avail; s += blockDim.x) {
    float kr[CI];
#pragma unroll
    for (int j = 0; j < CI; j += V) load_vec_f32<T>(K + (long long)s * CI + j, kr + j);
    float acc = 0.f;
    for (int h = 0; h < a.nhI; ++h) {
      const float4* qh = reinterpret_cast<const float4*>(q_s + h * CI);
      float dot = 0.f;
#pragma unroll
      for (int j = 0; j < CI / 4; ++j) {
        const float4 qv = qh[j];
        dot = fmaf(qv.x, kr[4 * j + 0], dot);
        dot = fmaf(qv.y, kr[4 * j + 1], dot);
        dot = fmaf(qv.z, kr[4 * j + 2], dot);
        dot = fmaf(qv.w, kr[4 * j + 3], dot);
      }
      acc = fmaf(w_s[h], fmaxf(dot, 0.f), acc);
    }
    sc[s] = acc;
  }
  __syncthreads();
  cta_topk_ascending(sc, avail, a.topk, out, hist, ws);
}

}  // namespace csa
