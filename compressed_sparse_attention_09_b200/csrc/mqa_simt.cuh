// Shared-KV MQA over the selected compressed entries (eqs. 9-11 of
// "Compressed Sparse Attention", cnblogs), CUDA-core version: one CTA per
// query row, each warp owns heads, lanes split the c channels, and an online
// softmax (base-2, the 1/sqrt(c) scale folded into log2 e) runs over the
// selected entries, each entry serving as key and value.  Used for the fp32
// configuration; the bf16 path runs the tcgen05 MQA kernel.
#pragma once
#include "common.cuh"

namespace csa {

struct MqaArgs {
  const void* q; long long ld_q;   // [rows, nh*c]
  const void* C;                   // entries [*, c]
  const int* idx;                  // [rows, topk]
  void* O; long long ld_O;         // [rows, nh*c]
  int topk, nh;
  float scale_log2;                // log2(e) / sqrt(c)
  RowMap rm;
};

template <typename T, int VEC>
__device__ __forceinline__ void load_lane(const T* p, float* out) {
  if constexpr ((VEC * sizeof(T)) % 16 == 0) {
#pragma unroll
    for (int j = 0; j < VEC; j += Vec16<T>::V) load_vec_f32<T>(p + j, out + j);
  } else {
#pragma unroll
    for (int j = 0; j < VEC; ++j) out[j] = to_f32(p[j]);
  }
}

// VEC = c / 32 channels per lane; two heads per warp pass.
template <typename T, int VEC>
__global__ void __launch_bounds__(256) mqa_simt_kernel(MqaArgs a) {
  extern __shared__ int idx_s[];   // [topk]
  constexpr int C = VEC * 32;
  const int row = blockIdx.x;
  long long base;
  int avail;
  row_entries(a.rm, row, base, avail);
  const int* ir = a.idx + (long long)row * a.topk;
  for (int j = threadIdx.x; j < a.topk; j += blockDim.x) idx_s[j] = ir[j];
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const T* qrow = static_cast<const T*>(a.q) + (long long)row * a.ld_q;
  const T* Cb = static_cast<const T*>(a.C) + base * C;
  for (int h0 = 2 * warp; h0 < a.nh; h0 += 2 * nw) {
    const int nhp = min(2, a.nh - h0);
    float qv[2][VEC], o[2][VEC], mx[2], l[2];
#pragma unroll
    for (int hp = 0; hp < 2; ++hp) {
      if (hp < nhp) load_lane<T, VEC>(qrow + (long long)(h0 + hp) * C + lane * VEC, qv[hp]);
      else
#pragma unroll
        for (int e = 0; e < VEC; ++e) qv[hp][e] = 0.f;
#pragma unroll
      for (int e = 0; e < VEC; ++e) o[hp][e] = 0.f;
      mx[hp] = -INFINITY;
      l[hp] = 0.f;
    }
    for (int j = 0; j < a.topk; ++j) {
      const int s = idx_s[j];
      if (s == -1) continue;
      if (s < 0 || s >= avail) {
        if (lane == 0 && h0 == 2 * warp && warp == 0) flag_status(kStatusBadIndex);
        continue;
      }
      if (!dcheck(base + s < rowmap_entries(a.rm, gridDim.x))) continue;
      float cv[VEC];
      load_lane<T, VEC>(Cb + (long long)s * C + lane * VEC, cv);
#pragma unroll
      for (int hp = 0; hp < 2; ++hp) {
        float d = 0.f;
#pragma unroll
        for (int e = 0; e < VEC; ++e) d = fmaf(qv[hp][e], cv[e], d);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
        d *= a.scale_log2;
        const float mnew = fmaxf(mx[hp], d);
        const float alpha = exp2f(mx[hp] - mnew);   // exp2(-inf) = 0 on the first entry
        const float p = exp2f(d - mnew);
        l[hp] = fmaf(l[hp], alpha, p);
#pragma unroll
        for (int e = 0; e < VEC; ++e) o[hp][e] = fmaf(o[hp][e], alpha, p * cv[e]);
        mx[hp] = mnew;
      }
    }
#pragma unroll
    for (int hp = 0; hp < 2; ++hp) {
      if (hp >= nhp) continue;
      const float inv = l[hp] > 0.f ? 1.f / l[hp] : 0.f;
      T* orow = static_cast<T*>(a.O) + (long long)row * a.ld_O + (long long)(h0 + hp) * C + lane * VEC;
#pragma unroll
      for (int e = 0; e < VEC; ++e) orow[e] = from_f32<T>(o[hp][e] * inv);
    }
  }
}

}  // namespace csa
