// Overlapping softmax compression, eqs. (3)-(4) of "Compressed Sparse
// Attention" (cnblogs): every m tokens become one entry, each channel a
// softmax over 2m logits (the block's own Z^a + B^a and the previous block's
// Z^b + B^b) weighting the matching C^a / C^b rows.
//
// The work is a pure stream: each C/Z element is read once and each entry
// written once, so the kernel is HBM-bound.  One thread owns 4 channels of
// one entry: its 4m row loads are 4-element vector loads (8 bytes for bf16,
// 16 for fp32), coalesced across the warp (neighbouring threads own
// neighbouring channels of the same rows), and the 2m-wide softmax and the
// weighted sum run in fp32 registers.  Four channels per thread keep the
// live registers low enough for many resident warps, which is what keeps
// enough loads in flight to stream at HBM rate.
#pragma once
#include "common.cuh"

namespace csa {

// One compressed channel value.  la/lb: the m logits of the block and of the
// block before (already biased); ca/cb: the matching C^a / C^b values.
// has_prev = false is the i = 0 padding (Z^b = -inf, C^b = 0).
template <int M>
__device__ __forceinline__ float compress_channel(const float* la, const float* lb, const float* ca,
                                                  const float* cb, bool has_prev) {
  float mx = la[0];
#pragma unroll
  for (int r = 1; r < M; ++r) mx = fmaxf(mx, la[r]);
  if (has_prev) {
#pragma unroll
    for (int r = 0; r < M; ++r) mx = fmaxf(mx, lb[r]);
  }
  float den = 0.f, num = 0.f;
#pragma unroll
  for (int r = 0; r < M; ++r) {
    float e = expf(la[r] - mx);
    den += e;
    num = fmaf(e, ca[r], num);
  }
  if (has_prev) {
#pragma unroll
    for (int r = 0; r < M; ++r) {
      float e = expf(lb[r] - mx);
      den += e;
      num = fmaf(e, cb[r], num);
    }
  }
  return num / den;
}

struct CompressSeg {
  const void* Ca;
  const void* Cb;
  const void* Za;
  const void* Zb;
  long long ld;        // row stride of Ca/Cb/Za/Zb in elements
  const float* Ba;     // [m, width]
  const float* Bb;     // [m, width]
  int width;
  void* out;           // [total_blocks, width]
};

struct CompressArgs {
  CompressSeg seg[2];
  int nseg;
  int vecs0;           // 4-channel groups per entry row of segment 0
  int vecs_total;      // 4-channel groups per entry over all segments
  const int* cu_seqlens;
  const int* cu_blocks;
  int nseq;
  int total_tokens;
  int total_blocks;
};

// 4 consecutive elements as fp32 (one 8-byte or 16-byte load)
template <typename T> __device__ __forceinline__ void load4(const T* p, float* o);
template <> __device__ __forceinline__ void load4<float>(const float* p, float* o) {
  const float4 v = *reinterpret_cast<const float4*>(p);
  o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
}
template <> __device__ __forceinline__ void load4<__nv_bfloat16>(const __nv_bfloat16* p, float* o) {
  const uint2 v = *reinterpret_cast<const uint2*>(p);
  const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&v.x);
  const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&v.y);
  const float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
  o[0] = fa.x; o[1] = fa.y; o[2] = fb.x; o[3] = fb.y;
}
template <typename T> __device__ __forceinline__ void store4(T* p, const float* v);
template <> __device__ __forceinline__ void store4<float>(float* p, const float* v) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
template <> __device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* p, const float* v) {
  const __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]);
  const __nv_bfloat162 b = __floats2bfloat162_rn(v[2], v[3]);
  uint2 u;
  u.x = *reinterpret_cast<const uint32_t*>(&a);
  u.y = *reinterpret_cast<const uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = u;
}

// grid-stride over (entry, 4-channel group) pairs of all segments
template <typename T, int M>
__global__ void __launch_bounds__(256) compress_kernel(CompressArgs a) {
  constexpr int V = 4;
  const long long n_items = (long long)a.total_blocks * a.vecs_total;
  for (long long it = (long long)blockIdx.x * blockDim.x + threadIdx.x; it < n_items;
       it += (long long)gridDim.x * blockDim.x) {
    const int g = (int)(it / a.vecs_total);
    int v = (int)(it - (long long)g * a.vecs_total);
    const int s = v < a.vecs0 ? 0 : 1;
    if (s) v -= a.vecs0;
    const CompressSeg& sg = a.seg[s];
    // the sequence owning entry g
    int lo = 0, hi = a.nseq;
    while (hi - lo > 1) {
      int mid = (lo + hi) >> 1;
      if (a.cu_blocks[mid] <= g) lo = mid; else hi = mid;
    }
    const int i = g - a.cu_blocks[lo];
    const long long tok = (long long)a.cu_seqlens[lo] + (long long)M * i;
    if (i < 0 || tok + M > a.cu_seqlens[lo + 1] || tok + M > a.total_tokens) {
      flag_status(kStatusMetadata);
      continue;
    }
    const bool has_prev = i > 0;
    const int col = v * V;
    float la[M][V], lb[M][V], ca[M][V], cb[M][V];
#pragma unroll
    for (int r = 0; r < M; ++r) {
      const long long ra = (tok + r) * sg.ld + col;
      load4<T>(static_cast<const T*>(sg.Za) + ra, la[r]);
      load4<T>(static_cast<const T*>(sg.Ca) + ra, ca[r]);
      if (has_prev) {
        const long long rb = (tok - M + r) * sg.ld + col;
        load4<T>(static_cast<const T*>(sg.Zb) + rb, lb[r]);
        load4<T>(static_cast<const T*>(sg.Cb) + rb, cb[r]);
      }
    }
#pragma unroll
    for (int r = 0; r < M; ++r) {
      const float4 ba = *reinterpret_cast<const float4*>(sg.Ba + (long long)r * sg.width + col);
      la[r][0] += ba.x; la[r][1] += ba.y; la[r][2] += ba.z; la[r][3] += ba.w;
      if (has_prev) {
        const float4 bb = *reinterpret_cast<const float4*>(sg.Bb + (long long)r * sg.width + col);
        lb[r][0] += bb.x; lb[r][1] += bb.y; lb[r][2] += bb.z; lb[r][3] += bb.w;
      }
    }
    float res[V];
#pragma unroll
    for (int e = 0; e < V; ++e) {
      float l_a[M], l_b[M], c_a[M], c_b[M];
#pragma unroll
      for (int r = 0; r < M; ++r) {
        l_a[r] = la[r][e]; c_a[r] = ca[r][e];
        l_b[r] = has_prev ? lb[r][e] : 0.f;
        c_b[r] = has_prev ? cb[r][e] : 0.f;
      }
      res[e] = compress_channel<M>(l_a, l_b, c_a, c_b, has_prev);
    }
    store4<T>(static_cast<T*>(sg.out) + (long long)g * sg.width + col, res);
  }
}

// ---------------------------------------------------------------- decode append
struct AppendArgs {
  const void* rows;     // [B, ld_rows]: first ring_w elements are the new token's ring row
  long long ld_rows;
  const int* pos;       // [B]
  void* ring;           // [B, 2m, ring_w]
  void* Ccache;         // [B, cap, c]
  void* KIcache;        // [B, cap, cI]
  int* cache_len;       // [B]
  const float* Ba; const float* Bb;     // [m, c]
  const float* BaI; const float* BbI;   // [m, cI]
  int c, cI, cap, ring_w;
};

// One CTA per sequence: store the token's row in ring slot t mod 2m, then, if
// t closes block i = (t+1)/m - 1, compress that block from the ring.
template <typename T, int M>
__global__ void __launch_bounds__(256) cache_append_kernel(AppendArgs a) {
  const int b = blockIdx.x;
  const int t = a.pos[b];
  if (t < 0) {
    if (threadIdx.x == 0) flag_status(kStatusMetadata);
    return;
  }
  const int slot = t % (2 * M);
  const T* src = static_cast<const T*>(a.rows) + (long long)b * a.ld_rows;
  T* ring = static_cast<T*>(a.ring) + (long long)b * 2 * M * a.ring_w;
  for (int e = threadIdx.x; e < a.ring_w; e += blockDim.x) ring[(long long)slot * a.ring_w + e] = src[e];
  __syncthreads();
  if ((t + 1) % M != 0) return;
  const int i = (t + 1) / M - 1;
  if (a.cache_len[b] != t / M || i >= a.cap) {
    if (threadIdx.x == 0) flag_status(i >= a.cap ? kStatusBadIndex : kStatusMetadata);
    if (i >= a.cap) return;
  }
  const bool has_prev = i > 0;
  // column offsets of the eight parts of a ring row
  const int c = a.c, cI = a.cI;
  const int offC[4] = {0, c, 2 * c, 3 * c};
  const int offI[4] = {4 * c, 4 * c + cI, 4 * c + 2 * cI, 4 * c + 3 * cI};
  for (int j = threadIdx.x; j < c + cI; j += blockDim.x) {
    const bool main = j < c;
    const int ch = main ? j : j - c;
    const int* off = main ? offC : offI;
    const float* Ba = main ? a.Ba : a.BaI;
    const float* Bb = main ? a.Bb : a.BbI;
    const int w = main ? c : cI;
    float la[M], lb[M], ca[M], cb[M];
#pragma unroll
    for (int r = 0; r < M; ++r) {
      const T* ra = ring + (long long)((M * i + r) % (2 * M)) * a.ring_w;
      ca[r] = to_f32(ra[off[0] + ch]);
      la[r] = to_f32(ra[off[2] + ch]) + Ba[r * w + ch];
      if (has_prev) {
        const T* rb = ring + (long long)((M * (i - 1) + r) % (2 * M)) * a.ring_w;
        cb[r] = to_f32(rb[off[1] + ch]);
        lb[r] = to_f32(rb[off[3] + ch]) + Bb[r * w + ch];
      } else {
        cb[r] = 0.f;
        lb[r] = 0.f;
      }
    }
    const float v = compress_channel<M>(la, lb, ca, cb, has_prev);
    if (main) static_cast<T*>(a.Ccache)[((long long)b * a.cap + i) * c + ch] = from_f32<T>(v);
    else static_cast<T*>(a.KIcache)[((long long)b * a.cap + i) * cI + ch] = from_f32<T>(v);
  }
  __syncthreads();
  if (threadIdx.x == 0) a.cache_len[b] = i + 1;
}

}  // namespace csa
