// Overlapping softmax compression, eqs. (3)-(4) of "Compressed Sparse
// Attention" (cnblogs): every m tokens become one entry, each channel a
// softmax over 2m logits (the block's own Z^a + B^a and the previous block's
// Z^b + B^b) weighting the matching C^a / C^b rows.
//
// The work is a pure stream: each C/Z element is read once and each entry
// written once, so the kernel is HBM-bound.  One thread owns 4 consecutive
// channels of one entry (8-byte loads for bf16, 16-byte for fp32: more
// resident threads measured faster than 16-byte bf16 groups): its 4m row
// loads are 4-element vector loads, coalesced across the warp
// (neighbouring threads own neighbouring channels of the same rows), all
// issued before any arithmetic, and the 2m-wide softmax and the weighted sum
// run in fp32 registers.  One launch covers both entry widths (C^Comp and
// K^IComp): the grid is the concatenation of each segment's blocks, and each
// thread takes exactly one (entry, channel group), so no thread waits on a
// second round of loads.
#pragma once
#include <cuda_fp8.h>

#include "common.cuh"

namespace csa {

// One compressed channel value.  la/lb: the m logits of the block and of the
// block before (already biased); ca/cb: the matching C^a / C^b values.
// has_prev = false is the i = 0 padding (Z^b = -inf, C^b = 0).  The softmax
// runs in base 2 (logits scaled by log2 e once, exponentials by the hardware
// 2^x), and the weighted sum is divided by the normaliser (in [1, 2m]) with
// the fast approximate division.
template <int M>
__device__ __forceinline__ float compress_channel(const float* la, const float* lb, const float* ca,
                                                  const float* cb, bool has_prev) {
  constexpr float kLog2e = 1.4426950408889634f;
  float a2[M], b2[M];
#pragma unroll
  for (int r = 0; r < M; ++r) {
    a2[r] = la[r] * kLog2e;
    b2[r] = lb[r] * kLog2e;
  }
  float mx = a2[0];
#pragma unroll
  for (int r = 1; r < M; ++r) mx = fmaxf(mx, a2[r]);
  if (has_prev) {
#pragma unroll
    for (int r = 0; r < M; ++r) mx = fmaxf(mx, b2[r]);
  }
  float den = 0.f, num = 0.f;
#pragma unroll
  for (int r = 0; r < M; ++r) {
    const float e = ex2_approx_f32(a2[r] - mx);
    den += e;
    num = fmaf(e, ca[r], num);
  }
  if (has_prev) {
#pragma unroll
    for (int r = 0; r < M; ++r) {
      const float e = ex2_approx_f32(b2[r] - mx);
      den += e;
      num = fmaf(e, cb[r], num);
    }
  }
  return __fdividef(num, den);
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
  int groups;          // channel groups per entry: width / V
  int blk0;            // first CTA of this segment in the grid
};

struct CompressArgs {
  CompressSeg seg[2];
  int nseg;
  const int* cu_seqlens;
  const int* cu_blocks;
  int nseq;
  int total_tokens;
  int total_blocks;
};

// V = 4 consecutive elements of T as one vector load (8 or 16 bytes)
template <typename T, int V> struct RawVec;
// a bf16 is the upper half of the fp32 with the same value
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
template <> struct RawVec<__nv_bfloat16, 4> {
  uint2 u;
  __device__ __forceinline__ float at(int e) const {
    const uint32_t w = e < 2 ? u.x : u.y;
    return (e & 1) ? bf16_hi(w) : bf16_lo(w);
  }
};
template <> struct RawVec<float, 4> {
  float4 u;
  __device__ __forceinline__ float at(int e) const { return reinterpret_cast<const float*>(&u)[e]; }
};

template <typename T, int V>
__device__ __forceinline__ RawVec<T, V> load_raw(const T* p) {
  RawVec<T, V> r;
  r.u = __ldcs(reinterpret_cast<const decltype(r.u)*>(p));   // streamed: read once
  return r;
}

template <typename T, int V>
__device__ __forceinline__ void store_raw(T* p, const float* v) {
  if constexpr (sizeof(T) == 2) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]);
    const __nv_bfloat162 b = __floats2bfloat162_rn(v[2], v[3]);
    uint2 u;
    u.x = *reinterpret_cast<const uint32_t*>(&a);
    u.y = *reinterpret_cast<const uint32_t*>(&b);
    *reinterpret_cast<uint2*>(p) = u;
  } else {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
}

// One thread per (segment, entry, channel group); see the header.
template <typename T, int M, int V>
__global__ void __launch_bounds__(256) compress_kernel(CompressArgs a) {
  const int s = (a.nseg > 1 && (int)blockIdx.x >= a.seg[1].blk0) ? 1 : 0;
  const CompressSeg& sg = a.seg[s];
  const int l = ((int)blockIdx.x - sg.blk0) * (int)blockDim.x + (int)threadIdx.x;
  const int g = l / sg.groups;
  if (g >= a.total_blocks) return;
  const int col = (l - g * sg.groups) * V;
  // the sequence owning entry g
  int lo = 0, hi = a.nseq;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (a.cu_blocks[mid] <= g) lo = mid; else hi = mid;
  }
  const int i = g - a.cu_blocks[lo];
  const int tok = a.cu_seqlens[lo] + M * i;
  if (i < 0 || tok + M > a.cu_seqlens[lo + 1] || tok + M > a.total_tokens) {
    flag_status(kStatusMetadata);
    return;
  }
  const bool has_prev = i > 0;
  const T* Za = static_cast<const T*>(sg.Za) + col;
  const T* Ca = static_cast<const T*>(sg.Ca) + col;
  const T* Zb = static_cast<const T*>(sg.Zb) + col;
  const T* Cb = static_cast<const T*>(sg.Cb) + col;
  RawVec<T, V> za[M], ca[M], zb[M], cb[M];
#pragma unroll
  for (int r = 0; r < M; ++r) {
    const long long ra = (long long)(tok + r) * sg.ld;
    za[r] = load_raw<T, V>(Za + ra);
    ca[r] = load_raw<T, V>(Ca + ra);
  }
  if (has_prev) {
#pragma unroll
    for (int r = 0; r < M; ++r) {
      const long long rb = (long long)(tok - M + r) * sg.ld;
      zb[r] = load_raw<T, V>(Zb + rb);
      cb[r] = load_raw<T, V>(Cb + rb);
    }
  }
  float res[V];
#pragma unroll
  for (int q = 0; q < V / 4; ++q) {
    // position biases of these four channels, every row of both halves
    float4 ba[M], bb[M];
#pragma unroll
    for (int r = 0; r < M; ++r) {
      ba[r] = __ldg(reinterpret_cast<const float4*>(sg.Ba + r * sg.width + col + 4 * q));
      bb[r] = has_prev ? __ldg(reinterpret_cast<const float4*>(sg.Bb + r * sg.width + col + 4 * q))
                       : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int e4 = 0; e4 < 4; ++e4) {
      const int e = 4 * q + e4;
      float la[M], lb[M], c_a[M], c_b[M];
#pragma unroll
      for (int r = 0; r < M; ++r) {
        const float bav = reinterpret_cast<const float*>(&ba[r])[e4];
        const float bbv = reinterpret_cast<const float*>(&bb[r])[e4];
        la[r] = za[r].at(e) + bav;
        c_a[r] = ca[r].at(e);
        lb[r] = has_prev ? zb[r].at(e) + bbv : 0.f;
        c_b[r] = has_prev ? cb[r].at(e) : 0.f;
      }
      res[e] = compress_channel<M>(la, lb, c_a, c_b, has_prev);
    }
  }
  if (!dcheck(g < a.total_blocks && (!has_prev || tok - M >= a.cu_seqlens[lo]))) return;
  store_raw<T, V>(static_cast<T*>(sg.out) + (long long)g * sg.width + col, res);
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
  uint8_t* KIcodes;     // quantised key cache (Q8): [B, cap, cI] E4M3 codes
  float* KIscale;       // [B, cap] scales
  int wait_late;        // 1: the previous kernel on the stream reads and writes none of the above
                        // and was scheduled after everything before it had completed (decode:
                        // the c^Q-side projection), so the append runs beside it and waits for it
                        // only at its end; 0: wait for the previous kernel before any access
};

// One CTA per sequence: store the token's row in ring slot t mod 2m, then, if
// t closes block i = (t+1)/m - 1, compress that block from the ring.  Q8:
// the indexer-key entry goes to an E4M3 cache (its bf16 value quantised with
// one scale, max |v| / 448) instead of a bf16 one.
template <typename T, int M, bool Q8>
__device__ __forceinline__ void cache_append_cta(const AppendArgs& a, float* ki_s) {
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
    else if (Q8) ki_s[ch] = to_f32(from_f32<T>(v));   // the entry as stored in T, then quantised below
    else static_cast<T*>(a.KIcache)[((long long)b * a.cap + i) * cI + ch] = from_f32<T>(v);
  }
  __syncthreads();
  if constexpr (Q8) {
    if (threadIdx.x < 32) {
      float amax = 0.f;
      for (int j = threadIdx.x; j < cI; j += 32) amax = fmaxf(amax, fabsf(ki_s[j]));
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      const float scale = amax > 0.f ? amax / 448.f : 1.f;
      uint8_t* dst = a.KIcodes + ((long long)b * a.cap + i) * cI;
      for (int j = threadIdx.x; j < cI; j += 32)
        dst[j] = (uint8_t)__nv_cvt_float_to_fp8(ki_s[j] / scale, __NV_SATFINITE, __NV_E4M3);
      if (threadIdx.x == 0) a.KIscale[(long long)b * a.cap + i] = scale;
    }
  }
  if (threadIdx.x == 0) a.cache_len[b] = i + 1;
}

// With a.wait_late the wait for the previous kernel comes after the append's
// own work, so the kernel after it sees both complete.
template <typename T, int M, bool Q8 = false>
__global__ void __launch_bounds__(256) cache_append_kernel(AppendArgs a) {
  __shared__ float ki_s[1024];
  if (!a.wait_late) pdl_prologue_done();
  cache_append_cta<T, M, Q8>(a, ki_s);
  if (a.wait_late) pdl_prologue_done();
}

}  // namespace csa
