// Exact block-wide top-k over scores held in shared memory (eq. (9) of
// "Compressed Sparse Attention", cnblogs): the k largest scores, equal scores
// ordered by the lower block index, written as ascending block indices.
//
// Selection is a most-significant-digit-first radix select on order-preserving
// 32-bit keys (4 passes of 8-bit histograms) that finds the k-th largest key
// `thr` and how many keys equal to it are taken; a final ordered pass writes
// every key > thr and the first `need_eq` keys == thr.
#pragma once
#include "common.cuh"

namespace csa {

// Exclusive prefix count of `flag` over the CTA (all threads must call);
// *total receives the CTA-wide count.  `ws` holds >= 32 ints of shared memory.
__device__ __forceinline__ int cta_excl_count(bool flag, int* ws, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const unsigned bal = __ballot_sync(0xffffffffu, flag);
  if (lane == 0) ws[warp] = __popc(bal);
  __syncthreads();
  int before = 0, tot = 0;
  for (int w = 0; w < nw; ++w) {
    const int v = ws[w];
    before += (w < warp) ? v : 0;
    tot += v;
  }
  __syncthreads();
  *total = tot;
  return before + __popc(bal & ((1u << lane) - 1u));
}

// Select the top-k of sc[0..n) (n > k) into out[0..k) in ascending index
// order.  `hist` is 256 unsigned of shared memory, `ws` 32+4 ints of shared
// memory.  blockDim.x must be a multiple of 32 and >= 256 is not required.
__device__ void cta_topk_ascending(const float* sc, int n, int k, int* out, unsigned* hist, int* ws) {
  uint32_t prefix = 0, mask = 0;
  int kk = k;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int s = threadIdx.x; s < n; s += blockDim.x) {
      const uint32_t key = ordered_key(sc[s]);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int cum = 0, d = 255;
      for (; d > 0; --d) {
        if (cum + (int)hist[d] >= kk) break;
        cum += hist[d];
      }
      ws[32] = (int)(prefix | ((uint32_t)d << shift));
      ws[33] = kk - cum;
    }
    __syncthreads();
    prefix = (uint32_t)ws[32];
    kk = ws[33];
    mask |= 255u << shift;
    __syncthreads();
  }
  const uint32_t thr = prefix;
  const int need_eq = kk;
  int out_off = 0, eq_seen = 0;
  for (int base = 0; base < n; base += blockDim.x) {
    const int s = base + threadIdx.x;
    const uint32_t key = s < n ? ordered_key(sc[s]) : 0u;
    const bool gt = s < n && key > thr;
    const bool eq = s < n && key == thr;
    int eq_tot, tk_tot;
    const int eq_rank = eq_seen + cta_excl_count(eq, ws, &eq_tot);
    const bool take = gt || (eq && eq_rank < need_eq);
    const int p = out_off + cta_excl_count(take, ws, &tk_tot);
    if (take && p < k) out[p] = s;
    out_off += tk_tot;
    eq_seen += eq_tot;
  }
}

}  // namespace csa
