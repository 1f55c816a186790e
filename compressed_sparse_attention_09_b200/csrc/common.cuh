// Shared device helpers of libcsa: element conversion, the per-device status
// word, and the mapping from a query row to its visible compressed entries.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace csa {

// ---------------------------------------------------------------- status word
// Error bits recorded by kernels instead of faulting; read (and cleared) by
// csa_get_device_status().
enum : unsigned {
  kStatusTimeout = 1u,   // a bounded wait gave up
  kStatusBadIndex = 2u,  // an out-of-range block index was skipped
  kStatusMetadata = 4u,  // cu_seqlens / cu_blocks / cache_len inconsistent
  kStatusBounds = 8u,    // a debug-build index check failed (the access was skipped)
};

__device__ unsigned g_status;

__device__ __forceinline__ void flag_status(unsigned bits) { atomicOr(&g_status, bits); }

// Index checks of the debug build (compiled with CSA_DEBUG): dcheck(ok)
// records kStatusBounds when `ok` is false and returns `ok`, so that the
// caller skips the access it guards; the release build compiles every check
// to `true`.  They restate, next to a global access, the invariant that the
// kernel's own logic guarantees (an entry row inside the entry array, a
// selected index inside the visible range, k indices written per row), so
// that a logic error shows up as a status bit instead of a stray access.
// dguard(ok) is for a guard the release build keeps as a silent skip
// (returns `ok` in both builds; the debug build also records the bit).
#ifdef CSA_DEBUG
constexpr bool kDebugBuild = true;
__device__ __forceinline__ bool dcheck(bool ok) {
  if (!ok) flag_status(kStatusBounds);
  return ok;
}
__device__ __forceinline__ bool dguard(bool ok) { return dcheck(ok); }
#else
constexpr bool kDebugBuild = false;
__device__ __forceinline__ constexpr bool dcheck(bool) { return true; }
__device__ __forceinline__ constexpr bool dguard(bool ok) { return ok; }
#endif

// Limit of every bounded device wait, in ns of %globaltimer (set per device
// by csa_set_wait_limit_ns; read by a wait when its first poll fails).
constexpr unsigned long long kDefaultWaitNs = 1500000000ull;   // 1.5 s
__device__ unsigned long long g_wait_ns = kDefaultWaitNs;

// ---------------------------------------------------------------- programmatic dependent launch
// Kernels launched with programmatic stream serialization may be scheduled
// while the previous kernel on the stream is still finishing.  Each such
// kernel calls pdl_prologue_done() once its prologue (barrier set-up, TMEM
// allocation, descriptor prefetch; no global memory) is over: it waits until
// the previous kernel has completed and its writes are visible, then lets
// the next kernel be scheduled.  Waiting first means that a kernel scheduled
// early after this one may rely on everything before this one on the stream
// being complete (only this kernel's own writes are still in flight).
// Without a programmatic predecessor the wait returns at once.
__device__ __forceinline__ void pdl_prologue_done() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- conversions
template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// 16-byte vector of V elements of T (V = 4 for fp32, 8 for bf16).
template <typename T> struct Vec16 {
  static constexpr int V = 16 / sizeof(T);
  union {
    uint4 u;
    T e[V];
  };
};

template <typename T>
__device__ __forceinline__ void load_vec_f32(const T* p, float* out) {
  Vec16<T> v;
  v.u = *reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int i = 0; i < Vec16<T>::V; ++i) out[i] = to_f32(v.e[i]);
}

// 2^x by the hardware approximation (ex2.approx.ftz.f32: relative error of
// about 2^-22, 2^-inf = +0).
__device__ __forceinline__ float ex2_approx_f32(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Map an fp32 score to an unsigned key whose unsigned order is the float
// order (-0 is folded onto +0 first so that equal scores get equal keys).
__device__ __forceinline__ uint32_t ordered_key(float f) {
  f = f + 0.0f;
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---------------------------------------------------------------- rows
// Where the compressed entries visible to one query row live.  Prefill rows
// are packed sequences (cu_seqlens / cu_blocks); decode rows are one token of
// sequence b over that sequence's cache of capacity `cap`.
struct RowMap {
  const int* cu_seqlens;  // prefill: [nseq+1]
  const int* cu_blocks;   // prefill: [nseq+1]
  int nseq;
  int total_blocks;
  const int* pos;         // decode: [B] token index of the new token
  int cap;                // decode: cache capacity per sequence (0 = prefill)
  int m;
  int pos0;               // prefill: position of the first row of a sequence (0, or the
                          // start of a context-parallel chunk of a single sequence)
};

// Number of entries behind a RowMap: the packed entry array of a prefill
// (total_blocks) or the rows x cap caches of a decode step.
__device__ __forceinline__ long long rowmap_entries(const RowMap& rm, int rows) {
  return rm.cap > 0 ? (long long)rows * rm.cap : (long long)rm.total_blocks;
}

// Visible entries of `row`: global entry index of block 0 and the count
// floor(t/m).  Inconsistent metadata is flagged and clamped so that no access
// leaves [0, total entries).
__device__ __forceinline__ void row_entries(const RowMap& rm, int row, long long& base, int& avail) {
  if (rm.cap > 0) {
    int t = rm.pos[row];
    int a = t >= 0 ? t / rm.m : 0;
    if (a > rm.cap) {
      flag_status(kStatusMetadata);
      a = rm.cap;
    }
    base = (long long)row * rm.cap;
    avail = a;
    return;
  }
  int lo = 0, hi = rm.nseq;  // find the sequence: cu_seqlens[lo] <= row < cu_seqlens[lo+1]
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (rm.cu_seqlens[mid] <= row) lo = mid; else hi = mid;
  }
  int t = row - rm.cu_seqlens[lo] + rm.pos0;
  int a = t / rm.m;
  int b0 = rm.cu_blocks[lo], b1 = rm.cu_blocks[lo + 1];
  if (b0 < 0 || b0 + a > b1 || b1 > rm.total_blocks) {
    flag_status(kStatusMetadata);
    b0 = max(0, min(b0, rm.total_blocks));
    a = max(0, min(a, rm.total_blocks - b0));
  }
  base = b0;
  avail = a;
}

}  // namespace csa
