// Decode over a quantised indexer-key cache: K^IComp held as FP8 E4M3 codes
// with one fp32 scale per entry (a cache format of this implementation; the
// page stores C^Comp / K^IComp without fixing a precision).  The indexer
// reads half the bytes of a bf16 cache, which is the largest stream of a
// decode step.
//
// Format: for an entry v (its c^I values as stored in bf16), scale =
// max_j |v_j| / 448 in fp32 (1 for an all-zero entry) and code_j =
// E4M3(v_j / scale), rounded to nearest even and saturated to +-448.  The
// entry stands for code * scale.  Because the scale is positive,
//     I[t, s] = sum_h w_h ReLU(q_h . (scale_s code_s))
//             = scale_s * sum_h w_h ReLU(q_h . code_s)
// so the tensor cores multiply the codes themselves (widened to fp16, which
// holds every E4M3 value exactly) by q^I in fp16, and the epilogue applies
// scale_s to the head-weighted sum.
#pragma once
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "sm100.cuh"

namespace csa {

// One warp per row: row r of src (w bf16 values, w a multiple of 32, row
// stride ld) to w E4M3 codes and one scale.
__global__ void quantize_rows_e4m3_kernel(const __nv_bfloat16* src, long long ld, int n, int w, uint8_t* codes,
                                          float* scales) {
  const int warp = (int)((blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5), lane = threadIdx.x & 31;
  if (warp >= n) return;
  const __nv_bfloat16* row = src + (long long)warp * ld;
  float amax = 0.f;
  for (int j = lane; j < w; j += 32) amax = fmaxf(amax, fabsf(__bfloat162float(row[j])));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const float scale = amax > 0.f ? amax / 448.f : 1.f;
  for (int j = lane; j < w; j += 32)
    codes[(long long)warp * w + j] =
        (uint8_t)__nv_cvt_float_to_fp8(__bfloat162float(row[j]) / scale, __NV_SATFINITE, __NV_E4M3);
  if (lane == 0) scales[warp] = scale;
}

// q^I rows (bf16, row stride ld) to fp16 [n, w]: the quantised indexer
// multiplies the fp16 codes by fp16 queries (one operand type per MMA).
__global__ void bf16_to_f16_rows_kernel(const __nv_bfloat16* src, long long ld, int n, int w, __half* dst) {
  pdl_prologue_done();
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)n * w) return;
  const int r = (int)(i / w), j = (int)(i % w);
  dst[i] = __float2half_rn(__bfloat162float(src[(long long)r * ld + j]));
}

struct IdxDecQ8Args {
  const float* wI; long long ld_wI;   // [B, nhI]
  const int* pos;                     // [B]
  const float* kscale;                // [B, cap]
  float* scratch;                     // [B, cap] scores
  int B, cap, m, nhI, tiles_per_seq;
};

namespace idxq8 {
constexpr int kM = 128, kCI = 128, kStages = 7, kKBufs = 2, kQSlots = 2;
constexpr int kQBytes = 64 * 128 * 2;          // q^I fp16, up to 64 heads x 128, two 64-column chunks
constexpr int kCodeBytes = kM * kCI;           // 128 entries x 128 codes (128-byte swizzled rows)
constexpr int kKChunk = kM * 128;              // fp16 [128 entries x 64 channels]
constexpr int kKBytes = 2 * kKChunk;
constexpr int kOffC = kQSlots * kQBytes;       // code stages
constexpr int kOffK = kOffC + kStages * kCodeBytes;
constexpr int kOffW = kOffK + kKBufs * kKBytes;
constexpr int kEpiWarps = 8;                   // warps 2-5 and 10-13: even and odd items of the CTA
constexpr size_t kSmem = 1024 + (size_t)kOffW + kEpiWarps * 64 * 4 + 256;
constexpr int kCvtWarps = 4;                   // warps 6-9 widen the codes
constexpr int kThreads = 32 * (2 + kEpiWarps + kCvtWarps);
}  // namespace idxq8

// Two E4M3 codes (the low and high byte of v) to an fp16 pair, low code in
// the low half (the hardware conversion).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t v) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(v));
  return r;
}

// Instruction descriptor of kind::f16 with fp16 A/B, fp32 D, both K-major.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Score rows of the decode queries over their FP8 key caches, one work item
// per (sequence, 128-entry tile), items of a CTA contiguous.  Warp 0: TMA
// (q^I fp16 once per sequence, the tile's codes per stage); warps 6-9: widen the codes to
// fp16 in the MMA's swizzled K-major layout (two buffers); warp 1: MMA
// issuer and TMEM owner (D[128 entries x n_h^I], two accumulators); warps
// 2-5 and 10-13: epilogue (ReLU, head weights, entry scale), one group per
// accumulator.  All waits are bounded.
__global__ void __launch_bounds__(idxq8::kThreads, 1)
    indexer_decode_q8_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
                             IdxDecQ8Args a) {
  using namespace sm100;
  using namespace idxq8;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* kbuf = sm + kOffK;
  float* w_s = reinterpret_cast<float*>(sm + kOffW);            // 4 epilogue warps x 64
  uint64_t* bars = reinterpret_cast<uint64_t*>(w_s + kEpiWarps * 64);
  uint64_t* full = bars;                   // [kStages] codes landed
  uint64_t* empty = full + kStages;        // [kStages] codes widened (kCvtWarps arrivals)
  uint64_t* kfull = empty + kStages;       // [kKBufs] fp16 tile written (kCvtWarps arrivals)
  uint64_t* kfree = kfull + kKBufs;        // [kKBufs] MMA done with the fp16 tile
  uint64_t* t_full = kfree + kKBufs;       // [2]
  uint64_t* t_empty = t_full + 2;          // [2]
  uint64_t* q_full = t_empty + 2;          // [kQSlots] q^I of a sequence landed
  uint64_t* q_empty = q_full + kQSlots;    // [kQSlots] the sequence's last MMA done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_empty + kQSlots);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = a.nhI;
  const int items = a.B * a.tiles_per_seq;
  const int qchunk = N * 128;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], kCvtWarps); }
    for (int s = 0; s < kKBufs; ++s) { mbar_init(&kfull[s], kCvtWarps); mbar_init(&kfree[s], 1); }
    for (int s = 0; s < 2; ++s) { mbar_init(&t_full[s], 1); mbar_init(&t_empty[s], 4); }
    for (int s = 0; s < kQSlots; ++s) { mbar_init(&q_full[s], 1); mbar_init(&q_empty[s], 1); }
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmQ);
  }
  if (warp == 1) tmem_alloc(tmem_slot, 128);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_prologue_done();
  const uint32_t tmem = *tmem_slot;

  const int per = (items + gridDim.x - 1) / gridDim.x;
  const int it0 = blockIdx.x * per, it1 = min(items, it0 + per);
  // the sequence's visible count is read once per sequence, not per item
  int cached_b = -1, cached_avail = 0;
  auto item_ok = [&](int it, int& b, int& j, int& avail) {
    b = it / a.tiles_per_seq;
    j = it - b * a.tiles_per_seq;
    if (b != cached_b) {
      const int t = a.pos[b];
      cached_avail = t >= 0 ? min(t / a.m, a.cap) : 0;
      cached_b = b;
    }
    avail = cached_avail;
    return j * kM < avail;
  };

  // q^I (fp16) is loaded once per sequence (a CTA's items are contiguous)
  // into one of kQSlots slots; the ring stages carry only codes, and the
  // widening warps free a stage as soon as they have read it.
  if (warp == 0) {
    if (lane == 0) {
      uint32_t g = 0, nq = 0;
      int qb = -1;
      for (int it = it0; it < it1 && !*abort_flag; ++it) {
        int b, j, avail;
        if (!item_ok(it, b, j, avail)) continue;
        if (b != qb) {
          const int qs = nq % kQSlots;
          if (!mbar_wait(&q_empty[qs], ((nq / kQSlots) & 1) ^ 1)) { *abort_flag = 1; break; }
          mbar_arrive_expect_tx(&q_full[qs], (uint32_t)(2 * qchunk));
          for (int c = 0; c < 2; ++c) tma_load_3d(&tmQ, &q_full[qs], sm + qs * kQBytes + c * qchunk, 64 * c, 0, b);
          qb = b;
          ++nq;
        }
        const int st = g % kStages;
        if (!mbar_wait(&empty[st], ((g / kStages) & 1) ^ 1)) { *abort_flag = 1; break; }
        mbar_arrive_expect_tx(&full[st], (uint32_t)kCodeBytes);
        tma_load_2d(&tmK, &full[st], sm + kOffC + st * kCodeBytes, 0, b * a.cap + j * kM);
        ++g;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_f16_f32(kM, N);
      uint32_t g = 0, nq = 0;
      int qb = -1;
      for (int it = it0; it < it1 && !*abort_flag; ++it) {
        int b, j, avail;
        if (!item_ok(it, b, j, avail)) continue;
        if (b != qb) {
          // the previous sequence's slot is free once its MMAs complete
          if (nq > 0) mma_commit(&q_empty[(nq - 1) % kQSlots]);
          if (!mbar_wait(&q_full[nq % kQSlots], (nq / kQSlots) & 1)) { *abort_flag = 1; break; }
          qb = b;
          ++nq;
        }
        const int kb = g % kKBufs, acc = g & 1;
        if (!mbar_wait(&kfull[kb], (g / kKBufs) & 1) || !mbar_wait(&t_empty[acc], ((g >> 1) & 1) ^ 1)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint64_t qd = sdesc_k_sw128(smem_u32(sm + ((nq - 1) % kQSlots) * kQBytes));
        const uint64_t kd = sdesc_k_sw128(smem_u32(kbuf + kb * kKBytes));
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_bf16(tmem + (uint32_t)(acc * 64), desc_add(kd, c * kKChunk + ks * 32),
                     desc_add(qd, c * qchunk + ks * 32), idesc, (c | ks) != 0);
        mma_commit(&kfree[kb]);
        mma_commit(&t_full[acc]);
        ++g;
      }
    }
  } else if (warp >= 6 && warp < 6 + kCvtWarps) {
    // ---------------------------------------------------------------- code widening (warps 6-9)
    // thread -> 16-byte unit u = t % 8 (16 codes) of rows t / 8 + 16 i; all
    // of a thread's row loads are issued before any conversion
    const int t = threadIdx.x - 192, u = t & 7, r0 = t >> 3;
    constexpr int kRows = kM / (4 * kCvtWarps);   // rows per thread
    uint32_t g = 0;
    for (int it = it0; it < it1; ++it) {
      if (warp_aborted(abort_flag)) break;
      int b, j, avail;
      if (!item_ok(it, b, j, avail)) continue;
      const int st = g % kStages, kb = g % kKBufs;
      if (!warp_wait(&full[st], (g / kStages) & 1) || !warp_wait(&kfree[kb], ((g / kKBufs) & 1) ^ 1)) {
        if (lane == 0) *abort_flag = 1;
        break;
      }
      const uint8_t* codes = sm + kOffC + st * kCodeBytes;
      uint8_t* dst = kbuf + kb * kKBytes + (u >> 2) * kKChunk;   // channels 16 u .. are in chunk u / 4
      uint4 cw[kRows];
#pragma unroll
      for (int i = 0; i < kRows; ++i) {
        const int r = r0 + (4 * kCvtWarps) * i;
        cw[i] = *reinterpret_cast<const uint4*>(codes + r * 128 + ((u ^ (r & 7)) << 4));
      }
      // 16 fp16 channels = units uu and uu + 1 of the chunk's row; the upper
      // four threads of each 8 store them in the other order, so that each
      // store of 8 threads covers all 8 bank groups (the chunks are 16 KB apart)
      const int uu = 2 * (u & 3), s0 = uu + (u >> 2), s1 = uu + 1 - (u >> 2);
#pragma unroll
      for (int i = 0; i < kRows; ++i) {
        const int r = r0 + (4 * kCvtWarps) * i;
        const uint32_t w4[4] = {cw[i].x, cw[i].y, cw[i].z, cw[i].w};
        uint32_t h[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          h[2 * q] = e4m3x2_to_f16x2((uint16_t)(w4[q] & 0xFFFFu));
          h[2 * q + 1] = e4m3x2_to_f16x2((uint16_t)(w4[q] >> 16));
        }
        const uint4 lo = make_uint4(h[0], h[1], h[2], h[3]), hi = make_uint4(h[4], h[5], h[6], h[7]);
        *reinterpret_cast<uint4*>(dst + r * 128 + ((s0 ^ (r & 7)) << 4)) = (u >> 2) ? hi : lo;
        *reinterpret_cast<uint4*>(dst + r * 128 + ((s1 ^ (r & 7)) << 4)) = (u >> 2) ? lo : hi;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&kfull[kb]);
        mbar_arrive(&empty[st]);   // every code of the stage has been read and used
      }
      ++g;
    }
  } else {
    // ---------------------------------------------------------------- epilogue (warps 2-5 and 10-13)
    // warps 2-5 take the CTA's even items (accumulator 0), warps 10-13 the
    // odd ones (accumulator 1), so two items are folded at a time
    const int sub = warp & 3, grp = warp < 6 ? 0 : 1;
    float* w_my = w_s + (warp < 6 ? warp - 2 : warp - 6 - kCvtWarps + 4) * 64;
    const uint32_t lane_base = (uint32_t)(32 * sub) << 16;
    uint32_t g = 0;
    int wb = -1;
    for (int it = it0; it < it1; ++it) {
      if (warp_aborted(abort_flag)) break;
      int b, j, avail;
      if (!item_ok(it, b, j, avail)) continue;
      if ((int)(g & 1) != grp) { ++g; continue; }
      if (b != wb) {
        for (int hh = lane; hh < N; hh += 32) w_my[hh] = a.wI[(long long)b * a.ld_wI + hh];
        __syncwarp();
        wb = b;
      }
      // the entry's scale is fetched before the wait, so that its memory
      // latency overlaps the MMA instead of following the epilogue
      const int s = j * kM + 32 * sub + lane;
      const float kscale = s < avail ? __ldg(a.kscale + (long long)b * a.cap + s) : 0.f;
      const int acc = g & 1;
      if (!warp_wait(&t_full[acc], (g >> 1) & 1)) { *abort_flag = 1; break; }
      tc_fence_after();
      float sc4[4] = {0.f, 0.f, 0.f, 0.f};   // four partial sums (heads e mod 4)
      for (int hc = 0; hc < N; hc += 32) {
        float v[32];
        tmem_ld_32x32b_x32(tmem + lane_base + (uint32_t)(acc * 64 + hc), v);
#pragma unroll
        for (int e = 0; e < 32; ++e) sc4[e & 3] = fmaf(w_my[hc + e], fmaxf(v[e], 0.f), sc4[e & 3]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&t_empty[acc]);
      if (s < avail && dcheck(s < a.cap))
        __stcg(a.scratch + (long long)b * a.cap + s, ((sc4[0] + sc4[1]) + (sc4[2] + sc4[3])) * kscale);
      ++g;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

}  // namespace csa
