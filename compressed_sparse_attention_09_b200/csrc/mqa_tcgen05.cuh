// Shared-KV MQA over the selected compressed entries, eqs. (9)-(11) of
// "Compressed Sparse Attention" (cnblogs), on the sm_100a tensor cores.
//
// Work item = one query row and a group of 64 of its heads (decode rows with
// n_h = 128 make two items).  For each item the CTA gathers the selected
// entries 128 at a time and computes, per tile, the transposed products
//     S^T = C_tile . q^T            tcgen05.mma M=128 (entries)  N=64 (heads) K=512
//     P   = exp2(S * log2e/sqrt(c) - m_ref)   per head
//     O^T += C_tile^T . P^T         tcgen05.mma M=128 (channels) x4, N=64, K=128
// Both products keep M = 128, which on sm_100a runs at ~4870 FLOP/clk/SM for
// N = 64, where every M = 64 form (heads as rows) is capped at half rate
// (4094).  The gathered tile sits in shared memory once, in the
// 128-byte-swizzled layout, as 8 channel chunks of [128 entries x 64
// channels]: S^T reads it as a K-major A operand (rows = entries) and O^T
// reads the very same bytes as an MN-major A operand (channels contiguous,
// K = entries): every entry is loaded once and serves as key and value.  A
// 128-entry tile is 128 KB, so there is one tile buffer whose chunks are
// released as the O^T blocks consume them; the next tile's gather overlaps
// the rest of O^T.
//
// Softmax over entries = across TMEM lanes.  Eight softmax warps each own one
// lane quarter (32 entries) and 32 of the 64 heads.  A per-head reference
// maximum m_ref is shared by all of them; P = exp2(s - m_ref) needs no
// reduction, and each thread keeps per-head partial sums l_part that are
// reduced once per query.  Only when some score exceeds m_ref + 8 (always on
// a query's first tile) do the warps agree, through a rotating flag word and
// a group barrier, to compute the tile's exact per-head maximum and rescale
// O^T and l_part; otherwise the stale reference is kept, which is exact
// because O^T and l share it.
//
// Warp roles (320 threads): warp 0 gathers the entry chunks with 16-byte
// cp.async (completion tracked by the chunk's mbarrier) and loads q with a
// 3-D TMA; warp 1 issues the MMAs (one thread) and owns TMEM; warps 2-9 run
// the softmax and the output epilogue.  All waits are bounded
// (sm100::mbar_wait).
#pragma once
#include "common.cuh"
#include "sm100.cuh"

namespace csa {

struct MqaTcArgs {
  const __nv_bfloat16* C;                   // entries [*, 512]
  const int* idx;                           // [rows, topk]
  __nv_bfloat16* O; long long ld_O;         // [rows, nh*512]
  int topk, nh, rows;
  float scale_log2;                         // log2(e) / sqrt(c)
  RowMap rm;
};

namespace mqa {
constexpr int kC = 512, kHeads = 64, kTile = 128;
constexpr int kQChunk = 64 * 128;           // [64 heads x 64 bf16], 128-byte rows, swizzled
constexpr int kCChunk = kTile * 128;        // [128 entries x 64 bf16]
constexpr int kPChunk = 64 * 128;           // [64 heads x 64 entries]
constexpr int kQBytes = 8 * kQChunk;        // 64 x 512
constexpr int kCBytes = 8 * kCChunk;        // one tile: 128 entries x 512
constexpr int kPBytes = 2 * kPChunk;        // P^T: 64 heads x 128 entries
constexpr int kMaxTopk = 2048;
constexpr int kProducers = 32;              // threads of warp 0
constexpr int kSoftmaxWarps = 8;
constexpr int kOffQ = 0;
constexpr int kOffC = kOffQ + kQBytes;
constexpr int kOffP = kOffC + kCBytes;
constexpr int kOffIdx = kOffP + kPBytes;
constexpr int kOffRed = kOffIdx + kMaxTopk * 4;   // [4 quarters][64 heads] floats x 2, + [8 warps][32] floats
constexpr int kOffMisc = kOffRed + 4 * 256 * 4;
constexpr int kMiscBytes = 256;
constexpr size_t kSmem = 1024 + kOffMisc + kMiscBytes;
constexpr int kThreads = 32 * (2 + kSoftmaxWarps);
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColS = 256;  // O^T: 4 blocks x 64 columns; S^T: 64 columns
}  // namespace mqa

// byte offset of 16-byte unit u (0..7) of row r in a 128-byte-swizzled chunk
__device__ __forceinline__ uint32_t sw128(int r, int u) { return (uint32_t)(r * 128 + ((u ^ (r & 7)) << 4)); }

// Number of kTile-entry tiles a query row needs: up to its last valid slot
// (0 <= s < avail).  Every warp role derives it on its own from the index
// row, so no role depends on another's shared-memory copy of it.
__device__ __forceinline__ int mqa_ntiles(const int* ir, int topk, int avail) {
  const int lane = threadIdx.x & 31;
  int last = -1;
  for (int j = lane; j < topk; j += 32) {
    const int s = ir[j];
    if (s >= 0 && s < avail) last = j;
  }
  last = __reduce_max_sync(0xffffffffu, last);
  return (last + mqa::kTile) / mqa::kTile;
}

__global__ void __launch_bounds__(mqa::kThreads, 1)
    mqa_tc_kernel(const __grid_constant__ CUtensorMap tmQ, MqaTcArgs a) {
  using namespace sm100;
  using namespace mqa;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_s = sm + kOffQ;
  uint8_t* c_s = sm + kOffC;
  uint8_t* p_s = sm + kOffP;
  int* idx_s = reinterpret_cast<int*>(sm + kOffIdx);
  float* red_m = reinterpret_cast<float*>(sm + kOffRed);     // per-quarter maxima [4][64]
  float* red_l = red_m + 4 * 64;                             // per-quarter sums    [4][64]
  float* alpha_s = red_l + 4 * 64;                           // per-warp rescale factors [8][32]
  float* mref_s = alpha_s + 8 * 32;                          // per-warp reference maxima [8][32]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kOffMisc);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* c_full = bars + 2;                 // [8] channel chunk of the tile gathered
  uint64_t* c_free = c_full + 8;               // [8] chunk consumed by the tile's MMAs
  uint64_t* s_full = c_free + 8;
  uint64_t* s_free = s_full + 1;
  uint64_t* p_full = s_free + 1;
  uint64_t* t_done = p_full + 1;               // O^T of the tile done (P buffer free)
  uint64_t* o_free = t_done + 1;
  uint64_t* g_sync = o_free + 1;               // softmax-group barrier
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(g_sync + 1);
  int* ovf = reinterpret_cast<int*>(tmem_slot + 1);                  // [3] rotating flag words
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ovf + 3);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hgroups = a.nh / kHeads;
  const int items = a.rows * hgroups;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int c = 0; c < 8; ++c) {
      mbar_init(&c_full[c], kProducers);
      mbar_init(&c_free[c], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, kSoftmaxWarps);
    mbar_init(p_full, kSoftmaxWarps);
    mbar_init(t_done, 1);
    mbar_init(o_free, kSoftmaxWarps);
    mbar_init(g_sync, kSoftmaxWarps);
    ovf[0] = ovf[1] = ovf[2] = 0;
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmQ);
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer (warp 0)
    uint32_t g = 0, qw = 0;
    for (int it = blockIdx.x; it < items; it += gridDim.x) {
      if (warp_aborted(abort_flag)) break;
      const int row = a.rows - 1 - it / hgroups, hg = it % hgroups;
      long long base;
      int avail;
      row_entries(a.rm, row, base, avail);
      const int* ir = a.idx + (long long)row * a.topk;
      const int ntiles = mqa_ntiles(ir, a.topk, avail);
      // the previous item's gathers were issued from idx_s before this loop iteration
      for (int j = lane; j < ntiles * kTile; j += 32) {
        const int s = j < a.topk ? ir[j] : -1;
        const bool v = s >= 0 && s < avail;
        if (!v && s != -1) flag_status(kStatusBadIndex);
        idx_s[j] = v ? s : -1;
      }
      __syncwarp();
      if (ntiles > 0) {
        if (lane == 0) {
          if (!mbar_wait(q_empty, (qw & 1) ^ 1)) {
            *abort_flag = 1;
          } else {
            mbar_arrive_expect_tx(q_full, (uint32_t)kQBytes);
            for (int kc = 0; kc < 8; ++kc) tma_load_3d(&tmQ, q_full, q_s + kc * kQChunk, 64 * kc, 64 * hg, row);
          }
        }
        ++qw;
      }
      bool ok = true;
      for (int j = 0; j < ntiles && ok; ++j, ++g) {
        for (int kc = 0; kc < 8; ++kc) {
          if (!warp_wait(&c_free[kc], (g & 1) ^ 1)) { ok = false; break; }
          uint8_t* dst = c_s + kc * kCChunk;
#pragma unroll 8
          for (int i = 0; i < kTile * 8 / kProducers; ++i) {
            const int u = lane + kProducers * i, r = u >> 3, unit = u & 7;
            const int s = idx_s[j * kTile + r];
            const __nv_bfloat16* src = s >= 0 ? a.C + (base + s) * kC + kc * 64 + unit * 8 : a.C;
            cp_async16(dst + sw128(r, unit), src, s >= 0 ? 16u : 0u);
          }
          cp_async_arrive_noinc(&c_full[kc]);
        }
      }
      __syncwarp();
      if (!ok) { *abort_flag = 1; break; }
    }
    cp_async_wait_all();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (warp 1, lane 0 issues)
    constexpr uint32_t idS = idesc_bf16_f32(128, 64);
    constexpr uint32_t idO = idesc_bf16_f32_amn(128, 64);
    const uint32_t q_addr = smem_u32(q_s), c_addr = smem_u32(c_s), p_addr = smem_u32(p_s);
    uint32_t g = 0, qw = 0, oi = 0;
    for (int it = blockIdx.x; it < items; it += gridDim.x, ++oi) {
      if (warp_aborted(abort_flag)) break;
      const int row = a.rows - 1 - it / hgroups;
      long long base;
      int avail;
      row_entries(a.rm, row, base, avail);
      const int ntiles = mqa_ntiles(a.idx + (long long)row * a.topk, a.topk, avail);
      int ok = 1;
      if (lane == 0) {
        if (ntiles == 0) {
          if (!mbar_wait(o_free, (oi & 1) ^ 1)) ok = 0;     // keep one o_free phase per item
        } else if (!mbar_wait(q_full, qw & 1)) {
          ok = 0;
        } else {
          for (int j = 0; j < ntiles && ok; ++j) {
            const uint32_t ph = (g + j) & 1;
            // S^T = C_tile . q^T, chunk by chunk as the gathers land
            if (!mbar_wait(s_free, ph ^ 1)) { ok = 0; break; }
            for (int kc = 0; kc < 8 && ok; ++kc) {
              if (!mbar_wait(&c_full[kc], ph)) { ok = 0; break; }
              fence_proxy_async_smem();
              tc_fence_after();
#pragma unroll
              for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tmem + kColS, sdesc_k_sw128(c_addr + kc * kCChunk + ks * 32),
                         sdesc_k_sw128(q_addr + kc * kQChunk + ks * 32), idS, (kc | ks) != 0);
            }
            if (!ok) break;
            mma_commit(s_full);
            if (j == ntiles - 1) mma_commit(q_empty);
            // O^T += C_tile^T . P^T, channel block by channel block, releasing its two chunks
            if (!mbar_wait(p_full, ph)) { ok = 0; break; }
            if (j == 0 && !mbar_wait(o_free, (oi & 1) ^ 1)) { ok = 0; break; }   // previous item's O stored
            tc_fence_after();
#pragma unroll
            for (int b = 0; b < 4; ++b) {
#pragma unroll
              for (int ks = 0; ks < kTile / 16; ++ks)
                mma_bf16(tmem + kColO + 64 * b,
                         sdesc_mn_sw128(c_addr + 2 * b * kCChunk + ks * 2048, kCChunk, 1024),
                         sdesc_k_sw128(p_addr + (ks >> 2) * kPChunk + (ks & 3) * 32), idO, (j > 0 || ks > 0));
              mma_commit(&c_free[2 * b]);
              mma_commit(&c_free[2 * b + 1]);
            }
            mma_commit(t_done);
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) { if (lane == 0) *abort_flag = 1; break; }
      if (ntiles > 0) ++qw;
      g += ntiles;
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue (warps 2-9)
    const int qd = warp & 3;                   // TMEM lane quarter: entries / channels 32qd .. 32qd+31
    const int hf = (warp - 2) >> 2;            // heads 32hf .. 32hf+31
    const uint32_t lane_base = (uint32_t)(32 * qd) << 16;
    const int e_loc = 32 * qd + lane;          // this thread's entry within a tile
    uint32_t g = 0, gs = 0;                    // tiles seen, group barriers passed
    auto group_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(g_sync);
      const bool okw = warp_wait(g_sync, gs & 1);
      ++gs;
      return okw;
    };
    for (int it = blockIdx.x; it < items; it += gridDim.x) {
      if (warp_aborted(abort_flag)) break;
      const int row = a.rows - 1 - it / hgroups, hg = it % hgroups;
      long long base;
      int avail;
      row_entries(a.rm, row, base, avail);
      const int* ir = a.idx + (long long)row * a.topk;
      const int ntiles = mqa_ntiles(ir, a.topk, avail);
      __nv_bfloat16* orow = a.O + (long long)row * a.ld_O + (long long)(hg * kHeads + 32 * hf) * kC;
      if (ntiles == 0) {
        // zeros: this warp writes channels 32qd..32qd+31 of each block for its 32 heads
        for (int h = 0; h < 32; ++h)
          for (int b = 0; b < 4; ++b) orow[(long long)h * kC + 128 * b + e_loc] = __float2bfloat16_rn(0.f);
        __syncwarp();
        if (lane == 0) mbar_arrive(o_free);   // one o_free phase per item, as for the others
        continue;
      }
      float* m_ref = mref_s + (warp - 2) * 32;   // warp-uniform values: read as broadcasts
      float l_part[32];
      if (lane == 0)
#pragma unroll
        for (int h = 0; h < 32; ++h) m_ref[h] = -INFINITY;
#pragma unroll
      for (int h = 0; h < 32; ++h) l_part[h] = 0.f;
      __syncwarp();
      bool ok = true;
      for (int j = 0; j < ntiles; ++j) {
        const uint32_t gj = g + j, ph = gj & 1;
        const int sidx = ir[j * kTile + e_loc < a.topk ? j * kTile + e_loc : 0];
        const bool valid = (j * kTile + e_loc < a.topk) && sidx >= 0 && sidx < avail;
        if (!warp_wait(s_full, ph)) { ok = false; break; }
        tc_fence_after();
        float sv[32];
        tmem_ld_32x32b_x32(tmem + lane_base + kColS + 32 * hf, sv);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free);
        bool over = false;
#pragma unroll
        for (int h = 0; h < 32; ++h) {
          sv[h] = valid ? sv[h] * a.scale_log2 : -INFINITY;
          over |= sv[h] > m_ref[h] + 8.f;
        }
        // agree on whether the reference maximum must move (flag words rotate over 3 tiles)
        const int fw = gj % 3;
        if (__any_sync(0xffffffffu, over) && lane == 0) atomicOr(&ovf[fw], 1);
        if (!group_sync()) { ok = false; break; }
        if (warp == 2 && lane == 0) ovf[(gj + 2) % 3] = 0;   // the word of tile gj-1: every warp has read it
        if (*reinterpret_cast<volatile int*>(&ovf[fw])) {
          // exact per-head maximum of this tile: lanes, then the four quarters
#pragma unroll
          for (int h = 0; h < 32; ++h) {
            float v = sv[h];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
            if (lane == h) red_m[qd * 64 + 32 * hf + h] = v;   // lane h publishes head h of this slice
          }
          if (!group_sync()) { ok = false; break; }
          float* alpha = alpha_s + (warp - 2) * 32;   // this warp's private factors
#pragma unroll
          for (int h = 0; h < 32; ++h) {
            const int hh = 32 * hf + h;
            const float tm = fmaxf(fmaxf(red_m[hh], red_m[64 + hh]), fmaxf(red_m[128 + hh], red_m[192 + hh]));
            const float mo = m_ref[h];
            const float mn = fmaxf(mo, tm);
            const float al = (mn == -INFINITY) ? 1.f : exp2f(mo - mn);   // exp2(-inf) = 0 on the first tile
            l_part[h] *= al;
            __syncwarp();
            if (lane == 0) { alpha[h] = al; m_ref[h] = mn; }
          }
          __syncwarp();
          if (j > 0) {
            // rescale O^T columns of this warp's heads (rows = its channel lanes) once the
            // earlier tiles' O^T MMAs are done
            if (!warp_wait(t_done, (gj - 1) & 1)) { ok = false; break; }
            tc_fence_after();
#pragma unroll 1
            for (int b = 0; b < 4; ++b) {
              float v[32];
              tmem_ld_32x32b_x32(tmem + lane_base + kColO + 64 * b + 32 * hf, v);
#pragma unroll
              for (int h = 0; h < 32; ++h) v[h] *= alpha[h];
              tmem_st_32x32b_x32(tmem + lane_base + kColO + 64 * b + 32 * hf, v);
            }
            tmem_st_wait();
            tc_fence_before();
          }
          // the reductions' shared words are read by every warp before the next reuse
          if (!group_sync()) { ok = false; break; }
        } else if (j > 0) {
          if (!warp_wait(t_done, (gj - 1) & 1)) { ok = false; break; }   // P is single-buffered
        }
        // P^T[h][e] = exp2(s - m_ref[h]) for this thread's entry and 32 heads
        {
          const int chunk = e_loc >> 6, ee = e_loc & 63;
          uint8_t* pch = p_s + chunk * kPChunk + (ee & 7) * 2;
#pragma unroll
          for (int h = 0; h < 32; ++h) {
            const float p = (sv[h] == -INFINITY) ? 0.f : exp2f(sv[h] - m_ref[h]);
            l_part[h] += p;
            const int hh = 32 * hf + h;
            *reinterpret_cast<__nv_bfloat16*>(pch + sw128(hh, ee >> 3)) = __float2bfloat16_rn(p);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
      }
      if (!ok) { *abort_flag = 1; break; }
      // l = sum of the partial sums over all entries (lanes, then quarters)
#pragma unroll
      for (int h = 0; h < 32; ++h) {
        float v = l_part[h];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == h) red_l[qd * 64 + 32 * hf + h] = v;
      }
      if (!group_sync()) { *abort_flag = 1; break; }
#pragma unroll
      for (int h = 0; h < 32; ++h) {
        const int hh = 32 * hf + h;
        const float l = red_l[hh] + red_l[64 + hh] + red_l[128 + hh] + red_l[192 + hh];
        l_part[h] = l > 0.f ? 1.f / l : 0.f;   // reused as 1 / l
      }
      // epilogue: O[row, head, channel] = O^T[channel, head] / l
      const uint32_t glast = g + ntiles - 1;
      if (!warp_wait(t_done, glast & 1)) { *abort_flag = 1; break; }
      tc_fence_after();
#pragma unroll 1
      for (int b = 0; b < 4; ++b) {
        float v[32];
        tmem_ld_32x32b_x32(tmem + lane_base + kColO + 64 * b + 32 * hf, v);
#pragma unroll
        for (int h = 0; h < 32; ++h) orow[(long long)h * kC + 128 * b + e_loc] = __float2bfloat16_rn(v[h] * l_part[h]);
      }
      tc_fence_before();
      // red_l is rewritten by the next item only after this barrier
      if (!group_sync()) { *abort_flag = 1; break; }
      if (lane == 0) mbar_arrive(o_free);
      g += ntiles;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace csa
