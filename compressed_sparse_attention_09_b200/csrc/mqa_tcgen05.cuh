// Shared-KV MQA over the selected compressed entries, eqs. (9)-(11) of
// "Compressed Sparse Attention" (cnblogs), on the sm_100a tensor cores.
//
// Work item = one query row and a group of 64 of its heads (decode rows with
// n_h = 128 make two items).  For each item the CTA gathers the selected
// entries 32 at a time and, per tile,
//     S  = q . C_tile^T          tcgen05.mma M=64 (heads) N=32 (entries) K=512
//     P  = exp2(S * log2e/sqrt(c) - m)     online softmax, one head per thread
//     O += P . C_tile            tcgen05.mma M=64 (heads) N=256 (x2)  K=32
// The gathered tile sits in shared memory once, in the 128-byte-swizzled
// layout; the S product reads it as a K-major operand (rows = entries) and
// the O product reads the very same bytes as an MN-major operand (rows =
// entries = K, channels contiguous): every entry is loaded once and serves as
// key and value.  With M = 64 the accumulator occupies half of each TMEM lane
// quarter, so the 64 x 512 fp32 O lives in 256 columns (channels 0-255 in the
// lower 16 lanes of every quarter, 256-511 in the upper 16) next to two
// 32-column S buffers.  Each softmax thread owns one head row of S: max, sum
// and the P row need no cross-thread reduction.  O is rescaled (TMEM load,
// multiply, store) only when a head's running maximum grows by more than 8 in
// log2 units; otherwise the stale maximum is kept, which is exact because O
// and the normaliser l share it.
//
// Warp roles (224 threads): warps 0-1 gather the entry tiles with 16-byte
// cp.async into a 4-deep ring (completion is tracked by the stage's mbarrier,
// so the gathers never block); thread 0 also loads q with a 3-D TMA; warp 2
// issues the MMAs (one thread) and owns TMEM; warps 3-6 run the softmax and
// the output epilogue.  All waits are bounded (sm100::mbar_wait).
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
constexpr int kC = 512, kHeads = 64, kTile = 32, kStages = 4;
constexpr int kQChunk = 64 * 128;           // [64 heads x 64 bf16], 128-byte rows, swizzled
constexpr int kCChunk = kTile * 128;        // [32 entries x 64 bf16]
constexpr int kQBytes = 8 * kQChunk;        // 64 x 512
constexpr int kCBytes = 8 * kCChunk;        // one tile: 32 entries x 512
constexpr int kPBytes = 64 * 128;           // 64 heads x 32 entries (rows padded to 128 B), swizzled
constexpr int kMaxTopk = 4096;
constexpr int kProducers = 64;              // threads of warps 0-1
constexpr int kOffQ = 0;
constexpr int kOffC = kOffQ + kQBytes;
constexpr int kOffP = kOffC + kStages * kCBytes;
constexpr int kOffIdx = kOffP + 2 * kPBytes;
constexpr int kOffMisc = kOffIdx + kMaxTopk * 4;
constexpr int kMiscBytes = 256;
constexpr size_t kSmem = 1024 + kOffMisc + kMiscBytes;
constexpr int kThreads = 224;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColS = 256;
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
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kOffMisc);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* c_full = bars + 2;                 // [kStages]
  uint64_t* t_done = c_full + kStages;         // [kStages]  O of the tile done: frees its C stage
  uint64_t* s_full = t_done + kStages;         // [2]
  uint64_t* s_free = s_full + 2;               // [2]
  uint64_t* p_full = s_free + 2;               // [2]
  uint64_t* o_free = p_full + 2;
  uint64_t* i_free = o_free + 1;               // both producer warps done with an item's idx copy
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(i_free + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hgroups = a.nh / kHeads;
  const int items = a.rows * hgroups;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&c_full[s], kProducers);
      mbar_init(&t_done[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], 4);
      mbar_init(&p_full[s], 4);
    }
    mbar_init(o_free, 4);
    mbar_init(i_free, 2);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmQ);
  }
  if (warp == 2) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 2) {
    // ------------------------------------------------------------ producers (warps 0-1)
    const int tid = threadIdx.x;   // 0..63
    uint32_t g = 0, qw = 0, ii = 0;
    for (int it = blockIdx.x; it < items; it += gridDim.x, ++ii) {
      if (warp_aborted(abort_flag)) break;
      const int row = a.rows - 1 - it / hgroups, hg = it % hgroups;
      long long base;
      int avail;
      row_entries(a.rm, row, base, avail);
      const int* ir = a.idx + (long long)row * a.topk;
      const int ntiles = mqa_ntiles(ir, a.topk, avail);
      // both producer warps must be done reading the previous item's idx copy
      if (ii > 0 && !warp_wait(i_free, (ii - 1) & 1)) { *abort_flag = 1; break; }
      // each warp writes the whole copy (identical values), so its own reads need only __syncwarp
      for (int j = lane; j < ntiles * kTile; j += 32) {
        const int s = j < a.topk ? ir[j] : -1;
        const bool v = s >= 0 && s < avail;
        if (warp == 0 && !v && s != -1) flag_status(kStatusBadIndex);
        idx_s[j] = v ? s : -1;
      }
      __syncwarp();
      if (ntiles > 0) {
        if (tid == 0) {
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
      for (int j = 0; j < ntiles; ++j, ++g) {
        const int st = g % kStages;
        if (!warp_wait(&t_done[st], ((g / kStages) & 1) ^ 1)) { ok = false; break; }
        uint8_t* cst = c_s + st * kCBytes;
#pragma unroll 4
        for (int i = 0; i < kTile * 64 / kProducers; ++i) {
          const int u = tid + kProducers * i, r = u >> 6, c16 = u & 63;
          const int s = idx_s[j * kTile + r];
          const __nv_bfloat16* src = s >= 0 ? a.C + (base + s) * kC + c16 * 8 : a.C;
          cp_async16(cst + (c16 >> 3) * kCChunk + sw128(r, c16 & 7), src, s >= 0 ? 16u : 0u);
        }
        cp_async_arrive_noinc(&c_full[st]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(i_free);
      if (!ok) { *abort_flag = 1; break; }
    }
    cp_async_wait_all();
  } else if (warp == 2) {
    // ------------------------------------------------------------ MMA issuer (warp 2, lane 0 issues)
    constexpr uint32_t idS = idesc_bf16_f32(64, kTile);
    constexpr uint32_t idO = idesc_bf16_f32_bmn(64, 256);
    const uint64_t qd0 = sdesc_k_sw128(smem_u32(q_s));
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
        auto issue_o = [&](uint32_t gj, uint32_t jj) -> bool {
          const int st = gj % kStages, pb = gj & 1;
          if (!mbar_wait(&p_full[pb], (gj >> 1) & 1)) return false;
          if (jj == 0 && !mbar_wait(o_free, (oi & 1) ^ 1)) return false;   // previous item's O stored
          tc_fence_after();
          const uint64_t pd = sdesc_k_sw128(smem_u32(p_s + pb * kPBytes));
          const uint64_t cd = sdesc_mn_sw128(smem_u32(c_s + st * kCBytes), kCChunk, 1024);
#pragma unroll
          for (int ks = 0; ks < kTile / 16; ++ks) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
              mma_bf16(tmem + ((uint32_t)(16 * hh) << 16) + kColO, desc_add(pd, ks * 32),
                       desc_add(cd, 4 * hh * kCChunk + ks * 2048), idO, (jj > 0 || ks > 0));
          }
          mma_commit(&t_done[st]);
          return true;
        };
        if (ntiles == 0) {
          if (!mbar_wait(o_free, (oi & 1) ^ 1)) ok = 0;     // keep one o_free phase per item
        } else if (!mbar_wait(q_full, qw & 1)) {
          ok = 0;
        } else {
          tc_fence_after();
          for (int j = 0; j < ntiles && ok; ++j) {
            const uint32_t gj = g + j;
            const int st = gj % kStages, sb = gj & 1;
            if (!mbar_wait(&c_full[st], (gj / kStages) & 1) || !mbar_wait(&s_free[sb], ((gj >> 1) & 1) ^ 1)) {
              ok = 0;
              break;
            }
            fence_proxy_async_smem();
            tc_fence_after();
            const uint64_t cd = sdesc_k_sw128(smem_u32(c_s + st * kCBytes));
#pragma unroll
            for (int kc = 0; kc < 8; ++kc)
#pragma unroll
              for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tmem + kColS + kTile * sb, desc_add(qd0, kc * kQChunk + ks * 32),
                         desc_add(cd, kc * kCChunk + ks * 32), idS, (kc | ks) != 0);
            mma_commit(&s_full[sb]);
            if (j == ntiles - 1) mma_commit(q_empty);
            if (j >= 1 && !issue_o(gj - 1, j - 1)) ok = 0;
          }
          if (ok && !issue_o(g + ntiles - 1, ntiles - 1)) ok = 0;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) { if (lane == 0) *abort_flag = 1; break; }
      if (ntiles > 0) ++qw;
      g += ntiles;
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue (warps 3-6)
    const int sub = warp & 3;                  // TMEM lane quarter of this warp
    const int hrow = 16 * sub + (lane & 15);   // head row (within the group) of lanes 0-15
    const int half = lane >> 4;                // O channel half held by this lane
    const uint32_t lane_base = (uint32_t)(32 * sub) << 16;
    uint32_t g = 0;
    for (int it = blockIdx.x; it < items; it += gridDim.x) {
      if (warp_aborted(abort_flag)) break;
      const int row = a.rows - 1 - it / hgroups, hg = it % hgroups;
      long long base;
      int avail;
      row_entries(a.rm, row, base, avail);
      const int* ir = a.idx + (long long)row * a.topk;
      const int ntiles = mqa_ntiles(ir, a.topk, avail);
      __nv_bfloat16* orow = a.O + (long long)row * a.ld_O + (long long)(hg * kHeads + hrow) * kC + half * 256;
      if (ntiles == 0) {
        const uint4 z = make_uint4(0, 0, 0, 0);
        for (int i = 0; i < 32; ++i) reinterpret_cast<uint4*>(orow)[i] = z;
        __syncwarp();
        if (lane == 0) mbar_arrive(o_free);   // one o_free phase per item, as for the others
        continue;
      }
      float m_run = -INFINITY, l_run = 0.f;
      bool ok = true;
      for (int j = 0; j < ntiles; ++j) {
        const uint32_t gj = g + j;
        const int sb = gj & 1;
        // validity of this tile's 32 rows, from the index row itself
        const int e = j * kTile + lane;
        const int sidx = e < a.topk ? ir[e] : -1;
        const uint32_t vmask = __ballot_sync(0xffffffffu, sidx >= 0 && sidx < avail);
        if (!warp_wait(&s_full[sb], (gj >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        float sv[kTile];
        tmem_ld_32x32b_x32(tmem + lane_base + kColS + kTile * sb, sv);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[sb]);
        float tmax = -INFINITY;
#pragma unroll
        for (int q = 0; q < kTile; ++q) {
          sv[q] = ((vmask >> q) & 1u) ? sv[q] * a.scale_log2 : -INFINITY;
          tmax = fmaxf(tmax, sv[q]);
        }
        const float m_new = fmaxf(m_run, tmax);
        const bool grow = half == 0 && m_new > m_run + 8.f;   // also true on the first finite tile
        const float m_use = grow ? m_new : m_run;
        if (__any_sync(0xffffffffu, grow && j > 0)) {
          // rescale O: the O MMAs of the earlier tiles must have completed
          const uint32_t gp = gj - 1;
          if (!warp_wait(&t_done[gp % kStages], (gp / kStages) & 1)) { ok = false; break; }
          tc_fence_after();
          float alpha = grow ? exp2f(m_run - m_new) : 1.f;    // exp2(-inf) = 0 when nothing was seen
          alpha = __shfl_sync(0xffffffffu, alpha, lane & 15);
#pragma unroll 1
          for (int ch = 0; ch < 8; ++ch) {
            float v[32];
            tmem_ld_32x32b_x32(tmem + lane_base + kColO + ch * 32, v);
#pragma unroll
            for (int q = 0; q < 32; ++q) v[q] *= alpha;
            tmem_st_32x32b_x32(tmem + lane_base + kColO + ch * 32, v);
          }
          tmem_st_wait();
          tc_fence_before();
          l_run *= alpha;
        }
        m_run = m_use;
        // P rows (lanes 0-15), once the P buffer's previous reader (tile gj-2) is done
        if (gj >= 2) {
          const uint32_t gp = gj - 2;
          if (!warp_wait(&t_done[gp % kStages], (gp / kStages) & 1)) { ok = false; break; }
        }
        if (half == 0) {
          uint8_t* prow = p_s + sb * kPBytes;
          float sum = 0.f;
#pragma unroll
          for (int u = 0; u < kTile / 8; ++u) {
            Vec16<__nv_bfloat16> pk;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float x = sv[8 * u + q];
              const float p = (x == -INFINITY) ? 0.f : exp2f(x - m_use);
              sum += p;
              pk.e[q] = __float2bfloat16_rn(p);
            }
            *reinterpret_cast<uint4*>(prow + sw128(hrow, u)) = pk.u;
          }
          l_run += sum;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[sb]);
      }
      if (!ok) { *abort_flag = 1; break; }
      // epilogue: O / l for this warp's 16 heads
      const uint32_t glast = g + ntiles - 1;
      if (!warp_wait(&t_done[glast % kStages], (glast / kStages) & 1)) { *abort_flag = 1; break; }
      tc_fence_after();
      float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      inv = __shfl_sync(0xffffffffu, inv, lane & 15);
#pragma unroll 1
      for (int ch = 0; ch < 8; ++ch) {
        float v[32];
        tmem_ld_32x32b_x32(tmem + lane_base + kColO + ch * 32, v);
#pragma unroll
        for (int qd = 0; qd < 4; ++qd) {
          Vec16<__nv_bfloat16> pk;
#pragma unroll
          for (int q = 0; q < 8; ++q) pk.e[q] = __float2bfloat16_rn(v[8 * qd + q] * inv);
          reinterpret_cast<uint4*>(orow + ch * 32)[qd] = pk.u;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_free);
      g += ntiles;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace csa
