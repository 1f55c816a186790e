// Shared-KV MQA over the selected compressed entries, eqs. (9)-(11) of
// "Compressed Sparse Attention" (cnblogs), on the sm_100a tensor cores.
//
// Work item = one query row and a group of 64 of its heads (decode rows with
// n_h = 128 make two items).  For each item the CTA gathers the selected
// entries 32 at a time and, per tile,
//     S  = q . C_tile^T          tcgen05.mma M=64 (heads) N=32 (entries) K=512
//     P  = exp2(S * log2e/sqrt(c) - m)     online softmax
//     O += P . C_tile            tcgen05.mma M=64 (heads) N=256 (x2)  K=32
// The gathered tile sits in shared memory once, in the 128-byte-swizzled
// layout; the S product reads it as a K-major operand (rows = entries) and
// the O product reads the very same bytes as an MN-major operand (rows =
// entries = K, channels contiguous): every entry is loaded once and serves as
// key and value.
//
// Issue rate.  One thread issuing tcgen05.mma waits ~54 cycles per
// instruction whatever its size below N = 128, so the S product of a 32-entry
// tile (32 instructions) would leave the tensor pipe three-quarters idle.
// Four threads (one per S-issuer warp) therefore issue it together, each over
// a quarter of the channels (K = 128) into its own partial accumulator; the
// softmax adds the four partials.  A fifth warp issues the O products only,
// so the S issuers never wait for the softmax: they run up to four tiles
// ahead, one S buffer each.
//
// Gather rate.  The tiles are gathered with 16-byte cp.async by eight warps
// into a 4-deep ring (completion tracked by the stage's mbarrier, so the
// gathers never block): a random-row gather from L2 reaches ~9 bytes/clock
// per warp, and the MMAs consume ~32 bytes/clock.
//
// TMEM (512 columns): O (64 x 512 fp32) in columns 0-255 (channels 0-255 in
// the lower 16 lanes of every lane quarter, 256-511 in the upper 16); four S
// buffers of 64 columns, each holding the four partials (issuer i at column
// offset 32 (i / 2) and lane offset 16 (i % 2)).  A softmax thread owns one
// head and half of a tile (16 entries) and writes its piece of the P row into
// one of four P buffers (64-byte rows in the 64-byte swizzle).  O is rescaled
// (TMEM load, multiply, store) only when a head's running maximum grows by
// more than 8 in log2 units; otherwise the stale maximum is kept, which is
// exact because O and the normaliser l share it.
//
// Warp roles (544 threads): warps 0-7 gather the entry tiles (thread 0 also
// loads q with a 3-D TMA); warps 8-11 issue the S products and warp 12 the O
// products (lane 0 of each; warp 8 owns TMEM); warps 13-16 run the softmax
// and the output epilogue.  All waits are bounded (sm100::mbar_wait).
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
constexpr int kPBytes = 64 * 64;            // 64 heads x 32 entries, 64-byte rows, swizzled
constexpr int kPBufs = 4;                   // P buffers
constexpr int kProducers = 256;             // threads of warps 0-7
constexpr int kIssuers = 4;                 // S issuers: warps 8-11
constexpr int kSBufs = 4;                   // S buffers in TMEM
constexpr int kOffQ = 0;
constexpr int kOffC = kOffQ + kQBytes;
constexpr int kOffP = kOffC + kStages * kCBytes;
constexpr int kStageBytes = 4 * 32 * 128;     // O staging: 32 rows of 128 B per softmax warp
constexpr int kOffStage = kOffP + kPBufs * kPBytes;
constexpr int kOffMisc = kOffStage + kStageBytes;
constexpr int kMiscBytes = 256;
constexpr size_t kSmem = 1024 + kOffMisc + kMiscBytes;
constexpr int kThreads = 544;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColS = 256;
}  // namespace mqa

// byte offset of 16-byte unit u (0..7) of row r in a 128-byte-swizzled chunk
__device__ __forceinline__ uint32_t sw128(int r, int u) { return (uint32_t)(r * 128 + ((u ^ (r & 7)) << 4)); }
// byte offset of 16-byte unit u (0..3) of row r in a 64-byte-swizzled block
__device__ __forceinline__ uint32_t sw64(int r, int u) { return (uint32_t)(r * 64 + ((u ^ ((r >> 1) & 3)) << 4)); }

// Number of kTile-entry tiles a query row needs: up to its last valid slot
// (0 <= s < avail).  Called by a whole warp; every warp role derives it on
// its own from the index row.  The loads go out 16 per lane at a time, so a
// row of up to 512 slots costs one memory latency.
__device__ __forceinline__ int mqa_ntiles(const int* ir, int topk, int avail) {
  const int lane = threadIdx.x & 31;
  int last = -1;
  for (int j0 = 0; j0 < topk; j0 += 32 * 16) {
    int v[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int j = j0 + 32 * u + lane;
      v[u] = j < topk ? __ldg(ir + j) : -1;
    }
#pragma unroll
    for (int u = 0; u < 16; ++u)
      if (v[u] >= 0 && v[u] < avail) last = j0 + 32 * u + lane;
  }
  last = __reduce_max_sync(0xffffffffu, last);
  return (last + mqa::kTile) / mqa::kTile;
}

__global__ void __launch_bounds__(mqa::kThreads, 1)
    mqa_tc_kernel(const __grid_constant__ CUtensorMap tmQ, MqaTcArgs a) {
  using namespace sm100;
  using namespace mqa;
  constexpr uint32_t kFull = 0xffffffffu;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_s = sm + kOffQ;
  uint8_t* c_s = sm + kOffC;
  uint8_t* p_s = sm + kOffP;
  uint8_t* o_stage = sm + kOffStage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kOffMisc);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;                // every issuer's last S of the item done with q
  uint64_t* c_full = bars + 2;                 // [kStages]
  uint64_t* t_done = c_full + kStages;         // [kStages] O product of the stage's tile done (frees it)
  uint64_t* s_full = t_done + kStages;         // [kSBufs] all four S partials written
  uint64_t* s_free = s_full + kSBufs;          // [kSBufs]
  uint64_t* p_full = s_free + kSBufs;          // [kPBufs]
  uint64_t* o_free = p_full + kPBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_free + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hgroups = a.nh / kHeads;
  const int items = a.rows * hgroups;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, kIssuers);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&c_full[s], kProducers);
      mbar_init(&t_done[s], 1);
    }
    for (int s = 0; s < kSBufs; ++s) {
      mbar_init(&s_full[s], kIssuers);
      mbar_init(&s_free[s], 4);
    }
    for (int s = 0; s < kPBufs; ++s) mbar_init(&p_full[s], 4);
    mbar_init(o_free, 4);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmQ);
  }
  if (warp == 8) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_prologue_done();
  const uint32_t tmem = *tmem_slot;

  if (warp < 8) {
    // ------------------------------------------------------------ producers (warps 0-7)
    // thread -> column piece c16 = tid % 64 of rows tid / 64 + 4 i (i = 0..7) of every tile
    const int tid = threadIdx.x, c16 = tid & 63, r0 = tid >> 6;
    uint32_t g = 0, qw = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < items && ok; it += gridDim.x) {
      if (warp_aborted(abort_flag)) break;
      const int row = a.rows - 1 - it / hgroups, hg = it % hgroups;
      long long base;
      int avail;
      row_entries(a.rm, row, base, avail);
      const long long n_ent = rowmap_entries(a.rm, a.rows);
      const int* ir = a.idx + (long long)row * a.topk;
      const int ntiles = mqa_ntiles(ir, a.topk, avail);
      if (ntiles == 0) continue;
      if (tid == 0) {
        if (!mbar_wait(q_empty, (qw & 1) ^ 1)) {
          *abort_flag = 1;
        } else {
          mbar_arrive_expect_tx(q_full, (uint32_t)kQBytes);
          for (int kc = 0; kc < 8; ++kc) tma_load_3d(&tmQ, q_full, q_s + kc * kQChunk, 64 * kc, 64 * hg, row);
        }
      }
      ++qw;
      // slots of this thread's rows, one tile ahead: the index loads of tile
      // j + 1 are in flight while tile j waits for its stage
      int sn[kTile / 4];
#pragma unroll
      for (int i = 0; i < kTile / 4; ++i) {
        const int e = r0 + 4 * i;
        sn[i] = e < a.topk ? __ldg(ir + e) : -1;
      }
      for (int j = 0; j < ntiles; ++j, ++g) {
        const int st = (int)(g % kStages);
        int s[kTile / 4];
#pragma unroll
        for (int i = 0; i < kTile / 4; ++i) {
          s[i] = sn[i];
          const int e = (j + 1) * kTile + r0 + 4 * i;
          sn[i] = (j + 1 < ntiles && e < a.topk) ? __ldg(ir + e) : -1;
        }
        if (!warp_wait(&t_done[st], ((g / kStages) & 1) ^ 1)) { ok = false; break; }
        uint8_t* cst = c_s + st * kCBytes + (c16 >> 3) * kCChunk;
#pragma unroll
        for (int i = 0; i < kTile / 4; ++i) {
          const int r = r0 + 4 * i;
          const bool v = s[i] >= 0 && s[i] < avail && dcheck(base + s[i] < n_ent);
          if (c16 == 0 && !v && s[i] != -1) flag_status(kStatusBadIndex);
          const __nv_bfloat16* src = v ? a.C + (base + s[i]) * kC + c16 * 8 : a.C;
          cp_async16(cst + sw128(r, c16 & 7), src, v ? 16u : 0u);
        }
        cp_async_arrive_noinc(&c_full[st]);
      }
    }
    if (!ok && lane == 0) *abort_flag = 1;
    cp_async_wait_all();
  } else if (warp < 12) {
    // ------------------------------------------------------------ S issuers (warps 8-11, lane 0 issues)
    const int iw = warp - 8;
    constexpr uint32_t idS = idesc_bf16_f32(64, kTile);
    const uint64_t qd0 = sdesc_k_sw128(smem_u32(q_s));
    const uint64_t cd0 = sdesc_k_sw128(smem_u32(c_s));   // stages as K-major operands
    // this issuer's S partial: channels 128 iw .. + 127 (K chunks 2 iw and 2 iw + 1)
    const uint32_t s_col = tmem + kColS + 32u * (uint32_t)(iw >> 1) + ((uint32_t)(16 * (iw & 1)) << 16);
    uint32_t g = 0, qw = 0;
    for (int it = blockIdx.x; it < items; it += gridDim.x) {
      if (warp_aborted(abort_flag)) break;
      const int row = a.rows - 1 - it / hgroups;
      long long base;
      int avail;
      row_entries(a.rm, row, base, avail);
      const int ntiles = mqa_ntiles(a.idx + (long long)row * a.topk, a.topk, avail);
      if (ntiles == 0) continue;
      int ok = 1;
      if (lane == 0) {
        if (!mbar_wait(q_full, qw & 1)) {
          ok = 0;
        } else {
          tc_fence_after();
          for (int j = 0; j < ntiles; ++j) {
            const uint32_t gj = g + j;
            const int st = (int)(gj % kStages), sb = (int)(gj % kSBufs);
            if (!mbar_wait(&c_full[st], (gj / kStages) & 1) ||
                !mbar_wait(&s_free[sb], ((gj / kSBufs) & 1) ^ 1)) {
              ok = 0;
              break;
            }
            fence_proxy_async_smem();
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 2; ++kk)
#pragma unroll
              for (int ks = 0; ks < 4; ++ks) {
                const int kc = 2 * iw + kk;
                mma_bf16(s_col + 64u * (uint32_t)sb, desc_add(qd0, kc * kQChunk + ks * 32),
                         desc_add(cd0, st * kCBytes + kc * kCChunk + ks * 32), idS, (kk | ks) != 0 ? 1u : 0u);
              }
            mma_commit(&s_full[sb]);
            if (j == ntiles - 1) mma_commit(q_empty);
          }
        }
      }
      ok = __shfl_sync(kFull, ok, 0);
      if (!ok) {
        if (lane == 0) *abort_flag = 1;
        break;
      }
      ++qw;
      g += ntiles;
    }
  } else if (warp == 12) {
    // ------------------------------------------------------------ O issuer (warp 12, lane 0 issues)
    // The stage of a tile is released after its O product, which is issued
    // only once P is written, i.e. after all four S partials have completed.
    constexpr uint32_t idO = idesc_bf16_f32_bmn(64, 256);
    const uint64_t od0 = sdesc_mn_sw128(smem_u32(c_s), kCChunk, 1024);  // stages as MN-major operands
    const uint64_t pd0 = sdesc_k_sw64(smem_u32(p_s));
    uint32_t g = 0, oi = 0;
    for (int it = blockIdx.x; it < items; it += gridDim.x) {
      if (warp_aborted(abort_flag)) break;
      const int row = a.rows - 1 - it / hgroups;
      long long base;
      int avail;
      row_entries(a.rm, row, base, avail);
      const int ntiles = mqa_ntiles(a.idx + (long long)row * a.topk, a.topk, avail);
      if (ntiles == 0) continue;
      int ok = 1;
      if (lane == 0) {
        for (int j = 0; j < ntiles; ++j) {
          const uint32_t gj = g + j;
          const int st = (int)(gj % kStages), pb = (int)(gj % kPBufs);
          if (!mbar_wait(&p_full[pb], (gj / kPBufs) & 1) ||
              (j == 0 && !mbar_wait(o_free, (oi & 1) ^ 1))) {   // previous item's O stored
            ok = 0;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int hh = 0; hh < 2; ++hh)
#pragma unroll
            for (int ks = 0; ks < kTile / 16; ++ks)
              mma_bf16(tmem + ((uint32_t)(16 * hh) << 16) + kColO, desc_add(pd0, pb * kPBytes + ks * 32),
                       desc_add(od0, st * kCBytes + 4 * hh * kCChunk + ks * 2048), idO,
                       (j > 0 || ks > 0) ? 1u : 0u);
          mma_commit(&t_done[st]);
        }
      }
      ok = __shfl_sync(kFull, ok, 0);
      if (!ok) {
        if (lane == 0) *abort_flag = 1;
        break;
      }
      ++oi;
      g += ntiles;
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue (warps 13-16)
    const int sub = warp & 3;                  // TMEM lane quarter of this warp
    const int hrow = 16 * sub + (lane & 15);   // head row (within the group)
    const int half = lane >> 4;                // S: entries 16 half .. + 15 of a tile; O: channels 256 half ..
    const uint32_t lane_base = (uint32_t)(32 * sub) << 16;
    uint8_t* ostage = o_stage + (warp - 13) * (32 * 128);   // this warp's 32 staging rows
    uint32_t g = 0;
    for (int it = blockIdx.x; it < items; it += gridDim.x) {
      if (warp_aborted(abort_flag)) break;
      const int row = a.rows - 1 - it / hgroups, hg = it % hgroups;
      long long base;
      int avail;
      row_entries(a.rm, row, base, avail);
      const int* ir = a.idx + (long long)row * a.topk;
      const int ntiles = mqa_ntiles(ir, a.topk, avail);
      if (ntiles == 0) {   // nothing visible: the attention output is zero
        __nv_bfloat16* orow = a.O + (long long)row * a.ld_O + (long long)(hg * kHeads + hrow) * kC + half * 256;
        const uint4 z = make_uint4(0, 0, 0, 0);
        for (int i = 0; i < 32; ++i) reinterpret_cast<uint4*>(orow)[i] = z;
        continue;
      }
      float m_run = -INFINITY, l_run = 0.f;    // l_run: this lane's half of the normaliser
      bool ok = true;
      int sidx = lane < a.topk ? __ldg(ir + lane) : -1;   // slot of this lane in tile 0
      for (int j = 0; j < ntiles; ++j) {
        const uint32_t gj = g + j;
        const int sb = (int)(gj % kSBufs), pb = (int)(gj % kPBufs);
        // validity of this tile's 32 slots; the next tile's slot is fetched meanwhile
        const uint32_t vmask = __ballot_sync(kFull, sidx >= 0 && sidx < avail);
        {
          const int e = (j + 1) * kTile + lane;
          sidx = (j + 1 < ntiles && e < a.topk) ? __ldg(ir + e) : -1;
        }
        if (!warp_wait(&s_full[sb], (gj / kSBufs) & 1)) { ok = false; break; }
        tc_fence_after();
        // partials of issuers `half` (x) and `half + 2` (y) for all 32 entries of head hrow
        float x[kTile], y[kTile];
        tmem_ld_32x32b_x32_pair(tmem + lane_base + kColS + 64u * (uint32_t)sb,
                                tmem + lane_base + kColS + 64u * (uint32_t)sb + 32u, x, y);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[sb]);
        // S of this lane's 16 entries: own two partials plus the partner lane's two
        float sv[16];
        float tmax = -INFINITY;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const float mine = half ? x[16 + k] + y[16 + k] : x[k] + y[k];
          const float other = half ? x[k] + y[k] : x[16 + k] + y[16 + k];
          const float sk = mine + __shfl_xor_sync(kFull, other, 16);
          sv[k] = ((vmask >> (16 * half + k)) & 1u) ? sk * a.scale_log2 : -INFINITY;
          tmax = fmaxf(tmax, sv[k]);
        }
        tmax = fmaxf(tmax, __shfl_xor_sync(kFull, tmax, 16));
        const float m_new = fmaxf(m_run, tmax);
        const bool grow = m_new > m_run + 8.f;   // also true on the first finite tile
        const float m_use = grow ? m_new : m_run;
        // P of this lane's 16 entries (bf16) and their sum
        float sum = 0.f;
        uint4 pk[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          uint32_t w[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float x0 = sv[8 * u + 2 * q], x1 = sv[8 * u + 2 * q + 1];
            const float p0 = x0 == -INFINITY ? 0.f : ex2_approx_f32(x0 - m_use);
            const float p1 = x1 == -INFINITY ? 0.f : ex2_approx_f32(x1 - m_use);
            sum += p0 + p1;
            __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
            w[q] = *reinterpret_cast<uint32_t*>(&h2);
          }
          pk[u] = make_uint4(w[0], w[1], w[2], w[3]);
        }
        if (__any_sync(kFull, grow && j > 0)) {
          // rescale O: the O products of the earlier tiles must have completed
          const uint32_t gp = gj - 1;
          if (!warp_wait(&t_done[gp % kStages], (gp / kStages) & 1)) { ok = false; break; }
          tc_fence_after();
          const float alpha = grow ? ex2_approx_f32(m_run - m_new) : 1.f;   // 2^-inf = 0 when nothing was seen
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
        l_run += sum;
        // P rows, once the P buffer's previous reader (tile gj - kPBufs) is done
        if (gj >= (uint32_t)kPBufs) {
          const uint32_t gp = gj - kPBufs;
          if (!warp_wait(&t_done[gp % kStages], (gp / kStages) & 1)) { ok = false; break; }
        }
        uint8_t* prow = p_s + pb * kPBytes;
        *reinterpret_cast<uint4*>(prow + sw64(hrow, 2 * half)) = pk[0];
        *reinterpret_cast<uint4*>(prow + sw64(hrow, 2 * half + 1)) = pk[1];
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[pb]);
      }
      if (!ok) {
        if (lane == 0) *abort_flag = 1;
        break;
      }
      // epilogue: O / l in four passes of 64 channels per lane (channels
      // 64 p .. for the lanes of half 0, 256 + 64 p .. for half 1).  Each
      // pass goes through this warp's 32 staging rows (row = lane) and leaves
      // as whole 128-byte rows: 4 rows per warp store instead of 32 pieces.
      const float l = l_run + __shfl_xor_sync(kFull, l_run, 16);
      const uint32_t glast = g + ntiles - 1;
      if (!warp_wait(&t_done[glast % kStages], (glast / kStages) & 1)) {
        if (lane == 0) *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* obase = a.O + (long long)row * a.ld_O + (long long)(hg * kHeads + 16 * sub) * kC;
#pragma unroll 1
      for (int p = 0; p < 4; ++p) {
        float v0[32], v1[32];
        tmem_ld_32x32b_x32_pair(tmem + lane_base + kColO + 64u * (uint32_t)p,
                                tmem + lane_base + kColO + 64u * (uint32_t)p + 32u, v0, v1);
        if (p == 3) {   // O is in registers: the next item's O products may start
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(o_free);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float* vv = u < 4 ? v0 : v1;
          Vec16<__nv_bfloat16> pkv;
#pragma unroll
          for (int q = 0; q < 8; ++q) pkv.e[q] = __float2bfloat16_rn(vv[8 * (u & 3) + q] * inv);
          *reinterpret_cast<uint4*>(ostage + sw128(lane, u)) = pkv.u;
        }
        __syncwarp();
        // staging row r holds head 16 sub + r % 16, channels 256 (r / 16) + 64 p ..
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = 4 * i + (lane >> 3), u = lane & 7;
          const uint4 val = *reinterpret_cast<const uint4*>(ostage + sw128(r, u));
          *reinterpret_cast<uint4*>(obase + (r & 15) * kC + 256 * (r >> 4) + 64 * p + 8 * u) = val;
        }
        __syncwarp();
      }
      g += ntiles;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace csa
