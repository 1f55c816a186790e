// H-side projection with the compression fused into its epilogue, eqs. (1),
// (2), the indexer-key projections, (3), (4), (5) and (7) of "Compressed
// Sparse Attention" (cnblogs), on the sm_100a tensor cores.
//
// One persistent GEMM D[T, N] = H[T, d] . W1^T over two kinds of 256-column
// tiles:
//   * compression tiles: 64 channels of one key set (C^Comp or K^IComp) as
//     the four column blocks [C^a | C^b | Z^a | Z^b] of those channels (four
//     64-row TMA boxes of the packed weights per stage, so the packed layout
//     is the plain one).  Their epilogue never stores C or Z: it rounds the
//     accumulators to bf16 (the storage point of the unfused path), stages
//     them in shared memory and compresses every entry whose 2m-row window
//     (its own block and the block before) lies inside the 128-row tile,
//     with the same per-channel arithmetic as the stand-alone compression
//     kernel, so C^Comp and K^IComp are bit-identical to it.
//   * plain tiles: the c^Q and w^I columns, stored as the plain GEMM stores
//     them (bf16 c^Q rows, fp32 w^I).
// Entries whose window straddles a row-tile boundary: both tiles next to the
// boundary write their 2m rows nearest to it into a small halo buffer, make
// them visible device-wide and count their arrival on the boundary's
// counter; the tile that arrives second compresses the straddling entries
// from the halo rows and resets the counter.  No tile ever waits for
// another (no spin-wait across CTAs).
//
// Warp roles (192 threads, one CTA per SM) as in the plain projection GEMM:
// warp 0 TMA producer, warp 1 TMEM owner and MMA issuer, warps 2-5 epilogue.
// Two TMEM accumulators of 256 columns.  All waits are bounded.
#pragma once
#include "compress.cuh"
#include "gemm_tcgen05.cuh"
#include "sm100.cuh"

namespace csa {

struct ProjCompressArgs {
  int M, K;                       // tokens, d
  int m;                          // compression block (== template M_BLK)
  int c, cI;                      // key widths (multiples of 64)
  int n_cg;                       // channel groups: c/64 of C^Comp, then cI/64 of K^IComp
  int n_plain;                    // plain column tiles (256 wide) over columns [plain_col0, plain_col0 + plain_N)
  int plain_col0, plain_N;
  int group_m;                    // tile order: groups of group_m row tiles
  GemmOut out;                    // plain columns, col0 relative to plain_col0
  const float* Ba; const float* Bb;     // [m, c] fp32
  const float* BaI; const float* BbI;   // [m, cI] fp32
  __nv_bfloat16* Ccomp;           // [total_blocks, c]
  __nv_bfloat16* KIcomp;          // [total_blocks, cI]
  const int* cu_seqlens; const int* cu_blocks;
  int nseq, total_blocks;
  __nv_bfloat16* halo;            // [(m_tiles + 1) * n_cg][4m rows][256]
  int* counters;                  // [(m_tiles + 1) * n_cg], zero on entry
};

namespace pcx {
constexpr int BM = 128, BN = 256, BK = 64, kStages = 4;
constexpr int A_BYTES = BM * BK * 2, B_BYTES = BN * BK * 2, STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int BOX_BYTES = 64 * BK * 2;          // one 64-row box of B
constexpr int STAGE_OUT = 128 * 256;            // 128 rows x 256 B: compression staging / plain-store staging
constexpr int MAX_ENT = 128;                    // entries per tile (m = 1)
constexpr int MISC = 1536;
constexpr size_t SMEM = 1024 + (size_t)kStages * STAGE_BYTES + STAGE_OUT + MISC;
}  // namespace pcx

// byte offset of the 16-byte unit u (0..15) of staged row r (256 B per row),
// XOR-swizzled so that rows read at the same unit spread over the banks
__device__ __forceinline__ uint32_t pcx_off(int r, int u) { return (uint32_t)(r * 256 + ((u ^ (r & 15)) << 4)); }

// Whether global token row `row` closes a block of its sequence; if so, the
// global entry index, whether the entry has a block before it, and the first
// row of its window (the block before, or the block itself at i = 0).
__device__ __forceinline__ bool pcx_entry(const ProjCompressArgs& a, int row, int& entry, bool& has_prev,
                                          int& wstart) {
  if (row >= a.M) return false;
  int lo = 0, hi = a.nseq;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (a.cu_seqlens[mid] <= row) lo = mid; else hi = mid;
  }
  const int t = row - a.cu_seqlens[lo];
  const int L = a.cu_seqlens[lo + 1] - a.cu_seqlens[lo];
  if ((t + 1) % a.m != 0 || t + 1 > a.m * (L / a.m)) return false;
  const int i = (t + 1) / a.m - 1;
  entry = a.cu_blocks[lo] + i;
  if (entry < 0 || entry >= a.total_blocks || i >= a.cu_blocks[lo + 1] - a.cu_blocks[lo]) {
    flag_status(kStatusMetadata);
    return false;
  }
  has_prev = i > 0;
  wstart = row - (has_prev ? 2 * a.m : a.m) + 1;
  return true;
}

// Compresses 8 channels (ch0 .. ch0 + 7 of channel group cg's 64) of one
// entry from 2m staged rows.  rows_at(r) gives the byte address of the
// 256-column bf16 row r ([C^a | C^b | Z^a | Z^b] x 64 channels) in the
// generic address space together with its swizzle key; here the staging is
// either shared memory (swizzled) or the halo buffer (plain).
template <int MB>
__device__ __forceinline__ void pcx_compress8(const ProjCompressArgs& a, int cg, int ch0, int entry, bool has_prev,
                                              const uint4* za, const uint4* ca, const uint4* zb, const uint4* cb) {
  const bool main = cg < a.c / 64;
  const int w = main ? a.c : a.cI;
  const int chg = (main ? cg : cg - a.c / 64) * 64 + ch0;   // channel within the key set
  const float* Ba = main ? a.Ba : a.BaI;
  const float* Bb = main ? a.Bb : a.BbI;
  float res[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    float la[MB], lb[MB], c_a[MB], c_b[MB];
#pragma unroll
    for (int r = 0; r < MB; ++r) {
      const uint32_t* zaw = reinterpret_cast<const uint32_t*>(&za[r]);
      const uint32_t* caw = reinterpret_cast<const uint32_t*>(&ca[r]);
      const uint32_t* zbw = reinterpret_cast<const uint32_t*>(&zb[r]);
      const uint32_t* cbw = reinterpret_cast<const uint32_t*>(&cb[r]);
      const float zav = (e & 1) ? bf16_hi(zaw[e >> 1]) : bf16_lo(zaw[e >> 1]);
      const float cav = (e & 1) ? bf16_hi(caw[e >> 1]) : bf16_lo(caw[e >> 1]);
      la[r] = zav + __ldg(Ba + r * w + chg + e);
      c_a[r] = cav;
      if (has_prev) {
        const float zbv = (e & 1) ? bf16_hi(zbw[e >> 1]) : bf16_lo(zbw[e >> 1]);
        const float cbv = (e & 1) ? bf16_hi(cbw[e >> 1]) : bf16_lo(cbw[e >> 1]);
        lb[r] = zbv + __ldg(Bb + r * w + chg + e);
        c_b[r] = cbv;
      } else {
        lb[r] = 0.f;
        c_b[r] = 0.f;
      }
    }
    res[e] = compress_channel<MB>(la, lb, c_a, c_b, has_prev);
  }
  Vec16<__nv_bfloat16> pk;
#pragma unroll
  for (int e = 0; e < 8; ++e) pk.e[e] = __float2bfloat16_rn(res[e]);
  if (!dcheck(entry >= 0 && entry < a.total_blocks)) return;
  __nv_bfloat16* dst = main ? a.Ccomp + (long long)entry * a.c + chg : a.KIcomp + (long long)entry * a.cI + chg;
  *reinterpret_cast<uint4*>(dst) = pk.u;
}

template <int MB>
__global__ void __launch_bounds__(192, 1)
    proj_compress_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                            ProjCompressArgs a) {
  using namespace sm100;
  using namespace pcx;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* smA = smem;
  uint8_t* smB = smem + kStages * A_BYTES;
  uint8_t* stg = smem + kStages * STAGE_BYTES;                  // STAGE_OUT bytes
  uint8_t* misc = stg + STAGE_OUT;
  int2* ent = reinterpret_cast<int2*>(misc);                     // [MAX_ENT] (entry, local row | has_prev << 8)
  int* wcount = reinterpret_cast<int*>(misc + MAX_ENT * 8);      // [4] entries found by each epilogue warp
  volatile int* wflag = wcount + 4;                              // [4] per-warp wait outcomes, [4] abort, [5..6] fixups
  uint64_t* full = reinterpret_cast<uint64_t*>(misc + MAX_ENT * 8 + 64);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_tiles = (a.M + BM - 1) / BM;
  const int n_tiles = a.n_cg + a.n_plain;
  const int k_blocks = (a.K + BK - 1) / BK;
  const int total = m_tiles * n_tiles;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int q = 0; q < 2; ++q) {
      mbar_init(&tfull[q], 1);
      mbar_init(&tempty[q], 4);
    }
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_prologue_done();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {  // ---------------- TMA producer: A box of 128 rows, B as four 64-row boxes
      int stage = 0;
      uint32_t phase = 0;
      for (int tile = blockIdx.x; tile < total && !*abort_flag; tile += gridDim.x) {
        int mt, nt;
        gemm_tile_coords(tile, m_tiles, n_tiles, a.group_m, mt, nt);
        int brow[4];
        if (nt < a.n_cg) {
          const bool main = nt < a.c / 64;
          const int w = main ? a.c : a.cI, base = main ? 0 : 4 * a.c, g = main ? nt : nt - a.c / 64;
#pragma unroll
          for (int j = 0; j < 4; ++j) brow[j] = base + j * w + 64 * g;
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j) brow[j] = a.plain_col0 + (nt - a.n_cg) * BN + 64 * j;
        }
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1)) { *abort_flag = 1; break; }
          mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
          tma_load_2d(&tmA, &full[stage], smA + stage * A_BYTES, kb * BK, mt * BM);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            tma_load_2d(&tmB, &full[stage], smB + stage * B_BYTES + j * BOX_BYTES, kb * BK, brow[j]);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // ---------------- MMA issuer
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int tile = blockIdx.x; tile < total && !*abort_flag; tile += gridDim.x) {
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1)) { *abort_flag = 1; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(&full[stage], phase)) { *abort_flag = 1; break; }
          tc_fence_after();
          const uint64_t ad = sdesc_k_sw128(smem_u32(smA + stage * A_BYTES));
          const uint64_t bd = sdesc_k_sw128(smem_u32(smB + stage * B_BYTES));
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            mma_bf16(d_tmem, desc_add(ad, k * 32), desc_add(bd, k * 32), idesc, (kb != 0 || k != 0) ? 1u : 0u);
          mma_commit(&empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
        mma_commit(&tfull[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
    }
  } else {  // ---------------- epilogue warps 2..5 (128 threads; thread = TMEM lane = tile row)
    // The four warps meet at named barriers (bar.sync 1, 128), so every
    // decision that could end the loop (the CTA's abort flag, a wait that ran
    // out) is agreed among them first: each warp posts its view in shared
    // memory, and all four act on the same combined value.
    const int sub = warp & 3;
    const int et = threadIdx.x - 64;            // 0..127
    const int r = sub * 32 + lane;              // tile row of this thread
    const int HR = 2 * MB;                      // halo rows on each side of a boundary
    auto epi_sync = [] { asm volatile("bar.sync 1, 128;" ::: "memory"); };
    // bounded wait of every epilogue warp on `bar`; true only if all four saw it complete
    auto epi_wait = [&](uint64_t* bar, uint32_t parity) {
      const bool ok = warp_wait(bar, parity);
      if (lane == 0) wflag[sub] = ok ? 1 : 0;
      epi_sync();
      const bool all = wflag[0] && wflag[1] && wflag[2] && wflag[3];
      epi_sync();
      return all;
    };
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      if (et == 0) wflag[4] = *abort_flag;
      epi_sync();
      const bool aborted = wflag[4] != 0;
      epi_sync();
      if (aborted) break;
      int mt, nt;
      gemm_tile_coords(tile, m_tiles, n_tiles, a.group_m, mt, nt);
      const int row = mt * BM + r;
      if (nt >= a.n_cg) {
        // ---------------- plain tile: c^Q (bf16, staged whole-row stores) and w^I (fp32)
        if (!epi_wait(&tfull[acc], acc_phase)) { *abort_flag = 1; break; }
        tc_fence_after();
        uint8_t* stage_out = stg + (warp - 2) * (32 * 128);
#pragma unroll 1
        for (int ch = 0; ch < BN / 64; ++ch) {
          float v0[32], v1[32];
          const uint32_t ta = tmem_base + ((uint32_t)(sub * 32) << 16) + (uint32_t)(acc * BN + ch * 64);
          tmem_ld_32x32b_x32_pair(ta, ta + 32u, v0, v1);
          const int c0 = (nt - a.n_cg) * BN + ch * 64;   // column within the plain part
          const int sidx = staged_segment(a.out, c0, a.plain_N);
          if (sidx < 0) {
            if (row < a.M && c0 < a.plain_N) store_chunk32<__nv_bfloat16>(a.out, row, c0, a.plain_N, v0);
            if (row < a.M && c0 + 32 < a.plain_N) store_chunk32<__nv_bfloat16>(a.out, row, c0 + 32, a.plain_N, v1);
            continue;
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const float* vv = u < 4 ? v0 : v1;
            Vec16<__nv_bfloat16> pk;
#pragma unroll
            for (int e = 0; e < 8; ++e) pk.e[e] = __float2bfloat16_rn(vv[8 * (u & 3) + e]);
            *reinterpret_cast<uint4*>(stage_out + r_sw128(lane, u)) = pk.u;
          }
          __syncwarp();
          const OutSeg& sg = a.out.seg[sidx];
          __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(sg.ptr) + (c0 - sg.col0);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int rr = 4 * i + (lane >> 3), u = lane & 7;
            const long long orow = (long long)mt * BM + sub * 32 + rr;
            const uint4 val = *reinterpret_cast<const uint4*>(stage_out + r_sw128(rr, u));
            if (orow < a.M) *reinterpret_cast<uint4*>(dst + orow * sg.ld + 8 * u) = val;
          }
          __syncwarp();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
        continue;
      }
      // ---------------- compression tile (channel group nt)
      // (0) the entries whose whole window lies in this tile, listed in shared memory
      {
        int entry = 0, ws = 0;
        bool hp = false;
        const bool mine = pcx_entry(a, row, entry, hp, ws) && ws >= mt * BM;
        const unsigned bal = __ballot_sync(0xffffffffu, mine);
        if (lane == 0) wcount[sub] = __popc(bal);
        epi_sync();
        int off = 0;
        for (int q = 0; q < sub; ++q) off += wcount[q];
        if (mine) ent[off + __popc(bal & ((1u << lane) - 1u))] = make_int2(entry, r | (hp ? 256 : 0));
      }
      if (!epi_wait(&tfull[acc], acc_phase)) { *abort_flag = 1; break; }
      tc_fence_after();
      const int n_ent = wcount[0] + wcount[1] + wcount[2] + wcount[3];
      const bool top_halo = r < HR, bot_halo = r >= BM - HR;
      __nv_bfloat16* halo_cg_top = a.halo + ((size_t)mt * a.n_cg + nt) * (size_t)(2 * HR) * BN;
      __nv_bfloat16* halo_cg_bot = a.halo + ((size_t)(mt + 1) * a.n_cg + nt) * (size_t)(2 * HR) * BN;
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        // (1) this thread's row: 32 channels of each of C^a, C^b, Z^a, Z^b,
        // rounded to bf16 and staged (16-byte unit u = set * 4 + channel octet)
        const uint32_t tl = tmem_base + ((uint32_t)(sub * 32) << 16) + (uint32_t)(acc * BN + 32 * h);
#pragma unroll 1
        for (int set = 0; set < 4; set += 2) {
          float v0[32], v1[32];
          tmem_ld_32x32b_x32_pair(tl + 64u * set, tl + 64u * (set + 1), v0, v1);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            Vec16<__nv_bfloat16> p0, p1;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              p0.e[e] = __float2bfloat16_rn(v0[8 * q + e]);
              p1.e[e] = __float2bfloat16_rn(v1[8 * q + e]);
            }
            *reinterpret_cast<uint4*>(stg + pcx_off(r, set * 4 + q)) = p0.u;
            *reinterpret_cast<uint4*>(stg + pcx_off(r, (set + 1) * 4 + q)) = p1.u;
            if (row < a.M && (top_halo || bot_halo)) {
              // halo row: [C^a | C^b | Z^a | Z^b] x 64 channels, plain layout
              __nv_bfloat16* hr = top_halo ? halo_cg_top + (size_t)(HR + r) * BN
                                           : halo_cg_bot + (size_t)(r - (BM - HR)) * BN;
              *reinterpret_cast<uint4*>(hr + set * 64 + 32 * h + 8 * q) = p0.u;
              *reinterpret_cast<uint4*>(hr + (set + 1) * 64 + 32 * h + 8 * q) = p1.u;
            }
          }
        }
        if (h == 1) {   // the accumulator is in registers / shared memory now
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[acc]);
        }
        epi_sync();
        // (2) entries x channel octets of this half
        for (int wk = et; wk < n_ent * 4; wk += 128) {
          const int2 e = ent[wk >> 2];
          const int q = wk & 3, rl = e.y & 255;
          const bool hp = (e.y >> 8) != 0;
          uint4 za[MB], ca[MB], zb[MB], cb[MB];
#pragma unroll
          for (int rr = 0; rr < MB; ++rr) {
            const int ra = rl - MB + 1 + rr, rb = rl - 2 * MB + 1 + rr;
            za[rr] = *reinterpret_cast<const uint4*>(stg + pcx_off(ra, 8 + q));
            ca[rr] = *reinterpret_cast<const uint4*>(stg + pcx_off(ra, q));
            if (hp) {
              zb[rr] = *reinterpret_cast<const uint4*>(stg + pcx_off(rb, 12 + q));
              cb[rr] = *reinterpret_cast<const uint4*>(stg + pcx_off(rb, 4 + q));
            } else {
              zb[rr] = make_uint4(0, 0, 0, 0);
              cb[rr] = make_uint4(0, 0, 0, 0);
            }
          }
          pcx_compress8<MB>(a, nt, 32 * h + 8 * q, e.x, hp, za, ca, zb, cb);
        }
        epi_sync();
      }
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      // (3) boundaries: arrive on the counters of the boundaries next to this
      // tile; the second arrival compresses the entries straddling it
      __threadfence();
      epi_sync();
      if (et < 2) {
        const int b = et == 0 ? mt : mt + 1;
        int last = 0;
        if (b > 0 && b < m_tiles) last = atomicAdd(&a.counters[b * a.n_cg + nt], 1) == 1;
        wflag[5 + et] = last;
      }
      epi_sync();
      const int do_top = wflag[5], do_bot = wflag[6];
      epi_sync();
#pragma unroll 1
      for (int side = 0; side < 2; ++side) {
        if (!(side == 0 ? do_top : do_bot)) continue;
        __threadfence();
        const int b = side == 0 ? mt : mt + 1;
        const int R = b * BM;
        const __nv_bfloat16* hb = a.halo + ((size_t)b * a.n_cg + nt) * (size_t)(2 * HR) * BN;   // rows R - HR ..
        // straddling entries: last row in [R, R + 2m - 2], window start < R;
        // work item = (candidate last row, channel octet of 64)
        for (int wk = et; wk < (2 * MB - 1) * 8; wk += 128) {
          const int e_row = R + wk / 8, q = wk % 8;
          int entry = 0, ws = 0;
          bool hp = false;
          if (!pcx_entry(a, e_row, entry, hp, ws) || ws >= R) continue;
          const int hl = e_row - (R - HR);                   // halo row of the entry's last token
          uint4 za[MB], ca[MB], zb[MB], cb[MB];
#pragma unroll
          for (int rr = 0; rr < MB; ++rr) {
            const __nv_bfloat16* ra = hb + (size_t)(hl - MB + 1 + rr) * BN + 8 * q;
            za[rr] = __ldcg(reinterpret_cast<const uint4*>(ra + 128));
            ca[rr] = __ldcg(reinterpret_cast<const uint4*>(ra));
            if (hp) {
              const __nv_bfloat16* rb = hb + (size_t)(hl - 2 * MB + 1 + rr) * BN + 8 * q;
              zb[rr] = __ldcg(reinterpret_cast<const uint4*>(rb + 192));
              cb[rr] = __ldcg(reinterpret_cast<const uint4*>(rb + 64));
            } else {
              zb[rr] = make_uint4(0, 0, 0, 0);
              cb[rr] = make_uint4(0, 0, 0, 0);
            }
          }
          pcx_compress8<MB>(a, nt, 8 * q, entry, hp, za, ca, zb, cb);
        }
        if (et == 0) atomicExch(&a.counters[b * a.n_cg + nt], 0);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace csa
