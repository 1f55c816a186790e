// Tensor-core projection GEMM for sm_100a:  D[M, N] = A[M, K] . B[N, K]^T,
// bf16 operands, fp32 accumulation in TMEM, routed epilogue (gemm_simt.cuh's
// GemmOut).  This carries eqs. (1), (2), (5), (7) (A = H, B = packed H-side
// weights) and eqs. (6), (10) (A = c^Q, B = packed up-projections) of
// "Compressed Sparse Attention" (cnblogs).
//
// Persistent, warp-specialised CTA (one per SM, 192 threads):
//   warp 0      TMA producer: 128 x 64 A tiles and BN x 64 B tiles, both
//               K-major with 128-byte swizzle, into a kStages-deep ring;
//   warp 1      allocates TMEM; one thread issues tcgen05.mma (M = 128,
//               N = BN, K = 16) and commits stage releases / tile completions;
//   warps 2..5  epilogue: tcgen05.ld of their 32 TMEM lanes, conversion, and
//               stores routed to the output segments: bf16 columns go through
//               a per-warp shared-memory transpose and leave as whole 128-byte
//               rows (four rows per warp store).
// Two TMEM accumulators (2 x BN columns) let the epilogue of tile i overlap
// the main loop of tile i+1.  Tiles are visited M-fastest so that the CTAs
// running at one time share the same few B (weight) column blocks in L2.
// Every wait is bounded (sm100::mbar_wait); a wait that runs out records a
// timeout in the status word and the CTA leaves its loop.
#pragma once
#include "gemm_simt.cuh"
#include "sm100.cuh"

namespace csa {

struct TcGemmArgs {
  int M, N, K;
  GemmOut out;
  int transpose_out;   // 1: D[i][j] is stored at output row j, column i (swap-AB use)
  int group_m;         // tile order: groups of group_m row tiles, each group's tiles column by column
  // Split of K (swap-AB use only): k_split > 1 gives every tile k_split work
  // units over equal ranges of K blocks; each stores its fp32 sum for rows
  // r < M at part[(ks * N + j) * Mpad + r] (Mpad = row tiles x 128) instead of
  // `out`, and gemm_split_reduce_kernel adds the slices in order.
  int k_split;
  float* part;
};

// Tile `tile` of the visiting order -> (row tile, column tile).  Within a
// group of group_m row tiles the row tile runs fastest, so the CTAs running
// at one time share a few column blocks of B; with group_m = m_tiles this is
// plain row-fastest order.  Smaller groups keep the A rows of a group and
// all of B resident in L2 when A is too large to stay there.
__device__ __forceinline__ void gemm_tile_coords(int tile, int m_tiles, int n_tiles, int group_m, int& mt, int& nt) {
  const int per_group = group_m * n_tiles;
  const int grp = tile / per_group;
  const int r = tile - grp * per_group;
  const int gm = min(group_m, m_tiles - grp * group_m);
  mt = grp * group_m + r % gm;
  nt = r / gm;
}

template <int BN, int kStages>
struct TcGemmCfg {
  static constexpr int BM = 128, BK = 64;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = 2 * BN <= 256 ? 256 : 512;   // two accumulators (power of two)
  static constexpr int OUT_STAGE = 4 * 32 * 128;  // epilogue staging: 32 rows x 128 B per epilogue warp
  static constexpr size_t SMEM =
      1024 /*align slack*/ + (size_t)kStages * STAGE_BYTES + OUT_STAGE + 256 /*barriers*/;
};

// byte offset of 16-byte piece u (0..7) of row r in 128-byte rows, XOR-swizzled
// so that a warp writing one piece of 32 rows spreads over the banks
__device__ __forceinline__ uint32_t r_sw128(int r, int u) { return (uint32_t)(r * 128 + ((u ^ (r & 7)) << 4)); }

template <typename T>
__device__ __forceinline__ void store_chunk32(const GemmOut& o, long long row, int col0, int N, const float* v) {
  // fast path: the 32 columns lie in one segment and are in range
  for (int s = 0; s < o.nseg; ++s) {
    const OutSeg& sg = o.seg[s];
    if (col0 >= sg.col0 && col0 + 32 <= sg.col0 + sg.ncols && col0 + 32 <= N) {
      const long long off = row * sg.ld + (col0 - sg.col0);
      const uintptr_t addr = reinterpret_cast<uintptr_t>(sg.ptr) + (uintptr_t)off * (sg.f32 ? 4 : sizeof(T));
      if (addr % 16) break;   // unaligned destination: per-element stores below
      if (sg.f32) {
        float4* p = reinterpret_cast<float4*>(static_cast<float*>(sg.ptr) + off);
#pragma unroll
        for (int q = 0; q < 8; ++q) p[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
      } else {
        uint4* p = reinterpret_cast<uint4*>(static_cast<T*>(sg.ptr) + off);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          Vec16<T> pk;
#pragma unroll
          for (int e = 0; e < 8; ++e) pk.e[e] = from_f32<T>(v[8 * q + e]);
          p[q] = pk.u;
        }
      }
      return;
    }
  }
#pragma unroll
  for (int j = 0; j < 32; ++j)
    if (col0 + j < N) store_out<T>(o, row, col0 + j, v[j]);
}

// The bf16 segment that holds output columns [c0, c0 + 64) in full, with
// 16-byte aligned rows there (or -1): those columns can leave through the
// staged, coalesced path.
__device__ __forceinline__ int staged_segment(const GemmOut& o, int c0, int N) {
  if (c0 + 64 > N) return -1;
#pragma unroll
  for (int s = 0; s < kMaxSeg; ++s) {
    if (s >= o.nseg) break;
    const OutSeg& sg = o.seg[s];
    if (sg.f32 || c0 < sg.col0 || c0 + 64 > sg.col0 + sg.ncols) continue;
    const bool aligned = (reinterpret_cast<uintptr_t>(sg.ptr) % 16) == 0 && sg.ld % 8 == 0 && (c0 - sg.col0) % 8 == 0;
    return aligned ? s : -1;
  }
  return -1;
}

template <int BN, int kStages>
__global__ void __launch_bounds__(192, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, TcGemmArgs g) {
  using Cfg = TcGemmCfg<BN, kStages>;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* smA = smem;
  uint8_t* smB = smem + kStages * Cfg::A_BYTES;
  uint8_t* smOut = smem + kStages * Cfg::STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(smOut + Cfg::OUT_STAGE);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_tiles = (g.M + Cfg::BM - 1) / Cfg::BM;
  const int n_tiles = (g.N + BN - 1) / BN;
  const int k_blocks = (g.K + Cfg::BK - 1) / Cfg::BK;
  const int kbs = (k_blocks + g.k_split - 1) / g.k_split;   // K blocks per work unit
  const int total = m_tiles * n_tiles * g.k_split;          // work units: (tile, K slice)

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
    }
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_prologue_done();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {  // ---------------- TMA producer
      int stage = 0;
      uint32_t phase = 0;
      for (int unit = blockIdx.x; unit < total && !*abort_flag; unit += gridDim.x) {
        const int tile = unit / g.k_split, kb0 = (unit % g.k_split) * kbs, kb1 = min(k_blocks, kb0 + kbs);
        int mt, nt;
        gemm_tile_coords(tile, m_tiles, n_tiles, g.group_m, mt, nt);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1)) { *abort_flag = 1; break; }
          mbar_arrive_expect_tx(&full[stage], Cfg::STAGE_BYTES);
          tma_load_2d(&tmA, &full[stage], smA + stage * Cfg::A_BYTES, kb * Cfg::BK, mt * Cfg::BM);
          tma_load_2d(&tmB, &full[stage], smB + stage * Cfg::B_BYTES, kb * Cfg::BK, nt * BN);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // ---------------- MMA issuer
      constexpr uint32_t idesc = idesc_bf16_f32(Cfg::BM, BN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int unit = blockIdx.x; unit < total && !*abort_flag; unit += gridDim.x) {
        const int kb0 = (unit % g.k_split) * kbs, kb1 = min(k_blocks, kb0 + kbs);
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1)) { *abort_flag = 1; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase)) { *abort_flag = 1; break; }
          tc_fence_after();
          const uint64_t ad = sdesc_k_sw128(smem_u32(smA + stage * Cfg::A_BYTES));
          const uint64_t bd = sdesc_k_sw128(smem_u32(smB + stage * Cfg::B_BYTES));
#pragma unroll
          for (int k = 0; k < Cfg::BK / 16; ++k)
            mma_bf16(d_tmem, desc_add(ad, k * 32), desc_add(bd, k * 32), idesc, (kb != kb0 || k != 0) ? 1u : 0u);
          mma_commit(&empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
        mma_commit(&tfull[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
    }
  } else {  // ---------------- epilogue warps 2..5
    // 64 columns per TMEM wait.  Where the 64 columns go to one bf16 segment,
    // each thread converts its row into this warp's 32 staging rows (row =
    // lane) and the warp writes them out as whole 128-byte rows, four rows
    // per store instruction; other columns (fp32 w^I, ragged edges, the
    // transposed decode form) are stored per thread.
    const int sub = warp & 3;   // TMEM lane quarter this warp may access
    uint8_t* stage_out = smOut + (warp - 2) * (32 * 128);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int unit = blockIdx.x; unit < total && !*abort_flag; unit += gridDim.x) {
      const int tile = unit / g.k_split, ks = unit % g.k_split;
      int mt, nt;
      gemm_tile_coords(tile, m_tiles, n_tiles, g.group_m, mt, nt);
      if (!mbar_wait(&tfull[acc], acc_phase)) { *abort_flag = 1; break; }
      tc_fence_after();
      const int r = mt * Cfg::BM + sub * 32 + lane;
#pragma unroll 1
      for (int ch = 0; ch < BN / 64; ++ch) {
        float v0[32], v1[32];
        const uint32_t ta = tmem_base + ((uint32_t)(sub * 32) << 16) + (uint32_t)(acc * BN + ch * 64);
        tmem_ld_32x32b_x32_pair(ta, ta + 32u, v0, v1);
        const int c0 = nt * BN + ch * 64;
        if (g.k_split > 1) {   // this K slice's fp32 sum, column c0 + j of row r at part[(ks N + c0 + j) Mpad + r]
          if (r < g.M) {
            float* dst = g.part + (size_t)ks * g.N * ((size_t)m_tiles * Cfg::BM) + r;
            const size_t ld = (size_t)m_tiles * Cfg::BM;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (c0 + j < g.N) dst[(size_t)(c0 + j) * ld] = v0[j];
              if (c0 + 32 + j < g.N) dst[(size_t)(c0 + 32 + j) * ld] = v1[j];
            }
          }
          continue;
        }
        if (g.transpose_out) {
          // D[r][c0 + j] goes to output row c0 + j, column r: one segment
          // per thread (its column), consecutive lanes write consecutive
          // columns of the same output row
          if (r < g.M) {
            int sidx = -1;
#pragma unroll
            for (int s = 0; s < kMaxSeg; ++s)
              if (s < g.out.nseg && r >= g.out.seg[s].col0 && r < g.out.seg[s].col0 + g.out.seg[s].ncols) sidx = s;
            if (sidx >= 0) {
              const OutSeg& sg = g.out.seg[sidx];
              const long long col = r - sg.col0;
              if (sg.f32) {
                float* dst = static_cast<float*>(sg.ptr) + col;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                  if (c0 + j < g.N) dst[(long long)(c0 + j) * sg.ld] = v0[j];
                  if (c0 + 32 + j < g.N) dst[(long long)(c0 + 32 + j) * sg.ld] = v1[j];
                }
              } else {
                __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(sg.ptr) + col;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                  if (c0 + j < g.N) dst[(long long)(c0 + j) * sg.ld] = __float2bfloat16_rn(v0[j]);
                  if (c0 + 32 + j < g.N) dst[(long long)(c0 + 32 + j) * sg.ld] = __float2bfloat16_rn(v1[j]);
                }
              }
            }
          }
          continue;
        }
        const int sidx = staged_segment(g.out, c0, g.N);
        if (sidx < 0) {
          if (r < g.M && c0 < g.N) store_chunk32<__nv_bfloat16>(g.out, r, c0, g.N, v0);
          if (r < g.M && c0 + 32 < g.N) store_chunk32<__nv_bfloat16>(g.out, r, c0 + 32, g.N, v1);
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
        const OutSeg& sg = g.out.seg[sidx];
        __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(sg.ptr) + (c0 - sg.col0);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int rr = 4 * i + (lane >> 3), u = lane & 7;
          const long long row = (long long)mt * Cfg::BM + sub * 32 + rr;
          const uint4 val = *reinterpret_cast<const uint4*>(stage_out + r_sw128(rr, u));
          if (row < g.M) *reinterpret_cast<uint4*>(dst + row * sg.ld + 8 * u) = val;
        }
        __syncwarp();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

// The K slices of a split swap-AB GEMM added in slice order (the same sum
// whatever the timing of the slices) and stored as that GEMM stores its
// output: D[r][j] at output row j, column r, through the segments of `out`.
__global__ void gemm_split_reduce_kernel(const float* part, int k_split, int M, int Mpad, int N, GemmOut out) {
  pdl_prologue_done();
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)N * M) return;
  const int j = (int)(i / M), r = (int)(i % M);
  float acc = 0.f;
  for (int q = 0; q < k_split; ++q) acc += part[((size_t)q * N + j) * Mpad + r];
  store_out<__nv_bfloat16>(out, j, r, acc);
}

}  // namespace csa
