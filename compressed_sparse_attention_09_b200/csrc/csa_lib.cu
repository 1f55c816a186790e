// libcsa: the C ABI of include/csa.h.  Host code here validates arguments,
// carves the caller's workspace and enqueues the kernels of the other files
// of this directory on the caller's stream; every step of the path is one of
// those kernels.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#ifdef CSA_NVTX
#include <nvtx3/nvToolsExt.h>
#endif

#include "../../include/csa.h"
#include "common.cuh"
#include "compress.cuh"
#include "decode_q8.cuh"
#include "gemm_simt.cuh"
#include "gemm_tcgen05.cuh"
#include "indexer_simt.cuh"
#include "indexer_tcgen05.cuh"
#include "mqa_simt.cuh"
#include "mqa_tcgen05.cuh"
#include "pack.cuh"
#include "proj_compress_tcgen05.cuh"
#include "selfcheck.cuh"

using namespace csa;
using bf16 = __nv_bfloat16;

namespace {

constexpr size_t kAlign = 1024;     // internal sub-buffer alignment
constexpr size_t kPtrAlign = 256;   // required alignment of caller buffers
inline size_t align_up(size_t x, size_t a = kAlign) { return (x + a - 1) / a * a; }
inline int round_up_int(int x, int a) { return (x + a - 1) / a * a; }

std::atomic<uint64_t> g_launches{0};

// Follows every kernel launch: counts it and maps a launch error.
#define CSA_CHECK_LAUNCH()                                      \
  do {                                                          \
    g_launches.fetch_add(1, std::memory_order_relaxed);         \
    if (cudaGetLastError() != cudaSuccess) return CSA_ERR_CUDA; \
  } while (0)

// Launch with programmatic stream serialization: the kernel may be scheduled
// while the previous kernel on the stream finishes, and overlaps its
// prologue with that kernel's tail.  Every kernel launched this way calls
// pdl_prologue_done() (common.cuh) before its first global-memory access.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args... args) {
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr;
  memset(&attr, 0, sizeof(attr));
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// NVTX ranges around each stage's launches (host side), compiled in only
// with -DCSA_NVTX so that a profiler timeline shows the stages by name.
#ifdef CSA_NVTX
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};
#define CSA_RANGE(name) NvtxRange csa_nvtx_range(name)
#else
#define CSA_RANGE(name) ((void)0)
#endif

size_t elem_size(const csa_dims* d) { return d->dtype == CSA_BF16 ? 2 : 4; }

// Host-side shape checks shared by every entry point.
csa_status check_dims(const csa_dims* d) {
  if (!d) return CSA_ERR_INVALID_ARG;
  if (d->d <= 0 || d->c <= 0 || d->m <= 0 || d->cI <= 0 || d->nhI <= 0 || d->nh <= 0 ||
      d->dc <= 0 || d->topk <= 0)
    return CSA_ERR_INVALID_ARG;
  if (d->dtype != CSA_F32 && d->dtype != CSA_BF16) return CSA_ERR_INVALID_ARG;
  if (d->m != 1 && d->m != 2 && d->m != 4 && d->m != 8) return CSA_ERR_UNSUPPORTED;
  if (d->c != 64 && d->c != 128 && d->c != 256 && d->c != 512 && d->c != 1024) return CSA_ERR_UNSUPPORTED;
  if (d->cI != 32 && d->cI != 64 && d->cI != 128) return CSA_ERR_UNSUPPORTED;
  const int v = d->dtype == CSA_BF16 ? 8 : 4;  // elements per 16-byte vector
  if (d->dc % v || d->d % v) return CSA_ERR_UNSUPPORTED;
  if (d->topk > 8192) return CSA_ERR_UNSUPPORTED;
  if ((size_t)d->nhI * d->cI > 16384) return CSA_ERR_UNSUPPORTED;
  return CSA_OK;
}

// ------------------------------------------------------------------ device facts
int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cached[dev] = n > 0 ? n : 148;
  }
  return cached[dev];
}

// Scratch of the tensor-core indexer: two buffers of one row of candidate
// scores per query of an item, per CTA.  Rows are padded to a multiple of 4
// floats so that every row starts 16-byte aligned.
inline int padded_cap(int sc_cap) { return (sc_cap + 3) & ~3; }
size_t indexer_scratch_bytes(int sc_cap) { return (size_t)sm_count() * 2 * 4 * (size_t)padded_cap(sc_cap) * 4; }

// ------------------------------------------------------------------ layouts
struct PackLayout {
  int N1b;    // bf16/f32 block of the H-side output: C^a C^b Z^a Z^b C^aI C^bI Z^aI Z^bI c^Q
  int N1;     // N1b + nhI (w^I columns)
  int N1p;    // N1 padded to the tile
  int N2;     // nhI*cI + nh*c
  int N2p;
  size_t w1, w2, ba, bb, baI, bbI, total;
};

PackLayout pack_layout(const csa_dims* d) {
  PackLayout L;
  const size_t es = elem_size(d);
  L.N1b = 4 * d->c + 4 * d->cI + d->dc;
  L.N1 = L.N1b + d->nhI;
  L.N1p = round_up_int(L.N1, 256);
  L.N2 = d->nhI * d->cI + d->nh * d->c;
  L.N2p = round_up_int(L.N2, 256);
  size_t off = 0;
  L.w1 = off; off = align_up(off + (size_t)L.N1p * d->d * es);
  L.w2 = off; off = align_up(off + (size_t)L.N2p * d->dc * es);
  L.ba = off; off = align_up(off + (size_t)d->m * d->c * 4);
  L.bb = off; off = align_up(off + (size_t)d->m * d->c * 4);
  L.baI = off; off = align_up(off + (size_t)d->m * d->cI * 4);
  L.bbI = off; off = align_up(off + (size_t)d->m * d->cI * 4);
  L.total = off;
  return L;
}

// Whether the H-side projection runs with the compression in its epilogue
// (bf16, key widths in 64-channel groups).
bool fused_compress_ok(const csa_dims* d) {
  return d->dtype == CSA_BF16 && d->c % 64 == 0 && d->cI % 64 == 0 && (d->c + d->cI) / 64 <= 64;
}

// Halo rows and boundary counters of the fused projection + compression.
struct FusedLayout {
  size_t halo, counters, total;
};
FusedLayout fused_layout(const csa_dims* d, int T) {
  FusedLayout L;
  const size_t m_tiles = (size_t)(T + 127) / 128, n_cg = (size_t)(d->c + d->cI) / 64;
  L.halo = 0;
  L.counters = align_up((m_tiles + 1) * n_cg * (size_t)(4 * d->m) * 256 * 2);
  L.total = align_up(L.counters + (m_tiles + 1) * n_cg * 4);
  return L;
}

struct FwdLayout {
  size_t y1, wI, y2, ccomp, kicomp, idx, scratch, fused, total;
};

FwdLayout fwd_layout(const csa_dims* d, int T) {
  const PackLayout P = pack_layout(d);
  const size_t es = elem_size(d);
  const size_t nbmax = (size_t)(T / d->m);
  FwdLayout L;
  size_t off = 0;
  L.y1 = off; off = align_up(off + (size_t)T * P.N1b * es);
  L.wI = off; off = align_up(off + (size_t)T * d->nhI * 4);
  L.y2 = off; off = align_up(off + (size_t)T * P.N2 * es);
  L.ccomp = off; off = align_up(off + nbmax * d->c * es);
  L.kicomp = off; off = align_up(off + nbmax * d->cI * es);
  L.idx = off; off = align_up(off + (size_t)T * d->topk * 4);
  L.scratch = off; off = align_up(off + indexer_scratch_bytes(T / d->m + 1));
  L.fused = off; off = align_up(off + (fused_compress_ok(d) ? fused_layout(d, T).total : 0));
  L.total = off;
  return L;
}

inline char* at(void* base, size_t off) { return static_cast<char*>(base) + off; }

// ------------------------------------------------------------------ TMA descriptors
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Row-major bf16 matrix [outer, inner] with row stride row_bytes, read in
// boxes of box_inner (= 64, one 128-byte swizzle span) x box_outer rows.
bool make_tmap_bf16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                    uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  if (reinterpret_cast<uintptr_t>(base) % 16 || row_bytes % 16) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 tensor [d2, d1, d0] (d0 innermost) with byte strides s1 (between
// d1 rows) and s2 (between d2 slabs), read in boxes b0 x b1 x b2.
bool make_tmap_bf16_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1,
                       uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  if (reinterpret_cast<uintptr_t>(base) % 16 || s1 % 16 || s2 % 16) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {s1, s2};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Row-major byte matrix [outer, inner] (row stride row_bytes), boxes of
// box_inner bytes x box_outer rows, 128-byte swizzle.
bool make_tmap_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                  uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  if (reinterpret_cast<uintptr_t>(base) % 16 || row_bytes % 16) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp16 tensor [d2, d1, d0] as make_tmap_bf16_3d.
bool make_tmap_f16_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1,
                      uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  if (reinterpret_cast<uintptr_t>(base) % 16 || s1 % 16 || s2 % 16) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {s1, s2};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ launchers
template <int BN, int kStages>
csa_status launch_tc_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const TcGemmArgs& g, cudaStream_t st) {
  using Cfg = TcGemmCfg<BN, kStages>;
  auto k = gemm_tc_kernel<BN, kStages>;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::SMEM) != cudaSuccess)
    return CSA_ERR_CUDA;
  const int tiles = ((g.M + Cfg::BM - 1) / Cfg::BM) * ((g.N + BN - 1) / BN) * g.k_split;
  const int grid = tiles < sm_count() ? tiles : sm_count();
  if (launch_pdl(k, dim3(grid), dim3(192), Cfg::SMEM, st, ta, tb, g) != cudaSuccess) return CSA_ERR_CUDA;
  CSA_CHECK_LAUNCH();
  if (g.k_split > 1) {
    const int m_pad = ((g.M + Cfg::BM - 1) / Cfg::BM) * Cfg::BM;
    const long long n = (long long)g.N * g.M;
    if (launch_pdl(gemm_split_reduce_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, g.part, g.k_split,
                   g.M, m_pad, g.N, g.out) != cudaSuccess)
      return CSA_ERR_CUDA;
    CSA_CHECK_LAUNCH();
  }
  return CSA_OK;
}

// fp32 bytes of the K-split partial sums a swap-AB GEMM with n_out output
// features and m_rows activation rows may use (four slices).
size_t gemm_split_bytes(int n_out, int m_rows) { return (size_t)4 * round_up_int(n_out, 128) * m_rows * 4; }

// D[M, N] = A[M, K] . B[N, K]^T routed to `out`.  A: activations (row stride
// lda), B: packed K-major weights with at least round_up(N, 256) rows.
csa_status launch_gemm(const csa_dims* d, const void* A, long long lda, const void* B, long long ldb,
                       int M, int N, int K, const GemmOut& out, cudaStream_t st, float* split_ws = nullptr,
                       size_t split_ws_bytes = 0) {
  if (M == 0) return CSA_OK;
  if (d->dtype == CSA_BF16) {
    CUtensorMap ta, tb;
    TcGemmArgs g;
    g.K = K;
    g.out = out;
    g.k_split = 1;
    g.part = nullptr;
    if (M > 64) {  // activations as the M operand, 128 x BN tiles (rows past M read as zero, not stored)
      // BN = 192 where it fills the last wave and the padded columns better
      // (the packed weights are padded to 256 rows, so both widths stay in range)
      auto wave_eff = [&](int bn) {
        const long long nt = (N + bn - 1) / bn, tiles = nt * ((M + 127) / 128), sms = sm_count();
        return (double)N / (double)(nt * bn) * (double)tiles / (double)(((tiles + sms - 1) / sms) * sms);
      };
      const int BN = wave_eff(192) > 1.03 * wave_eff(256) ? 192 : 256;
      const uint64_t nrows_b = (uint64_t)round_up_int(N, 256);
      if (!make_tmap_bf16(&ta, A, K, M, lda * 2, 64, 128) || !make_tmap_bf16(&tb, B, K, nrows_b, ldb * 2, 64, BN))
        return CSA_ERR_UNSUPPORTED;
      g.M = M; g.N = N; g.transpose_out = 0;
      // A too large to stay in L2 across the column bands: visit groups of
      // row tiles, each group sweeping every column tile.  A group holds at
      // least a wave of tiles and at least ~sqrt(SMs) row tiles, so that the
      // tiles in flight form a square-ish block: each B column tile is read
      // from DRAM about once per group (a group of one row tile would sweep
      // all of B per row tile: 126 MB of W2 per 128 rows of c^Q).
      const int m_tiles = (M + 127) / 128, n_tiles = (N + BN - 1) / BN;
      const int sq = std::max(1, (int)lrint(sqrt((double)sm_count())));
      g.group_m = (size_t)M * K * 2 > ((size_t)32 << 20)
                      ? std::max(sq, (sm_count() + n_tiles - 1) / n_tiles) : m_tiles;
      if (g.group_m > m_tiles) g.group_m = m_tiles;
      return BN == 192 ? launch_tc_gemm<192, 4>(ta, tb, g, st) : launch_tc_gemm<256, 4>(ta, tb, g, st);
    }
    // few rows (decode): swap A and B so the weights fill the 128-row MMA
    // operand and the tokens are the N = 64 operand; the epilogue transposes.
    const uint64_t nrows_w = (uint64_t)round_up_int(N, 256);
    if (!make_tmap_bf16(&ta, B, K, nrows_w, ldb * 2, 64, 128) || !make_tmap_bf16(&tb, A, K, M, lda * 2, 64, 64))
      return CSA_ERR_UNSUPPORTED;
    g.M = N; g.N = M; g.transpose_out = 1;
    g.group_m = (N + 127) / 128;
    // Few weight tiles (fewer than half the SMs): split K over 4 or 2 work
    // units per tile so that more SMs stream the weights; the slices' fp32
    // sums go through split_ws and one reduction kernel.
    const int w_tiles = (N + 127) / 128, k_blocks = (K + 63) / 64;
    for (int ks = 4; split_ws && ks >= 2; ks /= 2) {
      if ((long long)w_tiles * ks <= sm_count() && k_blocks % ks == 0 && k_blocks / ks >= 4 &&
          (size_t)ks * (size_t)w_tiles * 128 * (size_t)M * 4 <= split_ws_bytes) {
        g.k_split = ks;
        g.part = split_ws;
        break;
      }
    }
    return launch_tc_gemm<64, 8>(ta, tb, g, st);
  }
  SimtGemmArgs g{A, lda, B, ldb, M, N, K, out};
  dim3 grid((N + 127) / 128, (M + 127) / 128);
  gemm_simt_kernel<float><<<grid, 256, 0, st>>>(g);
  CSA_CHECK_LAUNCH();
  return CSA_OK;
}

template <typename T, int M, int V>
void compress_launch(CompressArgs a, cudaStream_t st) {
  // one thread per (entry, group of V channels); each segment's CTAs in turn
  int blocks = 0;
  for (int s = 0; s < a.nseg; ++s) {
    a.seg[s].groups = a.seg[s].width / V;
    a.seg[s].blk0 = blocks;
    blocks += (int)(((long long)a.total_blocks * a.seg[s].groups + 255) / 256);
  }
  compress_kernel<T, M, V><<<(unsigned)blocks, 256, 0, st>>>(a);
}

csa_status launch_compress(const csa_dims* d, const CompressArgs& a, cudaStream_t st) {
  if ((long long)a.total_blocks * (a.seg[0].width + (a.nseg > 1 ? a.seg[1].width : 0)) == 0) return CSA_OK;
#define CSA_COMPRESS_CASE(MM)                                                         \
  case MM:                                                                            \
    if (d->dtype != CSA_BF16) compress_launch<float, MM, 4>(a, st);                   \
    else compress_launch<bf16, MM, 4>(a, st);                                         \
    break;
  switch (d->m) {
    CSA_COMPRESS_CASE(1)
    CSA_COMPRESS_CASE(2)
    CSA_COMPRESS_CASE(4)
    CSA_COMPRESS_CASE(8)
    default: return CSA_ERR_UNSUPPORTED;
  }
#undef CSA_COMPRESS_CASE
  CSA_CHECK_LAUNCH();
  return CSA_OK;
}

size_t indexer_smem(const csa_dims* d, int sc_cap) {
  return (size_t)(d->nhI * d->cI + d->nhI) * 4 + 256 * 4 + 40 * 4 + (size_t)sc_cap * 4;
}

constexpr size_t kMaxSmem = 227 * 1024;

template <typename T, int CI>
csa_status indexer_launch(const IndexerArgs& a, int rows, size_t smem, cudaStream_t st) {
  auto k = indexer_topk_simt_kernel<T, CI>;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return CSA_ERR_CUDA;
  k<<<rows, 256, smem, st>>>(a);
  CSA_CHECK_LAUNCH();
  return CSA_OK;
}

// Whether the tensor-core indexer covers these dims (prefill rows only).
bool indexer_tc_ok(const csa_dims* d) {
  return d->dtype == CSA_BF16 && d->m == 4 && (d->nhI == 32 || d->nhI == 64) && (d->cI == 64 || d->cI == 128);
}


csa_status launch_indexer_tc(const csa_dims* d, const IndexerArgs& a, int T, int NB, void* ws, size_t ws_bytes,
                             cudaStream_t st, bool chunk = false) {
  CSA_RANGE("A4 indexer_topk");
  const int sc_cap = padded_cap(a.sc_cap > 0 ? a.sc_cap : 1);
  if (!ws || ws_bytes < indexer_scratch_bytes(sc_cap) || reinterpret_cast<uintptr_t>(ws) % 16)
    return CSA_ERR_WORKSPACE;
  CUtensorMap tk, tq;
  const uint64_t krows = NB > 0 ? (uint64_t)NB : 1;
  if (!make_tmap_bf16(&tk, a.KI, d->cI, krows, (uint64_t)d->cI * 2, 64, idxtc::kM) ||
      !make_tmap_bf16_3d(&tq, a.qI, d->cI, d->nhI, T, (uint64_t)d->cI * 2, (uint64_t)a.ld_qI * 2, 64, d->nhI, 4))
    return CSA_ERR_UNSUPPORTED;
  IdxTcArgs t;
  t.wI = a.wI; t.ld_wI = a.ld_wI; t.idx = a.idx; t.scratch = static_cast<float*>(ws); t.sc_cap = sc_cap;
  t.topk = d->topk; t.nhI = d->nhI; t.cI = d->cI;
  t.cu_seqlens = a.rm.cu_seqlens; t.cu_blocks = a.rm.cu_blocks; t.nseq = a.rm.nseq; t.total_blocks = NB;
  t.total_tokens = T;
  t.pos0 = a.rm.pos0;
  t.chunk = chunk ? 1 : 0;
  t.q_blocks = chunk ? T / d->m : NB;   // a chunk of one sequence: its own blocks of queries
  auto kern = d->nhI == 64 ? indexer_tc_kernel<64> : indexer_tc_kernel<32>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)idxtc::kSmem) != cudaSuccess)
    return CSA_ERR_CUDA;
  const long long items = (long long)t.q_blocks + a.rm.nseq;
  const int grid = items < sm_count() ? (int)items : sm_count();
  if (launch_pdl(kern, dim3(grid), dim3(idxtc::kThreads), idxtc::kSmem, st, tk, tq, t) != cudaSuccess)
    return CSA_ERR_CUDA;
  CSA_CHECK_LAUNCH();
  return CSA_OK;
}

csa_status launch_indexer(const csa_dims* d, const IndexerArgs& a, int rows, cudaStream_t st) {
  CSA_RANGE("A4 indexer_topk");
  if (rows == 0) return CSA_OK;
  const size_t smem = indexer_smem(d, a.sc_cap);
  if (smem > kMaxSmem) return CSA_ERR_UNSUPPORTED;
  const bool b = d->dtype == CSA_BF16;
  switch (d->cI) {
    case 32: return b ? indexer_launch<bf16, 32>(a, rows, smem, st) : indexer_launch<float, 32>(a, rows, smem, st);
    case 64: return b ? indexer_launch<bf16, 64>(a, rows, smem, st) : indexer_launch<float, 64>(a, rows, smem, st);
    case 128: return b ? indexer_launch<bf16, 128>(a, rows, smem, st) : indexer_launch<float, 128>(a, rows, smem, st);
  }
  return CSA_ERR_UNSUPPORTED;
}

template <typename T, int VEC>
csa_status mqa_launch(const MqaArgs& a, int rows, cudaStream_t st) {
  const size_t smem = (size_t)a.topk * 4;
  auto k = mqa_simt_kernel<T, VEC>;
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return CSA_ERR_CUDA;
  k<<<rows, 256, smem, st>>>(a);
  CSA_CHECK_LAUNCH();
  return CSA_OK;
}

csa_status launch_mqa(const csa_dims* d, const MqaArgs& a, int rows, cudaStream_t st) {
  CSA_RANGE("A5 sparse_mqa");
  if (rows == 0) return CSA_OK;
  const bool b = d->dtype == CSA_BF16;
  if (b && d->c == mqa::kC && d->nh % mqa::kHeads == 0 && a.topk >= 1 && a.ld_q % 8 == 0 && a.ld_O % 8 == 0 &&
      reinterpret_cast<uintptr_t>(a.q) % 16 == 0 && reinterpret_cast<uintptr_t>(a.O) % 16 == 0 &&
      reinterpret_cast<uintptr_t>(a.C) % 16 == 0) {
    // tensor-core path: c = 512, heads in groups of 64, q read through a 3-D tensor map
    CUtensorMap tq;
    if (!make_tmap_bf16_3d(&tq, a.q, mqa::kC, d->nh, rows, (uint64_t)mqa::kC * 2, (uint64_t)a.ld_q * 2, 64,
                           mqa::kHeads, 1))
      return CSA_ERR_UNSUPPORTED;
    MqaTcArgs t;
    t.C = static_cast<const bf16*>(a.C); t.idx = a.idx;
    t.O = static_cast<bf16*>(a.O); t.ld_O = a.ld_O;
    t.topk = a.topk; t.nh = a.nh; t.rows = rows; t.scale_log2 = a.scale_log2; t.rm = a.rm;
    if (cudaFuncSetAttribute(mqa_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)mqa::kSmem) !=
        cudaSuccess)
      return CSA_ERR_CUDA;
    const long long items = (long long)rows * (d->nh / mqa::kHeads);
    const int grid = items < sm_count() ? (int)items : sm_count();
    if (launch_pdl(mqa_tc_kernel, dim3(grid), dim3(mqa::kThreads), mqa::kSmem, st, tq, t) != cudaSuccess)
      return CSA_ERR_CUDA;
    CSA_CHECK_LAUNCH();
    return CSA_OK;
  }
  switch (d->c / 32) {
    case 2: return b ? mqa_launch<bf16, 2>(a, rows, st) : mqa_launch<float, 2>(a, rows, st);
    case 4: return b ? mqa_launch<bf16, 4>(a, rows, st) : mqa_launch<float, 4>(a, rows, st);
    case 8: return b ? mqa_launch<bf16, 8>(a, rows, st) : mqa_launch<float, 8>(a, rows, st);
    case 16: return b ? mqa_launch<bf16, 16>(a, rows, st) : mqa_launch<float, 16>(a, rows, st);
    case 32: return b ? mqa_launch<bf16, 32>(a, rows, st) : mqa_launch<float, 32>(a, rows, st);
  }
  return CSA_ERR_UNSUPPORTED;
}

// A1: eqs. (1), (2), (5), (7) and the indexer-key projections, one GEMM
csa_status project_hidden(const csa_dims* d, const void* packed, const void* H, int T, void* Y1, float* wI,
                          cudaStream_t st, float* split_ws = nullptr, size_t split_ws_bytes = 0) {
  CSA_RANGE("A1 project_hidden");
  const PackLayout P = pack_layout(d);
  GemmOut o;
  memset(&o, 0, sizeof(o));
  o.seg[0] = {0, P.N1b, Y1, P.N1b, 0};
  o.seg[1] = {P.N1b, d->nhI, wI, d->nhI, 1};
  o.nseg = 2;
  return launch_gemm(d, H, d->d, at((void*)packed, P.w1), d->d, T, P.N1, d->d, o, st, split_ws, split_ws_bytes);
}

// A2: eqs. (6), (10) from the shared c^Q
csa_status project_query(const csa_dims* d, const void* packed, const void* cQ, long long ld_cQ, int T,
                         void* Y2, cudaStream_t st) {
  CSA_RANGE("A2 project_query");
  const PackLayout P = pack_layout(d);
  GemmOut o;
  memset(&o, 0, sizeof(o));
  o.seg[0] = {0, P.N2, Y2, P.N2, 0};
  o.nseg = 1;
  return launch_gemm(d, cQ, ld_cQ, at((void*)packed, P.w2), d->dc, T, P.N2, d->dc, o, st);
}

CompressArgs make_compress_args(const csa_dims* d, const int* cu_seqlens, const int* cu_blocks,
                                int nseq, int T, int NB) {
  CompressArgs a;
  memset(&a, 0, sizeof(a));
  a.cu_seqlens = cu_seqlens;
  a.cu_blocks = cu_blocks;
  a.nseq = nseq;
  a.total_tokens = T;
  a.total_blocks = NB;
  return a;
}

// A3 as the forward runs it: both key sets from the Y1 projection rows.
csa_status compress_kv(const csa_dims* d, const void* packed, const void* Y1, int T, const int* cu_seqlens,
                       const int* cu_blocks, int nseq, int NB, void* Cc, void* KIc, cudaStream_t st) {
  CSA_RANGE("A3 compress");
  const PackLayout P = pack_layout(d);
  const size_t es = elem_size(d);
  const int c = d->c, cI = d->cI;
  const char* y1 = static_cast<const char*>(Y1);
  CompressArgs ca = make_compress_args(d, cu_seqlens, cu_blocks, nseq, T, NB);
  ca.seg[0] = {y1, y1 + (size_t)c * es, y1 + (size_t)2 * c * es, y1 + (size_t)3 * c * es, P.N1b,
               reinterpret_cast<const float*>(at((void*)packed, P.ba)),
               reinterpret_cast<const float*>(at((void*)packed, P.bb)), c, Cc, 0, 0};
  const char* yI = y1 + (size_t)4 * c * es;
  ca.seg[1] = {yI, yI + (size_t)cI * es, yI + (size_t)2 * cI * es, yI + (size_t)3 * cI * es, P.N1b,
               reinterpret_cast<const float*>(at((void*)packed, P.baI)),
               reinterpret_cast<const float*>(at((void*)packed, P.bbI)), cI, KIc, 0, 0};
  ca.nseg = 2;
  return launch_compress(d, ca, st);
}

// A1 and A3 in one kernel: the H-side projection with the compression of
// both key sets in its epilogue (bf16, fused_compress_ok).  Writes c^Q into
// its Y1 columns (row stride N1b) and w^I; C^Comp and K^IComp directly.
csa_status project_hidden_compress(const csa_dims* d, const void* packed, const void* H, int T,
                                   const int* cu_seqlens, const int* cu_blocks, int nseq, int NB, void* Y1,
                                   float* wI, void* Cc, void* KIc, void* fws, cudaStream_t st) {
  CSA_RANGE("A1+A3 project_hidden_compress");
  if (T == 0) return CSA_OK;
  const PackLayout P = pack_layout(d);
  const FusedLayout F = fused_layout(d, T);
  CUtensorMap ta, tb;
  if (!make_tmap_bf16(&ta, H, d->d, T, (uint64_t)d->d * 2, 64, 128) ||
      !make_tmap_bf16(&tb, at((void*)packed, P.w1), d->d, P.N1p, (uint64_t)d->d * 2, 64, 64))
    return CSA_ERR_UNSUPPORTED;
  ProjCompressArgs a;
  memset(&a, 0, sizeof(a));
  a.M = T; a.K = d->d; a.m = d->m; a.c = d->c; a.cI = d->cI;
  a.n_cg = (d->c + d->cI) / 64;
  a.plain_col0 = 4 * d->c + 4 * d->cI;
  a.plain_N = d->dc + d->nhI;
  a.n_plain = (a.plain_N + pcx::BN - 1) / pcx::BN;
  if (a.plain_col0 + a.n_plain * pcx::BN > P.N1p) return CSA_ERR_UNSUPPORTED;   // B boxes stay inside the packed rows
  a.out.seg[0] = {0, d->dc, static_cast<char*>(Y1) + (size_t)a.plain_col0 * 2, P.N1b, 0};
  a.out.seg[1] = {d->dc, d->nhI, wI, d->nhI, 1};
  a.out.nseg = 2;
  a.Ba = reinterpret_cast<const float*>(at((void*)packed, P.ba));
  a.Bb = reinterpret_cast<const float*>(at((void*)packed, P.bb));
  a.BaI = reinterpret_cast<const float*>(at((void*)packed, P.baI));
  a.BbI = reinterpret_cast<const float*>(at((void*)packed, P.bbI));
  a.Ccomp = static_cast<bf16*>(Cc);
  a.KIcomp = static_cast<bf16*>(KIc);
  a.cu_seqlens = cu_seqlens; a.cu_blocks = cu_blocks; a.nseq = nseq; a.total_blocks = NB;
  a.halo = reinterpret_cast<bf16*>(at(fws, F.halo));
  a.counters = reinterpret_cast<int*>(at(fws, F.counters));
  const int m_tiles = (T + 127) / 128, n_tiles = a.n_cg + a.n_plain;
  const int sq = std::max(1, (int)lrint(sqrt((double)sm_count())));
  a.group_m = (size_t)T * d->d * 2 > ((size_t)32 << 20) ? std::max(sq, (sm_count() + n_tiles - 1) / n_tiles)
                                                        : m_tiles;
  if (a.group_m > m_tiles) a.group_m = m_tiles;
  if (cudaMemsetAsync(a.counters, 0, (size_t)(m_tiles + 1) * a.n_cg * 4, st) != cudaSuccess) return CSA_ERR_CUDA;
  const long long tiles = (long long)m_tiles * n_tiles;
  const int grid = tiles < sm_count() ? (int)tiles : sm_count();
#define CSA_PCX_CASE(MM)                                                                                 \
  case MM: {                                                                                             \
    auto k = proj_compress_tc_kernel<MM>;                                                                \
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pcx::SMEM) != cudaSuccess) \
      return CSA_ERR_CUDA;                                                                               \
    k<<<grid, 192, pcx::SMEM, st>>>(ta, tb, a);                                                          \
    break;                                                                                               \
  }
  switch (d->m) {
    CSA_PCX_CASE(1)
    CSA_PCX_CASE(2)
    CSA_PCX_CASE(4)
    CSA_PCX_CASE(8)
    default: return CSA_ERR_UNSUPPORTED;
  }
#undef CSA_PCX_CASE
  CSA_CHECK_LAUNCH();
  return CSA_OK;
}

}  // namespace

// ====================================================================== ABI
extern "C" {

const char* csa_status_string(csa_status s) {
  switch (s) {
    case CSA_OK: return "ok";
    case CSA_ERR_INVALID_ARG: return "invalid argument";
    case CSA_ERR_UNSUPPORTED: return "unsupported shape or configuration";
    case CSA_ERR_CUDA: return "CUDA runtime error";
    case CSA_ERR_DEVICE_TIMEOUT: return "a bounded device wait ran out";
    case CSA_ERR_BAD_INDEX: return "out-of-range block index seen on the device";
    case CSA_ERR_BAD_METADATA: return "inconsistent cu_seqlens / cu_blocks / cache metadata";
    case CSA_ERR_WORKSPACE: return "workspace too small";
    case CSA_ERR_DEVICE_BOUNDS: return "a debug-build index check failed on the device";
  }
  return "unknown status";
}

csa_status csa_get_device_status(void* stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return CSA_ERR_CUDA;
  unsigned v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess) return CSA_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return CSA_ERR_CUDA;
  if (v & kStatusTimeout) return CSA_ERR_DEVICE_TIMEOUT;
  if (v & kStatusBadIndex) return CSA_ERR_BAD_INDEX;
  if (v & kStatusMetadata) return CSA_ERR_BAD_METADATA;
  if (v & kStatusBounds) return CSA_ERR_DEVICE_BOUNDS;
  return CSA_OK;
}

int csa_debug_build(void) { return kDebugBuild ? 1 : 0; }

uint64_t csa_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

csa_status csa_set_wait_limit_ns(unsigned long long ns) {
  if (ns < 1000ull || ns > 60000000000ull) return CSA_ERR_INVALID_ARG;
  if (cudaMemcpyToSymbol(g_wait_ns, &ns, sizeof(ns)) != cudaSuccess) return CSA_ERR_CUDA;
  return CSA_OK;
}

csa_status csa_check_wait_timeout(unsigned long long* out, void* stream) {
  if (!out || reinterpret_cast<uintptr_t>(out) % 8) return CSA_ERR_INVALID_ARG;
  wait_selfcheck_kernel<<<1, 64, 0, (cudaStream_t)stream>>>(out);
  CSA_CHECK_LAUNCH();
  return CSA_OK;
}

int csa_hidden_row_elems(const csa_dims* d) {
  if (check_dims(d) != CSA_OK) return 0;
  return pack_layout(d).N1b;
}

int csa_query_row_elems(const csa_dims* d) {
  if (check_dims(d) != CSA_OK) return 0;
  return pack_layout(d).N2;
}

csa_status csa_project_hidden(const csa_dims* d, const void* packed, const void* H, int T, void* Y1, float* wI,
                              void* stream) {
  csa_status s = check_dims(d);
  if (s != CSA_OK) return s;
  if (!packed || !H || !Y1 || !wI || T < 0) return CSA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(packed) % kPtrAlign) return CSA_ERR_INVALID_ARG;
  return project_hidden(d, packed, H, T, Y1, wI, (cudaStream_t)stream);
}

csa_status csa_project_query(const csa_dims* d, const void* packed, const void* cQ, int ld_cQ, int T, void* Y2,
                             void* stream) {
  csa_status s = check_dims(d);
  if (s != CSA_OK) return s;
  if (!packed || !cQ || !Y2 || T < 0 || ld_cQ < d->dc) return CSA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(packed) % kPtrAlign) return CSA_ERR_INVALID_ARG;
  return project_query(d, packed, cQ, ld_cQ, T, Y2, (cudaStream_t)stream);
}

size_t csa_packed_weights_bytes(const csa_dims* d) {
  if (check_dims(d) != CSA_OK) return 0;
  return pack_layout(d).total;
}

csa_status csa_pack_weights(const csa_dims* d, const csa_weights* w, void* packed, size_t packed_bytes,
                            void* stream) {
  csa_status s = check_dims(d);
  if (s != CSA_OK) return s;
  if (!w || !packed) return CSA_ERR_INVALID_ARG;
  const void* all[] = {w->W_aKV, w->W_bKV, w->W_aZ, w->W_bZ, w->B_a, w->B_b, w->W_aKV_I, w->W_bKV_I,
                       w->W_aZ_I, w->W_bZ_I, w->B_a_I, w->B_b_I, w->W_DQ, w->W_IUQ, w->W_UQ, w->W_w};
  for (const void* p : all)
    if (!p) return CSA_ERR_INVALID_ARG;
  const PackLayout P = pack_layout(d);
  if (packed_bytes < P.total) return CSA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(packed) % kPtrAlign) return CSA_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaMemsetAsync(packed, 0, P.total, st) != cudaSuccess) return CSA_ERR_CUDA;
  const size_t es = elem_size(d);
  // H-side: rows of W1t in the order of the GEMM's output columns
  struct Part { const void* W; int in, out; char* dst; long long ld; };
  char* w1 = at(packed, P.w1);
  char* w2 = at(packed, P.w2);
  const int c = d->c, cI = d->cI;
  long long r1 = 0;
  auto row1 = [&](int n) { char* p = w1 + r1 * d->d * es; r1 += n; return p; };
  Part parts[16];
  int np = 0;
  parts[np++] = {w->W_aKV, d->d, c, row1(c), d->d};
  parts[np++] = {w->W_bKV, d->d, c, row1(c), d->d};
  parts[np++] = {w->W_aZ, d->d, c, row1(c), d->d};
  parts[np++] = {w->W_bZ, d->d, c, row1(c), d->d};
  parts[np++] = {w->W_aKV_I, d->d, cI, row1(cI), d->d};
  parts[np++] = {w->W_bKV_I, d->d, cI, row1(cI), d->d};
  parts[np++] = {w->W_aZ_I, d->d, cI, row1(cI), d->d};
  parts[np++] = {w->W_bZ_I, d->d, cI, row1(cI), d->d};
  parts[np++] = {w->W_DQ, d->d, d->dc, row1(d->dc), d->d};
  parts[np++] = {w->W_w, d->d, d->nhI, row1(d->nhI), d->d};
  parts[np++] = {w->W_IUQ, d->dc, d->nhI * cI, w2, d->dc};
  parts[np++] = {w->W_UQ, d->dc, d->nh * c, w2 + (size_t)d->nhI * cI * d->dc * es, d->dc};
  for (int i = 0; i < np; ++i) {
    const Part& p = parts[i];
    dim3 grid((p.out + 31) / 32, (p.in + 31) / 32), block(32, 8);
    if (d->dtype == CSA_BF16)
      transpose_kernel<bf16><<<grid, block, 0, st>>>(static_cast<const bf16*>(p.W), p.in, p.out,
                                                     reinterpret_cast<bf16*>(p.dst), p.ld);
    else
      transpose_kernel<float><<<grid, block, 0, st>>>(static_cast<const float*>(p.W), p.in, p.out,
                                                      reinterpret_cast<float*>(p.dst), p.ld);
    CSA_CHECK_LAUNCH();
  }
  struct Bias { const void* src; size_t off; long long n; };
  const Bias biases[4] = {{w->B_a, P.ba, (long long)d->m * c}, {w->B_b, P.bb, (long long)d->m * c},
                          {w->B_a_I, P.baI, (long long)d->m * cI}, {w->B_b_I, P.bbI, (long long)d->m * cI}};
  for (const Bias& b : biases) {
    float* dst = reinterpret_cast<float*>(at(packed, b.off));
    if (d->dtype == CSA_BF16) widen_kernel<bf16><<<64, 256, 0, st>>>(static_cast<const bf16*>(b.src), dst, b.n);
    else widen_kernel<float><<<64, 256, 0, st>>>(static_cast<const float*>(b.src), dst, b.n);
    CSA_CHECK_LAUNCH();
  }
  return CSA_OK;
}

csa_status csa_compress(const csa_dims* d, const void* Ca, const void* Cb, const void* Za, const void* Zb,
                        int ld, const float* Ba, const float* Bb, int width, const int* cu_seqlens,
                        const int* cu_blocks, int nseq, int total_tokens, int total_blocks, void* out,
                        void* stream) {
  csa_status s = check_dims(d);
  if (s != CSA_OK) return s;
  if (!Ca || !Cb || !Za || !Zb || !Ba || !Bb || !cu_seqlens || !cu_blocks || !out) return CSA_ERR_INVALID_ARG;
  if (nseq <= 0 || total_tokens < 0 || total_blocks < 0 || width <= 0 || ld < width) return CSA_ERR_INVALID_ARG;
  if (total_blocks > total_tokens / d->m) return CSA_ERR_INVALID_ARG;
  if (width % 4 || ld % 4) return CSA_ERR_UNSUPPORTED;
  const uintptr_t va = 4 * elem_size(d);   // 4-element vectors
  for (const void* p : {Ca, Cb, Za, Zb, (const void*)out})
    if (reinterpret_cast<uintptr_t>(p) % va) return CSA_ERR_UNSUPPORTED;
  if (reinterpret_cast<uintptr_t>(Ba) % 16 || reinterpret_cast<uintptr_t>(Bb) % 16) return CSA_ERR_UNSUPPORTED;
  CompressArgs a = make_compress_args(d, cu_seqlens, cu_blocks, nseq, total_tokens, total_blocks);
  a.seg[0] = {Ca, Cb, Za, Zb, ld, Ba, Bb, width, out, 0, 0};
  a.nseg = 1;
  return launch_compress(d, a, (cudaStream_t)stream);
}

csa_status csa_compress_kv(const csa_dims* d, const void* packed, const void* Y1, int T, const int* cu_seqlens,
                           const int* cu_blocks, int nseq, int total_blocks, void* Ccomp, void* KIcomp,
                           void* stream) {
  csa_status s = check_dims(d);
  if (s != CSA_OK) return s;
  if (!packed || !Y1 || !cu_seqlens || !cu_blocks || !Ccomp || !KIcomp) return CSA_ERR_INVALID_ARG;
  if (nseq <= 0 || T < 0 || total_blocks < 0 || total_blocks > T / d->m) return CSA_ERR_INVALID_ARG;
  const uintptr_t va = 4 * elem_size(d);
  for (const void* p : {Y1, (const void*)Ccomp, (const void*)KIcomp})
    if (reinterpret_cast<uintptr_t>(p) % va) return CSA_ERR_UNSUPPORTED;
  if (reinterpret_cast<uintptr_t>(packed) % kPtrAlign) return CSA_ERR_UNSUPPORTED;
  return compress_kv(d, packed, Y1, T, cu_seqlens, cu_blocks, nseq, total_blocks, Ccomp, KIcomp,
                     (cudaStream_t)stream);
}

size_t csa_project_compress_workspace_bytes(const csa_dims* d, int T) {
  if (check_dims(d) != CSA_OK || T < 0 || !fused_compress_ok(d)) return 0;
  return fused_layout(d, T).total;
}

csa_status csa_project_hidden_compress(const csa_dims* d, const void* packed, const void* H, int T,
                                       const int* cu_seqlens, const int* cu_blocks, int nseq, int total_blocks,
                                       void* Y1, float* wI, void* Ccomp, void* KIcomp, void* ws, size_t ws_bytes,
                                       void* stream) {
  csa_status s = check_dims(d);
  if (s != CSA_OK) return s;
  if (!fused_compress_ok(d)) return CSA_ERR_UNSUPPORTED;
  if (!packed || !H || !cu_seqlens || !cu_blocks || !Y1 || !wI || !Ccomp || !KIcomp || !ws) return CSA_ERR_INVALID_ARG;
  if (nseq <= 0 || T < 0 || total_blocks < 0 || total_blocks > T / d->m) return CSA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(packed) % kPtrAlign || reinterpret_cast<uintptr_t>(ws) % kPtrAlign)
    return CSA_ERR_INVALID_ARG;
  for (const void* p : {H, (const void*)Y1, (const void*)wI, (const void*)Ccomp, (const void*)KIcomp})
    if (reinterpret_cast<uintptr_t>(p) % 16) return CSA_ERR_INVALID_ARG;
  if (ws_bytes < fused_layout(d, T).total) return CSA_ERR_WORKSPACE;
  return project_hidden_compress(d, packed, H, T, cu_seqlens, cu_blocks, nseq, total_blocks, Y1, wI, Ccomp, KIcomp,
                                 ws, (cudaStream_t)stream);
}

size_t csa_indexer_workspace_bytes(const csa_dims* d, int total_tokens, int nseq, int max_seqlen) {
  if (check_dims(d) != CSA_OK || total_tokens < 0 || nseq <= 0 || max_seqlen < 0) return 0;
  return align_up(indexer_scratch_bytes(max_seqlen / d->m + 1));
}

csa_status csa_indexer_topk(const csa_dims* d, const void* qI, int ld_qI, const float* wI, int ld_wI,
                            const void* KI, const int* cu_seqlens, const int* cu_blocks, int nseq,
                            int total_tokens, int total_blocks, int max_seqlen, int* idx, void* ws,
                            size_t ws_bytes, void* stream) {
  csa_status s = check_dims(d);
  if (s != CSA_OK) return s;
  if (!qI || !wI || !KI || !cu_seqlens || !cu_blocks || !idx) return CSA_ERR_INVALID_ARG;
  if (nseq <= 0 || total_tokens < 0 || total_blocks < 0 || max_seqlen < 0) return CSA_ERR_INVALID_ARG;
  if (ld_qI < d->nhI * d->cI || ld_wI < d->nhI) return CSA_ERR_INVALID_ARG;
  const int v = 16 / (int)elem_size(d);
  if (ld_qI % v || reinterpret_cast<uintptr_t>(KI) % 16) return CSA_ERR_UNSUPPORTED;
  IndexerArgs a;
  a.qI = qI; a.ld_qI = ld_qI; a.wI = wI; a.ld_wI = ld_wI; a.KI = KI; a.idx = idx;
  a.topk = d->topk; a.nhI = d->nhI;
  a.sc_cap = max_seqlen / d->m;
  a.rm = RowMap{cu_seqlens, cu_blocks, nseq, total_blocks, nullptr, 0, d->m};
  if (indexer_tc_ok(d) && ld_qI % 8 == 0 && reinterpret_cast<uintptr_t>(qI) % 16 == 0) {
    if (total_tokens == 0) return CSA_OK;
    a.sc_cap = max_seqlen / d->m + 1;
    return launch_indexer_tc(d, a, total_tokens, total_blocks, ws, ws_bytes, (cudaStream_t)stream);
  }
  return launch_indexer(d, a, total_tokens, (cudaStream_t)stream);
}

csa_status csa_sparse_mqa(const csa_dims* d, const void* q, int ld_q, const void* Ccomp, const int* idx,
                          const int* cu_seqlens, const int* cu_blocks, int nseq, int total_tokens,
                          int total_blocks, void* O, void* stream) {
  csa_status s = check_dims(d);
  if (s != CSA_OK) return s;
  if (!q || !Ccomp || !idx || !cu_seqlens || !cu_blocks || !O) return CSA_ERR_INVALID_ARG;
  if (nseq <= 0 || total_tokens < 0 || total_blocks < 0 || ld_q < d->nh * d->c) return CSA_ERR_INVALID_ARG;
  const int v = 16 / (int)elem_size(d);
  if (ld_q % v) return CSA_ERR_UNSUPPORTED;
  MqaArgs a;
  a.q = q; a.ld_q = ld_q; a.C = Ccomp; a.idx = idx; a.O = O; a.ld_O = (long long)d->nh * d->c;
  a.topk = d->topk; a.nh = d->nh;
  a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)d->c));
  a.rm = RowMap{cu_seqlens, cu_blocks, nseq, total_blocks, nullptr, 0, d->m};
  return launch_mqa(d, a, total_tokens, (cudaStream_t)stream);
}

}  // extern "C"

// ---------------------------------------------------------------- indexer without a caller workspace
// Scratch of csa_indexer_topk_noalloc: the tensor-core indexer's per-CTA
// score rows (2 buffers x 4 rows of up to kNoAllocMaxBlocks scores for each
// of up to kNoAllocMaxCtas CTAs), held in module memory for the life of the
// process on every GPU that loads the library (20 MiB).
constexpr int kNoAllocMaxCtas = 160;
constexpr int kNoAllocMaxBlocks = 4096;
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocMaxCtas * 2 * 4 * kNoAllocMaxBlocks];

namespace {
// Device address of g_noalloc_scratch on the current device.  The host-side
// name is only a stand-in, so the address is looked up once per device (with
// that device current) and cached.
float* noalloc_scratch() {
  static std::atomic<float*> cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  float* p = cached[dev].load(std::memory_order_acquire);
  if (!p) {
    void* q = nullptr;
    if (cudaGetSymbolAddress(&q, g_noalloc_scratch) != cudaSuccess) return nullptr;
    p = static_cast<float*>(q);
    cached[dev].store(p, std::memory_order_release);
  }
  return p;
}
}  // namespace

extern "C" {

csa_status csa_indexer_topk_noalloc(const csa_dims* d, const void* qI, int ld_qI, const float* wI, int ld_wI,
                                    const void* KI, const int* cu_seqlens, const int* cu_blocks, int nseq,
                                    int total_tokens, int total_blocks, int max_seqlen, int* idx, void* stream) {
  csa_status s = check_dims(d);
  if (s != CSA_OK) return s;
  if (!qI || !wI || !KI || !cu_seqlens || !cu_blocks || !idx) return CSA_ERR_INVALID_ARG;
  if (nseq <= 0 || total_tokens < 0 || total_blocks < 0 || max_seqlen < 0) return CSA_ERR_INVALID_ARG;
  if (ld_qI < d->nhI * d->cI || ld_wI < d->nhI) return CSA_ERR_INVALID_ARG;
  if (!indexer_tc_ok(d) || ld_qI % 8 || reinterpret_cast<uintptr_t>(qI) % 16 ||
      reinterpret_cast<uintptr_t>(KI) % 16)
    return CSA_ERR_UNSUPPORTED;
  const int sc_cap = max_seqlen / d->m + 1;
  if (sc_cap > kNoAllocMaxBlocks || sm_count() > kNoAllocMaxCtas) return CSA_ERR_UNSUPPORTED;
  float* scratch = noalloc_scratch();
  if (!scratch) return CSA_ERR_CUDA;
  if (total_tokens == 0) return CSA_OK;
  IndexerArgs a;
  a.qI = qI; a.ld_qI = ld_qI; a.wI = wI; a.ld_wI = ld_wI; a.KI = KI; a.idx = idx;
  a.topk = d->topk; a.nhI = d->nhI; a.sc_cap = sc_cap;
  a.rm = RowMap{cu_seqlens, cu_blocks, nseq, total_blocks, nullptr, 0, d->m};
  return launch_indexer_tc(d, a, total_tokens, total_blocks, scratch, sizeof(g_noalloc_scratch),
                           (cudaStream_t)stream);
}

size_t csa_forward_workspace_bytes(const csa_dims* d, int total_tokens, int nseq) {
  if (check_dims(d) != CSA_OK || total_tokens < 0 || nseq <= 0) return 0;
  return fwd_layout(d, total_tokens).total;
}

}  // extern "C"

namespace {
// Records events[i] on st when a stage-event array was given (staged entries).
inline csa_status mark(void* const* events, int i, cudaStream_t st) {
  if (events && cudaEventRecord((cudaEvent_t)events[i], st) != cudaSuccess) return CSA_ERR_CUDA;
  return CSA_OK;
}

csa_status forward_impl(const csa_dims* d, const void* packed, const void* H, const int* cu_seqlens,
                        const int* cu_blocks, int nseq, int total_tokens, int total_blocks, int max_seqlen,
                        void* O, void* Ccomp_out, void* KI_out, int* idx_out, void* ws, size_t ws_bytes,
                        void* const* ev, void* stream) {
  CSA_RANGE("csa_forward");
  csa_status s = check_dims(d);
  if (s != CSA_OK) return s;
  if (!packed || !H || !cu_seqlens || !cu_blocks || !O || !ws) return CSA_ERR_INVALID_ARG;
  if (nseq <= 0 || total_tokens < 0 || total_blocks < 0 || max_seqlen < 0) return CSA_ERR_INVALID_ARG;
  if (total_blocks > total_tokens / d->m) return CSA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(ws) % kPtrAlign || reinterpret_cast<uintptr_t>(packed) % kPtrAlign)
    return CSA_ERR_INVALID_ARG;
  for (const void* p : {H, (const void*)O, (const void*)Ccomp_out, (const void*)KI_out})
    if (reinterpret_cast<uintptr_t>(p) % 16) return CSA_ERR_INVALID_ARG;
  const int T = total_tokens, NB = total_blocks;
  const FwdLayout L = fwd_layout(d, T);
  if (ws_bytes < L.total) return CSA_ERR_WORKSPACE;
  if (T == 0) return CSA_OK;
  if (max_seqlen > T) max_seqlen = T;   // no sequence is longer than the batch
  // the CUDA-core indexer holds a query's candidate scores in shared memory: a
  // bound it cannot hold is refused here, before the first launch
  if (!indexer_tc_ok(d) && indexer_smem(d, max_seqlen / d->m) > kMaxSmem) return CSA_ERR_UNSUPPORTED;
  const PackLayout P = pack_layout(d);
  cudaStream_t st = (cudaStream_t)stream;
  const size_t es = elem_size(d);
  const int c = d->c, cI = d->cI;
  char* y1 = at(ws, L.y1);
  float* wI = reinterpret_cast<float*>(at(ws, L.wI));
  char* y2 = at(ws, L.y2);
  void* Cc = Ccomp_out ? Ccomp_out : at(ws, L.ccomp);
  void* KIc = KI_out ? KI_out : at(ws, L.kicomp);
  int* idx = idx_out ? idx_out : reinterpret_cast<int*>(at(ws, L.idx));

  if ((s = mark(ev, 0, st)) != CSA_OK) return s;
  const bool fused = fused_compress_ok(d);
  // A1 (with A3 in its epilogue where the shapes allow)
  s = fused ? project_hidden_compress(d, packed, H, T, cu_seqlens, cu_blocks, nseq, NB, y1, wI, Cc, KIc,
                                      at(ws, L.fused), st)
            : project_hidden(d, packed, H, T, y1, wI, st);
  if (s != CSA_OK || (s = mark(ev, 1, st)) != CSA_OK) return s;
  s = project_query(d, packed, y1 + (size_t)(4 * c + 4 * cI) * es, P.N1b, T, y2, st);
  if (s != CSA_OK || (s = mark(ev, 2, st)) != CSA_OK) return s;
  // A3: eqs. (3), (4) for C^Comp and K^IComp in one launch (already done by A1 when fused)
  if (!fused) s = compress_kv(d, packed, y1, T, cu_seqlens, cu_blocks, nseq, NB, Cc, KIc, st);
  if (s != CSA_OK || (s = mark(ev, 3, st)) != CSA_OK) return s;
  // A4: eqs. (8), (9)
  IndexerArgs ia;
  ia.qI = y2; ia.ld_qI = P.N2; ia.wI = wI; ia.ld_wI = d->nhI; ia.KI = KIc; ia.idx = idx;
  ia.topk = d->topk; ia.nhI = d->nhI; ia.sc_cap = max_seqlen / d->m;
  ia.rm = RowMap{cu_seqlens, cu_blocks, nseq, NB, nullptr, 0, d->m};
  if (indexer_tc_ok(d)) {
    ia.sc_cap = max_seqlen / d->m + 1;   // scratch rows are sized for T / m blocks
    s = launch_indexer_tc(d, ia, T, NB, at(ws, L.scratch), L.total - L.scratch, st);
  } else {
    s = launch_indexer(d, ia, T, st);
  }
  if (s != CSA_OK || (s = mark(ev, 4, st)) != CSA_OK) return s;
  // A5: eq. (11)
  MqaArgs ma;
  ma.q = y2 + (size_t)d->nhI * cI * es; ma.ld_q = P.N2; ma.C = Cc; ma.idx = idx;
  ma.O = O; ma.ld_O = (long long)d->nh * c; ma.topk = d->topk; ma.nh = d->nh;
  ma.scale_log2 = (float)(1.4426950408889634 / sqrt((double)c));
  ma.rm = RowMap{cu_seqlens, cu_blocks, nseq, NB, nullptr, 0, d->m};
  s = launch_mqa(d, ma, T, st);
  if (s != CSA_OK) return s;
  return mark(ev, 5, st);
}
}  // namespace

extern "C" {

csa_status csa_forward(const csa_dims* d, const void* packed, const void* H, const int* cu_seqlens,
                       const int* cu_blocks, int nseq, int total_tokens, int total_blocks, int max_seqlen,
                       void* O, void* Ccomp_out, void* KI_out, int* idx_out, void* ws, size_t ws_bytes,
                       void* stream) {
  return forward_impl(d, packed, H, cu_seqlens, cu_blocks, nseq, total_tokens, total_blocks, max_seqlen, O,
                      Ccomp_out, KI_out, idx_out, ws, ws_bytes, nullptr, stream);
}

csa_status csa_forward_staged(const csa_dims* d, const void* packed, const void* H, const int* cu_seqlens,
                              const int* cu_blocks, int nseq, int total_tokens, int total_blocks, int max_seqlen,
                              void* O, void* Ccomp_out, void* KI_out, int* idx_out, void* ws, size_t ws_bytes,
                              void* const* events, void* stream) {
  if (!events) return CSA_ERR_INVALID_ARG;
  for (int i = 0; i < 6; ++i)
    if (!events[i]) return CSA_ERR_INVALID_ARG;
  return forward_impl(d, packed, H, cu_seqlens, cu_blocks, nseq, total_tokens, total_blocks, max_seqlen, O,
                      Ccomp_out, KI_out, idx_out, ws, ws_bytes, events, stream);
}

// ------------------------------------------------------------------ context-parallel prefill
}  // extern "C"

namespace {
// [0, a] and [0, b]: the single-sequence metadata of a context-parallel chunk
__global__ void cp_meta_kernel(int* cu, int* cb, int a, int b) {
  if (threadIdx.x == 0) {
    cu[0] = 0; cu[1] = a;
    cb[0] = 0; cb[1] = b;
  }
}

struct CpLayout {
  size_t meta, cc, ki, fused, y2, idx, scratch, total;
};
// Workspace of the two context-parallel calls for a chunk of T tokens whose
// queries see at most ctx / m blocks (ctx = position of the chunk's end).
CpLayout cp_layout(const csa_dims* d, int T, int ctx) {
  const PackLayout P = pack_layout(d);
  const size_t es = elem_size(d);
  const int Tp = T + d->m;   // chunk plus the halo block
  CpLayout L;
  size_t off = 0;
  L.meta = off; off = align_up(off + 16 * sizeof(int));
  L.cc = off; off = align_up(off + (size_t)(Tp / d->m + 1) * d->c * es);
  L.ki = off; off = align_up(off + (size_t)(Tp / d->m + 1) * d->cI * es);
  L.fused = off; off = align_up(off + (fused_compress_ok(d) ? fused_layout(d, Tp).total : 0));
  L.y2 = off; off = align_up(off + (size_t)T * P.N2 * es);
  L.idx = off; off = align_up(off + (size_t)T * d->topk * 4);
  L.scratch = off; off = align_up(off + indexer_scratch_bytes(ctx / d->m + 1));
  L.total = off;
  return L;
}
}  // namespace

extern "C" {

size_t csa_cp_workspace_bytes(const csa_dims* d, int T, int ctx) {
  if (check_dims(d) != CSA_OK || T <= 0 || ctx < T) return 0;
  return cp_layout(d, T, ctx).total;
}

csa_status csa_cp_compress(const csa_dims* d, const void* packed, const void* H, int T, int pos0, void* Y1,
                           float* wI, void* Ccomp_chunk, void* KIcomp_chunk, void* ws, size_t ws_bytes,
                           void* stream) {
  csa_status s = check_dims(d);
  if (s != CSA_OK) return s;
  if (!packed || !H || !Y1 || !wI || !Ccomp_chunk || !KIcomp_chunk || !ws) return CSA_ERR_INVALID_ARG;
  if (T <= 0 || pos0 < 0 || pos0 % d->m) return CSA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(ws) % kPtrAlign || reinterpret_cast<uintptr_t>(packed) % kPtrAlign)
    return CSA_ERR_INVALID_ARG;
  for (const void* p : {H, (const void*)Y1, (const void*)wI, (const void*)Ccomp_chunk, (const void*)KIcomp_chunk})
    if (reinterpret_cast<uintptr_t>(p) % 16) return CSA_ERR_INVALID_ARG;
  const CpLayout L = cp_layout(d, T, pos0 + T);
  if (ws_bytes < L.total) return CSA_ERR_WORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  const int halo = pos0 > 0 ? d->m : 0;
  const int Tp = halo + T, nb = Tp / d->m, nb_out = T / d->m;
  int* cu = reinterpret_cast<int*>(at(ws, L.meta));
  int* cb = cu + 4;
  cp_meta_kernel<<<1, 32, 0, st>>>(cu, cb, Tp, nb);
  CSA_CHECK_LAUNCH();
  // the halo block and the chunk as one sequence: its entry 0 (the halo
  // block itself, which lacks its predecessor) is dropped, entries 1.. are
  // the chunk's blocks exactly as the whole sequence would compress them
  void* Cc = at(ws, L.cc);
  void* KIc = at(ws, L.ki);
  if (fused_compress_ok(d)) {
    s = project_hidden_compress(d, packed, H, Tp, cu, cb, 1, nb, Y1, wI, Cc, KIc, at(ws, L.fused), st);
  } else {
    s = project_hidden(d, packed, H, Tp, Y1, wI, st);
    if (s == CSA_OK) s = compress_kv(d, packed, Y1, Tp, cu, cb, 1, nb, Cc, KIc, st);
  }
  if (s != CSA_OK) return s;
  const size_t es = elem_size(d), skip = (size_t)(halo / d->m);
  if (nb_out > 0) {
    if (cudaMemcpyAsync(Ccomp_chunk, static_cast<char*>(Cc) + skip * d->c * es, (size_t)nb_out * d->c * es,
                        cudaMemcpyDeviceToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(KIcomp_chunk, static_cast<char*>(KIc) + skip * d->cI * es, (size_t)nb_out * d->cI * es,
                        cudaMemcpyDeviceToDevice, st) != cudaSuccess)
      return CSA_ERR_CUDA;
  }
  return CSA_OK;
}

csa_status csa_cp_queries(const csa_dims* d, const void* packed, const void* Y1, const float* wI, int T, int pos0,
                          const void* Ccomp, const void* KIcomp, int total_blocks, void* O, int* idx_out, void* ws,
                          size_t ws_bytes, void* stream) {
  csa_status s = check_dims(d);
  if (s != CSA_OK) return s;
  if (!packed || !Y1 || !wI || !Ccomp || !KIcomp || !O || !ws) return CSA_ERR_INVALID_ARG;
  if (T <= 0 || pos0 < 0 || pos0 % d->m || total_blocks < (pos0 + T) / d->m) return CSA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(ws) % kPtrAlign || reinterpret_cast<uintptr_t>(packed) % kPtrAlign)
    return CSA_ERR_INVALID_ARG;
  for (const void* p : {Y1, (const void*)wI, (const void*)O, Ccomp, KIcomp})
    if (reinterpret_cast<uintptr_t>(p) % 16) return CSA_ERR_INVALID_ARG;
  const CpLayout L = cp_layout(d, T, pos0 + T);
  if (ws_bytes < L.total) return CSA_ERR_WORKSPACE;
  if (!indexer_tc_ok(d) && indexer_smem(d, (pos0 + T) / d->m) > kMaxSmem) return CSA_ERR_UNSUPPORTED;
  cudaStream_t st = (cudaStream_t)stream;
  const PackLayout P = pack_layout(d);
  const size_t es = elem_size(d);
  const int c = d->c, cI = d->cI, NB = total_blocks;
  int* cu = reinterpret_cast<int*>(at(ws, L.meta)) + 8;
  int* cb = cu + 4;
  cp_meta_kernel<<<1, 32, 0, st>>>(cu, cb, T, NB);
  CSA_CHECK_LAUNCH();
  char* y2 = at(ws, L.y2);
  int* idx = idx_out ? idx_out : reinterpret_cast<int*>(at(ws, L.idx));
  s = project_query(d, packed, static_cast<const char*>(Y1) + (size_t)(4 * c + 4 * cI) * es, P.N1b, T, y2, st);
  if (s != CSA_OK) return s;
  IndexerArgs ia;
  ia.qI = y2; ia.ld_qI = P.N2; ia.wI = wI; ia.ld_wI = d->nhI; ia.KI = KIcomp; ia.idx = idx;
  ia.topk = d->topk; ia.nhI = d->nhI; ia.sc_cap = (pos0 + T) / d->m;
  ia.rm = RowMap{cu, cb, 1, NB, nullptr, 0, d->m, pos0};
  if (indexer_tc_ok(d)) {
    ia.sc_cap = (pos0 + T) / d->m + 1;
    s = launch_indexer_tc(d, ia, T, NB, at(ws, L.scratch), L.total - L.scratch, st, true);
  } else {
    s = launch_indexer(d, ia, T, st);
  }
  if (s != CSA_OK) return s;
  MqaArgs ma;
  ma.q = y2 + (size_t)d->nhI * cI * es; ma.ld_q = P.N2; ma.C = Ccomp; ma.idx = idx;
  ma.O = O; ma.ld_O = (long long)d->nh * c; ma.topk = d->topk; ma.nh = d->nh;
  ma.scale_log2 = (float)(1.4426950408889634 / sqrt((double)c));
  ma.rm = RowMap{cu, cb, 1, NB, nullptr, 0, d->m, pos0};
  return launch_mqa(d, ma, T, st);
}

// ------------------------------------------------------------------ decode
int csa_ring_row_elems(const csa_dims* d) {
  if (check_dims(d) != CSA_OK) return 0;
  return 4 * d->c + 4 * d->cI;
}

namespace {
csa_status launch_append(const csa_dims* d, const void* packed, const void* rows, long long ld_rows,
                         const int* pos, void* ring, void* Ccache, void* KIcache, int* cache_len, int cap,
                         int B, cudaStream_t st, uint8_t* KIcodes = nullptr, float* KIscale = nullptr,
                         bool wait_late = false) {
  CSA_RANGE("A6 cache_append");
  if (B == 0) return CSA_OK;
  const bool q8 = KIcodes != nullptr;
  const PackLayout P = pack_layout(d);
  AppendArgs a;
  a.rows = rows; a.ld_rows = ld_rows; a.pos = pos; a.ring = ring; a.Ccache = Ccache; a.KIcache = KIcache;
  a.cache_len = cache_len;
  a.Ba = reinterpret_cast<const float*>(at((void*)packed, P.ba));
  a.Bb = reinterpret_cast<const float*>(at((void*)packed, P.bb));
  a.BaI = reinterpret_cast<const float*>(at((void*)packed, P.baI));
  a.BbI = reinterpret_cast<const float*>(at((void*)packed, P.bbI));
  a.c = d->c; a.cI = d->cI; a.cap = cap; a.ring_w = 4 * d->c + 4 * d->cI;
  a.KIcodes = KIcodes; a.KIscale = KIscale;
  a.wait_late = wait_late ? 1 : 0;
#define CSA_APPEND_CASE(MM)                                                                    \
  case MM: {                                                                                   \
    const cudaError_t e_ = q8 ? launch_pdl(cache_append_kernel<bf16, MM, true>, dim3(B), dim3(256), 0, st, a) \
                         : d->dtype == CSA_BF16                                                \
                             ? launch_pdl(cache_append_kernel<bf16, MM>, dim3(B), dim3(256), 0, st, a)       \
                             : launch_pdl(cache_append_kernel<float, MM>, dim3(B), dim3(256), 0, st, a);     \
    if (e_ != cudaSuccess) return CSA_ERR_CUDA;                                                \
    break;                                                                                     \
  }
  switch (d->m) {
    CSA_APPEND_CASE(1)
    CSA_APPEND_CASE(2)
    CSA_APPEND_CASE(4)
    CSA_APPEND_CASE(8)
    default: return CSA_ERR_UNSUPPORTED;
  }
#undef CSA_APPEND_CASE
  CSA_CHECK_LAUNCH();
  return CSA_OK;
}

struct DecLayout {
  size_t y1, wI, y2, idx, scratch, split, qf16, total;
};
DecLayout dec_layout(const csa_dims* d, int B, int cap) {
  const PackLayout P = pack_layout(d);
  const size_t es = elem_size(d);
  DecLayout L;
  size_t off = 0;
  L.y1 = off; off = align_up(off + (size_t)B * P.N1b * es);
  L.wI = off; off = align_up(off + (size_t)B * d->nhI * 4);
  L.y2 = off; off = align_up(off + (size_t)B * P.N2 * es);
  L.idx = off; off = align_up(off + (size_t)B * d->topk * 4);
  L.scratch = off; off = align_up(off + (size_t)B * (size_t)cap * 4);
  L.split = off; off = align_up(off + gemm_split_bytes(P.N1, B));   // K-split sums of the A1 projection
  L.qf16 = off; off = align_up(off + (size_t)B * d->nhI * d->cI * 2);   // q^I in fp16 (quantised key cache)
  L.total = off;
  return L;
}

// Decode rows through the tensor-core indexer: split-s scores into the
// workspace, then one selection CTA per sequence.
csa_status launch_indexer_decode_tc(const csa_dims* d, const IndexerArgs& a, int B, int cap, float* scratch,
                                    cudaStream_t st, cudaEvent_t after_scores = nullptr) {
  CSA_RANGE("A4 indexer_topk (decode)");
  CUtensorMap tk, tq;
  if (!make_tmap_bf16(&tk, a.KI, d->cI, (uint64_t)B * cap, (uint64_t)d->cI * 2, 64, idxdec::kM) ||
      !make_tmap_bf16_3d(&tq, a.qI, d->cI, d->nhI, B, (uint64_t)d->cI * 2, (uint64_t)a.ld_qI * 2, 64, d->nhI, 1))
    return CSA_ERR_UNSUPPORTED;
  IdxDecArgs t;
  t.wI = a.wI; t.ld_wI = a.ld_wI; t.pos = a.rm.pos; t.scratch = scratch; t.B = B; t.cap = cap; t.m = d->m;
  t.nhI = d->nhI; t.cI = d->cI; t.tiles_per_seq = (cap + idxdec::kM - 1) / idxdec::kM;
  if (cudaFuncSetAttribute(indexer_decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)idxdec::kSmem) != cudaSuccess)
    return CSA_ERR_CUDA;
  const long long items = (long long)B * t.tiles_per_seq;
  const int grid = items < sm_count() ? (int)items : sm_count();
  if (launch_pdl(indexer_decode_tc_kernel, dim3(grid), dim3(idxdec::kThreads), idxdec::kSmem, st, tk, tq, t) !=
      cudaSuccess)
    return CSA_ERR_CUDA;
  CSA_CHECK_LAUNCH();
  if (after_scores && cudaEventRecord(after_scores, st) != cudaSuccess) return CSA_ERR_CUDA;
  if (cudaFuncSetAttribute(decode_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dsel::kSmem) !=
      cudaSuccess)
    return CSA_ERR_CUDA;
  if (launch_pdl(decode_select_kernel, dim3(B), dim3(dsel::kThreads), dsel::kSmem, st, (const float*)scratch,
                 a.rm.pos, cap, d->m, d->topk, a.idx) != cudaSuccess)
    return CSA_ERR_CUDA;
  CSA_CHECK_LAUNCH();
  return CSA_OK;
}
// Decode rows over an E4M3 key cache: q^I to fp16, the score rows (codes
// widened in shared memory, entry scales in the epilogue), then the same
// per-sequence selection as the bf16 cache.
csa_status launch_indexer_decode_q8(const csa_dims* d, const IndexerArgs& a, const uint8_t* codes,
                                    const float* scales, int B, int cap, float* scratch, void* qf16, cudaStream_t st,
                                    cudaEvent_t after_scores = nullptr) {
  CSA_RANGE("A4 indexer_topk (decode, e4m3 keys)");
  const int w = d->nhI * d->cI;
  if (launch_pdl(bf16_to_f16_rows_kernel, dim3((unsigned)(((long long)B * w + 255) / 256)), dim3(256), 0, st,
                 static_cast<const bf16*>(a.qI), (long long)a.ld_qI, B, w, static_cast<__half*>(qf16)) != cudaSuccess)
    return CSA_ERR_CUDA;
  CSA_CHECK_LAUNCH();
  CUtensorMap tk, tq;
  if (!make_tmap_u8(&tk, codes, d->cI, (uint64_t)B * cap, (uint64_t)d->cI, 128, idxq8::kM) ||
      !make_tmap_f16_3d(&tq, qf16, d->cI, d->nhI, B, (uint64_t)d->cI * 2, (uint64_t)w * 2, 64, d->nhI, 1))
    return CSA_ERR_UNSUPPORTED;
  IdxDecQ8Args t;
  t.wI = a.wI; t.ld_wI = a.ld_wI; t.pos = a.rm.pos; t.kscale = scales; t.scratch = scratch; t.B = B; t.cap = cap;
  t.m = d->m; t.nhI = d->nhI; t.tiles_per_seq = (cap + idxq8::kM - 1) / idxq8::kM;
  if (cudaFuncSetAttribute(indexer_decode_q8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)idxq8::kSmem) != cudaSuccess)
    return CSA_ERR_CUDA;
  const long long items = (long long)B * t.tiles_per_seq;
  const int grid = items < sm_count() ? (int)items : sm_count();
  if (launch_pdl(indexer_decode_q8_kernel, dim3(grid), dim3(idxq8::kThreads), idxq8::kSmem, st, tk, tq, t) !=
      cudaSuccess)
    return CSA_ERR_CUDA;
  CSA_CHECK_LAUNCH();
  if (after_scores && cudaEventRecord(after_scores, st) != cudaSuccess) return CSA_ERR_CUDA;
  if (cudaFuncSetAttribute(decode_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dsel::kSmem) !=
      cudaSuccess)
    return CSA_ERR_CUDA;
  if (launch_pdl(decode_select_kernel, dim3(B), dim3(dsel::kThreads), dsel::kSmem, st, (const float*)scratch,
                 a.rm.pos, cap, d->m, d->topk, a.idx) != cudaSuccess)
    return CSA_ERR_CUDA;
  CSA_CHECK_LAUNCH();
  return CSA_OK;
}

// The quantised key cache's requirements: bf16 path, c^I = 128, n_h^I in {32, 64}.
bool q8_ok(const csa_dims* d) { return d->dtype == CSA_BF16 && d->cI == 128 && (d->nhI == 32 || d->nhI == 64); }
}  // namespace

csa_status csa_cache_append(const csa_dims* d, const void* packed, const void* rows, const int* pos,
                            void* ring, void* Ccache, void* KIcache, int* cache_len, int cap, int B,
                            void* stream) {
  csa_status s = check_dims(d);
  if (s != CSA_OK) return s;
  if (!packed || !rows || !pos || !ring || !Ccache || !KIcache || !cache_len) return CSA_ERR_INVALID_ARG;
  if (cap <= 0 || B < 0) return CSA_ERR_INVALID_ARG;
  return launch_append(d, packed, rows, 4 * d->c + 4 * d->cI, pos, ring, Ccache, KIcache, cache_len, cap, B,
                       (cudaStream_t)stream);
}

size_t csa_decode_workspace_bytes(const csa_dims* d, int B, int cap) {
  if (check_dims(d) != CSA_OK || B < 0 || cap <= 0) return 0;
  return dec_layout(d, B, cap).total;
}

}  // extern "C"

namespace {
csa_status decode_impl(const csa_dims* d, const void* packed, const void* h, const int* pos, void* ring,
                       void* Ccache, void* KIcache, int* cache_len, int cap, int B, void* O, int* idx_out,
                       void* ws, size_t ws_bytes, void* const* ev, void* stream, uint8_t* KIcodes = nullptr,
                       float* KIscale = nullptr) {
  CSA_RANGE("csa_decode");
  csa_status s = check_dims(d);
  if (s != CSA_OK) return s;
  const bool q8 = KIcodes != nullptr;
  if (q8) {
    if (!KIscale) return CSA_ERR_INVALID_ARG;
    if (!q8_ok(d) || reinterpret_cast<uintptr_t>(KIcodes) % 16) return CSA_ERR_UNSUPPORTED;
    KIcache = KIcodes;   // stands in for the (absent) bf16 key cache in the checks below
  }
  if (!packed || !h || !pos || !ring || !Ccache || !KIcache || !cache_len || !O || !ws) return CSA_ERR_INVALID_ARG;
  if (cap <= 0 || B < 0) return CSA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(ws) % kPtrAlign || reinterpret_cast<uintptr_t>(packed) % kPtrAlign)
    return CSA_ERR_INVALID_ARG;
  const DecLayout L = dec_layout(d, B, cap);
  if (ws_bytes < L.total) return CSA_ERR_WORKSPACE;
  if (B == 0) return CSA_OK;
  const bool idx_tc = !q8 && d->dtype == CSA_BF16 && (d->nhI == 32 || d->nhI == 64) &&
                      (d->cI == 64 || d->cI == 128) && reinterpret_cast<uintptr_t>(KIcache) % 16 == 0;
  // the CUDA-core indexer holds a row of cap scores in shared memory: refused
  // here, before the append changes any cache
  if (!q8 && !idx_tc && indexer_smem(d, cap) > kMaxSmem) return CSA_ERR_UNSUPPORTED;
  const PackLayout P = pack_layout(d);
  cudaStream_t st = (cudaStream_t)stream;
  const size_t es = elem_size(d);
  const int c = d->c, cI = d->cI;
  char* y1 = at(ws, L.y1);
  float* wI = reinterpret_cast<float*>(at(ws, L.wI));
  char* y2 = at(ws, L.y2);
  int* idx = idx_out ? idx_out : reinterpret_cast<int*>(at(ws, L.idx));
  if ((s = mark(ev, 0, st)) != CSA_OK) return s;
  s = project_hidden(d, packed, h, B, y1, wI, st, reinterpret_cast<float*>(at(ws, L.split)),
                     L.total - L.split);
  if (s != CSA_OK || (s = mark(ev, 1, st)) != CSA_OK) return s;
  s = project_query(d, packed, y1 + (size_t)(4 * c + 4 * cI) * es, P.N1b, B, y2, st);
  if (s != CSA_OK || (s = mark(ev, 2, st)) != CSA_OK) return s;
  // the append touches nothing the c^Q-side projection reads or writes: it runs beside it and
  // waits for it at its end (the projection lets it start only once the H-side rows are complete)
  s = launch_append(d, packed, y1, P.N1b, pos, ring, Ccache, KIcache, cache_len, cap, B, st, KIcodes, KIscale,
                    /*wait_late=*/true);
  if (s != CSA_OK || (s = mark(ev, 3, st)) != CSA_OK) return s;
  IndexerArgs ia;
  ia.qI = y2; ia.ld_qI = P.N2; ia.wI = wI; ia.ld_wI = d->nhI; ia.KI = KIcache; ia.idx = idx;
  ia.topk = d->topk; ia.nhI = d->nhI; ia.sc_cap = cap;
  ia.rm = RowMap{nullptr, nullptr, 0, 0, pos, cap, d->m};
  if (q8) {
    s = launch_indexer_decode_q8(d, ia, KIcodes, KIscale, B, cap, reinterpret_cast<float*>(at(ws, L.scratch)),
                                 at(ws, L.qf16), st, ev ? (cudaEvent_t)ev[4] : nullptr);
  } else if (idx_tc) {
    s = launch_indexer_decode_tc(d, ia, B, cap, reinterpret_cast<float*>(at(ws, L.scratch)), st,
                                 ev ? (cudaEvent_t)ev[4] : nullptr);
  } else {
    s = launch_indexer(d, ia, B, st);   // scores and selection in one kernel: both events after it
    if (s == CSA_OK) s = mark(ev, 4, st);
  }
  if (s != CSA_OK || (s = mark(ev, 5, st)) != CSA_OK) return s;
  MqaArgs ma;
  ma.q = y2 + (size_t)d->nhI * cI * es; ma.ld_q = P.N2; ma.C = Ccache; ma.idx = idx;
  ma.O = O; ma.ld_O = (long long)d->nh * c; ma.topk = d->topk; ma.nh = d->nh;
  ma.scale_log2 = (float)(1.4426950408889634 / sqrt((double)c));
  ma.rm = RowMap{nullptr, nullptr, 0, 0, pos, cap, d->m};
  s = launch_mqa(d, ma, B, st);
  if (s != CSA_OK) return s;
  return mark(ev, 6, st);
}
}  // namespace

extern "C" {

csa_status csa_decode(const csa_dims* d, const void* packed, const void* h, const int* pos, void* ring,
                      void* Ccache, void* KIcache, int* cache_len, int cap, int B, void* O, int* idx_out,
                      void* ws, size_t ws_bytes, void* stream) {
  return decode_impl(d, packed, h, pos, ring, Ccache, KIcache, cache_len, cap, B, O, idx_out, ws, ws_bytes,
                     nullptr, stream);
}

csa_status csa_decode_staged(const csa_dims* d, const void* packed, const void* h, const int* pos, void* ring,
                             void* Ccache, void* KIcache, int* cache_len, int cap, int B, void* O, int* idx_out,
                             void* ws, size_t ws_bytes, void* const* events, void* stream) {
  if (!events) return CSA_ERR_INVALID_ARG;
  for (int i = 0; i < 7; ++i)
    if (!events[i]) return CSA_ERR_INVALID_ARG;
  return decode_impl(d, packed, h, pos, ring, Ccache, KIcache, cache_len, cap, B, O, idx_out, ws, ws_bytes,
                     events, stream);
}

csa_status csa_quantize_keys_e4m3(const void* KI, long long ld, int n, int w, void* codes, float* scales,
                                  void* stream) {
  if (!KI || !codes || !scales || n < 0 || w <= 0 || w % 32 || ld < w) return CSA_ERR_INVALID_ARG;
  if (n == 0) return CSA_OK;
  const long long threads = (long long)n * 32;
  quantize_rows_e4m3_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, (cudaStream_t)stream>>>(
      static_cast<const bf16*>(KI), ld, n, w, static_cast<uint8_t*>(codes), scales);
  CSA_CHECK_LAUNCH();
  return CSA_OK;
}

csa_status csa_decode_q8(const csa_dims* d, const void* packed, const void* h, const int* pos, void* ring,
                         void* Ccache, void* KIcodes, float* KIscale, int* cache_len, int cap, int B, void* O,
                         int* idx_out, void* ws, size_t ws_bytes, void* stream) {
  if (!KIcodes) return CSA_ERR_INVALID_ARG;
  return decode_impl(d, packed, h, pos, ring, Ccache, nullptr, cache_len, cap, B, O, idx_out, ws, ws_bytes,
                     nullptr, stream, static_cast<uint8_t*>(KIcodes), KIscale);
}

csa_status csa_decode_q8_staged(const csa_dims* d, const void* packed, const void* h, const int* pos, void* ring,
                                void* Ccache, void* KIcodes, float* KIscale, int* cache_len, int cap, int B,
                                void* O, int* idx_out, void* ws, size_t ws_bytes, void* const* events,
                                void* stream) {
  if (!KIcodes || !events) return CSA_ERR_INVALID_ARG;
  for (int i = 0; i < 7; ++i)
    if (!events[i]) return CSA_ERR_INVALID_ARG;
  return decode_impl(d, packed, h, pos, ring, Ccache, nullptr, cache_len, cap, B, O, idx_out, ws, ws_bytes, events,
                     stream, static_cast<uint8_t*>(KIcodes), KIscale);
}

}  // extern "C"
