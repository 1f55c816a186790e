// Lightning indexer (eq. 8) and top-k selector (eq. 9) of "Compressed
// Sparse Attention" (cnblogs) on the sm_100a tensor cores, prefill form.
//
// Work item = the 4 query tokens of one compression block (m = 4): they see
// the same blocks s < floor(t/m), so they share every K^IComp tile.  Per
// 128-block tile the MMA computes
//     D[s, (q, h)] = K^IComp_s . q^I_{t_q, h}      M = 128 blocks, N = 4 x n_h^I, K = c^I
// into one of two TMEM accumulators, and the epilogue warps (one TMEM lane =
// one block s per thread) fold it straight into the index score (stored as
// its order-preserving 32-bit key)
//     I[t_q, s] = sum_h w_{t_q, h} ReLU(D[s, (q, h)])
// so the per-head products never leave the SM.  The four score rows of the
// item go to one of two per-CTA scratch buffers (written and read back
// through L2 only; the n x n/m score matrix never exists), and four
// selection warps each pick the exact top-k of one query with a warp-level
// radix select, writing its indices in ascending order (ties to the lower
// block), while the epilogue warps already fill the other buffer with the
// next item's scores.  Sequence tails (L mod 4 tokens) are extra items with
// fewer than 4 queries; items whose queries see at most k blocks keep them
// all without any MMA.
//
// Warp roles (320 threads): warp 0 TMA producer (q^I of the item once, then
// the K^IComp tiles through a kStages ring), warp 1 MMA issuer + TMEM owner,
// warps 2-5 epilogue (TMEM -> scores), warps 6-9 selection.  All waits are
// bounded.
#pragma once
#include "common.cuh"
#include "sm100.cuh"
#include "topk.cuh"

namespace csa {

struct IdxTcArgs {
  const float* wI; long long ld_wI;   // [T, nhI]
  int* idx;                           // [T, topk]
  float* scratch;                     // [gridDim, 2 buffers, 4, sc_cap]
  int sc_cap;                         // >= max blocks of any sequence
  int topk, nhI, cI;
  const int* cu_seqlens; const int* cu_blocks;
  int nseq, total_blocks, total_tokens;
  int q_blocks;                       // blocks of 4 queries (= total_blocks unless chunk)
  int pos0;                           // chunk: position of its first query
  int chunk;                          // 1: the queries are one chunk of one sequence (cu_blocks = [0, all blocks])
};

namespace idxtc {
constexpr int kM = 128;                 // blocks per tile
constexpr int kStages = 3;
constexpr int kQChunk = 256 * 128;      // [4 x nhI <= 256 rows x 64 bf16]
constexpr int kKChunk = kM * 128;       // [128 rows x 64 bf16]
constexpr int kSelChunk = 1536;         // scores staged in shared memory per selection warp
constexpr int kHistBins = 2048;         // radix histogram per selection warp (11-bit digits)
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + 2 * kQChunk;
constexpr int kOffW = kOffK + kStages * 2 * kKChunk;   // 4 warps x [4 x 64] floats
constexpr int kOffH = kOffW + 4 * 256 * 4;             // 4 warps x kHistBins counts
constexpr int kOffS = kOffH + 4 * kHistBins * 4;       // 4 warps x kSelChunk staged scores
constexpr int kOffB = kOffS + 4 * kSelChunk * 4;
constexpr size_t kSmem = 1024 + kOffB + 256;
constexpr int kThreads = 320;
}  // namespace idxtc

// Item `it` of the work list: blocks of 4 queries from the last one down,
// then one tail item per sequence.  Normally the query blocks are the
// compression blocks (q_blocks = total_blocks); for a context-parallel chunk
// of one sequence whose first query sits at position pos0 (a multiple of 4),
// query block i sees pos0/4 + i blocks of the whole sequence.  Returns false
// for an empty tail item and for an item the metadata cannot place: its
// score rows would not fit the scratch rows (more visible blocks than
// sc_cap, i.e. a max_seqlen below the real length), its queries lie outside
// [0, total_tokens) or its blocks outside [0, total_blocks).  Such an item is
// skipped by every role alike (each evaluates the same test) and
// kStatusMetadata is raised.
__device__ __forceinline__ bool idx_item(const IdxTcArgs& a, int it, int& tok0, int& nq, int& avail,
                                         long long& kbase) {
  if (it < a.q_blocks) {
    const int g = a.q_blocks - 1 - it;
    int lo = 0, hi = a.nseq;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (a.cu_blocks[mid] <= g) lo = mid; else hi = mid;
    }
    const int i = g - a.cu_blocks[lo];
    tok0 = a.cu_seqlens[lo] + 4 * i;
    nq = 4;
    avail = i + (a.pos0 >> 2);
    kbase = a.cu_blocks[lo];
    if (i < 0 || tok0 < 0 || tok0 + 4 > a.cu_seqlens[lo + 1] || a.cu_seqlens[lo + 1] > a.total_tokens ||
        avail >= a.sc_cap || kbase + avail > a.total_blocks) {
      flag_status(kStatusMetadata);
      return false;
    }
    return true;
  }
  const int b = it - a.q_blocks;
  const int L = a.cu_seqlens[b + 1] - a.cu_seqlens[b];
  nq = L & 3;
  tok0 = a.cu_seqlens[b + 1] - nq;
  avail = (L >> 2) + (a.pos0 >> 2);
  kbase = a.cu_blocks[b];
  // every sequence's tail item also checks that cu_blocks gives the sequence
  // floor(L/4) blocks (for a chunk: at least the blocks its queries see), so
  // that no block of queries goes unvisited unnoticed
  const int have = a.cu_blocks[b + 1] - kbase;
  if (L < 0 || a.cu_seqlens[b] < 0 || a.cu_seqlens[b + 1] > a.total_tokens || kbase < 0 ||
      (a.chunk ? have < avail : have != avail) || kbase + avail > a.total_blocks ||
      (nq > 0 && avail >= a.sc_cap)) {
    flag_status(kStatusMetadata);
    return false;
  }
  return nq > 0;
}

// Exact top-k of a score row by one warp, written to out[0..k) as ascending
// indices; equal scores are taken lowest index first.  The row sc[0..n)
// holds the scores' order-preserving 32-bit keys (ordered_key), written by
// the epilogue in place of the floats, so no pass converts them again (the
// rows are handled as 32-bit words: float-typed pointers only for the
// 16-byte copies).
//
// Radix select on the order-preserving 32-bit keys, most significant digit
// first, in three passes of 11, 11 and 10 bits: each pass histograms the
// digit of the keys that share the digits found so far and picks the digit
// holding the kk-th largest of them; the last pass leaves the k-th largest
// key `thr` itself and how many keys equal to it are taken.  An ordered pass
// then writes every key > thr and the first `need_eq` keys == thr.
//
// A row that fits in `buf` (kSelChunk words of shared memory) is read from
// global memory once and every pass runs on shared memory; a longer row is
// read straight into registers on every pass, kStreamVecs 16-byte loads per
// lane in flight.  Each lane takes four consecutive scores per step, so that
// four independent key/histogram chains are in flight per lane.
__device__ __forceinline__ void warp_stage_chunk(const float* src, int n, float* buf) {
  constexpr int kBatch = 8;   // 16-byte loads in flight per lane
  const int lane = threadIdx.x & 31;
  if ((reinterpret_cast<uintptr_t>(src) & 15) == 0) {
    const int n4 = n >> 2;
    for (int i0 = 0; i0 < n4; i0 += 32 * kBatch) {
      float4 r[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int i = i0 + lane + 32 * u;
        if (i < n4) r[u] = __ldcg(reinterpret_cast<const float4*>(src) + i);
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int i = i0 + lane + 32 * u;
        if (i < n4) reinterpret_cast<float4*>(buf)[i] = r[u];
      }
    }
    for (int i = (n4 << 2) + lane; i < n; i += 32) buf[i] = __ldcg(src + i);
  } else {
#pragma unroll 8
    for (int i = lane; i < n; i += 32) buf[i] = __ldcg(src + i);
  }
  __syncwarp();
}

// 16-byte loads per lane in flight when a row is read straight from global memory
constexpr int kStreamVecs = 8;

__device__ __forceinline__ int warp_incl_scan(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, v, off);
    if (lane >= off) v += t;
  }
  return v;
}

// One radix pass over the keys k of sc[0..n) with (k & mask) == prefix:
// returns the WIDTH-bit digit at `shift` that holds the kk-th largest of
// them (kk >= 1, at most their number) and, in *above, how many of them have
// a larger digit, and in *in_bin how many have the returned digit.  hist
// holds 2^WIDTH ints of shared memory.  FIRST: the first pass (mask = 0:
// every key takes part).
template <int WIDTH, bool FIRST>
__device__ __noinline__ uint32_t warp_radix_pass(const float* sc, int n, bool resident, float* buf, int* hist,
                                                 int shift, uint32_t mask, uint32_t prefix, int kk, int* above,
                                                 int* in_bin) {
  constexpr int NB = 1 << WIDTH, PER = NB / 32, SUB = PER / 32;
  constexpr unsigned kFull = 0xffffffffu;
  const int lane = threadIdx.x & 31;
#pragma unroll 4
  for (int i = lane; i < NB / 4; i += 32) reinterpret_cast<int4*>(hist)[i] = make_int4(0, 0, 0, 0);
  __syncwarp();
  if (resident) {
    // whole 16-byte vectors first, then the last n % 4 keys one per lane
    const int nv = n >> 2;
#pragma unroll 2
    for (int i = lane; i < nv; i += 32) {
      const uint4 v = reinterpret_cast<const uint4*>(buf)[i];
      const uint32_t e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (FIRST || (e[u] & mask) == prefix) atomicAdd(&hist[(e[u] >> shift) & (uint32_t)(NB - 1)], 1);
    }
    if (lane < n - 4 * nv) {
      const uint32_t key = __float_as_uint(buf[4 * nv + lane]);
      if (FIRST || (key & mask) == prefix) atomicAdd(&hist[(key >> shift) & (uint32_t)(NB - 1)], 1);
    }
  } else {
    // a row longer than the staging buffer is read straight into registers,
    // kStreamVecs 16-byte loads per lane in flight
    const uint4* src4 = reinterpret_cast<const uint4*>(sc);
    const int nv = n >> 2;
    for (int i0 = 0; i0 < nv; i0 += 32 * kStreamVecs) {
      uint4 v[kStreamVecs];
#pragma unroll
      for (int u = 0; u < kStreamVecs; ++u) {
        const int i = i0 + lane + 32 * u;
        v[u] = i < nv ? __ldcg(src4 + i) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < kStreamVecs; ++u) {
        if (i0 + lane + 32 * u < nv) {
          const uint32_t e[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
          for (int j = 0; j < 4; ++j)
            if (FIRST || (e[j] & mask) == prefix) atomicAdd(&hist[(e[j] >> shift) & (uint32_t)(NB - 1)], 1);
        }
      }
    }
    if (lane < n - 4 * nv) {
      const uint32_t key = __ldcg(reinterpret_cast<const unsigned*>(sc) + 4 * nv + lane);
      if (FIRST || (key & mask) == prefix) atomicAdd(&hist[(key >> shift) & (uint32_t)(NB - 1)], 1);
    }
  }
  __syncwarp();
  // Position p = NB - 1 - digit (p = 0 is the largest digit).  Lane L sums
  // positions [PER L, PER L + PER), visiting them in a lane-rotated order so
  // that the 32 lanes read 32 different banks.
  int tot = 0;
#pragma unroll
  for (int j = 0; j < PER; ++j) tot += hist[NB - 1 - (PER * lane + ((j + lane) & (PER - 1)))];
  int incl = tot;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(kFull, incl, off);
    if (lane >= off) incl += v;
  }
  const int excl = incl - tot;
  const int src = __ffs(__ballot_sync(kFull, excl < kk && incl >= kk)) - 1;
  const int excl_src = __shfl_sync(kFull, excl, src);
  const int kk2 = kk - excl_src;
  // within the range of lane `src`: SUB positions per lane
  const int p0 = PER * src + SUB * lane;
  int c2 = 0;
#pragma unroll
  for (int u = 0; u < SUB; ++u) c2 += hist[NB - 1 - (p0 + u)];
  int incl2 = c2;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(kFull, incl2, off);
    if (lane >= off) incl2 += v;
  }
  const int excl2 = incl2 - c2;
  const int src2 = __ffs(__ballot_sync(kFull, excl2 < kk2 && incl2 >= kk2)) - 1;
  int pos = 0, before = 0, cnt = 0;
  if (lane == src2) {
    int c = excl2;
#pragma unroll
    for (int u = 0; u < SUB; ++u) {
      const int v = hist[NB - 1 - (p0 + u)];
      if (c + v >= kk2) { pos = p0 + u; before = c; cnt = v; break; }
      c += v;
    }
  }
  pos = __shfl_sync(kFull, pos, src2);
  before = __shfl_sync(kFull, before, src2);
  cnt = __shfl_sync(kFull, cnt, src2);
  __syncwarp();
  *above = excl_src + before;
  *in_bin = cnt;
  return (uint32_t)(NB - 1 - pos);
}

__device__ __noinline__ void warp_topk_ascending(const float* sc, int n, int k, int* out, int* hist, float* buf) {
  constexpr unsigned kFull = 0xffffffffu;
  const int lane = threadIdx.x & 31;
  const bool resident = n <= idxtc::kSelChunk;
  if (resident) warp_stage_chunk(sc, n, buf);
  // When every key of the digit's bin is needed (in_bin == kk after the
  // pass), the selection is already decided: exactly the keys >= the bin's
  // lowest key value (prefix, low bits 0), and the later passes are skipped.
  // After the second pass a bin spans 2^-13 of a binade, so at prefill sizes
  // it usually holds the k-th key alone.
  int kk = k, above, in_bin;
  uint32_t prefix = warp_radix_pass<11, true>(sc, n, resident, buf, hist, 21, 0u, 0u, kk, &above, &in_bin) << 21;
  kk -= above;
  bool settled = in_bin == kk;
  if (!settled) {
    prefix |= warp_radix_pass<11, false>(sc, n, resident, buf, hist, 10, 0xFFE00000u, prefix, kk, &above, &in_bin)
              << 10;
    kk -= above;
    settled = in_bin == kk;
  }
  if (!settled) {
    prefix |= warp_radix_pass<10, false>(sc, n, resident, buf, hist, 0, 0xFFFFFC00u, prefix, kk, &above, &in_bin);
    kk -= above;
  }
  const uint32_t thr = prefix;
  const int need_eq = kk;
  // after the third pass in_bin = the number of keys equal to thr: when all
  // of them are taken (the usual case) the choice is simply key >= thr, as it
  // is for a selection settled early
  const bool all_eq = settled || need_eq == in_bin;
  int out_off = 0, eq_seen = 0;
  const unsigned lt = (1u << lane) - 1u;
  if (!resident) {
    // long row, straight from global memory: lane l takes the four keys
    // 4 (i0 + l) .. + 3 of each 128-key step, and the positions follow from a
    // prefix over the lanes' take counts (ascending index order)
    const uint4* src4 = reinterpret_cast<const uint4*>(sc);
    const int nv = n >> 2;
    for (int i0 = 0; i0 < nv; i0 += 32 * kStreamVecs) {
      uint4 v[kStreamVecs];
#pragma unroll
      for (int u = 0; u < kStreamVecs; ++u) {
        const int i = i0 + lane + 32 * u;
        v[u] = i < nv ? __ldcg(src4 + i) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < kStreamVecs; ++u) {
        const int i = i0 + lane + 32 * u;
        const bool valid = i < nv;
        const uint32_t e[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
        bool take[4];
        if (all_eq) {
#pragma unroll
          for (int j = 0; j < 4; ++j) take[j] = valid && e[j] >= thr;
        } else {
          int ceq = 0;
#pragma unroll
          for (int j = 0; j < 4; ++j) ceq += (valid && e[j] == thr) ? 1 : 0;
          const int incl_eq = warp_incl_scan(ceq);
          int eqr = eq_seen + incl_eq - ceq;   // equal keys before this lane's four
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const bool eq = valid && e[j] == thr;
            take[j] = (valid && e[j] > thr) || (eq && eqr < need_eq);
            eqr += eq ? 1 : 0;
          }
          eq_seen += __shfl_sync(kFull, incl_eq, 31);
        }
        int cnt = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) cnt += take[j] ? 1 : 0;
        const int incl = warp_incl_scan(cnt);
        int p = out_off + incl - cnt;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (take[j]) {
            if (dguard(p < k)) out[p] = 4 * i + j;
            ++p;
          }
        out_off += __shfl_sync(kFull, incl, 31);
      }
    }
    // the last n % 4 keys, one per lane
    {
      const int s = 4 * nv + lane;
      const bool in = s < n;
      const uint32_t key = in ? __ldcg(reinterpret_cast<const unsigned*>(sc) + s) : 0u;
      const bool gt = in && key > thr;
      const bool eq = in && key == thr;
      const unsigned beq = __ballot_sync(kFull, eq);
      const bool take = gt || (eq && eq_seen + __popc(beq & lt) < need_eq);
      const unsigned btk = __ballot_sync(kFull, take);
      const int p = out_off + __popc(btk & lt);
      if (take && dguard(p < k)) out[p] = s;
    }
    return;
  }
  for (int c0 = 0; c0 < n; c0 += idxtc::kSelChunk) {
    const int cn = min(idxtc::kSelChunk, n - c0);
    for (int base = 0; base < cn; base += 128) {
      // four 32-score groups: keys first (independent loads), then the
      // ordered compaction group by group
      uint32_t key[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int s = base + 32 * u + lane;
        key[u] = s < cn ? __float_as_uint(buf[s]) : 0u;
      }
      if (all_eq) {
        unsigned btk[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) btk[u] = __ballot_sync(kFull, base + 32 * u + lane < cn && key[u] >= thr);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int p = out_off + __popc(btk[u] & lt);
          if (((btk[u] >> lane) & 1u) && dguard(p < k)) out[p] = c0 + base + 32 * u + lane;
          out_off += __popc(btk[u]);
        }
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int s = base + 32 * u + lane;
          const bool gt = s < cn && key[u] > thr;
          const bool eq = s < cn && key[u] == thr;
          const unsigned beq = __ballot_sync(kFull, eq);
          const bool take = gt || (eq && eq_seen + __popc(beq & lt) < need_eq);
          const unsigned btk = __ballot_sync(kFull, take);
          const int p = out_off + __popc(btk & lt);
          if (take && dguard(p < k)) out[p] = c0 + s;
          out_off += __popc(btk);
          eq_seen += __popc(beq);
        }
      }
    }
    __syncwarp();
  }
}

// NHI = n_h^I (32 or 64; a.nhI must equal it).
template <int NHI>
__global__ void __launch_bounds__(idxtc::kThreads, 1)
    indexer_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ, IdxTcArgs a) {
  using namespace sm100;
  using namespace idxtc;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_s = sm + kOffQ;
  uint8_t* k_s = sm + kOffK;
  float* w_s = reinterpret_cast<float*>(sm + kOffW);
  int* h_s = reinterpret_cast<int*>(sm + kOffH);
  float* sel_s = reinterpret_cast<float*>(sm + kOffS);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kOffB);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;                 // [kStages]
  uint64_t* k_empty = k_full + kStages;        // [kStages]
  uint64_t* t_full = k_empty + kStages;        // [2]
  uint64_t* t_empty = t_full + 2;              // [2]
  uint64_t* sc_full = t_empty + 2;             // [2] score buffer written (4 epilogue warps)
  uint64_t* sc_free = sc_full + 2;             // [2] score buffer selected from (4 selection warps)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sc_free + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int N = 4 * NHI;                    // MMA N: (query, head) pairs
  const int kchunks = a.cI / 64;
  constexpr uint32_t tmem_cols = N <= 128 ? 256 : 512;
  const int items = a.q_blocks + a.nseq;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&t_full[s], 1);
      mbar_init(&t_empty[s], 4);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sc_full[s], 4);
      mbar_init(&sc_free[s], 4);
    }
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmQ);
  }
  if (warp == 1) tmem_alloc(tmem_slot, tmem_cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_prologue_done();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t g = 0, qi = 0;
      for (int it = blockIdx.x; it < items && !*abort_flag; it += gridDim.x) {
        int tok0, nq, avail;
        long long kbase;
        if (!idx_item(a, it, tok0, nq, avail, kbase) || avail <= a.topk) continue;
        const int ntiles = (avail + kM - 1) / kM;
        if (!mbar_wait(q_empty, (qi & 1) ^ 1)) { *abort_flag = 1; break; }
        mbar_arrive_expect_tx(q_full, (uint32_t)(kchunks * N * 128));
        for (int c = 0; c < kchunks; ++c) tma_load_3d(&tmQ, q_full, q_s + c * kQChunk, 64 * c, 0, tok0);
        ++qi;
        {
          // the next item's q^I and w^I rows go to L2 while this item runs,
          // so that its q^I load (issued only once this item's MMAs are
          // done) and its head weights come from L2
          int tok1, nq1, av1;
          long long kb1;
          const int nx = it + (int)gridDim.x;
          if (nx < items && idx_item(a, nx, tok1, nq1, av1, kb1) && av1 > a.topk) {
            for (int c = 0; c < kchunks; ++c) tma_prefetch_3d(&tmQ, 64 * c, 0, tok1);
            for (int q = 0; q < nq1; ++q)
              for (int h = 0; h < NHI; h += 32) prefetch_l2(a.wI + (long long)(tok1 + q) * a.ld_wI + h);
          }
        }
        bool ok = true;
        for (int j = 0; j < ntiles; ++j, ++g) {
          const int st = g % kStages;
          if (!mbar_wait(&k_empty[st], ((g / kStages) & 1) ^ 1)) { ok = false; break; }
          mbar_arrive_expect_tx(&k_full[st], (uint32_t)(kchunks * kKChunk));
          for (int c = 0; c < kchunks; ++c)
            tma_load_2d(&tmK, &k_full[st], k_s + (st * 2 + c) * kKChunk, 64 * c, (int)(kbase + (long long)kM * j));
        }
        if (!ok) { *abort_flag = 1; break; }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kM, N);
      uint32_t g = 0, qi = 0, acc_it = 0;
      for (int it = blockIdx.x; it < items && !*abort_flag; it += gridDim.x) {
        int tok0, nq, avail;
        long long kbase;
        if (!idx_item(a, it, tok0, nq, avail, kbase) || avail <= a.topk) continue;
        const int ntiles = (avail + kM - 1) / kM;
        if (!mbar_wait(q_full, qi & 1)) { *abort_flag = 1; break; }
        ++qi;
        bool ok = true;
        for (int j = 0; j < ntiles; ++j, ++g, ++acc_it) {
          const int st = g % kStages, acc = acc_it & 1;
          if (!mbar_wait(&k_full[st], (g / kStages) & 1) || !mbar_wait(&t_empty[acc], ((acc_it >> 1) & 1) ^ 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t kd = sdesc_k_sw128(smem_u32(k_s + st * 2 * kKChunk)), qd = sdesc_k_sw128(smem_u32(q_s));
          for (int c = 0; c < kchunks; ++c)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              mma_bf16(tmem + (uint32_t)(acc * N), desc_add(kd, c * kKChunk + ks * 32),
                       desc_add(qd, c * kQChunk + ks * 32), idesc, (c | ks) != 0);
          mma_commit(&k_empty[st]);
          mma_commit(&t_full[acc]);
        }
        if (!ok) { *abort_flag = 1; break; }
        mma_commit(q_empty);
      }
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ epilogue (warps 2-5): TMEM -> scores
    const int sub = warp & 3;            // TMEM lane quarter
    const int ew = warp - 2;             // private smem slice for the head weights
    float* w_my = w_s + ew * 256;
    const uint32_t lane_base = (uint32_t)(32 * sub) << 16;
    uint32_t acc_it = 0, wi = 0;
    for (int it = blockIdx.x; it < items; it += gridDim.x) {
      if (warp_aborted(abort_flag)) break;
      int tok0, nq, avail;
      long long kbase;
      if (!idx_item(a, it, tok0, nq, avail, kbase) || avail <= a.topk) continue;
      const int ntiles = (avail + kM - 1) / kM;
      const int buf = wi & 1;
      float* scr = a.scratch + ((size_t)blockIdx.x * 2 + buf) * 4 * a.sc_cap;
      for (int e = lane; e < 4 * NHI; e += 32) {
        const int q = e / NHI, h = e - q * NHI;
        w_my[q * 64 + h] = q < nq ? a.wI[(long long)(tok0 + q) * a.ld_wI + h] : 0.f;
      }
      __syncwarp();
      // the selection of the item that used this buffer before must be over
      if (!warp_wait(&sc_free[buf], ((wi >> 1) & 1) ^ 1)) { *abort_flag = 1; break; }
      bool ok = true;
      for (int j = 0; j < ntiles; ++j, ++acc_it) {
        const int acc = acc_it & 1;
        if (!warp_wait(&t_full[acc], (acc_it >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const int s = j * kM + 32 * sub + lane;
        // four independent packed (fp32x2) partial sums per query keep the
        // FMA chains short and fold two heads per FMA instruction
        for (int q = 0; q < nq; ++q) {
          float2 p[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) p[e] = make_float2(0.f, 0.f);
#pragma unroll 1
          for (int hc = 0; hc < NHI; hc += 32) {
            float v[32];
            tmem_ld_32x32b_x32(tmem + lane_base + (uint32_t)(acc * N + q * NHI + hc), v);
            const float4* w4 = reinterpret_cast<const float4*>(w_my + q * 64 + hc);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float4 w = w4[e];
              p[(2 * e) & 3] = __ffma2_rn(make_float2(w.x, w.y),
                                          make_float2(fmaxf(v[4 * e + 0], 0.f), fmaxf(v[4 * e + 1], 0.f)),
                                          p[(2 * e) & 3]);
              p[(2 * e + 1) & 3] = __ffma2_rn(make_float2(w.z, w.w),
                                              make_float2(fmaxf(v[4 * e + 2], 0.f), fmaxf(v[4 * e + 3], 0.f)),
                                              p[(2 * e + 1) & 3]);
            }
          }
          const float sc = ((p[0].x + p[0].y) + (p[1].x + p[1].y)) + ((p[2].x + p[2].y) + (p[3].x + p[3].y));
          if (s < avail && dcheck(s < a.sc_cap))
            __stcg(reinterpret_cast<unsigned*>(scr) + (size_t)q * a.sc_cap + s, ordered_key(sc));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&t_empty[acc]);
      }
      if (!ok) { *abort_flag = 1; break; }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sc_full[buf]);
      ++wi;
    }
  } else {
    // ------------------------------------------------------------ selection (warps 6-9): one query each
    const int q = warp - 6;
    int* hist = h_s + q * kHistBins;
    uint32_t wi = 0;
    for (int it = blockIdx.x; it < items; it += gridDim.x) {
      if (warp_aborted(abort_flag)) break;
      int tok0, nq, avail;
      long long kbase;
      if (!idx_item(a, it, tok0, nq, avail, kbase)) continue;
      if (avail <= a.topk) {   // every visible block is kept
        if (q < nq) {
          int* out = a.idx + (long long)(tok0 + q) * a.topk;
          for (int j = lane; j < a.topk; j += 32) out[j] = j < avail ? j : -1;
        }
        continue;
      }
      const int buf = wi & 1;
      const float* scr = a.scratch + ((size_t)blockIdx.x * 2 + buf) * 4 * a.sc_cap;
      if (!warp_wait(&sc_full[buf], (wi >> 1) & 1)) { *abort_flag = 1; break; }
      if (q < nq)
        warp_topk_ascending(scr + (size_t)q * a.sc_cap, avail, a.topk, a.idx + (long long)(tok0 + q) * a.topk, hist,
                            sel_s + q * kSelChunk);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sc_free[buf]);
      ++wi;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
}

}  // namespace csa

namespace csa {

// ---------------------------------------------------------------- decode form
// One new query per sequence over that sequence's cached K^IComp: the score
// row I[b, s] = sum_h w_{b,h} ReLU(q^I_{b,h} . K^IComp_{b,s}) is split over
// all SMs in 128-block tiles (work item = (sequence, tile)), each tile one
// tcgen05.mma group D[128 blocks x n_h^I] with the ReLU / head weighting in
// the epilogue; the row goes to a [B, cap] scratch and decode_select_kernel
// then picks its exact top-k.  The cache streams from HBM once.
struct IdxDecArgs {
  const float* wI; long long ld_wI;   // [B, nhI]
  const int* pos;                     // [B]
  float* scratch;                     // [B, cap]
  int B, cap, m, nhI, cI, tiles_per_seq;
};

namespace idxdec {
constexpr int kM = 128, kStages = 5, kQSlots = 2;
constexpr int kQBytes = 64 * 128 * 2;    // up to [64 heads x 128] bf16 as two 64-column chunks
constexpr int kKBytes = kM * 128 * 2;    // [128 blocks x 128] bf16 as two chunks
constexpr int kOffK = kQSlots * kQBytes;
constexpr int kOffW = kOffK + kStages * kKBytes;
constexpr int kEpiWarps = 8;             // two groups of four: even and odd items of the CTA
constexpr size_t kSmem = 1024 + (size_t)kOffW + kEpiWarps * 64 * 4 + 256;
constexpr int kThreads = 32 * (2 + kEpiWarps);
}  // namespace idxdec

__global__ void __launch_bounds__(idxdec::kThreads, 1)
    indexer_decode_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
                             IdxDecArgs a) {
  using namespace sm100;
  using namespace idxdec;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* w_s = reinterpret_cast<float*>(sm + kOffW);     // kEpiWarps warps x 64
  uint64_t* bars = reinterpret_cast<uint64_t*>(w_s + kEpiWarps * 64);
  uint64_t* full = bars;                   // [kStages] key tile landed
  uint64_t* empty = full + kStages;        // [kStages]
  uint64_t* t_full = empty + kStages;      // [2]
  uint64_t* t_empty = t_full + 2;          // [2]
  uint64_t* q_full = t_empty + 2;          // [kQSlots] q^I of a sequence landed
  uint64_t* q_empty = q_full + kQSlots;    // [kQSlots] the sequence's last MMA done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_empty + kQSlots);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = a.nhI;
  const int kchunks = a.cI / 64;
  const int items = a.B * a.tiles_per_seq;
  const int qchunk = N * 128, kchunk = kM * 128;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
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

  // items of this CTA: a contiguous range, so consecutive items share a sequence
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

  // q^I is loaded once per sequence (a CTA's items are contiguous, so it
  // meets each of its sequences in one run) into one of kQSlots slots; the
  // ring stages carry only key tiles.
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
          mbar_arrive_expect_tx(&q_full[qs], (uint32_t)(kchunks * qchunk));
          for (int c = 0; c < kchunks; ++c) tma_load_3d(&tmQ, &q_full[qs], sm + qs * kQBytes + c * qchunk, 64 * c, 0, b);
          qb = b;
          ++nq;
        }
        const int st = g % kStages;
        if (!mbar_wait(&empty[st], ((g / kStages) & 1) ^ 1)) { *abort_flag = 1; break; }
        mbar_arrive_expect_tx(&full[st], (uint32_t)(kchunks * kchunk));
        for (int c = 0; c < kchunks; ++c)
          tma_load_2d(&tmK, &full[st], sm + kOffK + st * kKBytes + c * kchunk, 64 * c, b * a.cap + j * kM);
        ++g;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kM, N);
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
        const int st = g % kStages, acc = g & 1;
        if (!mbar_wait(&full[st], (g / kStages) & 1) || !mbar_wait(&t_empty[acc], ((g >> 1) & 1) ^ 1)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint64_t qd = sdesc_k_sw128(smem_u32(sm + ((nq - 1) % kQSlots) * kQBytes));
        const uint64_t kd = sdesc_k_sw128(smem_u32(sm + kOffK + st * kKBytes));
        for (int c = 0; c < kchunks; ++c)
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_bf16(tmem + (uint32_t)(acc * 64), desc_add(kd, c * kchunk + ks * 32),
                     desc_add(qd, c * qchunk + ks * 32), idesc, (c | ks) != 0);
        mma_commit(&empty[st]);
        mma_commit(&t_full[acc]);
        ++g;
      }
    }
  } else {
    // epilogue: warps 2-5 take the CTA's even items (accumulator 0), warps
    // 6-9 the odd ones (accumulator 1), so two items are folded at a time
    const int sub = warp & 3, grp = (warp - 2) >> 2;
    float* w_my = w_s + (warp - 2) * 64;
    const uint32_t lane_base = (uint32_t)(32 * sub) << 16;
    uint32_t g = 0;
    int wb = -1;
    for (int it = it0; it < it1; ++it) {
      if (warp_aborted(abort_flag)) break;
      int b, j, avail;
      if (!item_ok(it, b, j, avail)) continue;
      if ((int)(g & 1) != grp) { ++g; continue; }
      if (b != wb) {
        for (int h = lane; h < N; h += 32) w_my[h] = a.wI[(long long)b * a.ld_wI + h];
        __syncwarp();
        wb = b;
      }
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
      const int s = j * kM + 32 * sub + lane;
      if (s < avail && dcheck(s < a.cap)) __stcg(a.scratch + (long long)b * a.cap + s, (sc4[0] + sc4[1]) + (sc4[2] + sc4[3]));
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

// Exact top-k of each decode row's score row, one CTA of 32 warps per
// sequence, same selection rule as warp_topk_ascending (the k largest
// scores, equal scores lowest index first, ascending indices).  Radix select
// on the order-preserving keys in three passes of 11, 11 and 10 bits; each
// pair of warps builds its own histogram of its share of the row (so
// increments only collide within the pair), the 16 are summed, and warp 0
// picks the digit.  The ordered output splits the row into 32 contiguous
// segments: a counting pass, a prefix over the warps, and a writing pass.
// A row of up to kResident scores is read from global memory (L2) once and
// kept in shared memory as keys; a longer row is read on every pass.
namespace dsel {
constexpr int kWarps = 32, kThreads = 32 * kWarps, kHists = kWarps / 2, kBins = 2048;
constexpr int kWords = 128;        // scratch words: the pick (3) and two per-warp counts (2 x 32)
constexpr int kResident = 16384;   // rows of up to this many scores are selected from shared memory
constexpr size_t kSmem = (size_t)(kHists + 1) * kBins * 4 + kWords * 4 + (size_t)kResident * 4;
}  // namespace dsel

// Warp 0: the digit of the combined histogram hist[0..NB) holding the kk-th
// largest key, the count above it and the count in it (to ws[0..2]).
template <int NB>
__device__ __forceinline__ void dsel_pick(const int* hist, int kk, int* ws) {
  constexpr int PER = NB / 32, SUB = PER / 32 > 0 ? PER / 32 : 1;
  constexpr unsigned kFull = 0xffffffffu;
  const int lane = threadIdx.x & 31;
  int tot = 0;
#pragma unroll 8
  for (int j = 0; j < PER; ++j) tot += hist[NB - 1 - (PER * lane + ((j + lane) & (PER - 1)))];
  int incl = tot;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(kFull, incl, off);
    if (lane >= off) incl += v;
  }
  const int excl = incl - tot;
  const int src = __ffs(__ballot_sync(kFull, excl < kk && incl >= kk)) - 1;
  const int excl_src = __shfl_sync(kFull, excl, src);
  const int kk2 = kk - excl_src;
  const int p0 = PER * src + SUB * lane;
  int c2 = 0;
  for (int u = 0; u < SUB; ++u) c2 += hist[NB - 1 - (p0 + u)];
  int incl2 = c2;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(kFull, incl2, off);
    if (lane >= off) incl2 += v;
  }
  const int excl2 = incl2 - c2;
  const int src2 = __ffs(__ballot_sync(kFull, excl2 < kk2 && incl2 >= kk2)) - 1;
  if (lane == src2) {
    int c = excl2;
    for (int u = 0; u < SUB; ++u) {
      const int v = hist[NB - 1 - (p0 + u)];
      if (c + v >= kk2) {
        ws[0] = NB - 1 - (p0 + u);
        ws[1] = excl_src + c;
        ws[2] = v;
        break;
      }
      c += v;
    }
  }
}

__global__ void __launch_bounds__(dsel::kThreads) decode_select_kernel(const float* scratch, const int* pos, int cap, int m,
                                                            int topk, int* idx) {
  pdl_prologue_done();
  using namespace dsel;
  constexpr unsigned kFull = 0xffffffffu;
  extern __shared__ __align__(16) int dsm[];
  int* whist = dsm;                         // [kHists][kBins] histograms of the warp pairs
  int* hist = dsm + kHists * kBins;         // [kBins] combined
  int* ws = hist + kBins;                   // [kWords] scratch words
  uint32_t* keys = reinterpret_cast<uint32_t*>(ws + kWords);   // [kResident] the row's keys, when it fits
  const int b = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t = pos[b];
  int avail = t >= 0 ? t / m : 0;
  if (avail > cap) avail = cap;
  int* out = idx + (long long)b * topk;
  if (avail <= topk) {
    for (int j = tid; j < topk; j += blockDim.x) out[j] = j < avail ? j : -1;
    return;
  }
  const float* row = scratch + (long long)b * cap;
  // A row that fits is read from L2 once, with every thread's loads in
  // flight together, and kept as keys; the passes below then read shared
  // memory.  Longer rows are read from L2 on every pass.
  const bool resident = avail <= kResident;
  if (resident) {
    for (int i0 = tid; i0 < avail; i0 += kThreads * 8) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + kThreads * u;
        v[u] = i < avail ? __ldcg(row + i) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + kThreads * u;
        if (i < avail) keys[i] = ordered_key(v[u]);
      }
    }
  }
  auto key_at = [&](int i) -> uint32_t { return resident ? keys[i] : ordered_key(__ldcg(row + i)); };
  int* myh = whist + (warp >> 1) * kBins;
  uint32_t prefix = 0, mask = 0;
  int kk = topk;
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : pass == 1 ? 10 : 0;
    const int width = pass == 2 ? 10 : 11;
    const uint32_t dmask = (1u << width) - 1u;
    for (int i = 32 * (warp & 1) + lane; i < kBins / 4; i += 64) reinterpret_cast<int4*>(myh)[i] = make_int4(0, 0, 0, 0);
    __syncthreads();
    // this thread's scores: 4 consecutive per step, the CTA covering 4 kThreads per step
    for (int i0 = 4 * tid; i0 < avail; i0 += 4 * kThreads) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u;
        if (i < avail) {
          const uint32_t key = key_at(i);
          if ((key & mask) == prefix) atomicAdd(&myh[(key >> shift) & dmask], 1);
        }
      }
    }
    __syncthreads();
    for (int bin = tid; bin < kBins; bin += kThreads) {
      int c = 0;
#pragma unroll
      for (int w = 0; w < kHists; ++w) c += whist[w * kBins + bin];
      hist[bin] = c;
    }
    __syncthreads();
    if (warp == 0) {
      if (width == 11) dsel_pick<2048>(hist, kk, ws);
      else dsel_pick<1024>(hist, kk, ws);
    }
    __syncthreads();
    prefix |= (uint32_t)ws[0] << shift;
    mask |= dmask << shift;
    kk -= ws[1];
    const bool settled = ws[2] == kk;   // every key of the bin is needed: key >= prefix decides
    __syncthreads();
    if (settled) break;
  }
  const uint32_t thr = prefix;
  const int need_eq = kk;
  // ordered output over kWarps contiguous segments
  const int seg = (((avail + kWarps - 1) / kWarps) + 31) & ~31;
  const int s0 = min(avail, warp * seg), s1 = min(avail, s0 + seg);
  int n_gt = 0, n_eq = 0;
  for (int base = s0; base < s1; base += 32) {
    const int i = base + lane;
    const uint32_t key = i < s1 ? key_at(i) : 0u;
    n_gt += __popc(__ballot_sync(kFull, i < s1 && key > thr));
    n_eq += __popc(__ballot_sync(kFull, i < s1 && key == thr));
  }
  if (lane == 0) {
    ws[8 + warp] = n_gt;
    ws[8 + kWarps + warp] = n_eq;
  }
  __syncthreads();
  int gt_before = 0, eq_before = 0;
  for (int w = 0; w < warp; ++w) {
    gt_before += ws[8 + w];
    eq_before += ws[8 + kWarps + w];
  }
  int out_off = gt_before + min(eq_before, need_eq), eq_seen = eq_before;
  const unsigned lt = (1u << lane) - 1u;
  for (int base = s0; base < s1; base += 32) {
    const int i = base + lane;
    const uint32_t key = i < s1 ? key_at(i) : 0u;
    const bool gt = i < s1 && key > thr;
    const bool eq = i < s1 && key == thr;
    const unsigned beq = __ballot_sync(kFull, eq);
    const bool take = gt || (eq && eq_seen + __popc(beq & lt) < need_eq);
    const unsigned btk = __ballot_sync(kFull, take);
    const int p = out_off + __popc(btk & lt);
    if (take && dguard(p < topk)) out[p] = i;
    out_off += __popc(btk);
    eq_seen += __popc(beq);
  }
}

}  // namespace csa
