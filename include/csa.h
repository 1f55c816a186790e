/*
 * csa.h -- C ABI of libcsa.so, the B200 (sm_100a) forward path of
 * Compressed Sparse Attention (CSA).
 *
 * Every formula is the one of the page "Compressed Sparse Attention
 * (压缩稀疏注意力)" (cnblogs), equations (1)-(11); each entry point below names
 * the equations it evaluates.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Pointers marked [dev] are device pointers on the current CUDA device;
 *    [host] pointers are host memory.  The caller owns every buffer, the
 *    workspace included.  The library never allocates device memory, never
 *    frees caller memory and never synchronises, except in
 *    csa_get_device_status().
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream).  All work is enqueued asynchronously on it, in order.  Most
 *    kernels are launched with programmatic stream serialization: a kernel
 *    may start its on-chip set-up while the previous kernel on the stream
 *    finishes, but it waits for that kernel to complete before it reads or
 *    writes any memory, so the order of all memory effects is the stream
 *    order.  The one exception is inside csa_decode / csa_decode_q8: the
 *    cache append runs beside the c^Q-side projection of the same call,
 *    whose buffers (workspace rows, packed weights) it does not touch; the
 *    call as a whole keeps the stream order.
 *  - Matrices are dense row-major.  "ld" arguments are row strides in
 *    ELEMENTS.  Element type = csa_dims.dtype for activations and weights
 *    (fp32 or bf16); the indexer head weights w^I are always fp32 and block
 *    indices always int32.
 *  - Token indices t are 0-based and local to their sequence.  Packed
 *    sequences are described by cu_seqlens[nseq+1] (token offsets, [dev]
 *    int32, cu_seqlens[0] = 0) and cu_blocks[nseq+1] (offsets of each
 *    sequence's compressed entries, [dev] int32, cu_blocks[b+1] - cu_blocks[b]
 *    = floor(L_b / m)).  A sequence of L tokens has floor(L/m) compressed
 *    entries; the L mod m tail tokens are not compressed.  Compression
 *    blocks never cross a sequence boundary.
 *  - Errors: arguments and shapes are checked on the host before anything is
 *    launched (CSA_ERR_INVALID_ARG / CSA_ERR_UNSUPPORTED, nothing enqueued).
 *    A failed launch returns CSA_ERR_CUDA.  Conditions found on the device
 *    (an out-of-range block index given to csa_sparse_mqa, inconsistent
 *    cu_seqlens/cu_blocks, a bounded wait that ran out) never fault: the
 *    kernel skips the access, records a bit in a per-device status word and
 *    returns; csa_get_device_status() reports and clears it.
 *  - Nothing is thrown across this ABI.
 */
#ifndef CSA_H_
#define CSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  CSA_OK = 0,
  CSA_ERR_INVALID_ARG = 1,    /* NULL pointer, negative size, bad dims   */
  CSA_ERR_UNSUPPORTED = 2,    /* valid but outside the kernels' limits   */
  CSA_ERR_CUDA = 3,           /* a CUDA runtime call or launch failed     */
  CSA_ERR_DEVICE_TIMEOUT = 4, /* a bounded device wait ran out           */
  CSA_ERR_BAD_INDEX = 5,      /* out-of-range block index seen on device */
  CSA_ERR_BAD_METADATA = 6,   /* cu_seqlens / cu_blocks inconsistent     */
  CSA_ERR_WORKSPACE = 7,      /* workspace smaller than required         */
  CSA_ERR_DEVICE_BOUNDS = 8   /* debug build: an index check failed      */
} csa_status;

typedef enum { CSA_F32 = 0, CSA_BF16 = 1 } csa_dtype;

/* Problem dimensions, named as on the page:
 *   d    hidden size (H in R^{n x d})
 *   c    head dimension of the KV entries (C^a, C^b, Z^a, Z^b in R^{n x c})
 *   m    tokens per compressed entry
 *   cI   indexer head dimension (K^IComp in R^{n/m x cI})
 *   nhI  number of indexer query heads
 *   nh   number of attention query heads
 *   dc   query compression dimension (c^Q_t in R^{dc})
 *   topk number of compressed entries kept per query (eq. 9)
 *   dtype csa_dtype of activations and weights.  CSA_BF16 computes with
 *        fp32 accumulation and stores intermediates in bf16 (w^I in fp32);
 *        CSA_F32 computes and stores in fp32. */
typedef struct {
  int d, c, m, cI, nhI, nh, dc, topk;
  int dtype;
} csa_dims;

/* The trainable parameters, each [in, out] row-major as in "X . W" on the
 * page, all [dev] and of csa_dims.dtype.
 *   W_aKV, W_bKV, W_aZ, W_bZ      [d, c]   eqs. (1), (2)
 *   B_a, B_b                      [m, c]   position biases, eq. (3)
 *   W_aKV_I .. W_bZ_I             [d, cI]  the indexer keys' own compression
 *   B_a_I, B_b_I                  [m, cI]  parameters (same operation, width cI)
 *   W_DQ                          [d, dc]  eq. (5)
 *   W_IUQ                         [dc, nhI*cI]  eq. (6), heads concatenated
 *   W_UQ                          [dc, nh*c]    eq. (10), heads concatenated
 *   W_w                           [d, nhI]      eq. (7)                      */
typedef struct {
  const void *W_aKV, *W_bKV, *W_aZ, *W_bZ;
  const void *B_a, *B_b;
  const void *W_aKV_I, *W_bKV_I, *W_aZ_I, *W_bZ_I;
  const void *B_a_I, *B_b_I;
  const void *W_DQ, *W_IUQ, *W_UQ, *W_w;
} csa_weights;

/* ---------------------------------------------------------------------- */
/* Weights                                                                 */
/* ---------------------------------------------------------------------- */

/* Bytes of the packed-weight buffer for these dims (0 if dims are invalid). */
size_t csa_packed_weights_bytes(const csa_dims* dims);

/* Re-lays the parameters of eqs. (1)-(7), (10) out for the projection
 * kernels: the H-side matrices are concatenated along their output columns
 * and transposed (one [N1, d] K-major matrix), the c^Q-side ones likewise
 * ([N2, dc]); the biases are widened to fp32.  `packed` [dev] must hold
 * csa_packed_weights_bytes(dims) bytes and be 256-byte aligned.  Run once
 * per set of weights; every forward/decode call reads only `packed`. */
csa_status csa_pack_weights(const csa_dims* dims, const csa_weights* w, void* packed,
                            size_t packed_bytes, void* stream);

/* ---------------------------------------------------------------------- */
/* Stages                                                                  */
/* ---------------------------------------------------------------------- */

/* Row width (elements) of the H-side projection output: the concatenation
 * [C^a | C^b | Z^a | Z^b | C^aI | C^bI | Z^aI | Z^bI | c^Q] of one token,
 * 4c + 4cI + dc elements of dtype. */
int csa_hidden_row_elems(const csa_dims* dims);

/* Row width (elements) of the c^Q-side projection output [q^I | q] of one
 * token, nhI*cI + nh*c elements of dtype (heads concatenated, eqs. 6, 10). */
int csa_query_row_elems(const csa_dims* dims);

/* H-side projections, eqs. (1), (2), (5), (7) and the indexer-key
 * projections, as one GEMM over the packed weights.
 * H [dev]  : [T, d].   Y1 [dev] : [T, csa_hidden_row_elems] (row stride =
 * that width).   wI [dev] : [T, nhI] fp32, the indexer head weights. */
csa_status csa_project_hidden(const csa_dims* dims, const void* packed, const void* H, int T, void* Y1,
                              float* wI, void* stream);

/* c^Q-side projections, eqs. (6) and (10), from the shared latent query.
 * cQ [dev] : [T, dc] with row stride ld_cQ (the c^Q columns of Y1 qualify).
 * Y2 [dev] : [T, csa_query_row_elems] (row stride = that width). */
csa_status csa_project_query(const csa_dims* dims, const void* packed, const void* cQ, int ld_cQ, int T,
                             void* Y2, void* stream);

/* Overlapping softmax compression, eqs. (3)-(4), for packed sequences.
 * Ca, Cb, Za, Zb [dev] : [total_tokens, width] with row stride ld.
 * Ba, Bb [dev]         : [m, width] position biases, fp32.
 * out [dev]            : [total_blocks, width], row stride width.
 * Entry i of a sequence uses the C^a/Z^a rows of its block i and the
 * C^b/Z^b rows of block i-1; at i = 0 the Z^b logits are -inf and the C^b
 * rows 0.  The softmax runs over the 2m logits of each channel. */
csa_status csa_compress(const csa_dims* dims, const void* Ca, const void* Cb, const void* Za,
                        const void* Zb, int ld, const float* Ba, const float* Bb, int width,
                        const int* cu_seqlens, const int* cu_blocks, int nseq, int total_tokens,
                        int total_blocks, void* out, void* stream);

/* Compression of both key sets as the forward pass runs it, eqs. (3)-(4)
 * and the indexer-key copy of the same operation: C^Comp [total_blocks, c]
 * and K^IComp [total_blocks, cI] from the H-side projection rows, in one
 * launch.
 * Y1 [dev]     : [T, csa_hidden_row_elems] as csa_project_hidden writes it
 *                (its C^a, C^b, Z^a, Z^b and indexer column blocks are read).
 * packed [dev] : the packed weights (their fp32 position biases are read).
 * Ccomp, KIcomp [dev] : outputs, row strides c and cI.
 * Same entry rule as csa_compress; returns CSA_ERR_INVALID_ARG for null
 * pointers or inconsistent sizes before any launch. */
csa_status csa_compress_kv(const csa_dims* dims, const void* packed, const void* Y1, int T,
                           const int* cu_seqlens, const int* cu_blocks, int nseq, int total_blocks,
                           void* Ccomp, void* KIcomp, void* stream);

/* Workspace bytes csa_project_hidden_compress needs for T tokens (halo rows
 * of the row-tile boundaries and their counters; 0 if the dims are invalid
 * or the fused form does not apply: it needs bf16 and c, cI multiples of
 * 64). */
size_t csa_project_compress_workspace_bytes(const csa_dims* dims, int T);

/* The H-side projection with the compression in its epilogue: eqs. (1),
 * (2), the indexer-key projections, (3), (4), (5) and (7) in one kernel, as
 * csa_forward runs them when the fused form applies.  C^a, C^b, Z^a, Z^b
 * and their indexer copies never reach memory: each 128-token tile rounds
 * them to bf16 (the storage point of the unfused path) and compresses the
 * entries whose 2m-token window lies inside it; entries whose window
 * crosses a tile boundary are compressed from the boundary's halo rows by
 * whichever of the two neighbouring tiles finishes second.  C^Comp and
 * K^IComp are bit-identical to csa_project_hidden + csa_compress_kv.
 * H [dev]       : [T, d] bf16.
 * Y1 [dev]      : [T, csa_hidden_row_elems]; only its c^Q columns (from
 *                 column 4c + 4cI) are written.
 * wI [dev]      : [T, nhI] fp32.
 * Ccomp, KIcomp : [total_blocks, c], [total_blocks, cI] outputs.
 * ws [dev]      : >= csa_project_compress_workspace_bytes(dims, T), 256-byte
 *                 aligned; no initialisation needed (its counters are
 *                 cleared on the stream first).
 * Returns CSA_ERR_UNSUPPORTED if the fused form does not apply. */
csa_status csa_project_hidden_compress(const csa_dims* dims, const void* packed, const void* H, int T,
                                       const int* cu_seqlens, const int* cu_blocks, int nseq,
                                       int total_blocks, void* Y1, float* wI, void* Ccomp, void* KIcomp,
                                       void* ws, size_t ws_bytes, void* stream);

/* Lightning indexer (eq. 8) and top-k selector (eq. 9), prefill.
 * qI [dev]  : [total_tokens, nhI*cI] (row stride ld_qI), heads concatenated.
 * wI [dev]  : [total_tokens, nhI] fp32 (row stride ld_wI).
 * KI [dev]  : [total_blocks, cI] compressed indexer keys.
 * idx [dev] : [total_tokens, topk] int32 output.  Row t lists the chosen
 *             local block indices s < floor(t/m) in ascending order, then -1.
 *             k is clamped to floor(t/m); ties are broken by the lower s.
 * max_seqlen [host] : an upper bound of every sequence length (it sizes the
 *             per-query candidate storage).  A query of a longer sequence
 *             is not computed in full: the CUDA-core path clamps its
 *             candidates, the tensor-core path skips its block of queries
 *             (their idx rows keep their old contents); either way nothing
 *             is written outside the workspace and CSA_ERR_BAD_METADATA is
 *             flagged.  The same holds for cu_seqlens / cu_blocks that
 *             place a query or block outside total_tokens / total_blocks.
 * ws [dev]  : workspace of ws_bytes >= csa_indexer_workspace_bytes(), 256-byte
 *             aligned, no initialisation needed.
 * The score matrix is never written to memory.  The tensor-core indexer runs
 * for bf16 dims with m = 4, nhI in {32, 64} and cI in {64, 128}; otherwise
 * the CUDA-core indexer holds each query's candidate scores in shared memory
 * and requires 4 * (nhI*cI + nhI + 296 + floor(max_seqlen/m)) <= 227 KB
 * (CSA_ERR_UNSUPPORTED before any launch otherwise). */
csa_status csa_indexer_topk(const csa_dims* dims, const void* qI, int ld_qI, const float* wI,
                            int ld_wI, const void* KI, const int* cu_seqlens, const int* cu_blocks,
                            int nseq, int total_tokens, int total_blocks, int max_seqlen, int* idx,
                            void* ws, size_t ws_bytes, void* stream);

/* Workspace bytes csa_indexer_topk needs (per-CTA rows of candidate scores,
 * kept on chip / in L2; 0 if the dims are invalid). */
size_t csa_indexer_workspace_bytes(const csa_dims* dims, int total_tokens, int nseq, int max_seqlen);

/* csa_indexer_topk for callers that cannot allocate device memory.
 * The page has no counterpart: this is an interface addition, not a step of
 * the method.  Some callers own no allocator: code that runs where a
 * cudaMalloc is not allowed (a process whose device memory is handed out by
 * another framework's pool, or a latency-critical loop that must not
 * allocate after start-up) cannot provide the indexer's workspace.  This
 * entry point takes the same arguments minus the workspace and instead uses
 * a fixed scratch array that lives in the library's module memory (20 MiB on
 * every GPU that loads the library, held until the process exits).
 * Limits: the tensor-core indexer's shapes only (bf16, m = 4, nhI in {32, 64},
 * cI in {64, 128}, qI and KI 16-byte aligned, ld_qI a multiple of 8) and
 * floor(max_seqlen / m) + 1 <= 4096 (max_seqlen <= 16383 for m = 4); anything
 * else returns CSA_ERR_UNSUPPORTED before any launch.  It calls no allocating
 * routine.  The first call on a device looks up the scratch array's device
 * address (cudaGetSymbolAddress) with that device current; make that first
 * call before any stream capture.  Every call shares the one array: calls
 * whose kernels overlap on the GPU (e.g. on two streams) race on it; calls in
 * one stream are safe.  The array's contents carry over between calls; no
 * part of it needs to start at zero (each score is written before it is
 * read).  Output identical to csa_indexer_topk. */
csa_status csa_indexer_topk_noalloc(const csa_dims* dims, const void* qI, int ld_qI, const float* wI,
                                    int ld_wI, const void* KI, const int* cu_seqlens,
                                    const int* cu_blocks, int nseq, int total_tokens, int total_blocks,
                                    int max_seqlen, int* idx, void* stream);

/* Shared-KV MQA over the selected entries, eqs. (10)-(11).
 * q [dev]     : [total_tokens, nh*c] (row stride ld_q), heads concatenated.
 * Ccomp [dev] : [total_blocks, c] compressed entries (keys AND values).
 * idx [dev]   : [total_tokens, topk] int32 as produced by csa_indexer_topk;
 *               -1 entries are skipped; an index outside [0, floor(t/m)) is
 *               skipped and flags CSA_ERR_BAD_INDEX in the status word.
 * O [dev]     : [total_tokens, nh*c] output, o_{t,h} = softmax(q K^T/sqrt(c)) V.
 *               Rows with no selected entry are 0. */
csa_status csa_sparse_mqa(const csa_dims* dims, const void* q, int ld_q, const void* Ccomp,
                          const int* idx, const int* cu_seqlens, const int* cu_blocks, int nseq,
                          int total_tokens, int total_blocks, void* O, void* stream);

/* ---------------------------------------------------------------------- */
/* Whole forward pass (prefill)                                            */
/* ---------------------------------------------------------------------- */

/* Workspace bytes csa_forward needs for total_tokens tokens in nseq packed
 * sequences (0 if the dims are invalid). */
size_t csa_forward_workspace_bytes(const csa_dims* dims, int total_tokens, int nseq);

/* CSA forward pass, eqs. (1)-(11).
 * packed [dev]     : output of csa_pack_weights.
 * H [dev]          : [total_tokens, d] hidden states.
 * max_seqlen [host]: upper bound of every sequence length (as for
 *                    csa_indexer_topk); a bound above total_tokens is
 *                    taken as total_tokens.  Where the CUDA-core indexer
 *                    runs, its limit on floor(max_seqlen/m) (see
 *                    csa_indexer_topk) is checked before any launch.
 * O [dev]          : [total_tokens, nh*c] attention outputs o_{t,i}.
 * Ccomp_out, KI_out, idx_out [dev, optional, may be NULL]: copies of
 *                    C^Comp [total_blocks, c], K^IComp [total_blocks, cI]
 *                    and the top-k indices [total_tokens, topk].
 * ws [dev]         : workspace of ws_bytes >= csa_forward_workspace_bytes(),
 *                    256-byte aligned; its contents need no initialisation. */
csa_status csa_forward(const csa_dims* dims, const void* packed, const void* H,
                       const int* cu_seqlens, const int* cu_blocks, int nseq, int total_tokens,
                       int total_blocks, int max_seqlen, void* O, void* Ccomp_out, void* KI_out, int* idx_out,
                       void* ws, size_t ws_bytes, void* stream);

/* csa_forward with stage timing: the same launches and results, plus a
 * CUDA event recorded on `stream` before the first stage and after each
 * stage: events[0] before A1, then after A1 (eqs. 1, 2, 5, 7 projection),
 * A2 (eqs. 6, 10), A3 (eqs. 3-4 compression), A4 (eqs. 8-9 indexer +
 * top-k) and A5 (eq. 11 MQA), i.e. events[1..5].  Where the compression
 * runs inside the A1 kernel (bf16, c and cI multiples of 64), events[3]
 * follows events[2] with nothing between them and the A1 interval includes
 * A3.
 * events [host] : 6 cudaEvent_t handles (passed as void*), created by the
 *                 caller; a NULL array or handle returns CSA_ERR_INVALID_ARG
 *                 before any launch.  Recording adds no kernel. */
csa_status csa_forward_staged(const csa_dims* dims, const void* packed, const void* H,
                              const int* cu_seqlens, const int* cu_blocks, int nseq, int total_tokens,
                              int total_blocks, int max_seqlen, void* O, void* Ccomp_out, void* KI_out,
                              int* idx_out, void* ws, size_t ws_bytes, void* const* events, void* stream);

/* ---------------------------------------------------------------------- */
/* Context-parallel prefill of one sequence                                */
/* ---------------------------------------------------------------------- */
/* The forward pass of one sequence split into chunks of consecutive tokens
 * (chunk starts on block boundaries), for processes that each own some
 * chunks.  Entry i needs only tokens m(i-1) .. m(i+1)-1 (eqs. 3-4) and query
 * t needs only the entries s < floor(t/m) (eq. 8), so a rank compresses its
 * chunks alone, the caller exchanges the entries (one all-gather), and each
 * rank then evaluates its chunks' queries alone.  Results are bit-identical
 * to csa_forward on the whole sequence. */

/* Workspace bytes for a chunk of T tokens that ends at position ctx (the
 * same buffer may serve both calls of that chunk; 0 if invalid). */
size_t csa_cp_workspace_bytes(const csa_dims* dims, int T, int ctx);

/* Step 1: eqs. (1), (2), (5), (7), the indexer-key projections and eqs.
 * (3)-(4) for a chunk of T tokens starting at position pos0 (a multiple of
 * m; T a multiple of m except for the sequence's last chunk).
 * H [dev]     : the m hidden rows before the chunk (when pos0 > 0), then the
 *               chunk's T rows.
 * Y1, wI [dev]: [m + T (or T when pos0 = 0), csa_hidden_row_elems] and
 *               [same rows, nhI] fp32 outputs (the projection rows step 2
 *               reads; the halo rows come first).
 * Ccomp_chunk, KIcomp_chunk [dev]: the chunk's floor(T/m) entries, i.e.
 *               global entries pos0/m .. pos0/m + floor(T/m) - 1.
 * ws [dev]    : >= csa_cp_workspace_bytes(dims, T, pos0 + T), 256-byte
 *               aligned. */
csa_status csa_cp_compress(const csa_dims* dims, const void* packed, const void* H, int T, int pos0,
                           void* Y1, float* wI, void* Ccomp_chunk, void* KIcomp_chunk, void* ws,
                           size_t ws_bytes, void* stream);

/* Step 2 (after the caller has gathered every chunk's entries): eqs. (6),
 * (10), (8), (9), (11) for the chunk's T queries at positions pos0 ..
 * pos0 + T - 1 over the whole sequence's entries.
 * Y1, wI [dev]: the chunk's own rows of step 1's outputs (without the halo
 *               rows).
 * Ccomp, KIcomp [dev]: [total_blocks, c] / [total_blocks, cI], every entry
 *               of the sequence; total_blocks >= (pos0 + T) / m.
 * O [dev]     : [T, nh*c];  idx_out [dev, optional]: [T, topk] (global
 *               block indices).
 * ws [dev]    : as for step 1.
 * Where the CUDA-core indexer runs, its limit (csa_indexer_topk) applies to
 * (pos0 + T) / m and is checked before any launch. */
csa_status csa_cp_queries(const csa_dims* dims, const void* packed, const void* Y1, const float* wI, int T,
                          int pos0, const void* Ccomp, const void* KIcomp, int total_blocks, void* O,
                          int* idx_out, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------- */
/* Decode over a compressed cache                                          */
/* ---------------------------------------------------------------------- */

/* Row width of the per-sequence ring: 4c + 4cI elements of dtype, the raw
 * rows [C^a | C^b | Z^a | Z^b | C^aI | C^bI | Z^aI | Z^bI] of one token. */
int csa_ring_row_elems(const csa_dims* dims);

/* Appends one token per sequence to the compressed cache.
 * rows [dev]      : [B, csa_ring_row_elems] the new tokens' rows (eqs. 1-2).
 * pos [dev]       : [B] int32, the new token's index t in its sequence.
 * ring [dev]      : [B, 2m, csa_ring_row_elems], slot t mod 2m holds token t.
 * Ccache [dev]    : [B, cap, c];  KIcache [dev] : [B, cap, cI].
 * cache_len [dev] : [B] int32, must equal floor(t/m) on entry.
 * The row is stored in slot t mod 2m; when (t+1) is a multiple of m, block
 * i = (t+1)/m - 1 is compressed with eqs. (3)-(4) (C^a rows of block i, C^b
 * rows of block i-1, or the i = 0 padding) into entry i of both caches and
 * cache_len becomes i+1.  i >= cap flags CSA_ERR_BAD_INDEX and skips. */
csa_status csa_cache_append(const csa_dims* dims, const void* packed, const void* rows,
                            const int* pos, void* ring, void* Ccache, void* KIcache,
                            int* cache_len, int cap, int B, void* stream);

/* Workspace bytes csa_decode needs for B sequences with caches of capacity
 * cap entries: the projections, the indexer scores [B, cap] fp32, the
 * selected indices and the fp32 partial sums of the K-split A1 projection. */
size_t csa_decode_workspace_bytes(const csa_dims* dims, int B, int cap);

/* One decode step: each of B independent sequences gets one new token h_b
 * at position pos[b] and attends over its cached entries s < floor(t/m).
 * h [dev] : [B, d].  O [dev] : [B, nh*c].  idx_out [dev, optional] : [B, topk].
 * The caches, cache_len and ring are updated as by csa_cache_append.
 * Unless the tensor-core decode indexer runs (bf16, nhI in {32, 64}, cI in
 * {64, 128}, KIcache 16-byte aligned), a row of cap scores must fit in one
 * block's shared memory: 4 * (nhI*cI + nhI + 296 + cap) <= 227 KB, else
 * CSA_ERR_UNSUPPORTED before any launch (no cache is changed). */
csa_status csa_decode(const csa_dims* dims, const void* packed, const void* h, const int* pos,
                      void* ring, void* Ccache, void* KIcache, int* cache_len, int cap, int B,
                      void* O, int* idx_out, void* ws, size_t ws_bytes, void* stream);

/* csa_decode with stage timing: the same launches and results, plus a CUDA
 * event recorded on `stream` before the first stage (events[0]) and after
 * each stage: the H-side projection with its K-split reduction (1), the
 * c^Q-side projection (2), the cache append (3), the indexer scores (4),
 * the top-k selection (5) and the MQA (6).  (csa_decode runs the append
 * beside the c^Q-side projection, which touches none of its buffers; the
 * event between them serialises the two here.)
 * events [host] : 7 cudaEvent_t handles (passed as void*), created by the
 *                 caller; a NULL array or handle returns CSA_ERR_INVALID_ARG
 *                 before any launch.  Recording adds no kernel. */
csa_status csa_decode_staged(const csa_dims* dims, const void* packed, const void* h, const int* pos,
                             void* ring, void* Ccache, void* KIcache, int* cache_len, int cap, int B,
                             void* O, int* idx_out, void* ws, size_t ws_bytes, void* const* events,
                             void* stream);

/* ---------------------------------------------------------------------- */
/* Decode over a quantised indexer-key cache (E4M3)                        */
/* ---------------------------------------------------------------------- */
/* A cache format of this library (the page stores C^Comp / K^IComp without
 * fixing a precision): K^IComp entries as FP8 E4M3 codes with one fp32 scale
 * per entry, half the bytes the indexer streams per decode step.  For an
 * entry v (its cI values as stored in bf16): scale = max_j |v_j| / 448 in
 * fp32 (1 for an all-zero entry), code_j = E4M3(v_j / scale) rounded to
 * nearest even and saturated to +-448; the entry stands for code * scale.
 * The indexer multiplies the codes (widened exactly to fp16) by q^I in fp16
 * and applies each entry's scale to its head-weighted sum (the scale is
 * positive, so it commutes with the ReLU).  C^Comp stays bf16. */

/* Quantises n rows of w bf16 values (row stride ld elements; w a multiple
 * of 32) into codes [n, w] (one byte each) and scales [n] (fp32), as above:
 * e.g. a bf16 key cache [B * cap, cI] into the quantised cache. */
csa_status csa_quantize_keys_e4m3(const void* KI, long long ld, int n, int w, void* codes, float* scales,
                                  void* stream);

/* csa_decode with the indexer-key cache quantised: KIcodes [B, cap, cI]
 * (E4M3 codes, 16-byte aligned) and KIscale [B, cap] fp32 replace KIcache.
 * A block closed by this step is compressed, rounded to bf16 and quantised
 * into both.  Requires bf16 dims with cI = 128 and nhI in {32, 64}
 * (CSA_ERR_UNSUPPORTED otherwise).  Workspace: csa_decode_workspace_bytes. */
csa_status csa_decode_q8(const csa_dims* dims, const void* packed, const void* h, const int* pos, void* ring,
                         void* Ccache, void* KIcodes, float* KIscale, int* cache_len, int cap, int B, void* O,
                         int* idx_out, void* ws, size_t ws_bytes, void* stream);

/* csa_decode_q8 with the stage events of csa_decode_staged. */
csa_status csa_decode_q8_staged(const csa_dims* dims, const void* packed, const void* h, const int* pos,
                                void* ring, void* Ccache, void* KIcodes, float* KIscale, int* cache_len,
                                int cap, int B, void* O, int* idx_out, void* ws, size_t ws_bytes,
                                void* const* events, void* stream);

/* ---------------------------------------------------------------------- */
/* Status                                                                  */
/* ---------------------------------------------------------------------- */

/* Synchronises `stream`, reads and clears the current device's status word
 * and returns the most severe condition recorded since the last call
 * (CSA_OK if none).  The only call that synchronises. */
csa_status csa_get_device_status(void* stream);

/* Static, NUL-terminated description of a status code. */
const char* csa_status_string(csa_status s);

/* 1 in the debug build of this library (libcsa_debug.so, compiled with
 * CSA_DEBUG), 0 in the release build (libcsa.so).  The debug build has the
 * same entry points and results; in addition its kernels check, before each
 * global access whose index the kernel computes (a gathered entry row, a
 * score or index written for a query row, a compressed entry, a cache slot),
 * that the index lies in its range, and where it does not they skip the
 * access and record CSA_ERR_DEVICE_BOUNDS in the status word. */
int csa_debug_build(void);

/* Number of kernels this library has enqueued in this process so far (all
 * devices, all streams).  A monotone counter for accounting; never reset. */
uint64_t csa_launch_count(void);

/* ---------------------------------------------------------------------- */
/* Failure detection                                                       */
/* ---------------------------------------------------------------------- */
/* Not steps of the method (the page describes no runtime): every wait
 * inside a kernel of this library is bounded, and one that runs out records
 * CSA_ERR_DEVICE_TIMEOUT in the status word and ends its kernel instead of
 * hanging the GPU. */

/* Sets the limit of every bounded device wait on the current device, in ns
 * of the GPU's global timer (default 1.5 s; accepted range 1 us .. 60 s,
 * else CSA_ERR_INVALID_ARG).  Each wait also ends after 2^30 polls whatever
 * the timer says.  Takes effect for kernels launched after the call
 * returns; call it while no kernel of this library is running.  Meant for
 * tests and diagnostics: a too-short limit turns slow but healthy waits
 * into timeouts. */
csa_status csa_set_wait_limit_ns(unsigned long long ns);

/* Self-check of the bounded waits: enqueues one small kernel whose first
 * warp waits on a barrier that nothing arrives on (the wait must run out at
 * the limit, return to its caller and record CSA_ERR_DEVICE_TIMEOUT) and
 * whose second warp waits on a barrier it completes itself.
 * out [dev] : 3 x uint64, 8-byte aligned: out[0] = 1 if the first wait
 *             claimed completion (it must not), out[1] = ns the first wait
 *             took, out[2] = 1 if the second wait completed.
 * Read the result with csa_get_device_status (CSA_ERR_DEVICE_TIMEOUT is the
 * expected answer). */
csa_status csa_check_wait_timeout(unsigned long long* out, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* CSA_H_ */
