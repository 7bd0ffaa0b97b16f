/*
 * hsa.h -- C ABI of libhsa: hierarchical chunk-sparse landmark attention
 * (HSA / HiLS / DHSA forward pass) on NVIDIA B200 (sm_100a).
 *
 * What is computed.  For query token t of head h in KV group g = h / G
 * (G = H / Hkv query heads share one KV head), with chunk size S,
 * c_t = floor(t / S) and scale = 1/sqrt(d) unless given:
 *
 *   s[t,h,i]  = scale * q[t,h] . l[g,i]                 landmark score of chunk i
 *   sbar[t,g,i] = mean over the G heads of s[t,h,i]     group score (shared selection)
 *   sel(t,g)  = the topk chunks i < c_t with the largest sbar; equal scores go
 *               to the lower chunk index; fewer visible chunks -> all of them
 *   w[t,h,k]  = softmax over k in sel(t,g) of s[t,h,k]  fusion weights
 *   o[t,h,i]  = softmax_j(scale * q[t,h] . k[g,j]) v[g,j] over the S keys of chunk i
 *   O[t,h]    = sum_k w[t,h,k] o[t,h,sel_k]
 *               + (own_chunk ? causal attention over keys c_t*S .. t : 0)
 *
 * Sources: chunk size 64, one landmark per chunk and per-token top-K
 * retrieval are from "Understanding and Improving Length Generalization in
 * Hierarchical Sparse Attention Models" (ai.info summary, "Methodology in
 * Plain English" and "Main Findings"); attention inside each retrieved chunk
 * with outputs fused by the retrieval scores is the HiLS Attention abstract
 * (mlsift "length extrapolation" tag page); the DHSA landmark sqrt(|C|) * mean
 * of a chunk's keys is from the Dynamic Hierarchical Sparse Attention review
 * (pith.science, "What carries the argument").  Where the pages leave a step
 * open the library takes the readings stated next to each call.
 *
 * Conventions for every call:
 *  - All tensor pointers are DEVICE pointers, row-major and densely packed in
 *    the layout given; they must be 16-byte aligned.  The caller owns every
 *    buffer, the workspace included.  The library allocates no memory.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Calls only enqueue work on it; none synchronises except
 *    hsa_check.
 *  - Arguments are checked before anything is launched.  A failed check
 *    returns HSA_ERR_INVALID_ARG, HSA_ERR_UNSUPPORTED or HSA_ERR_WORKSPACE and
 *    launches nothing.  A launch failure returns HSA_ERR_CUDA.
 *  - Supported shapes: d in {64, 128}; S = 64; 1 <= topk <= 32; H % Hkv == 0
 *    with G = H / Hkv in {1, 2, 4, 8, 16}; dtypes HSA_F32 or HSA_BF16.
 *    Accumulation is fp32 throughout; O is written in the input dtype.
 */
#ifndef HSA_H_
#define HSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    HSA_OK = 0,
    HSA_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, inconsistent sizes */
    HSA_ERR_UNSUPPORTED = 2,   /* valid request outside the supported shapes/dtypes */
    HSA_ERR_WORKSPACE = 3,     /* workspace missing or smaller than *_workspace_size */
    HSA_ERR_CUDA = 4,          /* a CUDA launch or runtime call failed */
    HSA_ERR_TIMEOUT = 5        /* a device-side bounded wait gave up (see hsa_check) */
} hsa_status_t;

typedef enum { HSA_F32 = 0, HSA_BF16 = 1 } hsa_dtype_t;

/* Kernel families a call launched (hsa_last_call_kernels). */
enum {
    HSA_K_LANDMARKS = 1u << 0,            /* DHSA landmarks (hsa_landmarks, or prefill with lm = NULL) */
    HSA_K_SPLIT_LANDMARKS = 1u << 1,      /* fp32 landmarks split into bf16 high/low planes */
    HSA_K_SELECT_TC_ONE_TILE = 1u << 2,   /* tensor-core selection, all chunks in one score tile */
    HSA_K_SELECT_TC_MULTI_TILE = 1u << 3, /* tensor-core selection over several score tiles */
    HSA_K_SELECT_SIMT = 1u << 4,          /* selection on CUDA cores */
    HSA_K_WORK_LISTS = 1u << 5,           /* chunk buckets and tile lists */
    HSA_K_ATTEND_TC = 1u << 6,            /* tensor-core in-chunk attention */
    HSA_K_FUSE = 1u << 7,                 /* fusion of the chunk outputs */
    HSA_K_ATTEND_SIMT = 1u << 8,          /* in-chunk attention + fusion on CUDA cores */
    HSA_K_DECODE_SCAN = 1u << 9,          /* decode landmark scan + top-K */
    HSA_K_DECODE_ATTEND = 1u << 10,       /* decode attend + fusion (or a shard's fusion state) */
    HSA_K_DECODE_CP_MERGE = 1u << 11,     /* global top-K over the shards' candidates */
    HSA_K_DECODE_CP_COMBINE = 1u << 12,   /* O from the shards' fusion states */
    HSA_K_BACKWARD = 1u << 13,            /* prefill gradients (hsa_prefill_backward) */
    HSA_K_BACKWARD_TC = 1u << 14          /* ... with the tensor-core key pass */
};

/* Path overrides (hsa_set_path_overrides). */
enum {
    HSA_PATH_SIMT_PREFILL = 1,            /* prefill (and its backward) on CUDA cores even where tensor cores apply */
    HSA_PATH_SIMT_SELECT = 2,             /* selection on CUDA cores even where tensor cores apply */
    HSA_PATH_MULTI_TILE_SELECT = 4        /* the multi-tile tensor-core selection at any length */
};

/*
 * hsa_landmarks_append -- incremental landmark update for growing caches: the
 * DHSA landmarks (sqrt(S) * mean of the chunk's keys, as hsa_landmarks) of the
 * chunks that became complete while sequence b grew from len_before[b] to
 * len_after[b] tokens, i.e. chunks floor(len_before[b]/S) ..
 * floor(len_after[b]/S) - 1; no other landmark row is touched.
 *   K           [B, Hkv, Lmax, d]      k_dt, the cache (Lmax % S == 0)
 *   lm          [B, Hkv, Lmax/S, d]    lm_dt: fp32, or bf16 (rounded to
 *                                      nearest even; the form hsa_decode
 *                                      streams fastest)
 *   len_before, len_after  [B] int32, DEVICE; clamped to 0 .. Lmax
 *   max_new_chunks  a bound on the new chunks of one sequence, used only to
 *                   size the grid (any value >= 0 gives the same result)
 * One warp per new chunk; K read once per new chunk.
 */
hsa_status_t hsa_landmarks_append(const void *K, hsa_dtype_t k_dt, void *lm, hsa_dtype_t lm_dt,
                                  int B, int Hkv, int64_t Lmax, int d, int S,
                                  const int32_t *len_before, const int32_t *len_after,
                                  int max_new_chunks, void *stream);

/*
 * hsa_landmarks -- DHSA landmarks: l[b,g,i] = sqrt(S) * mean of the S keys of
 * chunk i (Dynamic Hierarchical Sparse Attention review, "What carries the
 * argument": chunk representation sqrt(|C|) times the mean key).
 *   K       [B, Hkv, L, d]  in k_dt (bf16 or fp32)
 *   lm_out  [B, Hkv, floor(L/S), d] fp32 -- one landmark per complete chunk;
 *           a partial tail chunk has none (it is never selectable).
 * Kept in fp32 because bf16 rounding of a landmark (2^-9 relative) would move
 * selection scores by more than the separation of near-tied chunks.
 */
hsa_status_t hsa_landmarks(const void *K, hsa_dtype_t k_dt, float *lm_out,
                           int B, int Hkv, int64_t L, int d, int S, void *stream);

/*
 * hsa_prefill_workspace_size -- bytes of device workspace hsa_prefill needs
 * for these sizes (0 on invalid arguments).  The workspace holds the group
 * selection, the fusion weights, the chunk-bucketed work list, per-entry
 * partial outputs and a status word.  A new workspace must be zero-filled
 * once before its first use; every completed call leaves it reusable.
 */
size_t hsa_prefill_workspace_size(int B, int H, int Hkv, int64_t L, int d, int S, int topk);

/*
 * hsa_prefill -- causal prefill of L query tokens against their own K/V.
 *   Q        [B, L, H, d]    dt (the G heads of a group are adjacent)
 *   K, V     [B, Hkv, L, d]  dt (one chunk = S contiguous rows)
 *   lm       [B, Hkv, floor(L/S), d] in lm_dt (bf16 or fp32), or NULL to use
 *            the DHSA form computed from K (hsa_landmarks, written into the
 *            workspace)
 *   own_chunk 1: add causal attention over keys c_t*S .. t (query t's own,
 *            unfinished chunk is never selectable); 0: retrieved chunks only.
 *   scale    logit scale for landmark scores and in-chunk logits; 0 -> 1/sqrt(d)
 *   O        [B, L, H, d]    dt, written
 *   idx_out  [B, L, Hkv, topk] int32 or NULL: selected chunks in rank order
 *            (best first), -1 where fewer than topk chunks are visible
 *   w_out    [B, L, H, topk] fp32 or NULL: fusion weights (0 on padded slots)
 * L need not be a multiple of S.  A query with no visible chunk and
 * own_chunk = 0 gets O = 0.
 */
hsa_status_t hsa_prefill(const void *Q, const void *K, const void *V, hsa_dtype_t dt,
                         const void *lm, hsa_dtype_t lm_dt,
                         int B, int H, int Hkv, int64_t L, int d, int S, int topk,
                         int own_chunk, float scale,
                         void *O, int32_t *idx_out, float *w_out,
                         void *workspace, size_t ws_bytes, void *stream);

/*
 * Retrieval variants of the prefill (hsa_prefill_variant).  Zero-filled it is
 * hsa_prefill's method except retrieval_interval, which must then be 1.
 *  retrieval_interval  R >= 1 dividing S: one selection per block of R
 *                      consecutive tokens (blocks start at token 0), shared by
 *                      the block's tokens; 1 = per-token retrieval.  The HSA
 *                      summary ("Main Findings") compares per-token with
 *                      per-8-token retrieval (R = 8).
 *  pool_mean           0: the block's selection is that of its first token
 *                      (its group query, its visible chunks -- the block never
 *                      straddles a chunk, so all its tokens see the same ones);
 *                      1: the group query is the mean over the block's tokens
 *                      (with R = S, the DHSA chunk-level query: sqrt(|C|) times
 *                      the mean of the chunk's queries, "What carries the
 *                      argument"; the positive factor does not change the
 *                      ranking).  The fusion weights stay per token.
 *  union_softmax       0: softmax inside each selected chunk, outputs fused by
 *                      the softmax of the token's landmark scores (HiLS);
 *                      1: one softmax over the keys of all selected chunks and,
 *                      with own_chunk, of the own chunk's keys c_t*S .. t (the
 *                      DHSA form of attention under the selected-chunk mask);
 *                      w_out is then all zero.
 */
typedef struct {
    int retrieval_interval;
    int pool_mean;
    int union_softmax;
} hsa_variant_t;

/*
 * hsa_prefill_variant -- hsa_prefill with a retrieval variant (NULL: the
 * per-token HiLS method of hsa_prefill, which calls this).  Same arguments,
 * layouts, workspace (hsa_prefill_workspace_size) and statuses; an invalid
 * variant returns HSA_ERR_INVALID_ARG.
 */
hsa_status_t hsa_prefill_variant(const void *Q, const void *K, const void *V, hsa_dtype_t dt,
                                 const void *lm, hsa_dtype_t lm_dt,
                                 int B, int H, int Hkv, int64_t L, int d, int S, int topk,
                                 int own_chunk, float scale, const hsa_variant_t *variant,
                                 void *O, int32_t *idx_out, float *w_out,
                                 void *workspace, size_t ws_bytes, void *stream);

/*
 * Variable-length chunks (Dynamic Hierarchical Sparse Attention review, "What
 * carries the argument": chunks of varying size, each represented by
 * sqrt(|C|) times the mean of its keys, which keeps the landmark scores of
 * chunks of different sizes comparable).  The chunks are given by their
 * boundaries, shared by the batch:
 *   bounds   [n_chunks + 1] int32, DEVICE, 0 = b_0 < b_1 < ... < b_n = L;
 *            chunk c holds tokens b_c .. b_{c+1} - 1, at most 64 of them
 * Everything else is hsa_prefill's method with chunk c in place of the
 * fixed chunks: token t selects among the chunks before the chunk holding t,
 * attends inside each selected chunk (all its keys) and, with own_chunk,
 * causally over its own chunk from that chunk's first token.  With lm = NULL
 * the landmarks are sqrt(|C|) * mean of each chunk's keys; an lm given is
 * [B, Hkv, n_chunks, d].  union_softmax as in hsa_variant_t.  Every chunk has
 * a landmark (the last one too, unlike the fixed-size form's partial tail).
 * The boundaries are checked on the device: wrong ones make hsa_check return
 * HSA_ERR_INVALID_ARG, and the call then computes as if the boundaries were
 * the even split b_c = floor(c * L / n_chunks) (so no kernel reads or writes
 * outside its buffers).  On the host: HSA_ERR_INVALID_ARG unless
 * 1 <= n_chunks <= L <= 64 * n_chunks (L = 0 returns HSA_OK) and bounds is a
 * 16-byte aligned device pointer.  Two more kernels than hsa_prefill (the
 * check and the token-to-chunk table).
 */
size_t hsa_prefill_varlen_workspace_size(int B, int H, int Hkv, int64_t L, int d, int64_t n_chunks,
                                         int topk);
hsa_status_t hsa_prefill_varlen(const void *Q, const void *K, const void *V, hsa_dtype_t dt,
                                const void *lm, hsa_dtype_t lm_dt, int B, int H, int Hkv,
                                int64_t L, int d, const int32_t *bounds, int64_t n_chunks,
                                int topk, int own_chunk, float scale, int union_softmax,
                                void *O, int32_t *idx_out, float *w_out, void *workspace,
                                size_t ws_bytes, void *stream);

/*
 * Prefill backward (HiLS Attention abstract: the retrieval scores are trained
 * end to end by the language-model loss; HSA "Methodology in Plain English"
 * for the forward it differentiates).  Gradients of sum(dO * O) for the
 * hsa_prefill forward, with the selection held fixed (a hard top-K has no
 * gradient): `idx` is the forward's selection.  Per query row (t, h) of group
 * g with selected chunks i_1 .. i_K, w = softmax_k(scale q.l_{i_k}) and
 * p_k = softmax_j(scale q.k_j) over chunk i_k (own chunk: weight 1, keys
 * c_t*S .. t):
 *   u_kj = dO.v_j, dw_k = p_k.u_k, dz_k = w_k (dw_k - sum_k' w_k' dw_k'),
 *   da_kj = w_k p_kj (u_kj - dw_k);
 *   dQ[t,h]   = scale (sum_kj da_kj k_j + sum_k dz_k l_{i_k})
 *   dK[j]    += scale da_kj q,  dV[j] += w_k p_kj dO,  dlm[i_k] += scale dz_k q
 * and with DHSA landmarks (lm = NULL, l = sqrt(S) * mean of the chunk's keys,
 * as hsa_prefill computes them) dlm / sqrt(S) is added to every key of the
 * chunk instead of being returned.
 *   Q, dO    [B, L, H, d]       dt (bf16 or fp32)
 *   K, V     [B, Hkv, L, d]     dt
 *   lm       [B, Hkv, L/S, d]   lm_dt, or NULL (DHSA)
 *   idx      [B, L, Hkv, topk]  int32, the forward's selection (-1: empty
 *                               slot; an entry naming a chunk that is not
 *                               before the token's own chunk is skipped and
 *                               reported by hsa_check as HSA_ERR_INVALID_ARG)
 *   dQ       [B, L, H, d]       fp32, written
 *   dK, dV   [B, Hkv, L, d]     fp32, written (every row)
 *   dlm      [B, Hkv, L/S, d]   fp32, written; required when lm is given,
 *                               ignored (may be NULL) in DHSA mode
 * Gradients accumulate in fp32 in a fixed order: the results are
 * bit-reproducible run to run.  Two paths: bf16 inputs with G = 8 and d = 128
 * run the key pass on the tensor cores (per chunk tile S = Q.K^T, U = dO.V^T,
 * then dV^T += dO^T.(w P), dK^T += Q^T.dS and the dQ partial dS.K, with P and
 * dS rounded to bf16 as the forward rounds P: ~2^-9 relative per term);
 * every other shape (or HSA_PATH_SIMT_PREFILL) runs on CUDA cores in fp32: a
 * row pass (dQ and the fusion coefficients) and a key pass.  Both sort the
 * selection by chunk (stable), cut it into segments of at most 1024 query
 * rows and add the segments' partials in order.  Supports L < 2^26 and B*Hkv*L*topk < 2^31
 * (else HSA_ERR_UNSUPPORTED); workspace from
 * hsa_prefill_backward_workspace_size (dhsa = 1 when lm will be NULL), no
 * zero-fill needed.  All buffers 16-byte aligned.
 */
size_t hsa_prefill_backward_workspace_size(int B, int H, int Hkv, int64_t L, int d, int S,
                                           int topk, int dhsa);
hsa_status_t hsa_prefill_backward(const void *Q, const void *K, const void *V, hsa_dtype_t dt,
                                  const void *lm, hsa_dtype_t lm_dt, const int32_t *idx,
                                  const void *dO, int B, int H, int Hkv, int64_t L, int d, int S,
                                  int topk, int own_chunk, float scale, float *dQ, float *dK,
                                  float *dV, float *dlm, void *workspace, size_t ws_bytes,
                                  void *stream);

/*
 * hsa_decode_workspace_size -- bytes of device workspace hsa_decode needs
 * (0 on invalid arguments; the size depends on the current device's SM
 * count).  It holds a status word, per-(sequence, group) tickets and work
 * counters (right after the status word), the selection and the per-block
 * candidate lists.  The tickets and counters must be zero when a call starts:
 * zero-fill a workspace before its first use and whenever the previous call
 * on it had another B*Hkv or it held anything else in between (a completed
 * call leaves at zero only the tickets and counters it used; the selection
 * and candidates of a call with fewer (sequence, group) pairs lie where a
 * larger call's counters go).  Calls that share a workspace must be ordered
 * (same stream).
 */
size_t hsa_decode_workspace_size(int B, int H, int Hkv, int64_t Lc, int d, int S, int topk);

/*
 * hsa_decode -- one new query per sequence at position Lc against a KV cache
 * of Lc tokens (Lc % S == 0): every one of the Lc/S chunks is visible and
 * there is no own-chunk term (local attention around the new token belongs to
 * the model's sliding-window layers, not to this operator).
 *   q        [B, H, d]          dt
 *   Kc, Vc   [B, Hkv, Lc, d]    dt; only the selected chunks are read
 *   lm       [B, Hkv, Lc/S, d]  lm_dt (bf16 or fp32)
 *   O        [B, H, d]          dt, written
 *   idx_out  [B, Hkv, topk] int32 or NULL
 * Two kernels: the landmark scan is split over many thread blocks and the
 * last block of each (sequence, KV group) merges their top-K lists into the
 * selection; then a cluster of min(topk, 8) blocks per (sequence, group)
 * gathers the selected chunks, attends inside them and fuses the results into
 * O (launched as a programmatic dependent of the scan).  Cache offsets are
 * 64-bit (Lc up to 2^31 - 1 tokens).
 */
hsa_status_t hsa_decode(const void *q, const void *Kc, const void *Vc, hsa_dtype_t dt,
                        const void *lm, hsa_dtype_t lm_dt,
                        int B, int H, int Hkv, int64_t Lc, int d, int S, int topk, float scale,
                        void *O, int32_t *idx_out,
                        void *workspace, size_t ws_bytes, void *stream);

/*
 * hsa_decode_ragged -- hsa_decode over a batch of caches of different lengths
 * (ragged batch): sequence b holds lens[b] tokens of a cache allocated for
 * Lmax (Lmax % S == 0, the row stride of Kc, Vc and lm) and its new query
 * retrieves among its first floor(lens[b] / S) chunks, the complete ones (HSA
 * "Methodology in Plain English": the query retrieves among the chunks
 * before it; the incomplete chunk holding the newest tokens is the sliding
 * window's, as in hsa_decode).  A sequence with no complete chunk gets O = 0
 * and an all -1 selection.
 *   lens     [B] int32, DEVICE (16-byte aligned); a length outside 0 .. Lmax
 *            is clamped and makes hsa_check return HSA_ERR_INVALID_ARG
 * Everything else, including the workspace (hsa_decode_workspace_size with
 * Lc = Lmax), is hsa_decode's.  The scan reads only each sequence's visible
 * landmark rows.
 */
hsa_status_t hsa_decode_ragged(const void *q, const void *Kc, const void *Vc, hsa_dtype_t dt,
                               const void *lm, hsa_dtype_t lm_dt, int B, int H, int Hkv,
                               int64_t Lmax, int d, int S, int topk, float scale,
                               const int32_t *lens, void *O, int32_t *idx_out, void *workspace,
                               size_t ws_bytes, void *stream);

/*
 * hsa_decode_noalloc -- hsa_decode for callers that cannot allocate device
 * memory.  (The pages describe no such call; it is an interface convenience
 * of this library.)  Some callers cannot hand hsa_decode a workspace: a
 * plugin inside a host program that owns all device memory (for example a
 * serving engine that reserves the whole HBM for its KV cache at start-up and
 * passes a plugin only its inputs and outputs), or code on a latency-critical
 * path that must not call cudaMalloc/cudaFree because they can synchronise
 * the device.  This entry point takes the same arguments as hsa_decode minus
 * the workspace and allocates nothing: its scratch is one fixed array of
 * hsa_decode_noalloc_max_scratch() bytes (1 MiB) in device global memory that
 * the library declares statically, so every GPU that loads the library holds
 * it until the process exits.
 *  - Sizes whose scratch (hsa_decode_workspace_size) exceeds that array are
 *    rejected with HSA_ERR_WORKSPACE before anything is launched; invalid
 *    arguments return the same status hsa_decode would.
 *  - Every call looks up the array's device address on the stream's device
 *    (cudaGetSymbolAddress, with that device current); the first call on a
 *    device loads the array, so make it before any stream capture on that
 *    device.  The stream's device must be the current device, as for
 *    hsa_decode.
 *  - Every call on a device shares the one array, and the array keeps the
 *    previous call's contents.  Each call clears the part that must start at
 *    zero (tickets and work counters) with cudaMemsetAsync on `stream`.
 *    Calls that can overlap on the GPU (different streams, or several host
 *    threads without ordering) race on the array and give wrong results:
 *    order them on one stream.
 *  - The array starts with a status word.  A call whose device-side bounded
 *    wait runs out sets its timeout flag there; the flag survives later calls
 *    until hsa_check(NULL, stream) returns HSA_ERR_TIMEOUT and clears it.
 *  - No cudaMalloc, cudaFree or other allocating routine is called.
 */
hsa_status_t hsa_decode_noalloc(const void *q, const void *Kc, const void *Vc, hsa_dtype_t dt,
                                const void *lm, hsa_dtype_t lm_dt,
                                int B, int H, int Hkv, int64_t Lc, int d, int S, int topk,
                                float scale, void *O, int32_t *idx_out, void *stream);

/* hsa_decode_noalloc_max_scratch -- size in bytes of hsa_decode_noalloc's array. */
size_t hsa_decode_noalloc_max_scratch(void);

/*
 * Context-parallel decode: hsa_decode for a KV cache cut along the sequence
 * into R contiguous chunk ranges (shards), one per GPU, for contexts larger
 * than one GPU's memory (the HSA summary reports retrieval up to 32M tokens,
 * "Main Findings").  The method is unchanged; only where its steps run moves.
 * Each rank calls, in order:
 *   1. hsa_decode_cp_candidates on its shard: the shard's top-K chunks by the
 *      group score, as (score, global chunk index) candidates;
 *   2. an all-gather of the candidates over the R ranks (the caller's
 *      collective, e.g. NCCL), then hsa_decode_cp_merge: the global top-K in
 *      the single-GPU order (larger score first, lower index on ties).  A
 *      chunk of the global top-K is within its own shard's top K, so the
 *      selection equals hsa_decode's;
 *   3. hsa_decode_cp_attend on its shard: attention inside the selected
 *      chunks it holds, folded into a per-head fusion state m (largest fusion
 *      logit), Z (sum of exp(z - m)), acc (sum of exp(z - m) * chunk output);
 *   4. an all-gather of the states, then hsa_decode_cp_combine: O, the
 *      fusion softmax over the selection written as a sum over shards.
 * Every rank gets the same idx and O.  Shard r holds chunks
 * [chunk_offset, chunk_offset + Lc/S) of the whole cache, Lc its own length
 * (a multiple of S, may be 0); q is the same on every rank.
 */
/* Step 1.  lm [B, Hkv, Lc/S, d]; cand_score [B, Hkv, topk] fp32 and cand_idx
 * [B, Hkv, topk] int32 (global chunk indices, best first; -1 and score 0 where
 * the shard has fewer than topk chunks).  workspace as for hsa_decode with the
 * shard's sizes (hsa_decode_workspace_size(B, H, Hkv, Lc, d, S, topk)). */
hsa_status_t hsa_decode_cp_candidates(const void *q, hsa_dtype_t dt, const void *lm,
                                      hsa_dtype_t lm_dt, int B, int H, int Hkv, int64_t Lc, int d,
                                      int S, int topk, float scale, int64_t chunk_offset,
                                      float *cand_score, int32_t *cand_idx, void *workspace,
                                      size_t ws_bytes, void *stream);
/* Step 2.  cand_score / cand_idx [R, B, Hkv, topk] (the gathered step-1
 * outputs, in rank order) -> idx [B, Hkv, topk] (-1 padded). */
hsa_status_t hsa_decode_cp_merge(const float *cand_score, const int32_t *cand_idx, int R, int B,
                                 int Hkv, int topk, int32_t *idx, void *stream);
/* Step 3.  Kc, Vc [B, Hkv, Lc, d], lm [B, Hkv, Lc/S, d] (the shard's), idx
 * [B, Hkv, topk] from step 2 -> m, Z [B, H] and acc [B, H, d] fp32 (m = -inf,
 * Z = 0, acc = 0 for heads whose group has no selected chunk on this shard). */
hsa_status_t hsa_decode_cp_attend(const void *q, const void *Kc, const void *Vc, hsa_dtype_t dt,
                                  const void *lm, hsa_dtype_t lm_dt, int B, int H, int Hkv,
                                  int64_t Lc, int d, int S, int topk, float scale,
                                  int64_t chunk_offset, const int32_t *idx, float *m, float *Z,
                                  float *acc, void *stream);
/* Step 4.  m, Z [R, B, H], acc [R, B, H, d] (gathered, rank order) ->
 * O [B, H, d] in dt: O = sum_r e^{m_r - M} acc_r / sum_r e^{m_r - M} Z_r,
 * M = max_r m_r (O = 0 where no shard held a selected chunk). */
hsa_status_t hsa_decode_cp_combine(const float *m, const float *Z, const float *acc, int R, int B,
                                   int H, int d, hsa_dtype_t dt, void *O, void *stream);

/*
 * hsa_selftest_wait_expiry -- exercises the failure path of the kernels'
 * bounded waits (see hsa_check): launches one block whose mbarrier wait can
 * never complete, because nothing arrives on it; after `budget_cycles` SM
 * cycles the block gives up, sets the timeout flag in the status word at the
 * head of `workspace` and exits, as every kernel of the library does when one
 * of its waits runs out.  A following hsa_check(workspace, stream) returns
 * HSA_ERR_TIMEOUT and clears the flag; the CUDA context stays usable.
 *   workspace     any workspace of this library (>= 16 bytes), zero-filled;
 *                 NULL aims at the status word of hsa_decode_noalloc's array
 *                 on the stream's device (then hsa_check(NULL, stream)
 *                 reports the flag)
 *   budget_cycles 1 .. 4e9 (2e6 is about 1 ms)
 * Returns HSA_ERR_INVALID_ARG for a bad argument, HSA_ERR_CUDA if the launch
 * fails, else HSA_OK (the expiry itself is reported by hsa_check).
 */
hsa_status_t hsa_selftest_wait_expiry(void *workspace, size_t ws_bytes, int64_t budget_cycles,
                                      void *stream);

/*
 * hsa_check -- synchronises `stream`, then reads the status word at the head
 * of `workspace` (the one given to the preceding hsa_prefill / hsa_decode).
 * Returns HSA_ERR_TIMEOUT if a device-side bounded wait gave up,
 * HSA_ERR_INVALID_ARG if hsa_prefill_varlen found its chunk boundaries wrong,
 * hsa_decode_ragged a length outside 0 .. Lmax or hsa_prefill_backward a
 * selection entry that names no visible chunk
 * (either clears the word), HSA_ERR_CUDA if the stream reports an error,
 * HSA_OK otherwise.
 * With workspace = NULL it reads the status word of hsa_decode_noalloc's
 * array on the stream's device (if this process has used that array there),
 * which collects the flags of every hsa_decode_noalloc call since the last
 * check.
 */
hsa_status_t hsa_check(void *workspace, void *stream);

/*
 * hsa_set_stage_events -- timing hook for benchmarks.  Until called again
 * with n = 0, hsa_prefill and hsa_decode calls made by the CALLING THREAD
 * record events[i] (cudaEvent_t values passed as void*) on their stream at
 * stage boundary i, for i < n:
 *   hsa_prefill: 0 start, 1 after the landmark kernel (DHSA mode), 2 after
 *                selection, 3 after the work-list build, 4 after the
 *                attention kernel, 5 after the fusion kernel (end of the
 *                call; 4 and 5 coincide on the path that fuses in place);
 *   hsa_decode, hsa_prefill_backward:  0 start, 1 end.
 * Boundaries a call does not reach are not recorded.  n must be 0..8.  The
 * events belong to the caller.  No effect on results.
 */
hsa_status_t hsa_set_stage_events(void *const *events, int n);

/*
 * hsa_last_call_launches -- number of kernels the calling thread's most
 * recent hsa_prefill* / hsa_decode* / hsa_landmarks / hsa_prefill_backward
 * call launched.
 */
int hsa_last_call_launches(void);

/*
 * hsa_last_call_kernels -- the kernel families (HSA_K_* bits) that the calling
 * thread's most recent hsa_prefill* / hsa_decode* / hsa_landmarks /
 * hsa_prefill_backward call launched: which path the dispatch took for those
 * sizes and dtypes.
 */
unsigned hsa_last_call_kernels(void);

/*
 * hsa_set_path_overrides -- testing and measurement hook.  Until called again,
 * hsa_prefill and hsa_prefill_workspace_size calls made by the CALLING THREAD
 * take the paths named by `flags` (HSA_PATH_* bits; 0 = the library's own
 * choice) and, if window_tokens > 0, split the tensor-core work lists into
 * token windows of that many tokens (rounded down to a multiple of 256; 0 =
 * the library's own choice).  Results are the same on every path up to the
 * rounding of each; a workspace must be sized under the same overrides as
 * the call that uses it.  Returns HSA_ERR_INVALID_ARG for unknown flags or a
 * window of 1..255 tokens.  The library reads no environment variables.
 */
hsa_status_t hsa_set_path_overrides(int flags, int64_t window_tokens);

/* hsa_status_string -- static, NUL-terminated description of a status. */
const char *hsa_status_string(hsa_status_t status);

/* hsa_version -- library version as major*10000 + minor*100 + patch. */
int hsa_version(void);

#ifdef __cplusplus
}
#endif
#endif /* HSA_H_ */
