/*
 * lsa.h -- C ABI of the LSA (LongCat Sparse Attention) hot path for NVIDIA B200 (sm_100a).
 *
 * Sources.  The operations follow the LongCat-2.0 pages:
 *   [release]   "美团大模型LongCat-2.0 正式发布，总参数量达 1.6 万亿，使用国产算力集群",
 *               section "LongCat 稀疏注意力" (SI, CLI and HI bullets; MTP paragraph) and
 *               section "确定性与可靠性" (deterministic operators, tree reductions);
 *   [explainer] "如何在 5 万张国产芯片训练出 1.6T 万亿参数模型？", section
 *               "① LSA：从“每个 Query 全量扫”改成“先索引、再稀疏读”" and section
 *               "③ KVP 解码切分示意" (partial attention per KV shard, then merged).
 * The pages give no formula; the indexer score is the DSA form
 *   I(t,s) = sum_h w[t,h] * ReLU(q[t,h,:] . k[s,:]),
 * and the top-k order is (score descending, position ascending).
 *
 * Conventions for every entry point.
 *   - All tensor pointers are DEVICE pointers, allocated and owned by the caller; the
 *     library allocates, frees and synchronises nothing on these paths.  Structs
 *     (lsa_batch, lsa_cache, lsa_layer, lsa_decode_params) are read on the host during
 *     the call and may be discarded when it returns.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is enqueued
 *     asynchronously; outputs are valid once the stream reaches that point.
 *   - Host-side argument validation fails with a status and launches nothing.
 *     A launch failure returns LSA_ERR_CUDA.
 *   - Bad DEVICE data (q_pos >= seq_len, an index outside 0..seq_len-1, a NaN score,
 *     a sequence id outside 0..B-1) is detected in the kernels: the offending access is
 *     skipped and, when `dev_status` is not NULL, an lsa_status code is stored there
 *     (the first error wins).  `dev_status` points to one int32 in device memory that
 *     the caller zeroes before use; read it with lsa_read_device_status.  Kernels never
 *     trap.
 *   - Deterministic: identical inputs and parameters (including n_split) give bitwise
 *     identical outputs.  No floating-point atomics are used; every reduction has a
 *     fixed order.
 *   - Element strides are counted in elements of the cache's dtype.
 *   - No exception crosses this boundary.  Calls on different streams may run
 *     concurrently as long as their output buffers do not overlap.
 *   - One call handles at most 65,535 query tokens and 65,535 sequences (some kernels put
 *     the token in a grid dimension of that size); larger batches return
 *     LSA_ERR_UNSUPPORTED before anything is launched.
 */
#ifndef LSA_H_
#define LSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LSA_OK = 0,
    LSA_ERR_INVALID_ARG = 1,   /* host validation: null pointer, bad size, misalignment */
    LSA_ERR_UNSUPPORTED = 2,   /* valid request outside what the kernels implement */
    LSA_ERR_WORKSPACE = 3,     /* workspace missing or smaller than the *_workspace_size result */
    LSA_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed */
    LSA_ERR_DEVICE_DATA = 5,   /* (device) bad lengths / positions / indices, NaN score */
    LSA_ERR_TIMEOUT = 6        /* (device) a bounded wait gave up */
} lsa_status;

typedef enum { LSA_BF16 = 0, LSA_FP8_E4M3 = 1, LSA_FP32 = 2 } lsa_dtype;

/* lsa_topk flags */
#define LSA_TOPK_RAW (1u << 0) /* output the selected COLUMN ids, no sink/window union (HI recall) */
#define LSA_TOPK_EXCLUDES_FIXED (1u << 1) /* fixed-budget SI: top-k drawn outside sinks and window */
#define LSA_TOPK_WINDOW_ALIGNED (1u << 2) /* SI window starts on a 64-row boundary */

/* A per-sequence cache: row r of sequence b starts at
 *   data + b * seq_stride + r * tok_stride            (elements of `dtype`),
 * and its FP8 scale (one float per row, FP8 caches only) at
 *   scale[b * scale_seq_stride + r].
 * A row's value is data (BF16) or scale * data (FP8 e4m3, OCP definition). */
typedef struct {
    const void*  data;
    const float* scale;            /* FP8: per-token scale (> 0); BF16: NULL */
    int32_t      dtype;            /* LSA_BF16 or LSA_FP8_E4M3 */
    int32_t      dim;              /* elements per row */
    int64_t      seq_stride;       /* elements between sequences */
    int64_t      tok_stride;       /* elements between rows (>= dim) */
    int64_t      scale_seq_stride; /* floats between sequences in `scale` */
} lsa_cache;

/* The query tokens of one call.  Token t belongs to sequence q_seq[t] and sits at
 * position q_pos[t]; it sees keys 0..q_pos[t] (causal).  Tokens are grouped in runs of
 * `q_group` consecutive tokens of the same sequence (1 for plain decode, the verify
 * length for speculative decoding, the chunk length for prefill); kernels read a
 * sequence's keys once per group. */
typedef struct {
    int32_t        B;          /* sequences */
    int32_t        T;          /* query tokens, a multiple of q_group */
    int32_t        q_group;    /* consecutive tokens sharing a sequence */
    int32_t        L_alloc;    /* rows allocated per sequence in the caches */
    const int32_t* seq_len;    /* device [B], 1 <= seq_len[b] <= L_alloc */
    const int32_t* q_seq;      /* device [T], 0 <= q_seq[t] < B */
    const int32_t* q_pos;      /* device [T], 0 <= q_pos[t] < seq_len[q_seq[t]] */
} lsa_batch;

/* ---------------------------------------------------------------- a1 / a4: indexer
 * Indexer scores  I(t,s) = sum_h w[t,h] * ReLU(q_idx[t,h,:] . k(s))  for the key rows k(s)
 * of the indexer cache ([release] "LongCat 稀疏注意力": the lightweight indexer that
 * scores keys for each query; DSA form).  FP8 keys contribute scale(s) * code(s).
 *   q_idx  [T][H_I][d_I] BF16, d_I = k_idx->dim (64 or 128);  w [T][H_I] float.
 *   Flat (cand_blocks == NULL): scores[t * ld_scores + s] for s < n_cols, the score when
 *     s <= q_pos[t], -INFINITY otherwise.
 *   Fine stage of HI (cand_blocks != NULL): cand_blocks [T][n_cand] int32 block ids
 *     (ascending, -1 = unused); column c < n_cand * block_size is position
 *     cand_blocks[t][c / block_size] * block_size + c % block_size; its score, or
 *     -INFINITY when the block id is -1 or the position is beyond q_pos[t].
 *   Requires H_I % 8 == 0, H_I <= 128, ld_scores >= number of columns, 16-byte aligned
 *   q_idx / data / rows. */
lsa_status lsa_index_score(const lsa_batch* batch, const void* q_idx, const float* w, int H_I,
                           const lsa_cache* k_idx, const int32_t* cand_blocks, int n_cand,
                           int block_size, float* scores, int64_t ld_scores, int n_cols,
                           int32_t* dev_status, void* stream);

/* lsa_index_score in FP8-query mode: the DSA-style indexer's e4m3 queries.  Each row
 * q_idx[t,h,:] is scaled by the power of two 2^s (s = 7 - floor(log2 max|q_idx[t,h,:]|),
 * clamped to [-126, 126]; 0 for an all-zero row), rounded to e4m3 (nearest, ties to even,
 * saturating) and scaled back, and the scores use those queries: half the tensor-core work of
 * the exact BF16-query mode.  Same arguments and results otherwise.  Needs the tensor-core
 * path (FP8 keys, d_I = 128, H_I a multiple of 32, block_size 64 for HI); returns
 * LSA_ERR_UNSUPPORTED elsewhere. */
lsa_status lsa_index_score_q8(const lsa_batch* batch, const void* q_idx, const float* w, int H_I,
                              const lsa_cache* k_idx, const int32_t* cand_blocks, int n_cand,
                              int block_size, float* scores, int64_t ld_scores, int n_cols,
                              int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------- a2: HI block keys
 * Block key of block j of sequence b = arithmetic mean of the dequantised indexer keys
 * of rows j*block_size .. min(seq_len[b], (j+1)*block_size) - 1 ([release] HI bullet:
 * block-level approximate scoring; the mean is this library's block summary).
 *   kbar: BF16 bits, sequence b at kbar + b * kbar_seq_stride (uint16 elements), 2 * d_I
 *   per block: row j holds hi[0..d_I) then lo[0..d_I), where m is the mean computed in FP32
 *   (fixed pairwise summation order), hi = m rounded to BF16 and lo = (m - hi) rounded to
 *   BF16; the block key is hi + lo (16 significant bits, relative error <= 2^-17 of m).
 *   Blocks 0 .. ceil(seq_len[b] / block_size) - 1 are written.  Requires
 *   kbar_seq_stride >= ceil(L_alloc / block_size) * 2 * d_I, a multiple of 8, and kbar
 *   16-byte aligned.  Cache maintenance: rerun for the blocks whose rows changed (here: all). */
lsa_status lsa_block_keys(const lsa_batch* batch, const lsa_cache* k_idx, int block_size,
                          void* kbar, int64_t kbar_seq_stride, int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------- a2: HI block scores
 * J(t,j) = sum_h w[t,h] * ReLU(q_idx[t,h,:] . kbar(q_seq[t], j)) for block columns
 * j < n_cols, kbar(b, j) = hi + lo as written by lsa_block_keys: the score when block j is
 * visible (j * block_size <= q_pos[t]), else -INFINITY.  d_I = dimension of q_idx rows
 * (64 or 128).  Same layout requirements on kbar as lsa_block_keys.  For H_I a multiple of
 * 32 the scores come from the tensor cores (BF16 MMA over K = 2 d_I: [hi | lo] against
 * [q | q], exact products, FP32 accumulation); otherwise from FP32 CUDA-core dot products. */
lsa_status lsa_block_score(const lsa_batch* batch, const void* q_idx, const float* w, int H_I, int d_I,
                           const void* kbar, int64_t kbar_seq_stride, int block_size,
                           float* scores, int64_t ld_scores, int n_cols,
                           int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------- a3 / a5: top-k and union
 * Per query row t: candidates are the columns c < n_cols with scores[t * ld + c] != -inf.
 * The k candidates ranked first by (score desc, column asc) are selected (all of them if
 * fewer); -0 ranks equal to +0; a NaN score sets LSA_ERR_DEVICE_DATA and is ignored.
 *   Default: columns map to positions (identity, or through cand_blocks as in
 *   lsa_index_score); the output is the ascending, de-duplicated union of the selected
 *   positions, the sinks 0..n_sink-1 and the SI window q_pos-window+1..q_pos, all clipped
 *   to 0..q_pos ([explainer] "① LSA": top-k keys plus a few fixed sink tokens; [release]
 *   SI bullet: a contiguous, hardware-aligned window beside the dynamic picks).
 *   LSA_TOPK_RAW: the output is the selected column ids, ascending (HI coarse recall);
 *   n_sink and window must be 0.
 *   LSA_TOPK_EXCLUDES_FIXED: fixed-budget SI -- columns at sink or window positions are no
 *   candidates, so the k picks come from the other visible positions and the (disjoint) list
 *   holds min(k, those) + the sinks + the window ([release] SI bullet, read as a budget split
 *   between the contiguous part and the dynamic picks).  Not with LSA_TOPK_RAW.
 *   LSA_TOPK_WINDOW_ALIGNED: the window starts at max(0, q_pos - window + 1) rounded down to a
 *   multiple of 64, so it covers whole 64-row blocks up to the query (window .. window + 63
 *   positions; [release] SI bullet: hardware-aligned contiguous reads).  Combines with
 *   LSA_TOPK_EXCLUDES_FIXED; not with LSA_TOPK_RAW.
 *   idx [T][ld_idx] int32, entries beyond count[t] set to -1; count [T] int32.
 *   ld_idx >= k + n_sink + window (+ 63 with LSA_TOPK_WINDOW_ALIGNED and window > 0). */
lsa_status lsa_topk(const lsa_batch* batch, const float* scores, int64_t ld_scores, int n_cols,
                    const int32_t* cand_blocks, int n_cand, int block_size,
                    int k, int n_sink, int window, uint32_t flags,
                    int32_t* idx, int64_t ld_idx, int32_t* count,
                    int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------- a7 / a8: sparse attention
 * For each query token t and head h, softmax attention over the rows idx[t][0..count[t]-1]
 * of sequence q_seq[t] ([explainer] "① LSA": attention reads only the selected keys):
 *   z_j = sm_scale * q[t,h,:] . K_j,  o[t,h,:] = sum_j softmax(z)_j V_j,
 *   lse[t,h] = log sum_j exp(z_j)  (natural log; -inf and o = 0 for an empty list).
 * K_j is row j of `kv` (dim = Dqk).  V_j is row j of `v` (dim = Dv) or, when v == NULL,
 * the first Dv elements of K_j (MLA absorbed layout).  FP8 rows are scale * code.
 * The list is cut into n_split contiguous chunks processed in parallel; the partial
 * results are merged with the log-sum-exp rule in chunk order ([explainer]
 * "③ KVP 解码切分示意": partial attention per KV shard, then merged -- here the shards are
 * chunks of one GPU's work).
 *   q [T][H][Dqk] BF16, o [T][H][Dv] BF16, lse [T][H] float (may be NULL).
 *   Supported: (Dqk, Dv) = (576, 512) with H % 32 == 0, or (128, 128) with H % 16 == 0;
 *   1 <= n_split <= 64.  ws: lsa_attn_workspace_size(T, H, Dv, n_split) bytes (0 when
 *   n_split == 1; ws may then be NULL). */
lsa_status lsa_sparse_attn(const lsa_batch* batch, const void* q, int H, int Dqk,
                           const lsa_cache* kv, const lsa_cache* v, int Dv,
                           const int32_t* idx, int64_t ld_idx, const int32_t* count,
                           float sm_scale, int n_split, void* o, float* lse,
                           void* ws, size_t ws_bytes, int32_t* dev_status, void* stream);

size_t lsa_attn_workspace_size(int T, int H, int Dv, int n_split);

/* ---------------------------------------------------------------- sparse attention without allocation
 * The pages have no counterpart to this entry point; it exists for callers that cannot
 * allocate device memory (a serving runtime whose memory pool forbids new allocations, a
 * plugin host that owns every cudaMalloc) and so cannot provide lsa_sparse_attn's
 * workspace.  Same arguments, results and determinism as lsa_sparse_attn, minus the
 * workspace: the split-KV partials live in one static device array of
 * LSA_NOALLOC_SCRATCH_BYTES inside this library, which every GPU that loads the library
 * holds until the process exits.  The call allocates nothing.
 *   - Returns LSA_ERR_WORKSPACE when lsa_attn_workspace_size(T, H, Dv, n_split) exceeds
 *     LSA_NOALLOC_SCRATCH_BYTES (at Dv = 512: T * n_split * H at most 16,352);
 *     n_split == 1 needs no scratch.
 *   - Arguments are checked exactly as lsa_sparse_attn checks them (same statuses); the
 *     scratch size is checked after those checks.
 *   - The first call with n_split > 1 on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call before any
 *     stream capture.  The address is kept per device and CUDA context: after a device
 *     reset (which destroys the context and the array with it) the next call looks it up
 *     again in the new context, so that call too should come before any capture.
 *   - Every call shares the one array and it keeps the last call's contents; nothing in
 *     it needs to start at zero (each call writes every partial it reads).  Calls whose
 *     execution overlaps on the GPU (other streams, other threads, concurrent graphs)
 *     race on the array and corrupt each other's results: serialise them. */
#define LSA_NOALLOC_SCRATCH_BYTES (32u << 20)
lsa_status lsa_sparse_attn_noalloc(const lsa_batch* batch, const void* q, int H, int Dqk,
                                   const lsa_cache* kv, const lsa_cache* v, int Dv,
                                   const int32_t* idx, int64_t ld_idx, const int32_t* count,
                                   float sm_scale, int n_split, void* o, float* lse,
                                   int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------- partial attention and its merge
 * lsa_sparse_attn with the result in FP32 and not normalised across calls: o_part [T][H][Dv]
 * float and lse_part [T][H] float (both required), the attention of each (token, head) over the
 * rows of its list only.  The partial results of disjoint row sets combine with
 * lsa_merge_partials ([explainer] "③ KVP 解码切分示意": per-shard partial attention, then the
 * merge).  Same arguments, workspace and determinism as lsa_sparse_attn otherwise. */
lsa_status lsa_sparse_attn_partial(const lsa_batch* batch, const void* q, int H, int Dqk,
                                   const lsa_cache* kv, const lsa_cache* v, int Dv,
                                   const int32_t* idx, int64_t ld_idx, const int32_t* count,
                                   float sm_scale, int n_split, float* o_part, float* lse_part,
                                   void* ws, size_t ws_bytes, int32_t* dev_status, void* stream);

/* Log-sum-exp merge of n_parts partial attentions over disjoint row sets, in part order:
 * with m = max_p lse_p and w_p = exp(lse_p - m), o = sum_p (w_p / sum w) o_p and
 * lse = m + log(sum w); a part with lse = -inf (no rows) contributes nothing, and all parts
 * empty give o = 0, lse = -inf.  o_parts [n_parts][T][H][Dv] float, lse_parts [n_parts][T][H]
 * float, o [T][H][Dv] BF16 (rounded to nearest even), lse [T][H] float or NULL.  Dv a multiple of
 * 8, 16-byte aligned o_parts and o; 1 <= n_parts <= 1024. */
lsa_status lsa_merge_partials(const float* o_parts, const float* lse_parts, int n_parts, int T, int H, int Dv,
                              void* o, float* lse, void* stream);

/* ---------------------------------------------------------------- KVP: one context over several ranks
 * [explainer] "③ KVP 解码切分示意" and [release] "推理" (decode nodes): the KV cache of a long
 * sequence is split over devices, each computes partial results over its shard, and the partial
 * results are merged.  Shard r of sequence b is the contiguous row range
 * shard_start[b] .. shard_start[b] + shard_len[b] - 1; the rank that holds it stores those rows as
 * rows 0 .. shard_len[b] - 1 of its own caches (indexer keys and KV).  Shards of a sequence are
 * disjoint, cover 0 .. seq_len[b] - 1 and are numbered in position order.  One step over R shards:
 *   1. lsa_kvp_shard_batch: the shard's local batch (local lengths and positions);
 *   2. lsa_index_score with the local batch and caches: the shard's scores;
 *   3. lsa_kvp_candidates: the shard's top-k as (global position, score) pairs;
 *   4. the caller gathers every shard's candidates, in shard order (an all-gather over ranks);
 *   5. lsa_kvp_select: the global top-k with sinks and window, the same on every rank and the same
 *      list as the single-device selection (each key of the global top-k is in the top-k of its
 *      shard, and the order (score desc, position asc) is kept);
 *   6. lsa_kvp_local_index: the selected rows of this shard, as local rows;
 *   7. lsa_sparse_attn_partial with the local batch and caches;
 *   8. the caller gathers every shard's partial results, in shard order;
 *   9. lsa_merge_partials.
 * Only the plain union (no LSA_TOPK_EXCLUDES_FIXED) and flat indexing are covered. */

/* local_seq_len[b] = shard_len[b]; local_q_pos[t] = clamp(q_pos[t] - shard_start[b], 0,
 * shard_len[b] - 1) (device [B] and [T] outputs).  The local batch is the global one with these
 * two arrays and L_alloc_local.  A shard outside 0 .. seq_len[b] - 1, or longer than
 * L_alloc_local, is bad device data. */
lsa_status lsa_kvp_shard_batch(const lsa_batch* global, int L_alloc_local, const int32_t* shard_start,
                               const int32_t* shard_len, int32_t* local_seq_len, int32_t* local_q_pos,
                               int32_t* dev_status, void* stream);

/* The top-k of the shard's local scores (scores [T][ld_scores], columns = local rows, as
 * lsa_index_score wrote them for the local batch) as global positions, ascending, and their
 * scores: cand_pos [T][k] int32 and cand_score [T][k] float, padded with (-1, -INFINITY);
 * cand_count [T] the number of pairs.  A token whose global position q_pos_global[t] precedes the
 * shard sees none of its keys and gets no pair. */
lsa_status lsa_kvp_candidates(const lsa_batch* local, const int32_t* q_pos_global, const int32_t* shard_start,
                              const float* scores, int64_t ld_scores, int n_cols, int k, int32_t* cand_pos,
                              float* cand_score, int32_t* cand_count, int32_t* dev_status, void* stream);

/* The global selection from every shard's candidates: cand_pos / cand_score [n_parts][T][k_part]
 * in shard order (as lsa_kvp_candidates wrote them, gathered).  The k pairs ranked first by
 * (score desc, position asc), unioned with the sinks and the window of the global batch, as
 * lsa_topk's default mode: idx [T][ld_idx] ascending, -1 padded, count [T].
 * ws: lsa_kvp_select_workspace_size(T, n_parts, k_part) bytes, 256-byte aligned. */
size_t lsa_kvp_select_workspace_size(int T, int n_parts, int k_part);
lsa_status lsa_kvp_select(const lsa_batch* global, const int32_t* cand_pos, const float* cand_score, int n_parts,
                          int k_part, int k, int n_sink, int window, int32_t* idx, int64_t ld_idx, int32_t* count,
                          void* ws, size_t ws_bytes, int32_t* dev_status, void* stream);

/* The entries of each token's global list idx[t][0..count[t]) that fall in the shard, minus
 * shard_start (local rows, ascending): local_idx [T][ld_local] (-1 padded), local_count [T].
 * ld_local >= ld_idx. */
lsa_status lsa_kvp_local_index(const lsa_batch* global, const int32_t* shard_start, const int32_t* shard_len,
                               const int32_t* idx, int64_t ld_idx, const int32_t* count, int32_t* local_idx,
                               int64_t ld_local, int32_t* local_count, int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------- fused decode / prefill step
 * One attention layer consuming a shared index list (cross-layer indexing: [release] CLI
 * bullet, one index serves consecutive layers; MTP paragraph, draft steps 2 and 3 reuse
 * step 1's index). */
typedef struct {
    const void* q;         /* [T][H][Dqk] BF16 */
    lsa_cache   kv;        /* K rows (and V = first Dv dims when v.data == NULL) */
    lsa_cache   v;         /* separate V cache, or v.data == NULL */
    void*       o;         /* [T][H][Dv] BF16 */
    float*      lse;       /* [T][H] or NULL */
} lsa_layer;

typedef struct {
    lsa_batch        batch;
    /* indexer */
    const void*      q_idx;      /* [T][H_I][d_I] BF16 */
    const float*     w;          /* [T][H_I] */
    int32_t          H_I;
    lsa_cache        k_idx;
    /* selection */
    int32_t          k, n_sink, window;
    /* hierarchical indexing (hi != 0): block keys kbar from lsa_block_keys */
    int32_t          hi, block_size, n_recall;
    const void*      kbar;            /* BF16 (hi, lo) pairs, as written by lsa_block_keys */
    int64_t          kbar_seq_stride; /* uint16 elements between sequences */
    /* attention layers sharing the index */
    int32_t          H, Dqk, Dv;
    float            sm_scale;
    int32_t          n_split;
    int32_t          n_layers;
    const lsa_layer* layers;     /* host array [n_layers] */
    /* optional: the index list and its counts are also written here ([T][idx_ld], [T]) */
    int32_t*         idx_out;
    int64_t          idx_ld;
    int32_t*         count_out;
    /* indexer queries: 0 = BF16 (exact), 1 = FP8-query mode (as lsa_index_score_q8; flat and
     * the fine stage of HI -- HI block scores keep the BF16 queries) */
    int32_t          idx_q_fp8;
    /* selection: 0 = top-k over all visible keys, then the union with sinks and window;
     * 1 = fixed budget (LSA_TOPK_EXCLUDES_FIXED) */
    int32_t          si_fixed_budget;
    /* 1 = the SI window starts on a 64-row boundary (LSA_TOPK_WINDOW_ALIGNED) */
    int32_t          si_window_aligned;
    /* Optional cudaEvent_t (NULL: none) recorded by the caller once every layer's attention query
     * `q` is written -- typically on another stream, at the end of the MLA prolog (norm,
     * projections, RoPE).  The indexer and the top-k do not wait for it; the attention layers do.
     * So the index selection runs while the prolog still computes the attention queries
     * ([release] "推理 · 模型层面优化", Attention paragraph: the indexer computed in parallel with
     * the MLA prolog).  The indexer's own inputs (q_idx, w) must be ready on `stream`. */
    void*            attn_q_ready;
} lsa_decode_params;

/* Runs indexer (flat, or HI: block scores -> recall -> fine scores), top-k + union, then
 * attention for every layer (after attn_q_ready, when given), with no host synchronisation.  Everything is ordered after the
 * work already queued on `stream`, and work queued on `stream` afterwards runs after all of
 * it.  With two or more layers the layers alternate between `stream` and a second stream of
 * the calling thread (created on first use, with two events; forked from `stream` after
 * top-k and joined back before returning), so that two layers' attention kernels can share
 * the GPU; captured into a CUDA graph this becomes two branches.  Scores, index lists and the
 * split partials of each branch live in `ws` (lsa_decode_workspace_size bytes). */
lsa_status lsa_decode_fused(const lsa_decode_params* p, void* ws, size_t ws_bytes,
                            int32_t* dev_status, void* stream);

size_t lsa_decode_workspace_size(const lsa_decode_params* p);
/* Entries per token of the step's index list: k + n_sink + window, plus 63 with
 * si_window_aligned and window > 0 (the minimum idx_ld). */
int    lsa_decode_index_capacity(const lsa_decode_params* p);

/* ---------------------------------------------------------------- pipelined host I/O
 * A decode driver for callers whose queries and outputs live in host memory (pinned, so that
 * the copies are asynchronous).  Each lsa_pipeline_step copies one step's inputs from host to
 * device buffers (`h2d`, one cudaMemcpyAsync each, in order), runs lsa_decode_fused for each of
 * the step's `n_params` parameter sets (with workspace ws[i] of ws_bytes[i] bytes), then copies
 * the outputs back (`d2h`): the copy-in on a stream of the pipeline, the decode on the stream
 * given at creation, the copy-out on a second stream of the pipeline, ordered by events, so that
 * one step's copies overlap the decode of the steps next to it.  The caller keeps `n_slots`
 * sets of device input / output buffers and passes slot = step index mod n_slots: a slot's
 * copy-in waits until the decode that last read that slot's inputs has finished, and its
 * decode waits until the copy-out that last read that slot's outputs has finished.
 * Workspaces, dev_status and the index outputs may be shared between slots (the decodes run in
 * order on one stream).  Host buffers must stay valid and unchanged until the copies that
 * read or write them have run.  A slot's decode is captured into a CUDA graph on its first
 * step (on a stream of the pipeline) and replayed while the slot's parameter sets, workspaces
 * and dev_status are the same as at the capture (compared byte for byte, layer arrays
 * included); otherwise it is captured again.  When the decode stream is itself being
 * captured, or a capture fails, the decode is launched directly. 
 *
 * lsa_pipeline_create: n_slots in [1, 8]; creates two streams and 3 n_slots + 1 events on the
 *   current device (a third stream and the slot graphs on first use; no device memory of
 *   its own).  *out receives the pipeline.
 * lsa_pipeline_step: LSA_ERR_INVALID_ARG for a bad slot, count or NULL array; any error of
 *   lsa_decode_fused; LSA_ERR_CUDA when a copy or event call fails.  Nothing is synchronised.
 * lsa_pipeline_join: makes the decode stream wait for every copy issued so far, so that work
 *   queued on it afterwards (an event, a synchronisation) follows all of the host outputs.
 * lsa_pipeline_destroy: waits for the pipeline's streams, then releases them, its events and
 *   its graphs. */
typedef struct {
    void*       dst;
    const void* src;
    size_t      bytes;
} lsa_copy;

typedef struct lsa_pipeline lsa_pipeline;

lsa_status lsa_pipeline_create(lsa_pipeline** out, int n_slots, void* stream);
lsa_status lsa_pipeline_step(lsa_pipeline* pl, int slot, const lsa_decode_params* const* params, int n_params,
                             void* const* ws, const size_t* ws_bytes, const lsa_copy* h2d, int n_h2d,
                             const lsa_copy* d2h, int n_d2h, int32_t* dev_status);
lsa_status lsa_pipeline_join(lsa_pipeline* pl);
lsa_status lsa_pipeline_destroy(lsa_pipeline* pl);

/* ---------------------------------------------------------------- helpers
 * Synchronises `stream`, then returns the status stored at dev_status (LSA_OK when 0),
 * or LSA_ERR_CUDA if the copy fails. */
lsa_status  lsa_read_device_status(const int32_t* dev_status, void* stream);
const char* lsa_status_string(lsa_status s);
int         lsa_version(void);

/* Diagnostic: the wall-time limit, in nanoseconds, of the pipeline waits of the tensor-core
 * indexer (lsa_index_score, lsa_index_score_q8, the indexer of lsa_decode_fused) and of the
 * tensor-core block scores, for launches issued after the call; 0 restores the default (2 s).  A
 * CTA whose wait runs out stops its pipeline, waits (with the 2 s bound) for its copies and MMAs
 * in flight, frees its tensor memory and stores LSA_ERR_TIMEOUT in dev_status; its outputs are
 * then incomplete.  A limit shorter than the kernel's own waits makes it give up on purpose: the
 * way to check that path.  Process-wide; returns the previous setting. */
uint64_t    lsa_set_wait_limit_ns(uint64_t ns);

#ifdef __cplusplus
}
#endif
#endif /* LSA_H_ */
