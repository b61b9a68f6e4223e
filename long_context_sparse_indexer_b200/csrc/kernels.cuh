// Internal kernel interfaces of the LSA library (argument blocks and host launchers).
#pragma once

#include "common.cuh"

namespace lsa {

struct IndexArgs {
    const int32_t* seq_len;
    const int32_t* q_seq;
    const int32_t* q_pos;
    int B, T, q_group, L_alloc;
    const uint16_t* q;       // bf16 bits [T][H_I][D_I]
    const float* w;          // [T][H_I]
    const uint8_t* kdata;    // cache base (bytes)
    const float* kscale;     // per-token scale or NULL
    int64_t seq_stride_b, tok_stride_b, scale_seq_stride;
    const int32_t* cand;     // [T][n_cand] or NULL
    int n_cand, block_size;
    float* scores;
    int64_t ld;
    int n_cols;              // columns to write
    int group;               // tokens per CTA (<= 4)
    int q_fp8;               // 1: FP8-query mode (queries rounded once to e4m3, tensor-core path only)
    uint64_t wait_ns;        // limit of the tensor-core kernel's pipeline waits (drains keep 2 s)
    int32_t* status;
};

struct BlockKeyArgs {
    const int32_t* seq_len;
    int B, L_alloc;
    const uint8_t* kdata;
    const float* kscale;
    int64_t seq_stride_b, tok_stride_b, scale_seq_stride;
    int d_I, block_size;
    bool fp8;
    uint16_t* kbar;          // [B][*][2][d_I] bf16 bits: (hi, lo) of each block key
    int64_t kbar_seq_stride; // uint16 elements between sequences
    int32_t* status;
};

struct BlockScoreArgs {
    const int32_t* seq_len;
    const int32_t* q_seq;
    const int32_t* q_pos;
    int B, T, L_alloc;
    const uint16_t* q;   // bf16 [T][H_I][d_I]
    const float* w;      // [T][H_I]
    const uint16_t* kbar;    // [B][*][2][d_I] bf16 bits (hi, lo)
    int64_t kbar_seq_stride; // uint16 elements between sequences
    int L_blocks;            // block rows allocated per sequence (ceil(L_alloc / block_size))
    int q_group;
    int d_I, block_size;
    float* scores;
    int64_t ld;
    int n_cols;
    uint64_t wait_ns;        // limit of the tensor-core kernel's pipeline waits (drains keep 2 s)
    int32_t* status;
};

// Indexer-form scores of BF16 rows on the tensor cores (row_score_tc.cu): HI block keys stored
// as [hi | lo] pairs (halves = 2, row_span = block size) or BF16 indexer keys (halves = 1,
// row_span = 1).  Row j of token t is visible when j * row_span <= q_pos[t].
struct RowScoreArgs {
    const int32_t* seq_len;
    const int32_t* q_seq;
    const int32_t* q_pos;
    int B, T, L_alloc, q_group;
    const uint16_t* q;       // bf16 [T][H_I][d_I]
    const float* w;          // [T][H_I]
    int H_I, d_I;
    int halves;              // row = halves x d_I BF16 values
    int row_span;            // positions per row
    float* scores;
    int64_t ld;
    int n_cols;
    uint64_t wait_ns;
    int32_t* status;
};

struct TopkArgs {
    const int32_t* seq_len;
    const int32_t* q_seq;
    const int32_t* q_pos;
    int B, T, L_alloc;
    const float* scores;
    int64_t ld;
    int n_cols;
    const int32_t* cand;
    int n_cand, block_size;
    int k, n_sink, window;
    bool raw;
    bool fixed_budget;       // top-k drawn outside the sinks and the window
    int window_align;        // 0, or the block the SI window's start is rounded down to (64)
    int32_t* idx;
    int64_t ld_idx;
    int32_t* count;
    int32_t* status;
};

struct AttnArgs {
    const int32_t* seq_len;
    const int32_t* q_seq;
    int B, T, L_alloc;
    const uint16_t* q;          // [T][H][DQK] bf16
    int H;
    const uint8_t* kv;          // bytes
    const float* kv_scale;
    int64_t kv_seq_b, kv_tok_b, kv_scale_seq;
    const uint8_t* v;           // separate V cache or NULL
    const float* v_scale;
    int64_t v_seq_b, v_tok_b, v_scale_seq;
    const int32_t* idx;
    int64_t ld_idx;
    const int32_t* count;
    float sm_scale_log2;        // sm_scale * log2(e)
    int n_split;
    uint16_t* o;                // [T][H][DV] bf16
    float* lse;                 // [T][H] or NULL
    float* part_o;              // [T][n_split][H][DV] (n_split > 1, or f32_out)
    float* part_lse;            // [T][n_split][H]
    int f32_out;                // the result in FP32: o32 / lse32 instead of o / lse
    float* o32;                 // [T][H][DV] (f32_out)
    float* lse32;               // [T][H] (f32_out)
    int32_t* status;
};

cudaError_t launch_index_score(IndexArgs a, int H_I, int D_I, bool fp8, cudaStream_t st);
bool index_score_tc_supported(const IndexArgs& a, int H_I, int D_I, bool fp8);
cudaError_t launch_index_score_tc(IndexArgs a, int H_I, cudaStream_t st);
cudaError_t launch_block_keys(const BlockKeyArgs& a, cudaStream_t st);
cudaError_t launch_block_score(const BlockScoreArgs& a, int H_I, cudaStream_t st);
int row_score_group(int q_group, int H_I);
bool row_score_tc_supported(const RowScoreArgs& a, int row_elems, int64_t row_stride_b, int64_t seq_stride_b,
                            const void* rows);
cudaError_t launch_row_score_tc(const RowScoreArgs& a, int n_rows, int64_t row_stride_b, int64_t seq_stride_b,
                                const void* rows, cudaStream_t st);
cudaError_t launch_topk(const TopkArgs& a, cudaStream_t st);
cudaError_t launch_sparse_attn(const AttnArgs& a, int DQK, int DV, bool kv_fp8, bool sep_v, cudaStream_t st);
bool sparse_attn_tc_supported(const AttnArgs& a, int DQK, int DV, bool sep_v);
cudaError_t launch_sparse_attn_tc(const AttnArgs& a, bool kv_fp8, cudaStream_t st);
// Log-sum-exp merge of n_part partial attentions: partial p of (token t, head h) at row
// p * part_stride + t * tok_stride + h of part_o ([row][DV]) and part_lse; result BF16 (o) or
// FP32 (o32), lse optional.
cudaError_t launch_merge_partials(const float* part_o, const float* part_lse, int n_part, int64_t part_stride,
                                  int64_t tok_stride, int T, int H, int DV, uint16_t* o, float* o32, float* lse,
                                  cudaStream_t st);

// KVP helpers (kvp.cu).
cudaError_t launch_kvp_shard_batch(int B, int T, int L_alloc_local, const int32_t* seq_len, const int32_t* q_seq,
                                   const int32_t* q_pos, const int32_t* shard_start, const int32_t* shard_len,
                                   int32_t* local_seq_len, int32_t* local_q_pos, int32_t* status, cudaStream_t st);
cudaError_t launch_kvp_candidates(int T, int k, const int32_t* q_seq, const int32_t* q_pos,
                                  const int32_t* shard_start, int B, const float* scores, int64_t ld,
                                  const int32_t* count, int32_t* cand_pos, float* cand_score, cudaStream_t st);
cudaError_t launch_kvp_gather(int T, int n_parts, int k_part, const int32_t* cand_pos, const float* cand_score,
                              int32_t* pos_out, float* score_out, cudaStream_t st);
cudaError_t launch_kvp_local_index(int T, int B, const int32_t* q_seq, const int32_t* shard_start,
                                   const int32_t* shard_len, const int32_t* idx, int64_t ld_idx,
                                   const int32_t* count, int32_t* local_idx, int64_t ld_local, int32_t* local_count,
                                   int32_t* status, cudaStream_t st);

// Wait limit the tensor-core indexer and block-score kernels are launched with (api.cu).
uint64_t wait_limit_ns();

// Host-side checks of lsa_sparse_attn's arguments other than its workspace (api.cu).
lsa_status attn_validate(const lsa_batch* batch, const void* q, int H, int Dqk, const lsa_cache* kv,
                         const lsa_cache* v, int Dv, const int32_t* idx, int64_t ld_idx, const int32_t* count,
                         float sm_scale, int n_split, const void* o);

}  // namespace lsa
