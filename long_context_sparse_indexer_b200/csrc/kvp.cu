// KVP: one sequence's context sharded over several ranks (GPUs), decode merged across them.
//
// Explainer page ("如何在 5 万张国产芯片训练出 1.6T 万亿参数模型？"), section "③ KVP 解码切分示意":
// the KV cache of a long sequence is split over devices, each computes a partial result over
// its shard, and the partial results are merged.  Release post, section "推理" (decode nodes):
// KVP splits the KV cache.  Here a shard is a contiguous range of rows [start, start + len) of
// every sequence (its indexer keys and its KV rows).  The selection stays exactly the
// single-device one: every key of the global top-k is in the top-k of its own shard, so each
// rank's top-k candidates (score, position), gathered over the ranks in shard order, contain the
// global top-k, which one more selection with the same order (score desc, position asc) finds.
// Attention is then computed per shard over the selected rows it holds, and the per-shard
// partial results are merged by log-sum-exp in shard order.  The exchanges between the steps
// (candidates, partial results) are collectives of the caller (NCCL all-gathers); every
// computation is one of the calls below or of the single-device path.
#include "kernels.cuh"

namespace lsa {

namespace {

constexpr int kKvpThreads = 256;

// local_seq_len[b] = shard_len[b]; local_q_pos[t] = clamp(q_pos[t] - shard_start[b], 0, len - 1).
__global__ void kvp_shard_batch_kernel(int B, int T, int L_alloc_local, const int32_t* seq_len, const int32_t* q_seq,
                                       const int32_t* q_pos, const int32_t* shard_start, const int32_t* shard_len,
                                       int32_t* local_seq_len, int32_t* local_q_pos, int32_t* status) {
    const int i = blockIdx.x * kKvpThreads + threadIdx.x;
    if (i < B) {
        const int st = shard_start[i], ln = shard_len[i];
        const bool ok = st >= 0 && ln >= 1 && ln <= L_alloc_local && st + ln <= seq_len[i];
        if (!ok) report(status, LSA_ERR_DEVICE_DATA);
        local_seq_len[i] = ok ? ln : 1;
    }
    if (i < T) {
        const int b = q_seq[i];
        int p = 0;
        if (b >= 0 && b < B) {
            const int st = shard_start[b], ln = max(shard_len[b], 1);
            p = min(max(q_pos[i] - st, 0), ln - 1);
        } else {
            report(status, LSA_ERR_DEVICE_DATA);
        }
        local_q_pos[i] = p;
    }
}

// Token t (one CTA): the top-k local columns cand_pos[t][0..count) (ascending) become global
// positions with their scores; slots past the count, and every slot of a token whose position
// precedes the shard (it sees none of its keys), become (-1, -inf).
__global__ void kvp_candidates_kernel(int k, const int32_t* q_seq, const int32_t* q_pos, const int32_t* shard_start,
                                      int B, const float* scores, int64_t ld, const int32_t* count,
                                      int32_t* cand_pos, float* cand_score) {
    const int t = blockIdx.x;
    const int b = q_seq[t];
    const bool bok = b >= 0 && b < B;
    const int st = bok ? shard_start[b] : 0;
    const int n = (bok && q_pos[t] >= st) ? count[t] : 0;
    for (int i = threadIdx.x; i < k; i += kKvpThreads) {
        const size_t o = (size_t)t * k + i;
        if (i < n) {
            const int c = cand_pos[o];
            cand_score[o] = scores[(size_t)t * ld + c];
            cand_pos[o] = c + st;
        } else {
            cand_score[o] = kNegInf;
            cand_pos[o] = -1;
        }
    }
}

// Candidates of n_parts parts, [part][T][k_part], to one row per token, [T][part * k_part].
__global__ void kvp_gather_kernel(int T, int n_parts, int k_part, const int32_t* cand_pos, const float* cand_score,
                                  int32_t* pos_out, float* score_out) {
    const int t = blockIdx.y;
    const int i = blockIdx.x * kKvpThreads + threadIdx.x;          // part * k_part + j
    if (i >= n_parts * k_part) return;
    const int part = i / k_part, j = i % k_part;
    const size_t src = ((size_t)part * T + t) * k_part + j;
    pos_out[(size_t)t * n_parts * k_part + i] = cand_pos[src];
    score_out[(size_t)t * n_parts * k_part + i] = cand_score[src];
}

// Token t (one CTA): the entries of its ascending global list inside [start, start + len) --
// one contiguous run -- as local rows.
__global__ void kvp_local_index_kernel(int B, const int32_t* q_seq, const int32_t* shard_start,
                                       const int32_t* shard_len, const int32_t* idx, int64_t ld_idx,
                                       const int32_t* count, int32_t* local_idx, int64_t ld_local,
                                       int32_t* local_count, int32_t* status) {
    const int t = blockIdx.x;
    const int b = q_seq[t];
    int st = 0, en = 0;
    if (b >= 0 && b < B) { st = shard_start[b]; en = st + shard_len[b]; }
    const int n = min(max(count[t], 0), (int)ld_idx);
    const int32_t* row = idx + (size_t)t * ld_idx;
    __shared__ int s_below, s_inside;
    if (threadIdx.x == 0) { s_below = 0; s_inside = 0; }
    __syncthreads();
    int below = 0, inside = 0;
    for (int i = threadIdx.x; i < n; i += kKvpThreads) {
        const int p = row[i];
        below += p < st;
        inside += p >= st && p < en;
    }
    atomicAdd(&s_below, below);                                    // integer counts: order-free
    atomicAdd(&s_inside, inside);
    __syncthreads();
    const int lo = s_below, m = s_inside;
    if (m > ld_local) {                                            // cannot happen with ld_local >= ld_idx
        if (threadIdx.x == 0) { report(status, LSA_ERR_DEVICE_DATA); local_count[t] = 0; }
        return;
    }
    int32_t* out = local_idx + (size_t)t * ld_local;
    for (int j = threadIdx.x; j < ld_local; j += kKvpThreads) out[j] = j < m ? row[lo + j] - st : -1;
    if (threadIdx.x == 0) local_count[t] = m;
}

}  // namespace

cudaError_t launch_kvp_shard_batch(int B, int T, int L_alloc_local, const int32_t* seq_len, const int32_t* q_seq,
                                   const int32_t* q_pos, const int32_t* shard_start, const int32_t* shard_len,
                                   int32_t* local_seq_len, int32_t* local_q_pos, int32_t* status, cudaStream_t st) {
    const int n = B > T ? B : T;
    kvp_shard_batch_kernel<<<(n + kKvpThreads - 1) / kKvpThreads, kKvpThreads, 0, st>>>(
        B, T, L_alloc_local, seq_len, q_seq, q_pos, shard_start, shard_len, local_seq_len, local_q_pos, status);
    return cudaGetLastError();
}

cudaError_t launch_kvp_candidates(int T, int k, const int32_t* q_seq, const int32_t* q_pos,
                                  const int32_t* shard_start, int B, const float* scores, int64_t ld,
                                  const int32_t* count, int32_t* cand_pos, float* cand_score, cudaStream_t st) {
    if (T <= 0 || k <= 0) return cudaSuccess;
    kvp_candidates_kernel<<<T, kKvpThreads, 0, st>>>(k, q_seq, q_pos, shard_start, B, scores, ld, count, cand_pos,
                                                     cand_score);
    return cudaGetLastError();
}

cudaError_t launch_kvp_gather(int T, int n_parts, int k_part, const int32_t* cand_pos, const float* cand_score,
                              int32_t* pos_out, float* score_out, cudaStream_t st) {
    if (T <= 0 || n_parts * k_part <= 0) return cudaSuccess;
    dim3 grid((n_parts * k_part + kKvpThreads - 1) / kKvpThreads, T);
    kvp_gather_kernel<<<grid, kKvpThreads, 0, st>>>(T, n_parts, k_part, cand_pos, cand_score, pos_out, score_out);
    return cudaGetLastError();
}

cudaError_t launch_kvp_local_index(int T, int B, const int32_t* q_seq, const int32_t* shard_start,
                                   const int32_t* shard_len, const int32_t* idx, int64_t ld_idx,
                                   const int32_t* count, int32_t* local_idx, int64_t ld_local, int32_t* local_count,
                                   int32_t* status, cudaStream_t st) {
    if (T <= 0) return cudaSuccess;
    kvp_local_index_kernel<<<T, kKvpThreads, 0, st>>>(B, q_seq, shard_start, shard_len, idx, ld_idx, count,
                                                      local_idx, ld_local, local_count, status);
    return cudaGetLastError();
}

}  // namespace lsa
