// C ABI of the LSA library: host-side validation, workspace carving and kernel dispatch.
// No device allocation, no synchronisation (except lsa_read_device_status), no exceptions.
#include <atomic>
#include <cmath>
#include <cstring>

#include "kernels.cuh"

using namespace lsa;

namespace {

constexpr size_t kAlign = 256;
constexpr int kMaxTokens = 65535;
constexpr int kWindowAlign = 64;             // rows of the block the aligned SI window starts on
inline size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
inline bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }
inline int elem_bytes(int dtype) { return dtype == LSA_FP8_E4M3 ? 1 : (dtype == LSA_BF16 ? 2 : 4); }

lsa_status check_batch(const lsa_batch* b) {
    if (!b || b->B < 1 || b->T < 0 || b->q_group < 1 || b->L_alloc < 1) return LSA_ERR_INVALID_ARG;
    if (b->T % b->q_group) return LSA_ERR_INVALID_ARG;
    // Several kernels put the query token in a grid dimension limited to 65535 blocks.
    if (b->T > kMaxTokens || b->B > kMaxTokens) return LSA_ERR_UNSUPPORTED;
    if (b->T > 0 && (!b->seq_len || !b->q_seq || !b->q_pos)) return LSA_ERR_INVALID_ARG;
    return LSA_OK;
}

// Checks a cache whose rows are read with 16-byte vector loads.
lsa_status check_cache(const lsa_cache* c, int dim_expected) {
    if (!c || !c->data) return LSA_ERR_INVALID_ARG;
    if (c->dtype != LSA_BF16 && c->dtype != LSA_FP8_E4M3) return LSA_ERR_UNSUPPORTED;
    if (c->dtype == LSA_FP8_E4M3 && !c->scale) return LSA_ERR_INVALID_ARG;
    if (dim_expected > 0 && c->dim != dim_expected) return LSA_ERR_INVALID_ARG;
    if (c->dim < 1 || c->tok_stride < c->dim || c->seq_stride < 0) return LSA_ERR_INVALID_ARG;
    const int eb = elem_bytes(c->dtype);
    if (!aligned16(c->data) || (c->tok_stride * eb) % 16 || (c->seq_stride * eb) % 16) return LSA_ERR_INVALID_ARG;
    if ((c->dim * eb) % 16) return LSA_ERR_UNSUPPORTED;
    return LSA_OK;
}

inline lsa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? LSA_OK : LSA_ERR_CUDA; }

bool supported_hi(int H_I) { return H_I == 8 || H_I == 16 || H_I == 32 || H_I == 64 || H_I == 128; }

IndexArgs make_index_args(const lsa_batch* batch, const void* q_idx, const float* w, const lsa_cache* k,
                          const int32_t* cand, int n_cand, int block_size, float* scores, int64_t ld,
                          int n_cols, int32_t* st) {
    IndexArgs a{};
    a.seq_len = batch->seq_len; a.q_seq = batch->q_seq; a.q_pos = batch->q_pos;
    a.B = batch->B; a.T = batch->T; a.q_group = batch->q_group; a.L_alloc = batch->L_alloc;
    a.q = static_cast<const uint16_t*>(q_idx); a.w = w;
    const int eb = elem_bytes(k->dtype);
    a.kdata = static_cast<const uint8_t*>(k->data);
    a.kscale = k->dtype == LSA_FP8_E4M3 ? k->scale : nullptr;
    a.seq_stride_b = k->seq_stride * eb; a.tok_stride_b = k->tok_stride * eb; a.scale_seq_stride = k->scale_seq_stride;
    a.cand = cand; a.n_cand = n_cand; a.block_size = block_size;
    a.scores = scores; a.ld = ld; a.n_cols = cand ? n_cand * block_size : n_cols;
    a.status = st;
    return a;
}

lsa_status index_score_impl(const lsa_batch* batch, const void* q_idx, const float* w, int H_I,
                            const lsa_cache* k_idx, const int32_t* cand, int n_cand, int block_size,
                            float* scores, int64_t ld, int n_cols, int32_t* st, cudaStream_t stream,
                            bool q_fp8 = false) {
    lsa_status s = check_batch(batch);
    if (s != LSA_OK) return s;
    if ((s = check_cache(k_idx, 0)) != LSA_OK) return s;
    if (!supported_hi(H_I) || (k_idx->dim != 64 && k_idx->dim != 128)) return LSA_ERR_UNSUPPORTED;
    if (batch->T == 0) return LSA_OK;
    if (!q_idx || !w || !scores) return LSA_ERR_INVALID_ARG;
    if (cand) {
        if (n_cand < 1 || block_size < 1 || (int64_t)n_cand * block_size > ld) return LSA_ERR_INVALID_ARG;
        if ((int64_t)n_cand * block_size > 0x7fffffff) return LSA_ERR_INVALID_ARG;
    } else {
        if (n_cols < 0 || n_cols > ld || n_cols > batch->L_alloc) return LSA_ERR_INVALID_ARG;
    }
    IndexArgs a = make_index_args(batch, q_idx, w, k_idx, cand, n_cand, block_size, scores, ld, n_cols, st);
    a.q_fp8 = q_fp8 ? 1 : 0;
    // The FP8-query mode exists on the tensor-core path only.
    if (q_fp8 && !index_score_tc_supported(a, H_I, k_idx->dim, k_idx->dtype == LSA_FP8_E4M3)) return LSA_ERR_UNSUPPORTED;
    return cuda_status(launch_index_score(a, H_I, k_idx->dim, k_idx->dtype == LSA_FP8_E4M3, stream));
}

lsa_status topk_impl(const lsa_batch* batch, const float* scores, int64_t ld, int n_cols,
                     const int32_t* cand, int n_cand, int block_size, int k, int n_sink, int window,
                     uint32_t flags, int32_t* idx, int64_t ld_idx, int32_t* count, int32_t* st,
                     cudaStream_t stream) {
    lsa_status s = check_batch(batch);
    if (s != LSA_OK) return s;
    const bool raw = flags & LSA_TOPK_RAW;
    const bool fixed = flags & LSA_TOPK_EXCLUDES_FIXED;
    if (k < 0 || n_sink < 0 || window < 0 || n_cols < 0 || n_cols > ld) return LSA_ERR_INVALID_ARG;
    if (raw && (n_sink || window || cand)) return LSA_ERR_INVALID_ARG;
    if ((int64_t)k + n_sink + window > ld_idx) return LSA_ERR_INVALID_ARG;
    if (cand && (n_cand < 1 || block_size < 1 || n_cols > (int64_t)n_cand * block_size)) return LSA_ERR_INVALID_ARG;
    const bool aligned = flags & LSA_TOPK_WINDOW_ALIGNED;
    if (flags & ~(LSA_TOPK_RAW | LSA_TOPK_EXCLUDES_FIXED | LSA_TOPK_WINDOW_ALIGNED)) return LSA_ERR_UNSUPPORTED;
    if (raw && (fixed || aligned)) return LSA_ERR_INVALID_ARG;
    // The aligned window holds up to 63 positions more than `window`.
    if (aligned && window > 0 && (int64_t)k + n_sink + window + kWindowAlign - 1 > ld_idx) return LSA_ERR_INVALID_ARG;
    if (batch->T == 0) return LSA_OK;
    if (!scores || !idx || !count) return LSA_ERR_INVALID_ARG;
    TopkArgs a{};
    a.seq_len = batch->seq_len; a.q_seq = batch->q_seq; a.q_pos = batch->q_pos;
    a.B = batch->B; a.T = batch->T; a.L_alloc = batch->L_alloc;
    a.scores = scores; a.ld = ld; a.n_cols = n_cols;
    a.cand = cand; a.n_cand = n_cand; a.block_size = block_size;
    a.k = k; a.n_sink = n_sink; a.window = window; a.raw = raw; a.fixed_budget = fixed;
    a.window_align = aligned ? kWindowAlign : 0;
    a.idx = idx; a.ld_idx = ld_idx; a.count = count; a.status = st;
    return cuda_status(launch_topk(a, stream));
}

size_t attn_ws(int T, int H, int Dv, int n_split) {
    if (n_split <= 1) return 0;
    return align_up((size_t)T * n_split * H * Dv * 4) + align_up((size_t)T * n_split * H * 4);
}

// Limit of the pipeline waits of the tensor-core indexer and block-score kernels (0: the 2 s
// default), set by lsa_set_wait_limit_ns.
std::atomic<uint64_t> g_wait_limit_ns{0};

}  // namespace

uint64_t lsa::wait_limit_ns() {
    const uint64_t v = g_wait_limit_ns.load(std::memory_order_relaxed);
    return v ? v : 2000000000ull;
}

// Argument checks of lsa_sparse_attn that do not involve the workspace (shared with the
// no-allocation entry point, which checks its own scratch size after these).
lsa_status lsa::attn_validate(const lsa_batch* batch, const void* q, int H, int Dqk, const lsa_cache* kv,
                              const lsa_cache* v, int Dv, const int32_t* idx, int64_t ld_idx, const int32_t* count,
                              float sm_scale, int n_split, const void* o) {
    lsa_status s = check_batch(batch);
    if (s != LSA_OK) return s;
    const bool sep_v = v && v->data;
    if ((s = check_cache(kv, Dqk)) != LSA_OK) return s;
    if (sep_v && (s = check_cache(v, Dv)) != LSA_OK) return s;
    const bool mla = Dqk == 576 && Dv == 512 && !sep_v && H > 0 && H % 32 == 0;
    const bool sep = Dqk == 128 && Dv == 128 && sep_v && H > 0 && H % 16 == 0 && kv->dtype == LSA_BF16 &&
                     v->dtype == LSA_BF16;
    if (!mla && !sep) return LSA_ERR_UNSUPPORTED;
    if (n_split < 1 || n_split > 64 || ld_idx < 1) return LSA_ERR_INVALID_ARG;
    if (!(sm_scale > 0.f) || !std::isfinite(sm_scale)) return LSA_ERR_INVALID_ARG;
    if (batch->T == 0) return LSA_OK;
    if (!q || !idx || !count || !o) return LSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(o)) return LSA_ERR_INVALID_ARG;
    return LSA_OK;
}

namespace {

// o32 / lse32 (FP32 result, both given) replace o / lse when not NULL.
lsa_status attn_impl(const lsa_batch* batch, const void* q, int H, int Dqk, const lsa_cache* kv,
                     const lsa_cache* v, int Dv, const int32_t* idx, int64_t ld_idx, const int32_t* count,
                     float sm_scale, int n_split, void* o, float* lse, void* ws, size_t ws_bytes,
                     int32_t* st, cudaStream_t stream, float* o32 = nullptr, float* lse32 = nullptr) {
    lsa_status s = attn_validate(batch, q, H, Dqk, kv, v, Dv, idx, ld_idx, count, sm_scale, n_split,
                                 o32 ? static_cast<const void*>(o32) : o);
    if (s != LSA_OK || batch->T == 0) return s;
    if (o32 && (!lse32 || ((uintptr_t)lse32 & 3))) return LSA_ERR_INVALID_ARG;
    const bool sep_v = v && v->data;
    const size_t need = attn_ws(batch->T, H, Dv, n_split);
    if (need && (!ws || ws_bytes < need || ((uintptr_t)ws % kAlign))) return LSA_ERR_WORKSPACE;
    AttnArgs a{};
    a.seq_len = batch->seq_len; a.q_seq = batch->q_seq;
    a.B = batch->B; a.T = batch->T; a.L_alloc = batch->L_alloc;
    a.q = static_cast<const uint16_t*>(q); a.H = H;
    const int eb = elem_bytes(kv->dtype);
    a.kv = static_cast<const uint8_t*>(kv->data);
    a.kv_scale = kv->dtype == LSA_FP8_E4M3 ? kv->scale : nullptr;
    a.kv_seq_b = kv->seq_stride * eb; a.kv_tok_b = kv->tok_stride * eb; a.kv_scale_seq = kv->scale_seq_stride;
    if (sep_v) {
        const int vb = elem_bytes(v->dtype);
        a.v = static_cast<const uint8_t*>(v->data);
        a.v_scale = v->dtype == LSA_FP8_E4M3 ? v->scale : nullptr;
        a.v_seq_b = v->seq_stride * vb; a.v_tok_b = v->tok_stride * vb; a.v_scale_seq = v->scale_seq_stride;
    }
    a.idx = idx; a.ld_idx = ld_idx; a.count = count;
    a.sm_scale_log2 = sm_scale * 1.4426950408889634f;
    a.n_split = n_split;
    a.o = static_cast<uint16_t*>(o); a.lse = lse;
    if (n_split > 1) {
        a.part_o = static_cast<float*>(ws);
        a.part_lse = reinterpret_cast<float*>(static_cast<char*>(ws) + align_up((size_t)batch->T * n_split * H * Dv * 4));
    }
    if (o32) {                    // FP32 result: one split writes it directly, more splits merge into it
        a.f32_out = 1;
        a.o32 = o32;
        a.lse32 = lse32;
        if (n_split == 1) { a.part_o = o32; a.part_lse = lse32; }
    }
    a.status = st;
    return cuda_status(launch_sparse_attn(a, Dqk, Dv, kv->dtype == LSA_FP8_E4M3, sep_v, stream));
}

// Workspace plan of the fused path.
struct FusedPlan {
    size_t scores = 0, bscores = 0, cand = 0, ccount = 0, idx = 0, count = 0, attn = 0, attn_one = 0, total = 0;
    int n_cols = 0, nblk = 0, cap = 0;
    int64_t ld = 0, bld = 0;
};

bool plan_fused(const lsa_decode_params* p, FusedPlan& f) {
    const int T = p->batch.T;
    f.cap = p->k + p->n_sink + p->window + (p->si_window_aligned && p->window > 0 ? kWindowAlign - 1 : 0);
    size_t off = 0;
    if (p->hi) {
        f.nblk = (p->batch.L_alloc + p->block_size - 1) / p->block_size;
        f.bld = (f.nblk + 3) / 4 * 4;
        f.bscores = off; off += align_up((size_t)T * f.bld * 4);
        f.cand = off; off += align_up((size_t)T * p->n_recall * 4);
        f.ccount = off; off += align_up((size_t)T * 4);
        f.n_cols = p->n_recall * p->block_size;
    } else {
        f.n_cols = p->batch.L_alloc;
    }
    f.ld = ((int64_t)f.n_cols + 3) / 4 * 4;
    f.scores = off; off += align_up((size_t)T * f.ld * 4);
    f.idx = off; off += align_up((size_t)T * f.cap * 4);
    f.count = off; off += align_up((size_t)T * 4);
    // One split-partial area per attention branch (layers alternate between two branches).
    f.attn_one = attn_ws(T, p->H, p->Dv, p->n_split);
    f.attn = off; off += (size_t)(p->n_layers > 1 ? 2 : 1) * f.attn_one;
    f.total = off;
    return true;
}

// A second stream of the calling thread on the current device, created on first use, with
// the two events that fork it from the caller's stream and join it back.  Under stream capture
// the fork and the join become dependencies of the captured graph.
struct AuxStream {
    cudaStream_t s = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};

AuxStream* aux_stream() {
    static thread_local AuxStream aux[16];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 16) return nullptr;
    AuxStream& a = aux[dev];
    if (!a.s) {
        cudaStream_t s = nullptr;
        cudaEvent_t f = nullptr, j = nullptr;
        if (cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
        if (cudaEventCreateWithFlags(&f, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&j, cudaEventDisableTiming) != cudaSuccess) {
            if (f) cudaEventDestroy(f);
            cudaStreamDestroy(s);
            return nullptr;
        }
        a.s = s; a.fork = f; a.join = j;
    }
    return &a;
}

}  // namespace

extern "C" {

lsa_status lsa_index_score(const lsa_batch* batch, const void* q_idx, const float* w, int H_I,
                           const lsa_cache* k_idx, const int32_t* cand_blocks, int n_cand, int block_size,
                           float* scores, int64_t ld_scores, int n_cols, int32_t* dev_status, void* stream) {
    return index_score_impl(batch, q_idx, w, H_I, k_idx, cand_blocks, n_cand, block_size, scores, ld_scores,
                            n_cols, dev_status, static_cast<cudaStream_t>(stream));
}

lsa_status lsa_index_score_q8(const lsa_batch* batch, const void* q_idx, const float* w, int H_I,
                              const lsa_cache* k_idx, const int32_t* cand_blocks, int n_cand, int block_size,
                              float* scores, int64_t ld_scores, int n_cols, int32_t* dev_status, void* stream) {
    return index_score_impl(batch, q_idx, w, H_I, k_idx, cand_blocks, n_cand, block_size, scores, ld_scores,
                            n_cols, dev_status, static_cast<cudaStream_t>(stream), true);
}

lsa_status lsa_block_keys(const lsa_batch* batch, const lsa_cache* k_idx, int block_size, void* kbar,
                          int64_t kbar_seq_stride, int32_t* dev_status, void* stream) {
    lsa_status s = check_batch(batch);
    if (s != LSA_OK) return s;
    if ((s = check_cache(k_idx, 0)) != LSA_OK) return s;
    if (!kbar || block_size < 1 || block_size > 1024 || k_idx->dim > 1024) return LSA_ERR_INVALID_ARG;
    const int64_t nblk = (batch->L_alloc + block_size - 1) / block_size;
    if (kbar_seq_stride < nblk * 2 * k_idx->dim || kbar_seq_stride % 8 || ((uintptr_t)kbar & 15)) return LSA_ERR_INVALID_ARG;
    if (!batch->seq_len) return LSA_ERR_INVALID_ARG;
    BlockKeyArgs a{};
    a.seq_len = batch->seq_len; a.B = batch->B; a.L_alloc = batch->L_alloc;
    const int eb = elem_bytes(k_idx->dtype);
    a.kdata = static_cast<const uint8_t*>(k_idx->data);
    a.kscale = k_idx->dtype == LSA_FP8_E4M3 ? k_idx->scale : nullptr;
    a.seq_stride_b = k_idx->seq_stride * eb; a.tok_stride_b = k_idx->tok_stride * eb;
    a.scale_seq_stride = k_idx->scale_seq_stride;
    a.d_I = k_idx->dim; a.block_size = block_size; a.fp8 = k_idx->dtype == LSA_FP8_E4M3;
    a.kbar = static_cast<uint16_t*>(kbar); a.kbar_seq_stride = kbar_seq_stride; a.status = dev_status;
    return cuda_status(launch_block_keys(a, static_cast<cudaStream_t>(stream)));
}

lsa_status lsa_block_score(const lsa_batch* batch, const void* q_idx, const float* w, int H_I, int d_I,
                           const void* kbar, int64_t kbar_seq_stride, int block_size, float* scores,
                           int64_t ld_scores, int n_cols, int32_t* dev_status, void* stream) {
    lsa_status s = check_batch(batch);
    if (s != LSA_OK) return s;
    if (!supported_hi(H_I) || (d_I != 64 && d_I != 128)) return LSA_ERR_UNSUPPORTED;
    if (block_size < 1 || n_cols < 0 || n_cols > ld_scores) return LSA_ERR_INVALID_ARG;
    const int64_t nblk = (batch->L_alloc + block_size - 1) / block_size;
    if (n_cols > nblk || kbar_seq_stride < nblk * 2 * d_I || kbar_seq_stride % 8) return LSA_ERR_INVALID_ARG;
    if (batch->T == 0) return LSA_OK;
    if (!q_idx || !w || !kbar || !scores || ((uintptr_t)kbar & 15) || ((uintptr_t)q_idx & 15)) return LSA_ERR_INVALID_ARG;
    BlockScoreArgs a{};
    a.seq_len = batch->seq_len; a.q_seq = batch->q_seq; a.q_pos = batch->q_pos;
    a.B = batch->B; a.T = batch->T; a.L_alloc = batch->L_alloc; a.q_group = batch->q_group;
    a.q = static_cast<const uint16_t*>(q_idx); a.w = w;
    a.kbar = static_cast<const uint16_t*>(kbar); a.kbar_seq_stride = kbar_seq_stride; a.L_blocks = (int)nblk;
    a.d_I = d_I; a.block_size = block_size;
    a.scores = scores; a.ld = ld_scores; a.n_cols = n_cols; a.status = dev_status;
    return cuda_status(launch_block_score(a, H_I, static_cast<cudaStream_t>(stream)));
}

lsa_status lsa_topk(const lsa_batch* batch, const float* scores, int64_t ld_scores, int n_cols,
                    const int32_t* cand_blocks, int n_cand, int block_size, int k, int n_sink, int window,
                    uint32_t flags, int32_t* idx, int64_t ld_idx, int32_t* count, int32_t* dev_status,
                    void* stream) {
    return topk_impl(batch, scores, ld_scores, n_cols, cand_blocks, n_cand, block_size, k, n_sink, window, flags,
                     idx, ld_idx, count, dev_status, static_cast<cudaStream_t>(stream));
}

lsa_status lsa_sparse_attn(const lsa_batch* batch, const void* q, int H, int Dqk, const lsa_cache* kv,
                           const lsa_cache* v, int Dv, const int32_t* idx, int64_t ld_idx, const int32_t* count,
                           float sm_scale, int n_split, void* o, float* lse, void* ws, size_t ws_bytes,
                           int32_t* dev_status, void* stream) {
    return attn_impl(batch, q, H, Dqk, kv, v, Dv, idx, ld_idx, count, sm_scale, n_split, o, lse, ws, ws_bytes,
                     dev_status, static_cast<cudaStream_t>(stream));
}

size_t lsa_attn_workspace_size(int T, int H, int Dv, int n_split) {
    if (T < 0 || H < 0 || Dv < 0) return 0;
    return attn_ws(T, H, Dv, n_split);
}

int lsa_decode_index_capacity(const lsa_decode_params* p) {
    if (!p) return 0;
    return p->k + p->n_sink + p->window + (p->si_window_aligned && p->window > 0 ? kWindowAlign - 1 : 0);
}

size_t lsa_decode_workspace_size(const lsa_decode_params* p) {
    if (!p) return 0;
    FusedPlan f;
    plan_fused(p, f);
    return f.total;
}

lsa_status lsa_decode_fused(const lsa_decode_params* p, void* ws, size_t ws_bytes, int32_t* dev_status,
                            void* stream) {
    if (!p) return LSA_ERR_INVALID_ARG;
    const lsa_batch* batch = &p->batch;
    lsa_status s = check_batch(batch);
    if (s != LSA_OK) return s;
    if (p->n_layers < 0 || (p->n_layers > 0 && !p->layers)) return LSA_ERR_INVALID_ARG;
    if (p->k < 0 || p->n_sink < 0 || p->window < 0) return LSA_ERR_INVALID_ARG;
    if (p->hi && (p->block_size < 1 || p->block_size > 1024 || p->n_recall < 1 || !p->kbar)) return LSA_ERR_INVALID_ARG;
    if (p->idx_out && p->idx_ld < (int64_t)lsa_decode_index_capacity(p)) return LSA_ERR_INVALID_ARG;
    if ((p->idx_out == nullptr) != (p->count_out == nullptr)) return LSA_ERR_INVALID_ARG;
    FusedPlan f;
    plan_fused(p, f);
    if (!ws || ws_bytes < f.total || ((uintptr_t)ws % kAlign)) return LSA_ERR_WORKSPACE;
    if (batch->T == 0) return LSA_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char* w = static_cast<char*>(ws);
    float* scores = reinterpret_cast<float*>(w + f.scores);
    int32_t* idx = p->idx_out ? p->idx_out : reinterpret_cast<int32_t*>(w + f.idx);
    int32_t* count = p->count_out ? p->count_out : reinterpret_cast<int32_t*>(w + f.count);
    const int64_t ld_idx = p->idx_out ? p->idx_ld : f.cap;
    const uint32_t topk_flags = (p->si_fixed_budget ? LSA_TOPK_EXCLUDES_FIXED : 0u) |
                                (p->si_window_aligned ? LSA_TOPK_WINDOW_ALIGNED : 0u);

    if (!p->hi) {
        s = index_score_impl(batch, p->q_idx, p->w, p->H_I, &p->k_idx, nullptr, 0, 0, scores, f.ld, f.n_cols,
                             dev_status, st, p->idx_q_fp8 != 0);
        if (s != LSA_OK) return s;
        s = topk_impl(batch, scores, f.ld, f.n_cols, nullptr, 0, 0, p->k, p->n_sink, p->window, topk_flags, idx,
                      ld_idx, count, dev_status, st);
        if (s != LSA_OK) return s;
    } else {
        float* bscores = reinterpret_cast<float*>(w + f.bscores);
        int32_t* cand = reinterpret_cast<int32_t*>(w + f.cand);
        int32_t* ccount = reinterpret_cast<int32_t*>(w + f.ccount);
        s = lsa_block_score(batch, p->q_idx, p->w, p->H_I, p->k_idx.dim, p->kbar, p->kbar_seq_stride,
                            p->block_size, bscores, f.bld, f.nblk, dev_status, st);
        if (s != LSA_OK) return s;
        s = topk_impl(batch, bscores, f.bld, f.nblk, nullptr, 0, 0, p->n_recall, 0, 0, LSA_TOPK_RAW, cand,
                      p->n_recall, ccount, dev_status, st);
        if (s != LSA_OK) return s;
        s = index_score_impl(batch, p->q_idx, p->w, p->H_I, &p->k_idx, cand, p->n_recall, p->block_size, scores,
                             f.ld, 0, dev_status, st, p->idx_q_fp8 != 0);
        if (s != LSA_OK) return s;
        s = topk_impl(batch, scores, f.ld, f.n_cols, cand, p->n_recall, p->block_size, p->k, p->n_sink, p->window,
                      topk_flags, idx, ld_idx, count, dev_status, st);
        if (s != LSA_OK) return s;
    }
    // The attention queries may come from a prolog still running elsewhere: everything below
    // waits for it, the selection above did not.
    if (p->attn_q_ready && p->n_layers > 0 &&
        cudaStreamWaitEvent(st, static_cast<cudaEvent_t>(p->attn_q_ready), 0) != cudaSuccess)
        return LSA_ERR_CUDA;
    // The layers depend only on the shared index list, not on one another: layer l runs on
    // branch l mod 2 (the caller's stream, and a second stream forked from it after top-k),
    // each branch with its own split partials, so that one layer's CTAs fill the SMs the
    // other's leave.  Without a second stream the layers run in order on the caller's.
    AuxStream* aux = p->n_layers > 1 ? aux_stream() : nullptr;
    if (aux) {
        if (cudaEventRecord(aux->fork, st) != cudaSuccess || cudaStreamWaitEvent(aux->s, aux->fork, 0) != cudaSuccess)
            return LSA_ERR_CUDA;
    }
    for (int l = 0; l < p->n_layers; ++l) {
        const lsa_layer& L = p->layers[l];
        const int br = aux ? (l & 1) : 0;
        float* part = reinterpret_cast<float*>(w + f.attn + (size_t)(l & 1) * f.attn_one);
        s = attn_impl(batch, L.q, p->H, p->Dqk, &L.kv, L.v.data ? &L.v : nullptr, p->Dv, idx, ld_idx, count,
                      p->sm_scale, p->n_split, L.o, L.lse, part, f.attn_one, dev_status, br ? aux->s : st);
        if (s != LSA_OK) break;
    }
    if (aux) {                                   // join, also after an error, so the caller's stream waits
        if (cudaEventRecord(aux->join, aux->s) != cudaSuccess || cudaStreamWaitEvent(st, aux->join, 0) != cudaSuccess)
            return LSA_ERR_CUDA;
    }
    if (s != LSA_OK) return s;
    return LSA_OK;
}

lsa_status lsa_sparse_attn_partial(const lsa_batch* batch, const void* q, int H, int Dqk, const lsa_cache* kv,
                                   const lsa_cache* v, int Dv, const int32_t* idx, int64_t ld_idx,
                                   const int32_t* count, float sm_scale, int n_split, float* o_part, float* lse_part,
                                   void* ws, size_t ws_bytes, int32_t* dev_status, void* stream) {
    if (batch && batch->T > 0 && (!o_part || !lse_part)) return LSA_ERR_INVALID_ARG;
    return attn_impl(batch, q, H, Dqk, kv, v, Dv, idx, ld_idx, count, sm_scale, n_split, nullptr, nullptr, ws,
                     ws_bytes, dev_status, static_cast<cudaStream_t>(stream), o_part, lse_part);
}

lsa_status lsa_merge_partials(const float* o_parts, const float* lse_parts, int n_parts, int T, int H, int Dv,
                              void* o, float* lse, void* stream) {
    if (n_parts < 1 || n_parts > 1024 || T < 0 || H < 1 || Dv < 8 || Dv % 8) return LSA_ERR_INVALID_ARG;
    if (T > kMaxTokens) return LSA_ERR_UNSUPPORTED;
    if (T == 0) return LSA_OK;
    if (!o_parts || !lse_parts || !o || !aligned16(o_parts) || !aligned16(o)) return LSA_ERR_INVALID_ARG;
    return cuda_status(launch_merge_partials(o_parts, lse_parts, n_parts, (int64_t)T * H, H, T, H, Dv,
                                             static_cast<uint16_t*>(o), nullptr, lse,
                                             static_cast<cudaStream_t>(stream)));
}

lsa_status lsa_kvp_shard_batch(const lsa_batch* global, int L_alloc_local, const int32_t* shard_start,
                               const int32_t* shard_len, int32_t* local_seq_len, int32_t* local_q_pos,
                               int32_t* dev_status, void* stream) {
    lsa_status s = check_batch(global);
    if (s != LSA_OK) return s;
    if (L_alloc_local < 1 || !shard_start || !shard_len || !local_seq_len || (global->T > 0 && !local_q_pos))
        return LSA_ERR_INVALID_ARG;
    return cuda_status(launch_kvp_shard_batch(global->B, global->T, L_alloc_local, global->seq_len, global->q_seq,
                                              global->q_pos, shard_start, shard_len, local_seq_len, local_q_pos,
                                              dev_status, static_cast<cudaStream_t>(stream)));
}

lsa_status lsa_kvp_candidates(const lsa_batch* local, const int32_t* q_pos_global, const int32_t* shard_start,
                              const float* scores, int64_t ld_scores, int n_cols, int k, int32_t* cand_pos,
                              float* cand_score, int32_t* cand_count, int32_t* dev_status, void* stream) {
    lsa_status s = check_batch(local);
    if (s != LSA_OK) return s;
    if (k < 1) return LSA_ERR_INVALID_ARG;
    if (local->T == 0) return LSA_OK;
    if (!q_pos_global || !shard_start || !cand_score || !cand_count) return LSA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    s = topk_impl(local, scores, ld_scores, n_cols, nullptr, 0, 0, k, 0, 0, LSA_TOPK_RAW, cand_pos, k, cand_count,
                  dev_status, st);
    if (s != LSA_OK) return s;
    return cuda_status(launch_kvp_candidates(local->T, k, local->q_seq, q_pos_global, shard_start, local->B, scores,
                                             ld_scores, cand_count, cand_pos, cand_score, st));
}

size_t lsa_kvp_select_workspace_size(int T, int n_parts, int k_part) {
    if (T < 0 || n_parts < 0 || k_part < 0) return 0;
    const size_t n = (size_t)T * n_parts * k_part;
    return align_up(n * 4) + align_up(n * 4);
}

lsa_status lsa_kvp_select(const lsa_batch* global, const int32_t* cand_pos, const float* cand_score, int n_parts,
                          int k_part, int k, int n_sink, int window, int32_t* idx, int64_t ld_idx, int32_t* count,
                          void* ws, size_t ws_bytes, int32_t* dev_status, void* stream) {
    lsa_status s = check_batch(global);
    if (s != LSA_OK) return s;
    if (n_parts < 1 || k_part < 1 || (int64_t)n_parts * k_part > 0x7fffffff) return LSA_ERR_INVALID_ARG;
    if (global->T == 0) return LSA_OK;
    if (!cand_pos || !cand_score) return LSA_ERR_INVALID_ARG;
    const size_t need = lsa_kvp_select_workspace_size(global->T, n_parts, k_part);
    if (!ws || ws_bytes < need || ((uintptr_t)ws % kAlign)) return LSA_ERR_WORKSPACE;
    const int n = n_parts * k_part;
    int32_t* pos_row = static_cast<int32_t*>(ws);
    float* score_row = reinterpret_cast<float*>(static_cast<char*>(ws) + align_up((size_t)global->T * n * 4));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    s = cuda_status(launch_kvp_gather(global->T, n_parts, k_part, cand_pos, cand_score, pos_row, score_row, st));
    if (s != LSA_OK) return s;
    // Columns in part order, each part's positions ascending and the parts' ranges ascending: the
    // column order is the position order, so the (score desc, column asc) selection of lsa_topk is
    // the (score desc, position asc) one; each column maps to its position as a block of one row.
    return topk_impl(global, score_row, n, n, pos_row, n, 1, k, n_sink, window, 0, idx, ld_idx, count, dev_status, st);
}

lsa_status lsa_kvp_local_index(const lsa_batch* global, const int32_t* shard_start, const int32_t* shard_len,
                               const int32_t* idx, int64_t ld_idx, const int32_t* count, int32_t* local_idx,
                               int64_t ld_local, int32_t* local_count, int32_t* dev_status, void* stream) {
    lsa_status s = check_batch(global);
    if (s != LSA_OK) return s;
    if (ld_idx < 1 || ld_local < ld_idx) return LSA_ERR_INVALID_ARG;
    if (global->T == 0) return LSA_OK;
    if (!shard_start || !shard_len || !idx || !count || !local_idx || !local_count) return LSA_ERR_INVALID_ARG;
    return cuda_status(launch_kvp_local_index(global->T, global->B, global->q_seq, shard_start, shard_len, idx, ld_idx,
                                              count, local_idx, ld_local, local_count, dev_status,
                                              static_cast<cudaStream_t>(stream)));
}

lsa_status lsa_read_device_status(const int32_t* dev_status, void* stream) {
    if (!dev_status) return LSA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t v = 0;
    if (cudaStreamSynchronize(st) != cudaSuccess) return LSA_ERR_CUDA;
    if (cudaMemcpy(&v, dev_status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return LSA_ERR_CUDA;
    return static_cast<lsa_status>(v);
}

const char* lsa_status_string(lsa_status s) {
    switch (s) {
        case LSA_OK: return "ok";
        case LSA_ERR_INVALID_ARG: return "invalid argument";
        case LSA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case LSA_ERR_WORKSPACE: return "workspace missing or too small";
        case LSA_ERR_CUDA: return "CUDA error";
        case LSA_ERR_DEVICE_DATA: return "bad device data (lengths, positions, indices or NaN scores)";
        case LSA_ERR_TIMEOUT: return "bounded device wait timed out";
    }
    return "unknown status";
}

int lsa_version(void) { return 1; }

uint64_t lsa_set_wait_limit_ns(uint64_t ns) { return g_wait_limit_ns.exchange(ns); }

}  // extern "C"
