// Sparse attention over the selected rows, split-KV partials and their log-sum-exp merge.
//
// Explainer page ("如何在 5 万张国产芯片训练出 1.6T 万亿参数模型？"), section "① LSA": attention
// reads only the top-k keys and the sink tokens the indexer selected; the model's
// attention is MLA in absorbed form, so all heads of a query share one latent KV row
// (K = the 576-dim row, V = its first 512 dims).  Section "③ KVP 解码切分示意": each KV
// shard computes a partial attention and the partial results are merged; here the shards
// are contiguous chunks of one query's index list (n_split), merged in split order, a fixed
// order, as the release post's section "确定性与可靠性" asks of reductions.
//
// CTA = (split, group of 16*MT heads, query token).  Warps 0..4*MT-1: warp w owns head
// tile (w % MT) and quarter (w / MT).  For S = Q K^T each quarter computes a partial over
// a quarter of the QK dims; the four partials meet in shared memory and are summed in a
// fixed order.  Every warp then runs the same online softmax on its head tile and
// accumulates P V for its quarter of the V dims.  FP8 rows are widened exactly to BF16;
// their per-row scale multiplies the scores and the probabilities.
#include "kernels.cuh"

namespace lsa {

constexpr int kNR = 32;          // rows per tile

template <int DQK, int DV, int MT, bool KV_FP8, bool SEP_V>
struct AttnCfg {
    static constexpr int WARPS = 4 * MT;
    static constexpr int THREADS = WARPS * 32;
    static constexpr int KLD = DQK + 8;              // padded smem row (elements): 16 B shift per row
    static constexpr int VLD = DV + 8;
    static constexpr int KQ = DQK / 4 / 16;          // k16 steps per quarter
    static constexpr int NV = DV / 4 / 8;            // n8 tiles of V per quarter
    static constexpr size_t K_BYTES = (size_t)kNR * KLD * 2;
    static constexpr size_t V_BYTES = SEP_V ? (size_t)kNR * VLD * 2 : 0;
    static constexpr size_t SP_BYTES = (size_t)4 * MT * 16 * kNR * 4;
    static constexpr size_t SMEM = K_BYTES + V_BYTES + SP_BYTES + 3 * kNR * 4;
};

template <int DQK, int DV, int MT, bool KV_FP8, bool SEP_V>
__global__ void __launch_bounds__(AttnCfg<DQK, DV, MT, KV_FP8, SEP_V>::THREADS)
sparse_attn_kernel(AttnArgs a) {
    using C = AttnCfg<DQK, DV, MT, KV_FP8, SEP_V>;
    static_assert(DQK % 64 == 0 && DV % 64 == 0, "dims");
    extern __shared__ __align__(16) unsigned char smem[];
    uint16_t* sK = reinterpret_cast<uint16_t*>(smem);
    uint16_t* sV = SEP_V ? reinterpret_cast<uint16_t*>(smem + C::K_BYTES) : sK;
    float* sP = reinterpret_cast<float*>(smem + C::K_BYTES + C::V_BYTES);          // [4][MT][16][kNR]
    float* sKs = reinterpret_cast<float*>(smem + C::K_BYTES + C::V_BYTES + C::SP_BYTES);  // [kNR] K scale
    float* sVs = sKs + kNR;                                                         // [kNR] V scale
    int* sOk = reinterpret_cast<int*>(sVs + kNR);                                   // [kNR] row valid
    const int vld = SEP_V ? C::VLD : C::KLD;

    const int split = blockIdx.x, hg = blockIdx.y, t = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    const int mw = warp % MT, qw = warp / MT;
    const int h0 = hg * 16 * MT + mw * 16;             // first head of this warp's tile

    const int b = a.q_seq[t];
    int len = 0;
    bool ok = b >= 0 && b < a.B;
    if (ok) { len = a.seq_len[b]; ok = len >= 1 && len <= a.L_alloc; }
    int n = ok ? a.count[t] : 0;
    if (n < 0 || n > a.ld_idx) { ok = false; n = 0; }
    if (!ok && threadIdx.x == 0 && split == 0 && hg == 0) report(a.status, LSA_ERR_DEVICE_DATA);
    const int per = (n + a.n_split - 1) / a.n_split;
    const int r_beg = min(n, split * per), r_end = min(n, r_beg + per);
    const int32_t* irow = a.idx + (size_t)t * a.ld_idx;
    const uint8_t* kvb = a.kv + (size_t)max(b, 0) * a.kv_seq_b;
    const float* kvs = KV_FP8 ? a.kv_scale + (size_t)max(b, 0) * a.kv_scale_seq : nullptr;
    const uint8_t* vb = SEP_V ? a.v + (size_t)max(b, 0) * a.v_seq_b : nullptr;

    // Q fragments for this warp's head tile and QK quarter (A operand, row-major).
    uint32_t qf[C::KQ][4];
    {
        const uint16_t* q0 = a.q + ((size_t)t * a.H + h0 + g) * DQK + qw * (DQK / 4);
        const uint16_t* q8 = q0 + (size_t)8 * DQK;
#pragma unroll
        for (int s = 0; s < C::KQ; ++s) {
            qf[s][0] = *reinterpret_cast<const uint32_t*>(q0 + s * 16 + 2 * c);
            qf[s][1] = *reinterpret_cast<const uint32_t*>(q8 + s * 16 + 2 * c);
            qf[s][2] = *reinterpret_cast<const uint32_t*>(q0 + s * 16 + 8 + 2 * c);
            qf[s][3] = *reinterpret_cast<const uint32_t*>(q8 + s * 16 + 8 + 2 * c);
        }
    }
    float oacc[C::NV][4];
#pragma unroll
    for (int i = 0; i < C::NV; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) oacc[i][e] = 0.f;
    float m_run[2] = {kNegInf, kNegInf}, l_run[2] = {0.f, 0.f};

    for (int r0 = r_beg; r0 < r_end; r0 += kNR) {
        const int nr = min(kNR, r_end - r0);
        // ---- gather the tile's rows into shared memory
        if (!KV_FP8) {
            constexpr int CPR = DQK * 2 / 16;           // 16-byte chunks per row
            for (int i = threadIdx.x; i < kNR * CPR; i += C::THREADS) {
                const int r = i / CPR, ch = i % CPR;
                int row = r < nr ? irow[r0 + r] : -1;
                bool valid = row >= 0 && row < len;
                if (r < nr && !valid) report(a.status, LSA_ERR_DEVICE_DATA);
                cp_async16(sK + (size_t)r * C::KLD + ch * 8, kvb + (size_t)(valid ? row : 0) * a.kv_tok_b + ch * 16, valid);
            }
            if (SEP_V) {
                constexpr int CPV = DV * 2 / 16;
                for (int i = threadIdx.x; i < kNR * CPV; i += C::THREADS) {
                    const int r = i / CPV, ch = i % CPV;
                    int row = r < nr ? irow[r0 + r] : -1;
                    bool valid = row >= 0 && row < len;
                    cp_async16(sV + (size_t)r * C::VLD + ch * 8, vb + (size_t)(valid ? row : 0) * a.v_tok_b + ch * 16, valid);
                }
            }
            cp_async_commit();
            if (threadIdx.x < kNR) {
                const int r = threadIdx.x;
                const int row = r < nr ? irow[r0 + r] : -1;
                sKs[r] = 1.f;
                sVs[r] = 1.f;
                sOk[r] = row >= 0 && row < len;
            }
            cp_async_wait<0>();
        } else {
            constexpr int CPR = DQK / 16;               // 16 codes per chunk
            for (int i = threadIdx.x; i < kNR * CPR; i += C::THREADS) {
                const int r = i / CPR, ch = i % CPR;
                int row = r < nr ? irow[r0 + r] : -1;
                bool valid = row >= 0 && row < len;
                if (r < nr && !valid) report(a.status, LSA_ERR_DEVICE_DATA);
                uint4 raw = valid ? ldg_nc16(kvb + (size_t)row * a.kv_tok_b + ch * 16) : make_uint4(0, 0, 0, 0);
                const uint32_t* wd = reinterpret_cast<const uint32_t*>(&raw);
                uint32_t outw[8];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    outw[2 * j] = e4m3x2_to_bf16x2((uint16_t)(wd[j] & 0xffff));
                    outw[2 * j + 1] = e4m3x2_to_bf16x2((uint16_t)(wd[j] >> 16));
                }
                uint4* dst = reinterpret_cast<uint4*>(sK + (size_t)r * C::KLD + ch * 16);
                dst[0] = make_uint4(outw[0], outw[1], outw[2], outw[3]);
                dst[1] = make_uint4(outw[4], outw[5], outw[6], outw[7]);
            }
            if (threadIdx.x < kNR) {
                const int r = threadIdx.x;
                int row = r < nr ? irow[r0 + r] : -1;
                bool valid = row >= 0 && row < len;
                const float s = valid ? kvs[row] : 0.f;
                sKs[r] = s;
                sVs[r] = s;
                sOk[r] = valid;
            }
        }
        __syncthreads();

        // ---- partial S over this warp's QK quarter: [16 heads] x [32 rows]
        float sacc[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) sacc[j][e] = 0.f;
#pragma unroll
        for (int s = 0; s < C::KQ; ++s) {
            const int k0 = qw * (DQK / 4) + s * 16;
#pragma unroll
            for (int jp = 0; jp < 2; ++jp) {              // pairs of n8 row tiles
                uint32_t bf[4];
                const int mi = lane >> 3, ri = lane & 7;
                const int row = jp * 16 + (mi >> 1) * 8 + ri;
                const int col = k0 + (mi & 1) * 8;
                ldmatrix_x4(bf, sK + (size_t)row * C::KLD + col);
                mma_bf16_16816(sacc[2 * jp], qf[s], bf[0], bf[1]);
                mma_bf16_16816(sacc[2 * jp + 1], qf[s], bf[2], bf[3]);
            }
        }
        float* myP = sP + ((size_t)(qw * MT + mw) * 16) * kNR;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            *reinterpret_cast<float2*>(myP + g * kNR + j * 8 + 2 * c) = make_float2(sacc[j][0], sacc[j][1]);
            *reinterpret_cast<float2*>(myP + (g + 8) * kNR + j * 8 + 2 * c) = make_float2(sacc[j][2], sacc[j][3]);
        }
        __syncthreads();

        // ---- full S (fixed order), mask, online softmax
        float sv[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int hr = g + 8 * (e >> 1), col = j * 8 + 2 * c + (e & 1);
                const float* base = sP + (size_t)mw * 16 * kNR + hr * kNR + col;
                const size_t qs = (size_t)MT * 16 * kNR;
                const float x = (base[0] + base[qs]) + (base[2 * qs] + base[3 * qs]);
                sv[j][e] = sOk[col] ? x * sKs[col] * a.sm_scale_log2 : kNegInf;
            }
        float alpha[2];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            float mx = kNegInf;
#pragma unroll
            for (int j = 0; j < 4; ++j) mx = fmaxf(mx, fmaxf(sv[j][2 * hf], sv[j][2 * hf + 1]));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            const float m_new = fmaxf(m_run[hf], mx);
            alpha[hf] = (m_new == kNegInf) ? 1.f : exp2f(m_run[hf] - m_new);
            float ls = 0.f;
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const float p = (m_new == kNegInf) ? 0.f : exp2f(sv[j][2 * hf + e] - m_new);
                    sv[j][2 * hf + e] = p;
                    ls += p;
                }
            ls += __shfl_xor_sync(0xffffffffu, ls, 1);
            ls += __shfl_xor_sync(0xffffffffu, ls, 2);
            l_run[hf] = l_run[hf] * alpha[hf] + ls;
            m_run[hf] = m_new;
        }
#pragma unroll
        for (int i = 0; i < C::NV; ++i) {
            oacc[i][0] *= alpha[0]; oacc[i][1] *= alpha[0];
            oacc[i][2] *= alpha[1]; oacc[i][3] *= alpha[1];
        }
        // ---- P (times the V scale) as the A operand; O += P V for this warp's V quarter
        uint32_t pf[2][4];
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
            const int ca = kk * 16 + 2 * c, cb = ca + 8;
            const float v0 = sVs[ca], v1 = sVs[ca + 1], v2 = sVs[cb], v3 = sVs[cb + 1];
            pf[kk][0] = pack_bf16x2(sv[2 * kk][0] * v0, sv[2 * kk][1] * v1);
            pf[kk][1] = pack_bf16x2(sv[2 * kk][2] * v0, sv[2 * kk][3] * v1);
            pf[kk][2] = pack_bf16x2(sv[2 * kk + 1][0] * v2, sv[2 * kk + 1][1] * v3);
            pf[kk][3] = pack_bf16x2(sv[2 * kk + 1][2] * v2, sv[2 * kk + 1][3] * v3);
        }
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
#pragma unroll
            for (int np = 0; np < C::NV / 2; ++np) {
                uint32_t bf[4];
                const int mi = lane >> 3, ri = lane & 7;
                const int row = kk * 16 + (mi & 1) * 8 + ri;
                const int col = qw * (DV / 4) + (2 * np + (mi >> 1)) * 8;
                ldmatrix_x4_trans(bf, sV + (size_t)row * vld + col);
                mma_bf16_16816(oacc[2 * np], pf[kk], bf[0], bf[1]);
                mma_bf16_16816(oacc[2 * np + 1], pf[kk], bf[2], bf[3]);
            }
        }
        __syncthreads();
    }

    // ---- epilogue
    const float kLn2 = 0.69314718055994530942f;
    float inv[2], lse_v[2];
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        inv[hf] = l_run[hf] > 0.f ? 1.f / l_run[hf] : 0.f;
        lse_v[hf] = l_run[hf] > 0.f ? (m_run[hf] + log2f(l_run[hf])) * kLn2 : kNegInf;
    }
    const int dv0 = qw * (DV / 4);
    if (a.n_split == 1 && !a.f32_out) {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            const int h = h0 + g + 8 * hf;
            uint16_t* orow = a.o + ((size_t)t * a.H + h) * DV + dv0;
#pragma unroll
            for (int i = 0; i < C::NV; ++i)
                *reinterpret_cast<uint32_t*>(orow + i * 8 + 2 * c) =
                    pack_bf16x2(oacc[i][2 * hf] * inv[hf], oacc[i][2 * hf + 1] * inv[hf]);
            if (a.lse && qw == 0 && c == 0) a.lse[(size_t)t * a.H + h] = lse_v[hf];
        }
    } else {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            const int h = h0 + g + 8 * hf;
            float* prow = a.part_o + (((size_t)t * a.n_split + split) * a.H + h) * DV + dv0;
#pragma unroll
            for (int i = 0; i < C::NV; ++i)
                *reinterpret_cast<float2*>(prow + i * 8 + 2 * c) =
                    make_float2(oacc[i][2 * hf] * inv[hf], oacc[i][2 * hf + 1] * inv[hf]);
            if (qw == 0 && c == 0) a.part_lse[((size_t)t * a.n_split + split) * a.H + h] = lse_v[hf];
        }
    }
}

// Split merge.  With m = max_s lse_s and w_s = exp(lse_s - m): o = sum_s (w_s / sum w) o_s and
// lse = m + log(sum w), both sums in split order (the values do not depend on the kernel below).
// Partial s of (token t, head h) is row s * part_stride + t * tok_stride + h; the splits of one
// call are [T][n_split][H] (part_stride = H, tok_stride = n_split * H), the per-rank partials of
// KVP [n_part][T][H] (part_stride = T * H, tok_stride = H).
//
// Up to 32 splits: warp = 128 consecutive V dims of one (token, head), lane = 4 of them.  Lane s
// loads lse_s and computes w_s; the others get it by shuffle, so the weights need no shared
// memory and no block barrier, and the first kMergeNS partial rows are loaded together with the
// lse values (one memory round trip).
constexpr int kMergeThreads = 128;
constexpr int kMergeNS = 24;

__device__ __forceinline__ void merge_store(const float4& acc, size_t out, uint16_t* o, float* o32) {
    if (o32) {
        *reinterpret_cast<float4*>(o32 + out) = acc;
    } else {
        uint2 pk;
        pk.x = pack_bf16x2(acc.x, acc.y);
        pk.y = pack_bf16x2(acc.z, acc.w);
        *reinterpret_cast<uint2*>(o + out) = pk;
    }
}

__device__ __forceinline__ void axpy4(float ws, const float4& x, float4& acc) {
    acc.x = fmaf(ws, x.x, acc.x); acc.y = fmaf(ws, x.y, acc.y);
    acc.z = fmaf(ws, x.z, acc.z); acc.w = fmaf(ws, x.w, acc.w);
}

__global__ void __launch_bounds__(kMergeThreads) merge_kernel(const float* part_o, const float* part_lse,
                                                              int n_split, int H, int DV, int64_t part_stride,
                                                              int64_t tok_stride, uint16_t* o, float* o32,
                                                              float* lse) {
    const int lane = threadIdx.x & 31;
    const int chunks = (DV + 127) / 128;
    const int64_t gw = (int64_t)blockIdx.x * (kMergeThreads / 32) + (threadIdx.x >> 5);
    const int t = blockIdx.y;
    if (gw >= (int64_t)H * chunks) return;                        // whole warps
    const int h = (int)(gw / chunks), d = (int)(gw % chunks) * 128 + lane * 4;
    const bool act = d < DV;
    const size_t row0 = (size_t)t * tok_stride + h;                // (split 0, head h)
    auto src = [&](int s) {
        return reinterpret_cast<const float4*>(part_o + (row0 + (size_t)s * part_stride) * DV + d);
    };
    float4 x[kMergeNS];
    if (act) {
#pragma unroll
        for (int s = 0; s < kMergeNS; ++s)
            if (s < n_split) x[s] = __ldcg(src(s));
    }
    const float l = lane < n_split ? __ldcg(part_lse + row0 + (size_t)lane * part_stride) : kNegInf;
    const float m = warp_max(l);
    const float e = lane < n_split && m != kNegInf ? expf(l - m) : 0.f;
    float wsum = 0.f;
    for (int s = 0; s < n_split; ++s) wsum += __shfl_sync(0xffffffffu, e, s);
    const float rs = wsum > 0.f ? 1.f / wsum : 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int s = 0; s < kMergeNS; ++s) {
        const float ws = __shfl_sync(0xffffffffu, e, s) * rs;
        if (s < n_split) axpy4(ws, x[s], acc);
    }
    for (int s = kMergeNS; s < n_split; ++s) {                     // 25..32 splits: a second round trip
        const float ws = __shfl_sync(0xffffffffu, e, s) * rs;
        if (act) axpy4(ws, __ldcg(src(s)), acc);
    }
    if (act) merge_store(acc, ((size_t)t * H + h) * DV + d, o, o32);
    if (lse && lane == 0 && (gw % chunks) == 0) lse[(size_t)t * H + h] = wsum > 0.f ? m + logf(wsum) : kNegInf;
}

// More than 32 splits: block = one (token, head), thread = 4 consecutive V dims (and every 512th
// dim after them); the lse values go through shared memory once, the rows in chunks of kMergeNS.
__global__ void __launch_bounds__(kMergeThreads) merge_wide_kernel(const float* part_o, const float* part_lse,
                                                                   int n_split, int DV, int64_t part_stride,
                                                                   int64_t tok_stride, uint16_t* o, float* o32,
                                                                   float* lse) {
    extern __shared__ float s_l[];                                 // lse of every split of this (token, head)
    const int h = blockIdx.x, t = blockIdx.y, H = gridDim.x;
    const size_t row0 = (size_t)t * tok_stride + h;
    for (int s = threadIdx.x; s < n_split; s += kMergeThreads)
        s_l[s] = __ldcg(part_lse + row0 + (size_t)s * part_stride);
    __syncthreads();
    float m = kNegInf, wsum = 0.f;
    for (int s = 0; s < n_split; ++s) m = fmaxf(m, s_l[s]);
    for (int s = 0; s < n_split; ++s) wsum += m == kNegInf ? 0.f : expf(s_l[s] - m);
    const float rs = wsum > 0.f ? 1.f / wsum : 0.f;
    for (int d = 4 * threadIdx.x; d < DV; d += 4 * kMergeThreads) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s0 = 0; s0 < n_split; s0 += kMergeNS) {
            float4 x[kMergeNS];
#pragma unroll
            for (int u = 0; u < kMergeNS; ++u)
                if (s0 + u < n_split)
                    x[u] = __ldcg(reinterpret_cast<const float4*>(part_o + (row0 + (size_t)(s0 + u) * part_stride) * DV + d));
#pragma unroll
            for (int u = 0; u < kMergeNS; ++u)
                if (s0 + u < n_split) axpy4((m == kNegInf ? 0.f : expf(s_l[s0 + u] - m)) * rs, x[u], acc);
        }
        merge_store(acc, ((size_t)t * H + h) * DV + d, o, o32);
    }
    if (lse && threadIdx.x == 0) lse[(size_t)t * H + h] = wsum > 0.f ? m + logf(wsum) : kNegInf;
}

cudaError_t launch_merge_partials(const float* part_o, const float* part_lse, int n_part, int64_t part_stride,
                                  int64_t tok_stride, int T, int H, int DV, uint16_t* o, float* o32, float* lse,
                                  cudaStream_t st) {
    if (T <= 0) return cudaSuccess;
    if (n_part <= 32) {
        const int64_t warps = (int64_t)H * ((DV + 127) / 128);
        dim3 mg((unsigned)((warps + kMergeThreads / 32 - 1) / (kMergeThreads / 32)), T);
        merge_kernel<<<mg, kMergeThreads, 0, st>>>(part_o, part_lse, n_part, H, DV, part_stride, tok_stride, o, o32,
                                                   lse);
    } else {
        merge_wide_kernel<<<dim3(H, T), kMergeThreads, (size_t)n_part * sizeof(float), st>>>(
            part_o, part_lse, n_part, DV, part_stride, tok_stride, o, o32, lse);
    }
    return cudaGetLastError();
}

// The merge of one call's split partials ([T][n_split][H]) into its BF16 (or FP32) result.
static cudaError_t launch_merge(const AttnArgs& a, int DV, cudaStream_t st) {
    return launch_merge_partials(a.part_o, a.part_lse, a.n_split, a.H, (int64_t)a.n_split * a.H, a.T, a.H, DV,
                                 a.f32_out ? nullptr : a.o, a.f32_out ? a.o32 : nullptr,
                                 a.f32_out ? a.lse32 : a.lse, st);
}

template <int DQK, int DV, int MT, bool KV_FP8, bool SEP_V>
static cudaError_t launch_attn_t(const AttnArgs& a, cudaStream_t st) {
    using C = AttnCfg<DQK, DV, MT, KV_FP8, SEP_V>;
    auto kern = sparse_attn_kernel<DQK, DV, MT, KV_FP8, SEP_V>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
    if (e != cudaSuccess) return e;
    dim3 grid(a.n_split, a.H / (16 * MT), a.T);
    kern<<<grid, C::THREADS, C::SMEM, st>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess || a.n_split == 1) return e;
    return launch_merge(a, DV, st);
}

// Supported: (576, 512) MLA layout, BF16 or FP8 rows, H % 32 == 0; (128, 128) with a
// separate BF16 V cache, H % 16 == 0.
cudaError_t launch_sparse_attn(const AttnArgs& a, int DQK, int DV, bool kv_fp8, bool sep_v, cudaStream_t st) {
    if (a.T <= 0) return cudaSuccess;
    if (sparse_attn_tc_supported(a, DQK, DV, sep_v)) {
        cudaError_t e = launch_sparse_attn_tc(a, kv_fp8, st);
        if (e != cudaSuccess || a.n_split == 1) return e;
        return launch_merge(a, DV, st);
    }
    if (DQK == 576 && DV == 512 && !sep_v)
        return kv_fp8 ? launch_attn_t<576, 512, 2, true, false>(a, st) : launch_attn_t<576, 512, 2, false, false>(a, st);
    if (DQK == 128 && DV == 128 && sep_v && !kv_fp8) return launch_attn_t<128, 128, 1, false, true>(a, st);
    return cudaErrorInvalidValue;
}

}  // namespace lsa
