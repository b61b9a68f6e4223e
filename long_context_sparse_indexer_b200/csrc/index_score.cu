// Indexer scores  I(t,s) = sum_h w[t,h] * ReLU(q[t,h,:] . k_s)  over an indexer key cache.
//
// LongCat-2.0 release post ("美团大模型LongCat-2.0 正式发布…"), section "LongCat 稀疏注意力":
// the lightweight indexer scores every cached key for each query and its scoring cost is
// what LSA attacks; the score takes the DSA lightning-indexer form (per-head dot product,
// ReLU, weighted head sum).  The HI bullet's fine stage is the same score restricted to
// the tokens of the recalled blocks (cand_blocks != NULL).
//
// Work decomposition.  A CTA of 4 warps owns 1024 consecutive score columns of one group
// of up to 4 query tokens that share a sequence, so each key row is read from HBM once
// per group.  A warp takes 32 key rows at a time as the A operand (two m16 tiles) of
// warp-level m16n8k16 MMAs; the group's queries (heads x dims) are the B operand, kept in
// shared memory.  FP8 keys are widened to f16 in registers (exact); each query head is
// scaled by a power of two into f16 range (exact for all but values 2^28 below the head's
// maximum), and the inverse power is folded into the head weight.  The epilogue applies
// ReLU, the weighted head sum (fixed order: per-lane partial sums, then a 2-step
// butterfly), and the per-token FP8 scale, which commutes with ReLU because it is
// positive.
#include "kernels.cuh"

namespace lsa {

constexpr int kIdxWarps = 4;
constexpr int kIdxColsPerCta = 1024;
constexpr int kIdxMaxGroup = 4;

template <bool FP8, int D_I, int NT>
__global__ void __launch_bounds__(kIdxWarps * 32)
index_score_kernel(IndexArgs a) {
    constexpr int H_I = NT * 8;
    constexpr int MT = (NT <= 8) ? 2 : 1;              // m16 tiles (16 keys each) per warp
    constexpr int ROWS = MT * 16;                       // keys per warp per step
    constexpr int EB = FP8 ? 1 : 2;                     // bytes per key element
    constexpr int EPC = 16 / EB;                        // elements per 16-byte chunk
    constexpr int SPC = EPC / 4;                        // k16 steps fed by one chunk (per lane)
    constexpr int CH = D_I * EB / 16;                   // chunks per key row
    constexpr int CPL = CH / 4;                         // chunks per lane per row
    constexpr int KS = D_I / 16;                        // k16 steps
    constexpr int QLD = D_I + 4;                        // padded smem row (elements)
    static_assert(CPL * SPC == KS, "k mapping");

    extern __shared__ __align__(16) unsigned char smem_raw[];
    uint16_t* sq = reinterpret_cast<uint16_t*>(smem_raw);                     // [group][H_I][QLD]
    float* sw = reinterpret_cast<float*>(smem_raw + (size_t)kIdxMaxGroup * H_I * QLD * 2);  // [group][H_I]
    __shared__ int s_pos[kIdxMaxGroup];
    __shared__ int s_ok[kIdxMaxGroup];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    const int t0 = blockIdx.y * a.group;
    const int G = min(a.group, a.T - t0);
    const int bseq = a.q_seq[t0];

    if (threadIdx.x < kIdxMaxGroup) {
        int t = t0 + threadIdx.x, ok = 0, pos = -1;
        if ((int)threadIdx.x < G) {
            int sq_ = a.q_seq[t];
            pos = a.q_pos[t];
            ok = 1;
            if (sq_ != bseq || sq_ < 0 || sq_ >= a.B) { report(a.status, LSA_ERR_DEVICE_DATA); ok = 0; }
            else {
                int len = a.seq_len[sq_];
                if (len < 1 || len > a.L_alloc || pos < 0 || pos >= len) { report(a.status, LSA_ERR_DEVICE_DATA); ok = 0; }
            }
        }
        s_pos[threadIdx.x] = ok ? pos : -1;
        s_ok[threadIdx.x] = ok;
    }
    // Queries of the group -> shared memory (f16 scaled per head for FP8 keys, bf16 as is).
    for (int hh = warp; hh < G * H_I; hh += kIdxWarps) {
        const int gi = hh / H_I, h = hh % H_I;
        const uint16_t* src = a.q + ((size_t)(t0 + gi) * H_I + h) * D_I;
        float v[D_I / 32];
        float m = 0.f;
#pragma unroll
        for (int i = 0; i < D_I / 32; ++i) {
            v[i] = bf16_bits_to_float(src[lane + 32 * i]);
            m = fmaxf(m, fabsf(v[i]));
        }
        m = warp_max(m);
        int k = 0;
        if (FP8) {
            int e = (int)((__float_as_uint(m) >> 23) & 0xff) - 127;   // m in [2^e, 2^(e+1)) when normal
            k = (m > 0.f) ? 14 - e : 0;
            k = max(-126, min(126, k));
        }
        const float sc = exp2i(k);
#pragma unroll
        for (int i = 0; i < D_I / 32; ++i) {
            uint16_t bits;
            if (FP8) bits = __half_as_ushort(__float2half_rn(v[i] * sc));
            else bits = src[lane + 32 * i];
            sq[((size_t)gi * H_I + h) * QLD + lane + 32 * i] = bits;
        }
        if (lane == 0) sw[gi * H_I + h] = a.w[(size_t)(t0 + gi) * H_I + h] * exp2i(-k);
    }
    __syncthreads();

    int max_pos = -1;
    for (int gi = 0; gi < G; ++gi) max_pos = max(max_pos, s_pos[gi]);

    const bool hi = a.cand != nullptr;
    const uint8_t* kseq = a.kdata + (size_t)max(bseq, 0) * a.seq_stride_b;
    const float* sseq = a.kscale ? a.kscale + (size_t)max(bseq, 0) * a.scale_seq_stride : nullptr;

    for (int it = 0; it < kIdxColsPerCta / (kIdxWarps * ROWS); ++it) {
        const int col0 = blockIdx.x * kIdxColsPerCta + (it * kIdxWarps + warp) * ROWS;
        if (col0 >= a.n_cols) break;

        // This lane's key rows: (mt, half) -> column col0 + mt*16 + g + 8*half.
        int rowid[MT][2];
        bool rv[MT][2];
        bool any = false;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int col = col0 + mt * 16 + g + 8 * hf;
                int row = -1;
                if (col < a.n_cols) {
                    if (!hi) row = col;
                    else {
                        const int blk = a.cand[(size_t)t0 * a.n_cand + col / a.block_size];
                        if (blk >= 0) row = blk * a.block_size + col % a.block_size;
                    }
                }
                rowid[mt][hf] = row;
                rv[mt][hf] = row >= 0 && row <= max_pos;
                any |= rv[mt][hf];
            }
        if (!__any_sync(0xffffffffu, any)) {
            // Nothing visible for any query of the group: -inf columns.
#pragma unroll
            for (int gi = 0; gi < kIdxMaxGroup; ++gi) {
                if (gi >= G) break;
                const int col = col0 + lane;
                if (lane < ROWS && col < a.n_cols) a.scores[(size_t)(t0 + gi) * a.ld + col] = kNegInf;
            }
            continue;
        }

        // Load and widen the A operand (keys).
        uint32_t afr[MT][KS][4];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            uint4 ch[2][CPL];
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const uint8_t* rp = kseq + (size_t)max(rowid[mt][hf], 0) * a.tok_stride_b;
#pragma unroll
                for (int hh = 0; hh < CPL; ++hh)
                    ch[hf][hh] = rv[mt][hf] ? ldg_nc16(rp + (size_t)(c + 4 * hh) * 16) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int s = 0; s < KS; ++s) {
                const int hh = s / SPC, u = s % SPC;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const uint32_t* wd = reinterpret_cast<const uint32_t*>(&ch[hf][hh]);
                    uint32_t lo, hi2;
                    if (FP8) {
                        lo = e4m3x2_to_f16x2((uint16_t)(wd[u] & 0xffff));
                        hi2 = e4m3x2_to_f16x2((uint16_t)(wd[u] >> 16));
                    } else {
                        lo = wd[2 * u];
                        hi2 = wd[2 * u + 1];
                    }
                    afr[mt][s][hf] = lo;          // a0 (row g) / a1 (row g+8)
                    afr[mt][s][2 + hf] = hi2;     // a2 / a3
                }
            }
        }

        float kscale_out = 1.f;
        const int my_mt = c >> 1, my_hf = c & 1;
        const int my_col = col0 + my_mt * 16 + g + 8 * my_hf;
        int my_row = -1;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf)
                if (mt == my_mt && hf == my_hf) my_row = rowid[mt][hf];
        if (FP8 && my_row >= 0 && my_row <= max_pos && sseq) kscale_out = sseq[my_row];

        for (int gi = 0; gi < G; ++gi) {
            float acc[MT][NT][4];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;
            const uint16_t* qg = sq + (size_t)gi * H_I * QLD;
#pragma unroll
            for (int s = 0; s < KS; ++s) {
                const int hh = s / SPC, u = s % SPC;
                const int dim = EPC * (c + 4 * hh) + 4 * u;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const uint2 bq = *reinterpret_cast<const uint2*>(qg + (size_t)(nt * 8 + g) * QLD + dim);
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) {
                        if (FP8) mma_f16_16816(acc[mt][nt], afr[mt][s], bq.x, bq.y);
                        else mma_bf16_16816(acc[mt][nt], afr[mt][s], bq.x, bq.y);
                    }
                }
            }
            // Epilogue: per key row, sum over heads of w' * ReLU(acc).
            const float* wg = sw + gi * H_I;
            float part[MT][2];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    float p = 0.f;
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        const float2 ww = *reinterpret_cast<const float2*>(wg + nt * 8 + 2 * c);
                        p = fmaf(ww.x, fmaxf(acc[mt][nt][2 * hf], 0.f), p);
                        p = fmaf(ww.y, fmaxf(acc[mt][nt][2 * hf + 1], 0.f), p);
                    }
                    p += __shfl_xor_sync(0xffffffffu, p, 1);
                    p += __shfl_xor_sync(0xffffffffu, p, 2);
                    part[mt][hf] = p;
                }
            float val = 0.f;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int hf = 0; hf < 2; ++hf)
                    if (mt == my_mt && hf == my_hf) val = part[mt][hf];
            if (my_mt < MT && my_col < a.n_cols) {
                const int pos = s_pos[gi];
                const bool vis = s_ok[gi] && my_row >= 0 && my_row <= pos;
                a.scores[(size_t)(t0 + gi) * a.ld + my_col] = vis ? val * kscale_out : kNegInf;
            }
        }
    }
}

template <bool FP8, int D_I, int NT>
static cudaError_t launch_index_t(const IndexArgs& a, cudaStream_t st) {
    constexpr int H_I = NT * 8;
    const size_t smem = (size_t)kIdxMaxGroup * H_I * (D_I + 4) * 2 + (size_t)kIdxMaxGroup * H_I * 4;
    auto kern = index_score_kernel<FP8, D_I, NT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((a.n_cols + kIdxColsPerCta - 1) / kIdxColsPerCta, (a.T + a.group - 1) / a.group);
    kern<<<grid, kIdxWarps * 32, smem, st>>>(a);
    return cudaGetLastError();
}

template <bool FP8, int D_I>
static cudaError_t launch_index_d(const IndexArgs& a, int H_I, cudaStream_t st) {
    switch (H_I) {
        case 8: return launch_index_t<FP8, D_I, 1>(a, st);
        case 16: return launch_index_t<FP8, D_I, 2>(a, st);
        case 32: return launch_index_t<FP8, D_I, 4>(a, st);
        case 64: return launch_index_t<FP8, D_I, 8>(a, st);
        case 128: return launch_index_t<FP8, D_I, 16>(a, st);
    }
    return cudaErrorInvalidValue;
}

// Host launcher; the caller has validated shapes (H_I in {8,16,32,64,128}, D_I in {64,128}).
cudaError_t launch_index_score(IndexArgs a, int H_I, int D_I, bool fp8, cudaStream_t st) {
    if (a.cand) a.group = 1;
    else a.group = a.q_group < kIdxMaxGroup ? a.q_group : (a.q_group % kIdxMaxGroup == 0 ? kIdxMaxGroup
                                                           : (a.q_group % 2 == 0 ? 2 : 1));
    if (a.n_cols <= 0 || a.T <= 0) return cudaSuccess;
    if (index_score_tc_supported(a, H_I, D_I, fp8)) return launch_index_score_tc(a, H_I, st);
    if (!fp8 && !a.cand) {
        // BF16 keys: the tensor-core row scorer (row_score_tc.cu), one key per row.
        RowScoreArgs r{};
        r.seq_len = a.seq_len; r.q_seq = a.q_seq; r.q_pos = a.q_pos;
        r.B = a.B; r.T = a.T; r.L_alloc = a.L_alloc; r.q_group = a.q_group;
        r.q = a.q; r.w = a.w; r.H_I = H_I; r.d_I = D_I; r.halves = 1; r.row_span = 1;
        r.scores = a.scores; r.ld = a.ld; r.n_cols = a.n_cols; r.status = a.status;
        if (row_score_tc_supported(r, D_I, a.tok_stride_b, a.seq_stride_b, a.kdata))
            return launch_row_score_tc(r, a.L_alloc, a.tok_stride_b, a.seq_stride_b, a.kdata, st);
    }
    if (fp8) return D_I == 64 ? launch_index_d<true, 64>(a, H_I, st) : launch_index_d<true, 128>(a, H_I, st);
    return D_I == 64 ? launch_index_d<false, 64>(a, H_I, st) : launch_index_d<false, 128>(a, H_I, st);
}

}  // namespace lsa
