// Hierarchical indexing (HI), coarse stage: block keys and block scores.
//
// LongCat-2.0 release post, section "LongCat 稀疏注意力", HI bullet: a coarse-to-fine,
// two-stage scoring -- block-level approximate scores recall candidate blocks, then a
// fine token-level selection runs inside the recalled candidates.  The pages do not say
// how a block is summarised; the block key here is the arithmetic mean of the block's
// dequantised indexer keys, and the block score is the indexer formula applied to it.
#include "kernels.cuh"

namespace lsa {

// One CTA per (block, sequence); thread d sums dimension d over the block's rows with a
// fixed pairwise tree (binary-counter order), then divides by the row count.
__global__ void block_keys_kernel(BlockKeyArgs a) {
    const int b = blockIdx.y, j = blockIdx.x, d = threadIdx.x;
    const int len = a.seq_len[b];
    if (len < 1 || len > a.L_alloc) {
        if (d == 0 && j == 0) report(a.status, LSA_ERR_DEVICE_DATA);
        return;
    }
    const int r0 = j * a.block_size;
    if (r0 >= len || d >= a.d_I) return;
    const int n = min(a.block_size, len - r0);
    const uint8_t* base = a.kdata + (size_t)b * a.seq_stride_b;
    const float* sc = a.kscale ? a.kscale + (size_t)b * a.scale_seq_stride : nullptr;
    float stack[12];
    for (int i = 0; i < n; ++i) {
        const uint8_t* rp = base + (size_t)(r0 + i) * a.tok_stride_b;
        float v;
        if (a.fp8) {
            const uint16_t pair = (uint16_t)rp[d];
            const uint32_t h2 = e4m3x2_to_f16x2(pair);
            v = __half2float(__ushort_as_half((unsigned short)(h2 & 0xffff))) * sc[r0 + i];
        } else {
            v = bf16_bits_to_float(reinterpret_cast<const uint16_t*>(rp)[d]);
        }
        int lvl = 0;
        for (int m = i; m & 1; m >>= 1, ++lvl) v = stack[lvl] + v;
        stack[lvl] = v;
    }
    // Fold the remaining partial sums, lowest level first.
    float tot = 0.f;
    bool have = false;
    for (int lvl = 0; lvl < 12; ++lvl)
        if ((n >> lvl) & 1) { tot = have ? stack[lvl] + tot : stack[lvl]; have = true; }
    a.kbar[(size_t)b * a.kbar_seq_stride + (size_t)j * a.d_I + d] = tot / (float)n;
}

cudaError_t launch_block_keys(const BlockKeyArgs& a, cudaStream_t st) {
    const int nblk = (a.L_alloc + a.block_size - 1) / a.block_size;
    dim3 grid(nblk, a.B);
    block_keys_kernel<<<grid, a.d_I, 0, st>>>(a);
    return cudaGetLastError();
}

constexpr int kBsThreads = 128;

// One thread per block column: J = sum_h w_h * ReLU(q_h . kbar_j), FP32, heads summed in order.
template <int H_I>
__global__ void __launch_bounds__(kBsThreads) block_score_kernel(BlockScoreArgs a) {
    extern __shared__ float sm[];
    float* sq = sm;                       // [H_I][d_I]
    float* sw = sm + H_I * a.d_I;         // [H_I]
    const int t = blockIdx.y;
    for (int i = threadIdx.x; i < H_I * a.d_I; i += kBsThreads)
        sq[i] = bf16_bits_to_float(a.q[(size_t)t * H_I * a.d_I + i]);
    for (int i = threadIdx.x; i < H_I; i += kBsThreads) sw[i] = a.w[(size_t)t * H_I + i];
    __syncthreads();
    const int j = blockIdx.x * kBsThreads + threadIdx.x;
    if (j >= a.n_cols) return;
    const int b = a.q_seq[t], pos = a.q_pos[t];
    bool ok = b >= 0 && b < a.B;
    int len = ok ? a.seq_len[b] : 0;
    if (!ok || len < 1 || len > a.L_alloc || pos < 0 || pos >= len) {
        if (j == 0) report(a.status, LSA_ERR_DEVICE_DATA);
        a.scores[(size_t)t * a.ld + j] = kNegInf;
        return;
    }
    if ((int64_t)j * a.block_size > pos) { a.scores[(size_t)t * a.ld + j] = kNegInf; return; }
    const float* kr = a.kbar + (size_t)b * a.kbar_seq_stride + (size_t)j * a.d_I;
    float acc[H_I];
#pragma unroll
    for (int h = 0; h < H_I; ++h) acc[h] = 0.f;
    for (int d0 = 0; d0 < a.d_I; d0 += 4) {
        const float4 kv = *reinterpret_cast<const float4*>(kr + d0);
#pragma unroll
        for (int h = 0; h < H_I; ++h) {
            const float* qh = sq + h * a.d_I + d0;
            acc[h] = fmaf(qh[0], kv.x, acc[h]);
            acc[h] = fmaf(qh[1], kv.y, acc[h]);
            acc[h] = fmaf(qh[2], kv.z, acc[h]);
            acc[h] = fmaf(qh[3], kv.w, acc[h]);
        }
    }
    float s = 0.f;
#pragma unroll
    for (int h = 0; h < H_I; ++h) s = fmaf(sw[h], fmaxf(acc[h], 0.f), s);
    a.scores[(size_t)t * a.ld + j] = s;
}

// Register-tiled form for d_I = 128 and H_I >= 16: a small GEMM per query (block keys x heads)
// followed by the ReLU-weighted head sum.  CTA = 64 block keys of one query; thread
// (kg = tid / 16, hg = tid % 16) accumulates 4 keys x H_I/16 heads over d = 0..127 in order,
// from d-major shared-memory copies of the block keys and the query (two 16-byte loads per
// 4 x H_I/16 FMAs).  Each thread then sums w_h * ReLU over its heads in order, and the 16
// threads of a key group combine their sums with a fixed xor butterfly.
constexpr int kTk = 64;             // block keys per CTA
constexpr int kTThreads = 256;

template <int H_I>
__global__ void __launch_bounds__(kTThreads) block_score_tiled_kernel(BlockScoreArgs a) {
    constexpr int D = 128, HT = H_I / 16, QS = H_I + 4, KS = kTk + 4;   // padded d-major strides
    extern __shared__ float sm[];
    float* sq = sm;                  // [D][QS]: query, d-major
    float* sk = sq + D * QS;         // [D][KS]: block keys, d-major
    float* sw = sk + D * KS;         // [H_I]
    const int t = blockIdx.y, j0 = blockIdx.x * kTk, tid = threadIdx.x;
    const int b = a.q_seq[t], pos = a.q_pos[t];
    bool ok = b >= 0 && b < a.B;
    const int len = ok ? a.seq_len[b] : 0;
    ok = ok && len >= 1 && len <= a.L_alloc && pos >= 0 && pos < len;
    if (!ok && blockIdx.x == 0 && tid == 0) report(a.status, LSA_ERR_DEVICE_DATA);
    const int n_vis = ok ? pos / a.block_size + 1 : 0;            // blocks whose first token <= pos
    if (j0 >= n_vis) {
        for (int i = tid; i < kTk; i += kTThreads)
            if (j0 + i < a.n_cols) a.scores[(size_t)t * a.ld + j0 + i] = kNegInf;
        return;
    }
    // Shared-memory fills, every load of a thread issued before its stores.  Query: item i =
    // (8-dim chunk i / H_I, head i % H_I), heads across lanes so the transposed stores are
    // conflict-free.  Block keys: item i = (4-dim chunk i / kTk, key i % kTk), likewise.
    constexpr int kQItems = H_I * (D / 8) / kTThreads, kKItems = kTk * (D / 4) / kTThreads;
    uint4 qraw[kQItems];
#pragma unroll
    for (int u = 0; u < kQItems; ++u) {
        const int i = tid + u * kTThreads, h = i % H_I, d8 = i / H_I;
        qraw[u] = *reinterpret_cast<const uint4*>(a.q + ((size_t)t * H_I + h) * D + d8 * 8);
    }
    const float* kb = a.kbar + (size_t)b * a.kbar_seq_stride;
    float4 kraw[kKItems];
#pragma unroll
    for (int u = 0; u < kKItems; ++u) {
        const int i = tid + u * kTThreads, key = i % kTk, d4 = i / kTk;
        const int j = min(j0 + key, n_vis - 1);                    // keys past the visible end: any valid row
        kraw[u] = *reinterpret_cast<const float4*>(kb + (size_t)j * D + d4 * 4);
    }
    for (int i = tid; i < H_I; i += kTThreads) sw[i] = a.w[(size_t)t * H_I + i];
#pragma unroll
    for (int u = 0; u < kQItems; ++u) {
        const int i = tid + u * kTThreads, h = i % H_I, d8 = i / H_I;
        const uint32_t wd[4] = {qraw[u].x, qraw[u].y, qraw[u].z, qraw[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            sq[(d8 * 8 + 2 * e) * QS + h] = bf16_bits_to_float((uint16_t)(wd[e] & 0xffff));
            sq[(d8 * 8 + 2 * e + 1) * QS + h] = bf16_bits_to_float((uint16_t)(wd[e] >> 16));
        }
    }
#pragma unroll
    for (int u = 0; u < kKItems; ++u) {
        const int i = tid + u * kTThreads, key = i % kTk, d4 = i / kTk;
        sk[(d4 * 4 + 0) * KS + key] = kraw[u].x;
        sk[(d4 * 4 + 1) * KS + key] = kraw[u].y;
        sk[(d4 * 4 + 2) * KS + key] = kraw[u].z;
        sk[(d4 * 4 + 3) * KS + key] = kraw[u].w;
    }
    __syncthreads();
    const int kg = tid >> 4, hg = tid & 15;
    float acc[4][HT];
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
        for (int h = 0; h < HT; ++h) acc[k][h] = 0.f;
#pragma unroll 4
    for (int d = 0; d < D; ++d) {
        const float4 kv = *reinterpret_cast<const float4*>(sk + d * KS + kg * 4);
        float qv[HT];
#pragma unroll
        for (int h = 0; h < HT; h += 4) {
            if (HT - h >= 4) {
                const float4 q4 = *reinterpret_cast<const float4*>(sq + d * QS + hg * HT + h);
                qv[h] = q4.x; qv[h + 1] = q4.y; qv[h + 2] = q4.z; qv[h + 3] = q4.w;
            } else {
#pragma unroll
                for (int e = 0; e < HT - h; ++e) qv[h + e] = sq[d * QS + hg * HT + h + e];
            }
        }
#pragma unroll
        for (int h = 0; h < HT; ++h) {
            acc[0][h] = fmaf(qv[h], kv.x, acc[0][h]);
            acc[1][h] = fmaf(qv[h], kv.y, acc[1][h]);
            acc[2][h] = fmaf(qv[h], kv.z, acc[2][h]);
            acc[3][h] = fmaf(qv[h], kv.w, acc[3][h]);
        }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        float sgrp = 0.f;
#pragma unroll
        for (int h = 0; h < HT; ++h) sgrp = fmaf(sw[hg * HT + h], fmaxf(acc[k][h], 0.f), sgrp);
#pragma unroll
        for (int o = 1; o < 16; o <<= 1) sgrp += __shfl_xor_sync(0xffffffffu, sgrp, o);
        const int j = j0 + kg * 4 + k;
        if (hg == 0 && j < a.n_cols) a.scores[(size_t)t * a.ld + j] = j < n_vis ? sgrp : kNegInf;
    }
}

template <int H_I>
static cudaError_t launch_bs_tiled(const BlockScoreArgs& a, cudaStream_t st) {
    const size_t smem = ((size_t)128 * (H_I + 4) + (size_t)128 * (kTk + 4) + H_I) * 4;
    auto kern = block_score_tiled_kernel<H_I>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((a.n_cols + kTk - 1) / kTk, a.T);
    kern<<<grid, kTThreads, smem, st>>>(a);
    return cudaGetLastError();
}

template <int H_I>
static cudaError_t launch_bs_t(const BlockScoreArgs& a, cudaStream_t st) {
    const size_t smem = ((size_t)H_I * a.d_I + H_I) * 4;
    auto kern = block_score_kernel<H_I>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((a.n_cols + kBsThreads - 1) / kBsThreads, a.T);
    kern<<<grid, kBsThreads, smem, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_block_score(const BlockScoreArgs& a, int H_I, cudaStream_t st) {
    if (a.n_cols <= 0 || a.T <= 0) return cudaSuccess;
    if (a.d_I == 128 && a.kbar_seq_stride % 4 == 0 && ((uintptr_t)a.kbar % 16) == 0) {
        switch (H_I) {
            case 16: return launch_bs_tiled<16>(a, st);
            case 32: return launch_bs_tiled<32>(a, st);
            case 64: return launch_bs_tiled<64>(a, st);
            case 128: return launch_bs_tiled<128>(a, st);
        }
    }
    switch (H_I) {
        case 8: return launch_bs_t<8>(a, st);
        case 16: return launch_bs_t<16>(a, st);
        case 32: return launch_bs_t<32>(a, st);
        case 64: return launch_bs_t<64>(a, st);
        case 128: return launch_bs_t<128>(a, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace lsa
