// Hierarchical indexing (HI), coarse stage: block keys and block scores.
//
// LongCat-2.0 release post, section "LongCat 稀疏注意力", HI bullet: a coarse-to-fine,
// two-stage scoring -- block-level approximate scores recall candidate blocks, then a
// fine token-level selection runs inside the recalled candidates.  The pages do not say
// how a block is summarised; the block key here is the arithmetic mean of the block's
// dequantised indexer keys, and the block score is the indexer formula applied to it.
//
// Storage of a block key.  The FP32 mean m is kept as the unevaluated sum of two BF16 values,
// hi = rn_bf16(m) and lo = rn_bf16(m - hi) (m - hi is exact in FP32), i.e. 16 significant bits,
// relative error at most 2^-17, in the same 4 bytes per dimension as FP32.  Row j of a sequence
// holds hi[0..d_I) followed by lo[0..d_I).  The block scores then run on the tensor cores
// (row_score_tc.cu) as one BF16 MMA chain over K = 2 d_I: the block-key row [hi | lo] against the
// query row [q | q].  Products of two BF16 values are exact in FP32, so q . (hi + lo) is formed
// with FP32 accumulation only, as a CUDA-core FP32 dot product would.
#include "kernels.cuh"

namespace lsa {

// One CTA per (block, sequence); thread d sums dimension d over the block's rows with a
// fixed pairwise tree (binary-counter order), divides by the row count and stores the
// (hi, lo) split of the mean.
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
    const float m = tot / (float)n;
    const __nv_bfloat16 hi = __float2bfloat16_rn(m);
    const __nv_bfloat16 lo = __float2bfloat16_rn(m - __bfloat162float(hi));
    uint16_t* row = a.kbar + (size_t)b * a.kbar_seq_stride + (size_t)j * 2 * a.d_I;
    row[d] = __bfloat16_as_ushort(hi);
    row[a.d_I + d] = __bfloat16_as_ushort(lo);
}

cudaError_t launch_block_keys(const BlockKeyArgs& a, cudaStream_t st) {
    const int nblk = (a.L_alloc + a.block_size - 1) / a.block_size;
    dim3 grid(nblk, a.B);
    block_keys_kernel<<<grid, a.d_I, 0, st>>>(a);
    return cudaGetLastError();
}

// Validity of query token t for the block scores: its sequence, and the number of blocks whose
// first token it sees (0 when the token is invalid; the caller reports that).
__device__ __forceinline__ int visible_blocks(const BlockScoreArgs& a, int t, int* seq) {
    const int b = a.q_seq[t], pos = a.q_pos[t];
    *seq = b;
    if (b < 0 || b >= a.B) return -1;
    const int len = a.seq_len[b];
    if (len < 1 || len > a.L_alloc || pos < 0 || pos >= len) return -1;
    return pos / a.block_size + 1;
}

// ---------------------------------------------------------------- CUDA-core form (layouts TMA cannot read)

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
    int b;
    const int n_vis = visible_blocks(a, t, &b);
    if (n_vis < 0) {
        if (j == 0) report(a.status, LSA_ERR_DEVICE_DATA);
        a.scores[(size_t)t * a.ld + j] = kNegInf;
        return;
    }
    if (j >= n_vis) { a.scores[(size_t)t * a.ld + j] = kNegInf; return; }
    const uint16_t* kr = a.kbar + (size_t)b * a.kbar_seq_stride + (size_t)j * 2 * a.d_I;
    float acc[H_I];
#pragma unroll
    for (int h = 0; h < H_I; ++h) acc[h] = 0.f;
    for (int d0 = 0; d0 < a.d_I; d0 += 8) {
        const uint4 hv = *reinterpret_cast<const uint4*>(kr + d0);
        const uint4 lv = *reinterpret_cast<const uint4*>(kr + a.d_I + d0);
        const uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w}, lw[4] = {lv.x, lv.y, lv.z, lv.w};
        float kv[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            kv[2 * e] = bf16_bits_to_float((uint16_t)(hw[e] & 0xffff)) + bf16_bits_to_float((uint16_t)(lw[e] & 0xffff));
            kv[2 * e + 1] = bf16_bits_to_float((uint16_t)(hw[e] >> 16)) + bf16_bits_to_float((uint16_t)(lw[e] >> 16));
        }
#pragma unroll
        for (int h = 0; h < H_I; ++h) {
            const float* qh = sq + h * a.d_I + d0;
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[h] = fmaf(qh[e], kv[e], acc[h]);
        }
    }
    float s = 0.f;
#pragma unroll
    for (int h = 0; h < H_I; ++h) s = fmaf(sw[h], fmaxf(acc[h], 0.f), s);
    a.scores[(size_t)t * a.ld + j] = s;
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
    // Tensor cores (row_score_tc.cu) when the block keys and the queries allow TMA.
    RowScoreArgs r{};
    r.seq_len = a.seq_len; r.q_seq = a.q_seq; r.q_pos = a.q_pos;
    r.B = a.B; r.T = a.T; r.L_alloc = a.L_alloc; r.q_group = a.q_group;
    r.q = a.q; r.w = a.w; r.H_I = H_I; r.d_I = a.d_I; r.halves = 2; r.row_span = a.block_size;
    r.scores = a.scores; r.ld = a.ld; r.n_cols = a.n_cols; r.status = a.status;
    if (a.kbar_seq_stride >= (int64_t)a.L_blocks * 2 * a.d_I &&
        row_score_tc_supported(r, 2 * a.d_I, 4 * a.d_I, a.kbar_seq_stride * 2, a.kbar))
        return launch_row_score_tc(r, a.L_blocks, 4 * a.d_I, a.kbar_seq_stride * 2, a.kbar, st);
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
