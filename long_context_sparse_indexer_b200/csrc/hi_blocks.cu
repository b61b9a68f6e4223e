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
// holds hi[0..d_I) followed by lo[0..d_I).  The block score then runs on the tensor cores as one
// BF16 MMA chain over K = 2 d_I: the block-key row [hi | lo] against the query row [q | q].
// Products of two BF16 values are exact in FP32, so q . (hi + lo) is formed with FP32
// accumulation only, as a CUDA-core FP32 dot product would.
#include <cstring>

#include "kernels.cuh"
#include "tc.cuh"

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

// ---------------------------------------------------------------- CUDA-core form (small H_I)

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

// ---------------------------------------------------------------- tensor-core form
//
// CTA = 128 block keys (one M = 128 MMA tile) x one group of G query tokens of one sequence
// (N = G * H_I query-head rows share every block key).  128 threads:
//   set-up : thread 0 initialises the barriers and issues the TMA loads -- the block-key tile as
//            2 d_I / 64 boxes of 128 rows x 128 bytes (128-byte swizzle: the K-major operand
//            layout), the group's query rows as d_I / 64 boxes of N rows x 128 bytes; warp 0
//            allocates N TMEM columns; every thread stages the head weights.
//   MMA    : one thread issues 2 d_I / 16 tcgen05.mma kind::f16 (BF16, M = 128, N, K = 16) --
//            K steps 0 .. d_I/16 - 1 against the hi half of the tile, the rest against the lo
//            half, the query operand the same for both -- and commits to an mbarrier.
//   epilog : thread r = TMEM lane r = block key j0 + r: per token, H_I accumulator columns,
//            ReLU, weighted head sum (eight partial sums combined in a fixed order), store.
// Several CTAs share an SM (80 KB of shared memory at N = 64, d_I = 128), so one CTA's loads
// overlap another's MMA and epilogue.  All waits are bounded; a CTA that gives up reports
// LSA_ERR_TIMEOUT after its copies and MMAs in flight have landed, and frees its TMEM.

constexpr int kBtThreads = 128;
constexpr int kBtRows = 128;            // block keys per CTA (M)
constexpr int kBtMaxG = 4;

struct BtArgs {
    BlockScoreArgs a;
    int G, H_I;
};

template <int N, int D>
struct BtSmem {
    alignas(1024) uint8_t key[2 * D / 64][kBtRows * 128];   // [hi atoms..., lo atoms...], SW128
    alignas(1024) uint8_t q[D / 64][N * 128];               // query rows, SW128
    alignas(16) float w[N];
    int nvis[kBtMaxG];
    int seq[kBtMaxG];
    uint64_t full, done;
    uint32_t tmem_base;
    int abort;
    int issued;                                             // the MMAs were issued (and committed)
};

template <int N, int D>
__global__ void __launch_bounds__(kBtThreads)
block_score_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap, BtArgs pa) {
    using Smem = BtSmem<N, D>;
    constexpr int kKeyAtoms = 2 * D / 64, kQAtoms = D / 64, kKSteps = 2 * D / 16;
    constexpr uint32_t kTxBytes = kKeyAtoms * kBtRows * 128 + kQAtoms * N * 128;
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const BlockScoreArgs& a = pa.a;
    const int G = pa.G, H_I = pa.H_I;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int t0 = blockIdx.y * G, j0 = blockIdx.x * kBtRows;
    volatile int* abort_flag = &sm.abort;

    if (tid < G) {
        int b;
        int nv = visible_blocks(a, t0 + tid, &b);
        if (nv >= 0 && tid > 0 && b != a.q_seq[t0]) nv = -1;       // a group shares one sequence
        if (nv < 0 && blockIdx.x == 0) report(a.status, LSA_ERR_DEVICE_DATA);
        sm.nvis[tid] = max(nv, 0);
        sm.seq[tid] = b;
    }
    if (tid == 0) {
        tc::mbar_init(&sm.full, 1);
        tc::mbar_init(&sm.done, 1);
        sm.abort = 0;
        sm.issued = 0;
        tc::fence_barrier_init();
    }
    __syncthreads();
    int nvis_max = 0;
    for (int g = 0; g < G; ++g) nvis_max = max(nvis_max, sm.nvis[g]);
    if (j0 >= nvis_max) {                              // no visible block in this tile: -inf
        for (int g = 0; g < G; ++g)
            if (j0 + tid < a.n_cols) a.scores[(size_t)(t0 + g) * a.ld + j0 + tid] = kNegInf;
        return;
    }
    const int bseq = min(max(sm.seq[0], 0), a.B - 1);
    if (warp == 0) {
        if (tc::elect_one()) {
            tc::prefetch_tmap(&kmap);
            tc::prefetch_tmap(&qmap);
            tc::mbar_expect_tx(&sm.full, kTxBytes);
#pragma unroll
            for (int i = 0; i < kKeyAtoms; ++i) tc::tma_load_3d(sm.key[i], &kmap, &sm.full, 64 * i, j0, bseq);
#pragma unroll
            for (int i = 0; i < kQAtoms; ++i) tc::tma_load_2d(sm.q[i], &qmap, &sm.full, 64 * i, t0 * H_I);
        }
        __syncwarp();
        tc::tmem_alloc(&sm.tmem_base, N);
    }
    for (int n = tid; n < N; n += kBtThreads) sm.w[n] = a.w[(size_t)t0 * H_I + n];
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == 0) {
        if (tc::elect_one()) {
            if (tc::mbar_wait(&sm.full, 0, abort_flag, a.wait_ns)) {
                tc::tc_fence_after();
                const uint32_t idesc = tc::idesc_f16(128, N, 1);      // bf16 x bf16 -> f32, K-major
#pragma unroll
                for (int k = 0; k < kKSteps; ++k) {
                    const uint64_t da = tc::sdesc_sw128(tc::smem_u32(sm.key[k / 4])) + 2 * (k & 3);
                    const uint64_t db = tc::sdesc_sw128(tc::smem_u32(sm.q[(k % (D / 16)) / 4])) + 2 * (k & 3);
                    tc::mma_f16_ss(tmem, da, db, idesc, k > 0);
                }
                tc::mma_commit(&sm.done);
                sm.issued = 1;
            } else {
                // The loads never completed in time: wait (bounded) for them before the CTA exits.
                volatile int drain_abort = 0;
                tc::mbar_wait(&sm.full, 0, &drain_abort);
            }
        }
        __syncwarp();
    }
    const bool ok = tc::mbar_wait(&sm.done, 0, abort_flag, a.wait_ns);
    if (ok) {
        tc::tc_fence_after();
        const int j = j0 + tid;
        const uint32_t lane_tm = tmem + ((uint32_t)(warp * 32) << 16);
        for (int g = 0; g < G; ++g) {
            float part[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) part[i] = 0.f;
            for (int h0 = 0; h0 < H_I; h0 += 32) {
                uint32_t v[32];
                tc::tmem_ld32(lane_tm + g * H_I + h0, v);
                tc::tmem_wait_ld();
                const float* wr = sm.w + g * H_I + h0;
#pragma unroll
                for (int i = 0; i < 32; ++i) part[i & 7] = fmaf(wr[i], fmaxf(__uint_as_float(v[i]), 0.f), part[i & 7]);
            }
            const float tot = ((part[0] + part[1]) + (part[2] + part[3])) + ((part[4] + part[5]) + (part[6] + part[7]));
            if (j < a.n_cols) a.scores[(size_t)(t0 + g) * a.ld + j] = j < sm.nvis[g] ? tot : kNegInf;
        }
    }
    __syncthreads();
    if (!ok && warp == 0 && sm.issued) {
        // Gave up while the MMAs were in flight: they complete before TMEM is freed (bounded).
        volatile int drain_abort = 0;
        tc::mbar_wait(&sm.done, 0, &drain_abort);
    }
    tc::tc_fence_before();
    __syncthreads();
    if (sm.abort && tid == 0) report(a.status, LSA_ERR_TIMEOUT);
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, N);
    }
}

template <int N, int D>
static cudaError_t launch_bt(const CUtensorMap& km, const CUtensorMap& qm, const BtArgs& pa, cudaStream_t st) {
    const size_t smem = sizeof(BtSmem<N, D>) + 1024;
    auto kern = block_score_tc_kernel<N, D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((pa.a.n_cols + kBtRows - 1) / kBtRows, pa.a.T / pa.G);
    kern<<<grid, kBtThreads, smem, st>>>(km, qm, pa);
    return cudaGetLastError();
}

static int bt_group(const BlockScoreArgs& a, int H_I) {
    int G = a.q_group % 4 == 0 ? 4 : (a.q_group % 2 == 0 ? 2 : 1);
    while (G > 1 && G * H_I > 256) G >>= 1;
    return G;
}

// Tensor-core form when the shapes and the alignment of the block keys and the queries allow
// TMA (16-byte aligned bases, 16-byte multiple strides) and the encoder is available.
static cudaError_t launch_block_score_tc(const BlockScoreArgs& a, int H_I, cudaStream_t st, bool* used) {
    *used = false;
    if ((a.d_I != 64 && a.d_I != 128) || H_I % 32 != 0 || H_I > 256) return cudaSuccess;
    const int G = bt_group(a, H_I), N = G * H_I;
    if (a.T % G != 0 || (N != 32 && N != 64 && N != 128 && N != 256)) return cudaSuccess;
    if ((uintptr_t)a.kbar % 16 || (a.kbar_seq_stride * 2) % 16 || (uintptr_t)a.q % 16) return cudaSuccess;
    if (a.kbar_seq_stride < (int64_t)a.L_blocks * 2 * a.d_I || tc::encode_tiled() == nullptr) return cudaSuccess;
    CUtensorMap km, qm;
    const cuuint64_t kdims[3] = {(cuuint64_t)(2 * a.d_I), (cuuint64_t)a.L_blocks, (cuuint64_t)a.B};
    const cuuint64_t kstr[2] = {(cuuint64_t)(4 * a.d_I), (cuuint64_t)a.kbar_seq_stride * 2};
    const cuuint32_t kbox[3] = {64, kBtRows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = tc::encode_tiled()(&km, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<uint16_t*>(a.kbar), kdims, kstr,
                                    kbox, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaSuccess;
    const cuuint64_t qdims[2] = {(cuuint64_t)a.d_I, (cuuint64_t)a.T * H_I};
    const cuuint64_t qstr[1] = {(cuuint64_t)a.d_I * 2};
    const cuuint32_t qbox[2] = {64, (cuuint32_t)N};
    r = tc::encode_tiled()(&qm, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<uint16_t*>(a.q), qdims, qstr, qbox, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaSuccess;
    BtArgs pa{a, G, H_I};
    pa.a.wait_ns = wait_limit_ns();
    *used = true;
    if (a.d_I == 128) {
        switch (N) {
            case 32: return launch_bt<32, 128>(km, qm, pa, st);
            case 64: return launch_bt<64, 128>(km, qm, pa, st);
            case 128: return launch_bt<128, 128>(km, qm, pa, st);
            case 256: return launch_bt<256, 128>(km, qm, pa, st);
        }
    } else {
        switch (N) {
            case 32: return launch_bt<32, 64>(km, qm, pa, st);
            case 64: return launch_bt<64, 64>(km, qm, pa, st);
            case 128: return launch_bt<128, 64>(km, qm, pa, st);
            case 256: return launch_bt<256, 64>(km, qm, pa, st);
        }
    }
    *used = false;
    return cudaSuccess;
}

cudaError_t launch_block_score(const BlockScoreArgs& a, int H_I, cudaStream_t st) {
    if (a.n_cols <= 0 || a.T <= 0) return cudaSuccess;
    bool used = false;
    cudaError_t e = launch_block_score_tc(a, H_I, st, &used);
    if (used || e != cudaSuccess) return e;
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
