// Indexer-form scores of BF16 rows on the tensor cores:
//   S(t, j) = sum_h w[t,h] * ReLU(q[t,h,:] . row_j)
// for two kinds of rows (LongCat-2.0 release post, section "LongCat 稀疏注意力": the lightweight
// indexer, DSA form; HI bullet: block-level approximate scores):
//   * HI block keys (halves = 2): row j = [hi | lo], the block key split into two BF16 values
//     (see hi_blocks.cu); the MMA chain runs over K = 2 d_I, the query row used for both halves,
//     so the accumulator holds q . (hi + lo).  Row j is visible when j * block_size <= q_pos.
//   * BF16 indexer keys (halves = 1): row j = the key of position j; visible when j <= q_pos.
// Products of two BF16 values are exact in FP32: the only rounding is the FP32 accumulation.
//
// CTA = 128 rows (one M = 128 MMA tile) x one group of G query tokens of one sequence, N = G * H_I
// query-head rows padded to at least 32 (padded rows carry weight 0 and are never read back).
// 128 threads:
//   set-up : thread 0 initialises the barriers and issues the TMA loads -- the row tile as
//            halves * d_I / 64 boxes of 128 rows x 128 bytes (128-byte swizzle: the K-major operand
//            layout), the group's query rows as d_I / 64 boxes of N rows x 128 bytes; warp 0
//            allocates N TMEM columns; every thread stages the head weights.
//   MMA    : one thread issues halves * d_I / 16 tcgen05.mma kind::f16 (BF16, M = 128, N, K = 16)
//            and commits to an mbarrier.
//   epilog : thread r = TMEM lane r = row j0 + r: per token, its H_I accumulator columns, ReLU,
//            weighted head sum (eight partial sums combined in a fixed order), store.
// Several CTAs share an SM (80 KB of shared memory for 128 block keys at N = 64, d_I = 128), so
// one CTA's loads overlap another's MMA and epilogue.  All waits are bounded; a CTA that gives
// up reports LSA_ERR_TIMEOUT after its copies and MMAs in flight have landed, and frees its TMEM.
#include <cstring>

#include "kernels.cuh"
#include "tc.cuh"

namespace lsa {

namespace {

constexpr int kRsThreads = 128;
constexpr int kRsRows = 128;             // rows per CTA (M)
constexpr int kRsMaxG = 4;

struct RsArgs {
    RowScoreArgs a;
    int G, N;                            // tokens per CTA, query rows of the MMA (>= G * H_I)
};

template <int N, int D, int KH>
struct RsSmem {
    alignas(1024) uint8_t rows[KH * D / 64][kRsRows * 128];   // row atoms (KH = 2: hi atoms, then lo atoms)
    alignas(1024) uint8_t q[D / 64][N * 128];                 // query rows, SW128
    alignas(16) float w[N];
    int nvis[kRsMaxG];
    int seq[kRsMaxG];
    uint64_t full, done;
    uint32_t tmem_base;
    int abort;
    int issued;                                               // the MMAs were issued (and committed)
};

// 32 lanes x 8 columns of 32-bit: thread i of the warp holds lane (base + i), 8 columns.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
}

// Rows of token t it sees (j * row_span <= q_pos), or -1 for an invalid token; its sequence.
__device__ __forceinline__ int visible_rows(const RowScoreArgs& a, int t, int* seq) {
    const int b = a.q_seq[t], pos = a.q_pos[t];
    *seq = b;
    if (b < 0 || b >= a.B) return -1;
    const int len = a.seq_len[b];
    if (len < 1 || len > a.L_alloc || pos < 0 || pos >= len) return -1;
    return pos / a.row_span + 1;
}

template <int N, int D, int KH>
__global__ void __launch_bounds__(kRsThreads)
row_score_tc_kernel(const __grid_constant__ CUtensorMap rmap, const __grid_constant__ CUtensorMap qmap, RsArgs pa) {
    using Smem = RsSmem<N, D, KH>;
    constexpr int kRowAtoms = KH * D / 64, kQAtoms = D / 64, kKSteps = KH * D / 16;
    constexpr uint32_t kTxBytes = kRowAtoms * kRsRows * 128 + kQAtoms * N * 128;
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const RowScoreArgs& a = pa.a;
    const int G = pa.G, H_I = a.H_I;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int t0 = blockIdx.y * G, j0 = blockIdx.x * kRsRows;
    volatile int* abort_flag = &sm.abort;

    if (tid < G) {
        int b;
        int nv = visible_rows(a, t0 + tid, &b);
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
    if (j0 >= nvis_max) {                              // no visible row in this tile: -inf
        for (int g = 0; g < G; ++g)
            if (j0 + tid < a.n_cols) a.scores[(size_t)(t0 + g) * a.ld + j0 + tid] = kNegInf;
        return;
    }
    const int bseq = min(max(sm.seq[0], 0), a.B - 1);
    if (warp == 0) {
        if (tc::elect_one()) {
            tc::prefetch_tmap(&rmap);
            tc::prefetch_tmap(&qmap);
            tc::mbar_expect_tx(&sm.full, kTxBytes);
#pragma unroll
            for (int i = 0; i < kRowAtoms; ++i) tc::tma_load_3d(sm.rows[i], &rmap, &sm.full, 64 * i, j0, bseq);
#pragma unroll
            for (int i = 0; i < kQAtoms; ++i) tc::tma_load_2d(sm.q[i], &qmap, &sm.full, 64 * i, t0 * H_I);
        }
        __syncwarp();
        tc::tmem_alloc(&sm.tmem_base, N);
    }
    // Query rows past the group's G * H_I (the padding of N) get weight 0.
    for (int n = tid; n < N; n += kRsThreads) sm.w[n] = n < G * H_I ? a.w[(size_t)t0 * H_I + n] : 0.f;
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
                    const uint64_t da = tc::sdesc_sw128(tc::smem_u32(sm.rows[k / 4])) + 2 * (k & 3);
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
            if (H_I % 32 == 0) {
                for (int h0 = 0; h0 < H_I; h0 += 32) {
                    uint32_t v[32];
                    tc::tmem_ld32(lane_tm + g * H_I + h0, v);
                    tc::tmem_wait_ld();
                    const float* wr = sm.w + g * H_I + h0;
#pragma unroll
                    for (int i = 0; i < 32; ++i) part[i & 7] = fmaf(wr[i], fmaxf(__uint_as_float(v[i]), 0.f), part[i & 7]);
                }
            } else {                                   // H_I = 8 or 16: eight columns at a time
                for (int h0 = 0; h0 < H_I; h0 += 8) {
                    uint32_t v[8];
                    tmem_ld8(lane_tm + g * H_I + h0, v);
                    tc::tmem_wait_ld();
                    const float* wr = sm.w + g * H_I + h0;
#pragma unroll
                    for (int i = 0; i < 8; ++i) part[i] = fmaf(wr[i], fmaxf(__uint_as_float(v[i]), 0.f), part[i]);
                }
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

template <int N, int D, int KH>
cudaError_t launch_rs(const CUtensorMap& rm, const CUtensorMap& qm, const RsArgs& pa, cudaStream_t st) {
    const size_t smem = sizeof(RsSmem<N, D, KH>) + 1024;
    auto kern = row_score_tc_kernel<N, D, KH>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((pa.a.n_cols + kRsRows - 1) / kRsRows, pa.a.T / pa.G);
    kern<<<grid, kRsThreads, smem, st>>>(rm, qm, pa);
    return cudaGetLastError();
}

template <int D, int KH>
cudaError_t launch_rs_n(const CUtensorMap& rm, const CUtensorMap& qm, const RsArgs& pa, cudaStream_t st) {
    switch (pa.N) {
        case 32: return launch_rs<32, D, KH>(rm, qm, pa, st);
        case 64: return launch_rs<64, D, KH>(rm, qm, pa, st);
        case 128: return launch_rs<128, D, KH>(rm, qm, pa, st);
        case 256: return launch_rs<256, D, KH>(rm, qm, pa, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

// Query tokens per CTA: 4, 2 or 1 (the largest dividing q_group) with G * H_I <= 256.
int row_score_group(int q_group, int H_I) {
    int G = q_group % 4 == 0 ? 4 : (q_group % 2 == 0 ? 2 : 1);
    while (G > 1 && G * H_I > 256) G >>= 1;
    return G;
}

bool row_score_tc_supported(const RowScoreArgs& a, int row_elems, int64_t row_stride_b, int64_t seq_stride_b,
                            const void* rows) {
    if ((a.d_I != 64 && a.d_I != 128) || (a.halves != 1 && a.halves != 2) || a.H_I % 8 != 0 || a.H_I > 256) return false;
    if (row_elems != a.halves * a.d_I) return false;
    const int G = row_score_group(a.q_group, a.H_I);
    if (a.T % G != 0) return false;
    if ((uintptr_t)rows % 16 || row_stride_b % 16 || seq_stride_b % 16 || (uintptr_t)a.q % 16) return false;
    return tc::encode_tiled() != nullptr;
}

cudaError_t launch_row_score_tc(const RowScoreArgs& a, int n_rows, int64_t row_stride_b, int64_t seq_stride_b,
                                const void* rows, cudaStream_t st) {
    if (a.n_cols <= 0 || a.T <= 0) return cudaSuccess;
    const int G = row_score_group(a.q_group, a.H_I);
    int N = 32;
    while (N < G * a.H_I) N <<= 1;                     // 32, 64, 128 or 256
    CUtensorMap rm, qm;
    const cuuint64_t rdims[3] = {(cuuint64_t)(a.halves * a.d_I), (cuuint64_t)n_rows, (cuuint64_t)a.B};
    const cuuint64_t rstr[2] = {(cuuint64_t)row_stride_b, (cuuint64_t)seq_stride_b};
    const cuuint32_t rbox[3] = {64, kRsRows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = tc::encode_tiled()(&rm, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void*>(rows), rdims, rstr, rbox,
                                    estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    // The query map covers every token's heads; a box of N rows past the last token reads zeros.
    const cuuint64_t qdims[2] = {(cuuint64_t)a.d_I, (cuuint64_t)a.T * a.H_I};
    const cuuint64_t qstr[1] = {(cuuint64_t)a.d_I * 2};
    const cuuint32_t qbox[2] = {64, (cuuint32_t)N};
    r = tc::encode_tiled()(&qm, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<uint16_t*>(a.q), qdims, qstr, qbox, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    RsArgs pa{a, G, N};
    pa.a.wait_ns = wait_limit_ns();
    if (a.halves == 2) return a.d_I == 128 ? launch_rs_n<128, 2>(rm, qm, pa, st) : launch_rs_n<64, 2>(rm, qm, pa, st);
    return a.d_I == 128 ? launch_rs_n<128, 1>(rm, qm, pa, st) : launch_rs_n<64, 1>(rm, qm, pa, st);
}

}  // namespace lsa
