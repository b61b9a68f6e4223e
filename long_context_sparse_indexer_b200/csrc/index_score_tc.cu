// Indexer scores on the 5th-generation tensor cores (tcgen05), FP8 e4m3 keys with d_I = 128.
//
// Same operation as index_score.cu (LongCat-2.0 release post, section "LongCat 稀疏注意力":
// the lightweight indexer scoring every cached key; DSA form sum_h w_h * ReLU(q_h . k)),
// restated for sm_100a.  One CTA owns 2048 score columns of a group of G <= 4 query tokens
// of one sequence, so every key row is read from HBM once per group.
//
//   warp 0      : TMA producer -- 128-key tiles (two 64-row boxes, 128-byte swizzle) and their
//                 per-token scales into a 4-stage shared-memory ring; allocates / frees TMEM.
//   warp 1      : MMA issuer -- per tile, 8 x tcgen05.mma kind::f16 (M = 128 keys, N = G*H_I,
//                 K = 16) with A read from TMEM and B (the queries) from shared memory.
//   warps 2..5  : converters -- thread = key row (= TMEM lane): widen the row's 128 FP8 codes
//                 to f16 (exact) and store them as the A operand in TMEM.
//   warps 6..9  : epilogue -- thread = key row: load the accumulator row (G*H_I scores), apply
//                 ReLU, the weighted head sum (four partial sums combined in a fixed order)
//                 and the token's FP8 scale, store.
//
// Queries are scaled per head by a power of two into f16 range (exact for all values within
// 2^28 of the head's maximum); the inverse power is folded into the head weight.  Products
// of f16 values are exact in the FP32 accumulator.  All waits are bounded (2 s of wall time);
// a CTA that gives up reports LSA_ERR_TIMEOUT and returns after freeing its TMEM.
#include <algorithm>
#include <cstring>
#include <mutex>

#include "kernels.cuh"
#include "tc.cuh"

namespace lsa {

namespace {

constexpr int kTcThreads = 320;
constexpr int kTcCols = 2048;          // score columns per CTA
constexpr int kTile = 128;             // keys per MMA tile
constexpr int kStages = 4;             // key-tile ring
constexpr int kKeyTileBytes = kTile * 128;
constexpr int kMaxG = 4;

struct TcArgs {
    IndexArgs a;
    int G, H_I, N, d_stages, tmem_cols;
    int scale_tma;          // per-token scales arrive by TMA with the keys (else: epilogue reads global)
};

template <int N>
struct TcSmem {
    alignas(1024) uint8_t keys[kStages][kKeyTileBytes];
    alignas(1024) uint8_t q[2][N * 128];          // B operand: two 64-element K atoms, SW128
    alignas(16) float scl[kStages][kTile];        // per-token FP8 scales of each key tile
    alignas(16) float w[N];                       // head weights (inverse query scale folded in)
    uint64_t full_k[kStages], empty_k[kStages];
    uint64_t a_full[2], a_empty[2];
    uint64_t d_full[2], d_empty[2];
    uint32_t tmem_base;
    int pos[kMaxG];
    int ok[kMaxG];
    int abort;
};

template <int N>
__global__ void __launch_bounds__(kTcThreads, (N <= 128 ? 2 : 1))
index_score_tc_kernel(const __grid_constant__ CUtensorMap tmap, const __grid_constant__ CUtensorMap smap,
                      TcArgs ta) {
    extern __shared__ uint8_t smem_raw[];
    TcSmem<N>& sm = *reinterpret_cast<TcSmem<N>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const IndexArgs& a = ta.a;
    const int G = ta.G, H_I = ta.H_I, DS = ta.d_stages;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = blockIdx.y * G;
    const int col_beg = blockIdx.x * kTcCols;
    const int col_end = min(a.n_cols, col_beg + kTcCols);
    const bool hi = a.cand != nullptr;
    volatile int* abort_flag = &sm.abort;

    // ---- set-up: barriers, TMEM, query group validity
    if (threadIdx.x == 0) {
        // A stage is free once the converters have read its keys and the epilogue its scales.
        for (int s = 0; s < kStages; ++s) { tc::mbar_init(&sm.full_k[s], 1); tc::mbar_init(&sm.empty_k[s], 256); }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&sm.a_full[i], 128); tc::mbar_init(&sm.a_empty[i], 1);
            tc::mbar_init(&sm.d_full[i], 1); tc::mbar_init(&sm.d_empty[i], 128);
        }
        sm.abort = 0;
        tc::fence_barrier_init();
        tc::prefetch_tmap(&tmap);
        if (ta.scale_tma) tc::prefetch_tmap(&smap);
    }
    if (warp == 0) tc::tmem_alloc(&sm.tmem_base, ta.tmem_cols);
    const int bseq = a.q_seq[t0];
    if (threadIdx.x < kMaxG) {
        const int gi = threadIdx.x;
        int ok = 0, pos = -1;
        if (gi < G) {
            const int s = a.q_seq[t0 + gi];
            pos = a.q_pos[t0 + gi];
            ok = s == bseq && s >= 0 && s < a.B;
            if (ok) {
                const int len = a.seq_len[s];
                ok = len >= 1 && len <= a.L_alloc && pos >= 0 && pos < len;
            }
            if (!ok) report(a.status, LSA_ERR_DEVICE_DATA);
        }
        sm.pos[gi] = ok ? pos : -1;
        sm.ok[gi] = ok;
    }
    // Queries -> f16, scaled per head, into the 128-byte-swizzled K-major B layout.  Thread i
    // handles 16-byte chunk i (8 elements) of the group's N rows; the 16 chunks of a row sit in
    // 16 consecutive lanes, which reduce the row maximum by shuffles.  All loads of a batch are
    // issued before use.
    {
        constexpr int kQB = 4;
        const int nchunks = N * 16;                       // a multiple of 32
        for (int base = threadIdx.x; base < nchunks; base += kTcThreads * kQB) {
            uint4 raw[kQB];
#pragma unroll
            for (int u = 0; u < kQB; ++u) {
                const int i = base + u * kTcThreads;
                const int rowi = i >> 4;
                raw[u] = i < nchunks ? *reinterpret_cast<const uint4*>(
                                           a.q + ((size_t)(t0 + rowi / H_I) * H_I + rowi % H_I) * 128 + (i & 15) * 8)
                                     : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < kQB; ++u) {
                const int i = base + u * kTcThreads;
                if (i >= nchunks) break;                  // warp-uniform: nchunks is a multiple of 32
                const int rowi = i >> 4, cc = i & 15;
                const uint32_t* wd = reinterpret_cast<const uint32_t*>(&raw[u]);
                float v[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    v[2 * e] = bf16_bits_to_float((uint16_t)(wd[e] & 0xffff));
                    v[2 * e + 1] = bf16_bits_to_float((uint16_t)(wd[e] >> 16));
                }
                float m = 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(v[e]));
#pragma unroll
                for (int o = 1; o < 16; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                const int ex = (int)((__float_as_uint(m) >> 23) & 0xff) - 127;
                int k = m > 0.f ? 14 - ex : 0;
                k = max(-126, min(126, k));
                const float sc = exp2i(k);
                uint32_t hv[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    hv[e] = (uint32_t)__half_as_ushort(__float2half_rn(v[2 * e] * sc)) |
                            ((uint32_t)__half_as_ushort(__float2half_rn(v[2 * e + 1] * sc)) << 16);
                const int atom = cc >> 3, c16 = cc & 7;
                uint8_t* dst = sm.q[atom] + (rowi >> 3) * 1024 + (rowi & 7) * 128 + ((c16 ^ (rowi & 7)) << 4);
                *reinterpret_cast<uint4*>(dst) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
                if (cc == 0) sm.w[rowi] = a.w[(size_t)(t0 + rowi / H_I) * H_I + rowi % H_I] * exp2i(-k);
            }
        }
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const uint32_t a_col = tmem, d_col = tmem + 128;

    int max_pos = -1;
    for (int gi = 0; gi < G; ++gi) max_pos = max(max_pos, sm.pos[gi]);
    // Active tiles: flat mode, the tiles holding a column <= max_pos; HI mode, all.
    int n_active = 0;
    if (col_end > col_beg) {
        const int last = hi ? col_end : min(col_end, max_pos + 1);
        n_active = last > col_beg ? (last - col_beg + kTile - 1) / kTile : 0;
    }

    if (warp == 0) {
        // ---------------- TMA producer
        if (tc::elect_one()) {
            int issued = 0;
            for (int j = 0; j < n_active; ++j) {
                const int s = j % kStages;
                if (!tc::mbar_wait(&sm.empty_k[s], ((j / kStages) + 1) & 1, abort_flag)) break;
                ++issued;
                tc::mbar_expect_tx(&sm.full_k[s], kKeyTileBytes + (ta.scale_tma ? kTile * 4 : 0));
                const int c = col_beg + j * kTile;
                int r0 = c, r1 = c + 64;
                if (hi) {
                    const int nb = a.n_cand;
                    const int b0 = (c / 64) < nb ? a.cand[(size_t)t0 * nb + c / 64] : -1;
                    const int b1 = (c / 64 + 1) < nb ? a.cand[(size_t)t0 * nb + c / 64 + 1] : -1;
                    r0 = b0 >= 0 ? b0 * 64 : 0;
                    r1 = b1 >= 0 ? b1 * 64 : 0;
                }
                tc::tma_load_3d(sm.keys[s], &tmap, &sm.full_k[s], 0, r0, max(bseq, 0));
                tc::tma_load_3d(sm.keys[s] + kKeyTileBytes / 2, &tmap, &sm.full_k[s], 0, r1, max(bseq, 0));
                if (ta.scale_tma) {
                    tc::tma_load_2d(sm.scl[s], &smap, &sm.full_k[s], r0, max(bseq, 0));
                    tc::tma_load_2d(sm.scl[s] + 64, &smap, &sm.full_k[s], r1, max(bseq, 0));
                }
            }
            // Drain: every issued tile has landed before the CTA can exit (bounded; already true
            // unless the consumers gave up early).
            volatile int drain_abort = 0;
            for (int j = max(0, issued - kStages); j < issued; ++j)
                tc::mbar_wait(&sm.full_k[j % kStages], (j / kStages) & 1, &drain_abort);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        const uint32_t idesc = tc::idesc_f16(128, N, 0);
        const uint32_t qaddr0 = tc::smem_u32(sm.q[0]), qaddr1 = tc::smem_u32(sm.q[1]);
        if (tc::elect_one()) {
            int last = -1;
            for (int j = 0; j < n_active; ++j) {
                const int ab = j & 1, db = j % DS;
                if (!tc::mbar_wait(&sm.a_full[ab], (j >> 1) & 1, abort_flag)) break;
                if (!tc::mbar_wait(&sm.d_empty[db], ((j / DS) + 1) & 1, abort_flag)) break;
                tc::tc_fence_after();
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t qa = (k < 4 ? qaddr0 : qaddr1) + (k & 3) * 32;
                    tc::mma_f16_ts(d_col + db * N, a_col + ab * 64 + k * 8, tc::sdesc_sw128(qa), idesc, k > 0);
                }
                tc::mma_commit(&sm.a_empty[ab]);
                tc::mma_commit(&sm.d_full[db]);
                last = j;
            }
            // Drain: the MMAs issued so far have completed before TMEM is freed.
            if (last >= 0) {
                volatile int drain_abort = 0;
                tc::mbar_wait(&sm.d_full[last % DS], (last / DS) & 1, &drain_abort);
            }
        }
    } else if (warp < 6) {
        // ---------------- converters: thread = TMEM lane = key row of the tile
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        for (int j = 0; j < n_active; ++j) {
            const int s = j % kStages, ab = j & 1;
            if (!tc::mbar_wait(&sm.full_k[s], (j / kStages) & 1, abort_flag)) break;
            const uint8_t* rowp = sm.keys[s] + r * 128;          // 128-byte rows, 16-byte chunks XOR-swizzled
            uint4 ch[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) ch[c] = *reinterpret_cast<const uint4*>(rowp + ((c ^ (r & 7)) << 4));
            tc::mbar_arrive(&sm.empty_k[s]);
            if (!tc::mbar_wait(&sm.a_empty[ab], ((j >> 1) + 1) & 1, abort_flag)) break;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t wv[32];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint32_t* wd = reinterpret_cast<const uint32_t*>(&ch[half * 4 + c]);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        wv[c * 8 + 2 * u] = e4m3x2_to_f16x2((uint16_t)(wd[u] & 0xffff));
                        wv[c * 8 + 2 * u + 1] = e4m3x2_to_f16x2((uint16_t)(wd[u] >> 16));
                    }
                }
                tc::tmem_st32(a_col + ab * 64 + half * 32 + lane_off, wv);
            }
            tc::tmem_wait_st();
            tc::tc_fence_before();
            tc::mbar_arrive(&sm.a_full[ab]);
        }
    } else {
        // ---------------- epilogue: thread = TMEM lane = key row of the tile
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const bool fp8 = a.kscale != nullptr;
        for (int j = 0; j < n_active; ++j) {
            const int s = j % kStages, db = j % DS;
            if (!tc::mbar_wait(&sm.full_k[s], (j / kStages) & 1, abort_flag)) break;
            const int col = col_beg + j * kTile + r;
            int row = col;
            if (hi) {
                const int bi = col / 64;
                const int blk = (col < a.n_cols && bi < a.n_cand) ? a.cand[(size_t)t0 * a.n_cand + bi] : -1;
                row = blk >= 0 ? blk * 64 + (col & 63) : -1;
            }
            float ks = 1.f;
            if (fp8) {
                if (ta.scale_tma) ks = sm.scl[s][r];
                else if (row >= 0 && row <= max_pos) ks = a.kscale[(size_t)max(bseq, 0) * a.scale_seq_stride + row];
            }
            tc::mbar_arrive(&sm.empty_k[s]);
            if (!tc::mbar_wait(&sm.d_full[db], (j / DS) & 1, abort_flag)) break;
            tc::tc_fence_after();
            for (int gi = 0; gi < G; ++gi) {
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
                for (int h0 = 0; h0 < H_I; h0 += 32) {
                    uint32_t v[32];
                    tc::tmem_ld32(d_col + db * N + gi * H_I + h0 + lane_off, v);
                    tc::tmem_wait_ld();
                    const float4* wp = reinterpret_cast<const float4*>(sm.w + gi * H_I + h0);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float4 ww = wp[i];
                        acc[0] = fmaf(ww.x, fmaxf(__uint_as_float(v[4 * i + 0]), 0.f), acc[0]);
                        acc[1] = fmaf(ww.y, fmaxf(__uint_as_float(v[4 * i + 1]), 0.f), acc[1]);
                        acc[2] = fmaf(ww.z, fmaxf(__uint_as_float(v[4 * i + 2]), 0.f), acc[2]);
                        acc[3] = fmaf(ww.w, fmaxf(__uint_as_float(v[4 * i + 3]), 0.f), acc[3]);
                    }
                }
                const float total = (acc[0] + acc[1]) + (acc[2] + acc[3]);
                if (col < col_end) {
                    const bool vis = sm.ok[gi] && row >= 0 && row <= sm.pos[gi];
                    a.scores[(size_t)(t0 + gi) * a.ld + col] = vis ? total * ks : kNegInf;
                }
            }
            tc::tc_fence_before();
            tc::mbar_arrive(&sm.d_empty[db]);
        }
        // Columns of the chunk past the active tiles see no visible key.
        for (int col = col_beg + n_active * kTile + r; col < col_end; col += 128)
            for (int gi = 0; gi < G; ++gi) a.scores[(size_t)(t0 + gi) * a.ld + col] = kNegInf;
    }

    tc::tc_fence_before();
    __syncthreads();
    if (sm.abort && threadIdx.x == 0) report(a.status, LSA_ERR_TIMEOUT);
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, ta.tmem_cols);
    }
}

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encode_fn() {
    static EncodeTiled fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiled>(p);
    });
    return fn;
}

template <int N>
cudaError_t launch_n(const CUtensorMap& m, const CUtensorMap& sm, const TcArgs& ta, cudaStream_t st) {
    // At least 80 KB so that no more than two CTAs share an SM: two 256-column TMEM
    // allocations fill the SM's 512 columns (a third CTA would wait for one to finish).
    const size_t smem = std::max(sizeof(TcSmem<N>) + 1024, (size_t)80 * 1024);
    auto kern = index_score_tc_kernel<N>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((ta.a.n_cols + kTcCols - 1) / kTcCols, ta.a.T / ta.G);
    kern<<<grid, kTcThreads, smem, st>>>(m, sm, ta);
    return cudaGetLastError();
}

}  // namespace

bool index_score_tc_supported(const IndexArgs& a, int H_I, int D_I, bool fp8) {
    if (!fp8 || D_I != 128 || H_I % 32 != 0) return false;
    if (a.cand && a.block_size != 64) return false;
    const int G = a.cand ? 1 : (a.q_group % 4 == 0 ? 4 : (a.q_group % 2 == 0 ? 2 : 1));
    const int N = G * H_I;
    if (N > 256) return false;
    return ((uintptr_t)a.kdata % 16 == 0) && (a.tok_stride_b % 16 == 0) && (a.seq_stride_b % 16 == 0) &&
           a.kscale != nullptr && encode_fn() != nullptr;
}

cudaError_t launch_index_score_tc(IndexArgs a, int H_I, cudaStream_t st) {
    if (a.n_cols <= 0 || a.T <= 0) return cudaSuccess;
    TcArgs ta{};
    ta.a = a;
    ta.H_I = H_I;
    ta.G = a.cand ? 1 : (a.q_group % 4 == 0 ? 4 : (a.q_group % 2 == 0 ? 2 : 1));
    while (ta.G * H_I > 256) ta.G >>= 1;
    ta.N = ta.G * H_I;
    ta.d_stages = ta.N <= 192 ? 2 : 1;
    const int need = 128 + ta.d_stages * ta.N;
    ta.tmem_cols = need <= 256 ? 256 : 512;

    CUtensorMap m;
    const cuuint64_t dims[3] = {128, (cuuint64_t)a.L_alloc, (cuuint64_t)a.B};
    const cuuint64_t strides[2] = {(cuuint64_t)a.tok_stride_b, (cuuint64_t)a.seq_stride_b};
    const cuuint32_t box[3] = {128, 64, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = encode_fn()(&m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(a.kdata), dims, strides, box,
                             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    // Per-token scales: [B][L_alloc] floats, boxes of 64 rows (zero fill past the end); TMA needs
    // a 16-byte aligned base and sequence stride, otherwise the epilogue reads them directly.
    ta.scale_tma = ((uintptr_t)a.kscale % 16 == 0) && (a.scale_seq_stride % 4 == 0) && a.B * (int64_t)a.scale_seq_stride > 0;
    CUtensorMap sc;
    memset(&sc, 0, sizeof(sc));
    const cuuint64_t sdims[2] = {(cuuint64_t)a.L_alloc, (cuuint64_t)a.B};
    const cuuint64_t sstr[1] = {(cuuint64_t)a.scale_seq_stride * 4};
    const cuuint32_t sbox[2] = {64, 1};
    const cuuint32_t sestr[2] = {1, 1};
    if (ta.scale_tma) {
        r = encode_fn()(&sc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(a.kscale), sdims, sstr, sbox,
                        sestr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) ta.scale_tma = 0;
    }
    switch (ta.N) {
        case 32: return launch_n<32>(m, sc, ta, st);
        case 64: return launch_n<64>(m, sc, ta, st);
        case 128: return launch_n<128>(m, sc, ta, st);
        case 192: return launch_n<192>(m, sc, ta, st);
        case 256: return launch_n<256>(m, sc, ta, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace lsa
