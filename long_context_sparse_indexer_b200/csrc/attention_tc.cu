// Sparse MLA-absorbed attention on the 5th-generation tensor cores (tcgen05).
//
// Same operation as attention.cu (explainer page, section "① LSA": attention reads only
// the selected keys and the sinks; MLA absorbed form: 128 query heads share one 576-dim
// latent row, V = its first 512 dims), restated for sm_100a.
//
// CTA = (split, V half, query token).  The two CTAs of a (split, token) each compute the
// full score tile S = Q K^T (M = 128 heads, K = 576) and accumulate O for their 256 V dims;
// the duplicated QK^T keeps every CTA independent (no cross-CTA exchange) at 1.53x the
// minimum tensor work.
//
//   warps 0..3 : gather -- two groups of two warps, group g fills stage g with the tiles
//                j = g, g+2, ...: the tile's 32 row indices (prefetched one tile ahead) are
//                staged in shared memory, then the rows are copied with 16-byte cp.async into
//                the 128-byte-swizzled K-major layout (FP8 rows are widened to BF16 on the way,
//                exactly); per-row scale and validity.  The two groups overlap their copies.
//   warp 8     : MMA issuer -- S_j = Q K_j^T into TMEM (36 MMAs, N = 32), then after the
//                softmax O += P_j V_j (2 MMAs, N = 256) with P read from TMEM and the same
//                shared-memory tile read as an MN-major B operand.
//   warps 4..7 : softmax -- thread = head (TMEM lane): online max / sum with lazy rescaling
//                of O (only when the running max grows by more than 2^8; warp-uniform, so
//                deterministic), P to TMEM as BF16; finally O / l and lse.
//
// All waits are bounded (2 s); a CTA that gives up reports LSA_ERR_TIMEOUT.
#include "kernels.cuh"
#include "tc.cuh"

namespace lsa {

namespace {

constexpr int kAThreads = 288;
constexpr int kRows = 32;                    // KV rows per tile
constexpr int kD = 576, kDv = 512, kHalf = 256;
constexpr int kAtoms = kD / 64;              // 64-element (128-byte) K atoms
constexpr int kTileBytes = kAtoms * kRows * 128;     // 36 KB
constexpr int kQBytes = kAtoms * 128 * 128;          // 144 KB
constexpr int kGroupThreads = 64;            // threads of one gather group

struct AttnSmem {
    alignas(1024) uint8_t q[kQBytes];
    alignas(1024) uint8_t kv[2][kTileBytes];
    float kscale[2][kRows];
    int valid[2][kRows];
    int rows[2][kRows];
    uint64_t kv_full[2], kv_empty[2], s_full[2], p_full[2], o_done;
    uint32_t tmem_base;
    int abort;
};

template <bool KV_FP8>
__global__ void __launch_bounds__(kAThreads, 1) sparse_attn_tc_kernel(AttnArgs a) {
    extern __shared__ uint8_t smem_raw[];
    AttnSmem& sm = *reinterpret_cast<AttnSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int split = blockIdx.x, half = blockIdx.y, t = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int* abort_flag = &sm.abort;

    const int b = a.q_seq[t];
    int len = 0;
    bool ok = b >= 0 && b < a.B;
    if (ok) { len = a.seq_len[b]; ok = len >= 1 && len <= a.L_alloc; }
    int n = ok ? a.count[t] : 0;
    if (n < 0 || n > a.ld_idx) { ok = false; n = 0; }
    if (!ok && threadIdx.x == 0 && split == 0 && half == 0) report(a.status, LSA_ERR_DEVICE_DATA);
    const int per = (n + a.n_split - 1) / a.n_split;
    const int r_beg = min(n, split * per), r_end = min(n, r_beg + per);
    const int n_tiles = (r_end - r_beg + kRows - 1) / kRows;
    const int32_t* irow = a.idx + (size_t)t * a.ld_idx;
    const uint8_t* kvb = a.kv + (size_t)max(b, 0) * a.kv_seq_b;
    const float* kvs = KV_FP8 ? a.kv_scale + (size_t)max(b, 0) * a.kv_scale_seq : nullptr;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&sm.kv_full[i], kGroupThreads);
            tc::mbar_init(&sm.kv_empty[i], 1);
            tc::mbar_init(&sm.s_full[i], 1);
            tc::mbar_init(&sm.p_full[i], 128);
        }
        tc::mbar_init(&sm.o_done, 1);
        sm.abort = 0;
        tc::fence_barrier_init();
    }
    if (warp == 0) tc::tmem_alloc(&sm.tmem_base, 512);
    // Q (all heads, all 576 dims) -> shared memory, K-major, 128-byte swizzle.
    {
        const uint16_t* qt = a.q + (size_t)t * 128 * kD;
        for (int i = threadIdx.x; i < 128 * (kD / 8); i += kAThreads) {
            const int h = i / (kD / 8), c = i % (kD / 8);
            const int atom = c >> 3, cc = c & 7;
            uint8_t* dst = sm.q + atom * (128 * 128) + h * 128 + ((cc ^ (h & 7)) << 4);
            cp_async16(dst, qt + (size_t)h * kD + c * 8, true);
        }
        cp_async_commit();
        cp_async_wait<0>();
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const uint32_t o_col = tmem, s_col = tmem + 256, p_col = tmem + 320;

    if (warp < 4) {
        // ---------------- gather producers: group g owns stage g and the tiles j = g, g + 2, ...
        const int g = warp >> 1;
        const int gt = threadIdx.x - g * kGroupThreads;          // 0..63
        auto fetch_row = [&](int j) -> int {
            if (j >= n_tiles || gt >= kRows) return -1;
            const int r0 = r_beg + j * kRows;
            return gt < min(kRows, r_end - r0) ? irow[r0 + gt] : -1;
        };
        int nxt = fetch_row(g);
        for (int j = g; j < n_tiles; j += 2) {
            const int cur = nxt;
            nxt = fetch_row(j + 2);                                // prefetch the group's next tile
            if (!tc::mbar_wait(&sm.kv_empty[g], ((j >> 1) + 1) & 1, abort_flag)) break;
            const int r0 = r_beg + j * kRows;
            const int nr = min(kRows, r_end - r0);
            if (gt < kRows) {
                const bool v = cur >= 0 && cur < len;
                if (gt < nr && !v) report(a.status, LSA_ERR_DEVICE_DATA);
                sm.rows[g][gt] = v ? cur : -1;
                sm.valid[g][gt] = v;
                sm.kscale[g][gt] = KV_FP8 ? (v ? kvs[cur] : 0.f) : 1.f;
            }
            asm volatile("bar.sync %0, %1;" :: "r"(1 + g), "r"(kGroupThreads) : "memory");
            uint8_t* tile = sm.kv[g];
            if (!KV_FP8) {
                for (int i = gt; i < kRows * (kD / 8); i += kGroupThreads) {
                    const int r = i / (kD / 8), c = i % (kD / 8);
                    const int row = sm.rows[g][r];
                    uint8_t* dst = tile + (c >> 3) * (kRows * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4);
                    cp_async16(dst, kvb + (size_t)(row >= 0 ? row : 0) * a.kv_tok_b + c * 16, row >= 0);
                }
                cp_async_commit();
                cp_async_wait<0>();
            } else {
                constexpr int kChunks = kRows * (kD / 16);             // 16 codes per chunk
                constexpr int kBatch = 6;
                for (int i0 = gt; i0 < kChunks; i0 += kGroupThreads * kBatch) {
                    uint4 raw[kBatch];
#pragma unroll
                    for (int u = 0; u < kBatch; ++u) {
                        const int i = i0 + u * kGroupThreads;
                        raw[u] = make_uint4(0, 0, 0, 0);
                        if (i < kChunks) {
                            const int row = sm.rows[g][i / (kD / 16)];
                            if (row >= 0) raw[u] = ldg_nc16(kvb + (size_t)row * a.kv_tok_b + (i % (kD / 16)) * 16);
                        }
                    }
#pragma unroll
                    for (int u = 0; u < kBatch; ++u) {
                        const int i = i0 + u * kGroupThreads;
                        if (i >= kChunks) break;
                        const int r = i / (kD / 16), c = i % (kD / 16);
                        const uint32_t* wd = reinterpret_cast<const uint32_t*>(&raw[u]);
                        uint32_t ow[8];
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            ow[2 * q] = e4m3x2_to_bf16x2((uint16_t)(wd[q] & 0xffff));
                            ow[2 * q + 1] = e4m3x2_to_bf16x2((uint16_t)(wd[q] >> 16));
                        }
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const int cb = 2 * c + hh;                  // bf16 chunk index (8 dims)
                            uint8_t* dst = tile + (cb >> 3) * (kRows * 128) + r * 128 + (((cb & 7) ^ (r & 7)) << 4);
                            *reinterpret_cast<uint4*>(dst) =
                                make_uint4(ow[4 * hh], ow[4 * hh + 1], ow[4 * hh + 2], ow[4 * hh + 3]);
                        }
                    }
                }
            }
            tc::fence_proxy_async_smem();
            tc::mbar_arrive(&sm.kv_full[g]);
        }
    } else if (warp == 8) {
        // ---------------- MMA issuer
        const uint32_t idesc_s = tc::idesc_f16(128, kRows, 1);
        const uint32_t idesc_o = tc::idesc_f16_bmn(128, kHalf, 1);
        const uint32_t qaddr = tc::smem_u32(sm.q);
        if (tc::elect_one() && n_tiles > 0) {
            auto issue_s = [&](int j) -> bool {
                const int s = j & 1;
                if (!tc::mbar_wait(&sm.kv_full[s], (j >> 1) & 1, abort_flag)) return false;
                tc::fence_proxy_async_smem();
                tc::tc_fence_after();
                const uint32_t kaddr = tc::smem_u32(sm.kv[s]);
#pragma unroll 4
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint64_t ad = tc::sdesc_sw128(qaddr + (kk >> 2) * (128 * 128) + (kk & 3) * 32);
                    const uint64_t bd = tc::sdesc_sw128(kaddr + (kk >> 2) * (kRows * 128) + (kk & 3) * 32);
                    tc::mma_f16_ss(s_col + s * 32, ad, bd, idesc_s, kk > 0);
                }
                tc::mma_commit(&sm.s_full[s]);
                return true;
            };
            int last_pv = -1;
            bool alive = issue_s(0);
            for (int j = 0; j < n_tiles && alive; ++j) {
                const int s = j & 1;
                if (j + 1 < n_tiles && !issue_s(j + 1)) break;
                if (!tc::mbar_wait(&sm.p_full[s], (j >> 1) & 1, abort_flag)) break;
                tc::tc_fence_after();
                const uint32_t vaddr = tc::smem_u32(sm.kv[s]) + (4 * half) * (kRows * 128);
#pragma unroll
                for (int kk = 0; kk < kRows / 16; ++kk) {
                    const uint64_t bd = tc::sdesc_sw128_lbo(vaddr + kk * 16 * 128, kRows * 128, 1024);
                    tc::mma_f16_ts(o_col, p_col + s * 16 + kk * 8, bd, idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
                }
                tc::mma_commit(&sm.kv_empty[s]);
                tc::mma_commit(&sm.o_done);
                last_pv = j;
            }
            if (last_pv >= 0) {                          // drain before TMEM is freed
                volatile int drain_abort = 0;
                tc::mbar_wait(&sm.o_done, last_pv & 1, &drain_abort);
            }
        }
    } else {
        // ---------------- softmax / epilogue: thread = head = TMEM lane
        const int quarter = warp & 3;
        const int h = quarter * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        float m_run = kNegInf, l_run = 0.f;
        bool alive = true;
        for (int j = 0; j < n_tiles; ++j) {
            const int s = j & 1;
            if (!tc::mbar_wait(&sm.s_full[s], (j >> 1) & 1, abort_flag)) { alive = false; break; }
            // The tile's row scales / validity were written by the gather warps before kv_full.
            if (!tc::mbar_wait(&sm.kv_full[s], (j >> 1) & 1, abort_flag)) { alive = false; break; }
            tc::tc_fence_after();
            uint32_t sv[32];
            tc::tmem_ld32(s_col + s * 32 + lane_off, sv);
            tc::tmem_wait_ld();
            if (j > 0 && !tc::mbar_wait(&sm.o_done, (j - 1) & 1, abort_flag)) { alive = false; break; }
            float x[32];
            float mt = kNegInf;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                x[i] = sm.valid[s][i] ? __uint_as_float(sv[i]) * sm.kscale[s][i] * a.sm_scale_log2 : kNegInf;
                mt = fmaxf(mt, x[i]);
            }
            float alpha = 1.f;
            bool rescale = false;
            if (mt > m_run + 8.f) {
                if (m_run != kNegInf) { alpha = exp2f(m_run - mt); rescale = true; }
                l_run *= alpha;
                m_run = mt;
            }
            uint32_t pw[16];
            float ls = 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float p0 = m_run == kNegInf ? 0.f : exp2f(x[2 * i] - m_run);
                const float p1 = m_run == kNegInf ? 0.f : exp2f(x[2 * i + 1] - m_run);
                ls += p0;
                ls += p1;
                pw[i] = pack_bf16x2(p0 * sm.kscale[s][2 * i], p1 * sm.kscale[s][2 * i + 1]);
            }
            l_run += ls;
            tc::tmem_st16(p_col + s * 16 + lane_off, pw);
            if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
                for (int c = 0; c < kHalf / 32; ++c) {
                    uint32_t ov[32];
                    tc::tmem_ld32(o_col + c * 32 + lane_off, ov);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
                    tc::tmem_st32(o_col + c * 32 + lane_off, ov);
                }
            }
            tc::tmem_wait_st();
            tc::tc_fence_before();
            tc::mbar_arrive(&sm.p_full[s]);
        }
        // Epilogue: O / l, lse.
        if (alive && n_tiles > 0 && !tc::mbar_wait(&sm.o_done, (n_tiles - 1) & 1, abort_flag)) alive = false;
        tc::tc_fence_after();
        const float kLn2 = 0.69314718055994530942f;
        const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
        const float lse = l_run > 0.f ? (m_run + log2f(l_run)) * kLn2 : kNegInf;
        const int dv0 = half * kHalf;
        for (int c = 0; c < kHalf / 32; ++c) {
            uint32_t ov[32];
            if (n_tiles > 0 && alive) {
                tc::tmem_ld32(o_col + c * 32 + lane_off, ov);
                tc::tmem_wait_ld();
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) ov[i] = 0u;
            }
            if (a.n_split == 1) {
                uint16_t* orow = a.o + ((size_t)t * 128 + h) * kDv + dv0 + c * 32;
#pragma unroll
                for (int i = 0; i < 32; i += 8) {
                    uint4 pk;
                    pk.x = pack_bf16x2(__uint_as_float(ov[i]) * inv, __uint_as_float(ov[i + 1]) * inv);
                    pk.y = pack_bf16x2(__uint_as_float(ov[i + 2]) * inv, __uint_as_float(ov[i + 3]) * inv);
                    pk.z = pack_bf16x2(__uint_as_float(ov[i + 4]) * inv, __uint_as_float(ov[i + 5]) * inv);
                    pk.w = pack_bf16x2(__uint_as_float(ov[i + 6]) * inv, __uint_as_float(ov[i + 7]) * inv);
                    *reinterpret_cast<uint4*>(orow + i) = pk;
                }
            } else {
                float* prow = a.part_o + (((size_t)t * a.n_split + split) * 128 + h) * kDv + dv0 + c * 32;
#pragma unroll
                for (int i = 0; i < 32; i += 4)
                    *reinterpret_cast<float4*>(prow + i) =
                        make_float4(__uint_as_float(ov[i]) * inv, __uint_as_float(ov[i + 1]) * inv,
                                    __uint_as_float(ov[i + 2]) * inv, __uint_as_float(ov[i + 3]) * inv);
            }
        }
        if (half == 0) {
            if (a.n_split == 1) { if (a.lse) a.lse[(size_t)t * 128 + h] = lse; }
            else a.part_lse[((size_t)t * a.n_split + split) * 128 + h] = lse;
        }
    }

    tc::tc_fence_before();
    __syncthreads();
    if (sm.abort && threadIdx.x == 0) report(a.status, LSA_ERR_TIMEOUT);
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, 512);
    }
}

template <bool KV_FP8>
cudaError_t launch_t(const AttnArgs& a, cudaStream_t st) {
    const size_t smem = sizeof(AttnSmem) + 1024;
    auto kern = sparse_attn_tc_kernel<KV_FP8>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(a.n_split, 2, a.T);
    kern<<<grid, kAThreads, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

bool sparse_attn_tc_supported(const AttnArgs& a, int DQK, int DV, bool sep_v) {
    return DQK == kD && DV == kDv && !sep_v && a.H == 128 && (a.kv_tok_b % 16) == 0 && (a.kv_seq_b % 16) == 0 &&
           ((uintptr_t)a.kv % 16) == 0 && ((uintptr_t)a.q % 16) == 0;
}

cudaError_t launch_sparse_attn_tc(const AttnArgs& a, bool kv_fp8, cudaStream_t st) {
    return kv_fp8 ? launch_t<true>(a, st) : launch_t<false>(a, st);
}

}  // namespace lsa
