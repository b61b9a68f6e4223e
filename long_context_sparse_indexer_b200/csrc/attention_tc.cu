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
// Memory plan.  TMEM (512 columns): O half [0,256), three S / P buffers [256,352) -- the
// softmax writes P (BF16, 16 columns) over the S it has just read, so S can run two tiles
// ahead of P V -- and Q dims 256..575 [352,512) as the A operand of the last 20 K-steps of S.  Shared memory: Q dims 0..255 (4 swizzled K atoms, 64 KB) as the A operand of the first
// 16 K-steps, and a 4-stage ring of 32-row KV tiles (36 KB each) in the 128-byte-swizzled
// K-major layout, read as the B operand of S (K-major) and of P V (MN-major).
//
//   warps 0..7 : gather -- warps 2s and 2s+1 fill stage s with the tiles j = s, s+4, ...: the
//                rows' indices (prefetched one tile ahead) and per-row scale and validity go
//                to shared memory; the two CTAs of a (split, token) form a cluster and each
//                copies only its half of the rows (16-byte cp.async; FP8 rows widened to BF16
//                exactly on the way), pushing them into the peer's stage with bulk
//                shared-to-shared copies, so each row crosses into the SMs once.
//   warp 12    : MMA issuer -- issues whatever is ready, in order per kind: S_j (16 SS + 20 TS
//                MMAs, N = 32) once tile j has landed and P V_{j-3} has been issued, and
//                O += P_j V_j (2 TS MMAs, N = 256) once the softmax of tile j is done.
//   warps 8..11: softmax -- thread = head (TMEM lane): online max / sum with lazy rescaling
//                of O (only when the running max grows by more than 2^8; warp-uniform, so
//                deterministic), P to TMEM as BF16; finally O / l and lse.
//
// All waits are bounded (2 s); a CTA that gives up reports LSA_ERR_TIMEOUT.
#include "kernels.cuh"
#include "tc.cuh"

namespace lsa {

namespace {

constexpr int kAThreads = 416;
constexpr int kRows = 32;                    // KV rows per tile
constexpr int kStagesA = 4;                  // KV tile ring
constexpr int kSP = 3;                       // S / P buffers in TMEM (P overwrites its own S)
constexpr int kD = 576, kDv = 512, kHalf = 256;
constexpr int kAtoms = kD / 64;              // 64-element (128-byte) K atoms of a KV row
constexpr int kQSmemAtoms = 4;               // Q dims 0..255 in shared memory
constexpr int kQTmemCols = (kD - kQSmemAtoms * 64) / 2;   // Q dims 256..575 in TMEM: 160 columns
constexpr int kTileBytes = kAtoms * kRows * 128;          // 36 KB
constexpr int kQBytes = kQSmemAtoms * 128 * 128;          // 64 KB

struct AttnSmem {
    alignas(1024) uint8_t q[kQBytes];
    alignas(1024) uint8_t kv[kStagesA][kTileBytes];
    alignas(16) float kscale[kStagesA][kRows];   // per-row FP8 scale x softmax scale (0 for masked rows)
    alignas(16) float kmask[kStagesA][kRows];    // 0, or -inf for masked rows (added to the scaled score)
    alignas(16) float vscale[kStagesA][kRows];   // per-row FP8 scale (1 for BF16)
    int rows[kStagesA][kRows];
    uint64_t kv_full[kStagesA], kv_empty[kStagesA], s_full[kSP], p_full[kSP], o_done[2], q_ready;
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

template <bool KV_FP8>
__global__ void __cluster_dims__(1, 2, 1) __launch_bounds__(kAThreads, 1) sparse_attn_tc_kernel(AttnArgs a) {
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
    const uint16_t* qt = a.q + (size_t)t * 128 * kD;

    if (threadIdx.x == 0) {
        // kv_full: this CTA's two gather warps (one of them also expecting the peer's rows);
        // kv_empty: the P V commits of both CTAs of the pair.
        for (int i = 0; i < kStagesA; ++i) { tc::mbar_init(&sm.kv_full[i], 64); tc::mbar_init(&sm.kv_empty[i], 2); }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&sm.o_done[i], 1);
        }
        for (int i = 0; i < kSP; ++i) { tc::mbar_init(&sm.s_full[i], 1); tc::mbar_init(&sm.p_full[i], 128); }
        tc::mbar_init(&sm.q_ready, 128);
        sm.abort = 0;
        tc::fence_barrier_init();
    }
    if (warp == 0) tc::tmem_alloc(&sm.tmem_base, 512);
    tc::tc_fence_before();
    __syncthreads();
    tc::cluster_sync_all();                      // the peer's barriers exist before any cross-CTA traffic
    tc::tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const uint32_t o_col = tmem, s_col = tmem + 256, qt_col = tmem + 256 + kSP * 32;   // O, S / P, Q tail
    // The softmax warps load Q while the gather warps already fetch KV tiles: dims 0..255 into
    // shared memory (K-major, 128-byte swizzle), dims 256..575 into TMEM (thread = head = lane).
    if (warp >= 8 && warp < 12) {
        const int tq = threadIdx.x - 256;
        prefetch_l2_bulk(qt + (size_t)tq * kD, kD * 2);              // head tq's row into L2
        for (int i = tq; i < 128 * (kQSmemAtoms * 8); i += 128) {
            const int h = i / (kQSmemAtoms * 8), c = i % (kQSmemAtoms * 8);
            uint8_t* dst = sm.q + (c >> 3) * (128 * 128) + h * 128 + (((c & 7) ^ (h & 7)) << 4);
            cp_async16(dst, qt + (size_t)h * kD + c * 8, true);
        }
        cp_async_commit();
        const int h = (warp & 3) * 32 + lane;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint4* src = reinterpret_cast<const uint4*>(qt + (size_t)h * kD + kQSmemAtoms * 64);
        // Software-pipelined: the loads of 32-column group c + 1 are in flight while group c is
        // stored to TMEM.
        uint4 cur[8], nxt[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) cur[u] = src[u];
#pragma unroll 1
        for (int c = 0; c < kQTmemCols / 32; ++c) {
            if (c + 1 < kQTmemCols / 32) {
#pragma unroll
                for (int u = 0; u < 8; ++u) nxt[u] = src[(c + 1) * 8 + u];
            }
            uint32_t v[32];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                v[4 * u] = cur[u].x; v[4 * u + 1] = cur[u].y; v[4 * u + 2] = cur[u].z; v[4 * u + 3] = cur[u].w;
            }
            tc::tmem_st32(qt_col + c * 32 + lane_off, v);
#pragma unroll
            for (int u = 0; u < 8; ++u) cur[u] = nxt[u];
        }
        tc::tmem_wait_st();
        cp_async_wait<0>();
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        tc::mbar_arrive(&sm.q_ready);
    }

    if (warp < 8) {
        // ---------------- gather producers: warps 2s, 2s + 1 own stage s (tiles j = s, s + 4, ...).
        // The two CTAs of the pair (V halves) gather the same rows: this CTA copies the 16 rows of
        // its own half of each tile (8 per warp) and pushes them into the peer's stage with
        // unicast bulk shared-to-shared copies, completing on the peer's kv_full; the peer does
        // the same for the other 16.  A stage is reused only once both CTAs' P V have read it.
        const int g = warp >> 1, wsub = warp & 1;
        const uint32_t peer = (uint32_t)(half ^ 1);
        const int rcopy = half * (kRows / 2) + wsub * (kRows / 4);  // first row this warp copies
        auto fetch_row = [&](int j) -> int {                       // lane l: index of row l of tile j
            if (j >= n_tiles) return -1;
            const int r0 = r_beg + j * kRows;
            return lane < min(kRows, r_end - r0) ? irow[r0 + lane] : -1;
        };
        int nxt = fetch_row(g);
        for (int j = g; j < n_tiles; j += kStagesA) {
            const int cur = nxt;
            nxt = fetch_row(j + kStagesA);                         // prefetch this warp's next tile
            if (!tc::mbar_wait(&sm.kv_empty[g], ((j / kStagesA) + 1) & 1, abort_flag)) break;
            const int nr = min(kRows, r_end - (r_beg + j * kRows));
            {
                // Both warps of the pair write the same metadata of all 32 rows (identical values).
                const bool v = cur >= 0 && cur < len;
                if (wsub == 0 && half == 0 && lane < nr && !v) report(a.status, LSA_ERR_DEVICE_DATA);
                const float vs = KV_FP8 ? (v ? kvs[cur] : 0.f) : 1.f;
                sm.rows[g][lane] = v ? cur : -1;
                sm.vscale[g][lane] = vs;
                sm.kscale[g][lane] = v ? vs * a.sm_scale_log2 : 0.f;
                sm.kmask[g][lane] = v ? 0.f : kNegInf;
            }
            __syncwarp();
            uint8_t* tile = sm.kv[g];
            if (!KV_FP8) {
#pragma unroll 3
                for (int i = lane; i < (kRows / 4) * (kD / 8); i += 32) {
                    const int r = rcopy + i / (kD / 8), c = i % (kD / 8);
                    const int row = sm.rows[g][r];
                    uint8_t* dst = tile + (c >> 3) * (kRows * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4);
                    cp_async16(dst, kvb + (size_t)(row >= 0 ? row : 0) * a.kv_tok_b + c * 16, row >= 0);
                }
                cp_async_commit();
                cp_async_wait<0>();
            } else {
                constexpr int kChunks = (kRows / 4) * (kD / 16);       // 16 codes per chunk
                constexpr int kBatch = 5;
                for (int i0 = lane; i0 < kChunks; i0 += 32 * kBatch) {
                uint4 raw[kBatch];
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {
                    const int i = i0 + u * 32;
                    raw[u] = make_uint4(0, 0, 0, 0);
                    if (i < kChunks) {
                        const int row = sm.rows[g][rcopy + i / (kD / 16)];
                        if (row >= 0) raw[u] = ldg_nc16(kvb + (size_t)row * a.kv_tok_b + (i % (kD / 16)) * 16);
                    }
                }
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {
                    const int i = i0 + u * 32;
                    if (i >= kChunks) break;
                    const int r = rcopy + i / (kD / 16), c = i % (kD / 16);
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
            tc::fence_proxy_async_smem();                          // this warp's rows, for the bulk copies
            __syncwarp();
            if (lane < kAtoms) {                                   // its 8 rows of atom `lane` to the peer
                const uint8_t* src = tile + lane * (kRows * 128) + rcopy * 128;
                tc::bulk_copy_to_peer(tc::peer_smem(src, peer), src, (kRows / 4) * 128, tc::peer_smem(&sm.kv_full[g], peer));
            }
            if (wsub == 0 && lane == 0) tc::mbar_expect_tx(&sm.kv_full[g], (kRows / 2) * 128 * kAtoms);   // the peer's rows
            else tc::mbar_arrive(&sm.kv_full[g]);
        }
    } else if (warp == 12) {
        // ---------------- MMA issuer: S_j and P_j V_j, each in order, whichever is ready
        const uint32_t idesc_s = tc::idesc_f16(128, kRows, 1);
        const uint32_t idesc_o = tc::idesc_f16_bmn(128, kHalf, 1);
        const uint32_t qaddr = tc::smem_u32(sm.q);
        if (tc::elect_one() && n_tiles > 0 && tc::mbar_wait(&sm.q_ready, 0, abort_flag)) {
            tc::fence_proxy_async_smem();
            tc::tc_fence_after();
            int ns = 0, npv = 0;                 // next S tile, next PV tile
            const uint64_t t0 = tc::global_ns();
            uint32_t polls = 0;
            while (npv < n_tiles) {
                bool progressed = false;
                // S_ns needs its KV tile and its S/P buffer free (P V_{ns-2} issued).
                if (ns < n_tiles && ns <= npv + kSP - 1 && tc::mbar_try_wait(&sm.kv_full[ns % kStagesA], (ns / kStagesA) & 1)) {
                    tc::fence_proxy_async_smem();
                    tc::tc_fence_after();
                    const int sb = ns % kSP;
                    const uint32_t kaddr = tc::smem_u32(sm.kv[ns % kStagesA]);
#pragma unroll
                    for (int kk = 0; kk < kQSmemAtoms * 4; ++kk) {
                        const uint64_t ad = tc::sdesc_sw128(qaddr + (kk >> 2) * (128 * 128) + (kk & 3) * 32);
                        const uint64_t bd = tc::sdesc_sw128(kaddr + (kk >> 2) * (kRows * 128) + (kk & 3) * 32);
                        tc::mma_f16_ss(s_col + sb * 32, ad, bd, idesc_s, kk > 0);
                    }
#pragma unroll
                    for (int kk = kQSmemAtoms * 4; kk < kD / 16; ++kk) {
                        const uint64_t bd = tc::sdesc_sw128(kaddr + (kk >> 2) * (kRows * 128) + (kk & 3) * 32);
                        tc::mma_f16_ts(s_col + sb * 32, qt_col + (kk - kQSmemAtoms * 4) * 8, bd, idesc_s, 1u);
                    }
                    tc::mma_commit(&sm.s_full[sb]);
                    ++ns;
                    progressed = true;
                }
                // P V_npv needs the softmax of tile npv.
                if (npv < ns && tc::mbar_try_wait(&sm.p_full[npv % kSP], (npv / kSP) & 1)) {
                    tc::tc_fence_after();
                    const uint32_t vaddr = tc::smem_u32(sm.kv[npv % kStagesA]) + (4 * half) * (kRows * 128);
#pragma unroll
                    for (int kk = 0; kk < kRows / 16; ++kk) {
                        const uint64_t bd = tc::sdesc_sw128_lbo(vaddr + kk * 16 * 128, kRows * 128, 1024);
                        tc::mma_f16_ts(o_col, s_col + (npv % kSP) * 32 + kk * 8, bd, idesc_o,
                                       (npv > 0 || kk > 0) ? 1u : 0u);
                    }
                    tc::mma_commit_cluster(&sm.kv_empty[npv % kStagesA], 0x3);   // both CTAs of the pair
                    tc::mma_commit(&sm.o_done[npv & 1]);
                    ++npv;
                    progressed = true;
                }
                if (!progressed && (++polls & 255) == 0) {
                    if (*abort_flag || tc::global_ns() - t0 > tc::kWaitNs * 4) { *abort_flag = 1; break; }
                }
            }
            if (npv > 0) {                          // drain before TMEM is freed
                volatile int drain_abort = 0;
                tc::mbar_wait(&sm.o_done[(npv - 1) & 1], ((npv - 1) >> 1) & 1, &drain_abort);
            }
        }
    } else if (warp >= 8 && warp < 12) {
        // ---------------- softmax / epilogue: thread = head = TMEM lane
        const int quarter = warp & 3;
        const int h = quarter * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        float m_run = kNegInf, l_run = 0.f;
        bool alive = true;
        for (int j = 0; j < n_tiles; ++j) {
            const int sb = j % kSP, st = j % kStagesA;
            if (!tc::mbar_wait(&sm.s_full[sb], (j / kSP) & 1, abort_flag)) { alive = false; break; }
            // The tile's row scales were written by the gather warp before kv_full.
            if (!tc::mbar_wait(&sm.kv_full[st], (j / kStagesA) & 1, abort_flag)) { alive = false; break; }
            tc::tc_fence_after();
            uint32_t sv[32];
            tc::tmem_ld32(s_col + sb * 32 + lane_off, sv);
            tc::tmem_wait_ld();
            float x[32];
            const float4* ks4 = reinterpret_cast<const float4*>(sm.kscale[st]);
            const float4* km4 = reinterpret_cast<const float4*>(sm.kmask[st]);
#pragma unroll
            for (int i = 0; i < 8; ++i) {                // scaled score, or -inf for a masked row
                const float4 k4 = ks4[i], m4 = km4[i];
                x[4 * i + 0] = fmaf(__uint_as_float(sv[4 * i + 0]), k4.x, m4.x);
                x[4 * i + 1] = fmaf(__uint_as_float(sv[4 * i + 1]), k4.y, m4.y);
                x[4 * i + 2] = fmaf(__uint_as_float(sv[4 * i + 2]), k4.z, m4.z);
                x[4 * i + 3] = fmaf(__uint_as_float(sv[4 * i + 3]), k4.w, m4.w);
            }
            float mx[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) mx[i] = fmaxf(x[2 * i], x[2 * i + 1]);
#pragma unroll
            for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
                for (int i = 0; i < w; ++i) mx[i] = fmaxf(mx[i], mx[i + w]);
            const float mt = mx[0];
            float alpha = 1.f;
            bool rescale = false;
            if (mt > m_run + 8.f) {
                if (m_run != kNegInf) { alpha = ex2(m_run - mt); rescale = true; }
                l_run *= alpha;
                m_run = mt;
            }
            const float mref = m_run == kNegInf ? 0.f : m_run;            // all rows masked so far: p = 0
            float p[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) p[i] = ex2(x[i] - mref);         // ex2(-inf) = 0
            float ps[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) ps[i] = p[2 * i] + p[2 * i + 1];
#pragma unroll
            for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
                for (int i = 0; i < w; ++i) ps[i] += ps[i + w];
            l_run += ps[0];
            uint32_t pw[16];
            if constexpr (KV_FP8) {                      // the row's FP8 scale goes into P
                const float4* vs4 = reinterpret_cast<const float4*>(sm.vscale[st]);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float4 v4 = vs4[i];
                    pw[2 * i] = pack_bf16x2(p[4 * i] * v4.x, p[4 * i + 1] * v4.y);
                    pw[2 * i + 1] = pack_bf16x2(p[4 * i + 2] * v4.z, p[4 * i + 3] * v4.w);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) pw[i] = pack_bf16x2(p[2 * i], p[2 * i + 1]);
            }
            tc::tmem_st16(s_col + sb * 32 + lane_off, pw);           // P over the S it came from
            if (__any_sync(0xffffffffu, rescale)) {
                // O must hold P V_{j-1} before it is rescaled.
                if (j >= 1 && !tc::mbar_wait(&sm.o_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag)) {
                    alive = false;
                    break;
                }
                tc::tc_fence_after();
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
            tc::mbar_arrive(&sm.p_full[sb]);
        }
        // Epilogue: O / l, lse.
        if (alive && n_tiles > 0 &&
            !tc::mbar_wait(&sm.o_done[(n_tiles - 1) & 1], ((n_tiles - 1) >> 1) & 1, abort_flag))
            alive = false;
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
    if (threadIdx.x == 0) {
        // The peer's copies into this CTA's last stages have landed (already true unless a wait gave
        // up; bounded) before either CTA can leave.
        volatile int drain_abort = 0;
        for (int j = max(0, n_tiles - kStagesA); j < n_tiles; ++j)
            tc::mbar_wait(&sm.kv_full[j % kStagesA], (j / kStagesA) & 1, &drain_abort);
    }
    __syncthreads();
    tc::cluster_sync_all();                      // every copy into either CTA has landed and been read
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
