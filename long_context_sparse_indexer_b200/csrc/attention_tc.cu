// Sparse MLA-absorbed attention on the 5th-generation tensor cores (tcgen05).
//
// Same operation as attention.cu (explainer page, section "① LSA": attention reads only
// the selected keys and the sinks; MLA absorbed form: 128 query heads share one 576-dim
// latent row, V = its first 512 dims), restated for sm_100a.
//
// Work split.  CTA = (split, half h, query token); the two halves of a (split, token) form a
// cluster.  CTA h owns latent dims D_h = [256h, 256h + 256) (its V half) plus the rope dims
// [512 + 32h, 512 + 32h + 32): it gathers only those 288 dims of every selected row (576 B of
// BF16), computes the partial score S_h = Q[:, D_h] K[:, D_h]^T (M = 128 heads, N = 32 rows,
// K = 288), and the two CTAs exchange their partials through distributed shared memory.
// Each adds the peer's partial to its own (x + y = y + x exactly, so both hold the same S),
// runs the same softmax (so both hold the same P) and accumulates O[:, V half h] += P V_h from
// its own rows.  Every byte of a row is read once and no product is computed twice.
//
// Memory plan.  TMEM (512 columns): O half [0,256), three S / P buffers [256,352) -- the
// softmax writes P (BF16) over the S it has just read, so S can run two tiles ahead of P V --
// and the query slice Q[:, D_h] [352,496) as the A operand of S.  Shared memory: a 7-stage
// ring of 32-row KV tiles (5 swizzled 64-dim K atoms, the last half used, 20 KB), read as the
// B operand of S (K-major) and of P V (MN-major); two 16 KB staging buffers for this CTA's
// partial S and two that receive the peer's.
//
//   warps 0..6 : gather -- warp s fills stage s with the tiles j = s, s + 7, ...: the rows'
//                indices (prefetched one tile ahead), per-row scale and validity to shared
//                memory, then the CTA's 288 dims of each row with 16-byte cp.async (FP8 rows
//                are widened to BF16 exactly on the way).
//   warp 7     : MMA issuer -- S_j (18 TS MMAs, N = 32) once tile j has landed and P V_{j-3}
//                has been issued; O += P_j V_j (2 TS MMAs, N = 256) once the softmax of tile
//                j is done; whichever is ready, each kind in order.
//   warps 8..11: softmax -- thread = head (TMEM lane).  Each warp exchanges its 32 heads'
//                rows on its own: it stages its partial S of tile j + 1 in shared memory and
//                one lane pushes the 4 KB to the peer with a bulk shared-to-shared copy that
//                completes on the peer's barrier (so the exchange runs under the softmax of
//                tile j); then it adds the peer's partial of tile j to its own, runs the
//                online max / sum with lazy rescaling of O (only when the running max grows
//                by more than 2^8; warp-uniform, so deterministic) and writes P to TMEM as
//                BF16; finally O / l and lse.
//
// All waits are bounded (2 s); a CTA that gives up reports LSA_ERR_TIMEOUT.
#include <cstring>

#include "kernels.cuh"
#include "tc.cuh"

namespace lsa {

namespace {

constexpr int kAThreads = 512;
constexpr int kRows = 32;                    // KV rows per tile
constexpr int kStagesA = 7;                  // KV tile ring (one gather warp per stage)
constexpr int kXB = 2;                       // partial-S exchange buffers (staging and receive)
constexpr int kSP = 3;                       // S / P buffers in TMEM (P overwrites its own S)
constexpr int kD = 576, kDv = 512, kHalf = 256;
constexpr int kAtomsA = 5;                   // K atoms of a CTA's slice: 4 V atoms + half a rope atom
constexpr int kKSteps = 4 * 4 + 2;           // 16-dim K steps of S per CTA (288 dims)
constexpr int kQCols = kKSteps * 8;          // TMEM columns of the query slice (144)
constexpr int kTileBytes = kAtomsA * kRows * 128;         // 20 KB
static_assert(256 + kSP * 32 + kQCols <= 512, "TMEM columns: O half, S / P buffers, query slice");
constexpr int kXBytes = 128 * kRows * 4;                  // one partial S: 128 heads x 32 rows FP32

struct AttnSmem {
    alignas(1024) uint8_t kv[kStagesA][kTileBytes];
    // Partial S exchange, per buffer [head][16-byte chunk ^ (head & 7)]; softmax warp q owns the
    // 4 KB of heads [32q, 32q + 32) in each.
    alignas(1024) uint8_t xs[kXB][kXBytes];      // the peer's partial S
    alignas(1024) uint8_t stg[kXB][kXBytes];     // this CTA's partial S, the source of the copy to the peer
    alignas(16) float kscale[kStagesA][kRows];   // per-row FP8 scale x softmax scale (0 for masked rows)
    alignas(16) float kmask[kStagesA][kRows];    // 0, or -inf for masked rows (added to the scaled score)
    alignas(16) float vscale[kStagesA][kRows];   // per-row FP8 scale (1 for BF16)
    int rows[kStagesA][kRows];
    uint64_t kv_full[kStagesA], kv_empty[kStagesA], s_full[kSP], p_full[kSP], o_done[2], q_ready;
    uint64_t s_sent[kSP];                        // the send warps have read S out of this buffer
    uint64_t rx_full[kXB][4];                    // a quarter of the peer's partial S has arrived (4 KB tx)
    uint64_t tx_free[kXB][4];                    // the peer has read the quarter this CTA sent into buffer x
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Global dim offset (in elements) of 16-byte chunk c8 of local atom la in CTA `half`'s slice.
// Atom 4 is the 64-dim rope atom at its natural position: CTA h uses chunks [4h, 4h + 4).
__device__ __forceinline__ int slice_dim(int half, int la, int c8) {
    return la < 4 ? half * kHalf + la * 64 + c8 * 8 : kDv + c8 * 8;
}

// KV_FP8: e4m3 rows with a per-row scale, widened to BF16 in shared memory by the gather warps.
// TMA (BF16 rows only): the gather warps issue tile::gather4 loads through `kvmap` (a 2-D map
// over all rows of the cache, box 64 dims x 1 row, 128-byte swizzle) instead of cp.async.
template <bool KV_FP8, bool TMA>
__global__ void __cluster_dims__(1, 2, 1) __launch_bounds__(kAThreads, 1)
    sparse_attn_tc_kernel(const __grid_constant__ CUtensorMap kvmap, AttnArgs a) {
    static_assert(!(KV_FP8 && TMA), "TMA gathers BF16 rows only");
    extern __shared__ uint8_t smem_raw[];
    AttnSmem& sm = *reinterpret_cast<AttnSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int split = blockIdx.x, half = blockIdx.y, t = blockIdx.z;
    const uint32_t peer = (uint32_t)(half ^ 1);
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
        for (int i = 0; i < kStagesA; ++i) {
            tc::mbar_init(&sm.kv_full[i], TMA ? 1 : 32);   // TMA: one expect_tx arrival + the bytes
            tc::mbar_init(&sm.kv_empty[i], 1);
        }
        for (int i = 0; i < kSP; ++i) {
            tc::mbar_init(&sm.s_full[i], 1);
            tc::mbar_init(&sm.s_sent[i], 4);
            tc::mbar_init(&sm.p_full[i], 128);
        }
        for (int x = 0; x < kXB; ++x)
            for (int q = 0; q < 4; ++q) {
                tc::mbar_init(&sm.rx_full[x][q], 1);     // the receiving warp's expect_tx + the copy's bytes
                tc::mbar_init(&sm.tx_free[x][q], 1);     // one remote arrival from the peer's warp q
            }
        for (int i = 0; i < 2; ++i) tc::mbar_init(&sm.o_done[i], 1);
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
    const uint32_t o_col = tmem, s_col = tmem + 256, qt_col = tmem + 256 + kSP * 32;   // O, S / P, Q slice

    // The softmax warps load the query slice Q[:, D_h] into TMEM (thread = head = lane) while the
    // gather warps already fetch KV tiles.  Column c of the slice holds dims (2c, 2c + 1) of
    // [256h, 256h + 256) for c < 128, then of the rope dims [512 + 32h, 512 + 32h + 32).
    if (warp >= 8 && warp < 12) {
        const int h = (warp & 3) * 32 + lane;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint4* src = reinterpret_cast<const uint4*>(qt + (size_t)h * kD + half * kHalf);
        const uint4* rope = reinterpret_cast<const uint4*>(qt + (size_t)h * kD + kDv + half * 32);
        uint4 cur[8], nxt[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) cur[u] = src[u];
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {                // 4 groups of 64 dims = 32 columns
            if (c + 1 < 4) {
#pragma unroll
                for (int u = 0; u < 8; ++u) nxt[u] = src[(c + 1) * 8 + u];
            } else {
#pragma unroll
                for (int u = 0; u < 4; ++u) nxt[u] = rope[u];
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
        {
            uint32_t v[16];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                v[4 * u] = cur[u].x; v[4 * u + 1] = cur[u].y; v[4 * u + 2] = cur[u].z; v[4 * u + 3] = cur[u].w;
            }
            tc::tmem_st16(qt_col + 128 + lane_off, v);
        }
        tc::tmem_wait_st();
        tc::tc_fence_before();
        tc::mbar_arrive(&sm.q_ready);
    }

    if (warp < kStagesA) {
        // ---------------- gather producers: warp s owns stage s and the tiles j = s, s + 7, ...
        const int g = warp;
        auto fetch_row = [&](int j) -> int {                       // lane l: index of row l of tile j
            if (j >= n_tiles) return -1;
            const int r0 = r_beg + j * kRows;
            return lane < min(kRows, r_end - r0) ? irow[r0 + lane] : -1;
        };
        if (TMA && lane == 0) tc::prefetch_tmap(&kvmap);
        // Row coordinate of this sequence's row 0 in the map (TMA): the cache is B sequences of
        // kv_seq_b / kv_tok_b rows.
        const int row0 = TMA ? (int)((int64_t)max(b, 0) * (a.kv_seq_b / a.kv_tok_b)) : 0;
        int nxt = fetch_row(g);
        for (int j = g; j < n_tiles; j += kStagesA) {
            const int cur = nxt;
            nxt = fetch_row(j + kStagesA);                         // prefetch this warp's next tile
            if (!__all_sync(0xffffffffu, tc::mbar_wait(&sm.kv_empty[g], ((j / kStagesA) + 1) & 1, abort_flag))) break;
            const int nr = min(kRows, r_end - (r_beg + j * kRows));
            {
                const bool v = cur >= 0 && cur < len;
                if (half == 0 && lane < nr && !v) report(a.status, LSA_ERR_DEVICE_DATA);
                const float vs = KV_FP8 ? (v ? kvs[cur] : 0.f) : 1.f;
                sm.rows[g][lane] = v ? cur : -1;
                sm.vscale[g][lane] = vs;
                sm.kscale[g][lane] = v ? vs * a.sm_scale_log2 : 0.f;
                sm.kmask[g][lane] = v ? 0.f : kNegInf;
            }
            __syncwarp();
            uint8_t* tile = sm.kv[g];
            if constexpr (TMA) {
                // 8 groups of 4 rows x 5 atoms (the V half and the whole rope atom), 512 B each;
                // a masked row reads as zeros (coordinate -1 is outside the map).
                const int grow = (cur >= 0 && cur < len) ? row0 + cur : -1;
                int rr[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) rr[i] = __shfl_sync(0xffffffffu, grow, ((lane & 7) << 2) + i);
                if (lane == 0) tc::mbar_expect_tx(&sm.kv_full[g], kTileBytes);
                __syncwarp();
                if (lane < 8) {
#pragma unroll
                    for (int la = 0; la < kAtomsA; ++la)
                        tc::tma_gather4(tile + la * (kRows * 128) + lane * 512, &kvmap, &sm.kv_full[g],
                                        la < 4 ? half * kHalf + la * 64 : kDv, rr[0], rr[1], rr[2], rr[3]);
                }
                continue;
            } else if (!KV_FP8) {
                // 36 chunks of 16 bytes per row: 32 of the V half (4 atoms x 8), 4 rope chunks.
#pragma unroll 4
                for (int i = lane; i < kRows * 36; i += 32) {
                    const int r = i / 36, q = i % 36;
                    const int la = q < 32 ? q >> 3 : 4, c8 = q < 32 ? q & 7 : 4 * half + q - 32;
                    const int row = sm.rows[g][r];
                    uint8_t* dst = tile + la * (kRows * 128) + r * 128 + ((c8 ^ (r & 7)) << 4);
                    cp_async16(dst, kvb + (size_t)(row >= 0 ? row : 0) * a.kv_tok_b + slice_dim(half, la, c8) * 2,
                               row >= 0);
                }
                cp_async_commit();
                cp_async_wait<0>();
            } else {
                // 18 chunks of 16 codes per row (16 of the V half, 2 rope), each widened to two
                // BF16 chunks.
                constexpr int kChunks = kRows * 18;
                constexpr int kBatch = 6;
                for (int i0 = lane; i0 < kChunks; i0 += 32 * kBatch) {
                    uint4 raw[kBatch];
#pragma unroll
                    for (int u = 0; u < kBatch; ++u) {
                        const int i = i0 + u * 32;
                        raw[u] = make_uint4(0, 0, 0, 0);
                        if (i < kChunks) {
                            const int r = i / 18, q = i % 18;
                            const int row = sm.rows[g][r];
                            const int code = q < 16 ? half * kHalf + q * 16 : kDv + half * 32 + (q - 16) * 16;
                            if (row >= 0) raw[u] = ldg_nc16(kvb + (size_t)row * a.kv_tok_b + code);
                        }
                    }
#pragma unroll
                    for (int u = 0; u < kBatch; ++u) {
                        const int i = i0 + u * 32;
                        if (i >= kChunks) break;
                        const int r = i / 18, q = i % 18;
                        const int la = q < 16 ? q >> 2 : 4, cb0 = q < 16 ? (q & 3) * 2 : 4 * half + (q - 16) * 2;
                        const uint32_t* wd = reinterpret_cast<const uint32_t*>(&raw[u]);
                        uint32_t ow[8];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            ow[2 * e] = e4m3x2_to_bf16x2((uint16_t)(wd[e] & 0xffff));
                            ow[2 * e + 1] = e4m3x2_to_bf16x2((uint16_t)(wd[e] >> 16));
                        }
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const int c8 = cb0 + hh;
                            uint8_t* dst = tile + la * (kRows * 128) + r * 128 + ((c8 ^ (r & 7)) << 4);
                            *reinterpret_cast<uint4*>(dst) =
                                make_uint4(ow[4 * hh], ow[4 * hh + 1], ow[4 * hh + 2], ow[4 * hh + 3]);
                        }
                    }
                }
            }
            tc::fence_proxy_async_smem();
            tc::mbar_arrive(&sm.kv_full[g]);
        }
        if constexpr (TMA) {
            // A CTA that gave up may still have gathers in flight into its shared memory: wait
            // (bounded) for this warp's last tile to land before the CTA can exit.
            const int last = g < n_tiles ? g + ((n_tiles - 1 - g) / kStagesA) * kStagesA : -1;
            if (last >= 0 && lane == 0 && *abort_flag) {
                volatile int drain_abort = 0;
                tc::mbar_wait(&sm.kv_full[g], (last / kStagesA) & 1, &drain_abort);
            }
        }
    } else if (warp == kStagesA) {
        // ---------------- MMA issuer: S_j and P_j V_j, each in order, whichever is ready
        const uint32_t idesc_s = tc::idesc_f16(128, kRows, 1);
        const uint32_t idesc_o = tc::idesc_f16_bmn(128, kHalf, 1);
        if (tc::elect_one() && n_tiles > 0 && tc::mbar_wait(&sm.q_ready, 0, abort_flag)) {
            tc::tc_fence_after();
            int ns = 0, npv = 0;                 // next S tile, next P V tile
            const uint64_t t0 = tc::global_ns();
            uint32_t polls = 0;
            while (npv < n_tiles) {
                bool progressed = false;
                // S_ns needs its KV tile and its S / P buffer free: P V_{ns-3} issued and S_{ns-3}
                // read by the send warps.
                if (ns < n_tiles && ns <= npv + kSP - 1 &&
                    (ns < kSP || tc::mbar_test_wait(&sm.s_sent[ns % kSP], ((ns / kSP) - 1) & 1)) &&
                    tc::mbar_try_wait(&sm.kv_full[ns % kStagesA], (ns / kStagesA) & 1)) {
                    tc::tc_fence_after();
                    const int sb = ns % kSP;
                    const uint32_t kaddr = tc::smem_u32(sm.kv[ns % kStagesA]);
#pragma unroll
                    for (int kk = 0; kk < kKSteps; ++kk) {
                        const int la = kk < 16 ? kk >> 2 : 4, ks = kk < 16 ? kk & 3 : 2 * half + kk - 16;
                        const uint64_t bd = tc::sdesc_sw128(kaddr + la * (kRows * 128) + ks * 32);
                        tc::mma_f16_ts(s_col + sb * 32, qt_col + kk * 8, bd, idesc_s, kk > 0);
                    }
                    tc::mma_commit(&sm.s_full[sb]);
                    ++ns;
                    progressed = true;
                }
                // P V_npv needs the softmax of tile npv.  V half = the tile's atoms 0..3, MN-major.
                if (npv < ns && tc::mbar_try_wait(&sm.p_full[npv % kSP], (npv / kSP) & 1)) {
                    tc::tc_fence_after();
                    const uint32_t vaddr = tc::smem_u32(sm.kv[npv % kStagesA]);
#pragma unroll
                    for (int kk = 0; kk < kRows / 16; ++kk) {
                        const uint64_t bd = tc::sdesc_sw128_lbo(vaddr + kk * 16 * 128, kRows * 128, 1024);
                        tc::mma_f16_ts(o_col, s_col + (npv % kSP) * 32 + kk * 8, bd, idesc_o,
                                       (npv > 0 || kk > 0) ? 1u : 0u);
                    }
                    tc::mma_commit(&sm.kv_empty[npv % kStagesA]);
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
        const int xoff = lane * 128;                 // this head's row within a quarter
        float m_run = kNegInf, l_run = 0.f;
        bool alive = true;
        if (lane == 0)                               // the first two tiles' partials may arrive at once
            for (int x = 0; x < kXB && x < n_tiles; ++x) tc::mbar_expect_tx(&sm.rx_full[x][quarter], 4096);
        for (int j = 0; j < n_tiles; ++j) {
            const int sb = j % kSP, st = j % kStagesA, xb = j % kXB;
            if (!__all_sync(0xffffffffu, tc::mbar_wait(&sm.s_full[sb], (j / kSP) & 1, abort_flag))) {
                alive = false;
                break;
            }
            // The tile's row scales were written by its gather warp before kv_full.
            if (!__all_sync(0xffffffffu, tc::mbar_wait(&sm.kv_full[st], (j / kStagesA) & 1, abort_flag))) {
                alive = false;
                break;
            }
            tc::tc_fence_after();
            uint32_t sv[32];
            tc::tmem_ld32(s_col + sb * 32 + lane_off, sv);
            // Receive the peer's partial and add it (the same sum in both CTAs).
            const bool got = tc::mbar_wait(&sm.rx_full[xb][quarter], (j / kXB) & 1, abort_flag);
            tc::tmem_wait_ld();
            if (!__all_sync(0xffffffffu, got)) { alive = false; break; }
            float x[32];
            {
                const uint8_t* xr = sm.xs[xb] + quarter * 4096 + xoff;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 pv = *reinterpret_cast<const uint4*>(xr + ((c ^ (lane & 7)) << 4));
                    x[4 * c + 0] = __uint_as_float(sv[4 * c + 0]) + __uint_as_float(pv.x);
                    x[4 * c + 1] = __uint_as_float(sv[4 * c + 1]) + __uint_as_float(pv.y);
                    x[4 * c + 2] = __uint_as_float(sv[4 * c + 2]) + __uint_as_float(pv.z);
                    x[4 * c + 3] = __uint_as_float(sv[4 * c + 3]) + __uint_as_float(pv.w);
                }
            }
            if (lane == 0 && j + kXB < n_tiles)      // buffer xb is ready for tile j + 2
                tc::mbar_expect_tx(&sm.rx_full[xb][quarter], 4096);
            const float4* ks4 = reinterpret_cast<const float4*>(sm.kscale[st]);
            const float4* km4 = reinterpret_cast<const float4*>(sm.kmask[st]);
#pragma unroll
            for (int i = 0; i < 8; ++i) {                // scaled score, or -inf for a masked row
                const float4 k4 = ks4[i], m4 = km4[i];
                x[4 * i + 0] = fmaf(x[4 * i + 0], k4.x, m4.x);
                x[4 * i + 1] = fmaf(x[4 * i + 1], k4.y, m4.y);
                x[4 * i + 2] = fmaf(x[4 * i + 2], k4.z, m4.z);
                x[4 * i + 3] = fmaf(x[4 * i + 3], k4.w, m4.w);
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
            // P goes over the S it came from, once the send warps have read that S.
            if (!__all_sync(0xffffffffu, tc::mbar_wait(&sm.s_sent[sb], (j / kSP) & 1, abort_flag))) {
                alive = false;
                break;
            }
            tc::tmem_st16(s_col + sb * 32 + lane_off, pw);
            // Every lane's max depends on every word it read from buffer xb, so once this vote has
            // run, the warp's reads of the buffer are complete and the peer may overwrite it.  (A
            // release arrive here stalls the warp for about half a tile's time.)
            const bool any_rescale = __any_sync(0xffffffffu, rescale);
            if (lane == 0) tc::mbar_arrive_remote_relaxed(tc::peer_smem(&sm.tx_free[xb][quarter], peer));
            if (any_rescale) {
                // O must hold P V_{j-1} before it is rescaled.
                if (j >= 1 &&
                    !__all_sync(0xffffffffu, tc::mbar_wait(&sm.o_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag))) {
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
            !__all_sync(0xffffffffu, tc::mbar_wait(&sm.o_done[(n_tiles - 1) & 1], ((n_tiles - 1) >> 1) & 1, abort_flag)))
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
    } else {
        // ---------------- send warps 12..15: warp q pushes heads [32q, 32q + 32) of every partial S
        // to the peer -- staged in shared memory, then one 4 KB bulk copy that completes on the
        // peer's rx_full -- as soon as the MMA has produced it, off the softmax's path.
        const int quarter = warp & 3;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const uint32_t xs_peer = tc::peer_smem(sm.xs[0], peer) + quarter * 4096;
        for (int jj = 0; jj < n_tiles; ++jj) {
            const int b = jj % kSP, x = jj % kXB;
            if (!__all_sync(0xffffffffu, tc::mbar_wait(&sm.s_full[b], (jj / kSP) & 1, abort_flag))) break;
            tc::tc_fence_after();
            uint32_t sv[32];
            tc::tmem_ld32(s_col + b * 32 + lane_off, sv);
            tc::tmem_wait_ld();
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&sm.s_sent[b]);          // buffer b may be overwritten
            // Staging buffer x and the peer's buffer x are free once the peer has read tile jj - 2
            // (which it received, so the copy out of staging buffer x is complete too).
            bool ok = true;
            if (jj >= kXB && lane == 0)
                ok = tc::mbar_wait_cluster(&sm.tx_free[x][quarter], ((jj / kXB) - 1) & 1, abort_flag);
            if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) break;
            uint8_t* row = sm.stg[x] + quarter * 4096 + lane * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c)
                *reinterpret_cast<uint4*>(row + ((c ^ (lane & 7)) << 4)) =
                    make_uint4(sv[4 * c], sv[4 * c + 1], sv[4 * c + 2], sv[4 * c + 3]);
            tc::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0)
                tc::bulk_copy_to_peer(xs_peer + x * kXBytes, sm.stg[x] + quarter * 4096, 4096,
                                      tc::peer_smem(&sm.rx_full[x][quarter], peer));
        }
    }

    tc::tc_fence_before();
    __syncthreads();
    tc::cluster_sync_all();                      // no CTA leaves while its peer may still store into it
    if (sm.abort && threadIdx.x == 0) report(a.status, LSA_ERR_TIMEOUT);
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, 512);
    }
}

template <bool KV_FP8, bool TMA>
cudaError_t launch_t(const CUtensorMap& m, const AttnArgs& a, cudaStream_t st) {
    const size_t smem = sizeof(AttnSmem) + 1024;
    auto kern = sparse_attn_tc_kernel<KV_FP8, TMA>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(a.n_split, 2, a.T);
    kern<<<grid, kAThreads, smem, st>>>(m, a);
    return cudaGetLastError();
}

// The BF16 cache as one 2-D tensor of rows (row of sequence b, token i = b * (kv_seq_b / kv_tok_b)
// + i) for tile::gather4.  False when the layout or the driver does not allow it.
bool make_kv_map(const AttnArgs& a, CUtensorMap* m) {
    if (tc::encode_tiled() == nullptr || a.B < 1 || a.kv_tok_b <= 0 || a.kv_seq_b % a.kv_tok_b != 0) return false;
    const int64_t rps = a.kv_seq_b / a.kv_tok_b;
    const int64_t rows = (int64_t)(a.B - 1) * rps + a.L_alloc;
    if (rows < 1 || rows >= ((int64_t)1 << 31) || (a.B > 1 && rps < 1)) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)a.kv_tok_b};
    const cuuint32_t box[2] = {64, 1};
    const cuuint32_t estr[2] = {1, 1};
    return tc::encode_tiled()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint8_t*>(a.kv), dims, strides, box,
                              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool sparse_attn_tc_supported(const AttnArgs& a, int DQK, int DV, bool sep_v) {
    return DQK == kD && DV == kDv && !sep_v && a.H == 128 && (a.kv_tok_b % 16) == 0 && (a.kv_seq_b % 16) == 0 &&
           ((uintptr_t)a.kv % 16) == 0 && ((uintptr_t)a.q % 16) == 0;
}

cudaError_t launch_sparse_attn_tc(const AttnArgs& a, bool kv_fp8, cudaStream_t st) {
    CUtensorMap m;
    memset(&m, 0, sizeof(m));
    if (kv_fp8) return launch_t<true, false>(m, a, st);
    if (make_kv_map(a, &m)) return launch_t<false, true>(m, a, st);
    memset(&m, 0, sizeof(m));
    return launch_t<false, false>(m, a, st);
}

}  // namespace lsa
