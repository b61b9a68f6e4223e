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
// Memory plan.  TMEM (512 columns): O half [0,256), four S / P buffers [256,384) -- the
// softmax writes P (BF16) over the S it has just read, so S can run three tiles ahead of P V --
// and the query's V-half dims [384,512) as the A operand of S; the query's 32 rope dims sit in
// shared memory (no swizzle, K-major) as the A operand of S's two rope steps.  Shared memory: an 8-stage
// ring of 32-row KV tiles, read as the B operand of S (K-major) and of P V (MN-major): each
// stage has its 4 swizzled 64-dim V-half atoms (16 KB), and two stages share one 64-dim rope
// atom, each in the half of its 128-byte rows that the other leaves (only 32 rope dims are this
// CTA's); two 16 KB staging buffers for this CTA's partial S and two that receive the peer's.
//
// Warp roles (512 threads).  With BF16 rows:
//   warps 0,2,3: gather -- tile j by the (j mod 3)-th: the rows' indices (prefetched three tiles
//                of the warp ahead) and validity to shared memory, then the V-half atoms with
//                tile::gather4 (4 rows x 64 dims per load; a tile of 32 consecutive valid rows,
//                as the window gives, with one TMA box of 32 rows per atom) and the 4 rope chunks
//                of each row with 16-byte cp.async; both complete on the tile's barrier by
//                themselves, so the warp moves on at once.  (Without a tensor map for the cache,
//                cp.async does it all.)
//   warp 1     : MMA issuer -- S_j (16 TS + 2 SS MMAs, N = 32) once tile j has landed, P V_{j-4}
//                has been issued and S_{j-4} has been sent; O += P_j V_j (2 TS MMAs, N = 256) once
//                the softmax of tile j is done; whichever is ready, each kind in order.
//   warps 4..7 : send -- warp q (mod 4) stages heads [32q, 32q + 32) of each partial S in shared
//                memory and pushes the 4 KB to the peer with one bulk shared-to-shared copy that
//                completes on the peer's barrier, as soon as the MMA has produced it.
//   warps 8..15: softmax -- two warpgroups taking alternate tiles; thread = head (TMEM lane).
//                Each adds the peer's partial of its tile to its own, then runs the online
//                softmax with lazy rescaling: the reference max is raised only when a tile's
//                max exceeds it by more than 2^8 (warp-uniform, so deterministic).  These
//                decisions form one chain over the tiles, handed from one warpgroup to the
//                other through shared memory, so that only the compare runs in tile order and
//                the exponentials of two tiles overlap; the warpgroup that raises the max
//                rescales O.  P goes to TMEM as BF16; finally O / l and lse, half the columns
//                each.
// With FP8 rows warps 0..6 gather (tile j by warp j mod 7; the codes are loaded and widened to
// BF16 exactly on the way), warp 7 issues the MMAs, warps 8..11 are a single softmax warpgroup
// and warps 12..15 send.
//
// All waits are bounded (2 s); a CTA that gives up reports LSA_ERR_TIMEOUT.
#include <cstring>

#include "kernels.cuh"
#include "tc.cuh"

namespace lsa {

namespace {

constexpr int kAThreads = 512;
constexpr int kRows = 32;                    // KV rows per tile
constexpr int kStagesA = 8;                  // KV tile ring
constexpr int kXB = 2;                       // partial-S exchange buffers (staging and receive)
constexpr int kSP = 4;                       // S / P buffers in TMEM (P overwrites its own S)
constexpr int kD = 576, kDv = 512, kHalf = 256;
constexpr int kKSteps = 4 * 4 + 2;           // 16-dim K steps of S per CTA (288 dims)
constexpr int kQCols = 16 * 8;               // TMEM columns of the query's V-half dims (128)
constexpr int kVBytes = 4 * kRows * 128;                  // a tile's 4 V-half atoms, 16 KB
constexpr int kRopeBytes = kRows * 128;                   // one rope atom, shared by two stages
static_assert(256 + kSP * 32 + kQCols <= 512, "TMEM columns: O half, S / P buffers, query slice");
constexpr int kXBytes = 128 * kRows * 4;                  // one partial S: 128 heads x 32 rows FP32

struct AttnSmem {
    alignas(1024) uint8_t kv[kStagesA][kVBytes];       // V-half atoms of each stage
    alignas(1024) uint8_t rope[kStagesA / 2][kRopeBytes];  // stage s: atom s / 2, chunk half (CTA half) ^ (s & 1)
    // Partial S exchange, per buffer [head][16-byte chunk ^ (head & 7)]; softmax warp q owns the
    // 4 KB of heads [32q, 32q + 32) in each.
    alignas(1024) uint8_t xs[kXB][kXBytes];      // the peer's partial S
    alignas(1024) uint8_t stg[kXB][kXBytes];     // this CTA's partial S, the source of the copy to the peer
    // The query's 32 rope dims of this CTA, K-major without swizzle: head h, 8-dim chunk c at
    // (h / 8) * 512 + c * 128 + (h % 8) * 16 -- the A operand of the two rope K steps of S.
    alignas(1024) uint8_t q_rope[128 * 64];
    alignas(16) float kscale[kStagesA][kRows];   // per-row FP8 scale x softmax scale (0 for masked rows)
    alignas(16) float kmask[kStagesA][kRows];    // 0, or -inf for masked rows (added to the scaled score)
    alignas(16) float vscale[kStagesA][kRows];   // per-row FP8 scale (1 for BF16)
    int rows[kStagesA][kRows];
    uint64_t kv_full[kStagesA], kv_empty[kStagesA], s_full[kSP], p_full[kSP], q_ready, q_tma;
    // P V_k completes phase k / kSP of o_done[k % kSP].  A parity wait tells two phases apart only
    // if the earlier one is complete: a thread that has seen S_j done knows P V_{j-4} done (the
    // commit after S_j covers every earlier MMA, and S_j is issued after P V_{j-4}), so it may
    // wait for P V_{j-1} on a ring of kSP barriers -- on two it could not, P V_{j-3} may still be
    // pending.  mma_done: committed once, after the last MMA (the issuer's drain).
    uint64_t o_done[kSP], mma_done;
    uint64_t s_sent[kSP];                        // the send warps have read S out of this buffer
    uint64_t hand[2][4];                         // softmax warpgroup w, quarter q: m_ref of its tile is out
    float m_ref[128];                            // the reference max after the latest decided tile
    float2 ml[2][128];                           // each softmax warpgroup's final (max, sum)
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

// Named barrier `id` over `count` threads (whole warps).
__device__ __forceinline__ void named_bar_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;" :: "r"(id), "r"(count) : "memory");
}

// KV_FP8: e4m3 rows with a per-row scale, widened to BF16 in shared memory by the gather warps.
// BF16 rows are copied as they are by three warps without waiting: the V-half atoms with TMA
// tile::gather4 through `kvmap` (a 2-D map over all rows of the cache, box 64 dims x 1 row,
// 128-byte swizzle) when TMA is set, else with cp.async; the rope chunks with cp.async.  Both
// complete on the tile's barrier by themselves.
// `qmap`: the queries as a 2-D tensor [T * 128 heads][576 dims], box 64 dims x 128 heads,
// 128-byte swizzle.
template <bool KV_FP8, bool TMA>
__global__ void __cluster_dims__(1, 2, 1) __launch_bounds__(kAThreads, 1)
    sparse_attn_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kvmap,
                          const __grid_constant__ CUtensorMap kvtile, AttnArgs a) {
    static_assert(!(KV_FP8 && TMA), "TMA gathers BF16 rows only");
    constexpr bool kAsync = !KV_FP8;             // gather by 3 warps that do not wait for their copies
    constexpr int kSmx = kAsync ? 2 : 1;         // softmax warpgroups
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
    const int32_t* irow = a.idx + (size_t)t * a.ld_idx;
    const uint8_t* kvb = a.kv + (size_t)max(b, 0) * a.kv_seq_b;
    const float* kvs = KV_FP8 ? a.kv_scale + (size_t)max(b, 0) * a.kv_scale_seq : nullptr;
    const uint16_t* qt = a.q + (size_t)t * 128 * kD;

    auto q_atom = [&](int at) -> uint8_t* { return at < 2 ? sm.xs[at] : (at < 4 ? sm.stg[at - 2] : sm.kv[7]); };
    if (threadIdx.x == 0) {
        for (int i = 0; i < kStagesA; ++i) {
            tc::mbar_init(&sm.kv_full[i], kAsync ? 33 : 32);   // async: 32 copy completions + 1 (scales)
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
        for (int i = 0; i < kSP; ++i) tc::mbar_init(&sm.o_done[i], 1);
        tc::mbar_init(&sm.mma_done, 1);
        for (int w = 0; w < 2; ++w)
            for (int q = 0; q < 4; ++q) tc::mbar_init(&sm.hand[w][q], 1);
        tc::mbar_init(&sm.q_ready, kSmx * 128);
        tc::mbar_init(&sm.q_tma, 1);
        sm.abort = 0;
        tc::fence_barrier_init();
        // Q[:, V half] as 4 swizzled 64-dim atoms into the exchange buffers and its rope atom into
        // KV stage 7, all idle until the softmax warps have moved Q to TMEM (the rope part to
        // shared memory).
        tc::prefetch_tmap(&qmap);
        tc::mbar_expect_tx(&sm.q_tma, 5 * 128 * 128);
        for (int at = 0; at < 5; ++at)
            tc::tma_load_2d(q_atom(at), &qmap, &sm.q_tma, at < 4 ? half * kHalf + at * 64 : kDv, t * 128);
    }
    if (warp == 0) tc::tmem_alloc(&sm.tmem_base, 512);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    int n = ok ? a.count[t] : 0;
    if (n < 0 || n > a.ld_idx) { ok = false; n = 0; }
    if (!ok && threadIdx.x == 0 && split == 0 && half == 0) report(a.status, LSA_ERR_DEVICE_DATA);
    const int per = (n + a.n_split - 1) / a.n_split;
    const int r_beg = min(n, split * per), r_end = min(n, r_beg + per);
    const int n_tiles = (r_end - r_beg + kRows - 1) / kRows;
    const uint32_t tmem = sm.tmem_base;
    const uint32_t o_col = tmem, s_col = tmem + 256, qt_col = tmem + 256 + kSP * 32;   // O, S / P, Q slice

    // Warp roles.  BF16 rows: warps 0, 2, 3 gather (tile j by the (j mod 3)-th), warp 1 issues the
    // MMAs, warps 4..7 send the partial S, and warps 8..11 and 12..15 are two softmax warpgroups
    // taking alternate tiles.  FP8 rows: warps 0..6 gather (warp s owns stage s), warp 7 issues
    // the MMAs, warps 8..11 are the softmax warpgroup and warps 12..15 send.
    constexpr int kGatherFp8 = 7;                // FP8 gather warps 0..6
    const int mma_warp = kAsync ? 1 : kGatherFp8;
    const bool send_warp = kAsync ? (warp >= 4 && warp < 8) : warp >= 12;
    const int wg = warp >= 8 ? (warp - 8) >> 2 : -1;                // softmax warpgroup
    const bool smx_warp = wg >= 0 && wg < kSmx;

    // The softmax warps move the query slice Q[:, D_h] into TMEM (thread = head = lane; with two
    // warpgroups each takes half the columns) while the gather warps already fetch KV tiles:
    // column c holds dims (2c, 2c + 1) of [256 half, 256 half + 256) for c < 128, then of the rope
    // dims [512 + 32 half, 512 + 32 half + 32), read from the staged atoms.
    // Every thread arrives on the cluster barrier once its CTA's barriers exist -- the softmax
    // warps only after their reads of the exchange buffers, so no copy from the peer lands there
    // before.
    if (smx_warp) {
        const int h = (warp & 3) * 32 + lane;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const bool got = tc::mbar_wait(&sm.q_tma, 0, abort_flag);
        const int at0 = kSmx == 2 ? 2 * wg : 0, at1 = kSmx == 2 ? at0 + 2 : 4;
        for (int at = at0; at < at1; ++at) {
            const uint8_t* row = q_atom(at) + h * 128;
            uint32_t w[32];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 v = got ? *reinterpret_cast<const uint4*>(row + ((c ^ (h & 7)) << 4)) : make_uint4(0, 0, 0, 0);
                w[4 * c] = v.x; w[4 * c + 1] = v.y; w[4 * c + 2] = v.z; w[4 * c + 3] = v.w;
            }
            tc::tmem_st32(qt_col + at * 32 + lane_off, w);
        }
        if (kSmx == 1 || wg == 1) {                  // this CTA's rope chunks 4 half .. 4 half + 3
            const uint8_t* row = q_atom(4) + h * 128;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint4 v = got ? *reinterpret_cast<const uint4*>(row + (((4 * half + c) ^ (h & 7)) << 4))
                                    : make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4*>(sm.q_rope + (h >> 3) * 512 + c * 128 + (h & 7) * 16) = v;
            }
            tc::fence_proxy_async_smem();            // for the tensor cores
        }
        tc::tmem_wait_st();
        tc::tc_fence_before();
        tc::mbar_arrive(&sm.q_ready);
    }
    tc::cluster_arrive();
    // Warps that touch the peer's shared memory wait for its barriers to exist; the others only
    // before leaving.
    const bool remote_warp = send_warp || smx_warp;
    if (remote_warp) tc::cluster_wait();

    if (kAsync ? (warp == 0 || warp == 2 || warp == 3) : warp < kGatherFp8) {
        // ---------------- gather producers: tiles j = first, first + step, ... into stage j % 8
        const int first = kAsync ? (warp == 0 ? 0 : warp - 1) : warp, step = kAsync ? 3 : kGatherFp8;
        auto fetch_row = [&](int j) -> int {                       // lane l: index of row l of tile j
            if (j >= n_tiles) return -1;
            const int r0 = r_beg + j * kRows;
            return lane < min(kRows, r_end - r0) ? irow[r0 + lane] : -1;
        };
        if (TMA && lane == 0) {
            tc::prefetch_tmap(&kvmap);
            tc::prefetch_tmap(&kvtile);
        }
        // Row coordinate of this sequence's row 0 in the map (TMA): the cache is B sequences of
        // kv_seq_b / kv_tok_b rows.
        const int row0 = TMA ? (int)((int64_t)max(b, 0) * (a.kv_seq_b / a.kv_tok_b)) : 0;
        // The row indices run three of this warp's tiles ahead (the warp does not wait for its
        // copies, so one tile ahead would leave the index load's latency exposed).
        int nxt1 = fetch_row(first), nxt2 = fetch_row(first + step), nxt3 = fetch_row(first + 2 * step);
        for (int j = first; j < n_tiles; j += step) {
            const int cur = nxt1, g = j % kStagesA;
            nxt1 = nxt2;
            nxt2 = nxt3;
            nxt3 = fetch_row(j + 3 * step);
            if (!__all_sync(0xffffffffu, tc::mbar_wait(&sm.kv_empty[g], ((j / kStagesA) + 1) & 1, abort_flag))) break;
            // Stage 7 holds the query's rope atom until the softmax warps have read it.
            if (j == 7 && !__all_sync(0xffffffffu, tc::mbar_wait(&sm.q_ready, 0, abort_flag))) break;
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
            // Destination of 16-byte chunk c8 of local atom la (4 = rope) of tile row r.
            const int rh = half ^ (g & 1);                         // rope chunk half of this stage
            auto dst_of = [&](int la, int r, int c8) -> uint8_t* {
                return (la < 4 ? sm.kv[g] + la * (kRows * 128) : sm.rope[g >> 1]) + r * 128 + ((c8 ^ (r & 7)) << 4);
            };
            if constexpr (!KV_FP8) {
                // A masked row reads as zeros.  Each lane's cp.async arrive on the barrier when
                // they complete (32 of its 33 arrivals); the 33rd is lane 0's, after the scales.
                if constexpr (TMA) {
                    // V half.  A tile of 32 valid consecutive rows (the window, or a context
                    // shorter than the selection) is one box of 32 rows per atom; any other tile
                    // is 8 groups of 4 rows x 4 atoms, 512 B per tile::gather4 (coordinate -1 is
                    // outside the map).  Both land the same swizzled bytes.
                    const int grow = (cur >= 0 && cur < len) ? row0 + cur : -1;
                    const int grow0 = __shfl_sync(0xffffffffu, grow, 0);
                    const bool run = __all_sync(0xffffffffu, grow >= 0 && grow == grow0 + lane);
                    if (lane == 0) tc::mbar_expect_tx(&sm.kv_full[g], kVBytes);
                    __syncwarp();
                    if (run) {
                        if (lane < 4)
                            tc::tma_load_2d(sm.kv[g] + lane * (kRows * 128), &kvtile, &sm.kv_full[g],
                                            half * kHalf + lane * 64, grow0);
                    } else {
                        int rr[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) rr[i] = __shfl_sync(0xffffffffu, grow, ((lane & 7) << 2) + i);
                        if (lane < 8) {
#pragma unroll
                            for (int la = 0; la < 4; ++la)
                                tc::tma_gather4(sm.kv[g] + la * (kRows * 128) + lane * 512, &kvmap, &sm.kv_full[g],
                                                half * kHalf + la * 64, rr[0], rr[1], rr[2], rr[3]);
                        }
                    }
                    // Rope: 4 chunks per row.
#pragma unroll
                    for (int i = lane; i < kRows * 4; i += 32) {
                        const int r = i >> 2, c = i & 3;
                        const int row = sm.rows[g][r];
                        cp_async16(dst_of(4, r, 4 * rh + c),
                                   kvb + (size_t)(row >= 0 ? row : 0) * a.kv_tok_b + (kDv + 32 * half + 8 * c) * 2, row >= 0);
                    }
                    cp_async_mbar_arrive_noinc(&sm.kv_full[g]);
                } else {
                    // 36 chunks of 16 bytes per row: 32 of the V half (4 atoms x 8), 4 rope chunks.
#pragma unroll 4
                    for (int i = lane; i < kRows * 36; i += 32) {
                        const int r = i / 36, q = i % 36;
                        const int la = q < 32 ? q >> 3 : 4, c = q < 32 ? q & 7 : q - 32;
                        const int row = sm.rows[g][r];
                        const int dim = la < 4 ? half * kHalf + la * 64 + c * 8 : kDv + 32 * half + 8 * c;
                        cp_async16(dst_of(la, r, la < 4 ? c : 4 * rh + c),
                                   kvb + (size_t)(row >= 0 ? row : 0) * a.kv_tok_b + dim * 2, row >= 0);
                    }
                    cp_async_mbar_arrive_noinc(&sm.kv_full[g]);
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(&sm.kv_full[g]);
                }
                continue;
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
                        const int la = q < 16 ? q >> 2 : 4, cb0 = q < 16 ? (q & 3) * 2 : 4 * rh + (q - 16) * 2;
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
                            uint8_t* dst = dst_of(la, r, c8);
                            *reinterpret_cast<uint4*>(dst) =
                                make_uint4(ow[4 * hh], ow[4 * hh + 1], ow[4 * hh + 2], ow[4 * hh + 3]);
                        }
                    }
                }
            }
            tc::fence_proxy_async_smem();
            tc::mbar_arrive(&sm.kv_full[g]);
        }
        if constexpr (kAsync) cp_async_wait_all();     // no copy outlives the CTA
    } else if (warp == mma_warp) {
        // ---------------- MMA issuer: S_j and P_j V_j, each in order, whichever is ready
        const uint32_t idesc_s = tc::idesc_f16(128, kRows, 1);
        const uint32_t idesc_o = tc::idesc_f16_bmn(128, kHalf, 1);
        const uint32_t qraddr = tc::smem_u32(sm.q_rope);
        if (tc::elect_one() && n_tiles > 0 && tc::mbar_wait(&sm.q_ready, 0, abort_flag)) {
            tc::tc_fence_after();
            int ns = 0, npv = 0;                 // next S tile, next P V tile
            const uint64_t t0 = tc::global_ns();
            uint32_t polls = 0;
            while (npv < n_tiles) {
                bool progressed = false;
                // S_ns needs its KV tile and its S / P buffer free: P V_{ns-4} issued and S_{ns-4}
                // read by the send warps.
                if (ns < n_tiles && ns <= npv + kSP - 1 &&
                    (ns < kSP || tc::mbar_test_wait(&sm.s_sent[ns % kSP], ((ns / kSP) - 1) & 1)) &&
                    tc::mbar_try_wait(&sm.kv_full[ns % kStagesA], (ns / kStagesA) & 1)) {
                    tc::tc_fence_after();
                    tc::fence_proxy_async_smem();    // the tile's cp.async writes, for the tensor cores
                    const int sb = ns % kSP;
                    const int st = ns % kStagesA;
                    const uint32_t kaddr = tc::smem_u32(sm.kv[st]), raddr = tc::smem_u32(sm.rope[st >> 1]);
                    const int rh = half ^ (st & 1);
#pragma unroll
                    for (int kk = 0; kk < kKSteps; ++kk) {
                        if (kk < 16) {                   // V-half dims: A (query) from TMEM
                            const uint64_t bd = tc::sdesc_sw128(kaddr + (kk >> 2) * (kRows * 128) + (kk & 3) * 32);
                            tc::mma_f16_ts(s_col + sb * 32, qt_col + kk * 8, bd, idesc_s, kk > 0);
                        } else {                         // rope dims: A from shared memory
                            const uint64_t ad = tc::sdesc_none(qraddr + (kk - 16) * 256, 128, 512);
                            const uint64_t bd = tc::sdesc_sw128(raddr + (2 * rh + kk - 16) * 32);
                            tc::mma_f16_ss(s_col + sb * 32, ad, bd, idesc_s, 1u);
                        }
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
                    tc::mma_commit(&sm.o_done[npv % kSP]);
                    ++npv;
                    progressed = true;
                }
                if (!progressed && (++polls & 255) == 0) {
                    if (*abort_flag || tc::global_ns() - t0 > tc::kWaitNs * 4) { *abort_flag = 1; break; }
                }
            }
            if (ns > 0) {                           // drain before TMEM is freed (every MMA issued)
                tc::mma_commit(&sm.mma_done);
                volatile int drain_abort = 0;
                tc::mbar_wait(&sm.mma_done, 0, &drain_abort);
            }
        }
    } else if (smx_warp) {
        // ---------------- softmax / epilogue: thread = head = TMEM lane; warpgroup wg takes the
        // tiles j = wg, wg + kSmx, ...
        const int quarter = warp & 3;
        const int h = quarter * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const int xoff = lane * 128;                 // this head's row within a quarter
        float m_w = kNegInf, l_w = 0.f;              // reference max this warpgroup last used, its sum
        bool alive = true;
        if (lane == 0)                               // the first partials may arrive at once
            for (int x = wg; x < kXB && x < n_tiles; x += kSmx) tc::mbar_expect_tx(&sm.rx_full[x][quarter], 4096);
        for (int j = wg; j < n_tiles; j += kSmx) {
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
            // Every lane's tile max depends on every word it read from buffer xb, so once this vote
            // has run the warp's reads of the buffer are complete: the peer may overwrite it (a
            // release arrive would stall the warp for about half a tile's time).  Released this
            // early, the peer's next copy into the buffer is not held up by this tile's softmax.
            {
                uint32_t v;                          // a warp vote on every lane's max (kept by volatile)
                asm volatile("{ .reg .pred p, q; setp.ne.f32 p, %1, %1; vote.sync.any.pred q, p, 0xffffffff; selp.u32 %0, 1, 0, q; }"
                             : "=r"(v) : "f"(mt));
                if (lane == 0) tc::mbar_arrive_remote_relaxed(tc::peer_smem(&sm.tx_free[xb][quarter], peer));
            }
            // The reference max is raised to the tile max only when that exceeds it by more than
            // 2^8 (lazy rescaling).  With two warpgroups the decisions form one chain over the
            // tiles: tile j's starts from tile j-1's, handed over through shared memory.
            float m_prev = m_w;
            if constexpr (kSmx == 2) {
                if (j > 0) {
                    if (!__all_sync(0xffffffffu,
                                    tc::mbar_wait(&sm.hand[wg ^ 1][quarter], ((j - 1) >> 1) & 1, abort_flag))) {
                        alive = false;
                        break;
                    }
                    m_prev = sm.m_ref[h];
                }
            }
            float m_new = m_prev, alpha = 1.f;
            bool rescale = false;
            if (mt > m_prev + 8.f) {
                if (m_prev != kNegInf) { alpha = ex2(m_prev - mt); rescale = true; }
                m_new = mt;
            }
            if constexpr (kSmx == 2) {
                if (j + 1 < n_tiles) {
                    sm.m_ref[h] = m_new;
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(&sm.hand[wg][quarter]);
                }
            }
            if (m_new != m_w) {                          // bring this warpgroup's sum to the new max
                l_w = m_w == kNegInf ? 0.f : l_w * ex2(m_w - m_new);
                m_w = m_new;
            }
            const float mref = m_w == kNegInf ? 0.f : m_w;                // all rows masked so far: p = 0
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
            l_w += ps[0];
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
            if (__any_sync(0xffffffffu, rescale)) {
                // O must hold P V_{j-1} before it is rescaled.
                if (j >= 1 &&
                    !__all_sync(0xffffffffu, tc::mbar_wait(&sm.o_done[(j - 1) % kSP], ((j - 1) / kSP) & 1, abort_flag))) {
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
        // Epilogue: O / l and lse.  The two warpgroups' sums are brought to the final reference max
        // (the larger of their last ones) and added; warpgroup w writes O columns [128w, 128w + 128).
        float m_f = m_w, l_f = l_w;
        if constexpr (kSmx == 2) {
            sm.ml[wg][h] = make_float2(m_w, l_w);
            // One barrier over both warpgroups.  bar.sync is the aligned form: a warp's arrival
            // counts all 32 threads, so the warp must be converged when it arrives -- after the
            // lane-divergent code of the tile loop, __syncwarp makes sure of it.  (Per-quarter
            // barriers of 64 threads without it let a warp read the other's pair before it was
            // written in a fraction of launches.)
            __syncwarp();
            named_bar_sync(6, 2 * 128);
            const float2 o = sm.ml[wg ^ 1][h];
            m_f = fmaxf(m_w, o.x);
            l_f = (m_w == kNegInf ? 0.f : l_w * ex2(m_w - m_f)) + (o.x == kNegInf ? 0.f : o.y * ex2(o.x - m_f));
        }
        if (alive && n_tiles > 0 &&
            !__all_sync(0xffffffffu,
                        tc::mbar_wait(&sm.o_done[(n_tiles - 1) % kSP], ((n_tiles - 1) / kSP) & 1, abort_flag)))
            alive = false;
        tc::tc_fence_after();
        const float kLn2 = 0.69314718055994530942f;
        const float inv = l_f > 0.f ? 1.f / l_f : 0.f;
        const float lse = l_f > 0.f ? (m_f + log2f(l_f)) * kLn2 : kNegInf;
        // The rows go out through shared memory (the idle KV ring; rows padded by 16 B so that
        // consecutive heads fall in different banks), one bulk copy per head row.
        const bool bf16_out = a.n_split == 1 && !a.f32_out;
        const int row_bytes = bf16_out ? kHalf * 2 : kHalf * 4, pitch = row_bytes + 16;
        uint8_t* srow = sm.kv[0] + h * pitch;
        const int c_beg = kSmx == 2 ? wg * (kHalf / 64) : 0, c_end = kSmx == 2 ? c_beg + kHalf / 64 : kHalf / 32;
        for (int c = c_beg; c < c_end; ++c) {
            uint32_t ov[32];
            if (n_tiles > 0 && alive) {
                tc::tmem_ld32(o_col + c * 32 + lane_off, ov);
                tc::tmem_wait_ld();
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) ov[i] = 0u;
            }
            if (bf16_out) {
#pragma unroll
                for (int i = 0; i < 32; i += 8) {
                    uint4 pk;
                    pk.x = pack_bf16x2(__uint_as_float(ov[i]) * inv, __uint_as_float(ov[i + 1]) * inv);
                    pk.y = pack_bf16x2(__uint_as_float(ov[i + 2]) * inv, __uint_as_float(ov[i + 3]) * inv);
                    pk.z = pack_bf16x2(__uint_as_float(ov[i + 4]) * inv, __uint_as_float(ov[i + 5]) * inv);
                    pk.w = pack_bf16x2(__uint_as_float(ov[i + 6]) * inv, __uint_as_float(ov[i + 7]) * inv);
                    *reinterpret_cast<uint4*>(srow + c * 64 + i * 2) = pk;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 32; i += 4)
                    *reinterpret_cast<float4*>(srow + c * 128 + i * 4) =
                        make_float4(__uint_as_float(ov[i]) * inv, __uint_as_float(ov[i + 1]) * inv,
                                    __uint_as_float(ov[i + 2]) * inv, __uint_as_float(ov[i + 3]) * inv);
            }
        }
        tc::fence_proxy_async_smem();
        named_bar_sync(5, kSmx * 128);               // every column of every row is staged
        if (wg == 0) {
            const int dv0 = half * kHalf;
            void* dst = bf16_out ? static_cast<void*>(a.o + ((size_t)t * 128 + h) * kDv + dv0)
                                 : static_cast<void*>(a.part_o + (((size_t)t * a.n_split + split) * 128 + h) * kDv + dv0);
            tc::bulk_store(dst, srow, row_bytes);
            tc::bulk_commit();
            tc::bulk_wait_all();
        }
        if (half == 0 && wg == 0) {
            if (bf16_out) { if (a.lse) a.lse[(size_t)t * 128 + h] = lse; }
            else a.part_lse[((size_t)t * a.n_split + split) * 128 + h] = lse;
        }
    } else if (send_warp) {
        // ---------------- send warps: warp q (mod 4) pushes heads [32q, 32q + 32) of every partial S
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

    __syncwarp();
    if (!remote_warp) tc::cluster_wait();
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
cudaError_t launch_t(const CUtensorMap& qm, const CUtensorMap& m, const CUtensorMap& mt, const AttnArgs& a,
                     cudaStream_t st) {
    const size_t smem = sizeof(AttnSmem) + 1024;
    auto kern = sparse_attn_tc_kernel<KV_FP8, TMA>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(a.n_split, 2, a.T);
    kern<<<grid, kAThreads, smem, st>>>(qm, m, mt, a);
    return cudaGetLastError();
}

// The queries [T][128][576] as a 2-D tensor of T * 128 rows, box 64 dims x 128 heads.
bool make_q_map(const AttnArgs& a, CUtensorMap* m) {
    if (tc::encode_tiled() == nullptr || a.T < 1 || (int64_t)a.T * 128 >= ((int64_t)1 << 31)) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)a.T * 128};
    const cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
    const cuuint32_t box[2] = {64, 128};
    const cuuint32_t estr[2] = {1, 1};
    return tc::encode_tiled()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(a.q), dims, strides, box,
                              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The BF16 cache as one 2-D tensor of rows (row of sequence b, token i = b * (kv_seq_b / kv_tok_b)
// + i), box 64 dims x `box_rows` rows: 1 for tile::gather4, kRows for a tile of consecutive rows.
// False when the layout or the driver does not allow it.
bool make_kv_map(const AttnArgs& a, CUtensorMap* m, int box_rows) {
    if (tc::encode_tiled() == nullptr || a.B < 1 || a.kv_tok_b <= 0 || a.kv_seq_b % a.kv_tok_b != 0) return false;
    const int64_t rps = a.kv_seq_b / a.kv_tok_b;
    const int64_t rows = (int64_t)(a.B - 1) * rps + a.L_alloc;
    if (rows < 1 || rows >= ((int64_t)1 << 31) || (a.B > 1 && rps < 1)) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)a.kv_tok_b};
    const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return tc::encode_tiled()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint8_t*>(a.kv), dims, strides, box,
                              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool sparse_attn_tc_supported(const AttnArgs& a, int DQK, int DV, bool sep_v) {
    return DQK == kD && DV == kDv && !sep_v && a.H == 128 && (a.kv_tok_b % 16) == 0 && (a.kv_seq_b % 16) == 0 &&
           ((uintptr_t)a.kv % 16) == 0 && ((uintptr_t)a.q % 16) == 0 && ((uintptr_t)a.o % 16) == 0 &&
           ((uintptr_t)a.part_o % 16) == 0 && tc::encode_tiled() != nullptr;
}

cudaError_t launch_sparse_attn_tc(const AttnArgs& a, bool kv_fp8, cudaStream_t st) {
    CUtensorMap qm, m, mt;
    memset(&m, 0, sizeof(m));
    memset(&mt, 0, sizeof(mt));
    if (!make_q_map(a, &qm)) return cudaErrorInvalidValue;
    if (kv_fp8) return launch_t<true, false>(qm, m, mt, a, st);
    if (make_kv_map(a, &m, 1) && make_kv_map(a, &mt, kRows)) return launch_t<false, true>(qm, m, mt, a, st);
    memset(&m, 0, sizeof(m));
    memset(&mt, 0, sizeof(mt));
    return launch_t<false, false>(qm, m, mt, a, st);
}

}  // namespace lsa
