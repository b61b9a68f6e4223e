// Indexer scores on the 5th-generation tensor cores (tcgen05), FP8 e4m3 keys with d_I = 128.
//
// Same operation as index_score.cu (LongCat-2.0 release post, section "LongCat 稀疏注意力":
// the lightweight indexer scoring every cached key; DSA form sum_h w_h * ReLU(q_h . k)),
// restated for sm_100a as a persistent kernel, one CTA per SM.
//
// Scheduling.  Query tokens come in groups of G <= 4 tokens of one sequence (N = G*H_I <= 256
// query rows share every key row).  A group's key range is cut into 128-key tiles; only tiles
// holding a visible key are active.  Every CTA counts the active tiles of all groups, takes an
// equal contiguous share of the concatenated list and runs it through one pipeline.  Tiles of
// one group reuse its prepared queries; a CTA prepares a group's queries once ("epoch"), into
// one of two buffers, so the next group's preparation overlaps the current group's tiles.
//
//   warp 0      : TMA producer -- key tiles (two 64-row boxes, 128-byte swizzle) and their
//                 per-token scales into a KS-stage shared-memory ring; allocates / frees TMEM.
//   warp 1      : MMA issuer -- per tile and accumulator slot, 8 x tcgen05.mma kind::f16
//                 (M = 128 keys, N = min(N, 128), K = 16), A from TMEM, B (queries) from smem.
//   warps 2..5  : converters -- thread = key row (= TMEM lane): widen the row's 128 FP8 codes to
//                 f16 (exact) into one of 4 TMEM A stages; at each epoch, prepare the group's
//                 queries: f16 scaled per head by a power of two, 128-byte-swizzled K-major.
//   warps 6..13 : epilogue, two warpgroups -- thread = key row: load the accumulator row, apply
//                 ReLU, the weighted head sum (four partial sums combined in a fixed order) and
//                 the token's FP8 scale, store.
//
// TMEM: 4 A stages x 64 columns, then 256 / min(N, 128) accumulator slots of min(N, 128)
// columns.  N <= 128: tile j uses slot j % slots and the epilogue warpgroups take alternate
// tiles.  N = 256: a tile's two halves go to slots 0 and 1 and warpgroup h always takes half h,
// so the epilogue of one half overlaps the MMA of the other.  Either way every slot has a
// single consumer warpgroup, which keeps the mbarrier phase parities unambiguous.
//
// The power-of-two query scaling is exact for all values within 2^28 of the head's maximum;
// its inverse is folded into the head weight.  Products of f16 values are exact in the FP32
// accumulator.  All waits are bounded (2 s); a CTA that gives up reports LSA_ERR_TIMEOUT and
// returns after its copies and MMAs in flight have landed and its TMEM is freed.
#include <algorithm>
#include <cstring>
#include <mutex>

#include "kernels.cuh"
#include "tc.cuh"

namespace lsa {

namespace {

constexpr int kPThreads = 448;         // 14 warps
constexpr int kPWarps = kPThreads / 32;
constexpr int kTile = 128;             // keys per MMA tile
constexpr int kKeyTileBytes = kTile * 128;
constexpr int kMaxG = 4;
constexpr int kMaxGroups = 2048;       // query-token groups one launch schedules
constexpr int kAStages = 4;            // A-operand (widened keys) stages in TMEM

struct PArgs {
    IndexArgs a;
    int G, H_I, n_groups, group0;      // groups [group0, group0 + n_groups) of this launch
    int scale_tma;                     // per-token scales arrive by TMA with the keys
};

template <int N, int KS>
struct PSmem {
    static constexpr int NS = N < 128 ? N : 128;          // accumulator slot width
    static constexpr int kSub = N / NS;                    // slots per tile
    static constexpr int kSlots = 256 / NS;
    alignas(1024) uint8_t keys[KS][kKeyTileBytes];
    alignas(1024) uint8_t q[2][2][N * 128];              // [buffer][K atom]: B operand, SW128
    alignas(16) float scl[KS][kTile];                    // per-token FP8 scales of each key tile
    alignas(16) float w[2][N];                           // head weights (inverse query scale folded in)
    int pos[2][kMaxG], ok[2][kMaxG];
    int tstart[kMaxGroups + 1];                          // exclusive prefix sums of active tiles
    uint64_t full_k[KS], empty_k[KS], a_full[kAStages], a_empty[kAStages];
    uint64_t d_full[kSlots], d_empty[kSlots];
    uint64_t q_full[2], q_free[2][2];                    // q_free[buffer][epilogue warpgroup]
    uint32_t tmem_base;
    int abort;
};

// Walks a CTA's tiles in order: group, tile within the group, and the CTA-local group epoch.
struct TileCursor {
    const int* tstart;
    int n_groups;
    int g = 0, epoch = -1, lt = 0;
    __device__ void seek(int k) {
        int ng = g;
        if (epoch < 0) {                                  // first tile: binary search
            int lo = 0, hi = n_groups - 1;
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (tstart[mid + 1] > k) hi = mid; else lo = mid + 1;
            }
            ng = lo;
        } else {
            while (tstart[ng + 1] <= k) ++ng;
        }
        if (ng != g || epoch < 0) ++epoch;
        g = ng;
        lt = k - tstart[g];
    }
};

// In place: counts tstart[0..n) -> exclusive prefix sums, tstart[n] = total.  Whole CTA.
__device__ void cta_exclusive_scan(int* tstart, int n, int* s_tmp) {
    const int per = (n + kPThreads - 1) / kPThreads;
    const int lo = min(n, (int)threadIdx.x * per), hi = min(n, lo + per);
    int local = 0;
    for (int i = lo; i < hi; ++i) local += tstart[i];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int v = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += x;
    }
    if (lane == 31) s_tmp[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int x = lane < kPWarps ? s_tmp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane < kPWarps) s_tmp[lane] = x;
    }
    __syncthreads();
    int run = v - local + (warp > 0 ? s_tmp[warp - 1] : 0);
    const int total = s_tmp[kPWarps - 1];
    for (int i = lo; i < hi; ++i) {
        const int c = tstart[i];
        tstart[i] = run;
        run += c;
    }
    if (threadIdx.x == 0) tstart[n] = total;
    __syncthreads();
}

template <int N, int KS>
__global__ void __launch_bounds__(kPThreads, 1)
index_score_tc_kernel(const __grid_constant__ CUtensorMap tmap, const __grid_constant__ CUtensorMap smap,
                      PArgs pa) {
    using Smem = PSmem<N, KS>;
    constexpr int NS = Smem::NS, kSub = Smem::kSub, kSlots = Smem::kSlots;
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ int s_tmp[32];
    const IndexArgs& a = pa.a;
    const int G = pa.G, H_I = pa.H_I, NG = pa.n_groups;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool hi = a.cand != nullptr;
    volatile int* abort_flag = &sm.abort;

    // ---- set-up: barriers, TMEM, active tiles per group and this CTA's share
    if (threadIdx.x == 0) {
        // A key stage is free once the converters have read its keys and the epilogue its scales.
        for (int s = 0; s < KS; ++s) { tc::mbar_init(&sm.full_k[s], 1); tc::mbar_init(&sm.empty_k[s], 128 + 128 * kSub); }
        for (int s = 0; s < kAStages; ++s) { tc::mbar_init(&sm.a_full[s], 128); tc::mbar_init(&sm.a_empty[s], 1); }
        for (int s = 0; s < kSlots; ++s) { tc::mbar_init(&sm.d_full[s], 1); tc::mbar_init(&sm.d_empty[s], 128); }
        for (int b = 0; b < 2; ++b) {
            tc::mbar_init(&sm.q_full[b], 128);
            tc::mbar_init(&sm.q_free[b][0], 128);
            tc::mbar_init(&sm.q_free[b][1], 128);
        }
        sm.abort = 0;
        tc::fence_barrier_init();
        tc::prefetch_tmap(&tmap);
        if (pa.scale_tma) tc::prefetch_tmap(&smap);
    }
    if (warp == 0) tc::tmem_alloc(&sm.tmem_base, 512);
    for (int gl = threadIdx.x; gl < NG; gl += kPThreads) {
        const int t0 = (pa.group0 + gl) * G;
        const int b0 = a.q_seq[t0];
        int max_pos = -1;
        for (int gi = 0; gi < G; ++gi) {
            const int s = a.q_seq[t0 + gi], p = a.q_pos[t0 + gi];
            bool ok = s == b0 && s >= 0 && s < a.B;
            if (ok) {
                const int len = a.seq_len[s];
                ok = len >= 1 && len <= a.L_alloc && p >= 0 && p < len;
            }
            if (ok) max_pos = max(max_pos, p);
            else if (blockIdx.x == 0) report(a.status, LSA_ERR_DEVICE_DATA);
        }
        const int cols = hi ? a.n_cols : min(a.n_cols, max_pos + 1);
        sm.tstart[gl] = (max_pos < 0 || cols <= 0) ? 0 : (cols + kTile - 1) / kTile;
    }
    __syncthreads();
    cta_exclusive_scan(sm.tstart, NG, s_tmp);
    const int total = sm.tstart[NG];
    const int k_lo = (int)((int64_t)blockIdx.x * total / gridDim.x);
    const int k_hi = (int)((int64_t)(blockIdx.x + 1) * total / gridDim.x);
    const int n_mine = k_hi - k_lo;
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const uint32_t a_col = tmem, d_col = tmem + kAStages * 64;

    if (warp == 0) {
        // ---------------- TMA producer
        if (tc::elect_one()) {
            TileCursor cur{sm.tstart, NG};
            int issued = 0;
            for (int j = 0; j < n_mine; ++j) {
                cur.seek(k_lo + j);
                const int s = j % KS;
                if (!tc::mbar_wait(&sm.empty_k[s], ((j / KS) + 1) & 1, abort_flag)) break;
                ++issued;
                const int t0 = (pa.group0 + cur.g) * G;
                const int bseq = max(a.q_seq[t0], 0);
                tc::mbar_expect_tx(&sm.full_k[s], kKeyTileBytes + (pa.scale_tma ? kTile * 4 : 0));
                const int c = cur.lt * kTile;
                int r0 = c, r1 = c + 64;
                if (hi) {
                    const int nb = a.n_cand;
                    const int bk0 = (c / 64) < nb ? a.cand[(size_t)t0 * nb + c / 64] : -1;
                    const int bk1 = (c / 64 + 1) < nb ? a.cand[(size_t)t0 * nb + c / 64 + 1] : -1;
                    r0 = bk0 >= 0 ? bk0 * 64 : 0;
                    r1 = bk1 >= 0 ? bk1 * 64 : 0;
                }
                tc::tma_load_3d(sm.keys[s], &tmap, &sm.full_k[s], 0, r0, bseq);
                tc::tma_load_3d(sm.keys[s] + kKeyTileBytes / 2, &tmap, &sm.full_k[s], 0, r1, bseq);
                if (pa.scale_tma) {
                    tc::tma_load_2d(sm.scl[s], &smap, &sm.full_k[s], r0, bseq);
                    tc::tma_load_2d(sm.scl[s] + 64, &smap, &sm.full_k[s], r1, bseq);
                }
            }
            // Drain: every issued tile has landed before the CTA can exit (bounded; already true
            // unless the consumers gave up early).
            volatile int drain_abort = 0;
            for (int j = max(0, issued - KS); j < issued; ++j)
                tc::mbar_wait(&sm.full_k[j % KS], (j / KS) & 1, &drain_abort);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        const uint32_t idesc = tc::idesc_f16(128, NS, 0);
        if (tc::elect_one()) {
            TileCursor cur{sm.tstart, NG};
            int last_slot = -1, last_ph = 0;
            for (int j = 0; j < n_mine; ++j) {
                const int prev_epoch = cur.epoch;
                cur.seek(k_lo + j);
                const int qb = cur.epoch & 1;
                if (cur.epoch != prev_epoch &&
                    !tc::mbar_wait(&sm.q_full[qb], (cur.epoch >> 1) & 1, abort_flag)) break;
                const int ab = j % kAStages;
                if (!tc::mbar_wait(&sm.a_full[ab], (j / kAStages) & 1, abort_flag)) break;
                const uint32_t q0 = tc::smem_u32(sm.q[qb][0]), q1 = tc::smem_u32(sm.q[qb][1]);
                bool ok = true;
#pragma unroll
                for (int h = 0; h < kSub; ++h) {
                    const int slot = kSub == 2 ? h : j % kSlots, ph = kSub == 2 ? j : j / kSlots;
                    if (!tc::mbar_wait(&sm.d_empty[slot], (ph + 1) & 1, abort_flag)) { ok = false; break; }
                    tc::tc_fence_after();
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint32_t qa = (k < 4 ? q0 : q1) + (k & 3) * 32 + h * NS * 128;
                        tc::mma_f16_ts(d_col + slot * NS, a_col + ab * 64 + k * 8, tc::sdesc_sw128(qa), idesc, k > 0);
                    }
                    tc::mma_commit(&sm.d_full[slot]);
                    last_slot = slot;
                    last_ph = ph;
                }
                if (!ok) break;
                tc::mma_commit(&sm.a_empty[ab]);
            }
            if (last_slot >= 0) {                     // drain: issued MMAs complete before TMEM is freed
                volatile int drain_abort = 0;
                tc::mbar_wait(&sm.d_full[last_slot], last_ph & 1, &drain_abort);
            }
        }
    } else if (warp < 6) {
        // ---------------- converters (thread = TMEM lane = key row) and query preparation
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const int ct = threadIdx.x - 64;                                // 0..127
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        TileCursor cur{sm.tstart, NG};
        for (int j = 0; j < n_mine; ++j) {
            const int prev_epoch = cur.epoch;
            cur.seek(k_lo + j);
            if (cur.epoch != prev_epoch) {
                // New group: its queries go to buffer e & 1 once both epilogue warpgroups have
                // released the group that used the buffer before (epoch e - 2).
                const int e = cur.epoch, qb = e & 1;
                if (e >= 2 && (!tc::mbar_wait(&sm.q_free[qb][0], ((e - 2) >> 1) & 1, abort_flag) ||
                               !tc::mbar_wait(&sm.q_free[qb][1], ((e - 2) >> 1) & 1, abort_flag)))
                    break;
                const int t0 = (pa.group0 + cur.g) * G;
                if (ct < kMaxG) {
                    int okv = 0, p = -1;
                    if (ct < G) {
                        const int b0 = a.q_seq[t0], s = a.q_seq[t0 + ct];
                        p = a.q_pos[t0 + ct];
                        okv = s == b0 && s >= 0 && s < a.B;
                        if (okv) {
                            const int len = a.seq_len[s];
                            okv = len >= 1 && len <= a.L_alloc && p >= 0 && p < len;
                        }
                    }
                    sm.pos[qb][ct] = okv ? p : -1;
                    sm.ok[qb][ct] = okv;
                }
                // Thread ct handles 16-byte chunks ct, ct + 128, ... of the N rows (16 chunks per
                // row, in 16 consecutive lanes that reduce the row maximum by shuffles).
                constexpr int kQB = 4;
                for (int base = ct; base < N * 16; base += 128 * kQB) {
                    uint4 raw[kQB];
#pragma unroll
                    for (int u = 0; u < kQB; ++u) {
                        const int i = base + u * 128;
                        const int rowi = i >> 4;
                        raw[u] = i < N * 16 ? *reinterpret_cast<const uint4*>(
                                                  a.q + ((size_t)(t0 + rowi / H_I) * H_I + rowi % H_I) * 128 + (i & 15) * 8)
                                            : make_uint4(0, 0, 0, 0);
                    }
#pragma unroll
                    for (int u = 0; u < kQB; ++u) {
                        const int i = base + u * 128;
                        if (i >= N * 16) break;                  // warp-uniform: N * 16 is a multiple of 128
                        const int rowi = i >> 4, cc = i & 15;
                        const uint32_t* wd = reinterpret_cast<const uint32_t*>(&raw[u]);
                        float v[8];
#pragma unroll
                        for (int e2 = 0; e2 < 4; ++e2) {
                            v[2 * e2] = bf16_bits_to_float((uint16_t)(wd[e2] & 0xffff));
                            v[2 * e2 + 1] = bf16_bits_to_float((uint16_t)(wd[e2] >> 16));
                        }
                        float m = 0.f;
#pragma unroll
                        for (int e2 = 0; e2 < 8; ++e2) m = fmaxf(m, fabsf(v[e2]));
#pragma unroll
                        for (int o = 1; o < 16; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                        const int ex = (int)((__float_as_uint(m) >> 23) & 0xff) - 127;
                        int k = m > 0.f ? 14 - ex : 0;
                        k = max(-126, min(126, k));
                        const float sc = exp2i(k);
                        uint32_t hv[4];
#pragma unroll
                        for (int e2 = 0; e2 < 4; ++e2)
                            hv[e2] = (uint32_t)__half_as_ushort(__float2half_rn(v[2 * e2] * sc)) |
                                     ((uint32_t)__half_as_ushort(__float2half_rn(v[2 * e2 + 1] * sc)) << 16);
                        const int atom = cc >> 3, c16 = cc & 7;
                        uint8_t* dst = sm.q[qb][atom] + (rowi >> 3) * 1024 + (rowi & 7) * 128 + ((c16 ^ (rowi & 7)) << 4);
                        *reinterpret_cast<uint4*>(dst) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
                        if (cc == 0) sm.w[qb][rowi] = a.w[(size_t)(t0 + rowi / H_I) * H_I + rowi % H_I] * exp2i(-k);
                    }
                }
                tc::fence_proxy_async_smem();
                tc::mbar_arrive(&sm.q_full[qb]);
            }
            const int s = j % KS, ab = j % kAStages;
            if (!tc::mbar_wait(&sm.full_k[s], (j / KS) & 1, abort_flag)) break;
            const uint8_t* rowp = sm.keys[s] + r * 128;          // 128-byte rows, 16-byte chunks XOR-swizzled
            uint4 ch[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) ch[c] = *reinterpret_cast<const uint4*>(rowp + ((c ^ (r & 7)) << 4));
            tc::mbar_arrive(&sm.empty_k[s]);
            if (!tc::mbar_wait(&sm.a_empty[ab], ((j / kAStages) + 1) & 1, abort_flag)) break;
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
        // ---------------- epilogue warpgroups: N <= 128, warpgroup wg takes the tiles j with
        // j % 2 == wg; N = 256, it takes half wg of every tile
        const int wg = (warp - 6) >> 2;
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const bool fp8 = a.kscale != nullptr;
        const int tps = NS / H_I;                            // query tokens per accumulator slot
        TileCursor cur{sm.tstart, NG};
        int released = -1, waited = -1;                      // last epoch released / whose queries are known ready
        for (int j = 0; j < n_mine; ++j) {
            cur.seek(k_lo + j);
            const int e = cur.epoch, qb = e & 1;
            // Every tile of this warpgroup before j is done: release the earlier groups' buffers.
            for (; released < e - 1; ++released) tc::mbar_arrive(&sm.q_free[(released + 1) & 1][wg]);
            if (kSub == 1 && (j & 1) != wg) continue;
            if (e != waited) {
                if (!tc::mbar_wait(&sm.q_full[qb], (e >> 1) & 1, abort_flag)) break;
                waited = e;
            }
            const int s = j % KS;
            const int t0 = (pa.group0 + cur.g) * G;
            const int col = cur.lt * kTile + r;
            int row = col;
            if (hi) {
                const int bi = col / 64;
                const int blk = (col < a.n_cols && bi < a.n_cand) ? a.cand[(size_t)t0 * a.n_cand + bi] : -1;
                row = blk >= 0 ? blk * 64 + (col & 63) : -1;
            }
            if (!tc::mbar_wait(&sm.full_k[s], (j / KS) & 1, abort_flag)) break;
            float ks = 1.f;
            if (fp8) {
                if (pa.scale_tma) ks = sm.scl[s][r];
                else if (row >= 0 && row < a.L_alloc) ks = a.kscale[(size_t)max(a.q_seq[t0], 0) * a.scale_seq_stride + row];
            }
            tc::mbar_arrive(&sm.empty_k[s]);
            {
                const int h = kSub == 2 ? wg : 0;
                const int slot = kSub == 2 ? wg : j % kSlots, ph = kSub == 2 ? j : j / kSlots;
                if (!tc::mbar_wait(&sm.d_full[slot], ph & 1, abort_flag)) break;
                tc::tc_fence_after();
                for (int ti = 0; ti < tps; ++ti) {
                    const int gi = h * tps + ti;
                    // Four partial sums (head h goes to sum h % 4), two per packed FMA.
                    float2 acc01 = make_float2(0.f, 0.f), acc23 = make_float2(0.f, 0.f);
                    for (int h0 = 0; h0 < H_I; h0 += 32) {
                        uint32_t v[32];
                        tc::tmem_ld32(d_col + slot * NS + ti * H_I + h0 + lane_off, v);
                        tc::tmem_wait_ld();
                        const float4* wp = reinterpret_cast<const float4*>(sm.w[qb] + gi * H_I + h0);
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const float4 ww = wp[i];
                            acc01 = ffma2(make_float2(ww.x, ww.y),
                                          make_float2(fmaxf(__uint_as_float(v[4 * i + 0]), 0.f),
                                                      fmaxf(__uint_as_float(v[4 * i + 1]), 0.f)), acc01);
                            acc23 = ffma2(make_float2(ww.z, ww.w),
                                          make_float2(fmaxf(__uint_as_float(v[4 * i + 2]), 0.f),
                                                      fmaxf(__uint_as_float(v[4 * i + 3]), 0.f)), acc23);
                        }
                    }
                    const float tot = (acc01.x + acc01.y) + (acc23.x + acc23.y);
                    if (col < a.n_cols) {
                        const bool vis = sm.ok[qb][gi] && row >= 0 && row <= sm.pos[qb][gi];
                        a.scores[(size_t)(t0 + gi) * a.ld + col] = vis ? tot * ks : kNegInf;
                    }
                }
                tc::tc_fence_before();
                tc::mbar_arrive(&sm.d_empty[slot]);
            }
        }
        // Columns past a group's active tiles (all columns of a group with no visible key) are
        // -inf; CTA b fills the groups g with g % grid == b.
        const int et = threadIdx.x - 192;                           // 0..255
        for (int gl = blockIdx.x; gl < NG; gl += gridDim.x) {
            const int t0 = (pa.group0 + gl) * G;
            const int from = (sm.tstart[gl + 1] - sm.tstart[gl]) * kTile;
            for (int gi = 0; gi < G; ++gi)
                for (int col = from + et; col < a.n_cols; col += 256)
                    a.scores[(size_t)(t0 + gi) * a.ld + col] = kNegInf;
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

int num_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 148;
    return n;
}

template <int N, int KS>
cudaError_t launch_n(const CUtensorMap& m, const CUtensorMap& sm, const PArgs& pa, cudaStream_t st) {
    const size_t smem = sizeof(PSmem<N, KS>) + 1024;
    auto kern = index_score_tc_kernel<N, KS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<num_sms(), kPThreads, smem, st>>>(m, sm, pa);
    return cudaGetLastError();
}

int group_size(const IndexArgs& a, int H_I) {
    if (a.cand) return 1;
    int G = a.q_group % 4 == 0 ? 4 : (a.q_group % 2 == 0 ? 2 : 1);
    while (G > 1 && G * H_I > 256) G >>= 1;
    return G;
}

}  // namespace

bool index_score_tc_supported(const IndexArgs& a, int H_I, int D_I, bool fp8) {
    if (!fp8 || D_I != 128 || H_I % 32 != 0 || H_I > 128) return false;
    if (a.cand && a.block_size != 64) return false;
    if (a.T % group_size(a, H_I) != 0) return false;
    const int N = group_size(a, H_I) * H_I;
    if (N != 32 && N != 64 && N != 128 && N != 256) return false;
    return ((uintptr_t)a.kdata % 16 == 0) && (a.tok_stride_b % 16 == 0) && (a.seq_stride_b % 16 == 0) &&
           a.kscale != nullptr && encode_fn() != nullptr;
}

cudaError_t launch_index_score_tc(IndexArgs a, int H_I, cudaStream_t st) {
    if (a.n_cols <= 0 || a.T <= 0) return cudaSuccess;
    PArgs pa{};
    pa.a = a;
    pa.H_I = H_I;
    pa.G = group_size(a, H_I);
    const int N = pa.G * H_I;

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
    pa.scale_tma = ((uintptr_t)a.kscale % 16 == 0) && (a.scale_seq_stride % 4 == 0) && a.scale_seq_stride > 0;
    CUtensorMap sc;
    memset(&sc, 0, sizeof(sc));
    if (pa.scale_tma) {
        const cuuint64_t sdims[2] = {(cuuint64_t)a.L_alloc, (cuuint64_t)a.B};
        const cuuint64_t sstr[1] = {(cuuint64_t)a.scale_seq_stride * 4};
        const cuuint32_t sbox[2] = {64, 1};
        const cuuint32_t sestr[2] = {1, 1};
        r = encode_fn()(&sc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(a.kscale), sdims, sstr, sbox, sestr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) { pa.scale_tma = 0; memset(&sc, 0, sizeof(sc)); }
    }
    const int total_groups = a.T / pa.G;
    for (int g0 = 0; g0 < total_groups; g0 += kMaxGroups) {
        pa.group0 = g0;
        pa.n_groups = std::min(kMaxGroups, total_groups - g0);
        cudaError_t e;
        switch (N) {
            case 32: e = launch_n<32, 8>(m, sc, pa, st); break;
            case 64: e = launch_n<64, 8>(m, sc, pa, st); break;
            case 128: e = launch_n<128, 8>(m, sc, pa, st); break;
            case 256: e = launch_n<256, 4>(m, sc, pa, st); break;
            default: return cudaErrorInvalidValue;
        }
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace lsa
