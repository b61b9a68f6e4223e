// Indexer scores on the 5th-generation tensor cores (tcgen05), FP8 e4m3 keys with d_I = 128.
//
// Same operation as index_score.cu (LongCat-2.0 release post, section "LongCat 稀疏注意力":
// the lightweight indexer scoring every cached key; DSA form sum_h w_h * ReLU(q_h . k)),
// restated for sm_100a as a persistent kernel, one CTA per SM.
//
// Arithmetic.  The key tile goes to the tensor core as it sits in the cache: 128 e4m3 codes per
// key row, MMA kind::f8f6f4 with A read from shared memory.  Each BF16 query row q_h is scaled by
// a power of two 2^s_h (its largest magnitude into [128, 256)) and split into two e4m3 rows,
// hi = rn(q_h 2^s_h) and lo = rn(q_h 2^s_h - hi).  The residual of a bf16 value after rounding
// to 4 significant bits has at most 4 significant bits, so hi + lo equals q_h 2^s_h exactly for
// every element whose magnitude is at least 2^-10 of the row maximum; smaller elements keep an
// absolute error below 2^-17 of the row maximum.  The MMA runs over K = 256 (the key row twice,
// against hi then lo), so the FP32 accumulator holds 2^s_h (q_h . k); products of e4m3 values are
// exact.  2^-s_h is folded into the head weight.
//
// FP8-query mode (IndexArgs::q_fp8): the query row is hi alone, rn(q_h 2^s_h) 2^-s_h, the
// per-(token, head) e4m3 query of the DSA-style indexer; the MMA runs over K = 128, half the
// tensor-core work.  Scores then differ from the BF16-query ones by the rounding of q.
//
// Scheduling.  Query tokens come in groups of G <= 4 tokens of one sequence (N = G*H_I <= 256
// query rows share every key row).  A group's key range is cut into tiles of NB blocks of 128
// keys (NB = 2, 256-key tiles, for N <= 128; NB = 1 at N = 256); only tiles holding a visible
// key are active.  Every CTA counts the active tiles of all groups, takes an
// equal contiguous share of the concatenated list and runs it through one pipeline.  Tiles of
// one group reuse its prepared queries; a CTA prepares a group's queries once ("epoch"), into
// one of two buffers, so the next group's preparation overlaps the current group's tiles.
//
//   warp 0      : TMA producer -- key tiles (64-row boxes, 128-byte swizzle, which is the
//                 K-major operand layout) and their per-token scales into a KS-stage ring; the
//                 first kEarlyTiles tiles are requested before the first queries are ready;
//                 allocates / frees TMEM.
//   warp 1      : MMA issuer -- per 128-key block, 8 (FP8 queries: 4) x tcgen05.mma kind::f8f6f4
//                 (M = 128 keys, N, K = 32) into one of min(8, 512 / (NB N)) accumulator slots;
//                 its commit frees the key stage.
//   warps 2..3  : query preparation, once per epoch (hi / lo split, 128-byte-swizzled K-major).
//   warps 4..11 : epilogue, two warpgroups taking alternate tiles -- thread = key row (= TMEM
//                 lane): load the accumulator row, apply ReLU, the weighted head sum (eight
//                 partial sums combined in a fixed order) and the token's FP8 scale, store.
//
// Every accumulator slot has a single consumer warpgroup (slot j % slots, an even count), which
// keeps the mbarrier phase parities unambiguous.  All waits are bounded (2 s); a CTA that gives
// up reports LSA_ERR_TIMEOUT and returns after its copies and MMAs in flight have landed and its
// TMEM is freed.
#include <algorithm>
#include <cstring>
#include <mutex>

#include "kernels.cuh"
#include "tc.cuh"

namespace lsa {

namespace {

constexpr int kPThreads = 384;         // 12 warps
constexpr int kPrepThreads = 64;       // warps 2..3
constexpr int kPWarps = kPThreads / 32;
constexpr int kBlock = 128;            // keys per MMA (M); a tile is NB such blocks
constexpr int kBlockBytes = kBlock * 128;
constexpr int kMaxG = 4;
constexpr int kMaxGroups = 2048;       // query-token groups one launch schedules
constexpr int kEarlyTiles = 2;         // key tiles requested before the first queries are ready

struct PArgs {
    IndexArgs a;
    int G, H_I, n_groups, group0;      // groups [group0, group0 + n_groups) of this launch
    int scale_tma;                     // per-token scales arrive by TMA with the keys
};

template <int N, int NB, int KS>
struct PSmem {
    static constexpr int kSlots = (512 / (NB * N)) < 8 ? (512 / (NB * N)) : 8;
    alignas(1024) uint8_t keys[KS][NB * kBlockBytes];
    alignas(1024) uint8_t q[2][2][N * 128];              // [buffer][hi, lo]: B operand, e4m3, SW128
    alignas(16) float scl[KS][NB * kBlock];              // per-token FP8 scales of each key tile
    alignas(16) float w[2][N];                           // head weights times 2^-s
    int pos[2][kMaxG], ok[2][kMaxG];
    int tstart[kMaxGroups + 1];                          // exclusive prefix sums of active tiles
    uint64_t full_k[KS], empty_k[KS];
    uint64_t d_full[kSlots], d_empty[kSlots];
    uint64_t q_full[2], q_free[2][2];                    // q_free[buffer][epilogue warpgroup]
    uint32_t tmem_base;
    int abort;
};

// Walks a CTA's tiles k_lo, k_lo + 1, ...: the group g of the current tile and the CTA-local
// group epoch (0 for the group of tile k_lo, +1 at every change of group).
struct Walk {
    const int* tstart;
    int g, next_b, epoch;
    __device__ Walk(const int* ts, int n_groups, int k) : tstart(ts), epoch(0) {
        int lo = 0, hi = n_groups - 1;                    // the group holding tile k
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (ts[mid + 1] > k) hi = mid; else lo = mid + 1;
        }
        g = lo;
        next_b = ts[g + 1];
    }
    // Moves to tile k (never backwards); true when the group changed.
    __device__ bool to(int k) {
        if (k < next_b) return false;
        do { ++g; next_b = tstart[g + 1]; } while (k >= next_b);
        ++epoch;
        return true;
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

// Two floats to two e4m3 codes (round to nearest even, saturating): x0 in the low byte.
__device__ __forceinline__ uint16_t f32x2_to_e4m3x2(float x0, float x1) {
    uint16_t r;
    asm("{ .reg .b16 t; cvt.rn.satfinite.e4m3x2.f32 t, %1, %2; mov.b16 %0, t; }" : "=h"(r) : "f"(x1), "f"(x0));
    return r;
}

// Decodes two e4m3 codes (low byte first) to floats, exactly.
__device__ __forceinline__ float2 e4m3x2_to_f32x2(uint16_t v) {
    const uint32_t h = e4m3x2_to_f16x2(v);
    return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

// One epoch's query preparation by nthr threads (thread ct; nthr a multiple of 32).  Work item
// i: row n = i / 8 (token
// n / H_I, head n % H_I), 16-element chunk c = i % 8; the 8 chunks of a row sit in 8 consecutive
// lanes, which reduce the row maximum by shuffles.  Loads are issued four items at a time.
// `mid` runs once, after the first batch's loads are issued (the caller's own loads then overlap
// them).  The head weight is loaded with its row.
template <int N, typename Mid>
__device__ void prepare_queries(const IndexArgs& a, int t0, int H_I, int ct, int nthr, uint8_t* q_hi,
                                uint8_t* q_lo, float* w_out, Mid mid) {
    constexpr int kB = 4;
    bool first = true;
    for (int i0 = ct; i0 < N * 8; i0 += nthr * kB) {
        uint4 raw[kB][2];
        float wv[kB];
#pragma unroll
        for (int u = 0; u < kB; ++u) {
            const int i = i0 + u * nthr;
            if (i < N * 8) {                                  // warp-uniform: N * 8 is a multiple of 32
                const int n = i >> 3, c = i & 7;
                const size_t row = (size_t)(t0 + n / H_I) * H_I + n % H_I;
                const uint16_t* src = a.q + row * 128 + c * 16;
                raw[u][0] = *reinterpret_cast<const uint4*>(src);
                raw[u][1] = *reinterpret_cast<const uint4*>(src + 8);
                wv[u] = c == 0 ? a.w[row] : 0.f;
            }
        }
        if (first) { mid(); first = false; }
#pragma unroll
        for (int u = 0; u < kB; ++u) {
            const int i = i0 + u * nthr;
            if (i >= N * 8) break;
            const int n = i >> 3, c = i & 7;
            const uint32_t wd[8] = {raw[u][0].x, raw[u][0].y, raw[u][0].z, raw[u][0].w,
                                    raw[u][1].x, raw[u][1].y, raw[u][1].z, raw[u][1].w};
            float v[16];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                v[2 * e] = bf16_bits_to_float((uint16_t)(wd[e] & 0xffff));
                v[2 * e + 1] = bf16_bits_to_float((uint16_t)(wd[e] >> 16));
            }
            float m = 0.f;
#pragma unroll
            for (int e = 0; e < 16; ++e) m = fmaxf(m, fabsf(v[e]));
#pragma unroll
            for (int o = 1; o < 8; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            // 2^s brings the maximum into [128, 256): s = 7 - floor(log2 m).
            const int ex = (int)((__float_as_uint(m) >> 23) & 0xff) - 127;
            int s = m > 0.f ? 7 - ex : 0;
            s = max(-126, min(126, s));
            const float sc = exp2i(s);
            uint32_t hw[4], lw[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float x0 = v[4 * e] * sc, x1 = v[4 * e + 1] * sc, x2 = v[4 * e + 2] * sc, x3 = v[4 * e + 3] * sc;
                const uint16_t h01 = f32x2_to_e4m3x2(x0, x1), h23 = f32x2_to_e4m3x2(x2, x3);
                const float2 d01 = e4m3x2_to_f32x2(h01), d23 = e4m3x2_to_f32x2(h23);
                // FP8-query mode: the row is its rounded hi part alone (lo is never read).
                const uint16_t l01 = a.q_fp8 ? 0 : f32x2_to_e4m3x2(x0 - d01.x, x1 - d01.y);
                const uint16_t l23 = a.q_fp8 ? 0 : f32x2_to_e4m3x2(x2 - d23.x, x3 - d23.y);
                hw[e] = (uint32_t)h01 | ((uint32_t)h23 << 16);
                lw[e] = (uint32_t)l01 | ((uint32_t)l23 << 16);
            }
            const int off = (n >> 3) * 1024 + (n & 7) * 128 + ((c ^ (n & 7)) << 4);
            *reinterpret_cast<uint4*>(q_hi + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
            *reinterpret_cast<uint4*>(q_lo + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            if (c == 0) w_out[n] = wv[u] * exp2i(-s);
        }
    }
}

// Token gi (< kMaxG) of the group starting at t0: its position, and whether it is a valid query of
// the group's sequence (a token of another sequence, or out of range, sees no key).  In two
// halves -- the token's sequence and position, then its sequence's length -- so that a caller can
// put other loads between them.
struct GroupValidity {
    int b0 = -1, sq = -1, p = -1, len = 0;
    bool in = false;
    __device__ void load(const IndexArgs& a, int t0, int G, int gi) {
        in = gi < G;
        if (in) { b0 = a.q_seq[t0]; sq = a.q_seq[t0 + gi]; p = a.q_pos[t0 + gi]; }
    }
    __device__ void load_len(const IndexArgs& a) {
        if (in && sq == b0 && sq >= 0 && sq < a.B) len = a.seq_len[sq];
    }
    __device__ void store(const IndexArgs& a, int gi, int* pos, int* ok) const {
        const bool okv = in && sq == b0 && sq >= 0 && sq < a.B && len >= 1 && len <= a.L_alloc && p >= 0 && p < len;
        if (in && !okv) report(a.status, LSA_ERR_DEVICE_DATA);
        pos[gi] = okv ? p : -1;
        ok[gi] = okv;
    }
};


// Weighted ReLU head sums of two accumulator rows held by this thread: item a (columns
// ca .. ca + H_I - 1 of the TMEM row, weights wa) and item b (cb, wb; skipped unless `two`).
// Head h goes to partial sum h % 8, two per packed FMA; the eight sums are combined pairwise in a
// fixed order.  The two items are interleaved 32 heads at a time for instruction-level
// parallelism; when both use the same weights (same token) they share the weight loads.
__device__ __forceinline__ void head_sums2(uint32_t ca, uint32_t cb, const float* wa, const float* wb, int H_I,
                                           bool two, float& out_a, float& out_b) {
    float2 aa[4], ab[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) { aa[i] = make_float2(0.f, 0.f); ab[i] = make_float2(0.f, 0.f); }
    const bool same = wa == wb;
    for (int h0 = 0; h0 < H_I; h0 += 32) {
        uint32_t va[32], vb[32];
        tc::tmem_ld32(ca + h0, va);
        if (two) tc::tmem_ld32(cb + h0, vb);
        tc::tmem_wait_ld();
        const float4* pa = reinterpret_cast<const float4*>(wa + h0);
        const float4* pb = reinterpret_cast<const float4*>(wb + h0);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float4 w4 = pa[i];
            aa[(i & 1) * 2] = ffma2(make_float2(w4.x, w4.y),
                                    make_float2(fmaxf(__uint_as_float(va[4 * i]), 0.f), fmaxf(__uint_as_float(va[4 * i + 1]), 0.f)),
                                    aa[(i & 1) * 2]);
            aa[(i & 1) * 2 + 1] = ffma2(make_float2(w4.z, w4.w),
                                        make_float2(fmaxf(__uint_as_float(va[4 * i + 2]), 0.f), fmaxf(__uint_as_float(va[4 * i + 3]), 0.f)),
                                        aa[(i & 1) * 2 + 1]);
            if (two) {
                float4 u4 = w4;
                if (!same) u4 = pb[i];
                ab[(i & 1) * 2] = ffma2(make_float2(u4.x, u4.y),
                                        make_float2(fmaxf(__uint_as_float(vb[4 * i]), 0.f), fmaxf(__uint_as_float(vb[4 * i + 1]), 0.f)),
                                        ab[(i & 1) * 2]);
                ab[(i & 1) * 2 + 1] = ffma2(make_float2(u4.z, u4.w),
                                            make_float2(fmaxf(__uint_as_float(vb[4 * i + 2]), 0.f), fmaxf(__uint_as_float(vb[4 * i + 3]), 0.f)),
                                            ab[(i & 1) * 2 + 1]);
            }
        }
    }
    out_a = ((aa[0].x + aa[0].y) + (aa[1].x + aa[1].y)) + ((aa[2].x + aa[2].y) + (aa[3].x + aa[3].y));
    out_b = ((ab[0].x + ab[0].y) + (ab[1].x + ab[1].y)) + ((ab[2].x + ab[2].y) + (ab[3].x + ab[3].y));
}

template <int N, int NB, int KS>
__global__ void __launch_bounds__(kPThreads, 1)
index_score_tc_kernel(const __grid_constant__ CUtensorMap tmap, const __grid_constant__ CUtensorMap smap,
                      PArgs pa) {
    using Smem = PSmem<N, NB, KS>;
    constexpr int kSlots = Smem::kSlots;
    constexpr int TK = NB * kBlock;                      // keys per tile
    constexpr int SW = NB * N;                           // TMEM columns per accumulator slot
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ int s_tmp[32];
    const IndexArgs& a = pa.a;
    const int G = pa.G, H_I = pa.H_I, NG = pa.n_groups;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool hi = a.cand != nullptr;
    volatile int* abort_flag = &sm.abort;
    const uint64_t wlim = a.wait_ns;                     // pipeline waits; the drains keep tc::kWaitNs

    // ---- set-up: barriers, TMEM, active tiles per group and this CTA's share
    if (threadIdx.x == 0) {
        // A key stage is free once the MMAs reading it have completed (one commit) and the
        // epilogue has read its scales (128 arrivals).
        for (int s = 0; s < KS; ++s) { tc::mbar_init(&sm.full_k[s], 1); tc::mbar_init(&sm.empty_k[s], 129); }
        for (int s = 0; s < kSlots; ++s) { tc::mbar_init(&sm.d_full[s], 1); tc::mbar_init(&sm.d_empty[s], 128); }
        for (int b = 0; b < 2; ++b) {
            tc::mbar_init(&sm.q_full[b], kPrepThreads);
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
        if (hi) {                                        // every group scores all n_cols candidates
            sm.tstart[gl] = a.n_cols > 0 ? (a.n_cols + TK - 1) / TK : 0;
            continue;
        }
        const int t0 = (pa.group0 + gl) * G;
        const int b0 = a.q_seq[t0];
        int max_pos = -1;
        for (int gi = 0; gi < G; ++gi) {
            // The tile count needs no sequence length (one round trip less before the first key
            // tile is requested): a position past its sequence only adds tiles whose columns the
            // epilogue writes as -inf, and is reported where the group's queries are prepared.
            const int s = a.q_seq[t0 + gi], p = a.q_pos[t0 + gi];
            const bool ok = s == b0 && s >= 0 && s < a.B && p >= 0;
            if (ok) max_pos = max(max_pos, p);
            else if (blockIdx.x == 0) report(a.status, LSA_ERR_DEVICE_DATA);
        }
        const int cols = min(a.n_cols, max_pos + 1);
        sm.tstart[gl] = (max_pos < 0 || cols <= 0) ? 0 : (cols + TK - 1) / TK;
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
    const uint32_t d_col = sm.tmem_base;

    // The first group's queries: prepared by the query-preparation and epilogue warps together
    // (the epilogue has nothing to do before the first accumulator is ready).
    if (warp >= 2 && n_mine > 0) {
        const int ct = threadIdx.x - 64;                                // 0..319
        const Walk w0(sm.tstart, NG, k_lo);
        const int t0 = (pa.group0 + w0.g) * G;
        // The validity loads go out with the query loads; the length load, which needs the
        // sequence, after them, so that it overlaps the query arithmetic.
        GroupValidity gv;
        if (ct < kMaxG) gv.load(a, t0, G, ct);
        prepare_queries<N>(a, t0, H_I, ct, kPThreads - 64, sm.q[0][0], sm.q[0][1], sm.w[0],
                           [&] { if (ct < kMaxG) gv.load_len(a); });
        if (ct < kMaxG) gv.store(a, ct, sm.pos[0], sm.ok[0]);
        tc::fence_proxy_async_smem();
        asm volatile("bar.sync 2, %0;" :: "n"(kPThreads - 64) : "memory");
        if (warp < 4) tc::mbar_arrive(&sm.q_full[0]);
    }

    if (warp == 0) {
        // ---------------- TMA producer
        if (tc::elect_one()) {
            Walk wk(sm.tstart, NG, k_lo);
            int t0 = (pa.group0 + wk.g) * G, bseq = max(a.q_seq[t0], 0);
            int s = 0, ph = 0, issued = 0;
            for (int k = k_lo; k < k_hi; ++k) {
                if (wk.to(k)) { t0 = (pa.group0 + wk.g) * G; bseq = max(a.q_seq[t0], 0); }
                // Two key tiles go out at once; the rest of the ring only once the first group's
                // queries are prepared.  Every CTA starts its key stream at the same moment, and a
                // full ring of them (≈24 MB over the GPU) queued ahead of the queries' own loads
                // delayed the first MMA; the tensor pipe cannot start before the queries anyway.
                if (k == k_lo + kEarlyTiles && !tc::mbar_wait(&sm.q_full[0], 0, abort_flag, wlim)) break;
                if (!tc::mbar_wait(&sm.empty_k[s], ph ^ 1, abort_flag, wlim)) break;
                ++issued;
                tc::mbar_expect_tx(&sm.full_k[s], NB * kBlockBytes + (pa.scale_tma ? TK * 4 : 0));
                const int c = (k - sm.tstart[wk.g]) * TK;
#pragma unroll
                for (int i = 0; i < 2 * NB; ++i) {               // 64-row boxes
                    int r0 = c + 64 * i;
                    if (hi) {
                        const int bi = c / 64 + i;
                        const int bk = bi < a.n_cand ? a.cand[(size_t)t0 * a.n_cand + bi] : -1;
                        r0 = bk >= 0 ? bk * 64 : 0;
                    }
                    tc::tma_load_3d(sm.keys[s] + i * (kBlockBytes / 2), &tmap, &sm.full_k[s], 0, r0, bseq);
                    if (pa.scale_tma) tc::tma_load_2d(sm.scl[s] + 64 * i, &smap, &sm.full_k[s], r0, bseq);
                }
                if (++s == KS) { s = 0; ph ^= 1; }
            }
            // Drain: every issued tile has landed before the CTA can exit (bounded; already true
            // unless the consumers gave up early).
            volatile int drain_abort = 0;
            for (int j = max(0, issued - KS); j < issued; ++j)
                tc::mbar_wait(&sm.full_k[j % KS], (j / KS) & 1, &drain_abort);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer: a lean loop (descriptors precomputed; K chunk kk of a
        // 128-byte swizzled row starts kk * 32 bytes in, i.e. 2 * kk in the descriptor's address
        // field, which cannot carry since shared addresses are below 256 KB)
        const uint32_t idesc = tc::idesc_f16(128, N, 0);      // e4m3 x e4m3 -> f32, both K-major
        const int n_k8 = a.q_fp8 ? 4 : 8;                      // FP8-query mode: no lo half
        if (tc::elect_one()) {
            const uint64_t da0 = tc::sdesc_sw128(tc::smem_u32(sm.keys[0]));
            const uint64_t dh0 = tc::sdesc_sw128(tc::smem_u32(sm.q[0][0])), dl0 = tc::sdesc_sw128(tc::smem_u32(sm.q[0][1]));
            const uint64_t dh1 = tc::sdesc_sw128(tc::smem_u32(sm.q[1][0])), dl1 = tc::sdesc_sw128(tc::smem_u32(sm.q[1][1]));
            Walk wk(sm.tstart, NG, k_lo);
            int s = 0, kph = 0, slot = 0, dph = 0, last_slot = -1, last_ph = 0;
            bool alive = n_mine == 0 || tc::mbar_wait(&sm.q_full[0], 0, abort_flag, wlim);
            for (int k = k_lo; alive && k < k_hi; ++k) {
                if (wk.to(k) && !tc::mbar_wait(&sm.q_full[wk.epoch & 1], (wk.epoch >> 1) & 1, abort_flag, wlim)) break;
                if (!tc::mbar_wait(&sm.full_k[s], kph, abort_flag, wlim)) break;
                if (!tc::mbar_wait(&sm.d_empty[slot], dph ^ 1, abort_flag, wlim)) break;
                tc::tc_fence_after();
                const uint64_t dh = (wk.epoch & 1) ? dh1 : dh0, dl = (wk.epoch & 1) ? dl1 : dl0;
#pragma unroll
                for (int b = 0; b < NB; ++b) {                   // block b: keys b*128 .. b*128+127
                    const uint64_t da = da0 + (uint64_t)((s * NB + b) * (kBlockBytes >> 4));
                    const uint32_t dc = d_col + slot * SW + b * N;
#pragma unroll
                    for (int k8 = 0; k8 < 8; ++k8)               // K steps 0..3: q_hi; 4..7: q_lo
                        if (k8 < n_k8)
                            tc::mma_f8_ss(dc, da + 2 * (k8 & 3), (k8 < 4 ? dh : dl) + 2 * (k8 & 3), idesc, k8 > 0);
                }
                tc::mma_commit(&sm.empty_k[s]);
                tc::mma_commit(&sm.d_full[slot]);
                last_slot = slot;
                last_ph = dph;
                if (++s == KS) { s = 0; kph ^= 1; }
                if (++slot == kSlots) { slot = 0; dph ^= 1; }
            }
            if (last_slot >= 0) {                     // drain: issued MMAs complete before TMEM is freed
                volatile int drain_abort = 0;
                tc::mbar_wait(&sm.d_full[last_slot], last_ph, &drain_abort);
            }
        }
    } else if (warp < 4) {
        // ---------------- query preparation, once per group epoch
        const int ct = threadIdx.x - 64;                                // 0..63
        Walk wk(sm.tstart, NG, k_lo);                                   // epoch 0 is prepared above
        for (int k = sm.tstart[wk.g + 1]; k < k_hi; k = sm.tstart[wk.g + 1]) {
            wk.to(k);
            // Group epoch e: its queries go to buffer e & 1 once both epilogue warpgroups have
            // released the group that used the buffer before (epoch e - 2).
            const int e = wk.epoch, qb = e & 1;
            if (e >= 2 && (!tc::mbar_wait(&sm.q_free[qb][0], ((e - 2) >> 1) & 1, abort_flag, wlim) ||
                           !tc::mbar_wait(&sm.q_free[qb][1], ((e - 2) >> 1) & 1, abort_flag, wlim)))
                break;
            const int t0 = (pa.group0 + wk.g) * G;
            GroupValidity gv;
            if (ct < kMaxG) gv.load(a, t0, G, ct);
            prepare_queries<N>(a, t0, H_I, ct, kPrepThreads, sm.q[qb][0], sm.q[qb][1], sm.w[qb],
                               [&] { if (ct < kMaxG) gv.load_len(a); });
            if (ct < kMaxG) gv.store(a, ct, sm.pos[qb], sm.ok[qb]);
            tc::fence_proxy_async_smem();
            tc::mbar_arrive(&sm.q_full[qb]);
        }
    } else {
        // ---------------- epilogue warpgroups: warpgroup wg takes the tiles j with j % 2 == wg
        const int wg = (warp - 4) >> 2;
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const bool fp8 = a.kscale != nullptr;
        Walk wk(sm.tstart, NG, k_lo);
        int t0 = (pa.group0 + wk.g) * G;
        int released = -1, waited = -1;                      // last epoch released / whose queries are known ready
        int s = 0, kph = 0, slot = 0, dph = 0;
        for (int k = k_lo, j = 0; k < k_hi; ++k, ++j) {
            if (wk.to(k)) t0 = (pa.group0 + wk.g) * G;
            const int e = wk.epoch, qb = e & 1;
            // Every tile of this warpgroup before j is done: release the earlier groups' buffers.
            for (; released < e - 1; ++released) tc::mbar_arrive(&sm.q_free[(released + 1) & 1][wg]);
            if ((j & 1) == wg) {
                if (e != waited) {
                    if (!tc::mbar_wait(&sm.q_full[qb], (e >> 1) & 1, abort_flag, wlim)) break;
                    waited = e;
                }
                int col[NB], row[NB];
                float ks[NB];
#pragma unroll
                for (int b = 0; b < NB; ++b) {
                    col[b] = (k - sm.tstart[wk.g]) * TK + b * kBlock + r;
                    row[b] = col[b];
                    if (hi) {
                        const int bi = col[b] / 64;
                        const int blk = (col[b] < a.n_cols && bi < a.n_cand) ? a.cand[(size_t)t0 * a.n_cand + bi] : -1;
                        row[b] = blk >= 0 ? blk * 64 + (col[b] & 63) : -1;
                    }
                }
                if (!tc::mbar_wait(&sm.full_k[s], kph, abort_flag, wlim)) break;
#pragma unroll
                for (int b = 0; b < NB; ++b) {
                    ks[b] = 1.f;
                    if (fp8) {
                        if (pa.scale_tma) ks[b] = sm.scl[s][b * kBlock + r];
                        else if (row[b] >= 0 && row[b] < a.L_alloc)
                            ks[b] = a.kscale[(size_t)max(a.q_seq[t0], 0) * a.scale_seq_stride + row[b]];
                    }
                }
                tc::mbar_arrive(&sm.empty_k[s]);
                if (!tc::mbar_wait(&sm.d_full[slot], dph, abort_flag, wlim)) break;
                tc::tc_fence_after();
                const uint32_t tb = d_col + slot * SW + lane_off;
                const auto store = [&](int gi, int b, float tot) {
                    if (col[b] < a.n_cols) {
                        const bool vis = sm.ok[qb][gi] && row[b] >= 0 && row[b] <= sm.pos[qb][gi];
                        a.scores[(size_t)(t0 + gi) * a.ld + col[b]] = vis ? tot * ks[b] : kNegInf;
                    }
                };
                // Items (block, token), two at a time: both blocks of one token when NB = 2 (same
                // weights), else two tokens of the one block.
                const int n_items = NB * G;
                for (int it = 0; it < n_items; it += 2) {
                    constexpr int ba = 0, bb = NB == 2 ? 1 : 0;
                    const int ga = NB == 2 ? it / 2 : it, gb = NB == 2 ? it / 2 : it + 1;
                    const bool two = it + 1 < n_items;
                    float ta, tv;
                    head_sums2(tb + ba * N + ga * H_I, tb + bb * N + gb * H_I, sm.w[qb] + ga * H_I, sm.w[qb] + gb * H_I,
                               H_I, two, ta, tv);
                    store(ga, ba, ta);
                    if (two) store(gb, bb, tv);
                }
                tc::tc_fence_before();
                tc::mbar_arrive(&sm.d_empty[slot]);
            }
            if (++s == KS) { s = 0; kph ^= 1; }
            if (++slot == kSlots) { slot = 0; dph ^= 1; }
        }
        // Columns past a group's active tiles (all columns of a group with no visible key) are
        // -inf; CTA b fills the groups g with g % grid == b.
        const int et = threadIdx.x - 128;                           // 0..255
        for (int gl = blockIdx.x; gl < NG; gl += gridDim.x) {
            const int tg = (pa.group0 + gl) * G;
            const int from = (sm.tstart[gl + 1] - sm.tstart[gl]) * TK;
            for (int gi = 0; gi < G; ++gi)
                for (int col = from + et; col < a.n_cols; col += 256)
                    a.scores[(size_t)(tg + gi) * a.ld + col] = kNegInf;
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (sm.abort && threadIdx.x == 0) report(a.status, LSA_ERR_TIMEOUT);
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(sm.tmem_base, 512);
    }
}

int num_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 148;
    return n;
}

template <int N, int NB, int KS>
cudaError_t launch_n(const CUtensorMap& m, const CUtensorMap& sm, const PArgs& pa, cudaStream_t st) {
    const size_t smem = sizeof(PSmem<N, NB, KS>) + 1024;
    auto kern = index_score_tc_kernel<N, NB, KS>;
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

namespace tc {

EncodeTiledFn encode_tiled() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

}  // namespace tc

bool index_score_tc_supported(const IndexArgs& a, int H_I, int D_I, bool fp8) {
    if (!fp8 || D_I != 128 || H_I % 32 != 0 || H_I > 128) return false;
    if (a.cand && a.block_size != 64) return false;
    if (a.T % group_size(a, H_I) != 0) return false;
    const int N = group_size(a, H_I) * H_I;
    if (N != 32 && N != 64 && N != 128 && N != 256) return false;
    return ((uintptr_t)a.kdata % 16 == 0) && (a.tok_stride_b % 16 == 0) && (a.seq_stride_b % 16 == 0) &&
           a.kscale != nullptr && tc::encode_tiled() != nullptr;
}

cudaError_t launch_index_score_tc(IndexArgs a, int H_I, cudaStream_t st) {
    if (a.n_cols <= 0 || a.T <= 0) return cudaSuccess;
    PArgs pa{};
    pa.a = a;
    pa.a.wait_ns = wait_limit_ns();
    pa.H_I = H_I;
    pa.G = group_size(a, H_I);
    const int N = pa.G * H_I;

    CUtensorMap m;
    const cuuint64_t dims[3] = {128, (cuuint64_t)a.L_alloc, (cuuint64_t)a.B};
    const cuuint64_t strides[2] = {(cuuint64_t)a.tok_stride_b, (cuuint64_t)a.seq_stride_b};
    const cuuint32_t box[3] = {128, 64, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = tc::encode_tiled()(&m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(a.kdata), dims, strides, box,
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
        r = tc::encode_tiled()(&sc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(a.kscale), sdims, sstr, sbox, sestr,
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
            case 32: e = launch_n<32, 2, 5>(m, sc, pa, st); break;
            case 64: e = launch_n<64, 2, 5>(m, sc, pa, st); break;
            case 128: e = launch_n<128, 2, 4>(m, sc, pa, st); break;
            case 256: e = launch_n<256, 1, 4>(m, sc, pa, st); break;
            default: return cudaErrorInvalidValue;
        }
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace lsa
