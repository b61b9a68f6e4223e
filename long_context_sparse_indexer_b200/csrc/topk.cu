// Top-k selection with the SI window and the sink tokens.
//
// Explainer page ("如何在 5 万张国产芯片训练出 1.6T 万亿参数模型？"), section "① LSA": each query
// reads only its top-k keys plus a few fixed sink tokens.  Release post, section
// "LongCat 稀疏注意力", SI bullet: the selection budget mixes a hardware-aligned contiguous
// part with the dynamic top-k picks.  The order on equal scores is the lower position
// first, which makes the selection unique and the output deterministic.
//
// Method: radix select on the order-preserving 32-bit key of each score, 12 + 12 + 8 bits.
// One query row is handled by a cluster of NC CTAs (8 for a few rows, 2 or 4 for many: see
// launch_topk); CTA r owns the r-th contiguous segment of the row (cached in shared memory as
// order keys when it has at most 40960 columns, else re-read from global memory).  Histograms
// are integer shared-memory counts (atomics; counts do not depend on atomic order).
//   1. Top 12 bits over the cluster: each CTA folds its 4096 bins into 64 super-bins; after one
//      cluster barrier every CTA reads the NC x 64 super-bin counts, then the NC x 64 bins inside
//      the threshold super-bin, through distributed shared memory, and finds the same bin b1.
//      When the keys at or above b1 would overflow the per-warp candidate lists, the next 12
//      bits are settled over the cluster as well, and the listing threshold becomes (b1, b2).
//   2. The keys at or above the threshold (usually a few thousand, about k after the second
//      digit) are compacted, in column order, into CTA 0's shared memory; CTA 0 alone finds the
//      next 12 and the last 8 bits, i.e. the k-th key v* and the number m of ties at v* to keep,
//      and emits every key > v* and the first m keys == v* (lowest columns first) in one walk:
//      each warp stages its kept positions in shared memory, and they are copied out at their
//      offsets after a prefix over the warps' counts.  When the candidates do not fit, the
//      cluster runs passes 2 and 3 over its segments and emits with cluster-wide prefix counts
//      instead.
// Positions are written in ascending order and merged with the sinks [0, a) and the window
// [b, pos], so the list comes out sorted and de-duplicated.  Fixed-budget mode: sink and window
// positions are no candidates at all, so the top-k is drawn from the other positions and the
// list holds exactly min(k, those) + a + (pos + 1 - b) entries.
#include <algorithm>
#include <cooperative_groups.h>

#include "kernels.cuh"
#include "tc.cuh"

namespace cg = cooperative_groups;

namespace lsa {

constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kTopkCluster = 8;

// First position of the SI window: pos - window + 1 clipped at 0, rounded down to a multiple of
// `align` when align > 0 (the block-aligned window).
__device__ __forceinline__ int window_start(int pos, int window, int align) {
    const int b = max(0, pos - window + 1);
    return align > 0 ? b - b % align : b;
}

// Inclusive prefix sum over the CTA (warp shuffles + one shared array of warp totals).
__device__ __forceinline__ int cta_inclusive_scan(int v, int* s_warp, int& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    if (lane == 31) s_warp[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int x = lane < kTopkWarps ? s_warp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += n;
        }
        if (lane < kTopkWarps) s_warp[lane] = x;
    }
    __syncthreads();
    total = s_warp[kTopkWarps - 1];
    const int res = v + (warp > 0 ? s_warp[warp - 1] : 0);
    __syncthreads();
    return res;
}

// Adds 1 to hist[bin] for every lane with `on` (shared-memory integer atomics).
__device__ __forceinline__ void hist_add(int* hist, int bin, bool on) {
    if (on) atomicAdd(&hist[bin], 1);
}

// Sums the histograms of all CTAs of the cluster into `sum` in every CTA, then finds the bin
// where the count from the top first reaches `need` (identical in every CTA).  CTA r adds up
// the r-th of NC equal shares of the bins over the cluster (distributed shared memory loads)
// and writes the sums into every CTA's `sum` (distributed shared memory stores).
template <int NC>
__device__ int cluster_threshold(cg::cluster_group& cl, int rank, int* hist, int* sum, int nb, int need,
                                 int* s_warp, int* s_bin, int* s_above) {
    cl.sync();                                           // all local histograms complete
    const int share = nb / NC;
    for (int i = threadIdx.x; i < share; i += kTopkThreads) {
        const int bin = rank * share + i;
        int v[NC];
#pragma unroll
        for (int r = 0; r < NC; ++r) v[r] = cl.map_shared_rank(hist, r)[bin];
        int s = 0;
#pragma unroll
        for (int r = 0; r < NC; ++r) s += v[r];
#pragma unroll
        for (int r = 0; r < NC; ++r) cl.map_shared_rank(sum, r)[bin] = s;
    }
    cl.sync();                                           // sums everywhere; peers done reading `hist`
    const int per = (nb + kTopkThreads - 1) / kTopkThreads;     // bins per thread, from the top
    int local = 0;
    for (int i = 0; i < per; ++i) {
        const int bin = nb - 1 - ((int)threadIdx.x * per + i);
        if (bin >= 0) local += sum[bin];
    }
    int total;
    const int incl = cta_inclusive_scan(local, s_warp, total);
    int run = incl - local;
    for (int i = 0; i < per; ++i) {
        const int bin = nb - 1 - ((int)threadIdx.x * per + i);
        if (bin < 0) break;
        const int h = sum[bin];
        if (run < need && run + h >= need) { *s_bin = bin; *s_above = run; }
        run += h;
    }
    __syncthreads();
    return total;
}

// One warp: over 64 counts c[0..63] taken from the top (index 63 first) after `base` counts
// above them, the index where the running count first reaches `need` (run < need <= run + c)
// and the count above it; lane 0 writes them to *bin / *above (-1 / unchanged when there is
// none) and, if `total` is given, the sum of the 64 counts to *total.
__device__ __forceinline__ void top_crossing(const int* c, int base, int need, int* bin, int* above, int* total) {
    const int lane = threadIdx.x & 31;
    const int hi = c[63 - 2 * lane], lo = c[62 - 2 * lane];
    int incl = hi + lo;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    const int run = base + incl - hi - lo;
    int found = -1, fa = 0;
    if (run < need && run + hi >= need) { found = 63 - 2 * lane; fa = run; }
    else if (run + hi < need && run + hi + lo >= need) { found = 62 - 2 * lane; fa = run + hi; }
    const uint32_t m = __ballot_sync(0xffffffffu, found >= 0);
    const int src = m ? __ffs(m) - 1 : 0;
    const int f = __shfl_sync(0xffffffffu, found, src), a = __shfl_sync(0xffffffffu, fa, src);
    const int tot = __shfl_sync(0xffffffffu, incl, 31);
    if (lane == 0) {
        *bin = m ? f : -1;
        if (m) *above = a;
        if (total) *total = tot;
    }
}

// Two-level form of cluster_threshold for the 4096-bin histogram of the top 12 bits, with one
// cluster barrier.  Each CTA folds its histogram into 64 super-bins of 64 bins (`sup`); after
// the barrier every CTA reads the cluster's NC x 64 super-bin counts, finds the super-bin where
// the count from the top reaches `need`, then reads the NC x 64 bin counts inside it and finds
// the bin (the same rule, so the same bin, as the one-level form).  Peers read `hist` and `sup`
// after this returns: the caller must pass another cluster barrier before changing either.
// Returns the cluster's total count; *s_bin / *s_above are left unchanged when no bin reaches
// `need` (need <= 0 or need > total).
template <int NC>
__device__ int cluster_threshold_4096(cg::cluster_group& cl, const int* hist, int* sup, int need, int* s_red,
                                      int* s_bin, int* s_above, int* s_total) {
    const int t = threadIdx.x, lane = t & 31;
    static_assert(kTopkThreads == 512 && NC >= 1 && NC <= 8 && (NC & (NC - 1)) == 0,
                  "one thread per 8 bins, 8 lanes per super-bin (lanes past the cluster size add 0)");
    __syncthreads();                                     // the local histogram is complete
    {
        int s = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) s += hist[8 * t + i];
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        s += __shfl_xor_sync(0xffffffffu, s, 4);
        if ((t & 7) == 0) sup[t >> 3] = s;
    }
    cl.sync();                                           // every CTA's histogram and super-bins complete
    // Thread t: super-bin t >> 3 of CTA t & 7; the 8 lanes of a super-bin add up the CTAs.
    {
        int v = (t & 7) < NC ? cl.map_shared_rank(sup, t & 7)[t >> 3] : 0;
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        if ((t & 7) == 0) s_red[t >> 3] = v;
    }
    __syncthreads();
    // Warp 0 walks the 64 totals from the top (lane l: super-bins 63 - 2l and 62 - 2l).
    if (t < 32) top_crossing(s_red, 0, need, s_red + 64, s_red + 65, s_total);
    __syncthreads();
    const int sb = s_red[64];
    if (sb >= 0) {
        // Thread t: bin 64 sb + (t >> 3) of CTA t & 7.
        int v = (t & 7) < NC ? cl.map_shared_rank(hist, t & 7)[64 * sb + (t >> 3)] : 0;
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        if ((t & 7) == 0) s_red[66 + (t >> 3)] = v;
        __syncthreads();
        if (t < 32) {
            int bin = -1, above = 0;
            top_crossing(s_red + 66, s_red[65], need, &bin, &above, nullptr);
            if (lane == 0 && bin >= 0) { *s_bin = 64 * sb + bin; *s_above = above; }
        }
    }
    __syncthreads();
    return *s_total;
}

// Cluster-wide exclusive prefix of one int per CTA (the value in `slot` of each CTA).  Every
// exchange uses its own slot, so the slot is never rewritten while a peer may still read it.
template <int NC>
__device__ int cluster_exclusive(cg::cluster_group& cl, int* slot, int rank, int& total) {
    cl.sync();
    int before = 0;
    total = 0;
    for (int r = 0; r < NC; ++r) {
        const int v = *cl.map_shared_rank(slot, r);
        if (r < rank) before += v;
        total += v;
    }
    return before;
}

// Within one CTA: finds the bin of `hist` where the count from the top first reaches `need`
// (same rule as cluster_threshold, CTA barriers only).
__device__ void local_threshold(const int* hist, int nb, int need, int* s_warp, int* s_bin, int* s_above) {
    const int per = (nb + kTopkThreads - 1) / kTopkThreads;
    int local = 0;
    for (int i = 0; i < per; ++i) {
        const int bin = nb - 1 - ((int)threadIdx.x * per + i);
        if (bin >= 0) local += hist[bin];
    }
    int total;
    const int incl = cta_inclusive_scan(local, s_warp, total);
    int run = incl - local;
    for (int i = 0; i < per; ++i) {
        const int bin = nb - 1 - ((int)threadIdx.x * per + i);
        if (bin < 0) break;
        const int h = hist[bin];
        if (run < need && run + h >= need) { *s_bin = bin; *s_above = run; }
        run += h;
    }
    __syncthreads();
}

// Segment length (columns) a CTA caches in shared memory as order keys.
constexpr int kTopkCacheCols = 40960;
// Candidate block ids of a row kept in shared memory (HI: the recalled blocks).
constexpr int kTopkCandCache = 1024;
// Candidate lists of the compacted finish: per CTA (in its `hsum` array) and merged in CTA 0.
// Above kTopkRefine expected candidates per warp the listing waits for the second radix digit.
constexpr int kTopkRefine = 96;
constexpr int kTopkLocalCap = 2048;
constexpr int kTopkWarpCap = kTopkLocalCap / kTopkWarps;   // per warp
constexpr int kTopkCap = 8192;

template <bool CACHED, int NC>
__global__ void __cluster_dims__(NC, 1, 1) __launch_bounds__(kTopkThreads, 2)
topk_kernel(TopkArgs a) {
    __shared__ int hist[4096];
    __shared__ int hsum[4096];
    __shared__ int s_warp[kTopkWarps];
    __shared__ int s_bin, s_above, s_slot[3], s_wmax;
    __shared__ int s_wcnt[kTopkWarps], s_wk[kTopkWarps];
    __shared__ int s_sup[64], s_red[130], s_total, hist3[256];
    __shared__ int s_cand[kTopkCandCache];        // the row's candidate block ids (HI), when they fit
    extern __shared__ uint32_t s_keys[];          // CACHED: order key of each column of the segment, 0 = invalid
    __shared__ uint64_t s_seg_full;               // CACHED: the segment's bulk copy has landed
    __shared__ int s_abort;
    cg::cluster_group cl = cg::this_cluster();
    const int rank = (int)cl.block_rank();
    const int t = blockIdx.x / NC;
    const float* row = a.scores + (size_t)t * a.ld;
    int32_t* out = a.idx + (size_t)t * a.ld_idx;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

    // Query position and its validity (identical in every CTA of the cluster).
    const int b = a.q_seq[t];
    const int pos = a.q_pos[t];
    bool ok = b >= 0 && b < a.B;
    if (ok) {
        const int len = a.seq_len[b];
        ok = len >= 1 && len <= a.L_alloc && pos >= 0 && pos < len;
    }
    if (!ok) {
        if (rank == 0) {
            if (threadIdx.x == 0) { report(a.status, LSA_ERR_DEVICE_DATA); a.count[t] = 0; }
            for (int i = threadIdx.x; i < a.ld_idx; i += kTopkThreads) out[i] = -1;
        }
        return;
    }

    // This CTA's segment, split further into contiguous warp segments (multiples of 32).
    const int per_cta = ((a.n_cols + NC - 1) / NC + 31) / 32 * 32;
    const int c0 = min(a.n_cols, rank * per_cta), c1 = min(a.n_cols, c0 + per_cta);
    const int per_warp = ((c1 - c0 + kTopkWarps - 1) / kTopkWarps + 31) / 32 * 32;
    const int w0 = min(c1, c0 + warp * per_warp), w1 = min(c1, w0 + per_warp);

    // Sinks [0, a_lo) and window [b_hi, pos] (positions), and the position of column cc.
    const int a_lo = a.raw ? 0 : min(a.n_sink, pos + 1);
    const int b_hi = a.raw ? 0x7fffffff : (a.window > 0 ? max(a_lo, window_start(pos, a.window, a.window_align)) : pos + 1);
    // Column -> position through the candidate blocks: from shared memory when they fit (the
    // emission maps every kept column; a dependent global load there would serialise its walks),
    // with shifts for a power-of-two block size.
    const bool cand_cached = !a.raw && a.cand && a.n_cand <= kTopkCandCache;
    const int bs_log = (a.block_size > 0 && (a.block_size & (a.block_size - 1)) == 0) ? __ffs(a.block_size) - 1 : -1;
    if (cand_cached) {                                // uniform over the CTA
        for (int i = threadIdx.x; i < a.n_cand; i += kTopkThreads) s_cand[i] = a.cand[(size_t)t * a.n_cand + i];
        __syncthreads();
    }
    auto position = [&](int cc) -> int {
        if (a.raw || !a.cand) return cc;
        const int bi = bs_log >= 0 ? cc >> bs_log : cc / a.block_size;
        const int off = bs_log >= 0 ? cc & (a.block_size - 1) : cc % a.block_size;
        const int blk = cand_cached ? s_cand[bi] : a.cand[(size_t)t * a.n_cand + bi];
        return blk * a.block_size + off;
    };
    // Fixed-budget selection: a column at a sink or window position is no candidate.
    auto fixed_pos = [&](int cc) -> bool {
        if (!a.fixed_budget) return false;
        const int p = position(cc);
        return p < a_lo || p >= b_hi;
    };

    // Order key of column cc of this warp's segment (0 = not a candidate; valid keys are > 0).
    auto key_at = [&](int cc) -> uint32_t {
        if (cc >= w1) return 0u;
        if (CACHED) return s_keys[cc - c0];
        const float f = row[cc];
        return (f != f || f == kNegInf || fixed_pos(cc)) ? 0u : order_key(f);
    };

    // ---- pass 1: top 12 bits (and, when cached, the segment's keys into shared memory)
    for (int i = threadIdx.x; i < 4096; i += kTopkThreads) hist[i] = 0;
    if (CACHED) {
        // The segment comes into shared memory as raw scores by one bulk copy (its 16-byte
        // multiple; the ragged tail, or a row not 16-byte aligned, by plain loads), then every
        // thread turns its columns into order keys in place and counts them in the same sweep.
        // One round trip instead of a register round trip per batch of loads, and one sweep of
        // the segment instead of two.
        const int n_seg = c1 - c0;
        const bool vec = (((uintptr_t)(row + c0)) & 15) == 0;
        const int n_bulk = vec ? (n_seg & ~3) : 0;
        if (threadIdx.x == 0) {
            s_abort = 0;
            if (n_bulk > 0) {
                tc::mbar_init(&s_seg_full, 1);
                tc::fence_barrier_init();
            }
        }
        __syncthreads();                                 // hist cleared, the barrier initialised
        if (threadIdx.x == 0 && n_bulk > 0) {
            tc::mbar_expect_tx(&s_seg_full, (uint32_t)n_bulk * 4);
            tc::bulk_load(s_keys, row + c0, (uint32_t)n_bulk * 4, &s_seg_full);
        }
        for (int i = n_bulk + threadIdx.x; i < n_seg; i += kTopkThreads) s_keys[i] = __float_as_uint(row[c0 + i]);
        if (n_bulk > 0 && !tc::mbar_wait(&s_seg_full, 0, &s_abort) && threadIdx.x == 0)
            report(a.status, LSA_ERR_TIMEOUT);           // the keys are then not the row's; every CTA goes on
        __syncthreads();                                 // the tail's plain stores
        for (int i = threadIdx.x; i < n_seg; i += kTopkThreads) {
            const float x = __uint_as_float(s_keys[i]);
            if (x != x) report(a.status, LSA_ERR_DEVICE_DATA);
            const uint32_t key = (x != x || x == kNegInf || fixed_pos(c0 + i)) ? 0u : order_key(x);
            s_keys[i] = key;
            hist_add(hist, (int)(key >> 20), key != 0u);
        }
    } else {
        __syncthreads();
        for (int c = w0; c < w1; c += 32) {
            const int cc = c + lane;
            if (cc < w1) {
                const float f = row[cc];
                if (f != f) report(a.status, LSA_ERR_DEVICE_DATA);
            }
            const uint32_t key = key_at(cc);
            hist_add(hist, (int)(key >> 20), key != 0u);
        }
    }
    // Cluster histogram of the top 12 bits; its total is the number of candidates.
    const int n_valid = cluster_threshold_4096<NC>(cl, hist, s_sup, a.k, s_red, &s_bin, &s_above, &s_total);
    const bool take_all = n_valid <= a.k;
    uint32_t tb = a.k <= 0 ? 0xffffffffu : (take_all ? 1u : ((uint32_t)s_bin << 20));   // listing threshold

    // ---- refinement before the listing.  When the keys at or above the threshold bin b1 would
    // fill more than kTopkRefine slots per warp on average (a wide bin, few warps per row: the
    // per-warp lists would overflow and the row would take the full passes), the next 12 bits
    // are settled first over the cluster, and only keys at or above (b1, b2) are listed.  The
    // counts are the cluster's, so every CTA takes the same branch.  CTA 0's finish then finds b2
    // again from the candidates (all keys of bin b1 at or above it are among them).
    if (!take_all && a.k > 0) {
        const uint32_t b1 = (uint32_t)s_bin;
        const int above1 = s_above;
        const int b1_count = s_red[66 + (b1 & 63)];              // the cluster's keys in bin b1
        if ((above1 + b1_count) / (NC * kTopkWarps) > kTopkRefine) {
            cl.sync();                                           // peers are done reading hist / sup
            for (int i = threadIdx.x; i < 4096; i += kTopkThreads) hist[i] = 0;
            __syncthreads();
            for (int c = w0; c < w1; c += 32) {
                const uint32_t key = key_at(c + lane);
                hist_add(hist, (int)((key >> 8) & 0xfff), key != 0u && (key >> 20) == b1);
            }
            cluster_threshold<NC>(cl, rank, hist, hsum, 4096, a.k - above1, s_warp, &s_bin, &s_above);
            tb = (b1 << 20) | ((uint32_t)s_bin << 8);
            __syncthreads();                                     // every thread has read b2
            if (threadIdx.x == 0) { s_bin = (int)b1; s_above = above1; }   // pass 1's, for what follows
            __syncthreads();
        }
    }

    // ---- compacted finish.  The top-k lies in the threshold bin b1 of pass 1 or above it, a few
    // thousand columns of the row: every warp lists its candidates (column order) in its region
    // of `hsum`; when they fit, every warp stores them into CTA 0's merged list, and CTA 0
    // completes the selection and the emission alone.
    {
        // One pass: warp w appends its candidates (column order) to its own region of kTopkWarpCap
        // slots of the CTA's list in `hsum` (keys, then columns).
        uint32_t* lkey = reinterpret_cast<uint32_t*>(hsum);
        int* lcol = hsum + kTopkLocalCap;
        int run = 0;
        for (int c = w0; c < w1; c += 32) {
            const uint32_t key = key_at(c + lane);
            const bool sel = key != 0u && key >= tb;
            const uint32_t m = __ballot_sync(0xffffffffu, sel);
            const int at = run + __popc(m & ((1u << lane) - 1));
            if (sel && at < kTopkWarpCap) { lkey[warp * kTopkWarpCap + at] = key; lcol[warp * kTopkWarpCap + at] = c + lane; }
            run += __popc(m);
        }
        if (lane == 0) s_wcnt[warp] = run;
        __syncthreads();
        if (threadIdx.x == 0) {
            int tot = 0, big = 0;
            for (int w = 0; w < kTopkWarps; ++w) { tot += s_wcnt[w]; big = max(big, s_wcnt[w]); }
            s_slot[2] = tot;
            s_wmax = big;
        }
        cl.sync();                                       // counts everywhere (CTA 0's cache is done)
        int total = 0, biggest = 0, before = 0;
        for (int r = 0; r < NC; ++r) {
            const int v = *cl.map_shared_rank(&s_slot[2], r);
            if (r < rank) before += v;
            total += v;
            biggest = max(biggest, *cl.map_shared_rank(&s_wmax, r));
        }
        if (biggest <= kTopkWarpCap && total <= kTopkCap) {
            uint32_t* ckey = s_keys;                     // CTA 0: merged candidates, column order
            int* ccol = reinterpret_cast<int*>(s_keys) + kTopkCap;
            {
                // Every warp stores its candidates straight into CTA 0's merged list.
                int wb = before;
                for (int w = 0; w < warp; ++w) wb += s_wcnt[w];
                uint32_t* dk = cl.map_shared_rank(ckey, 0);
                int* dc = cl.map_shared_rank(ccol, 0);
                for (int i = lane; i < s_wcnt[warp]; i += 32) {
                    dk[wb + i] = lkey[warp * kTopkWarpCap + i];
                    dc[wb + i] = lcol[warp * kTopkWarpCap + i];
                }
            }
            // No peer reads `hist` any more (the count barrier above): CTA 0 clears its
            // histograms for passes 2 and 3 while the candidates arrive.
            if (rank == 0) {
                for (int i = threadIdx.x; i < 4096; i += kTopkThreads) hist[i] = 0;
                if (threadIdx.x < 256) hist3[threadIdx.x] = 0;
            }
            cl.sync();                                   // every candidate has reached CTA 0
            if (rank != 0) return;
            const int n = total;
            uint32_t vs = 0;
            int m_keep = 0, n_eq = 0;
            if (!take_all && a.k > 0) {
                const uint32_t b1 = (uint32_t)s_bin;
                int above = s_above;
                for (int i = threadIdx.x; i < n; i += kTopkThreads) {
                    const uint32_t key = ckey[i];
                    if ((key >> 20) == b1) atomicAdd(&hist[(key >> 8) & 0xfff], 1);
                }
                __syncthreads();
                local_threshold(hist, 4096, a.k - above, s_warp, &s_bin, &s_above);
                const uint32_t pre = (b1 << 12) | (uint32_t)s_bin;
                above += s_above;
                for (int i = threadIdx.x; i < n; i += kTopkThreads) {
                    const uint32_t key = ckey[i];
                    if ((key >> 8) == pre) atomicAdd(&hist3[key & 0xff], 1);
                }
                __syncthreads();
                local_threshold(hist3, 256, a.k - above, s_warp, &s_bin, &s_above);
                above += s_above;
                vs = (pre << 8) | (uint32_t)s_bin;
                m_keep = a.k - above;                    // keys == vs to keep, lowest columns first
                n_eq = hist3[s_bin];                     // keys == vs among the candidates
            }
            const bool every = take_all || a.k <= 0;     // every candidate is selected (none when k = 0)
            const bool ties_all = every || m_keep >= n_eq;
            // Emission in column order: warp w owns a contiguous range of the candidates and walks
            // it 32 at a time; in-warp ranks come from ballots, warp bases from per-warp counts.
            const uint32_t lt = (1u << lane) - 1;
            const int cw = ((n + kTopkWarps - 1) / kTopkWarps + 31) / 32 * 32;
            const int e0 = min(n, warp * cw), e1 = min(n, e0 + cw);
            int eq_base = 0;
            if (!ties_all) {                             // ties at vs are cut: ranks among them needed
                int c = 0;
                for (int i = e0; i < e1; i += 32)
                    c += __popc(__ballot_sync(0xffffffffu, i + lane < e1 && ckey[i + lane] == vs));
                if (lane == 0) s_wcnt[warp] = c;
                __syncthreads();
                for (int w = 0; w < warp; ++w) eq_base += s_wcnt[w];
            }
            // kept(i): selected, and (unless raw) its position outside the sinks and the window.
            // One walk: warp w stages its kept positions in shared memory from its own candidate
            // offset e0 on (kept entries are a subset of its candidates, so the regions do not
            // meet; `hsum` then `hist`, both free by now, hold kTopkCap entries), then copies them
            // out once the warps' counts are known.
            static_assert(kTopkCap <= 2 * 4096, "the staging spans hsum and hist");
            auto stage = [&](int i) -> int& { return i < 4096 ? hsum[i] : hist[i - 4096]; };
            int kept_w = 0;
            {
                int eq_run = eq_base;
                for (int i = e0; i < e1; i += 32) {
                    const int ii = i + lane;
                    const bool in = ii < e1;
                    const uint32_t key = in ? ckey[ii] : 0u;
                    bool keep;
                    if (every) {
                        keep = in && a.k > 0;
                    } else {
                        const bool eq = in && key == vs;
                        const uint32_t em = ties_all ? 0u : __ballot_sync(0xffffffffu, eq);
                        keep = in && (key > vs || (eq && (ties_all || eq_run + __popc(em & lt) < m_keep)));
                        eq_run += __popc(em);
                    }
                    int pv = 0;
                    if (keep) {
                        pv = a.raw ? ccol[ii] : position(ccol[ii]);
                        if (!a.raw) keep = pv >= a_lo && pv < b_hi;
                    }
                    const uint32_t km = __ballot_sync(0xffffffffu, keep);
                    if (keep) stage(e0 + kept_w + __popc(km & lt)) = pv;
                    kept_w += __popc(km);
                }
            }
            if (lane == 0) s_wk[warp] = kept_w;
            __syncthreads();
            int keep_base = 0, written = 0;
            for (int w = 0; w < kTopkWarps; ++w) {
                const int v = s_wk[w];
                if (w < warp) keep_base += v;
                written += v;
            }
            for (int j = lane; j < kept_w; j += 32) out[a_lo + keep_base + j] = stage(e0 + j);
            int n_out = a_lo + written;
            if (!a.raw) {
                for (int i = threadIdx.x; i < a_lo; i += kTopkThreads) out[i] = i;
                const int tail = pos + 1 - b_hi;
                for (int i = threadIdx.x; i < tail; i += kTopkThreads) out[n_out + i] = b_hi + i;
                n_out += max(tail, 0);
            }
            for (int i = n_out + threadIdx.x; i < a.ld_idx; i += kTopkThreads) out[i] = -1;
            if (threadIdx.x == 0) a.count[t] = n_out;
            return;
        }
        // Too many candidates: the cluster continues with the full passes below.
    }
    uint32_t vstar = 0;
    int above = 0;
    if (!take_all && a.k > 0) {
        const uint32_t b1 = (uint32_t)s_bin;
        above = s_above;
        // ---- pass 2: next 12 bits among keys with prefix b1
        for (int i = threadIdx.x; i < 4096; i += kTopkThreads) hist[i] = 0;
        __syncthreads();
        for (int c = w0; c < w1; c += 32) {
            const uint32_t key = key_at(c + lane);
            hist_add(hist, (int)((key >> 8) & 0xfff), key != 0u && (key >> 20) == b1);
        }
        cluster_threshold<NC>(cl, rank, hist, hsum, 4096, a.k - above, s_warp, &s_bin, &s_above);
        const uint32_t b2 = (uint32_t)s_bin;
        above += s_above;
        // ---- pass 3: last 8 bits among keys with prefix (b1, b2)
        const uint32_t pre = (b1 << 12) | b2;
        for (int i = threadIdx.x; i < 256; i += kTopkThreads) hist[i] = 0;
        __syncthreads();
        for (int c = w0; c < w1; c += 32) {
            const uint32_t key = key_at(c + lane);
            hist_add(hist, (int)(key & 0xff), key != 0u && (key >> 8) == pre);
        }
        cluster_threshold<NC>(cl, rank, hist, hsum, 256, a.k - above, s_warp, &s_bin, &s_above);
        above += s_above;
        vstar = (pre << 8) | (uint32_t)s_bin;
    }
    const int m_ties = a.k - above;           // keys == v* to keep (lowest columns first)

    // ---- emission: ascending columns
    auto classify = [&](int cc, bool& eq, bool& gt, int& p) {
        eq = gt = false;
        p = -1;
        const uint32_t key = key_at(cc);
        if (key == 0u) return;
        if (a.k > 0) {
            gt = take_all || key > vstar;
            eq = !take_all && key == vstar;
        }
        p = position(cc);
    };
    // A: ties per warp -> CTA prefix -> cluster prefix.
    int eq_w = 0;
    for (int c = w0; c < w1; c += 32) {
        bool eq, gt;
        int p;
        classify(c + lane, eq, gt, p);
        eq_w += __popc(__ballot_sync(0xffffffffu, eq));
    }
    int eq_cta;
    const int eq_wbase = cta_inclusive_scan(lane == 0 ? eq_w : 0, s_warp, eq_cta) - (lane == 0 ? eq_w : 0);
    if (threadIdx.x == 0) s_slot[0] = eq_cta;
    int eq_all;
    const int eq_cbase = cluster_exclusive<NC>(cl, &s_slot[0], rank, eq_all);
    const int eq_base = eq_cbase + __shfl_sync(0xffffffffu, eq_wbase, 0);
    // B: kept entries per warp -> CTA prefix -> cluster prefix.
    int keep_w = 0;
    {
        int eq_run = eq_base;
        for (int c = w0; c < w1; c += 32) {
            bool eq, gt;
            int p;
            classify(c + lane, eq, gt, p);
            const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
            const int rk = eq_run + __popc(eqm & ((1u << lane) - 1));
            const bool sel = gt || (eq && rk < m_ties);
            const bool keep = sel && (a.raw || (p >= a_lo && p < b_hi));
            keep_w += __popc(__ballot_sync(0xffffffffu, keep));
            eq_run += __popc(eqm);
        }
    }
    int keep_cta;
    const int keep_wbase = cta_inclusive_scan(lane == 0 ? keep_w : 0, s_warp, keep_cta) - (lane == 0 ? keep_w : 0);
    if (threadIdx.x == 0) s_slot[1] = keep_cta;
    int written;
    const int keep_cbase = cluster_exclusive<NC>(cl, &s_slot[1], rank, written);
    // C: write.
    {
        int eq_run = eq_base;
        int out_run = a_lo + keep_cbase + __shfl_sync(0xffffffffu, keep_wbase, 0);
        for (int c = w0; c < w1; c += 32) {
            bool eq, gt;
            int p;
            classify(c + lane, eq, gt, p);
            const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
            const int rk = eq_run + __popc(eqm & ((1u << lane) - 1));
            const bool sel = gt || (eq && rk < m_ties);
            const bool keep = sel && (a.raw || (p >= a_lo && p < b_hi));
            const uint32_t km = __ballot_sync(0xffffffffu, keep);
            if (keep) out[out_run + __popc(km & ((1u << lane) - 1))] = a.raw ? c + lane : p;
            out_run += __popc(km);
            eq_run += __popc(eqm);
        }
    }
    cl.sync();                    // no CTA leaves while a peer may still read its shared memory
    if (rank != NC - 1) return;
    int n_out = a_lo + written;
    if (!a.raw) {
        for (int i = threadIdx.x; i < a_lo; i += kTopkThreads) out[i] = i;
        const int tail = pos + 1 - b_hi;
        for (int i = threadIdx.x; i < tail; i += kTopkThreads) out[n_out + i] = b_hi + i;
        n_out += max(tail, 0);
    }
    for (int i = n_out + threadIdx.x; i < a.ld_idx; i += kTopkThreads) out[i] = -1;
    if (threadIdx.x == 0) a.count[t] = n_out;
}

template <int NC>
static cudaError_t launch_topk_nc(const TopkArgs& a, cudaStream_t st) {
    const int per_cta = ((a.n_cols + NC - 1) / NC + 31) / 32 * 32;
    const size_t cand_smem = (size_t)kTopkCap * 8;             // merged candidates (keys, columns) in CTA 0
    if (per_cta <= kTopkCacheCols) {
        const size_t smem = std::max((size_t)per_cta * 4, cand_smem);
        cudaError_t e = cudaFuncSetAttribute(topk_kernel<true, NC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)std::max((size_t)kTopkCacheCols * 4, cand_smem));
        if (e != cudaSuccess) return e;
        topk_kernel<true, NC><<<a.T * NC, kTopkThreads, smem, st>>>(a);
    } else {
        cudaError_t e = cudaFuncSetAttribute(topk_kernel<false, NC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)cand_smem);
        if (e != cudaSuccess) return e;
        topk_kernel<false, NC><<<a.T * NC, kTopkThreads, cand_smem, st>>>(a);
    }
    return cudaGetLastError();
}

// Cluster size per launch.  A few rows (decode) take clusters of kTopkCluster = 8: the row's
// latency is what counts and eight CTAs share its passes.  From kTopkManyRows rows on, the SMs
// are busy with rows anyway and the cluster barriers, not the work, set the time of each row, so
// the smallest cluster whose segments still fit the shared-memory cache is taken (2, else 4):
// measured on one B200, 2,048 rows of 32,768 columns take 0.33 ms in clusters of 2 against 0.72
// ms in clusters of 8; 4 rows of 16,384 columns 12.9 us against 11.5 us.
constexpr int kTopkManyRows = 64;

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t st) {
    if (a.T <= 0) return cudaSuccess;
    auto cached = [&](int nc) { return ((a.n_cols + nc - 1) / nc + 31) / 32 * 32 <= kTopkCacheCols; };
    if (a.T >= kTopkManyRows) {
        if (cached(2)) return launch_topk_nc<2>(a, st);
        if (cached(4)) return launch_topk_nc<4>(a, st);
    }
    return launch_topk_nc<kTopkCluster>(a, st);
}

}  // namespace lsa
