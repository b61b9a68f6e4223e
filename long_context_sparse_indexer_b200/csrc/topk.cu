// Top-k selection with the SI window and the sink tokens.
//
// Explainer page ("如何在 5 万张国产芯片训练出 1.6T 万亿参数模型？"), section "① LSA": each query
// reads only its top-k keys plus a few fixed sink tokens.  Release post, section
// "LongCat 稀疏注意力", SI bullet: the selection budget mixes a hardware-aligned contiguous
// part with the dynamic top-k picks.  The order on equal scores is the lower position
// first, which makes the selection unique and the output deterministic.
//
// Method: radix select on the order-preserving 32-bit key of each score, 12 + 12 + 8 bits.
// One query row is handled by a cluster of kTopkCluster CTAs; CTA r owns the r-th
// contiguous segment of the row.  Each pass builds integer shared-memory histograms of
// its segment (warp-aggregated atomics; counts do not depend on atomic order), every CTA
// then reads all the cluster's histograms through distributed shared memory and finds
// the same threshold bin.  The result is the k-th key v* and the number m of ties at v*
// to keep.  The emission pass keeps every key > v* and the first m keys == v* (lowest
// columns first); ranks across CTAs, warps and lanes come from cluster-wide prefix
// counts, ballots and popcounts.  Positions are written in ascending order and merged
// with the sinks [0, a) and the window [b, pos], so the list comes out sorted and
// de-duplicated.  Segments of up to 40960 columns are first cached in shared memory as
// order keys (one coalesced read of the row); longer ones are re-read from global memory.
#include <algorithm>
#include <cooperative_groups.h>

#include "kernels.cuh"

namespace cg = cooperative_groups;

namespace lsa {

constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kTopkCluster = 8;

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
// the r-th eighth of the bins over the cluster (distributed shared memory loads) and writes
// the sums into every CTA's `sum` (distributed shared memory stores).
__device__ int cluster_threshold(cg::cluster_group& cl, int rank, int* hist, int* sum, int nb, int need,
                                 int* s_warp, int* s_bin, int* s_above) {
    cl.sync();                                           // all local histograms complete
    const int share = nb / kTopkCluster;
    for (int i = threadIdx.x; i < share; i += kTopkThreads) {
        const int bin = rank * share + i;
        int v[kTopkCluster];
#pragma unroll
        for (int r = 0; r < kTopkCluster; ++r) v[r] = cl.map_shared_rank(hist, r)[bin];
        int s = 0;
#pragma unroll
        for (int r = 0; r < kTopkCluster; ++r) s += v[r];
#pragma unroll
        for (int r = 0; r < kTopkCluster; ++r) cl.map_shared_rank(sum, r)[bin] = s;
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

// Cluster-wide exclusive prefix of one int per CTA (the value in `slot` of each CTA).  Every
// exchange uses its own slot, so the slot is never rewritten while a peer may still read it.
__device__ int cluster_exclusive(cg::cluster_group& cl, int* slot, int rank, int& total) {
    cl.sync();
    int before = 0;
    total = 0;
    for (int r = 0; r < kTopkCluster; ++r) {
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
// Candidate lists of the compacted finish: per CTA (in its `hsum` array) and merged in CTA 0.
constexpr int kTopkLocalCap = 2048;
constexpr int kTopkWarpCap = kTopkLocalCap / kTopkWarps;   // per warp
constexpr int kTopkCap = 8192;

template <bool CACHED>
__global__ void __cluster_dims__(kTopkCluster, 1, 1) __launch_bounds__(kTopkThreads)
topk_kernel(TopkArgs a) {
    __shared__ int hist[4096];
    __shared__ int hsum[4096];
    __shared__ int s_warp[kTopkWarps];
    __shared__ int s_bin, s_above, s_slot[3], s_wmax;
    __shared__ int s_wcnt[kTopkWarps];
    extern __shared__ uint32_t s_keys[];          // CACHED: order key of each column of the segment, 0 = invalid
    cg::cluster_group cl = cg::this_cluster();
    const int rank = (int)cl.block_rank();
    const int t = blockIdx.x / kTopkCluster;
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
    const int per_cta = ((a.n_cols + kTopkCluster - 1) / kTopkCluster + 31) / 32 * 32;
    const int c0 = min(a.n_cols, rank * per_cta), c1 = min(a.n_cols, c0 + per_cta);
    const int per_warp = ((c1 - c0 + kTopkWarps - 1) / kTopkWarps + 31) / 32 * 32;
    const int w0 = min(c1, c0 + warp * per_warp), w1 = min(c1, w0 + per_warp);

    // Order key of column cc of this warp's segment (0 = not a candidate; valid keys are > 0).
    auto key_at = [&](int cc) -> uint32_t {
        if (cc >= w1) return 0u;
        if (CACHED) return s_keys[cc - c0];
        const float f = row[cc];
        return (f != f || f == kNegInf) ? 0u : order_key(f);
    };

    // ---- pass 1: top 12 bits (and, when cached, the segment's keys into shared memory)
    for (int i = threadIdx.x; i < 4096; i += kTopkThreads) hist[i] = 0;
    if (CACHED) {
        // Batches of 8 independent 16-byte loads per thread, then conversion to keys.
        constexpr int kB = 8;
        const bool vec = (((uintptr_t)(row + c0)) & 15) == 0;
        for (int base = c0 + threadIdx.x * 4; base < c1; base += kTopkThreads * 4 * kB) {
            float f[kB][4];
#pragma unroll
            for (int u = 0; u < kB; ++u) {
                const int cc = base + u * kTopkThreads * 4;
                if (vec && cc + 3 < c1) {
                    const float4 v4 = *reinterpret_cast<const float4*>(row + cc);
                    f[u][0] = v4.x; f[u][1] = v4.y; f[u][2] = v4.z; f[u][3] = v4.w;
                } else {
#pragma unroll
                    for (int e = 0; e < 4; ++e) f[u][e] = cc + e < c1 ? row[cc + e] : kNegInf;
                }
            }
#pragma unroll
            for (int u = 0; u < kB; ++u) {
                const int cc = base + u * kTopkThreads * 4;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    if (cc + e >= c1) break;
                    const float x = f[u][e];
                    if (x != x) report(a.status, LSA_ERR_DEVICE_DATA);
                    s_keys[cc + e - c0] = (x != x || x == kNegInf) ? 0u : order_key(x);
                }
            }
        }
    }
    __syncthreads();
    for (int c = w0; c < w1; c += 32) {
        const int cc = c + lane;
        if (!CACHED && cc < w1) {
            const float f = row[cc];
            if (f != f) report(a.status, LSA_ERR_DEVICE_DATA);
        }
        const uint32_t key = key_at(cc);
        hist_add(hist, (int)(key >> 20), key != 0u);
    }
    // Cluster histogram of the top 12 bits; its total is the number of candidates.
    const int n_valid = cluster_threshold(cl, rank, hist, hsum, 4096, a.k, s_warp, &s_bin, &s_above);
    const bool take_all = n_valid <= a.k;
    const int a_lo = a.raw ? 0 : min(a.n_sink, pos + 1);
    const int b_hi = a.raw ? 0x7fffffff : (a.window > 0 ? max(a_lo, pos - a.window + 1) : pos + 1);
    auto position = [&](int cc) -> int {
        if (a.raw || !a.cand) return cc;
        return a.cand[(size_t)t * a.n_cand + cc / a.block_size] * a.block_size + cc % a.block_size;
    };

    // ---- compacted finish.  The top-k lies in the threshold bin b1 of pass 1 or above it, a few
    // thousand columns of the row: every warp lists its candidates (column order) in its region
    // of `hsum`; when they fit, every warp stores them into CTA 0's merged list, and CTA 0
    // completes the selection and the emission alone.
    {
        const uint32_t tb = a.k <= 0 ? 0xffffffffu : (take_all ? 1u : ((uint32_t)s_bin << 20));
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
        for (int r = 0; r < kTopkCluster; ++r) {
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
            cl.sync();                                   // every candidate has reached CTA 0
            if (rank != 0) return;
            __syncthreads();
            const int n = total;
            uint32_t vs = 0;
            int m_keep = 0;
            if (!take_all && a.k > 0) {
                const uint32_t b1 = (uint32_t)s_bin;
                int above = s_above;
                for (int i = threadIdx.x; i < 4096; i += kTopkThreads) hist[i] = 0;
                __syncthreads();
                for (int i = threadIdx.x; i < n; i += kTopkThreads) {
                    const uint32_t key = ckey[i];
                    if ((key >> 20) == b1) atomicAdd(&hist[(key >> 8) & 0xfff], 1);
                }
                __syncthreads();
                local_threshold(hist, 4096, a.k - above, s_warp, &s_bin, &s_above);
                const uint32_t pre = (b1 << 12) | (uint32_t)s_bin;
                above += s_above;
                for (int i = threadIdx.x; i < 256; i += kTopkThreads) hist[i] = 0;
                __syncthreads();
                for (int i = threadIdx.x; i < n; i += kTopkThreads) {
                    const uint32_t key = ckey[i];
                    if ((key >> 8) == pre) atomicAdd(&hist[key & 0xff], 1);
                }
                __syncthreads();
                local_threshold(hist, 256, a.k - above, s_warp, &s_bin, &s_above);
                above += s_above;
                vs = (pre << 8) | (uint32_t)s_bin;
                m_keep = a.k - above;                    // keys == vs to keep, lowest columns first
            }
            const bool every = take_all || a.k <= 0;     // every candidate is selected (none when k = 0)
            // Emission in column order: thread = contiguous chunk of the candidates.
            const int chunk = (n + kTopkThreads - 1) / kTopkThreads;
            const int i0 = min(n, (int)threadIdx.x * chunk), i1 = min(n, i0 + chunk);
            int eq_t = 0;
            if (!every)
                for (int i = i0; i < i1; ++i) eq_t += ckey[i] == vs;
            int eq_tot;
            const int eq_base = cta_inclusive_scan(eq_t, s_warp, eq_tot) - eq_t;
            auto kept = [&](int i, int& eq_seen) -> bool {
                const uint32_t key = ckey[i];
                bool sel;
                if (every) sel = a.k > 0;
                else if (key > vs) sel = true;
                else if (key == vs) sel = eq_base + eq_seen++ < m_keep;
                else sel = false;
                if (!sel) return false;
                if (a.raw) return true;
                const int p = position(ccol[i]);
                return p >= a_lo && p < b_hi;
            };
            int keep_t = 0;
            {
                int eq_seen = 0;
                for (int i = i0; i < i1; ++i) keep_t += kept(i, eq_seen);
            }
            int written;
            const int keep_base = cta_inclusive_scan(keep_t, s_warp, written) - keep_t;
            {
                int eq_seen = 0, o = a_lo + keep_base;
                for (int i = i0; i < i1; ++i)
                    if (kept(i, eq_seen)) out[o++] = a.raw ? ccol[i] : position(ccol[i]);
            }
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
        cluster_threshold(cl, rank, hist, hsum, 4096, a.k - above, s_warp, &s_bin, &s_above);
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
        cluster_threshold(cl, rank, hist, hsum, 256, a.k - above, s_warp, &s_bin, &s_above);
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
        if (a.raw || !a.cand) p = cc;
        else p = a.cand[(size_t)t * a.n_cand + cc / a.block_size] * a.block_size + cc % a.block_size;
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
    const int eq_cbase = cluster_exclusive(cl, &s_slot[0], rank, eq_all);
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
    const int keep_cbase = cluster_exclusive(cl, &s_slot[1], rank, written);
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
    if (rank != kTopkCluster - 1) return;
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

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t st) {
    if (a.T <= 0) return cudaSuccess;
    const int per_cta = ((a.n_cols + kTopkCluster - 1) / kTopkCluster + 31) / 32 * 32;
    const size_t cand_smem = (size_t)kTopkCap * 8;             // merged candidates (keys, columns) in CTA 0
    if (per_cta <= kTopkCacheCols) {
        const size_t smem = std::max((size_t)per_cta * 4, cand_smem);
        cudaError_t e = cudaFuncSetAttribute(topk_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)std::max((size_t)kTopkCacheCols * 4, cand_smem));
        if (e != cudaSuccess) return e;
        topk_kernel<true><<<a.T * kTopkCluster, kTopkThreads, smem, st>>>(a);
    } else {
        cudaError_t e = cudaFuncSetAttribute(topk_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)cand_smem);
        if (e != cudaSuccess) return e;
        topk_kernel<false><<<a.T * kTopkCluster, kTopkThreads, cand_smem, st>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace lsa
