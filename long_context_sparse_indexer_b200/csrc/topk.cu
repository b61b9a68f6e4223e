// Top-k selection with the SI window and the sink tokens, one CTA per query row.
//
// Explainer page ("如何在 5 万张国产芯片训练出 1.6T 万亿参数模型？"), section "① LSA": each query
// reads only its top-k keys plus a few fixed sink tokens.  Release post, section
// "LongCat 稀疏注意力", SI bullet: the selection budget mixes a hardware-aligned contiguous
// part with the dynamic top-k picks.  The order on equal scores is the lower position
// first, which makes the selection unique and the output deterministic.
//
// Method: radix select on the order-preserving 32-bit key of the score, 12 + 12 + 8 bits,
// with integer shared-memory histograms (counts do not depend on the order of the
// atomics).  That yields the k-th key v* and the number m of ties at v* to keep; a final
// ascending pass over the columns keeps every key > v* and the first m keys == v*
// (lowest columns), and writes the positions in ascending order, merged with the sinks
// [0, a) and the window [b, pos] so the list comes out sorted and de-duplicated.
#include "kernels.cuh"

namespace lsa {

constexpr int kTopkThreads = 1024;
constexpr int kTopkWarps = kTopkThreads / 32;

// Inclusive prefix sum over the block (warp shuffles + one shared array of warp totals).
__device__ __forceinline__ int block_inclusive_scan(int v, int* s_warp, int& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    if (lane == 31) s_warp[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int x = s_warp[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int n = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += n;
        }
        s_warp[lane] = x;
    }
    __syncthreads();
    total = s_warp[kTopkWarps - 1];
    const int res = v + (warp > 0 ? s_warp[warp - 1] : 0);
    __syncthreads();
    return res;
}

// Finds the bin where the count from the top first reaches `need` (bins: nb, 4 per thread).
// Returns via shared memory: the bin and the count of elements in higher bins.
__device__ void find_threshold(const int* hist, int nb, int need, int* s_warp, int* s_bin, int* s_above) {
    const int per = nb / kTopkThreads;   // 4 or (for 256 bins) handled by per == 0 below
    int local = 0;
    int bins[4];
    if (per > 0) {
        for (int i = 0; i < per; ++i) {
            bins[i] = nb - 1 - (threadIdx.x * per + i);     // from the top
            local += hist[bins[i]];
        }
    } else {
        bins[0] = (int)threadIdx.x < nb ? nb - 1 - (int)threadIdx.x : -1;
        local = bins[0] >= 0 ? hist[bins[0]] : 0;
    }
    int total;
    const int incl = block_inclusive_scan(local, s_warp, total);
    int run = incl - local;                                  // count in bins above this thread's first bin
    const int cnt = per > 0 ? per : 1;
    for (int i = 0; i < cnt; ++i) {
        if (bins[i] < 0) break;
        const int h = hist[bins[i]];
        if (run < need && run + h >= need) { *s_bin = bins[i]; *s_above = run; }
        run += h;
    }
    __syncthreads();
}

__global__ void __launch_bounds__(kTopkThreads) topk_kernel(TopkArgs a) {
    __shared__ int hist[4096];
    __shared__ int s_warp[kTopkWarps];
    __shared__ int s_bin, s_above, s_nvalid;
    const int t = blockIdx.x;
    const float* row = a.scores + (size_t)t * a.ld;
    int32_t* out = a.idx + (size_t)t * a.ld_idx;

    // Query position and its validity.
    const int b = a.q_seq[t];
    int pos = a.q_pos[t];
    bool ok = b >= 0 && b < a.B;
    if (ok) {
        const int len = a.seq_len[b];
        ok = len >= 1 && len <= a.L_alloc && pos >= 0 && pos < len;
    }
    if (!ok) {
        if (threadIdx.x == 0) { report(a.status, LSA_ERR_DEVICE_DATA); a.count[t] = 0; }
        for (int i = threadIdx.x; i < a.ld_idx; i += kTopkThreads) out[i] = -1;
        return;
    }

    // ---- pass 1: top 12 bits
    for (int i = threadIdx.x; i < 4096; i += kTopkThreads) hist[i] = 0;
    if (threadIdx.x == 0) s_nvalid = 0;
    __syncthreads();
    int nvalid = 0;
    for (int c = threadIdx.x; c < a.n_cols; c += kTopkThreads) {
        const float f = row[c];
        if (f != f) { report(a.status, LSA_ERR_DEVICE_DATA); continue; }
        if (f == kNegInf) continue;
        atomicAdd(&hist[order_key(f) >> 20], 1);
        ++nvalid;
    }
    atomicAdd(&s_nvalid, nvalid);
    __syncthreads();
    const int n_valid = s_nvalid;
    const bool take_all = n_valid <= a.k;
    uint32_t vstar = 0;
    int above = 0;
    if (!take_all && a.k > 0) {
        find_threshold(hist, 4096, a.k, s_warp, &s_bin, &s_above);
        const uint32_t b1 = (uint32_t)s_bin;
        above = s_above;
        // ---- pass 2: next 12 bits among keys with prefix b1
        for (int i = threadIdx.x; i < 4096; i += kTopkThreads) hist[i] = 0;
        __syncthreads();
        for (int c = threadIdx.x; c < a.n_cols; c += kTopkThreads) {
            const float f = row[c];
            if (f != f || f == kNegInf) continue;
            const uint32_t key = order_key(f);
            if ((key >> 20) == b1) atomicAdd(&hist[(key >> 8) & 0xfff], 1);
        }
        __syncthreads();
        find_threshold(hist, 4096, a.k - above, s_warp, &s_bin, &s_above);
        const uint32_t b2 = (uint32_t)s_bin;
        above += s_above;
        // ---- pass 3: last 8 bits among keys with prefix (b1, b2)
        const uint32_t pre = (b1 << 12) | b2;
        for (int i = threadIdx.x; i < 256; i += kTopkThreads) hist[i] = 0;
        __syncthreads();
        for (int c = threadIdx.x; c < a.n_cols; c += kTopkThreads) {
            const float f = row[c];
            if (f != f || f == kNegInf) continue;
            const uint32_t key = order_key(f);
            if ((key >> 8) == pre) atomicAdd(&hist[key & 0xff], 1);
        }
        __syncthreads();
        find_threshold(hist, 256, a.k - above, s_warp, &s_bin, &s_above);
        above += s_above;
        vstar = (pre << 8) | (uint32_t)s_bin;
    }
    const int m_ties = a.k - above;           // keys == v* to keep (lowest columns first)

    // ---- emission: ascending columns.  Warp w owns the contiguous column segment
    // [w * seg, (w + 1) * seg); ranks inside a warp come from ballots, across warps from
    // two block scans (ties at v*, then kept entries).
    const int a_lo = a.raw ? 0 : min(a.n_sink, pos + 1);
    const int b_hi = a.raw ? 0x7fffffff : (a.window > 0 ? max(a_lo, pos - a.window + 1) : pos + 1);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int seg = ((a.n_cols + kTopkThreads - 1) / kTopkThreads) * 32;
    const int c_beg = warp * seg, c_end = min(a.n_cols, c_beg + seg);
    auto classify = [&](int c, bool& eq, bool& gt, int& p) {
        eq = gt = false;
        p = -1;
        if (c >= c_end) return;
        const float f = row[c];
        if (f != f || f == kNegInf) return;
        if (a.k > 0) {
            const uint32_t key = order_key(f);
            gt = take_all || key > vstar;
            eq = !take_all && key == vstar;
        }
        if (a.raw || !a.cand) p = c;
        else p = a.cand[(size_t)t * a.n_cand + c / a.block_size] * a.block_size + c % a.block_size;
    };
    // A: ties per warp.
    int eq_w = 0;
    for (int c0 = c_beg; c0 < c_end; c0 += 32) {
        bool eq, gt;
        int p;
        classify(c0 + lane, eq, gt, p);
        eq_w += __popc(__ballot_sync(0xffffffffu, eq));
    }
    int eq_tot;
    const int eq_base = block_inclusive_scan(lane == 0 ? eq_w : 0, s_warp, eq_tot) - (lane == 0 ? eq_w : 0);
    const int eq_base_w = __shfl_sync(0xffffffffu, eq_base, 0);
    // B: kept entries per warp.
    int keep_w = 0;
    {
        int eq_run = eq_base_w;
        for (int c0 = c_beg; c0 < c_end; c0 += 32) {
            bool eq, gt;
            int p;
            classify(c0 + lane, eq, gt, p);
            const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
            const int rank = eq_run + __popc(eqm & ((1u << lane) - 1));
            const bool sel = gt || (eq && rank < m_ties);
            const bool keep = sel && (a.raw || (p >= a_lo && p < b_hi));
            keep_w += __popc(__ballot_sync(0xffffffffu, keep));
            eq_run += __popc(eqm);
        }
    }
    int written;
    const int keep_base = block_inclusive_scan(lane == 0 ? keep_w : 0, s_warp, written) - (lane == 0 ? keep_w : 0);
    // C: write.
    {
        int eq_run = eq_base_w;
        int out_run = a_lo + __shfl_sync(0xffffffffu, keep_base, 0);
        for (int c0 = c_beg; c0 < c_end; c0 += 32) {
            bool eq, gt;
            int p;
            classify(c0 + lane, eq, gt, p);
            const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
            const int rank = eq_run + __popc(eqm & ((1u << lane) - 1));
            const bool sel = gt || (eq && rank < m_ties);
            const bool keep = sel && (a.raw || (p >= a_lo && p < b_hi));
            const uint32_t km = __ballot_sync(0xffffffffu, keep);
            if (keep) out[out_run + __popc(km & ((1u << lane) - 1))] = a.raw ? c0 + lane : p;
            out_run += __popc(km);
            eq_run += __popc(eqm);
        }
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
}

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t st) {
    if (a.T <= 0) return cudaSuccess;
    topk_kernel<<<a.T, kTopkThreads, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace lsa
