// Pipelined host I/O around lsa_decode_fused: copy-in, decode and copy-out of consecutive
// steps on three streams, ordered per buffer slot by events (see lsa.h).
#include <new>

#include "kernels.cuh"

struct lsa_pipeline {
    static constexpr int kMaxSlots = 8;
    int dev = -1, n_slots = 0;
    cudaStream_t st = nullptr;                   // the caller's stream: the decodes
    cudaStream_t in = nullptr, out = nullptr;    // copy-in, copy-out
    cudaEvent_t in_done[kMaxSlots] = {}, dec_done[kMaxSlots] = {}, out_done[kMaxSlots] = {};
    cudaEvent_t joined = nullptr;
    bool used[kMaxSlots] = {};                   // the slot has events recorded
};

namespace {

void release(lsa_pipeline* pl) {
    for (int i = 0; i < lsa_pipeline::kMaxSlots; ++i) {
        if (pl->in_done[i]) cudaEventDestroy(pl->in_done[i]);
        if (pl->dec_done[i]) cudaEventDestroy(pl->dec_done[i]);
        if (pl->out_done[i]) cudaEventDestroy(pl->out_done[i]);
    }
    if (pl->joined) cudaEventDestroy(pl->joined);
    if (pl->in) cudaStreamDestroy(pl->in);
    if (pl->out) cudaStreamDestroy(pl->out);
    delete pl;
}

inline bool ok(cudaError_t e) { return e == cudaSuccess; }

}  // namespace

extern "C" {

lsa_status lsa_pipeline_create(lsa_pipeline** out, int n_slots, void* stream) {
    if (!out || n_slots < 1 || n_slots > lsa_pipeline::kMaxSlots) return LSA_ERR_INVALID_ARG;
    *out = nullptr;
    lsa_pipeline* pl = new (std::nothrow) lsa_pipeline;
    if (!pl) return LSA_ERR_CUDA;
    pl->n_slots = n_slots;
    pl->st = static_cast<cudaStream_t>(stream);
    bool good = ok(cudaGetDevice(&pl->dev)) && ok(cudaStreamCreateWithFlags(&pl->in, cudaStreamNonBlocking)) &&
                ok(cudaStreamCreateWithFlags(&pl->out, cudaStreamNonBlocking)) &&
                ok(cudaEventCreateWithFlags(&pl->joined, cudaEventDisableTiming));
    for (int i = 0; good && i < n_slots; ++i)
        good = ok(cudaEventCreateWithFlags(&pl->in_done[i], cudaEventDisableTiming)) &&
               ok(cudaEventCreateWithFlags(&pl->dec_done[i], cudaEventDisableTiming)) &&
               ok(cudaEventCreateWithFlags(&pl->out_done[i], cudaEventDisableTiming));
    if (!good) {
        release(pl);
        return LSA_ERR_CUDA;
    }
    *out = pl;
    return LSA_OK;
}

lsa_status lsa_pipeline_step(lsa_pipeline* pl, int slot, const lsa_decode_params* const* params, int n_params,
                             void* const* ws, const size_t* ws_bytes, const lsa_copy* h2d, int n_h2d,
                             const lsa_copy* d2h, int n_d2h, int32_t* dev_status) {
    if (!pl || slot < 0 || slot >= pl->n_slots || n_params < 0 || n_h2d < 0 || n_d2h < 0) return LSA_ERR_INVALID_ARG;
    if ((n_params && (!params || !ws || !ws_bytes)) || (n_h2d && !h2d) || (n_d2h && !d2h)) return LSA_ERR_INVALID_ARG;
    for (int i = 0; i < n_params; ++i)
        if (!params[i]) return LSA_ERR_INVALID_ARG;
    const bool again = pl->used[slot];
    // Copy-in, once the decode that last read this slot's inputs has finished.
    if (again && !ok(cudaStreamWaitEvent(pl->in, pl->dec_done[slot], 0))) return LSA_ERR_CUDA;
    for (int i = 0; i < n_h2d; ++i)
        if (h2d[i].bytes && !ok(cudaMemcpyAsync(h2d[i].dst, h2d[i].src, h2d[i].bytes, cudaMemcpyHostToDevice, pl->in)))
            return LSA_ERR_CUDA;
    if (!ok(cudaEventRecord(pl->in_done[slot], pl->in)) || !ok(cudaStreamWaitEvent(pl->st, pl->in_done[slot], 0)))
        return LSA_ERR_CUDA;
    // Decode, once the copy-out that last read this slot's outputs has finished.
    if (again && !ok(cudaStreamWaitEvent(pl->st, pl->out_done[slot], 0))) return LSA_ERR_CUDA;
    lsa_status s = LSA_OK;
    for (int i = 0; i < n_params && s == LSA_OK; ++i) s = lsa_decode_fused(params[i], ws[i], ws_bytes[i], dev_status, pl->st);
    // The events below are recorded also after an error, so that the slot's ordering holds.
    if (!ok(cudaEventRecord(pl->dec_done[slot], pl->st)) || !ok(cudaStreamWaitEvent(pl->out, pl->dec_done[slot], 0)))
        return LSA_ERR_CUDA;
    for (int i = 0; s == LSA_OK && i < n_d2h; ++i)
        if (d2h[i].bytes && !ok(cudaMemcpyAsync(d2h[i].dst, d2h[i].src, d2h[i].bytes, cudaMemcpyDeviceToHost, pl->out)))
            s = LSA_ERR_CUDA;
    if (!ok(cudaEventRecord(pl->out_done[slot], pl->out))) return LSA_ERR_CUDA;
    pl->used[slot] = true;
    return s;
}

lsa_status lsa_pipeline_join(lsa_pipeline* pl) {
    if (!pl) return LSA_ERR_INVALID_ARG;
    if (!ok(cudaEventRecord(pl->joined, pl->out)) || !ok(cudaStreamWaitEvent(pl->st, pl->joined, 0))) return LSA_ERR_CUDA;
    return LSA_OK;
}

lsa_status lsa_pipeline_destroy(lsa_pipeline* pl) {
    if (!pl) return LSA_ERR_INVALID_ARG;
    const bool synced = ok(cudaStreamSynchronize(pl->in)) && ok(cudaStreamSynchronize(pl->out));
    release(pl);
    return synced ? LSA_OK : LSA_ERR_CUDA;
}

}  // extern "C"
