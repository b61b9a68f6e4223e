// Pipelined host I/O around lsa_decode_fused: copy-in, decode and copy-out of consecutive
// steps on three streams, ordered per buffer slot by events (see lsa.h).  A slot's decode is
// captured once into a CUDA graph and replayed while its parameters stay the same.
#include <cstring>
#include <new>
#include <vector>

#include "kernels.cuh"

struct lsa_pipeline {
    static constexpr int kMaxSlots = 8;
    int dev = -1, n_slots = 0;
    cudaStream_t st = nullptr;                   // the caller's stream: the decodes
    cudaStream_t in = nullptr, out = nullptr;    // copy-in, copy-out
    cudaEvent_t in_done[kMaxSlots] = {}, dec_done[kMaxSlots] = {}, out_done[kMaxSlots] = {};
    cudaEvent_t joined = nullptr;
    bool used[kMaxSlots] = {};                   // the slot has events recorded
    cudaStream_t cap = nullptr;                  // capture stream of the slot graphs
    cudaGraphExec_t exec[kMaxSlots] = {};        // the slot's captured decode
    std::vector<unsigned char> sig[kMaxSlots];   // the parameters it was captured with
};

namespace {

void release(lsa_pipeline* pl) {
    for (int i = 0; i < lsa_pipeline::kMaxSlots; ++i) {
        if (pl->in_done[i]) cudaEventDestroy(pl->in_done[i]);
        if (pl->dec_done[i]) cudaEventDestroy(pl->dec_done[i]);
        if (pl->out_done[i]) cudaEventDestroy(pl->out_done[i]);
    }
    if (pl->joined) cudaEventDestroy(pl->joined);
    for (int i = 0; i < lsa_pipeline::kMaxSlots; ++i)
        if (pl->exec[i]) cudaGraphExecDestroy(pl->exec[i]);
    if (pl->cap) cudaStreamDestroy(pl->cap);
    if (pl->in) cudaStreamDestroy(pl->in);
    if (pl->out) cudaStreamDestroy(pl->out);
    delete pl;
}

inline bool ok(cudaError_t e) { return e == cudaSuccess; }

void append(std::vector<unsigned char>& v, const void* p, size_t n) {
    const unsigned char* c = static_cast<const unsigned char*>(p);
    v.insert(v.end(), c, c + n);
}

// Everything a captured decode depends on: every parameter set with its layer array, the
// workspaces and the status word.
std::vector<unsigned char> signature(const lsa_decode_params* const* params, int n, void* const* ws,
                                     const size_t* ws_bytes, const int32_t* dev_status) {
    std::vector<unsigned char> v;
    append(v, &n, sizeof(n));
    append(v, &dev_status, sizeof(dev_status));
    for (int i = 0; i < n; ++i) {
        append(v, params[i], sizeof(lsa_decode_params));
        if (params[i]->n_layers > 0 && params[i]->layers)
            append(v, params[i]->layers, sizeof(lsa_layer) * (size_t)params[i]->n_layers);
        append(v, &ws[i], sizeof(ws[i]));
        append(v, &ws_bytes[i], sizeof(ws_bytes[i]));
    }
    return v;
}

lsa_status decode_eager(const lsa_decode_params* const* params, int n, void* const* ws, const size_t* ws_bytes,
                        int32_t* dev_status, cudaStream_t st) {
    lsa_status s = LSA_OK;
    for (int i = 0; i < n && s == LSA_OK; ++i) s = lsa_decode_fused(params[i], ws[i], ws_bytes[i], dev_status, st);
    return s;
}

// Runs the slot's decode on pl->st: its graph when the parameters match the capture, else a new
// capture (on the pipeline's own stream, so the caller's stream is never in capture mode).
// Eager launches when the caller's stream is itself being captured or a capture fails.
lsa_status decode_slot(lsa_pipeline* pl, int slot, const lsa_decode_params* const* params, int n, void* const* ws,
                       const size_t* ws_bytes, int32_t* dev_status) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (!ok(cudaStreamIsCapturing(pl->st, &cs)) || cs != cudaStreamCaptureStatusNone)
        return decode_eager(params, n, ws, ws_bytes, dev_status, pl->st);
    // A wait on the caller's prolog event cannot be captured (the event lives outside the graph).
    for (int i = 0; i < n; ++i)
        if (params[i] && params[i]->attn_q_ready) return decode_eager(params, n, ws, ws_bytes, dev_status, pl->st);
    std::vector<unsigned char> sig = signature(params, n, ws, ws_bytes, dev_status);
    if (!pl->exec[slot] || sig != pl->sig[slot]) {
        if (pl->exec[slot]) {
            cudaGraphExecDestroy(pl->exec[slot]);
            pl->exec[slot] = nullptr;
        }
        if (!pl->cap && !ok(cudaStreamCreateWithFlags(&pl->cap, cudaStreamNonBlocking)))
            return decode_eager(params, n, ws, ws_bytes, dev_status, pl->st);
        if (!ok(cudaStreamBeginCapture(pl->cap, cudaStreamCaptureModeThreadLocal)))
            return decode_eager(params, n, ws, ws_bytes, dev_status, pl->st);
        const lsa_status s = decode_eager(params, n, ws, ws_bytes, dev_status, pl->cap);
        cudaGraph_t g = nullptr;
        const bool captured = ok(cudaStreamEndCapture(pl->cap, &g)) && g != nullptr;
        if (s != LSA_OK) {                       // invalid parameters: nothing was launched
            if (g) cudaGraphDestroy(g);
            return s;
        }
        cudaGraphExec_t e = nullptr;
        const bool inst = captured && ok(cudaGraphInstantiate(&e, g, 0));
        if (g) cudaGraphDestroy(g);
        if (!inst) {
            cudaGetLastError();
            return decode_eager(params, n, ws, ws_bytes, dev_status, pl->st);
        }
        pl->exec[slot] = e;
        pl->sig[slot] = std::move(sig);
    }
    return ok(cudaGraphLaunch(pl->exec[slot], pl->st)) ? LSA_OK : LSA_ERR_CUDA;
}

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
    lsa_status s = n_params ? decode_slot(pl, slot, params, n_params, ws, ws_bytes, dev_status) : LSA_OK;
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
