// Sparse attention for callers that cannot allocate device memory.
//
// lsa_sparse_attn needs a caller-provided workspace for its split-KV partial results when
// n_split > 1.  Some callers have no way to obtain one: code running under an allocator
// that forbids new device allocations after start-up (a serving runtime with a
// pre-reserved memory pool that is full, a plugin host that owns every cudaMalloc), or a
// caller without a CUDA allocator of its own.  lsa_sparse_attn_noalloc serves them: its
// split partials live in one file-scope device array, sized once at compile time and
// held by every GPU that loads this library until the process exits.  The call itself
// allocates nothing.
#include <mutex>

#include "kernels.cuh"

namespace {

static_assert(LSA_NOALLOC_SCRATCH_BYTES % 256 == 0, "scratch size");

// The scratch array.  In host code this name is only a host-side stand-in for the symbol,
// not a device address: the device address is obtained with cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_attn_scratch[LSA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once per device.
lsa_status scratch_for_current_device(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LSA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_attn_scratch);
        if (e != cudaSuccess || p == nullptr) {
            cudaGetLastError();   // clear the non-sticky error so it is not reported by a later call
            return LSA_ERR_CUDA;
        }
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return LSA_OK;
}

}  // namespace

extern "C" lsa_status lsa_sparse_attn_noalloc(const lsa_batch* batch, const void* q, int H, int Dqk,
                                              const lsa_cache* kv, const lsa_cache* v, int Dv, const int32_t* idx,
                                              int64_t ld_idx, const int32_t* count, float sm_scale, int n_split,
                                              void* o, float* lse, int32_t* dev_status, void* stream) {
    if (!batch || batch->T < 0 || H < 0 || Dv < 0) return LSA_ERR_INVALID_ARG;
    if (n_split < 1 || n_split > 64) return LSA_ERR_INVALID_ARG;
    const size_t need = lsa_attn_workspace_size(batch->T, H, Dv, n_split);
    if (need > (size_t)LSA_NOALLOC_SCRATCH_BYTES) return LSA_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (need > 0) {
        const lsa_status s = scratch_for_current_device(&scratch);
        if (s != LSA_OK) return s;
    }
    return lsa_sparse_attn(batch, q, H, Dqk, kv, v, Dv, idx, ld_idx, count, sm_scale, n_split, o, lse, scratch,
                           need > 0 ? (size_t)LSA_NOALLOC_SCRATCH_BYTES : 0, dev_status, stream);
}
