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
#include <cuda.h>

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
unsigned long long g_scratch_ctx[kMaxDevices] = {};   // context ID the address belongs to

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// The unique ID of the current CUDA context (IDs are never reused within a process), or 0
// when it cannot be read.  A device reset destroys the context and its module; the next
// runtime call creates a new one with a new ID, so an address cached under the old ID is
// never used again.
unsigned long long current_context_id() {
    static CtxGetCurrentFn get_cur = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_cur = reinterpret_cast<CtxGetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_cur || !get_id || get_cur(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of the scratch array in the current device's context: looked up once per
// device and context (with that device current), again after the context changes (or on
// every call while the context ID cannot be read).
lsa_status scratch_for_current_device(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LSA_ERR_CUDA;
    const unsigned long long ctx = current_context_id();
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev] || ctx == 0 || g_scratch_ctx[dev] != ctx) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_attn_scratch);
        if (e != cudaSuccess || p == nullptr) {
            cudaGetLastError();   // clear the non-sticky error so it is not reported by a later call
            g_scratch_ptr[dev] = nullptr;
            return LSA_ERR_CUDA;
        }
        g_scratch_ptr[dev] = p;
        g_scratch_ctx[dev] = ctx;
    }
    *out = g_scratch_ptr[dev];
    return LSA_OK;
}

}  // namespace

extern "C" lsa_status lsa_sparse_attn_noalloc(const lsa_batch* batch, const void* q, int H, int Dqk,
                                              const lsa_cache* kv, const lsa_cache* v, int Dv, const int32_t* idx,
                                              int64_t ld_idx, const int32_t* count, float sm_scale, int n_split,
                                              void* o, float* lse, int32_t* dev_status, void* stream) {
    // The same argument checks, in the same order, as lsa_sparse_attn; the scratch size after them.
    lsa_status s = lsa::attn_validate(batch, q, H, Dqk, kv, v, Dv, idx, ld_idx, count, sm_scale, n_split, o);
    if (s != LSA_OK || batch->T == 0) return s;
    const size_t need = lsa_attn_workspace_size(batch->T, H, Dv, n_split);
    if (need > (size_t)LSA_NOALLOC_SCRATCH_BYTES) return LSA_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (need > 0) {
        s = scratch_for_current_device(&scratch);
        if (s != LSA_OK) return s;
    }
    return lsa_sparse_attn(batch, q, H, Dqk, kv, v, Dv, idx, ld_idx, count, sm_scale, n_split, o, lse, scratch,
                           need > 0 ? (size_t)LSA_NOALLOC_SCRATCH_BYTES : 0, dev_status, stream);
}
