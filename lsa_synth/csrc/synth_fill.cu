// Device filler for the synthetic LSA inputs: writes the same bytes as the host generator
// (lsa_synth/gen.py) directly into GPU memory.  Integer hashing, an exact Irwin-Hall(12)
// normal, and single correctly rounded float32 operations (no contraction), so the two
// implementations agree bit for bit.  Input generation only: none of the LSA arithmetic.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr uint64_t kGold = 0x9E3779B97F4A7C15ull;

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

__device__ __forceinline__ float normal_at(uint64_t key, uint64_t ctr) {
    uint32_t s = 0;
    const uint64_t base = ctr * 3ull;
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        const uint64_t h = mix64(key + (base + j) * kGold);
        s += (uint32_t)(h & 0xffff) + (uint32_t)((h >> 16) & 0xffff) + (uint32_t)((h >> 32) & 0xffff) +
             (uint32_t)(h >> 48);
    }
    const int centred = 2 * (int)s - 786420;
    return __fmul_rn((float)centred, 0x1p-17f);
}

__device__ __forceinline__ uint8_t to_e4m3(float y) {
    uint16_t r;
    asm("{ .reg .b16 t; cvt.rn.satfinite.e4m3x2.f32 t, %1, %2; mov.b16 %0, t; }" : "=h"(r) : "f"(0.f), "f"(y));
    return (uint8_t)(r & 0xff);
}

__device__ __forceinline__ uint64_t row_ctr(int64_t r, int dim, int cache_mode, int L_alloc) {
    if (!cache_mode) return (uint64_t)r * (uint64_t)dim;
    const uint64_t b = (uint64_t)(r / L_alloc), l = (uint64_t)(r % L_alloc);
    return ((b << 22) | l) << 10;
}

// fmt: 0 = bf16, 1 = fp8 e4m3 + per-row scale, 2 = float32.  One warp per row.
template <int MAXV>
__global__ void fill_rows(void* out, float* scale_out, int fmt, int64_t n_rows, int dim, int cache_mode,
                          int L_alloc, uint64_t key, const int64_t* rows, const float* dirs) {
    const int lane = threadIdx.x & 31;
    const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (wid >= n_rows) return;
    const int64_t r = rows ? rows[wid] : wid;
    const uint64_t base = row_ctr(r, dim, cache_mode, L_alloc);
    const float* dir = rows ? dirs + (size_t)(r / L_alloc) * dim : nullptr;
    float v[MAXV];
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
        const int d = lane + 32 * i;
        float x = 0.f;
        if (d < dim) {
            x = normal_at(key, base + (uint64_t)d);
            if (dir) x = __fadd_rn(__fmul_rn(0.3f, x), dir[d]);
        }
        v[i] = x;
        amax = fmaxf(amax, fabsf(x));
    }
    if (fmt == 0) {
        __nv_bfloat16* o = static_cast<__nv_bfloat16*>(out) + (size_t)r * dim;
#pragma unroll
        for (int i = 0; i < MAXV; ++i)
            if (lane + 32 * i < dim) o[lane + 32 * i] = __float2bfloat16_rn(v[i]);
    } else if (fmt == 2) {
        float* o = static_cast<float*>(out) + (size_t)r * dim;
#pragma unroll
        for (int i = 0; i < MAXV; ++i)
            if (lane + 32 * i < dim) o[lane + 32 * i] = v[i];
    } else {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        float scale = 1.f, inv = 1.f;
        if (amax > 0.f) {
            scale = __fdiv_rn(amax, 448.f);
            inv = __fdiv_rn(448.f, amax);
        }
        uint8_t* o = static_cast<uint8_t*>(out) + (size_t)r * dim;
#pragma unroll
        for (int i = 0; i < MAXV; ++i)
            if (lane + 32 * i < dim) o[lane + 32 * i] = to_e4m3(__fmul_rn(v[i], inv));
        if (lane == 0) scale_out[r] = scale;
    }
}

__global__ void fill_uniform(float* out, int64_t n, uint64_t key) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const uint64_t h = mix64(key + (uint64_t)i * kGold);
    out[i] = __fmul_rn((float)(uint32_t)(h >> 40), 0x1p-24f);
}

}  // namespace

extern "C" {

// Fills n_rows rows of `dim` values (row r at out + r * dim) or, when `rows` is given, only
// the listed rows, overwriting them with the planted form dir[b] + 0.3 * noise (b = r / L_alloc).
// Returns a cudaError_t code.
int synth_fill_rows(void* out, float* scale_out, int fmt, int64_t n_rows, int dim, int cache_mode, int L_alloc,
                    uint64_t key, const int64_t* rows, const float* dirs, void* stream) {
    if (dim < 1 || dim > 1024 || n_rows < 0 || L_alloc < 1) return (int)cudaErrorInvalidValue;
    if (n_rows == 0) return 0;
    const int threads = 256;
    const int64_t blocks = (n_rows * 32 + threads - 1) / threads;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (dim <= 64) fill_rows<2><<<(unsigned)blocks, threads, 0, st>>>(out, scale_out, fmt, n_rows, dim, cache_mode, L_alloc, key, rows, dirs);
    else if (dim <= 128) fill_rows<4><<<(unsigned)blocks, threads, 0, st>>>(out, scale_out, fmt, n_rows, dim, cache_mode, L_alloc, key, rows, dirs);
    else if (dim <= 576) fill_rows<18><<<(unsigned)blocks, threads, 0, st>>>(out, scale_out, fmt, n_rows, dim, cache_mode, L_alloc, key, rows, dirs);
    else fill_rows<32><<<(unsigned)blocks, threads, 0, st>>>(out, scale_out, fmt, n_rows, dim, cache_mode, L_alloc, key, rows, dirs);
    return (int)cudaGetLastError();
}

int synth_fill_uniform(float* out, int64_t n, uint64_t key, void* stream) {
    if (n <= 0) return 0;
    fill_uniform<<<(unsigned)((n + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(out, n, key);
    return (int)cudaGetLastError();
}

}  // extern "C"
