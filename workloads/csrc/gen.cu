// gen.cu - device side of the workload generator (see workloads/gen.py for
// the definition).  Integer SplitMix64 streams, Irwin-Hall normals scaled by
// one binary32 multiply, Student-t(3) from four normals, 1% outliers; all
// binary32 operations are explicitly rounded so the bits equal the numpy
// implementation's.  This library holds no optimizer arithmetic.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

__device__ __forceinline__ uint64_t mix64(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

__device__ __forceinline__ uint64_t word(uint64_t key, uint64_t c) { return mix64(key + (c + 1) * kGamma); }

__device__ __forceinline__ int ih8(uint64_t key, uint64_t i, int j, int J)
{
    const uint64_t base = (i * (uint64_t)J + (uint64_t)j) * 2;
    int64_t s = 0;
    for (int off = 0; off < 2; off++) {
        const uint64_t w = word(key, base + off);
        s += (int64_t)(w & 0xFFFF) + (int64_t)((w >> 16) & 0xFFFF) + (int64_t)((w >> 32) & 0xFFFF) +
             (int64_t)(w >> 48);
    }
    return (int)(2 * s - 8 * 65535);
}

__device__ __forceinline__ float normal(uint64_t key, uint64_t i, float c, int j, int J)
{
    return __fmul_rn((float)ih8(key, i, j, J), c);
}

// dist: 0 normal(c), 1 normal(c) with 1% x100 outliers (key_o), 2 Student-t(3) * scale
__device__ __forceinline__ float draw(int dist, uint64_t key, uint64_t key_o, uint64_t i, float c,
                                      float c1, float scale)
{
    if (dist == 2) {
        const float z0 = normal(key, i, c1, 0, 4);
        const float z1 = normal(key, i, c1, 1, 4);
        const float z2 = normal(key, i, c1, 2, 4);
        const float z3 = normal(key, i, c1, 3, 4);
        float s = __fmul_rn(z1, z1);
        s = __fadd_rn(s, __fmul_rn(z2, z2));
        s = __fadd_rn(s, __fmul_rn(z3, z3));
        s = __fdiv_rn(s, 3.0f);
        const float t = __fdiv_rn(z0, __fsqrt_rn(s));
        return __fmul_rn(t, scale);
    }
    float z = normal(key, i, c, 0, 1);
    if (dist == 1 && (word(key_o, i) % 100ull) == 0ull) z = __fmul_rn(z, 100.0f);
    return z;
}

__global__ void gen_f32_kernel(float* out, int64_t n, int dist, uint64_t key, uint64_t key_o, float c,
                               float c1, float scale)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
        out[i] = draw(dist, key, key_o, (uint64_t)i, c, c1, scale);
}

__global__ void gen_16_kernel(uint16_t* out, int64_t n, int dist, uint64_t key, uint64_t key_o,
                              float c, float c1, float scale, int fp16)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        const float v = draw(dist, key, key_o, (uint64_t)i, c, c1, scale);
        out[i] = fp16 ? __half_as_ushort(__float2half_rn(v)) : __bfloat16_as_ushort(__float2bfloat16_rn(v));
    }
}

unsigned grid_of(int64_t n)
{
    int64_t g = (n + 255) / 256;
    return (unsigned)(g > 148 * 16 ? 148 * 16 : (g < 1 ? 1 : g));
}

}  // namespace

extern "C" {

int fo_gen_f32(float* out, int64_t n, int dist, uint64_t key, uint64_t key_o, float c, float c1,
               float scale, void* stream)
{
    if (n <= 0) return 0;
    gen_f32_kernel<<<grid_of(n), 256, 0, (cudaStream_t)stream>>>(out, n, dist, key, key_o, c, c1, scale);
    return (int)cudaGetLastError();
}

int fo_gen_16(uint16_t* out, int64_t n, int dist, uint64_t key, uint64_t key_o, float c, float c1,
              float scale, int fp16, void* stream)
{
    if (n <= 0) return 0;
    gen_16_kernel<<<grid_of(n), 256, 0, (cudaStream_t)stream>>>(out, n, dist, key, key_o, c, c1, scale,
                                                                  fp16);
    return (int)cudaGetLastError();
}

}  // extern "C"
