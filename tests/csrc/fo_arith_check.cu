// fo_arith_check.cu - exhaustive / dense GPU checks of the identities the
// step kernel's fast path relies on (test infrastructure, not the product).
// Each check runs the kernel's own device functions (fo_kernels.cuh) against
// the IEEE operation they replace and counts the inputs where the bits
// differ.  Every kernel is a grid-stride loop over an index range; it writes
// only to the counter / example arrays handed in by the host, at indices
// below their stated sizes.
#include <cstdint>
#include <cuda_runtime.h>

#include "fo_kernels.cuh"

namespace {

__device__ __forceinline__ float rcp_full(float x)
{
    float r;
    asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ float rsqrt_full(float x)
{
    float r;
    asm("rsqrt.approx.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ void note(unsigned long long* cnt, uint32_t* ex, int slot, uint32_t v)
{
    const unsigned long long k = atomicAdd(&cnt[slot], 1ull);
    if (k < 4) ex[4 * slot + (int)k] = v;
}

// cnt[0]: rcp flush-to-zero form != full form with a normal full result
// cnt[1]: rsqrt flush-to-zero form != full form
// over every positive normal binary32
__global__ void k_ftz(unsigned long long* cnt, uint32_t* ex)
{
    const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    for (uint64_t i = 0x00800000ull + (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < 0x7F800000ull;
         i += stride) {
        const float x = __uint_as_float((uint32_t)i);
        const float a = fo::rcp_approx(x), b = rcp_full(x);
        if (__float_as_uint(a) != __float_as_uint(b) && fabsf(b) >= 1.17549435e-38f) note(cnt, ex, 0, (uint32_t)i);
        if (__float_as_uint(fo::rsqrt_approx(x)) != __float_as_uint(rsqrt_full(x))) note(cnt, ex, 1, (uint32_t)i);
    }
}

// cnt[0]: sqrt2_nr(v) != sqrt.rn(v) for v = +0 and every binary32 in (0, 2^64)
// cnt[1]: sqrt2_nr(v) is not NaN for v in [2^64, inf]
__global__ void k_sqrt(unsigned long long* cnt, uint32_t* ex)
{
    const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i <= 0x7F800000ull; i += 2 * stride) {
        const uint32_t i0 = (uint32_t)i;
        const uint32_t i1 = (uint32_t)(i + stride <= 0x7F800000ull ? i + stride : i);
        const float2 v = make_float2(__uint_as_float(i0), __uint_as_float(i1));
        const float2 s = fo::sqrt2_nr(v);
        const uint32_t lim = 0x5F800000u;  // 2^64
        if (i0 < lim) {
            if (__float_as_uint(s.x) != __float_as_uint(__fsqrt_rn(v.x))) note(cnt, ex, 0, i0);
        } else if (!isnan(s.x)) {
            note(cnt, ex, 1, i0);
        }
        if (i1 < lim) {
            if (__float_as_uint(s.y) != __float_as_uint(__fsqrt_rn(v.y))) note(cnt, ex, 0, i1);
        } else if (!isnan(s.y)) {
            note(cnt, ex, 1, i1);
        }
    }
}

__device__ __forceinline__ uint64_t splitmix(uint64_t z)
{
    z += 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

// cnt[0]: div2_nr(x, b) != div.rn(x, b) on n random pairs with b in
// [2^-60, 2^20) and |x| in [2^-80, 2^61) (exponents uniform, significands
// uniform), plus x = +0
__global__ void k_div(uint64_t n, uint64_t seed, unsigned long long* cnt, uint32_t* ex)
{
    const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        const uint64_t r = splitmix(seed ^ (i * 0xD1B54A32D192ED03ull));
        const uint32_t eb = 127u - 60u + (uint32_t)((r >> 0) % 80u);    // 2^-60 .. 2^19
        const uint32_t ea = 127u - 80u + (uint32_t)((r >> 8) % 141u);   // 2^-80 .. 2^60
        const uint32_t mb = (uint32_t)(r >> 16) & 0x7FFFFFu;
        const uint32_t ma = (uint32_t)(r >> 39) & 0x7FFFFFu;
        const uint32_t sa = (uint32_t)(r >> 63) << 31;
        float a = __uint_as_float(sa | (ea << 23) | ma);
        if ((i & 1023u) == 0u) a = 0.0f;
        const float b = __uint_as_float((eb << 23) | mb);
        const float2 q = fo::div2_nr(make_float2(a, a), make_float2(b, b), make_float2(-b, -b));
        if (__float_as_uint(q.x) != __float_as_uint(__fdiv_rn(a, b))) {
            const unsigned long long k = atomicAdd(&cnt[0], 1ull);
            if (k < 2) {
                ex[2 * k] = __float_as_uint(a);
                ex[2 * k + 1] = __float_as_uint(b);
            }
        }
    }
}

// cnt[0]: largest ulp distance of rcp_approx(d) from RN(1/d) over every
// binary32 d in [1, 2]; cnt[1]: scale_recips(S, S) != (1/S, 255/S) by div.rn
// for every positive finite fp16 S (and S = 0 must give (0, 0))
__global__ void k_rcp_scales(unsigned long long* cnt, uint32_t* ex)
{
    const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i <= (1ull << 23); i += stride) {
        const float d = __uint_as_float(0x3F800000u + (uint32_t)i);  // [1, 2]
        const float r = fo::rcp_approx(d), e = __fdiv_rn(1.0f, d);
        const int u = (int)__float_as_uint(r) - (int)__float_as_uint(e);
        atomicMax(&cnt[0], (unsigned long long)(u < 0 ? -u : u));
    }
    for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < 0x7C00ull; i += stride) {
        const float S = __half2float(__ushort_as_half((unsigned short)i));
        const float2 q = fo::scale_recips(S, S);
        const float e1 = S == 0.0f ? 0.0f : __fdiv_rn(1.0f, S), e2 = S == 0.0f ? 0.0f : __fdiv_rn(255.0f, S);
        if (__float_as_uint(q.x) != __float_as_uint(e1) || __float_as_uint(q.y) != __float_as_uint(e2))
            note(cnt, ex, 1, (uint32_t)i);
    }
}

// The fast 16-bit-master ECC8 codec of the step kernel against the exact one
// (the device functions of the reference path), for W = bf16 (0) or fp16 (1):
// cnt[0]: decode mismatches over every 16-bit pattern x' with every code in
// [-127, 127] (pairs of elements, both lanes of a pair); cnt[1]: encode
// mismatches (x' bits or code) over every binary32 x with |x| below the fast
// path's limit (other x send the slice to the exact path).  Non-finite x'
// are skipped for the decode, whose fast result is then caught downstream,
// and so is a bf16 +-0 with an inward code, whose fast result must be out of
// range.
template <int W>
__global__ void k_codec(unsigned long long* cnt, uint32_t* ex)
{
    // The fp16 fast codec takes a warp vote, so every call below is made by
    // whole warps: the stride and both loop bounds are multiples of 32, and
    // the 32 consecutive items of a warp share one pattern h (128 items per h),
    // so a warp skips a non-finite h together.
    const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < (1ull << 16) * 128ull; i += stride) {
        const uint32_t h = (uint32_t)(i >> 7), k = (uint32_t)(i & 127u);
        if (fo::nonfinite16<W>(h)) continue;
        // codes k and -k for the two lanes of the pair
        const int r0 = (int)k, r1 = -(int)k;
        uint32_t e[2] = {((uint32_t)r0 & 0xFFu) | (((uint32_t)r1 & 0xFFu) << 8), 0u};
        const float2 x = fo::fast_decode_pair<W, 8>(h | (h << 16), e, 0);
        const float e0 = fo::ecc_decode<W, 8>(h, r0), e1 = fo::ecc_decode<W, 8>(h, r1);
        // bf16 +-0 with an inward code: the fast decode must land outside the
        // fast path's range (the slice is then redone exactly)
        const bool flagged1 = W == 0 && (h & 0x7FFFu) == 0u && r1 < 0;
        const bool ok1 = flagged1 ? !(fabsf(x.y) < 3.39615136e38f) : __float_as_uint(x.y) == __float_as_uint(e1);
        if (__float_as_uint(x.x) != __float_as_uint(e0) || !ok1) note(cnt, ex, 0, (uint32_t)i);
    }
    const uint32_t lim = W == 0 ? 0x7F7F8000u : 0x477FF000u;  // kDecodeLimit, 65520
    for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < (uint64_t)lim; i += stride) {
        const float xa = __uint_as_float((uint32_t)i), xb = -xa;
        uint32_t codes;
        const uint32_t wo = fo::fast_encode_pair<W, 8>(make_float2(xa, xb), codes);
        const int c0 = (int)(int16_t)(codes & 0xFFFFu), c1 = (int)(int16_t)(codes >> 16);
        const uint32_t pa = fo::downcast16<W>(xa), pb = fo::downcast16<W>(xb);
        if ((wo & 0xFFFFu) != pa || (wo >> 16) != pb || c0 != fo::ecc_encode<W, 8>(xa, pa) ||
            c1 != fo::ecc_encode<W, 8>(xb, pb))
            note(cnt, ex, 1, (uint32_t)i);
    }
}

// cnt[0]: div2_nr(x, b) != div.rn(x, b) over every pair of significands:
// x in [1, 2) (all 2^23) for each of the divisors b in [1, 2) with
// significands [b0, b0 + nb); x in pairs, both lanes.  Together with the
// power-of-two scaling check below this covers the divider's stated range.
__global__ void k_div_grid(uint32_t b0, uint32_t nb, unsigned long long* cnt, uint32_t* ex)
{
    const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    const uint64_t total = (uint64_t)nb << 22;  // (b, x pair) items
    for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
        const uint32_t mb = b0 + (uint32_t)(i >> 22);
        const uint32_t mx = (uint32_t)(i & ((1u << 22) - 1u)) << 1;
        const float b = __uint_as_float(0x3F800000u | mb);
        const float2 x = make_float2(__uint_as_float(0x3F800000u | mx), __uint_as_float(0x3F800000u | (mx + 1u)));
        const float2 q = fo::div2_nr(x, make_float2(b, b), make_float2(-b, -b));
        const bool bad0 = __float_as_uint(q.x) != __float_as_uint(__fdiv_rn(x.x, b));
        const bool bad1 = __float_as_uint(q.y) != __float_as_uint(__fdiv_rn(x.y, b));
        if (bad0 || bad1) {
            const unsigned long long k = atomicAdd(&cnt[0], 1ull);
            if (k < 2) {
                ex[2 * k] = __float_as_uint(bad0 ? x.x : x.y);
                ex[2 * k + 1] = __float_as_uint(b);
            }
        }
    }
}

// cnt[0]: rcp_approx(b 2^e) != rcp_approx(b) 2^-e for a binary32 b in [1, 2)
// and an exponent e in [-61, 61] (the approximate reciprocal scales exactly by
// powers of two there); cnt[1]: the same for rsqrt_approx(b 2^(2e)) =
// rsqrt_approx(b) 2^-e, e in [-30, 30]
__global__ void k_rcp_scaling(unsigned long long* cnt, uint32_t* ex)
{
    const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < (1ull << 23) * 123ull; i += stride) {
        const uint32_t m = (uint32_t)(i % (1ull << 23));
        const int e = (int)(i / (1ull << 23)) - 61;
        const float b = __uint_as_float(0x3F800000u | m);
        const float be = __uint_as_float((uint32_t)(127 + e) << 23 | m);
        const float r = fo::rcp_approx(b), re = fo::rcp_approx(be);
        if (__float_as_uint(re) != __float_as_uint(__fmul_rn(r, __uint_as_float((uint32_t)(127 - e) << 23))))
            note(cnt, ex, 0, __float_as_uint(be));
        if (e >= -30 && e <= 30) {
            const float b2 = __uint_as_float((uint32_t)(127 + 2 * e) << 23 | m);
            const float s = fo::rsqrt_approx(b), s2 = fo::rsqrt_approx(b2);
            if (__float_as_uint(s2) != __float_as_uint(__fmul_rn(s, __uint_as_float((uint32_t)(127 - e) << 23))))
                note(cnt, ex, 1, __float_as_uint(b2));
        }
    }
}

// The step kernel's bounded wait on an mbarrier (one block of 64 threads):
// warp 0 waits on a barrier nothing ever arrives on, with a limit of
// limit_ns; warp 1 waits on a barrier its lane 0 completed by arriving.
// cnt[0]: threads of warp 0 whose wait did not give up; cnt[1]: threads of
// warp 1 whose wait gave up; cnt[2]: the longest wait of warp 0 in ns;
// cnt[3]: the shortest.
__global__ void k_wait(unsigned long long limit_ns, unsigned long long* cnt)
{
    __shared__ __align__(8) uint64_t bars[2];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t bar = (uint32_t)__cvta_generic_to_shared(&bars[warp]);
    if (lane == 0) {
        fo::mbar_init(bar, 1);
        fo::mbar_init_fence();
    }
    __syncthreads();
    if (warp == 1 && lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
    __syncwarp();
    const unsigned long long t0 = fo::globaltimer();
    const bool done = fo::mbar_wait_bounded(bar, 0u, limit_ns);
    const unsigned long long dt = fo::globaltimer() - t0;
    if (warp == 0) {
        if (done) atomicAdd(&cnt[0], 1ull);
        atomicMax(&cnt[2], dt);
        atomicMin(&cnt[3], dt);
    } else if (!done) {
        atomicAdd(&cnt[1], 1ull);
    }
}

int launch_done(unsigned long long* hcnt, uint32_t* hex, unsigned long long* dcnt, uint32_t* dex)
{
    if (cudaGetLastError() != cudaSuccess) return 2;
    if (cudaDeviceSynchronize() != cudaSuccess) return 3;
    if (cudaMemcpy(hcnt, dcnt, 4 * sizeof(unsigned long long), cudaMemcpyDeviceToHost) != cudaSuccess) return 4;
    if (cudaMemcpy(hex, dex, 16 * sizeof(uint32_t), cudaMemcpyDeviceToHost) != cudaSuccess) return 4;
    return 0;
}

}  // namespace

// which: 0 ftz forms, 1 square root, 2 division (n pairs, seed), 3 rcp bound
// and scale reciprocals, 4 / 5 fast bf16 / fp16 ECC8 codec, 6 division over
// the significand grid (n divisor significands from seed), 7 power-of-two
// scaling of the approximate reciprocal and reciprocal square root, 8 the
// bounded mbarrier wait (n = its limit in ns).  cnt: 4 counters, ex: 16 example words (host memory).
extern "C" __attribute__((visibility("default"))) int fo_arith_check(int which, uint64_t n, uint64_t seed,
                                                                     unsigned long long* cnt, uint32_t* ex)
{
    unsigned long long* dcnt = nullptr;
    uint32_t* dex = nullptr;
    if (cudaMalloc(&dcnt, 4 * sizeof(unsigned long long)) != cudaSuccess) return 1;
    if (cudaMalloc(&dex, 16 * sizeof(uint32_t)) != cudaSuccess) {
        cudaFree(dcnt);
        return 1;
    }
    cudaMemset(dcnt, 0, 4 * sizeof(unsigned long long));
    cudaMemset(dex, 0, 16 * sizeof(uint32_t));
    const int grid = 148 * 8, block = 256;
    switch (which) {
    case 0: k_ftz<<<grid, block>>>(dcnt, dex); break;
    case 1: k_sqrt<<<grid, block>>>(dcnt, dex); break;
    case 2: k_div<<<grid, block>>>(n, seed, dcnt, dex); break;
    case 3: k_rcp_scales<<<grid, block>>>(dcnt, dex); break;
    case 4: k_codec<0><<<grid, block>>>(dcnt, dex); break;
    case 5: k_codec<1><<<grid, block>>>(dcnt, dex); break;
    case 6:
        // divisor significands [seed, seed + n) (n <= 2^23 - seed; a slice per
        // call keeps each launch short)
        if (seed >= (1ull << 23) || n == 0 || n > (1ull << 23) - seed) {
            cudaFree(dcnt);
            cudaFree(dex);
            return 5;
        }
        k_div_grid<<<grid, block>>>((uint32_t)seed, (uint32_t)n, dcnt, dex);
        break;
    case 7: k_rcp_scaling<<<grid, block>>>(dcnt, dex); break;
    case 8: {
        // n: the wait limit in ns (at most 1 s); cnt[3] starts at its maximum
        if (n == 0 || n > 1000000000ull) {
            cudaFree(dcnt);
            cudaFree(dex);
            return 5;
        }
        const unsigned long long big = ~0ull;
        cudaMemcpy(dcnt + 3, &big, sizeof big, cudaMemcpyHostToDevice);
        k_wait<<<1, 64>>>(n, dcnt);
        break;
    }
    default: break;
    }
    const int rc = launch_done(cnt, ex, dcnt, dex);
    cudaFree(dcnt);
    cudaFree(dex);
    return rc;
}
