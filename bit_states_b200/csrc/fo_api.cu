// fo_api.cu - host side of libfo: argument validation, the binary32 host
// scalars of one step, packing of the multi-tensor descriptor table into
// kernel parameters, and launches.  See include/fo.h for the contract.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <limits>
#include <mutex>
#include <string>

#include <cuda_runtime.h>

#include "fo.h"
#include "fo_kernels.cuh"

namespace {

thread_local std::string g_last_error;

fo_status fail(fo_status s, const std::string& msg)
{
    g_last_error = msg;
    return s;
}

fo_status cuda_fail(cudaError_t e, const char* where)
{
    return fail(FO_ERR_CUDA, std::string(where) + ": " + cudaGetErrorName(e) + " (" +
                                 cudaGetErrorString(e) + ")");
}

// ---- per-device launch constants -------------------------------------------

constexpr int kMaxDevices = 64;
std::once_flag g_dev_once[kMaxDevices];
int g_sm_count[kMaxDevices];

fo_status device_sms(int* sms)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(FO_ERR_CUDA, "device ordinal out of range");
    std::call_once(g_dev_once[dev], [dev] {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n = 0;
        g_sm_count[dev] = n;
    });
    if (g_sm_count[dev] <= 0) return fail(FO_ERR_CUDA, "could not query the SM count");
    *sms = g_sm_count[dev];
    return FO_OK;
}

// ---- validation ------------------------------------------------------------

bool aligned(const void* p, uintptr_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

fo_status check_format(const fo_format& f)
{
    if ((f.w_dtype != FO_DT_BF16 && f.w_dtype != FO_DT_FP16) ||
        (f.grad_dtype != FO_DT_BF16 && f.grad_dtype != FO_DT_FP16))
        return fail(FO_ERR_UNSUPPORTED, "w_dtype / grad_dtype must be FO_DT_BF16 or FO_DT_FP16");
    if (f.ecc_bits != 8 && f.ecc_bits != 16)
        return fail(FO_ERR_UNSUPPORTED, "ecc_bits must be 8 or 16");
    return FO_OK;
}

fo_status check_tensors(const fo_tensor* t, int n, const fo_format& f, bool adam)
{
    if (n < 0) return fail(FO_ERR_INVALID_ARG, "n_tensors < 0");
    if (n > FO_MAX_TENSORS_PER_CALL) return fail(FO_ERR_TOO_MANY_TENSORS, "n_tensors too large");
    if (n > 0 && t == nullptr) return fail(FO_ERR_INVALID_ARG, "tensor array is NULL");
    for (int i = 0; i < n; i++) {
        const fo_tensor& x = t[i];
        char where[64];
        snprintf(where, sizeof where, "tensor %d: ", i);
        if (x.numel < 0) return fail(FO_ERR_INVALID_ARG, std::string(where) + "numel < 0");
        if (x.numel > FO_MAX_NUMEL) return fail(FO_ERR_INVALID_ARG, std::string(where) + "numel > FO_MAX_NUMEL");
        if (x.numel == 0) continue;
        if (!x.w || !x.ecc || !x.grad || !x.m_q || !x.m_scale)
            return fail(FO_ERR_INVALID_ARG, std::string(where) + "NULL w / ecc / grad / m_q / m_scale");
        if (adam && (!x.v_q || !x.v_scale))
            return fail(FO_ERR_INVALID_ARG, std::string(where) + "NULL v_q / v_scale");
        if (!aligned(x.w, 2) || !aligned(x.grad, 2) || !aligned(x.m_scale, 2) ||
            (adam && !aligned(x.v_scale, 2)) || (f.ecc_bits == 16 && !aligned(x.ecc, 2)))
            return fail(FO_ERR_ALIGNMENT, std::string(where) + "16-bit array not 2-byte aligned");
    }
    return FO_OK;
}

// ---- launch of one step over a tensor list -----------------------------------

using StepKernel = void (*)(const fo::StepParams);
using SmallStepKernel = void (*)(const fo::StepParamsT<fo::kSmallTensors>);

// one step kernel (two parameter-table sizes) with its launch geometry
// (fo::Geometry)
struct StepLaunch {
    StepKernel k;
    SmallStepKernel ks;
    int threads;    // threads per block
    int smem;       // dynamic shared memory per block (stage buffers)
    int64_t chunk;  // elements per chunk
    int ecc_bits;
    int lane;       // elements per lane in a staged slice
};

template <int WDT, int GDT, int NB, int KIND>
StepLaunch step_launch()
{
    using G = fo::Geometry<NB, KIND>;
    return {fo::step_kernel<WDT, GDT, NB, KIND, fo::kMaxTensorsPerLaunch>,
            fo::step_kernel<WDT, GDT, NB, KIND, fo::kSmallTensors>,
            G::kBlockThreads, G::kSmemBytes, G::kChunk, NB, G::kLane};
}

// the step kernel of a format (k = nullptr if the format is not provided)
template <int KIND>
StepLaunch pick_step(const fo_format& f)
{
#define FO_PICK(W, G, N)                                                                  \
    if (f.w_dtype == W && f.grad_dtype == G && f.ecc_bits == N) return step_launch<W, G, N, KIND>();
    FO_PICK(0, 0, 8) FO_PICK(0, 1, 8) FO_PICK(1, 0, 8) FO_PICK(1, 1, 8)
    FO_PICK(0, 0, 16) FO_PICK(0, 1, 16) FO_PICK(1, 0, 16) FO_PICK(1, 1, 16)
#undef FO_PICK
    return {nullptr, nullptr, 0, 0, 0, 0, 0};
}

struct LaunchCache {
    std::mutex mu;
    int dev[128] = {};
    const void* fn[128] = {};
    int blocks[128] = {};
    int n = 0;
} g_launch;

// once per (device, kernel): allow the dynamic shared memory of the stage
// buffers and find how many blocks fit on one SM
template <class KERNEL>
fo_status prepare_kernel(KERNEL k, int threads, int smem, int* blocks_per_sm)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    std::lock_guard<std::mutex> lock(g_launch.mu);
    for (int i = 0; i < g_launch.n; i++)
        if (g_launch.fn[i] == (const void*)k && g_launch.dev[i] == dev) {
            *blocks_per_sm = g_launch.blocks[i];
            return FO_OK;
        }
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    int b = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, k, threads, smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
    if (b < 1) b = 1;
    if (g_launch.n < 128) {
        g_launch.fn[g_launch.n] = (const void*)k;
        g_launch.dev[g_launch.n] = dev;
        g_launch.blocks[g_launch.n] = b;
        g_launch.n++;
    }
    *blocks_per_sm = b;
    return FO_OK;
}

// Pack up to MAXT tensors from t[i..] (skipping empty ones) into P and
// launch; returns the index of the first tensor not packed.
template <int MAXT, class KERNEL>
fo_status launch_table(KERNEL kernel, const StepLaunch& L, const fo::Scalars& sc, const fo_tensor* t, int n,
                       int& i, int64_t cap, cudaStream_t stream)
{
    const int64_t chunk = L.chunk;
    const int warps = L.threads / 32;
    // kernel parameters are copied at launch, so one block of host memory
    // per thread serves every launch
    thread_local fo::StepParamsT<MAXT> P;
    std::memset(&P, 0, offsetof(fo::StepParamsT<MAXT>, t));
    P.sc = sc;
    int m = 0;
    int64_t chunks = 0;
    P.chunk_start[0] = 0;
    for (; i < n && m < MAXT; i++) {
        const fo_tensor& x = t[i];
        if (x.numel == 0) continue;
        fo::TensorDesc& d = P.t[m];
        d.w = x.w;
        d.ecc = x.ecc;
        d.grad = x.grad;
        d.mq = x.m_q;
        d.ms = x.m_scale;
        d.vq = x.v_q;
        d.vs = x.v_scale;
        d.numel = x.numel;
        // staged chunks: every array 16-byte aligned (bulk copies, 128-bit
        // stores) and the arrays written with 256-bit stores (weights, 16-bit
        // ECC codes, with 16 elements per lane) 32-byte aligned; other
        // tensors take the scalar path
        const uintptr_t a = (uintptr_t)x.w | (uintptr_t)x.grad | (uintptr_t)x.ecc | (uintptr_t)x.m_q |
                            (uintptr_t)x.m_scale | (uintptr_t)x.v_q | (uintptr_t)x.v_scale;
        const uintptr_t a32 = L.lane == 16 ? ((uintptr_t)x.w | (L.ecc_bits == 16 ? (uintptr_t)x.ecc : 0)) : 0;
        d.n_chunks = (int32_t)((x.numel + chunk - 1) / chunk);
        d.staged = ((a & 15u) == 0 && (a32 & 31u) == 0) ? 1 : 0;
        const int64_t last = x.numel - (int64_t)(d.n_chunks - 1) * chunk;  // elements of the last chunk
        d.last_slices = (int16_t)(last / (32 * L.lane));
        chunks += d.n_chunks;
        P.chunk_start[++m] = chunks;
    }
    if (m == 0) return FO_OK;
    P.n_tensors = m;
    P.total_chunks = chunks;
    // a sentinel past the last tensor keeps the device-side walk bounded
    for (int j = m + 1; j <= MAXT; j++) P.chunk_start[j] = INT64_MAX;
    int64_t grid = (chunks + warps - 1) / warps;
    if (grid > cap) grid = cap;
    // programmatic stream serialization: the kernel may be scheduled while
    // the previous kernel on the stream finishes; it waits for it
    // (griddepcontrol.wait) before touching global memory
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)L.threads);
    cfg.dynamicSmemBytes = (size_t)L.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, P);
    if (e != cudaSuccess) return cuda_fail(e, "step kernel launch");
    return FO_OK;
}

fo_status launch_step(const StepLaunch& L, const fo::Scalars& sc, const fo_tensor* t, int n, cudaStream_t stream)
{
    int live = 0;
    for (int j = 0; j < n; j++) live += t[j].numel > 0;
    if (live == 0) return FO_OK;
    int sms = 0;
    fo_status st = device_sms(&sms);
    if (st != FO_OK) return st;
    int bps = 1;
    if (live <= fo::kSmallTensors) {
        st = prepare_kernel(L.ks, L.threads, L.smem, &bps);
        if (st != FO_OK) return st;
        int i = 0;
        return launch_table<fo::kSmallTensors>(L.ks, L, sc, t, n, i, (int64_t)sms * bps, stream);
    }
    st = prepare_kernel(L.k, L.threads, L.smem, &bps);
    if (st != FO_OK) return st;
    int i = 0;
    while (i < n) {
        st = launch_table<fo::kMaxTensorsPerLaunch>(L.k, L, sc, t, n, i, (int64_t)sms * bps, stream);
        if (st != FO_OK) return st;
    }
    return FO_OK;
}

bool is_finite(double v) { return std::isfinite(v); }

int64_t grid_for(int64_t n, int sms)
{
    int64_t g = (n + fo::kThreads - 1) / fo::kThreads;
    const int64_t cap = (int64_t)sms * 8;
    if (g > cap) g = cap;
    return g < 1 ? 1 : g;
}

}  // namespace

extern "C" {

// Bounds of the kernel's fast path for AdamW (its Newton-Raphson update; see
// lane_adamw_fast): s[8] = -lr/(1-b1^t) * 2^-40, s[9] = the smallest
// |x (1-lr wd)| for which an update of at most
//   U = |lr/(1-b1^t)| (2^-119 / eps + 2^-126)
// cannot change x'' (U < |x (1-lr wd)| 2^-26), s[10] = the largest sqrt(v')
// that keeps the divisor sqrt(v') / sqrt(1-b2^t) + eps at or below 2^20 and
// the variance scale below its saturation at 65504 (the largest fp16).
// Where those conditions cannot hold (eps < 2^-60, a step size too small to
// scale by 2^-40) s[9] is +inf and every slice takes the exact path.
static void adamw_fast_bounds(fo::Scalars& sc)
{
    const float step = sc.s[4], ibc2 = sc.s[5], eps = sc.s[6];
    const float inf = std::numeric_limits<float>::infinity();
    sc.s[8] = -step * 0x1p-40f;
    const bool ok = eps >= 0x1p-60f && eps < 0x1p19f && (step == 0.0f || std::fabs(step) >= 0x1p-80f);
    if (!ok) {
        sc.s[9] = inf;
        sc.s[10] = 0.0f;
        return;
    }
    const double u = std::fabs((double)step) * (std::ldexp(1.0, -119) / (double)eps + std::ldexp(1.0, -126));
    const double thr = u * std::ldexp(1.0, 26) * (1.0 + std::ldexp(1.0, -10));
    float t = (float)thr;
    if ((double)t < thr) t = std::nextafter(t, inf);
    sc.s[9] = t;
    float b = (float)((std::ldexp(1.0, 20) - (double)eps) / (double)ibc2 * (1.0 - std::ldexp(1.0, -20)));
    sc.s[10] = b < 65504.0f ? b : 65504.0f;
}

fo_status fo_adamw_step(const fo_tensor* t, int n_tensors, fo_format f, const fo_adamw_hparams* h,
                        void* stream)
{
    g_last_error.clear();
    fo_status st = check_format(f);
    if (st != FO_OK) return st;
    if (!h) return fail(FO_ERR_INVALID_ARG, "hyper-parameters are NULL");
    if (!is_finite(h->lr) || !is_finite(h->eps) || !is_finite(h->weight_decay))
        return fail(FO_ERR_INVALID_ARG, "lr / eps / weight_decay must be finite");
    if (!(h->beta1 >= 0.0 && h->beta1 < 1.0) || !(h->beta2 >= 0.0 && h->beta2 < 1.0))
        return fail(FO_ERR_INVALID_ARG, "betas must lie in [0, 1)");
    if (h->step < 1) return fail(FO_ERR_INVALID_ARG, "step must be >= 1");
    st = check_tensors(t, n_tensors, f, true);
    if (st != FO_OK) return st;
    if (n_tensors == 0) return FO_OK;
    // host scalars: binary64, each rounded once to binary32
    const double bc1 = 1.0 - std::pow(h->beta1, (double)h->step);
    const double bc2 = 1.0 - std::pow(h->beta2, (double)h->step);
    fo::Scalars sc;
    sc.s[0] = (float)h->beta1;
    sc.s[1] = (float)h->beta2;
    sc.s[2] = (float)(1.0 - h->beta1);
    sc.s[3] = (float)(1.0 - h->beta2);
    sc.s[4] = (float)(h->lr / bc1);
    sc.s[5] = (float)(1.0 / std::sqrt(bc2));
    sc.s[6] = (float)h->eps;
    sc.s[7] = (float)(1.0 - h->lr * h->weight_decay);
    adamw_fast_bounds(sc);
    fo::fill_pairs(sc, true);
    const StepLaunch L = pick_step<fo::kAdamW>(f);
    if (!L.k) return fail(FO_ERR_UNSUPPORTED, "format not provided");
    return launch_step(L, sc, t, n_tensors, (cudaStream_t)stream);
}

fo_status fo_sgdm_step(const fo_tensor* t, int n_tensors, fo_format f, const fo_sgdm_hparams* h,
                       void* stream)
{
    g_last_error.clear();
    fo_status st = check_format(f);
    if (st != FO_OK) return st;
    if (!h) return fail(FO_ERR_INVALID_ARG, "hyper-parameters are NULL");
    if (!is_finite(h->lr) || !is_finite(h->weight_decay))
        return fail(FO_ERR_INVALID_ARG, "lr / weight_decay must be finite");
    if (!(h->momentum >= 0.0 && h->momentum <= 1.0) || !(h->dampening >= 0.0 && h->dampening <= 1.0))
        return fail(FO_ERR_INVALID_ARG, "momentum / dampening must lie in [0, 1]");
    if (h->step < 1) return fail(FO_ERR_INVALID_ARG, "step must be >= 1");
    st = check_tensors(t, n_tensors, f, false);
    if (st != FO_OK) return st;
    if (n_tensors == 0) return FO_OK;
    fo::Scalars sc;
    sc.s[0] = (float)h->lr;
    sc.s[1] = (float)h->momentum;
    sc.s[2] = (float)(1.0 - h->dampening);
    sc.s[3] = (float)h->weight_decay;
    sc.s[4] = h->nesterov ? 1.0f : 0.0f;
    sc.s[5] = h->step == 1 ? 1.0f : 0.0f;
    sc.s[6] = 0.0f;
    sc.s[7] = 0.0f;
    fo::fill_pairs(sc, false);
    const StepLaunch L = pick_step<fo::kSGDM>(f);
    if (!L.k) return fail(FO_ERR_UNSUPPORTED, "format not provided");
    return launch_step(L, sc, t, n_tensors, (cudaStream_t)stream);
}

fo_status fo_stream_copy(const fo_tensor* t, int n_tensors, fo_format f, int adamw_mix, void* stream)
{
    g_last_error.clear();
    fo_status st = check_format(f);
    if (st != FO_OK) return st;
    st = check_tensors(t, n_tensors, f, adamw_mix != 0);
    if (st != FO_OK) return st;
    if (n_tensors == 0) return FO_OK;
    fo::Scalars sc = {};
    // the copy moves bytes only: the 16-bit formats do not matter, the ECC width does
    StepLaunch L;
    if (adamw_mix)
        L = f.ecc_bits == 8 ? step_launch<0, 0, 8, fo::kCopyAdamW>() : step_launch<0, 0, 16, fo::kCopyAdamW>();
    else
        L = f.ecc_bits == 8 ? step_launch<0, 0, 8, fo::kCopySGDM>() : step_launch<0, 0, 16, fo::kCopySGDM>();
    return launch_step(L, sc, t, n_tensors, (cudaStream_t)stream);
}

fo_status fo_encode_master(const float* x32, void* w, void* ecc, int64_t n, fo_format f, void* stream)
{
    g_last_error.clear();
    fo_status st = check_format(f);
    if (st != FO_OK) return st;
    if (n < 0) return fail(FO_ERR_INVALID_ARG, "n < 0");
    if (n == 0) return FO_OK;
    if (!x32 || !w || !ecc) return fail(FO_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned(x32, 4) || !aligned(w, 2) || (f.ecc_bits == 16 && !aligned(ecc, 2)))
        return fail(FO_ERR_ALIGNMENT, "misaligned array");
    int sms = 0;
    st = device_sms(&sms);
    if (st != FO_OK) return st;
    const unsigned grid = (unsigned)grid_for(n, sms);
    cudaStream_t s = (cudaStream_t)stream;
    const bool bf = f.w_dtype == FO_DT_BF16;
    if (f.ecc_bits == 8) {
        if (bf) fo::encode_master_kernel<0, 8><<<grid, fo::kThreads, 0, s>>>(x32, w, ecc, n);
        else fo::encode_master_kernel<1, 8><<<grid, fo::kThreads, 0, s>>>(x32, w, ecc, n);
    } else {
        if (bf) fo::encode_master_kernel<0, 16><<<grid, fo::kThreads, 0, s>>>(x32, w, ecc, n);
        else fo::encode_master_kernel<1, 16><<<grid, fo::kThreads, 0, s>>>(x32, w, ecc, n);
    }
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? FO_OK : cuda_fail(e, "encode kernel launch");
}

fo_status fo_decode_master(const void* w, const void* ecc, float* x32, int64_t n, fo_format f,
                           void* stream)
{
    g_last_error.clear();
    fo_status st = check_format(f);
    if (st != FO_OK) return st;
    if (n < 0) return fail(FO_ERR_INVALID_ARG, "n < 0");
    if (n == 0) return FO_OK;
    if (!x32 || !w || !ecc) return fail(FO_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned(x32, 4) || !aligned(w, 2) || (f.ecc_bits == 16 && !aligned(ecc, 2)))
        return fail(FO_ERR_ALIGNMENT, "misaligned array");
    int sms = 0;
    st = device_sms(&sms);
    if (st != FO_OK) return st;
    const unsigned grid = (unsigned)grid_for(n, sms);
    cudaStream_t s = (cudaStream_t)stream;
    const bool bf = f.w_dtype == FO_DT_BF16;
    if (f.ecc_bits == 8) {
        if (bf) fo::decode_master_kernel<0, 8><<<grid, fo::kThreads, 0, s>>>(w, ecc, x32, n);
        else fo::decode_master_kernel<1, 8><<<grid, fo::kThreads, 0, s>>>(w, ecc, x32, n);
    } else {
        if (bf) fo::decode_master_kernel<0, 16><<<grid, fo::kThreads, 0, s>>>(w, ecc, x32, n);
        else fo::decode_master_kernel<1, 16><<<grid, fo::kThreads, 0, s>>>(w, ecc, x32, n);
    }
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? FO_OK : cuda_fail(e, "decode kernel launch");
}

fo_status fo_check_errors(void* stream)
{
    g_last_error.clear();
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    unsigned int n = 0;
    e = cudaMemcpyFromSymbol(&n, fo::g_wait_timeouts, sizeof n);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyFromSymbol");
    if (n == 0) return FO_OK;
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(fo::g_wait_timeouts, &zero, sizeof zero);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyToSymbol");
    return fail(FO_ERR_TIMEOUT, std::to_string(n) + " warp(s) gave up waiting for a staged copy; their chunks were "
                                                    "not stepped");
}

const char* fo_status_string(fo_status s)
{
    switch (s) {
    case FO_OK: return "FO_OK";
    case FO_ERR_INVALID_ARG: return "FO_ERR_INVALID_ARG";
    case FO_ERR_UNSUPPORTED: return "FO_ERR_UNSUPPORTED";
    case FO_ERR_ALIGNMENT: return "FO_ERR_ALIGNMENT";
    case FO_ERR_TOO_MANY_TENSORS: return "FO_ERR_TOO_MANY_TENSORS";
    case FO_ERR_CUDA: return "FO_ERR_CUDA";
    case FO_ERR_TIMEOUT: return "FO_ERR_TIMEOUT";
    }
    return "unknown fo_status";
}

const char* fo_last_error(void) { return g_last_error.c_str(); }

int fo_version(void) { return 200; }

}  // extern "C"
