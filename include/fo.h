/*
 * fo.h - C ABI of libfo: the FlashOptim-style fused optimizer step on
 * NVIDIA B200 (sm_100a).
 *
 * Method (web pages on FlashOptim):
 *   "FlashOptim: Breaking the Memory Wall with 24-bit Weights and Companded
 *   States" (wispaper blog), sections "1. ULP-based Weight Splitting" and
 *   "2. Companded Quantization"; Davis Blalock's FlashOptim release thread,
 *   posts on weight splitting, on the f32 interval that rounds to a downcast
 *   value, on 8-bit states with a 16-bit scale per 32 elements, on
 *   companding, and on gradients kept in backward precision.
 *
 * Storage formats (all little-endian, caller-owned device memory):
 *   w        numel 16-bit downcast weights x' (bf16 or fp16), round to
 *            nearest even of the f32 master.
 *   ecc      numel signed codes rho of ecc_bits (8 -> int8, 16 -> int16):
 *            rho = round_half_even((x - x') / (u / 2^N)), clamped to
 *            +-(2^(N-1) - 1); u is the spacing of the 16-bit format at x' on
 *            the side of x' where x lies (toward zero at a power of two the
 *            spacing halves).  The master is reconstructed as
 *            x = x' + rho * u / 2^N (one binary32 rounding).
 *   m_q      numel int8 momentum codes, companded: code = round(127 * phi(y)),
 *            phi(y) = 2y / (1 + |y|), y = m * (1 / S_m).
 *   m_scale  ceil(numel / 32) fp16 bit patterns S_m, one per group of 32
 *            consecutive elements counted from element 0 of the tensor:
 *            max |m| of the group rounded toward +inf to fp16, saturated at
 *            65504.
 *   v_q      numel uint8 variance codes: code = round(255 * sqrt(v) / S_v).
 *   v_scale  ceil(numel / 32) fp16 patterns S_v: max sqrt(v) of the group
 *            rounded toward +inf, saturated at 65504.
 *   grad     numel 16-bit gradients (bf16 or fp16), read only; gradients stay
 *            in backward precision.
 *
 * Non-finite values (the pages are silent; a fixed reading): a NaN master
 * is stored as the positive quiet NaN of its format (bf16 0x7FC0, fp16
 * 0x7E00) with code 0, an inf master as inf with code 0; inf and NaN values
 * of m' or sqrt(v') are left out of their group's maximum and stored as code
 * 0; all other arithmetic is IEEE binary32 (an inf gradient makes the AdamW
 * update inf / inf = NaN).
 *
 * Conventions for every call:
 *   - Memory: the caller owns every buffer; the library allocates nothing and
 *     keeps no state between calls other than per-device launch constants
 *     (SM count), found on the first call on a device, and a device word that
 *     counts bounded waits that gave up (read and cleared by fo_check_errors).
 *   - Asynchrony: work is enqueued on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream) and the call returns without waiting.  The
 *     descriptor array and hyper-parameter structs are copied into the launch
 *     before the call returns, so the caller may reuse them at once.  The
 *     grad buffer must stay valid until the work on `stream` has finished.
 *   - Validation happens on the host before any launch: a non-FO_OK status
 *     means nothing was enqueued and no buffer was touched
 *     (FO_ERR_CUDA from a later launch of a multi-launch call is the one
 *     exception: earlier launches of that call may have been enqueued).
 *     fo_last_error() then gives a one-line, thread-local explanation.
 *   - Kernel faults are asynchronous and surface at the caller's next
 *     synchronisation with the stream.
 *   - Alignment: 16-bit arrays need 2-byte alignment, int16 ECC arrays too.
 *     Any other alignment and any numel up to FO_MAX_NUMEL are accepted:
 *     tensors whose arrays are all 16-byte aligned take the vectorised path,
 *     others a scalar path inside the same kernel, with identical results.
 *   - numel == 0 tensors are skipped; n_tensors == 0 is a no-op.
 *   - Results do not depend on the number of tensors per call, their order,
 *     or on whether they are stepped in one call or one call per tensor.
 *   - Launch geometry (performance only, results identical): chunks of 1024
 *     elements for AdamW and 512 for SGD-momentum, staged in shared memory by
 *     bulk copies, one warp per chunk; the elements of a tensor's
 *     last chunk beyond its whole 512-element slices, and tensors whose
 *     arrays are not 16-byte aligned (or whose weights / 16-bit ECC codes are
 *     not 32-byte aligned), take a scalar path.
 *   - Waits inside the kernels are bounded in time; fo_check_errors reports
 *     a wait that gave up.
 */
#ifndef FO_H
#define FO_H

#include <stdint.h>

#if defined(__GNUC__)
#define FO_API __attribute__((visibility("default")))
#else
#define FO_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FO_OK = 0,
    FO_ERR_INVALID_ARG = 1,      /* null pointer, negative size, bad hyper-parameter */
    FO_ERR_UNSUPPORTED = 2,      /* dtype / ecc_bits combination not provided */
    FO_ERR_ALIGNMENT = 3,        /* a 16-bit array not 2-byte aligned */
    FO_ERR_TOO_MANY_TENSORS = 4, /* n_tensors above FO_MAX_TENSORS_PER_CALL */
    FO_ERR_CUDA = 5,             /* a CUDA runtime call or launch failed */
    FO_ERR_TIMEOUT = 6           /* a kernel gave up a bounded wait (fo_check_errors) */
} fo_status;

typedef enum { FO_DT_BF16 = 0, FO_DT_FP16 = 1 } fo_dtype;

/* Largest n_tensors accepted by one call.  Calls with more tensors than fit
   one launch's parameter block are split into several launches. */
#define FO_MAX_TENSORS_PER_CALL (1 << 20)

/* Largest numel of one tensor (2^36 elements, far beyond what one GPU's
   memory holds; larger ones are rejected with FO_ERR_INVALID_ARG). */
#define FO_MAX_NUMEL ((int64_t)1 << 36)

/* One parameter tensor.  All pointers are device memory owned by the caller.
   Optimizer fields that a call does not use may be NULL (v_q / v_scale for
   SGD-momentum). */
typedef struct {
    void* w;             /* numel 16-bit downcast weights, updated in place         */
    void* ecc;           /* numel codes of ecc_bits bits, updated in place          */
    const void* grad;    /* numel 16-bit gradients, read only                       */
    int8_t* m_q;         /* numel int8 momentum codes, updated in place             */
    uint16_t* m_scale;   /* ceil(numel/32) fp16 momentum scales, updated in place   */
    uint8_t* v_q;        /* numel uint8 variance codes (AdamW), updated in place    */
    uint16_t* v_scale;   /* ceil(numel/32) fp16 variance scales (AdamW)             */
    int64_t numel;       /* >= 0                                                     */
} fo_tensor;

/* AdamW as in torch.optim.AdamW: decoupled weight decay, bias correction,
   eps added outside the square root.  step is the 1-based count t of this
   update (the state holds t-1 previous updates). */
typedef struct {
    double lr, beta1, beta2, eps, weight_decay;
    int64_t step;
} fo_adamw_hparams;

/* SGD with momentum as in torch.optim.SGD: coupled weight decay
   (g += weight_decay * x), buf = momentum * buf + (1 - dampening) * g, and on
   step == 1 buf = g; Nesterov uses g + momentum * buf as the direction. */
typedef struct {
    double lr, momentum, dampening, weight_decay;
    int nesterov;
    int64_t step;
} fo_sgdm_hparams;

typedef struct {
    fo_dtype w_dtype;     /* downcast format of the weights */
    fo_dtype grad_dtype;  /* format of the gradients */
    int ecc_bits;         /* 8 (24-bit masters) or 16 (32-bit masters) */
} fo_format;

/*
 * fo_adamw_step - one fused AdamW step over n_tensors tensors.
 * Passage: "FlashOptim: Breaking the Memory Wall with 24-bit Weights and
 * Companded States" (wispaper blog), "Methodology" sections 1 (ULP-based
 * weight splitting) and 2 (companded quantization) and "Performance" (one
 * fused step); Davis Blalock's release thread, posts on the weight split,
 * on 8-bit states with a 16-bit scale per 32 elements, on companding and on
 * gradients kept in backward precision.
 * Per element: reconstruct x from (w, ecc); dequantize m and v with the
 * group scales; m' = b1*m + (1-b1)*g, v' = b2*v + (1-b2)*g^2 in binary32;
 * x'' = x*(1 - lr*wd) - lr/(1-b1^t) * m' / (sqrt(v')/sqrt(1-b2^t) + eps);
 * write back the downcast + ECC of x'' and the companded codes of m', sqrt(v')
 * with fresh per-group scales.  Supported formats: w bf16 or fp16, grad bf16
 * or fp16, ecc_bits 8 or 16.
 * Errors: FO_ERR_INVALID_ARG (t NULL with n_tensors > 0, h NULL, any
 * required pointer NULL for numel > 0, numel < 0, step < 1, lr / betas / eps
 * not finite, beta outside [0, 1)), FO_ERR_UNSUPPORTED, FO_ERR_ALIGNMENT,
 * FO_ERR_TOO_MANY_TENSORS, FO_ERR_CUDA.
 */
FO_API fo_status fo_adamw_step(const fo_tensor* t, int n_tensors, fo_format f,
                        const fo_adamw_hparams* h, void* stream);

/*
 * fo_sgdm_step - one fused SGD-momentum step over n_tensors tensors (uses the
 * momentum codes and scales only; v_q / v_scale are ignored).  Same format
 * support and error behaviour as fo_adamw_step; momentum and dampening must
 * lie in [0, 1].
 * Passage: Davis Blalock's release thread, the post listing the optimizers
 * the method wraps (Adam, SGD, ...), with the same weight split and momentum
 * compander as fo_adamw_step.
 */
FO_API fo_status fo_sgdm_step(const fo_tensor* t, int n_tensors, fo_format f,
                       const fo_sgdm_hparams* h, void* stream);

/*
 * fo_stream_copy - the byte traffic of one step without its arithmetic: reads
 * every array fo_adamw_step (adamw_mix != 0) or fo_sgdm_step (adamw_mix == 0)
 * reads and writes the same bytes back unchanged, through the same staging,
 * work split and stores.  A measurement aid, not part of the method (the
 * FlashOptim pages have no counterpart): its bandwidth is the practical
 * ceiling for the step on the same tensors.  Arguments, validation and errors
 * as fo_adamw_step / fo_sgdm_step; the 16-bit formats in f are not used, the
 * ECC width is.  Concurrent calls or steps on the same tensors race.
 * Passage: none (a measurement aid, not part of the method).
 */
FO_API fo_status fo_stream_copy(const fo_tensor* t, int n_tensors, fo_format f, int adamw_mix,
                        void* stream);

/*
 * fo_encode_master - split n binary32 masters x32 (device) into the 16-bit
 * downcast w (round to nearest even) and the ECC codes ecc (device).
 * Used to wrap existing f32 weights and to import checkpoints.
 * Errors: FO_ERR_INVALID_ARG (NULL pointer with n > 0, n < 0),
 * FO_ERR_UNSUPPORTED, FO_ERR_ALIGNMENT (x32 not 4-byte aligned, w or int16
 * ecc not 2-byte aligned), FO_ERR_CUDA.
 * Passage: the wispaper blog's "1. ULP-based Weight Splitting"; the release
 * thread's posts on the f32 interval that rounds to one downcast value and on
 * integer-quantizing the position inside it.
 */
FO_API fo_status fo_encode_master(const float* x32, void* w, void* ecc, int64_t n, fo_format f,
                           void* stream);

/*
 * fo_decode_master - reconstruct n binary32 masters x32 (device) from w and
 * ecc (device).  Used to export checkpoints.  Same errors as
 * fo_encode_master.  Non-finite x' decode to x' itself.
 * Passage: as fo_encode_master (the inverse of the split).
 */
FO_API fo_status fo_decode_master(const void* w, const void* ecc, float* x32, int64_t n, fo_format f,
                           void* stream);

/*
 * fo_check_errors - wait for the work on `stream` (a cudaStream_t), then
 * report whether any step kernel on the current device gave up a bounded
 * wait for one of its staged copies since the last check.  Such a kernel
 * leaves the chunks of the warp that gave up unstepped (their bytes are
 * unspecified); this never happens on a healthy device.  Returns FO_OK, or
 * FO_ERR_TIMEOUT (and clears the device's count), or FO_ERR_CUDA.
 * Passage: none (error reporting).
 */
FO_API fo_status fo_check_errors(void* stream);

/* Static English name of a status code.  Passage: none (error reporting). */
FO_API const char* fo_status_string(fo_status s);

/* Detail of the last non-FO_OK status returned on the calling thread
   ("" if none).  The pointer stays valid until the next call on the thread.
   Passage: none (error reporting). */
FO_API const char* fo_last_error(void);

/* Library version as major * 10000 + minor * 100 + patch.  Passage: none. */
FO_API int fo_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FO_H */
