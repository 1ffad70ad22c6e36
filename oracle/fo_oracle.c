/*
 * fo_oracle.c - plain, slow, scalar CPU oracle for the FlashOptim-style
 * compressed optimizer step.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file: only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark use it.  It shares no code, header, table or constant
 * generator with the CUDA library; the two are independent restatements of
 * the same definitions.
 *
 * Sources (web pages on FlashOptim):
 *   [BLOG] "FlashOptim: Breaking the Memory Wall with 24-bit Weights and
 *          Companded States" (wispaper blog), sections "1. ULP-based Weight
 *          Splitting", "2. Companded Quantization", "The Problem".
 *   [THREAD] Davis Blalock's release thread for FlashOptim: the posts on
 *          weight splitting into a B-bit downcast plus a (32-B)-bit ECC, on
 *          the fixed f32 interval that rounds to a downcast value, on
 *          integer-quantizing the position inside that interval, on 24-bit
 *          masters (16-bit downcast + 8-bit ECC), on 8-bit states with one
 *          16-bit scale per 32 elements, on companding (different functions
 *          for momentum-like and variance-like states), and on keeping
 *          gradients in backward precision.
 *
 * Precision.  The pages fix the master weight as a 32-bit float split into
 * a 16-bit downcast and an ECC; every quantity that decides an emitted code
 * (the optimizer update, the companders) is therefore computed in IEEE
 * binary32 with one rounding per operation, exactly as written below, and
 * fma only where written.  Interval arithmetic of the weight codec is done
 * in binary64, where every step is exact.  Compile with
 * -ffp-contract=off -fno-fast-math; MXCSR is forced to round-to-nearest,
 * no flush-to-zero, no denormals-are-zero inside every entry point.
 *
 * Readings where the pages are silent (each is listed with its reason in
 * the design notes of the repository):
 *   R1 downcast = IEEE round-to-nearest-even, overflow to inf, subnormals kept.
 *   R2 the ECC is a signed code centred on the downcast value x':
 *      rho = round_half_even((x - x') / (u / 2^N)), clamped to
 *      +-(2^(N-1)-1); u is the spacing of the downcast format on the side
 *      of x' that x lies on (half the spacing inward at a power of two).
 *   R3 decode is x' + rho * u / 2^N, rounded once to binary32.
 *   R4 groups of 32 consecutive elements per tensor, last group partial.
 *   R5 the 16-bit scale is an fp16 of max|z| rounded toward +inf, saturated
 *      at 65504; for the variance state z = sqrt(v) (scale in the sqrt
 *      domain).
 *   R6 momentum compander phi(y) = 2y / (1 + |y|) (twice the textbook
 *      softsign) applied to y = m * (1/S); int8 code round(127 * phi).
 *   R7 variance compander: uint8 code round(255 * sqrt(v) / S).
 *   R8 AdamW as in torch.optim.AdamW (decoupled decay, eps outside the
 *      root, bias correction), on the decoded f32 state; SGD-momentum as in
 *      torch.optim.SGD (coupled decay, dampening, optional Nesterov,
 *      first step copies the gradient into the buffer).
 *   R9 non-finite values: a NaN downcasts to the positive quiet NaN of the
 *      format (bf16 0x7FC0, fp16 0x7E00) whatever its sign and payload, with
 *      ECC 0 (as every non-finite x'); inf and NaN state values are left out
 *      of the group maximum and get code 0; everything else follows IEEE
 *      binary32 arithmetic (an inf gradient gives m' = inf, v' = inf and, in
 *      AdamW, the quotient inf/inf = NaN).
 *
 * Parity pins (tests/test_oracle_*.py): the downcast against numpy and torch
 * casts over all 2^32 binary32 patterns; the ECC against closed integer
 * forms and brute-force nearest-code search; the companders against
 * torch's softsign / numpy sqrt in binary64 and exhaustive code-grid
 * invertibility; the update against torch.optim.AdamW / torch.optim.SGD in
 * binary64.  The exact compander constants, the fp16 round-up of scales and
 * the binary32 operation order are fixed by this file alone; the pages do
 * not print them (parity unpinned by the pages for those three choices,
 * pinned only by invariants).
 */
#define _GNU_SOURCE
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <pthread.h>
#include <xmmintrin.h>

/* ------------------------------------------------------------------ */
/* floating formats                                                    */
/* ------------------------------------------------------------------ */

typedef struct {
    int p;      /* significand precision in bits, hidden bit included */
    int emin;   /* exponent of the smallest normal */
    int emax;   /* exponent of the largest finite */
    int ebits;  /* exponent field width */
    int bias;
} fmt_t;

static const fmt_t F_BF16 = {8, -126, 127, 8, 127};
static const fmt_t F_FP16 = {11, -14, 15, 5, 15};

static fmt_t fmt_of(int dtype) { return dtype == 0 ? F_BF16 : F_FP16; }

static uint16_t fmt_inf_bits(fmt_t f) { return (uint16_t)(((1u << f.ebits) - 1u) << (f.p - 1)); }

static uint16_t fmt_qnan_bits(fmt_t f)
{
    return (uint16_t)(fmt_inf_bits(f) | (1u << (f.p - 2)));
}

/* exact value of a 16-bit pattern */
static double fmt_value(fmt_t f, uint16_t bits)
{
    int neg = bits >> 15;
    unsigned ef = (bits >> (f.p - 1)) & ((1u << f.ebits) - 1u);
    unsigned mant = bits & ((1u << (f.p - 1)) - 1u);
    double v;
    if (ef == (1u << f.ebits) - 1u)
        v = mant ? NAN : INFINITY;
    else if (ef == 0)
        v = ldexp((double)mant, f.emin - (f.p - 1));
    else
        v = ldexp((double)(mant | (1u << (f.p - 1))), (int)ef - f.bias - (f.p - 1));
    return neg ? -v : v;
}

/* floor(log2 a) for finite a > 0 */
static int ilog2_of(double a)
{
    int e;
    frexp(a, &e);
    return e - 1;
}

/* pattern of an exactly representable, finite, positive value r */
static uint16_t fmt_pattern_exact(fmt_t f, double r)
{
    if (r < ldexp(1.0, f.emin))
        return (uint16_t)(r / ldexp(1.0, f.emin - (f.p - 1)));
    int E = ilog2_of(r);
    double m = r / ldexp(1.0, E - (f.p - 1)) - ldexp(1.0, f.p - 1);
    return (uint16_t)(((unsigned)(E + f.bias) << (f.p - 1)) | (unsigned)m);
}

/* R1: round-to-nearest-even downcast of a binary32 value.  R9: every NaN,
   whatever its sign and payload, becomes the one positive quiet NaN of the
   format (only the quiet bit set): a NaN carries no sign or payload that
   binary32 arithmetic on different machines would agree on. */
static uint16_t fmt_round_rne(fmt_t f, float xf)
{
    double x = xf;
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    if (isnan(x)) return fmt_qnan_bits(f);
    double a = fabs(x);
    if (isinf(a)) return (uint16_t)(sign | fmt_inf_bits(f));
    if (a == 0.0) return sign;
    int E = ilog2_of(a);
    if (E < f.emin) E = f.emin;
    double ulp = ldexp(1.0, E - (f.p - 1));
    double k = floor(a / ulp);           /* exact: power-of-two scaling */
    double rem = a - k * ulp;            /* exact */
    double half = ulp / 2;
    if (rem > half || (rem == half && fmod(k, 2.0) == 1.0)) k += 1.0;
    double r = k * ulp;
    if (r >= ldexp(1.0, f.emax + 1)) return (uint16_t)(sign | fmt_inf_bits(f));
    return (uint16_t)(sign | fmt_pattern_exact(f, r));
}

/* R5: fp16 pattern of a >= 0 rounded toward +inf, saturated at 65504 */
static uint16_t fp16_round_up_sat(float af)
{
    const fmt_t f = F_FP16;
    double a = af;
    if (!(a <= 65504.0)) return 0x7BFF;   /* also catches NaN and inf */
    if (a <= 0.0) return 0;               /* a is a max of absolute values */
    int E = ilog2_of(a);
    if (E < f.emin) E = f.emin;
    double ulp = ldexp(1.0, E - (f.p - 1));
    double k = ceil(a / ulp);
    double r = k * ulp;
    if (r > 65504.0) return 0x7BFF;
    return fmt_pattern_exact(f, r);
}

/* ------------------------------------------------------------------ */
/* ULP-normalised error-correction code (weight splitting)              */
/* [BLOG] section 1 "ULP-based Weight Splitting"; [THREAD] posts on the */
/* interval of f32 values rounding to x' and on quantizing the position */
/* inside it.                                                           */
/* ------------------------------------------------------------------ */

typedef struct {
    double a;      /* |x'| */
    double s;      /* sign of x' as +-1 */
    double u_out;  /* spacing of the downcast grid away from zero at x' */
    double u_in;   /* spacing toward zero (half at a power of two above emin) */
} interval_t;

static interval_t interval_of(fmt_t f, double xp)
{
    interval_t iv;
    iv.a = fabs(xp);
    iv.s = signbit(xp) ? -1.0 : 1.0;
    int E = f.emin;
    int pow2 = 0;
    if (iv.a > 0.0) {
        E = ilog2_of(iv.a);
        pow2 = (iv.a == ldexp(1.0, E));
        if (E < f.emin) E = f.emin;
    }
    iv.u_out = ldexp(1.0, E - (f.p - 1));
    iv.u_in = (pow2 && E > f.emin) ? iv.u_out / 2 : iv.u_out;
    return iv;
}

/* R2: code of x (binary32) relative to its downcast pattern xp_bits */
static int32_t ecc_encode(fmt_t f, int nbits, float x, uint16_t xp_bits)
{
    double xp = fmt_value(f, xp_bits);
    if (!isfinite(xp) || isnan((double)x)) return 0;
    interval_t iv = interval_of(f, xp);
    double e = iv.s * ((double)x - xp);          /* exact in binary64 */
    double u = (e >= 0.0) ? iv.u_out : iv.u_in;
    double t = ldexp(e, nbits) / u;              /* exact */
    double r = nearbyint(t);                     /* ties to even */
    double lim = ldexp(1.0, nbits - 1) - 1.0;
    if (r > lim) r = lim;
    if (r < -lim) r = -lim;
    return (int32_t)r;
}

/* R3: reconstruct the binary32 master */
static float ecc_decode(fmt_t f, int nbits, uint16_t xp_bits, int32_t rho)
{
    double xp = fmt_value(f, xp_bits);
    if (rho == 0 || !isfinite(xp)) return (float)xp;
    interval_t iv = interval_of(f, xp);
    double u = (rho > 0) ? iv.u_out : iv.u_in;
    double off = ldexp((double)rho * u, -nbits);  /* exact */
    return (float)(iv.s * (iv.a + off));          /* one rounding */
}

/* ------------------------------------------------------------------ */
/* companded 8-bit states, one fp16 scale per group of 32               */
/* [BLOG] section 2 "Companded Quantization"; [THREAD] posts on 8-bit   */
/* linear quantization with a 16-bit scale per 32 elements and on       */
/* companding.                                                          */
/* ------------------------------------------------------------------ */

#define GROUP 32

/* R9: a non-finite state value (inf or NaN) has no place on a scaled 8-bit
   grid; it is left out of its group's maximum and stored as code 0, so that
   one overflowed element does not flatten the codes of the other 31. */
static int finite_f(float z) { return isfinite(z) != 0; }

static float group_absmax(const float* z, int n)
{
    float A = 0.0f;
    for (int i = 0; i < n; i++)
        if (finite_f(z[i])) A = fmaxf(A, fabsf(z[i]));
    return A;
}

/* R6: momentum, signed int8 */
static void m_encode_group(const float* z, int n, int8_t* q, uint16_t* S_bits)
{
    uint16_t S = fp16_round_up_sat(group_absmax(z, n));
    *S_bits = S;
    float Sf = (float)fmt_value(F_FP16, S);
    if (Sf == 0.0f) {
        for (int i = 0; i < n; i++) q[i] = 0;
        return;
    }
    float r = 1.0f / Sf;
    for (int i = 0; i < n; i++) {
        if (!finite_f(z[i])) {
            q[i] = 0;
            continue;
        }
        float y = z[i] * r;
        float num = 2.0f * y;
        float den = 1.0f + fabsf(y);
        float c = num / den;
        float t = 127.0f * c;
        float k = nearbyintf(t);
        if (isnan(k)) k = 0.0f;
        if (k > 127.0f) k = 127.0f;
        if (k < -127.0f) k = -127.0f;
        q[i] = (int8_t)k;
    }
}

static float m_decode(int8_t q, uint16_t S_bits)
{
    float Sf = (float)fmt_value(F_FP16, S_bits);
    float c = (float)q / 127.0f;
    float y = c / (2.0f - fabsf(c));
    return y * Sf;
}

/* R7: variance, unsigned uint8 code of sqrt(v) */
static void v_encode_group(const float* sv, int n, uint8_t* q, uint16_t* S_bits)
{
    uint16_t S = fp16_round_up_sat(group_absmax(sv, n));
    *S_bits = S;
    float Sf = (float)fmt_value(F_FP16, S);
    if (Sf == 0.0f) {
        for (int i = 0; i < n; i++) q[i] = 0;
        return;
    }
    float k = 255.0f / Sf;
    for (int i = 0; i < n; i++) {
        if (!finite_f(sv[i])) {
            q[i] = 0;
            continue;
        }
        float t = sv[i] * k;
        float c = nearbyintf(t);
        if (isnan(c) || c < 0.0f) c = 0.0f;
        if (c > 255.0f) c = 255.0f;
        q[i] = (uint8_t)c;
    }
}

static float v_decode_sqrt(uint8_t q, uint16_t S_bits)
{
    float Sf = (float)fmt_value(F_FP16, S_bits);
    float u = (float)q / 255.0f;
    return u * Sf;
}

static float v_decode(uint8_t q, uint16_t S_bits)
{
    float sv = v_decode_sqrt(q, S_bits);
    return sv * sv;
}

/* ------------------------------------------------------------------ */
/* host scalars                                                         */
/* ------------------------------------------------------------------ */

typedef struct {
    float b1, b2, omb1, omb2, step, ibc2, eps, decay;
} adamw_sc_t;

static adamw_sc_t adamw_scalars(double lr, double beta1, double beta2, double eps,
                                double wd, int64_t t)
{
    adamw_sc_t s;
    double bc1 = 1.0 - pow(beta1, (double)t);
    double bc2 = 1.0 - pow(beta2, (double)t);
    s.b1 = (float)beta1;
    s.b2 = (float)beta2;
    s.omb1 = (float)(1.0 - beta1);
    s.omb2 = (float)(1.0 - beta2);
    s.step = (float)(lr / bc1);
    s.ibc2 = (float)(1.0 / sqrt(bc2));
    s.eps = (float)eps;
    s.decay = (float)(1.0 - lr * wd);
    return s;
}

/* ------------------------------------------------------------------ */
/* elementwise stream access                                            */
/* ------------------------------------------------------------------ */

static int32_t ecc_load(const void* ecc, int nbits, int64_t i)
{
    return nbits == 8 ? (int32_t)((const int8_t*)ecc)[i] : (int32_t)((const int16_t*)ecc)[i];
}

static void ecc_store(void* ecc, int nbits, int64_t i, int32_t v)
{
    if (nbits == 8)
        ((int8_t*)ecc)[i] = (int8_t)v;
    else
        ((int16_t*)ecc)[i] = (int16_t)v;
}

/* ------------------------------------------------------------------ */
/* one optimizer step over one tensor                                   */
/* ------------------------------------------------------------------ */

typedef struct {
    uint16_t* w;
    void* ecc;
    const uint16_t* grad;
    int8_t* mq;
    uint16_t* ms;
    uint8_t* vq;
    uint16_t* vs;
    int64_t n;
    int wdt, gdt, nbits;
    int kind;            /* 0 AdamW, 1 SGD-momentum */
    adamw_sc_t a;
    float lr, mu, omd, wd;
    int nesterov, first;
    int64_t g0, g1;      /* group range for this worker */
} step_job_t;

/* R8, AdamW: decode -> update -> re-encode one group */
static void adamw_group(const step_job_t* J, int64_t g)
{
    fmt_t fw = fmt_of(J->wdt), fg = fmt_of(J->gdt);
    int64_t b = g * GROUP;
    int n = (int)((J->n - b) < GROUP ? (J->n - b) : GROUP);
    float x2[GROUP], m1[GROUP], sv[GROUP];
    const adamw_sc_t* s = &J->a;
    for (int i = 0; i < n; i++) {
        int64_t k = b + i;
        float x = ecc_decode(fw, J->nbits, J->w[k], ecc_load(J->ecc, J->nbits, k));
        float m = m_decode(J->mq[k], J->ms[g]);
        float v = v_decode(J->vq[k], J->vs[g]);
        float gr = (float)fmt_value(fg, J->grad[k]);
        float mn = fmaf(s->b1, m, s->omb1 * gr);
        float vn = fmaf(s->b2, v, s->omb2 * (gr * gr));
        float r = sqrtf(vn);
        float den = fmaf(r, s->ibc2, s->eps);
        float x1 = x * s->decay;
        x2[i] = fmaf(-s->step, mn / den, x1);
        m1[i] = mn;
        sv[i] = r;
    }
    m_encode_group(m1, n, J->mq + b, J->ms + g);
    v_encode_group(sv, n, J->vq + b, J->vs + g);
    for (int i = 0; i < n; i++) {
        uint16_t xp = fmt_round_rne(fw, x2[i]);
        J->w[b + i] = xp;
        ecc_store(J->ecc, J->nbits, b + i, ecc_encode(fw, J->nbits, x2[i], xp));
    }
}

/* R8, SGD with momentum */
static void sgdm_group(const step_job_t* J, int64_t g)
{
    fmt_t fw = fmt_of(J->wdt), fg = fmt_of(J->gdt);
    int64_t b = g * GROUP;
    int n = (int)((J->n - b) < GROUP ? (J->n - b) : GROUP);
    float x2[GROUP], b1[GROUP];
    for (int i = 0; i < n; i++) {
        int64_t k = b + i;
        float x = ecc_decode(fw, J->nbits, J->w[k], ecc_load(J->ecc, J->nbits, k));
        float gr = (float)fmt_value(fg, J->grad[k]);
        float g1 = fmaf(J->wd, x, gr);
        float buf;
        if (J->first) {
            buf = g1;
        } else {
            float m = m_decode(J->mq[k], J->ms[g]);
            buf = fmaf(J->mu, m, J->omd * g1);
        }
        float d = J->nesterov ? fmaf(J->mu, buf, g1) : buf;
        x2[i] = fmaf(-J->lr, d, x);
        b1[i] = buf;
    }
    m_encode_group(b1, n, J->mq + b, J->ms + g);
    for (int i = 0; i < n; i++) {
        uint16_t xp = fmt_round_rne(fw, x2[i]);
        J->w[b + i] = xp;
        ecc_store(J->ecc, J->nbits, b + i, ecc_encode(fw, J->nbits, x2[i], xp));
    }
}

static void fpenv_enter(unsigned* saved)
{
    *saved = _mm_getcsr();
    /* round to nearest, all exceptions masked, FTZ and DAZ off */
    _mm_setcsr(0x1F80);
}

static void fpenv_leave(unsigned saved) { _mm_setcsr(saved); }

static void* step_worker(void* arg)
{
    step_job_t* J = (step_job_t*)arg;
    unsigned csr;
    fpenv_enter(&csr);
    for (int64_t g = J->g0; g < J->g1; g++) {
        if (J->kind == 0)
            adamw_group(J, g);
        else
            sgdm_group(J, g);
    }
    fpenv_leave(csr);
    return NULL;
}

static int run_groups(step_job_t* proto, int nthreads)
{
    int64_t ng = (proto->n + GROUP - 1) / GROUP;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (ng < nthreads) nthreads = ng > 0 ? (int)ng : 1;
    step_job_t jobs[256];
    pthread_t th[256];
    for (int t = 0; t < nthreads; t++) {
        jobs[t] = *proto;
        jobs[t].g0 = ng * t / nthreads;
        jobs[t].g1 = ng * (t + 1) / nthreads;
    }
    if (nthreads == 1) {
        step_worker(&jobs[0]);
        return 0;
    }
    for (int t = 0; t < nthreads; t++)
        if (pthread_create(&th[t], NULL, step_worker, &jobs[t]) != 0) return -1;
    for (int t = 0; t < nthreads; t++) pthread_join(th[t], NULL);
    return 0;
}

static int check_format(int wdt, int gdt, int nbits)
{
    if ((wdt != 0 && wdt != 1) || (gdt != 0 && gdt != 1)) return -1;
    if (nbits != 8 && nbits != 16) return -1;
    return 0;
}

/* ------------------------------------------------------------------ */
/* exported entry points (ctypes)                                      */
/* dtype: 0 = bf16, 1 = fp16.  ecc arrays are int8 (N=8) or int16.      */
/* ------------------------------------------------------------------ */

int oracle_adamw_step(uint16_t* w, void* ecc, const uint16_t* grad, int8_t* mq, uint16_t* ms,
                      uint8_t* vq, uint16_t* vs, int64_t n, int wdt, int gdt, int nbits,
                      double lr, double beta1, double beta2, double eps, double wd, int64_t t,
                      int nthreads)
{
    if (check_format(wdt, gdt, nbits) || n < 0 || t < 1) return -1;
    step_job_t J;
    memset(&J, 0, sizeof J);
    J.w = w; J.ecc = ecc; J.grad = grad; J.mq = mq; J.ms = ms; J.vq = vq; J.vs = vs;
    J.n = n; J.wdt = wdt; J.gdt = gdt; J.nbits = nbits; J.kind = 0;
    J.a = adamw_scalars(lr, beta1, beta2, eps, wd, t);
    return run_groups(&J, nthreads);
}

int oracle_sgdm_step(uint16_t* w, void* ecc, const uint16_t* grad, int8_t* mq, uint16_t* ms,
                     int64_t n, int wdt, int gdt, int nbits, double lr, double momentum,
                     double dampening, double wd, int nesterov, int64_t t, int nthreads)
{
    if (check_format(wdt, gdt, nbits) || n < 0 || t < 1) return -1;
    step_job_t J;
    memset(&J, 0, sizeof J);
    J.w = w; J.ecc = ecc; J.grad = grad; J.mq = mq; J.ms = ms;
    J.n = n; J.wdt = wdt; J.gdt = gdt; J.nbits = nbits; J.kind = 1;
    J.lr = (float)lr;
    J.mu = (float)momentum;
    J.omd = (float)(1.0 - dampening);
    J.wd = (float)wd;
    J.nesterov = nesterov != 0;
    J.first = (t == 1);
    return run_groups(&J, nthreads);
}

/* ---- codec-level entry points used by the pin tests ---- */

typedef struct {
    int op;  /* 0 encode master, 1 decode master, 2 downcast only */
    const float* x;
    uint16_t* w;
    void* ecc;
    float* out;
    int64_t i0, i1;
    int wdt, nbits;
} codec_job_t;

static void* codec_worker(void* arg)
{
    codec_job_t* J = (codec_job_t*)arg;
    fmt_t f = fmt_of(J->wdt);
    unsigned csr;
    fpenv_enter(&csr);
    for (int64_t i = J->i0; i < J->i1; i++) {
        if (J->op == 0) {
            uint16_t xp = fmt_round_rne(f, J->x[i]);
            J->w[i] = xp;
            ecc_store(J->ecc, J->nbits, i, ecc_encode(f, J->nbits, J->x[i], xp));
        } else if (J->op == 1) {
            J->out[i] = ecc_decode(f, J->nbits, J->w[i], ecc_load(J->ecc, J->nbits, i));
        } else {
            J->w[i] = fmt_round_rne(f, J->x[i]);
        }
    }
    fpenv_leave(csr);
    return NULL;
}

static int run_codec(codec_job_t* proto, int64_t n, int nthreads)
{
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    codec_job_t jobs[256];
    pthread_t th[256];
    for (int t = 0; t < nthreads; t++) {
        jobs[t] = *proto;
        jobs[t].i0 = n * t / nthreads;
        jobs[t].i1 = n * (t + 1) / nthreads;
    }
    if (nthreads == 1) {
        codec_worker(&jobs[0]);
        return 0;
    }
    for (int t = 0; t < nthreads; t++)
        if (pthread_create(&th[t], NULL, codec_worker, &jobs[t]) != 0) return -1;
    for (int t = 0; t < nthreads; t++) pthread_join(th[t], NULL);
    return 0;
}

int oracle_encode_master(const float* x, uint16_t* w, void* ecc, int64_t n, int wdt, int nbits,
                         int nthreads)
{
    if (check_format(wdt, 0, nbits) || n < 0) return -1;
    codec_job_t J = {0, x, w, ecc, NULL, 0, 0, wdt, nbits};
    return run_codec(&J, n, nthreads);
}

int oracle_decode_master(const uint16_t* w, const void* ecc, float* x, int64_t n, int wdt,
                         int nbits, int nthreads)
{
    if (check_format(wdt, 0, nbits) || n < 0) return -1;
    codec_job_t J = {1, NULL, (uint16_t*)w, (void*)ecc, x, 0, 0, wdt, nbits};
    return run_codec(&J, n, nthreads);
}

int oracle_downcast(const float* x, uint16_t* w, int64_t n, int wdt, int nthreads)
{
    if (check_format(wdt, 0, 8) || n < 0) return -1;
    codec_job_t J = {2, x, w, NULL, NULL, 0, 0, wdt, 8};
    return run_codec(&J, n, nthreads);
}

/* widen 16-bit patterns to binary32 (exact) */
int oracle_widen(const uint16_t* w, float* x, int64_t n, int wdt)
{
    if (check_format(wdt, 0, 8) || n < 0) return -1;
    fmt_t f = fmt_of(wdt);
    for (int64_t i = 0; i < n; i++) x[i] = (float)fmt_value(f, w[i]);
    return 0;
}

/* fp16 round-up of non-negative magnitudes (the scale rule) */
int oracle_scale_fp16(const float* a, uint16_t* s, int64_t n)
{
    unsigned csr;
    fpenv_enter(&csr);
    for (int64_t i = 0; i < n; i++) s[i] = fp16_round_up_sat(a[i]);
    fpenv_leave(csr);
    return 0;
}

/* quantize groups of 32 of z into codes + scales; kind 0 momentum
   (int8 codes), kind 1 variance (input is sqrt(v), uint8 codes) */
int oracle_quantize_state(const float* z, void* q, uint16_t* s, int64_t n, int kind)
{
    if (n < 0 || (kind != 0 && kind != 1)) return -1;
    unsigned csr;
    fpenv_enter(&csr);
    for (int64_t b = 0, g = 0; b < n; b += GROUP, g++) {
        int m = (int)((n - b) < GROUP ? (n - b) : GROUP);
        if (kind == 0)
            m_encode_group(z + b, m, (int8_t*)q + b, s + g);
        else
            v_encode_group(z + b, m, (uint8_t*)q + b, s + g);
    }
    fpenv_leave(csr);
    return 0;
}

/* dequantize: kind 0 momentum m, kind 1 variance v, kind 2 sqrt(v) */
int oracle_dequantize_state(const void* q, const uint16_t* s, float* z, int64_t n, int kind)
{
    if (n < 0 || kind < 0 || kind > 2) return -1;
    unsigned csr;
    fpenv_enter(&csr);
    for (int64_t i = 0; i < n; i++) {
        int64_t g = i / GROUP;
        if (kind == 0)
            z[i] = m_decode(((const int8_t*)q)[i], s[g]);
        else if (kind == 1)
            z[i] = v_decode(((const uint8_t*)q)[i], s[g]);
        else
            z[i] = v_decode_sqrt(((const uint8_t*)q)[i], s[g]);
    }
    fpenv_leave(csr);
    return 0;
}

/* quantize against a given (stored) scale, for the code-grid tests */
int oracle_quantize_fixed_scale(const float* z, void* q, uint16_t S, int64_t n, int kind)
{
    if (n < 0 || (kind != 0 && kind != 1)) return -1;
    unsigned csr;
    fpenv_enter(&csr);
    float Sf = (float)fmt_value(F_FP16, S);
    for (int64_t i = 0; i < n; i++) {
        float k;
        if (Sf == 0.0f || !finite_f(z[i])) {
            k = 0.0f;
        } else if (kind == 0) {
            float r = 1.0f / Sf;
            float y = z[i] * r;
            float c = (2.0f * y) / (1.0f + fabsf(y));
            k = nearbyintf(127.0f * c);
            if (isnan(k)) k = 0.0f;
            if (k > 127.0f) k = 127.0f;
            if (k < -127.0f) k = -127.0f;
        } else {
            float kk = 255.0f / Sf;
            k = nearbyintf(z[i] * kk);
            if (isnan(k) || k < 0.0f) k = 0.0f;
            if (k > 255.0f) k = 255.0f;
        }
        if (kind == 0)
            ((int8_t*)q)[i] = (int8_t)k;
        else
            ((uint8_t*)q)[i] = (uint8_t)k;
    }
    fpenv_leave(csr);
    return 0;
}

/* the f32 host scalars of one AdamW step, for inspection by tests */
int oracle_adamw_scalars(double lr, double beta1, double beta2, double eps, double wd,
                         int64_t t, float* out8)
{
    adamw_sc_t s = adamw_scalars(lr, beta1, beta2, eps, wd, t);
    out8[0] = s.b1; out8[1] = s.b2; out8[2] = s.omb1; out8[3] = s.omb2;
    out8[4] = s.step; out8[5] = s.ibc2; out8[6] = s.eps; out8[7] = s.decay;
    return 0;
}
