/*
 * opt2s oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, single-threaded CPU restatement of the 32-bit two-state
 * optimizer update (Adam/AdamW and AdEMAMix), used to check the CUDA path.
 * Only the test suite, the smoke check of the entry module and the CPU
 * baseline / reference legs of the benchmark may load it.  The product path
 * never calls it, and it shares no code, header, table or constant with the
 * CUDA library: every function below is written out here from the published
 * definitions.
 *
 * Sources of what it computes:
 *   [issue]    bitsandbytes issue "Investigate a 256-thread SM103 path for
 *              small 32-bit optimizer tensors":
 *                section "Problem"            -- the two-state 32-bit update,
 *                                                32-bit (fp32) state;
 *                section "Scope"              -- decoupled weight decay is
 *                                                applied before the Adam /
 *                                                AdEMAMix update;
 *                section "Correctness oracle" -- variants ADAM/AdamW and
 *                                                ADEMAMIX, FP16/BF16/FP32
 *                                                param+grad storage, weight
 *                                                decay and skip_zeros flags,
 *                                                gradient left unchanged.
 *   [Adam]     Kingma & Ba, "Adam: A Method for Stochastic Optimization",
 *              ICLR 2015, Algorithm 1 (moments, bias correction, eps outside
 *              the square root).
 *   [AdamW]    Loshchilov & Hutter, "Decoupled Weight Decay Regularization",
 *              ICLR 2019, Algorithm 2 (p <- p - lr*wd*p, decoupled from the
 *              gradient moments).
 *   [AdEMAMix] Pagliardini, Ablin & Grangier, "The AdEMAMix Optimizer:
 *              Better, Faster, Older", 2024, Algorithm 1 (a second, slow EMA
 *              m2 with rate beta3, not bias-corrected, mixed in with weight
 *              alpha).
 *   [LAMB]     You et al., "Large Batch Optimization for Deep Learning:
 *              Training BERT in 76 minutes", ICLR 2020, Algorithm 2 (per-layer
 *              trust ratio ||x|| / ||r + lambda x||).
 *   [8bit]     Dettmers, Lewis, Shleifer & Zettlemoyer, "8-bit Optimizers via
 *              Block-wise Quantization", ICLR 2022, sections 2.1 (block-wise
 *              absmax quantization, B = 2048), 2.2 (dynamic tree
 *              quantization) and 2.3 (dynamic quantization of the unsigned
 *              second state).  [issue] "Problem": tensors below
 *              min_8bit_size = 4096 elements keep the 32-bit state.
 *   [IEEE754]  IEEE 754-2008, section 4.3.1 (roundTiesToEven) and 3.6
 *              (binary16 format); bfloat16 is the upper half of binary32.
 *
 * Readings where the sources leave a step open (each one is also listed in
 * the design notes of the repository):
 *   - fp32 arithmetic, every operation rounded to fp32 in the order written
 *     below, with no fused multiply-add (built with -ffp-contract=off) and no
 *     flush-to-zero (the MXCSR FTZ/DAZ bits are cleared for the call).
 *   - bias corrections bc1 = 1 - beta1^t, bc2 = 1 - beta2^t and the decay
 *     factor 1 - lr*wd are evaluated in double and rounded to fp32 once.
 *   - skip_zeros: an element whose gradient compares equal to zero (+0 or -0)
 *     is left wholly unchanged: param, all moments, and no weight decay.
 *   - AdEMAMix state1 holds [m1(0..n) | m2(0..n)], 2*n floats.
 *   - fp16/bf16 params are widened exactly and narrowed with
 *     round-to-nearest-even; state is always fp32.
 *   - max_unorm > 0 (oracle_step_f32_max_unorm): the tensor's update norm is
 *     bounded by max_unorm times its weight norm, as written out above that
 *     function; the pages name the option without its arithmetic.
 *   - LAMB (oracle_step_f32_lamb): You et al. 2020, Algorithm 2, per tensor,
 *     with the readings written out above that function.
 *   - 8-bit blockwise state (oracle_step_8bit): [8bit], with the map and
 *     quantization readings written out above oracle_quant_map.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <xmmintrin.h>

#define OR_ADAM 0
#define OR_ADEMAMIX 1
#define OR_F32 0
#define OR_F16 1
#define OR_BF16 2

/* ------------------------------------------------------------------------ */
/* Storage conversions, written from the format definitions [IEEE754].       */
/* ------------------------------------------------------------------------ */

/* Split a finite, nonzero |x| (as binary32 bits without sign) into an exact
 * integer significand M and exponent k with |x| = M * 2^k. */
static void split_f32(uint32_t mag, uint64_t *M, int *k)
{
    uint32_t e = mag >> 23, f = mag & 0x7fffffu;
    if (e == 0) { *M = f; *k = -149; }                  /* subnormal */
    else        { *M = f | 0x800000u; *k = (int)e - 150; }
}

static int bit_length(uint64_t v)
{
    int n = 0;
    while (v) { n++; v >>= 1; }
    return n;
}

/* Round |x| = M*2^k to the nearest multiple of 2^Q, ties to an even multiple.
 * Returns the multiple count. */
static uint64_t round_to_quantum(uint64_t M, int k, int Q)
{
    int s = Q - k;
    if (s <= 0) return M << (-s);                       /* already exact */
    if (s >= 64) return 0;                              /* far below half a quantum */
    uint64_t count = M >> s;
    uint64_t rem = M & ((1ull << s) - 1);
    uint64_t half = 1ull << (s - 1);
    if (rem > half || (rem == half && (count & 1))) count++;
    return count;
}

/* Narrow binary32 -> a smaller binary format with `fbits` fraction bits,
 * exponent bias `bias`, round-to-nearest-even.  In that format a finite value
 * is count * 2^Q with Q = max(floor(log2|x|) - fbits, 1 - bias - fbits), and
 * its bit pattern (sign aside) is (Q - Qmin) * 2^fbits + count; the same
 * formula covers subnormals, normals, the carry into the next binade, and the
 * carry into the infinity pattern. */
static uint32_t narrow_rne(float x, int fbits, int bias, uint32_t inf_bits,
                           uint32_t qnan_bits, int total_bits)
{
    uint32_t u;
    memcpy(&u, &x, sizeof u);
    uint32_t sign = (u >> 31) << (total_bits - 1);
    uint32_t mag = u & 0x7fffffffu;
    if (mag > 0x7f800000u) return sign | qnan_bits;     /* NaN */
    if (mag == 0x7f800000u) return sign | inf_bits;     /* infinity */
    if (mag == 0) return sign;                          /* signed zero */
    uint64_t M;
    int k;
    split_f32(mag, &M, &k);
    int log2x = k + bit_length(M) - 1;                  /* floor(log2|x|) */
    int Qmin = 1 - bias - fbits;
    int Q = log2x - fbits;
    if (Q < Qmin) Q = Qmin;
    uint64_t count = round_to_quantum(M, k, Q);
    uint64_t bits = (uint64_t)(Q - Qmin) * (1ull << fbits) + count;
    if (bits >= inf_bits) return sign | inf_bits;       /* overflow */
    return sign | (uint32_t)bits;
}

uint16_t oracle_f32_to_f16(float x)
{
    return (uint16_t)narrow_rne(x, 10, 15, 0x7c00u, 0x7e00u, 16);
}

uint16_t oracle_f32_to_bf16(float x)
{
    return (uint16_t)narrow_rne(x, 7, 127, 0x7f80u, 0x7fc0u, 16);
}

float oracle_f16_to_f32(uint16_t h)
{
    int sign = h >> 15, e = (h >> 10) & 0x1f, f = h & 0x3ff;
    double mag;
    if (e == 0x1f) mag = f ? NAN : INFINITY;
    else if (e == 0) mag = ldexp((double)f, -24);       /* subnormal: f * 2^-24 */
    else mag = ldexp((double)(1024 + f), e - 25);       /* (1.f) * 2^(e-15) */
    return (float)(sign ? -mag : mag);                  /* exact in binary32 */
}

float oracle_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;                     /* bf16 = top half of binary32 */
    float x;
    memcpy(&x, &u, sizeof x);
    return x;
}

static float load_param(const void *p, int dtype, int64_t i)
{
    if (dtype == OR_F32) return ((const float *)p)[i];
    if (dtype == OR_F16) return oracle_f16_to_f32(((const uint16_t *)p)[i]);
    return oracle_bf16_to_f32(((const uint16_t *)p)[i]);
}

static void store_param(void *p, int dtype, int64_t i, float x)
{
    if (dtype == OR_F32) ((float *)p)[i] = x;
    else if (dtype == OR_F16) ((uint16_t *)p)[i] = oracle_f32_to_f16(x);
    else ((uint16_t *)p)[i] = oracle_f32_to_bf16(x);
}

/* ------------------------------------------------------------------------ */
/* Per-step scalars.                                                          */
/* ------------------------------------------------------------------------ */

/* 1 - beta^t in double, rounded to fp32 once. [Adam] Algorithm 1. */
float oracle_bias_correction(float beta, int t)
{
    return (float)(1.0 - pow((double)beta, (double)t));
}

/* 1 - lr*wd in double, rounded to fp32 once. [AdamW] Algorithm 2. */
float oracle_decay_factor(float lr, float wd)
{
    return (float)(1.0 - (double)lr * (double)wd);
}

/* ------------------------------------------------------------------------ */
/* The fp32 step.                                                            */
/* ------------------------------------------------------------------------ */

/*
 * One optimizer step, in place, over one tensor of n elements.
 *
 * algo      0 = Adam (AdamW when wd != 0), 1 = AdEMAMix.
 * dtype     storage of param and grad: 0 fp32, 1 fp16, 2 bf16.
 * state1    Adam: m (n floats).  AdEMAMix: [m1 | m2] (2n floats).
 * state2    v (n floats).
 * step      t >= 1, the 1-based index of this update.
 *
 * Per element, every operation rounded to fp32 in this order:
 *   m   = beta1*m + (1-beta1)*g                           [Adam]
 *   v   = beta2*v + ((1-beta2)*g)*g                       [Adam]
 *   num = m / bc1                                         [Adam]
 *   AdEMAMix only:
 *     m2  = beta3*m2 + (1-beta3)*g                        [AdEMAMix]
 *     num = num + alpha*m2                                [AdEMAMix]
 *   den = sqrt(v / bc2) + eps                             [Adam]
 *   p   = p*decay - lr*(num/den)       decay first, [AdamW]; [issue] "Scope"
 * Returns 0, or -1 on an argument the definitions do not cover.
 */
/* The new moments of one element and its update direction u = num/den
 * (m2 is read and written only for AdEMAMix). */
static void element_direction(int algo, float g, float m, float m2, float v,
                              float beta1, float beta2, float beta3, float alpha,
                              float eps, float bc1, float bc2, float one_minus_b1,
                              float one_minus_b2, float one_minus_b3,
                              float *mi, float *m2i, float *vi, float *u)
{
    *mi = beta1 * m + one_minus_b1 * g;
    *vi = beta2 * v + (one_minus_b2 * g) * g;
    float num = *mi / bc1;
    *m2i = m2;
    if (algo == OR_ADEMAMIX) {
        *m2i = beta3 * m2 + one_minus_b3 * g;
        num = num + alpha * *m2i;
    }
    float den = sqrtf(*vi / bc2) + eps;
    *u = num / den;
}

/* The per-element update of one step (shared by both fp32 step entries). */
static void update_element(int algo, float g, float *p, float *m, float *m2, float *v,
                           float lr, float beta1, float beta2, float beta3, float alpha,
                           float eps, float bc1, float bc2, float decay,
                           float one_minus_b1, float one_minus_b2, float one_minus_b3)
{
    float mi, m2i, vi, u;
    element_direction(algo, g, *m, algo == OR_ADEMAMIX ? *m2 : 0.0f, *v, beta1, beta2,
                      beta3, alpha, eps, bc1, bc2, one_minus_b1, one_minus_b2,
                      one_minus_b3, &mi, &m2i, &vi, &u);
    *p = *p * decay - lr * u;
    *m = mi;
    *v = vi;
    if (algo == OR_ADEMAMIX) *m2 = m2i;
}

/* One step over n elements whose gradient is read by get_grad(grad, i). */
static int step_core(int algo, int dtype, int skip_zeros, float lr, float beta1,
                     float beta2, float beta3, float alpha, float eps,
                     float weight_decay, int step, void *param, const void *grad,
                     float (*get_grad)(const void *, int, int64_t), int grad_dtype,
                     float *state1, float *state2, int64_t n)
{
    if (step < 1 || n < 0) return -1;
    if (algo != OR_ADAM && algo != OR_ADEMAMIX) return -1;
    if (dtype != OR_F32 && dtype != OR_F16 && dtype != OR_BF16) return -1;

    unsigned int csr = _mm_getcsr();
    _mm_setcsr(csr & ~(0x8000u | 0x0040u));             /* FTZ and DAZ off */

    const float bc1 = oracle_bias_correction(beta1, step);
    const float bc2 = oracle_bias_correction(beta2, step);
    const float decay = oracle_decay_factor(lr, weight_decay);
    const float one_minus_b1 = 1.0f - beta1;
    const float one_minus_b2 = 1.0f - beta2;
    const float one_minus_b3 = 1.0f - beta3;

    float *m = state1;
    float *m2 = state1 + n;                             /* AdEMAMix only */
    float *v = state2;

    for (int64_t i = 0; i < n; i++) {
        float g = get_grad(grad, grad_dtype, i);
        if (skip_zeros && g == 0.0f) continue;
        float p = load_param(param, dtype, i);
        update_element(algo, g, &p, &m[i], &m2[i], &v[i], lr, beta1, beta2, beta3,
                       alpha, eps, bc1, bc2, decay, one_minus_b1, one_minus_b2,
                       one_minus_b3);
        store_param(param, dtype, i, p);
    }

    _mm_setcsr(csr);
    return 0;
}

static float grad_in_storage(const void *grad, int dtype, int64_t i)
{
    return load_param(grad, dtype, i);
}

static float grad_in_f32(const void *grad, int dtype, int64_t i)
{
    (void)dtype;
    return ((const float *)grad)[i];
}

/*
 * One optimizer step, in place, over one tensor of n elements.
 *
 * algo      0 = Adam (AdamW when wd != 0), 1 = AdEMAMix.
 * dtype     storage of param and grad: 0 fp32, 1 fp16, 2 bf16.
 * state1    Adam: m (n floats).  AdEMAMix: [m1 | m2] (2n floats).
 * state2    v (n floats).
 * step      t >= 1, the 1-based index of this update.
 *
 * Per element, every operation rounded to fp32 in this order:
 *   m   = beta1*m + (1-beta1)*g                           [Adam]
 *   v   = beta2*v + ((1-beta2)*g)*g                       [Adam]
 *   num = m / bc1                                         [Adam]
 *   AdEMAMix only:
 *     m2  = beta3*m2 + (1-beta3)*g                        [AdEMAMix]
 *     num = num + alpha*m2                                [AdEMAMix]
 *   den = sqrt(v / bc2) + eps                             [Adam]
 *   p   = p*decay - lr*(num/den)       decay first, [AdamW]; [issue] "Scope"
 * Returns 0, or -1 on an argument the definitions do not cover.
 */
int oracle_step_f32(int algo, int dtype, int skip_zeros,
                    float lr, float beta1, float beta2, float beta3,
                    float alpha, float eps, float weight_decay, int step,
                    void *param, const void *grad, float *state1,
                    float *state2, int64_t n)
{
    return step_core(algo, dtype, skip_zeros, lr, beta1, beta2, beta3, alpha, eps,
                     weight_decay, step, param, grad, grad_in_storage, dtype, state1,
                     state2, n);
}

/* The same step with a gradient already in fp32 (whatever the param
 * storage), e.g. the data-parallel average below. */
int oracle_step_f32_fgrad(int algo, int dtype, int skip_zeros,
                          float lr, float beta1, float beta2, float beta3,
                          float alpha, float eps, float weight_decay, int step,
                          void *param, const float *grad, float *state1,
                          float *state2, int64_t n)
{
    return step_core(algo, dtype, skip_zeros, lr, beta1, beta2, beta3, alpha, eps,
                     weight_decay, step, param, grad, grad_in_f32, OR_F32, state1,
                     state2, n);
}

/*
 * The step with the update norm of the tensor clipped: max_unorm > 0.
 *
 * [issue] "Scope" keeps the existing kernel for "max-unorm/LAMB use" and
 * section "Correctness oracle" runs "max_unorm > 0" controls, so max_unorm
 * is an option of this same two-state update, but the pages never write out
 * its arithmetic.  Reading used here (the plainest one the name supports:
 * max_unorm bounds the norm of the update relative to the norm of the
 * weights, the tensor being the unit):
 *   u_i = num_i / den_i, the update direction of element i exactly as in the
 *         plain step (fp32); u_i = 0 for an element skip_zeros leaves alone;
 *   U   = sqrt(sum_i u_i^2) and P = sqrt(sum_i p_i^2) over the tensor, p the
 *         stored param before the step; squares, sums and roots in binary64,
 *         summed in index order;
 *   s   = max_unorm*P/U if U > max_unorm*P, else 1 (binary64, then rounded
 *         to fp32 once);
 *   p_i = p_i*decay - lr*(s*u_i) in fp32, with m, v (and m2) exactly as in
 *         the plain step.  s = 1 gives the plain step's bits.
 * The tensor is read twice: once for U and P, once for the update.
 * Returns 0, or -1 on an argument the definitions do not cover.
 */
int oracle_step_f32_max_unorm(int algo, int dtype, int skip_zeros,
                              float lr, float beta1, float beta2, float beta3,
                              float alpha, float eps, float weight_decay,
                              float max_unorm, int step, void *param,
                              const void *grad, float *state1, float *state2,
                              int64_t n, float *scale_out)
{
    if (step < 1 || n < 0 || !(max_unorm > 0.0f)) return -1;
    if (algo != OR_ADAM && algo != OR_ADEMAMIX) return -1;
    if (dtype != OR_F32 && dtype != OR_F16 && dtype != OR_BF16) return -1;

    unsigned int csr = _mm_getcsr();
    _mm_setcsr(csr & ~(0x8000u | 0x0040u));             /* FTZ and DAZ off */

    const float bc1 = oracle_bias_correction(beta1, step);
    const float bc2 = oracle_bias_correction(beta2, step);
    const float decay = oracle_decay_factor(lr, weight_decay);
    const float one_minus_b1 = 1.0f - beta1;
    const float one_minus_b2 = 1.0f - beta2;
    const float one_minus_b3 = 1.0f - beta3;
    float *m = state1;
    float *m2 = state1 + n;                             /* AdEMAMix only */
    float *v = state2;

    /* pass 1: the norms of the update and of the weights */
    double su = 0.0, sp = 0.0;
    for (int64_t i = 0; i < n; i++) {
        float p = load_param(param, dtype, i);
        sp += (double)p * (double)p;
        float g = load_param(grad, dtype, i);
        if (skip_zeros && g == 0.0f) continue;
        float mi, m2i, vi, u;
        element_direction(algo, g, m[i], algo == OR_ADEMAMIX ? m2[i] : 0.0f, v[i], beta1,
                          beta2, beta3, alpha, eps, bc1, bc2, one_minus_b1, one_minus_b2,
                          one_minus_b3, &mi, &m2i, &vi, &u);
        su += (double)u * (double)u;
    }
    const double U = sqrt(su), P = sqrt(sp);
    const double limit = (double)max_unorm * P;
    const float scale = (float)(U > limit ? limit / U : 1.0);
    if (scale_out) *scale_out = scale;

    /* pass 2: the update, scaled */
    for (int64_t i = 0; i < n; i++) {
        float g = load_param(grad, dtype, i);
        if (skip_zeros && g == 0.0f) continue;
        float p = load_param(param, dtype, i);
        float mi, m2i, vi, u;
        element_direction(algo, g, m[i], algo == OR_ADEMAMIX ? m2[i] : 0.0f, v[i], beta1,
                          beta2, beta3, alpha, eps, bc1, bc2, one_minus_b1, one_minus_b2,
                          one_minus_b3, &mi, &m2i, &vi, &u);
        p = p * decay - lr * (scale * u);
        store_param(param, dtype, i, p);
        m[i] = mi;
        v[i] = vi;
        if (algo == OR_ADEMAMIX) m2[i] = m2i;
    }

    _mm_setcsr(csr);
    return 0;
}

/*
 * LAMB: the layer-wise adaptive step of You et al., "Large Batch Optimization
 * for Deep Learning: Training BERT in 76 minutes", ICLR 2020, Algorithm 2,
 * over one tensor (the "layer").  [issue] "Scope" keeps the two-state kernel
 * "for max-unorm/LAMB use"; the pages do not write LAMB out, so the paper's
 * Algorithm 2 is followed, with these readings:
 *   u_i = num_i / den_i, the bias-corrected Adam direction of element i
 *         exactly as in the plain fp32 step (Algorithm 2's r_t);
 *   w_i = u_i + wd*p_i in fp32 (the weight decay lambda sits inside the
 *         trust ratio, as in Algorithm 2, not the decay-first AdamW form);
 *   W   = sqrt(sum_i w_i^2), P = sqrt(sum_i p_i^2) over the tensor, p the
 *         stored param before the step, squares, sums and roots in binary64,
 *         summed in index order;
 *   r   = P/W rounded to fp32 once, if P > 0 and W > 0, else 1: the scaling
 *         function phi is the identity (the paper's experiments), and a zero
 *         norm (a zero-initialised tensor, or no update) takes ratio 1 so
 *         that such a tensor still moves (the paper leaves 0/x and x/0 open);
 *   p_i = p_i - lr*(r*w_i) in fp32; m and v exactly as in the plain step.
 * skip_zeros: an element whose gradient is zero keeps p, m and v; its p_i
 * counts in P and it adds nothing to W.  Adam moments only (algo 0).
 * Returns 0, or -1 on an argument the definitions do not cover.
 */
int oracle_step_f32_lamb(int dtype, int skip_zeros, float lr, float beta1,
                         float beta2, float eps, float weight_decay, int step,
                         void *param, const void *grad, float *state1,
                         float *state2, int64_t n, float *ratio_out)
{
    if (step < 1 || n < 0) return -1;
    if (dtype != OR_F32 && dtype != OR_F16 && dtype != OR_BF16) return -1;

    unsigned int csr = _mm_getcsr();
    _mm_setcsr(csr & ~(0x8000u | 0x0040u));             /* FTZ and DAZ off */

    const float bc1 = oracle_bias_correction(beta1, step);
    const float bc2 = oracle_bias_correction(beta2, step);
    const float one_minus_b1 = 1.0f - beta1;
    const float one_minus_b2 = 1.0f - beta2;
    float *m = state1;
    float *v = state2;

    /* pass 1: the norms of the weights and of the decayed direction */
    double sw = 0.0, sp = 0.0;
    for (int64_t i = 0; i < n; i++) {
        float p = load_param(param, dtype, i);
        sp += (double)p * (double)p;
        float g = load_param(grad, dtype, i);
        if (skip_zeros && g == 0.0f) continue;
        float mi, m2i, vi, u;
        element_direction(OR_ADAM, g, m[i], 0.0f, v[i], beta1, beta2, 0.0f, 0.0f, eps,
                          bc1, bc2, one_minus_b1, one_minus_b2, 0.0f, &mi, &m2i, &vi, &u);
        float w = u + weight_decay * p;
        sw += (double)w * (double)w;
    }
    const double W = sqrt(sw), P = sqrt(sp);
    const float ratio = (P > 0.0 && W > 0.0) ? (float)(P / W) : 1.0f;
    if (ratio_out) *ratio_out = ratio;

    /* pass 2: the update along w, scaled by the trust ratio */
    for (int64_t i = 0; i < n; i++) {
        float g = load_param(grad, dtype, i);
        if (skip_zeros && g == 0.0f) continue;
        float p = load_param(param, dtype, i);
        float mi, m2i, vi, u;
        element_direction(OR_ADAM, g, m[i], 0.0f, v[i], beta1, beta2, 0.0f, 0.0f, eps,
                          bc1, bc2, one_minus_b1, one_minus_b2, 0.0f, &mi, &m2i, &vi, &u);
        float w = u + weight_decay * p;
        p = p - lr * (ratio * w);
        store_param(param, dtype, i, p);
        m[i] = mi;
        v[i] = vi;
    }

    _mm_setcsr(csr);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* 8-bit blockwise state [8bit].                                              */
/* ------------------------------------------------------------------------ */

#define OR_BLOCK8 2048                                  /* [8bit] 2.1: block size B */

/*
 * The quantization maps of [8bit]: the 256 values a state code stands for,
 * in ascending order, so that code c means the c-th smallest value.
 *
 * [8bit] 2.2 (dynamic tree quantization, for the signed first moments): a
 * code is a sign bit, then E zero bits (the value's decimal exponent,
 * 10^-E), then an indicator bit 1, then F = 6 - E bits f of a linear fraction
 * in [0.1, 1].  [8bit] 2.3 (dynamic quantization, for the non-negative
 * second moment): the sign bit becomes one more fraction bit, F = 7 - E.
 * E runs over 0..6 in both (the 7 decades down to 10^-7 the paper gives).
 * Readings where the paper leaves the detail open:
 *   - the F fraction bits split [0.1, 1] into 2^F equal bins and f stands
 *     for the midpoint of bin f: value = 10^-E * (0.1 + 0.9*(2f+1)/2^(F+1)),
 *     which is N/D with N = 2^(F+1) + 9*(2f+1) and D = 10^(E+1) * 2^(F+1),
 *     both exact binary32 integers, so one IEEE division rounds it once;
 *   - the bits with no indicator (all zeros after the sign, or all zeros in
 *     the unsigned code's first seven bits) give two patterns: one is 0, the
 *     other stands for 1.0, so that the element a block is normalised by
 *     (x = 1 after the division by the block's absmax) is stored exactly.
 * Returns 0.
 */
static int cmp_float_asc(const void *a, const void *b)
{
    float x = *(const float *)a, y = *(const float *)b;
    return (x > y) - (x < y);
}

int oracle_quant_map(int is_signed, float *map)
{
    int k = 0;
    const int f0 = is_signed ? 6 : 7;                   /* fraction bits at E = 0 */
    for (int E = 0; E <= 6; E++) {
        const int F = f0 - E;
        float D = (float)(1 << (F + 1));
        for (int e = 0; e <= E; e++) D *= 10.0f;       /* exact: 10^(E+1) 2^(F+1) < 2^31 */
        for (int f = 0; f < (1 << F); f++) {
            const float N = (float)((1 << (F + 1)) + 9 * (2 * f + 1));
            const float value = N / D;
            map[k++] = value;
            if (is_signed) map[k++] = -value;
        }
    }
    map[k++] = 0.0f;
    map[k++] = 1.0f;
    qsort(map, (size_t)k, sizeof(float), cmp_float_asc);
    return k == 256 ? 0 : -1;
}

/* [8bit] 2.1: the code of the map value nearest to x; the distances are
 * compared exactly (x and the map are binary32, whose differences binary64
 * holds exactly wherever two candidates are close), and an exact tie goes to
 * the lower code.  A NaN x gets code 0. */
int oracle_quantize(const float *map, float x)
{
    int best = 0;
    double bd = fabs((double)x - (double)map[0]);
    for (int j = 1; j < 256; j++) {
        double d = fabs((double)x - (double)map[j]);
        if (d < bd) { bd = d; best = j; }
    }
    return best;
}

static int zero_code(const float *map)
{
    for (int j = 0; j < 256; j++)
        if (map[j] == 0.0f) return j;
    return 0;
}

/* One block of one state quantity: values x[0..len) (fp32) -> codes and the
 * block's absmax.  [8bit] 2.1: N = max |x_i|, code_i = nearest(x_i / N) with
 * the division rounded to fp32; a block whose absmax is 0 stores the code of
 * 0 everywhere.  NaNs do not raise the absmax. */
static void quantize_block(const float *map, const float *x, int64_t len, uint8_t *codes,
                           float *absmax)
{
    float amax = 0.0f;
    for (int64_t i = 0; i < len; i++) {
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    const int zc = zero_code(map);
    for (int64_t i = 0; i < len; i++)
        codes[i] = (uint8_t)(amax > 0.0f ? oracle_quantize(map, x[i] / amax) : zc);
    *absmax = amax;
}

/*
 * One optimizer step over one tensor whose state is stored in 8 bits, block
 * by block ([8bit] section 2: dequantize the state of a block to fp32,
 * update, quantize the new state back with the block's new absmax).
 *
 * q1        Adam: codes of m (n bytes).  AdEMAMix: [m1 codes | m2 codes] (2n).
 * absmax1   Adam: absmax of m per block (ceil(n/2048) floats).  AdEMAMix:
 *           [m1 absmaxes | m2 absmaxes] (2*ceil(n/2048)).
 * q2        codes of v (n bytes); absmax2: absmax of v per block.
 * m and m2 use the signed map, v the unsigned one.  A block is elements
 * [2048k, 2048(k+1)) of the tensor.  State starting at zero: every absmax 0
 * (codes then do not matter).
 *
 * Per element: m = map_s[q1]*absmax (fp32 product), likewise v and m2; the
 * update is the plain fp32 step's (the same order, decay first), on these
 * values; p is stored as in the plain step.  With skip_zeros, an element
 * whose gradient is zero keeps p and its dequantized m, v (m2), which are
 * then quantized with the block's new absmax like the others.
 * Returns 0, or -1 on an argument the definitions do not cover.
 */
int oracle_step_8bit(int algo, int dtype, int skip_zeros, float lr, float beta1,
                     float beta2, float beta3, float alpha, float eps, float weight_decay,
                     int step, void *param, const void *grad, uint8_t *q1, uint8_t *q2,
                     float *absmax1, float *absmax2, int64_t n)
{
    if (step < 1 || n < 0) return -1;
    if (algo != OR_ADAM && algo != OR_ADEMAMIX) return -1;
    if (dtype != OR_F32 && dtype != OR_F16 && dtype != OR_BF16) return -1;

    unsigned int csr = _mm_getcsr();
    _mm_setcsr(csr & ~(0x8000u | 0x0040u));             /* FTZ and DAZ off */

    float smap[256], umap[256];
    oracle_quant_map(1, smap);
    oracle_quant_map(0, umap);
    const float bc1 = oracle_bias_correction(beta1, step);
    const float bc2 = oracle_bias_correction(beta2, step);
    const float decay = oracle_decay_factor(lr, weight_decay);
    const float one_minus_b1 = 1.0f - beta1;
    const float one_minus_b2 = 1.0f - beta2;
    const float one_minus_b3 = 1.0f - beta3;
    const int64_t nblocks = (n + OR_BLOCK8 - 1) / OR_BLOCK8;

    float m[OR_BLOCK8], v[OR_BLOCK8], m2[OR_BLOCK8];
    for (int64_t b = 0; b < nblocks; b++) {
        const int64_t lo = b * OR_BLOCK8;
        const int64_t len = (n - lo < OR_BLOCK8) ? n - lo : OR_BLOCK8;
        for (int64_t k = 0; k < len; k++) {
            const int64_t i = lo + k;
            m[k] = smap[q1[i]] * absmax1[b];
            v[k] = umap[q2[i]] * absmax2[b];
            m2[k] = algo == OR_ADEMAMIX ? smap[q1[n + i]] * absmax1[nblocks + b] : 0.0f;
            float g = load_param(grad, dtype, i);
            if (skip_zeros && g == 0.0f) continue;
            float p = load_param(param, dtype, i);
            update_element(algo, g, &p, &m[k], &m2[k], &v[k], lr, beta1, beta2, beta3, alpha,
                           eps, bc1, bc2, decay, one_minus_b1, one_minus_b2, one_minus_b3);
            store_param(param, dtype, i, p);
        }
        quantize_block(smap, m, len, q1 + lo, &absmax1[b]);
        quantize_block(umap, v, len, q2 + lo, &absmax2[b]);
        if (algo == OR_ADEMAMIX)
            quantize_block(smap, m2, len, q1 + n + lo, &absmax1[nblocks + b]);
    }

    _mm_setcsr(csr);
    return 0;
}

/*
 * Data-parallel gradient: the mean of `world` ranks' gradients (storage
 * dtype), widened exactly, summed in fp32 in rank order 0, 1, ..., world-1
 * (each addition rounded), then divided by world (rounded).  This is the
 * gradient the sharded step applies: the reduce-scatter of a ZeRO-style
 * data-parallel optimizer, with the order fixed so every run gives the same
 * bits.  Returns 0, or -1 on bad arguments.
 */
int oracle_average_grads(int dtype, int world, const void *const *grads,
                         float *out, int64_t n)
{
    if (world < 1 || n < 0) return -1;
    if (dtype != OR_F32 && dtype != OR_F16 && dtype != OR_BF16) return -1;
    unsigned int csr = _mm_getcsr();
    _mm_setcsr(csr & ~(0x8000u | 0x0040u));
    for (int64_t i = 0; i < n; i++) {
        float sum = load_param(grads[0], dtype, i);
        for (int q = 1; q < world; q++)
            sum = sum + load_param(grads[q], dtype, i);
        out[i] = sum / (float)world;
    }
    _mm_setcsr(csr);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* The fp64 shadow: the same definitions entirely in double, used to bound    */
/* the rounding error of the fp32 oracle.  m2 may be NULL for Adam.           */
/* ------------------------------------------------------------------------ */

int oracle_step_f64(int algo, int skip_zeros, double lr, double beta1,
                    double beta2, double beta3, double alpha, double eps,
                    double weight_decay, int step, double *param,
                    const double *grad, double *m, double *m2, double *v,
                    int64_t n)
{
    if (step < 1 || n < 0) return -1;
    if (algo != OR_ADAM && algo != OR_ADEMAMIX) return -1;
    if (algo == OR_ADEMAMIX && m2 == NULL && n > 0) return -1;

    const double bc1 = 1.0 - pow(beta1, (double)step);
    const double bc2 = 1.0 - pow(beta2, (double)step);
    const double decay = 1.0 - lr * weight_decay;

    for (int64_t i = 0; i < n; i++) {
        double g = grad[i];
        if (skip_zeros && g == 0.0) continue;
        m[i] = beta1 * m[i] + (1.0 - beta1) * g;
        v[i] = beta2 * v[i] + (1.0 - beta2) * g * g;
        double num = m[i] / bc1;
        if (algo == OR_ADEMAMIX) {
            m2[i] = beta3 * m2[i] + (1.0 - beta3) * g;
            num += alpha * m2[i];
        }
        double den = sqrt(v[i] / bc2) + eps;
        param[i] = param[i] * decay - lr * (num / den);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Array forms of the conversions, so the tests can sweep many values.        */
/* dtype 1 = fp16, 2 = bf16.                                                  */
/* ------------------------------------------------------------------------ */

int oracle_narrow_array(int dtype, const float *x, uint16_t *out, int64_t n)
{
    if (dtype != OR_F16 && dtype != OR_BF16) return -1;
    for (int64_t i = 0; i < n; i++)
        out[i] = dtype == OR_F16 ? oracle_f32_to_f16(x[i]) : oracle_f32_to_bf16(x[i]);
    return 0;
}

int oracle_widen_array(int dtype, const uint16_t *h, float *out, int64_t n)
{
    if (dtype != OR_F16 && dtype != OR_BF16) return -1;
    for (int64_t i = 0; i < n; i++)
        out[i] = dtype == OR_F16 ? oracle_f16_to_f32(h[i]) : oracle_bf16_to_f32(h[i]);
    return 0;
}
