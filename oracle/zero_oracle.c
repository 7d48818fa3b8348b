/*
 * CPU oracle for the ZeRO-DP partitioned mixed-precision Adam step.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline of the benchmark load this file's library.  The product path never
 * does, and this file shares no code with it.
 *
 * What it computes, and where each part comes from:
 *   - Mixed-precision model states: fp16 (or bf16) parameters and gradients,
 *     fp32 master weights, momentum and variance for Adam
 *     [ZeRO explainer (azimuth.plus), model-states paragraph].
 *   - Reduction of N replicas' gradients.  Plain data parallelism all-reduces
 *     them [ZeRO explainer, data-parallelism paragraph]; Stage 2 reduce-
 *     scatters them so that rank r gets only its 1/N slice
 *     [ZeRO explainer, "Stage 2 - Gradient Partitioning (P_os+g)"].
 *     The pages fix no summation order or precision; this oracle adds the N
 *     replicas in rank order 0..N-1 in fp32, starting from replica 0.
 *   - The Adam update of a partition of the fp32 states
 *     [ZeRO explainer, "Stage 1 - Optimizer State Partitioning (P_os)"].
 *     The pages name Adam and its states but print no formula; this oracle
 *     uses Adam with bias correction and epsilon outside the square root
 *     (Kingma & Ba), with decoupled weight decay (AdamW, decay factor
 *     1 - lr*wd), written in one fixed order of fp32 operations:
 *         g   = s * inv                      inv = 1/(divisor * loss_scale)
 *         m'  = fma(b1, m, (1-b1)*g)
 *         v'  = fma(b2, v, ((1-b2)*g)*g)
 *         den = fma(sqrt(v'), 1/sqrt(1-b2^t), eps)     = sqrt(v_hat) + eps
 *         u   = (m' * 1/(1-b1^t)) / den                = m_hat / den
 *         p'  = fma(-lr, u, p * (1 - lr*wd))
 *     The five scalar constants are computed in double and rounded once to
 *     float.  Division and square root are the IEEE correctly rounded ones.
 *   - The low-precision write-back of updated parameters, which is what the
 *     all-gather distributes [ZeRO explainer, Stage 1 and Stage 2]:
 *     round-to-nearest-even from fp32, written out from the IEEE 754
 *     definition below.
 *   - The all-gather reconstruct of N shards
 *     [ZeRO explainer, "Stage 3 - Parameter Partitioning (P_os+g+p)"].
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math (no contraction of a*b+c
 * into fma except where fmaf is written).  OpenMP, when enabled, only splits
 * the element loops; every element's arithmetic is unchanged.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* Storage formats (IEEE 754 binary16 and bfloat16)                          */
/* ------------------------------------------------------------------------ */

/* binary16 bits -> fp32, exact.  1 sign, 5 exponent (bias 15), 10 fraction. */
float orc_f16_to_f32(uint16_t h)
{
    uint32_t sign = (uint32_t)(h >> 15) & 1u;
    uint32_t e = (uint32_t)(h >> 10) & 0x1fu;
    uint32_t f = (uint32_t)h & 0x3ffu;
    float mag;
    if (e == 0x1f) {
        mag = f ? NAN : INFINITY;
    } else if (e == 0) {
        mag = ldexpf((float)f, -24);               /* subnormal: f * 2^-24 */
    } else {
        mag = ldexpf((float)(1024u + f), (int)e - 25); /* (1.f) * 2^(e-15) */
    }
    return sign ? -mag : mag;
}

/* bfloat16 bits -> fp32, exact: the top half of an fp32 word. */
float orc_bf16_to_f32(uint16_t b)
{
    uint32_t x = (uint32_t)b << 16;
    float f;
    memcpy(&f, &x, sizeof f);
    return f;
}

/* Round-half-to-even of an integer significand shifted right by `shift`. */
static uint32_t rne_shift(uint32_t sig, int shift)
{
    if (shift <= 0) return sig;
    if (shift >= 32) return 0;
    uint32_t q = sig >> shift;
    uint32_t rem = sig & ((1u << shift) - 1u);
    uint32_t half = 1u << (shift - 1);
    if (rem > half || (rem == half && (q & 1u))) q += 1u;
    return q;
}

/* fp32 -> binary16, round to nearest, ties to even; overflow gives inf. */
uint16_t orc_f32_to_f16(float x)
{
    uint32_t u;
    memcpy(&u, &x, sizeof u);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    uint32_t ex = (u >> 23) & 0xffu;
    uint32_t fr = u & 0x7fffffu;
    if (ex == 0xffu) return (uint16_t)(sign | (fr ? 0x7e00u : 0x7c00u));
    if (ex == 0) return sign;            /* fp32 zero/subnormal < 2^-126: rounds to 0 */
    int E = (int)ex - 127;               /* x = M * 2^(E-23), M has 24 bits */
    uint32_t M = 0x800000u | fr;
    if (E > 15) return (uint16_t)(sign | 0x7c00u);
    if (E >= -14) {
        /* normal target: keep 11 significant bits */
        uint32_t q = rne_shift(M, 13);   /* in [0x400, 0x800] */
        uint32_t bits = ((uint32_t)(E + 14) << 10) + q;   /* a carry bumps the exponent */
        if (bits >= 0x7c00u) return (uint16_t)(sign | 0x7c00u);
        return (uint16_t)(sign | bits);
    }
    /* subnormal target: units of 2^-24, x / 2^-24 = M * 2^(E+1) */
    uint32_t q = rne_shift(M, -(E + 1)); /* q == 0x400 is the smallest normal */
    return (uint16_t)(sign | q);
}

/* fp32 -> bfloat16, round to nearest, ties to even; overflow gives inf. */
uint16_t orc_f32_to_bf16(float x)
{
    uint32_t u;
    memcpy(&u, &x, sizeof u);
    uint32_t sign = u & 0x80000000u;
    uint32_t mag = u & 0x7fffffffu;
    if (mag > 0x7f800000u) return (uint16_t)((sign >> 16) | 0x7fc0u | ((mag >> 16) & 0x3fu));
    if (mag == 0x7f800000u) return (uint16_t)((sign >> 16) | 0x7f80u);
    /* drop 16 low bits of the magnitude with ties to even; a carry out of
     * the fraction increments the exponent, and out of the largest finite
     * exponent it produces the inf encoding 0x7f80 */
    uint32_t q = rne_shift(mag, 16);
    return (uint16_t)((sign >> 16) | q);
}

void orc_f16_to_f32_array(const uint16_t* h, float* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_f16_to_f32(h[i]);
}

void orc_bf16_to_f32_array(const uint16_t* h, float* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_bf16_to_f32(h[i]);
}

void orc_f32_to_f16_array(const float* x, uint16_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_f32_to_f16(x[i]);
}

void orc_f32_to_bf16_array(const float* x, uint16_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_f32_to_bf16(x[i]);
}

/* dtype codes shared only inside this oracle: 0 = binary16, 1 = bfloat16 */
static float to_f32(uint16_t bits, int dtype)
{
    return dtype == 0 ? orc_f16_to_f32(bits) : orc_bf16_to_f32(bits);
}

static uint16_t from_f32(float x, int dtype)
{
    return dtype == 0 ? orc_f32_to_f16(x) : orc_f32_to_bf16(x);
}

/* ------------------------------------------------------------------------ */
/* Gradient reduction                                                        */
/* ------------------------------------------------------------------------ */

/*
 * s[j] = fp32(G_0[begin+j]) + fp32(G_1[begin+j]) + ... + fp32(G_{N-1}[begin+j]),
 * added left to right in fp32.
 *
 * begin = 0, count = padded size: the all-reduce of plain data parallelism
 * (every rank gets the whole sum) [ZeRO explainer, data-parallelism paragraph].
 * begin = r*P, count = P: rank r's slice of a reduce-scatter
 * [ZeRO explainer, "Stage 2 - Gradient Partitioning (P_os+g)"].
 */
void orc_reduce(const uint16_t* const* G, int32_t N, int dtype,
                int64_t begin, int64_t count, float* s)
{
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < count; ++j) {
        float acc = to_f32(G[0][begin + j], dtype);
        for (int32_t k = 1; k < N; ++k) acc = acc + to_f32(G[k][begin + j], dtype);
        s[j] = acc;
    }
}

/* 1 if any reduced gradient is inf or NaN, else 0 (the overflow test of
 * dynamic loss scaling, applied to the fp32 sums). */
int32_t orc_any_nonfinite(const float* s, int64_t count)
{
    int32_t any = 0;
    for (int64_t j = 0; j < count; ++j)
        if (!isfinite(s[j])) any = 1;
    return any;
}

/* sum over j of (s[j]*inv)^2, the unscaled gradient computed in fp32 and
 * squared and summed in double. */
double orc_grad_sqnorm(const float* s, int64_t count, float inv)
{
    double acc = 0.0;
    for (int64_t j = 0; j < count; ++j) {
        float g = s[j] * inv;
        acc += (double)g * (double)g;
    }
    return acc;
}

/* The reduced gradient a rank keeps after the reduce-scatter (ZeRO explainer,
 * "Stage 2 - Gradient Partitioning (P_os+g)"), unscaled: g[j] = s[j]*inv in
 * fp32, the same g the update and the norm use. */
void orc_unscale(const float* s, int64_t count, float inv, float* g)
{
    for (int64_t j = 0; j < count; ++j) g[j] = s[j] * inv;
}

/* ------------------------------------------------------------------------ */
/* Adam                                                                     */
/* ------------------------------------------------------------------------ */

/* Derived constants, each computed in double and rounded once to float.
 * c[0] lr   c[1] beta1  c[2] beta2  c[3] eps
 * c[4] inv = 1/(divisor*loss_scale)
 * c[5] 1-beta1       c[6] 1-beta2
 * c[7] 1/(1-beta1^t) c[8] 1/sqrt(1-beta2^t)
 * c[9] 1 - lr*wd
 * t is the 1-based count of applied updates, this one included. */
void orc_adam_constants(float lr, float beta1, float beta2, float eps, float wd,
                        int64_t t, double divisor, float loss_scale, float* c)
{
    c[0] = lr;
    c[1] = beta1;
    c[2] = beta2;
    c[3] = eps;
    c[4] = (float)(1.0 / (divisor * (double)loss_scale));
    c[5] = (float)(1.0 - (double)beta1);
    c[6] = (float)(1.0 - (double)beta2);
    c[7] = (float)(1.0 / (1.0 - pow((double)beta1, (double)t)));
    c[8] = (float)(1.0 / sqrt(1.0 - pow((double)beta2, (double)t)));
    c[9] = (float)(1.0 - (double)lr * (double)wd);
}

/* One Adam/AdamW update of `count` elements of a partition, in place on the
 * fp32 master/m/v arrays; the new master is rounded into p16 (dtype 0 =
 * binary16, 1 = bfloat16).  s holds the reduced, still loss-scaled sums. */
void orc_adam_update(const float* s, int64_t count, const float* c,
                     float* master, float* m, float* v, uint16_t* p16, int pdtype)
{
    const float lr = c[0], b1 = c[1], b2 = c[2], eps = c[3], inv = c[4];
    const float omb1 = c[5], omb2 = c[6], rbc1 = c[7], rsbc2 = c[8], decay = c[9];
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < count; ++j) {
        float g = s[j] * inv;
        float mn = fmaf(b1, m[j], omb1 * g);
        float vn = fmaf(b2, v[j], (omb2 * g) * g);
        float den = fmaf(sqrtf(vn), rsbc2, eps);
        float u = (mn * rbc1) / den;
        float pn = fmaf(-lr, u, master[j] * decay);
        m[j] = mn;
        v[j] = vn;
        master[j] = pn;
        p16[j] = from_f32(pn, pdtype);
    }
}

/* Global-norm gradient clipping (not on the pages; the usual rule): the
 * unscaled gradient is multiplied by
 *     clip = min(1, max_norm / (sqrt(total_sqnorm) + 1e-6)),
 * computed in double and rounded once to float. */
float orc_clip_coefficient(double total_sqnorm, double max_norm)
{
    double coef = max_norm / (sqrt(total_sqnorm) + 1e-6);
    return coef < 1.0 ? (float)coef : 1.0f;
}

/* orc_adam_update with clipped gradients: g = (s * inv) * clip, the rest of
 * the update unchanged.  clip == 1 reproduces orc_adam_update exactly. */
void orc_adam_update_clipped(const float* s, int64_t count, const float* c, float clip,
                             float* master, float* m, float* v, uint16_t* p16, int pdtype)
{
    const float lr = c[0], b1 = c[1], b2 = c[2], eps = c[3], inv = c[4];
    const float omb1 = c[5], omb2 = c[6], rbc1 = c[7], rsbc2 = c[8], decay = c[9];
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < count; ++j) {
        float g = (s[j] * inv) * clip;
        float mn = fmaf(b1, m[j], omb1 * g);
        float vn = fmaf(b2, v[j], (omb2 * g) * g);
        float den = fmaf(sqrtf(vn), rsbc2, eps);
        float u = (mn * rbc1) / den;
        float pn = fmaf(-lr, u, master[j] * decay);
        m[j] = mn;
        v[j] = vn;
        master[j] = pn;
        p16[j] = from_f32(pn, pdtype);
    }
}

/* ------------------------------------------------------------------------ */
/* All-gather                                                               */
/* ------------------------------------------------------------------------ */

/* dst[r*P + j] = shards[r][offset + j] for r < N, j < P: every rank's
 * updated slice placed at its rank-major position
 * [ZeRO explainer, "Stage 3 - Parameter Partitioning (P_os+g+p)"]. */
void orc_allgather(const uint16_t* const* shards, int32_t N, int64_t offset,
                   int64_t P, uint16_t* dst)
{
    for (int32_t r = 0; r < N; ++r)
        for (int64_t j = 0; j < P; ++j)
            dst[(int64_t)r * P + j] = shards[r][offset + j];
}

/* threads OpenMP would use (1 without OpenMP) */
int32_t orc_threads(void)
{
#ifdef _OPENMP
    return (int32_t)omp_get_max_threads();
#else
    return 1;
#endif
}

void orc_set_threads(int32_t n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
