/*
 * mq_oracle.c -- plain, slow CPU reference for the NVFP4 W4A4 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library and
 * its Python binding) may call, link or load this file.  Only the tests, the
 * smoke check and the CPU-baseline leg of the benchmark use it.  It shares no
 * code, header, table or helper with the CUDA sources.
 *
 * What it computes (NVFP4 two-level microscaling, as stated in
 *   [P1] "Mix-Quant：面向智能体LLM的量化预填充与精确解码" (paper.rainbus.top
 *        digest), section 方法步骤详情, step (3), and section NVFP4 微缩放量化;
 *   [P3] "Mix-Quant: Quantized Prefilling, Precise Decoding for Agentic LLMs"
 *        (r9-hu paper digest), section Method, item 1):
 *
 *   sigma_b = Pi_E4M3( max_{i in b} |x_i| / (alpha_x * q_max) )      per block b
 *   q_i     = Pi_FP4 ( x_i / (alpha_x * sigma_b(i)) )               round to nearest
 *   xhat_i  = alpha_x * sigma_b(i) * q_i                             dequantization
 *
 * with blocks of g = 16 consecutive elements along K, E2M1 element codes,
 * E4M3 block scales and one fp32 tensor-level scale alpha_x.
 *
 * Where the pages are silent the following readings are used (each one is
 * listed in the design notes of the repository):
 *   R1  alpha_x = fl32(amax / (q_max * 448)) = fl32(amax / 2688), amax = max|x|
 *       over the whole tensor; alpha_x = 1 when amax = 0.
 *   R2  q_max = 6, the largest E2M1 magnitude.
 *   R3  Pi_E4M3 rounds to nearest, ties to even, onto the OCP E4M3FN grid and
 *       saturates to 448 (no infinity).  Its argument is t = fl32(amax_b / d)
 *       with d = fl32(6 * alpha_x).
 *   R4  A block whose scale rounds to 0 gets all codes +0 (0x0).
 *   R5  Pi_FP4 is applied to v = fl32(x_i * r), r = fl32(1 / s),
 *       s = fl32(alpha_x * sigma_b): one reciprocal per block, one multiply per
 *       element.  The exact-real reading is also provided
 *       (oracle_quantize_exact) so the two can be compared.
 *   R6  Pi_FP4 rounds to nearest, ties to even code, saturating at |6|.
 *   R7  The sign of a value that rounds to zero is kept (code 0x8 for -0).
 *   R8  Codes are packed two per byte, the lower K index in the low nibble.
 *
 * All float arithmetic below is IEEE binary32 or binary64 with round to
 * nearest even; build with -ffp-contract=off and without -ffast-math.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Threads the row loops below may use (OMP_NUM_THREADS), 1 without OpenMP. */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------- */
/* bf16 <-> binary32 / binary64                                               */
/* ------------------------------------------------------------------------- */

/* A bf16 value is the upper 16 bits of a binary32 value: widening is exact. */
float oracle_bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/*
 * Round a binary64 value to bf16, to nearest, ties to even, with overflow to
 * infinity.  Works on the exact value: split it as (integer mantissa) * 2^e
 * with 8 significant bits kept.
 */
uint16_t oracle_bf16_rne(double v)
{
    if (isnan(v)) return 0x7fc0;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0) return sign;
    int ex;
    frexp(a, &ex);                       /* a in [2^(ex-1), 2^ex)          */
    int unbiased = ex - 1;               /* a in [2^u, 2^(u+1))            */
    if (unbiased < -126) unbiased = -126; /* subnormal bf16 range          */
    double quantum = ldexp(1.0, unbiased - 7);   /* 7 fraction bits        */
    double n = nearbyint(a / quantum);   /* exact scaling, RNE to integer  */
    double r = n * quantum;
    if (r >= ldexp(1.0, 128)) return sign | 0x7f80;   /* overflow -> inf  */
    /* r is exactly representable in binary32 now */
    float f = (float)r;
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | (u >> 16));
}

/* ------------------------------------------------------------------------- */
/* E2M1 (FP4): 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit           */
/* ------------------------------------------------------------------------- */

/* Magnitudes of codes 0..7: the E2M1 grid {0, 0.5, 1, 1.5, 2, 3, 4, 6}. */
static const double E2M1_MAGNITUDE[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double oracle_e2m1_decode(uint8_t code)
{
    double m = E2M1_MAGNITUDE[code & 7];
    return (code & 8) ? -m : m;
}

/*
 * Pi_FP4 (R6, R7): nearest grid magnitude; on an exact midpoint between two
 * neighbouring codes the even code wins; magnitudes above 6 saturate to 6.
 */
uint8_t oracle_e2m1_encode(float v)
{
    uint8_t sign = signbit(v) ? 8 : 0;
    double a = fabs((double)v);
    for (int c = 0; c < 7; ++c) {
        double mid = 0.5 * (E2M1_MAGNITUDE[c] + E2M1_MAGNITUDE[c + 1]);
        if (a < mid) return sign | (uint8_t)c;
        if (a == mid) return sign | (uint8_t)((c % 2 == 0) ? c : c + 1);
    }
    return sign | 7;                     /* |v| above 5: nearest is 6, or saturate */
}

/* ------------------------------------------------------------------------- */
/* E4M3 (OCP E4M3FN): 1 sign, 4 exponent bits (bias 7), 3 mantissa bits,     */
/* no infinity, 0x7f/0xff are NaN, largest finite 448.                        */
/* ------------------------------------------------------------------------- */

double oracle_e4m3_decode(uint8_t code)
{
    int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);             /* (m/8) * 2^(1-7)   */
    else        v = ldexp((double)(8 + m), e - 10);   /* (1+m/8) * 2^(e-7) */
    return s ? -v : v;
}

/*
 * Pi_E4M3 (R3): round to nearest, ties to even code, saturate to 448.
 * In a binade [2^u, 2^(u+1)) the grid step is 2^(u-3); below 2^-6 the grid is
 * the subnormal step 2^-9.  Scaling by the step is exact, so rounding the
 * scaled value to an integer (ties to even) is rounding onto the grid, and an
 * even integer is an even mantissa, i.e. an even code.
 */
uint8_t oracle_e4m3_encode(float t)
{
    uint8_t sign = signbit(t) ? 0x80 : 0;
    double a = fabs((double)t);
    if (a >= 448.0) return sign | 0x7e;               /* satfinite           */
    if (a < ldexp(1.0, -6)) {                          /* subnormal binade    */
        double n = nearbyint(a / ldexp(1.0, -9));      /* 0..8                */
        return sign | (uint8_t)n;                      /* n = 8 is 2^-6 = 0x08 */
    }
    int ex;
    frexp(a, &ex);                                     /* a in [2^(ex-1), 2^ex) */
    double step = ldexp(1.0, ex - 1 - 3);
    double n = nearbyint(a / step);                    /* 8..16               */
    int biased = (ex - 1) + 7;
    return sign | (uint8_t)((biased << 3) + ((int)n - 8)); /* n = 16 carries up */
}

/* ------------------------------------------------------------------------- */
/* Tensor-level scale alpha_x (R1)                                           */
/* ------------------------------------------------------------------------- */

float oracle_tensor_scale(const uint16_t *x, int64_t numel)
{
    float amax = 0.0f;
    for (int64_t i = 0; i < numel; ++i) {
        float v = fabsf(oracle_bf16_to_f32(x[i]));
        if (v > amax) amax = v;
    }
    if (amax == 0.0f) return 1.0f;
    return amax / 2688.0f;               /* q_max * largest E4M3 = 6 * 448 */
}

/* ------------------------------------------------------------------------- */
/* Quantization of a [rows, K] bf16 tensor in 16-element blocks along K       */
/* ------------------------------------------------------------------------- */

/*
 * codes : [rows, K/2] bytes, element 2j in the low nibble of byte j (R8)
 * scales: [rows, K/16] E4M3 codes in plain row-major order
 */
void oracle_quantize(const uint16_t *x, int64_t rows, int64_t K, float alpha,
                     uint8_t *codes, uint8_t *scales)
{
    const int64_t nblk = K / 16;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nblk; ++b) {
            const uint16_t *xb = x + r * K + b * 16;
            float xf[16];
            float amax_b = 0.0f;
            for (int i = 0; i < 16; ++i) {
                xf[i] = oracle_bf16_to_f32(xb[i]);
                if (fabsf(xf[i]) > amax_b) amax_b = fabsf(xf[i]);
            }
            /* sigma_b = Pi_E4M3(amax_b / (alpha * q_max)) */
            float d = 6.0f * alpha;
            float t = amax_b / d;
            uint8_t sc = oracle_e4m3_encode(t);
            double sigma = oracle_e4m3_decode(sc);
            scales[r * nblk + b] = sc;

            uint8_t q[16];
            if (sigma == 0.0) {
                for (int i = 0; i < 16; ++i) q[i] = 0;       /* R4 */
            } else {
                /* q_i = Pi_FP4(x_i / (alpha * sigma_b)) via the block reciprocal */
                float s = alpha * (float)sigma;
                float rcp = 1.0f / s;
                for (int i = 0; i < 16; ++i) q[i] = oracle_e2m1_encode(xf[i] * rcp);
            }
            uint8_t *cb = codes + r * (K / 2) + b * 8;
            for (int j = 0; j < 8; ++j) cb[j] = (uint8_t)(q[2 * j] | (q[2 * j + 1] << 4));
        }
    }
}

/*
 * The exact-real reading of the same two formulas: sigma_b and q_i are the
 * round-to-nearest-even images of the exact real quotients.  Operands are
 * bf16 (8 significant bits), fp32 alpha (24 bits) and E4M3 (4 bits); their
 * products are exact in binary64 and a correctly rounded binary64 quotient
 * cannot cross a midpoint of the coarse E4M3/E2M1 grids unless the exact
 * quotient sits on it, so binary64 division followed by the grid rounding
 * gives the exact-real result.  The grid rounding is therefore applied to
 * the binary64 quotient directly (no binary32 step).
 */
static uint8_t e2m1_encode_f64(double v)
{
    uint8_t sign = signbit(v) ? 8 : 0;
    double a = fabs(v);
    for (int c = 0; c < 7; ++c) {
        double mid = 0.5 * (E2M1_MAGNITUDE[c] + E2M1_MAGNITUDE[c + 1]);
        if (a < mid) return sign | (uint8_t)c;
        if (a == mid) return sign | (uint8_t)((c % 2 == 0) ? c : c + 1);
    }
    return sign | 7;
}

static uint8_t e4m3_encode_f64(double a)
{
    if (a >= 448.0) return 0x7e;
    if (a < ldexp(1.0, -6)) return (uint8_t)nearbyint(a / ldexp(1.0, -9));
    int ex;
    frexp(a, &ex);
    double n = nearbyint(a / ldexp(1.0, ex - 4));
    return (uint8_t)(((ex + 6) << 3) + ((int)n - 8));
}

void oracle_quantize_exact(const uint16_t *x, int64_t rows, int64_t K, float alpha,
                           uint8_t *codes, uint8_t *scales)
{
    const int64_t nblk = K / 16;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nblk; ++b) {
            const uint16_t *xb = x + r * K + b * 16;
            double amax_b = 0.0;
            for (int i = 0; i < 16; ++i) {
                double v = fabs((double)oracle_bf16_to_f32(xb[i]));
                if (v > amax_b) amax_b = v;
            }
            uint8_t sc = e4m3_encode_f64(amax_b / (6.0 * (double)alpha));
            double sigma = oracle_e4m3_decode(sc);
            scales[r * nblk + b] = sc;
            uint8_t q[16];
            for (int i = 0; i < 16; ++i) {
                if (sigma == 0.0) { q[i] = 0; continue; }
                q[i] = e2m1_encode_f64((double)oracle_bf16_to_f32(xb[i]) / ((double)alpha * sigma));
            }
            uint8_t *cb = codes + r * (K / 2) + b * 8;
            for (int j = 0; j < 8; ++j) cb[j] = (uint8_t)(q[2 * j] | (q[2 * j + 1] << 4));
        }
    }
}

/* xhat_i = alpha * sigma_b(i) * q_i, exact in binary64 (30 significant bits). */
void oracle_dequantize(const uint8_t *codes, const uint8_t *scales, int64_t rows, int64_t K,
                       float alpha, double *out)
{
    const int64_t nblk = K / 16;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = codes[r * (K / 2) + k / 2];
            uint8_t q = (k % 2 == 0) ? (byte & 15) : (byte >> 4);
            double sigma = oracle_e4m3_decode(scales[r * nblk + k / 16]);
            out[r * K + k] = (double)alpha * sigma * oracle_e2m1_decode(q);
        }
    }
}

/* Round every element of a binary64 array to bf16 bits. */
void oracle_bf16_rne_array(const double *v, int64_t n, uint16_t *out)
{
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_bf16_rne(v[i]);
}

/* ------------------------------------------------------------------------- */
/* Block-scale storage order consumed by the Blackwell block-scaled MMA       */
/* ------------------------------------------------------------------------- */

/*
 * Scales are stored in atoms of 128 rows x 4 scale columns (512 bytes).  Atoms
 * are ordered row-tile major, k-tile minor.  Inside an atom, row r and scale
 * column c sit at byte (r % 32) * 16 + ((r / 32) % 4) * 4 + (c % 4).  Rows are
 * padded to a multiple of 128 and scale columns to a multiple of 4.
 */
int64_t oracle_scale_offset(int64_t row, int64_t kblock, int64_t K)
{
    int64_t katoms = (K / 16 + 3) / 4;
    int64_t atom = (row / 128) * katoms + kblock / 4;
    int64_t inner = (row % 32) * 16 + ((row / 32) % 4) * 4 + (kblock % 4);
    return atom * 512 + inner;
}

int64_t oracle_scale_bytes(int64_t rows, int64_t K)
{
    return ((rows + 127) / 128) * 128 * (((K / 16) + 3) / 4) * 4;
}

/* logical [rows, K/16] -> stored order (padding bytes are zero) */
void oracle_scales_to_stored(const uint8_t *logical, int64_t rows, int64_t K, uint8_t *stored)
{
    memset(stored, 0, (size_t)oracle_scale_bytes(rows, K));
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < K / 16; ++b)
            stored[oracle_scale_offset(r, b, K)] = logical[r * (K / 16) + b];
}

/* stored order -> logical [rows, K/16] */
void oracle_scales_from_stored(const uint8_t *stored, int64_t rows, int64_t K, uint8_t *logical)
{
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < K / 16; ++b)
            logical[r * (K / 16) + b] = stored[oracle_scale_offset(r, b, K)];
}

/* ------------------------------------------------------------------------- */
/* SwiGLU of a gate/up product (the MLP between the two W4A4 linears)        */
/* ------------------------------------------------------------------------- */

/*
 * The pages quantize the MLP's linears but give no numerics for the gated
 * activation between them (the down projection's input).  Readings:
 *   R11  The gate/up product is first rounded to bf16 exactly as the plain
 *        linear writes it: G = bf16(gate row products), U = bf16(up row
 *        products).  Then h = bf16( fl32( silu(G) * U ) ).
 *   R12  silu(g) = fl32( g / fl32(1 + e(-g)) ), where e(x) is a binary32
 *        exponential built from Cody and Waite's range reduction
 *        (x = k ln2 + r, ln2 split into a 16-bit head and a tail, |r| <= ln2/2)
 *        and the Taylor polynomial of e^r to degree 7 in Horner form, times
 *        2^k.  Every step is one IEEE binary32 operation (fmaf where written),
 *        so the value does not depend on where it is evaluated.  e(x) = +inf
 *        for x > 88 and 0 for x < -87 (k would leave the normal range).
 *   R13  The down projection quantizes H with its own tensor scale:
 *        alpha_h = fl32(max|h| / 2688) (R1), max over the whole [M, I] tensor.
 */
float oracle_exp_f32(float x)
{
    if (x > 88.0f) return INFINITY;
    if (x < -87.0f) return 0.0f;
    const float k = rintf(x * 0x1.715476p+0f);          /* nearest even of fl32(x log2 e) */
    float r = fmaf(-k, 0x1.62e4p-1f, x);                /* x - k ln2 (head, 16 bits)       */
    r = fmaf(-k, 0x1.7f7d1cp-20f, r);                   /* ... - k (ln2 - head)            */
    float p = 0x1.a01a02p-13f;                          /* 1/7!                            */
    p = fmaf(p, r, 0x1.6c16c2p-10f);                    /* 1/6!                            */
    p = fmaf(p, r, 0x1.111112p-7f);                     /* 1/5!                            */
    p = fmaf(p, r, 0x1.555556p-5f);                     /* 1/4!                            */
    p = fmaf(p, r, 0x1.555556p-3f);                     /* 1/3!                            */
    p = fmaf(p, r, 0.5f);
    p = fmaf(p, r, 1.0f);
    p = fmaf(p, r, 1.0f);
    const uint32_t eb = (uint32_t)((int)k + 127) << 23; /* 2^k, k in [-126, 127]          */
    float two_k;
    memcpy(&two_k, &eb, sizeof two_k);
    return p * two_k;
}

float oracle_silu_f32(float g)
{
    return g / (1.0f + oracle_exp_f32(-g));
}

/* h = bf16(fl32(silu(g) * u)) for bf16 g, u (R11, R12); binary32 -> bf16 RNE */
uint16_t oracle_swiglu_bf16(uint16_t g, uint16_t u)
{
    const float h = oracle_silu_f32(oracle_bf16_to_f32(g)) * oracle_bf16_to_f32(u);
    return oracle_bf16_rne((double)h);
}

void oracle_swiglu_array(const uint16_t *g, const uint16_t *u, int64_t n, uint16_t *h)
{
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) h[i] = oracle_swiglu_bf16(g[i], u[i]);
}
