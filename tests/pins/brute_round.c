/*
 * brute_round.c -- test-side brute-force references for the scalar roundings.
 *
 * Independent of the oracle's method: the grids are decoded here from the bit
 * fields of each format, and rounding is a nearest-value search with binary64
 * distances; a tie between two neighbouring grid points goes to the even code.
 * The checkers walk every binary32 bit pattern in a range and count the
 * patterns on which a given encoder (a function pointer handed in from the
 * test) disagrees.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

typedef uint8_t (*encode_fn)(float);

static float f32_from_bits(uint32_t u) { float f; memcpy(&f, &u, sizeof f); return f; }

/* E2M1 magnitude of a 3-bit code: exponent field e (bias 1), mantissa bit m. */
static double e2m1_mag_from_fields(int c)
{
    int e = (c >> 1) & 3, m = c & 1;
    if (e == 0) return 0.5 * m;                 /* subnormal: m * 2^-1 */
    return (1.0 + 0.5 * m) * ldexp(1.0, e - 1);
}

/* E4M3FN magnitude of a 7-bit code (0x7f is NaN and never used here). */
static double e4m3_mag_from_fields(int c)
{
    int e = (c >> 3) & 15, m = c & 7;
    if (e == 0) return (m / 8.0) * ldexp(1.0, -6);
    return (1.0 + m / 8.0) * ldexp(1.0, e - 7);
}

uint8_t brute_e2m1(float v)
{
    uint8_t sign = signbit(v) ? 8 : 0;
    double a = fabs((double)v);
    if (isinf(a) || a > 6.0) return sign | 7;
    int best = 0;
    double bestd = INFINITY;
    for (int c = 0; c < 8; ++c) {
        double d = fabs(a - e2m1_mag_from_fields(c));
        if (d < bestd || (d == bestd && (c % 2 == 0))) { best = c; bestd = d; }
    }
    return sign | (uint8_t)best;
}

static double E4M3_TABLE[127];
static int e4m3_table_ready = 0;

static void e4m3_table_init(void)
{
    if (e4m3_table_ready) return;
    for (int c = 0; c < 127; ++c) E4M3_TABLE[c] = e4m3_mag_from_fields(c);
    e4m3_table_ready = 1;
}

uint8_t brute_e4m3(float t)
{
    e4m3_table_init();
    uint8_t sign = signbit(t) ? 0x80 : 0;
    double a = fabs((double)t);
    if (isinf(a) || a >= 448.0) return sign | 0x7e;
    /* bisection: largest code whose value is <= a */
    int lo = 0, hi = 126;
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if (E4M3_TABLE[mid] <= a) lo = mid; else hi = mid - 1;
    }
    int c = lo;
    if (c < 126) {
        double d0 = a - E4M3_TABLE[c], d1 = E4M3_TABLE[c + 1] - a;
        if (d1 < d0 || (d1 == d0 && ((c + 1) % 2 == 0))) c = c + 1;
    }
    return sign | (uint8_t)c;
}

void brute_prepare(void) { e4m3_table_init(); }

/*
 * Count bit patterns u in [lo, hi) (NaN patterns skipped) where fn(u) differs
 * from brute(u).  which = 0: E2M1, which = 1: E4M3.  first_bad receives the
 * smallest disagreeing pattern (or 0xffffffff).
 */
uint64_t brute_count_mismatch(encode_fn fn, int which, uint64_t lo, uint64_t hi, uint32_t *first_bad)
{
    e4m3_table_init();
    uint64_t bad = 0;
    uint32_t first = 0xffffffffu;
    #pragma omp parallel for schedule(static, 1 << 16) reduction(+ : bad) reduction(min : first)
    for (uint64_t u = lo; u < hi; ++u) {
        float v = f32_from_bits((uint32_t)u);
        if (isnan(v)) continue;
        uint8_t want = which == 0 ? brute_e2m1(v) : brute_e4m3(v);
        if (fn(v) != want) { ++bad; if ((uint32_t)u < first) first = (uint32_t)u; }
    }
    *first_bad = first;
    return bad;
}
