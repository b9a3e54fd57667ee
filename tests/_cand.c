/* Candidate bf16 values of exact fp64 values, and the charged error of a
 * device tensor against them, in one pass (test infrastructure; the rule is
 * stated in tests/_parity.py).
 *
 * For each element: near = v rounded to bf16 (nearest, ties to even); the
 * other neighbour of v is also correct when the dropped bits of v (45 of the
 * 52 fraction bits) lie within window * 2^45 of the halfway pattern 2^44.
 * Values below the bf16 normal range (|v| < 2^-126) round on the bf16
 * subnormal grid (spacing 2^-133) and get no second value.
 *
 * Outputs: pick[i] = the device value where it is one of the candidates, else
 * near; stats[0] = max charged |error|, stats[1] = max |got - near|,
 * stats[2] = sum near^2, stats[3] = number of elements with two candidates.
 * A NaN device value is charged +inf.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

static inline double from_bits(uint64_t b) { double d; memcpy(&d, &b, 8); return d; }
static inline uint64_t to_bits(double d) { uint64_t b; memcpy(&b, &d, 8); return b; }
static inline double bf16_value(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static inline void cands(double v, double window, double* near, double* alt) {
    if (fabs(v) < 0x1p-126) {
        *near = *alt = nearbyint(v / 0x1p-133) * 0x1p-133;
        return;
    }
    const uint64_t one = 1ull << 45, half = 1ull << 44;
    const uint64_t b = to_bits(v);
    const uint64_t low = b & (one - 1), keep = b - low;
    const int up = low > half || (low == half && ((b >> 45) & 1));
    const uint64_t nb = keep + (up ? one : 0);
    const double dist = fabs((double)low - (double)half);
    *near = from_bits(nb);
    *alt = dist <= window * (double)one ? from_bits(keep + (up ? 0 : one)) : *near;
}

void cand_tally(const double* v, const uint16_t* g_bf16, const double* g_f64, int64_t n,
                double window, double* pick, double* stats) {
    double mch = 0.0, mst = 0.0, ss = 0.0, two = 0.0;
#pragma omp parallel for reduction(max : mch, mst) reduction(+ : ss, two) schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        double near, alt;
        cands(v[i], window, &near, &alt);
        const double g = g_bf16 ? bf16_value(g_bf16[i]) : g_f64[i];
        const double st = isnan(g) ? INFINITY : fabs(g - near);
        const double ch = isnan(g) ? INFINITY : fmin(st, fabs(g - alt));
        if (ch > mch) mch = ch;
        if (st > mst) mst = st;
        ss += near * near;
        two += (near != alt);
        pick[i] = (g == alt) ? alt : near;
    }
    stats[0] = mch;
    stats[1] = mst;
    stats[2] = ss;
    stats[3] = two;
}

void cand_only(const double* v, int64_t n, double window, double* near_out, double* alt_out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) cands(v[i], window, &near_out[i], &alt_out[i]);
}
