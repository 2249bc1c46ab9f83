// Normal-float codebook on the host (bbc_nf_codebook in include/bbc.h).
//
// Definition (bitsandbytes k-bit patch series, create_normal_float_codebook):
// for n = 2^K levels, the standard-normal quantile at the bin midpoints
// p_i = (2i+1)/(2n) (these are exact in fp32 and fp64 for n a power of two),
// evaluated in double, rounded to fp32, then divided in fp32 by the largest
// magnitude.
//
// The quantile is found by solving Phi(x) = p with the C library's erfc,
// Phi(x) = erfc(-x / sqrt 2) / 2: bisection to bracket the root to about one
// part in 2^50, then Newton steps x -= (Phi(x) - p) / phi(x) until the step
// vanishes. The error is set by erfc's accuracy (about one ulp of p), far below
// the half-ulp of fp32 that the final rounding keeps.
#include <cmath>
#include <string>

#include "bbc.h"

namespace {

double norm_cdf(double x) { return 0.5 * std::erfc(-x / std::sqrt(2.0)); }

double norm_quantile(double p) {
    double lo = -40.0, hi = 40.0;
    for (int i = 0; i < 60; i++) {
        const double mid = 0.5 * (lo + hi);
        if (norm_cdf(mid) < p) lo = mid;
        else hi = mid;
    }
    double x = 0.5 * (lo + hi);
    const double inv_sqrt_2pi = 0.39894228040143267794;
    for (int i = 0; i < 8; i++) {
        const double dens = inv_sqrt_2pi * std::exp(-0.5 * x * x);
        const double step = (norm_cdf(x) - p) / dens;
        x -= step;
        if (std::fabs(step) <= 1e-17 * std::fabs(x)) break;
    }
    return x;
}

}  // namespace

extern "C" int bbc_nf_codebook(int K, float* out) {
    if (!out || K < 1 || K > 8) return BBC_ERR_INVALID;
    const int n = 1 << K;
    float vmax = 0.0f;
    for (int i = 0; i < n; i++) {
        const double p = (2.0 * i + 1.0) / (2.0 * n);
        out[i] = (float)norm_quantile(p);
        const float a = std::fabs(out[i]);
        if (a > vmax) vmax = a;
    }
    for (int i = 0; i < n; i++) out[i] = out[i] / vmax;
    return BBC_OK;
}
