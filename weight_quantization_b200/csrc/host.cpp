// Host-side helpers of libwq_b200: the Gaussian Lloyd-Max codebook ("orbit_quant.py",
// gaussian_lloyd_max and OrbitQuantizer.quantize_), status strings and the version.
#include <cmath>
#include <cstdint>
#include <limits>

#include "wq.h"

namespace {

// Inverse error function by Newton's method on erf (erf' = 2/sqrt(pi) exp(-y^2)), started from
// a bracketed bisection so that every step stays inside (-6, 6) where erf is far from +-1.
double erfinv_newton(double t) {
    if (t <= -1.0) return -std::numeric_limits<double>::infinity();
    if (t >= 1.0) return std::numeric_limits<double>::infinity();
    double lo = -6.0, hi = 6.0, y = 0.0;
    for (int i = 0; i < 40; ++i) {  // coarse bracket
        y = 0.5 * (lo + hi);
        (std::erf(y) < t ? lo : hi) = y;
    }
    const double two_over_sqrt_pi = 1.1283791670955126;
    for (int i = 0; i < 8; ++i) {
        const double f = std::erf(y) - t;
        const double step = f / (two_over_sqrt_pi * std::exp(-y * y));
        const double next = y - step;
        if (next == y) break;
        y = next;
    }
    return y;
}

}  // namespace

extern "C" wq_status wq_gaussian_lloyd_max(int bits, int iters, float *out) {
    if (!out) return WQ_ERR_NULL;
    if (bits < 1 || bits > 4) return WQ_ERR_BITS;
    if (iters < 0) return WQ_ERR_SHAPE;
    const int levels = 1 << bits;
    const double inf = std::numeric_limits<double>::infinity();
    const double root2 = std::sqrt(2.0), root2pi = std::sqrt(2.0 * 3.141592653589793);
    double c[16], edge[17];
    // initial levels at the Gaussian quantiles of the cell midpoints
    for (int k = 0; k < levels; ++k) c[k] = root2 * erfinv_newton(2.0 * ((k + 0.5) / levels) - 1.0);
    for (int it = 0; it < iters; ++it) {
        // cells between midpoints; level = conditional mean of N(0,1) on its cell
        edge[0] = -inf;
        edge[levels] = inf;
        for (int k = 1; k < levels; ++k) edge[k] = (c[k - 1] + c[k]) / 2.0;
        for (int k = 0; k < levels; ++k) {
            const double a = edge[k], b = edge[k + 1];
            const double pdf_a = std::exp(-a * a / 2.0) / root2pi, pdf_b = std::exp(-b * b / 2.0) / root2pi;
            const double cdf_a = 0.5 * (1.0 + std::erf(a / root2)), cdf_b = 0.5 * (1.0 + std::erf(b / root2));
            c[k] = (pdf_a - pdf_b) / (cdf_b - cdf_a);
        }
    }
    for (int k = 0; k < levels; ++k) out[k] = (float)c[k];
    return WQ_OK;
}

extern "C" wq_status wq_rpbh_codebook(int bits, int64_t d, float *out) {
    if (!out) return WQ_ERR_NULL;
    if (bits < 2 || bits > 4) return WQ_ERR_BITS;
    if (d <= 0) return WQ_ERR_SHAPE;
    float c[16];
    wq_status st = wq_gaussian_lloyd_max(bits, 200, c);
    if (st != WQ_OK) return st;
    // gaussian_lloyd_max(bits) * d ** -0.5: an fp32 tensor times a Python float, i.e. in fp32
    const float scale = (float)std::pow((double)d, -0.5);
    for (int k = 0; k < (1 << bits); ++k) out[k] = c[k] * scale;
    return WQ_OK;
}

extern "C" const char *wq_status_string(int status) {
    switch (status) {
        case WQ_OK: return "ok";
        case WQ_ERR_NULL: return "a required pointer is NULL";
        case WQ_ERR_SHAPE: return "bad count or dimension";
        case WQ_ERR_DTYPE: return "unsupported dtype code";
        case WQ_ERR_ALIGN: return "pointer misaligned";
        case WQ_ERR_BITS: return "bits must be 2, 3 or 4";
        case WQ_ERR_NOT_QUANTIZABLE: return "power-of-two block d & -d is below 32";
        case WQ_ERR_CUDA: return "CUDA launch error";
        default: return "unknown status";
    }
}

extern "C" int wq_version(void) { return (0 << 16) | 1; }
