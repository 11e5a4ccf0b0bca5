// Design-time codebook: Lloyd-Max scalar quantizer of N(0, 1/d) at b bits.
//
// AXELRAM (arXiv 2604.02638), abstract: after the orthogonal transform every
// coordinate of a unit key is close to N(0, 1/d), so the best scalar quantizer is
// fixed at design time by (d, b).  The paper's repository names a Lloyd-Max
// solver for it (codebook.py: target pdf, conditional mean, solve_lloyd_max).
//
// This solver works on the positive half-line only: the normal density is
// symmetric and log-concave, so the optimal quantizer with an even number of
// levels is symmetric, has a boundary at 0, and is the unique fixed point of the
// Lloyd-Max conditions.  With m = 2^(b-1) positive centroids p_0 < ... < p_{m-1}:
//   cell i = (tau_{i-1}, tau_i], tau_{-1} = 0, tau_{m-1} = +inf,
//   tau_i  = (p_i + p_{i+1}) / 2                       (nearest-neighbour rule)
//   p_i    = E[X | X in cell i]
//          = (phi(lo) - phi(hi)) / (Q(lo) - Q(hi))      (centroid rule)
// with phi the standard normal density and Q its upper tail.  The iteration runs
// in long double until no centroid moves by more than 1e-18; the N(0,1) result
// is scaled by 1/sqrt(d) and rounded to fp32.
#include <cmath>
#include <map>
#include <mutex>
#include <utility>

#include "axr_internal.cuh"

namespace axr {
namespace {

using real = long double;

real normal_pdf(real x)
{
    if (std::isinf(x)) return 0.0L;
    static const real inv_sqrt_2pi = 1.0L / std::sqrt(2.0L * 3.141592653589793238462643383279502884L);
    return inv_sqrt_2pi * std::exp(-0.5L * x * x);
}

// upper tail P(X > x), x >= 0
real normal_upper_tail(real x)
{
    if (std::isinf(x)) return 0.0L;
    return 0.5L * std::erfc(x / std::sqrt(2.0L));
}

void solve_positive_half(int b, real *p)
{
    const int m = 1 << (b - 1);
    // start: evenly spaced on (0, 3)
    for (int i = 0; i < m; ++i) p[i] = 3.0L * (i + 0.5L) / m;
    real next[kMaxLevels];
    for (int it = 0; it < 1000000; ++it) {
        real moved = 0.0L;
        for (int i = 0; i < m; ++i) {
            const real lo = (i == 0) ? 0.0L : 0.5L * (p[i - 1] + p[i]);
            const real hi = (i == m - 1) ? INFINITY : 0.5L * (p[i] + p[i + 1]);
            next[i] = (normal_pdf(lo) - normal_pdf(hi)) / (normal_upper_tail(lo) - normal_upper_tail(hi));
            moved = std::fmax(moved, std::fabs(next[i] - p[i]));
        }
        for (int i = 0; i < m; ++i) p[i] = next[i];
        if (moved <= 1e-18L) break;
    }
}

bool supported(int d, int b)
{
    return d >= 8 && d <= 512 && (d & (d - 1)) == 0 && b >= 1 && b <= kMaxBits;
}

Codebook build(int d, int b)
{
    Codebook cb;
    cb.d = d;
    cb.b = b;
    const int L = 1 << b;
    const int m = L / 2;
    real p[kMaxLevels];
    solve_positive_half(b, p);
    const real sigma = 1.0L / std::sqrt(static_cast<real>(d));
    for (int i = 0; i < m; ++i) {
        const float v = static_cast<float>(p[i] * sigma);
        cb.centroids[m + i] = v;
        cb.centroids[m - 1 - i] = -v;
    }
    for (int i = 0; i + 1 < L; ++i)
        cb.boundaries[i] = static_cast<float>(
            0.5 * (static_cast<double>(cb.centroids[i]) + static_cast<double>(cb.centroids[i + 1])));
    return cb;
}

// Bucket width in sigma units: below the smallest gap between neighbouring
// boundaries (0.258 sigma at b = 4), so no bucket holds two of them; the first
// width whose boundaries all keep `kMinMargin` from the bucket edges is used.
constexpr float kWidths[] = {0.25f, 0.24f, 0.23f, 0.22f, 0.21f, 0.2f, 0.19f, 0.18f};
constexpr float kMinMargin = 0.05f;

bool build_table(const Codebook &cb, BucketTable *t)
{
    const int L = 1 << cb.b;
    const float sqrt_d = std::sqrt(static_cast<float>(cb.d));
    for (float h : kWidths) {
        BucketTable tab;
        tab.d = cb.d;
        tab.b = cb.b;
        tab.g_scale = sqrt_d / h;
        // |u| <= 1, so g stays within g_off +- g_scale (+ rounding)
        int nt = 1;
        while (nt < 2 * static_cast<int>(std::ceil(tab.g_scale)) + 8) nt *= 2;
        if (nt > kMaxBuckets) continue;
        tab.nt = nt;
        tab.g_off = static_cast<float>(nt / 2);
        float tg[kMaxLevels];
        float margin = 1.0f;
        bool ok = true;
        for (int i = 0; i + 1 < L; ++i) {
            tg[i] = std::fma(cb.boundaries[i], tab.g_scale, tab.g_off);
            const float frac = tg[i] - std::floor(tg[i]);
            margin = std::fmin(margin, std::fabs(frac - 0.5f));
            if (i > 0 && std::floor(tg[i] + 0.5f) == std::floor(tg[i - 1] + 0.5f)) ok = false;
        }
        if (!ok || margin < kMinMargin) continue;
        tab.margin = margin;
        for (int j = 0; j < nt; ++j) {
            tab.tau[j] = INFINITY;
            int below = 0;
            for (int i = 0; i + 1 < L; ++i) {
                if (tg[i] < j - 0.5f) ++below;
                else if (tg[i] < j + 0.5f) tab.tau[j] = tg[i];
            }
            tab.base[j] = below;
        }
        for (int j = nt; j < kMaxBuckets; ++j) {
            tab.tau[j] = INFINITY;
            tab.base[j] = L - 1;
        }
        *t = tab;
        return true;
    }
    return false;
}

}  // namespace

bool get_bucket_table(int d, int b, BucketTable *out)
{
    Codebook cb;
    if (!out || !get_codebook(d, b, &cb)) return false;
    static std::mutex mu;
    static std::map<std::pair<int, int>, BucketTable> cache;
    std::lock_guard<std::mutex> lock(mu);
    auto key = std::make_pair(d, b);
    auto it = cache.find(key);
    if (it == cache.end()) {
        BucketTable t;
        if (!build_table(cb, &t)) return false;
        it = cache.emplace(key, t).first;
    }
    *out = it->second;
    return true;
}

bool get_codebook(int d, int b, Codebook *out)
{
    if (!supported(d, b) || !out) return false;
    static std::mutex mu;
    static std::map<std::pair<int, int>, Codebook> cache;
    std::lock_guard<std::mutex> lock(mu);
    auto key = std::make_pair(d, b);
    auto it = cache.find(key);
    if (it == cache.end()) it = cache.emplace(key, build(d, b)).first;
    *out = it->second;
    return true;
}

}  // namespace axr
