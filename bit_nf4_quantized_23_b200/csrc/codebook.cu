// Host construction of the code values (NF4, and the uniform 4-bit grid it is
// compared with) and the quantize kernel's decision thresholds.
//
// The code values are normal quantiles ("Science Depth M5-131: PEFT (LoRA /
// QLoRA / Prefix Tuning)", section 3, NF4): 16 points with equal probability
// mass per bin, zero represented exactly and the end points at -1 and +1.  The
// printed formula q_i = (Phi^-1(i/16) + Phi^-1((i+1)/16)) / 2 has infinite end
// points, so the asymmetric construction is used: 8 positive quantiles at
// probabilities evenly spaced from delta towards 1/2, 7 negative ones, and 0,
// with delta = ((1 - 1/30) + (1 - 1/32)) / 2; all divided by the largest.
//
// Phi^-1 here: the rational approximation 26.2.23 of Abramowitz & Stegun
// (Handbook of Mathematical Functions) as a starting point, refined by Newton
// steps on Phi(x) = erfc(-x / sqrt(2)) / 2 until the step vanishes.
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "qlora_internal.cuh"

namespace qlora {
namespace {

double normal_cdf(double x) { return 0.5 * std::erfc(-x / std::sqrt(2.0)); }

double normal_pdf(double x) {
    const double inv_sqrt_2pi = 0.398942280401432677939946059934;
    return inv_sqrt_2pi * std::exp(-0.5 * x * x);
}

double normal_quantile(double p) {
    // A&S 26.2.23 for the upper tail probability pt = min(p, 1-p).
    const double pt = p < 0.5 ? p : 1.0 - p;
    const double t = std::sqrt(-2.0 * std::log(pt));
    const double c0 = 2.515517, c1 = 0.802853, c2 = 0.010328;
    const double d1 = 1.432788, d2 = 0.189269, d3 = 0.001308;
    double x = t - (c0 + c1 * t + c2 * t * t) / (1.0 + d1 * t + d2 * t * t + d3 * t * t * t);
    if (p < 0.5) x = -x;
    for (int it = 0; it < 50; ++it) {
        const double step = (normal_cdf(x) - p) / normal_pdf(x);
        const double nx = x - step;
        if (nx == x) break;
        x = nx;
    }
    return x;
}

NF4Tables build_tables(int codebook) {
    double v[16];
    double top = 1.0;
    if (codebook == QLORA_CODEBOOK_UNIFORM4) {
        // 16 evenly spaced values on [-1, 1]: i * (2/15) - 1 in double, the last exactly 1
        const double step = 2.0 / 15.0;
        for (int i = 0; i < 15; ++i) v[i] = (double)i * step + (-1.0);
        v[15] = 1.0;
    } else {
        const double delta = 0.5 * ((1.0 - 1.0 / 30.0) + (1.0 - 1.0 / 32.0));
        int n = 0;
        for (int j = 0; j < 8; ++j) v[n++] = normal_quantile(delta - j * (delta - 0.5) / 8.0);
        for (int j = 0; j < 7; ++j) v[n++] = -normal_quantile(delta - j * (delta - 0.5) / 7.0);
        v[n++] = 0.0;
        // insertion sort, ascending
        for (int i = 1; i < 16; ++i) {
            double key = v[i];
            int j = i - 1;
            while (j >= 0 && v[j] > key) { v[j + 1] = v[j]; --j; }
            v[j + 1] = key;
        }
        top = v[0];
        for (int i = 1; i < 16; ++i) top = v[i] > top ? v[i] : top;
    }
    NF4Tables tb;
    for (int i = 0; i < 16; ++i) tb.q[i] = (float)(v[i] / top);
    for (int j = 0; j < 15; ++j) {
        // exact midpoint in double (sum of two floats of similar magnitude), rounded down to float
        const double mid = ((double)tb.q[j] + (double)tb.q[j + 1]) / 2.0;
        float t = (float)mid;
        if ((double)t > mid) t = std::nextafter(t, -INFINITY);
        tb.t[j] = t;
    }
    return tb;
}

// Bucket table of the quantize kernel (see QuantBuckets).  bucket(x) =
// RNE(64 x + 64) is monotone in x, so a threshold in a lower bucket lies below
// every x of bucket k and one in a higher bucket above it.
int bucket_of(double x) { return (int)std::nearbyint(64.0 * x + 64.0); }   // default mode: ties to even

QuantBuckets build_buckets(const NF4Tables& tb) {
    QuantBuckets qb;
    for (int k = 0; k < kCodeBuckets; ++k) {
        int base = 0, inside = 0;
        float thr = INFINITY;
        for (int j = 0; j < 15; ++j) {
            const int b = bucket_of((double)tb.t[j]);
            if (b < k) ++base;
            else if (b == k) { thr = tb.t[j]; ++inside; }
        }
        if (inside > 1) std::abort();             // bucket narrower than every threshold gap
        int32_t bb = base;
        float bf;
        std::memcpy(&bf, &bb, 4);
        qb.e[k] = make_float2(thr, bf);
    }
    return qb;
}

}  // namespace

const QuantBuckets& host_buckets(int codebook) {
    static std::once_flag once[2];
    static QuantBuckets qb[2];
    const int c = codebook == QLORA_CODEBOOK_UNIFORM4 ? 1 : 0;
    std::call_once(once[c], [c] { qb[c] = build_buckets(host_tables(c)); });
    return qb[c];
}

const NF4Tables& host_tables(int codebook) {
    static std::once_flag once[2];
    static NF4Tables tables[2];
    const int c = codebook == QLORA_CODEBOOK_UNIFORM4 ? 1 : 0;
    std::call_once(once[c], [c] { tables[c] = build_tables(c); });
    return tables[c];
}

}  // namespace qlora
