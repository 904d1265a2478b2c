// Host-side generators of the TurboQuant library: the seeded random stream,
// the rotation / projection matrices and the Lloyd-Max codebook.
//
// Written from the method's description, not from any listing:
//  * "TurboQuant+ upstream guide", sec. 3 (Codex finding 6): the rotation is
//    generated deterministically from a seed -- QR of a Gaussian matrix gives
//    a Haar orthogonal matrix, with det forced to +1 -- instead of a static
//    table; sec. 4: the structured alternative D1 @ H @ D2.
//  * same guide, sec. 1.2 / 5.2: a Lloyd-Max codebook ("centroid table").
//
// The stream is SplitMix64 (Steele, Lea, Flood 2014); normals are
// Box-Muller pairs.  The codebook density is that of one coordinate of a
// uniform point on S^(block-1).  Integrals use the substitution x = sin(th):
// the mass of (a, b] is the integral of cos^(block-2) over (asin a, asin b],
// evaluated with the standard cosine-power reduction formula; the first
// moment has the closed form -(1 - x^2)^((block-1)/2) / (block - 1).

#include <cmath>
#include <cstdio>
#include <cstring>
#include <limits>
#include <string>
#include <vector>

#include "tq_internal.h"

namespace tq {

namespace {
thread_local std::string g_last_error;

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

bool is_pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }

// Householder QR of the n x n row-major matrix `a` (overwritten).  Returns the
// explicit orthogonal factor in `q` (row-major) and the diagonal of R.
void householder_qr(int n, std::vector<double> & a, std::vector<double> & q,
                    std::vector<double> & rdiag) {
    std::vector<double> v(n);
    std::vector<std::vector<double>> vs;
    std::vector<double> betas;
    rdiag.assign(n, 0.0);
    for (int k = 0; k < n; ++k) {
        double norm = 0.0;
        for (int i = k; i < n; ++i) norm += a[(size_t)i * n + k] * a[(size_t)i * n + k];
        norm = std::sqrt(norm);
        double x0 = a[(size_t)k * n + k];
        double alpha = (x0 >= 0.0) ? -norm : norm;  // avoid cancellation
        std::vector<double> vk(n, 0.0);
        vk[k] = x0 - alpha;
        for (int i = k + 1; i < n; ++i) vk[i] = a[(size_t)i * n + k];
        double vnorm2 = 0.0;
        for (int i = k; i < n; ++i) vnorm2 += vk[i] * vk[i];
        double beta = (vnorm2 > 0.0) ? 2.0 / vnorm2 : 0.0;
        // apply H = I - beta v v^T to columns k..n-1
        for (int j = k; j < n; ++j) {
            double s = 0.0;
            for (int i = k; i < n; ++i) s += vk[i] * a[(size_t)i * n + j];
            s *= beta;
            for (int i = k; i < n; ++i) a[(size_t)i * n + j] -= s * vk[i];
        }
        rdiag[k] = a[(size_t)k * n + k];
        vs.push_back(vk);
        betas.push_back(beta);
    }
    // Q = H_0 H_1 ... H_{n-1}: apply the reflections to the identity in reverse
    q.assign((size_t)n * n, 0.0);
    for (int i = 0; i < n; ++i) q[(size_t)i * n + i] = 1.0;
    for (int k = n - 1; k >= 0; --k) {
        const std::vector<double> & vk = vs[k];
        double beta = betas[k];
        if (beta == 0.0) continue;
        for (int j = 0; j < n; ++j) {
            double s = 0.0;
            for (int i = k; i < n; ++i) s += vk[i] * q[(size_t)i * n + j];
            s *= beta;
            for (int i = k; i < n; ++i) q[(size_t)i * n + j] -= s * vk[i];
        }
    }
}

// Sign of the determinant of an n x n row-major matrix (LU, partial pivoting).
int det_sign(int n, std::vector<double> m) {
    int sign = 1;
    for (int k = 0; k < n; ++k) {
        int p = k;
        double best = std::fabs(m[(size_t)k * n + k]);
        for (int i = k + 1; i < n; ++i) {
            double v = std::fabs(m[(size_t)i * n + k]);
            if (v > best) { best = v; p = i; }
        }
        if (best == 0.0) return 0;
        if (p != k) {
            for (int j = 0; j < n; ++j) std::swap(m[(size_t)k * n + j], m[(size_t)p * n + j]);
            sign = -sign;
        }
        double piv = m[(size_t)k * n + k];
        if (piv < 0) sign = -sign;
        for (int i = k + 1; i < n; ++i) {
            double f = m[(size_t)i * n + k] / piv;
            if (f == 0.0) continue;
            for (int j = k; j < n; ++j) m[(size_t)i * n + j] -= f * m[(size_t)k * n + j];
        }
    }
    return sign;
}

// Integral of cos^p over [0, th], |th| <= pi/2, by the reduction formula
// I_k = cos^(k-1) sin / k + (k-1)/k I_(k-2), with I_0 = th and I_1 = sin th.
double cos_power_integral(int p, double th) {
    const double s = std::sin(th), c = std::cos(th);
    double integral = (p & 1) ? s : th;
    double cpow = (p & 1) ? c * c : c;   // cos^(k-1) for the first k of the chain
    for (int k = (p & 1) ? 3 : 2; k <= p; k += 2) {
        integral = cpow * s / k + (double)(k - 1) / k * integral;
        cpow *= c * c;
    }
    return integral;
}

}  // namespace

tq_status fail(tq_status s, const std::string & why) {
    g_last_error = why;
    return s;
}

const char * last_error_cstr() { return g_last_error.c_str(); }

void splitmix64_fill(uint64_t seed, uint64_t * out, int64_t n) {
    uint64_t state = seed;
    for (int64_t i = 0; i < n; ++i) {
        state += kGamma;
        out[i] = mix64(state);
    }
}

void signs_fill(uint64_t seed, double * out, int64_t n) {
    std::vector<uint64_t> z((size_t)n);
    splitmix64_fill(seed, z.data(), n);
    for (int64_t i = 0; i < n; ++i) out[i] = (z[i] >> 63) ? -1.0 : 1.0;
}

void gaussians_fill(uint64_t seed, double * out, int64_t n) {
    int64_t pairs = (n + 1) / 2;
    std::vector<uint64_t> z((size_t)(2 * pairs));
    splitmix64_fill(seed, z.data(), 2 * pairs);
    const double two_pi = 6.283185307179586476925286766559;
    for (int64_t k = 0; k < pairs; ++k) {
        double u1 = 1.0 - (double)(z[2 * k] >> 11) * 0x1.0p-53;
        double u2 = (double)(z[2 * k + 1] >> 11) * 0x1.0p-53;
        double r = std::sqrt(-2.0 * std::log(u1));
        double g0 = r * std::cos(two_pi * u2);
        double g1 = r * std::sin(two_pi * u2);
        out[2 * k] = g0;
        if (2 * k + 1 < n) out[2 * k + 1] = g1;
    }
}

bool generate_matrix(int32_t kind, int32_t rows, int32_t cols, uint64_t seed, double * out,
                     std::string * why) {
    if (kind == TQ_ROT_WHT) {
        if (rows != cols || !is_pow2(rows) || rows > 4096) {
            *why = "WHT rotation needs rows == cols, a power of two <= 4096";
            return false;
        }
        int d = rows;
        std::vector<double> s((size_t)2 * d);
        signs_fill(seed, s.data(), 2 * d);
        double scale = 1.0 / std::sqrt((double)d);
        for (int i = 0; i < d; ++i)
            for (int j = 0; j < d; ++j) {
                double h = (__builtin_popcount((unsigned)(i & j)) & 1) ? -1.0 : 1.0;
                out[(size_t)i * d + j] = scale * s[i] * h * s[d + j];
            }
        return true;
    }
    if (kind == TQ_ROT_HAAR) {
        if (rows != cols || rows < 1 || rows > 1024) {
            *why = "Haar rotation needs rows == cols in [1, 1024]";
            return false;
        }
        int d = rows;
        std::vector<double> g((size_t)d * d), q, rdiag;
        gaussians_fill(seed, g.data(), (int64_t)d * d);
        householder_qr(d, g, q, rdiag);
        for (int j = 0; j < d; ++j) {
            double sgn = (rdiag[j] < 0.0) ? -1.0 : 1.0;
            for (int i = 0; i < d; ++i) q[(size_t)i * d + j] *= sgn;
        }
        if (det_sign(d, q) < 0)
            for (int i = 0; i < d; ++i) q[(size_t)i * d] = -q[(size_t)i * d];
        std::memcpy(out, q.data(), sizeof(double) * (size_t)d * d);
        return true;
    }
    if (kind == TQ_ROT_GAUSS) {
        if (rows < 1 || cols < 1 || (int64_t)rows * cols > (1 << 24)) {
            *why = "Gaussian projection needs 1 <= rows*cols <= 2^24";
            return false;
        }
        gaussians_fill(seed, out, (int64_t)rows * cols);
        return true;
    }
    *why = "unknown rotation kind";
    return false;
}

bool lloyd_max(int32_t bits, int32_t block, std::vector<double> * centroids,
               std::string * why) {
    if (bits < 1 || bits > 4) { *why = "bits must be in [1, 4]"; return false; }
    if (block < 3 || block > 4096) { *why = "block must be in [3, 4096]"; return false; }
    const int p = block - 2;                       // cos power after x = sin(th)
    const double half_pi = 1.5707963267948966192313216916398;
    const double total = 2.0 * cos_power_integral(p, half_pi);  // B(1/2, (block-1)/2)
    const double e = 0.5 * (block - 1);            // exponent of the first-moment closed form
    auto cdf_raw = [&](double x) {                 // integral of f from 0 to x, unnormalised
        if (x >= 1.0) return 0.5 * total;
        if (x <= -1.0) return -0.5 * total;
        return cos_power_integral(p, std::asin(x));
    };
    auto moment_raw = [&](double x) {              // antiderivative of x f(x), unnormalised
        double s = 1.0 - x * x;
        if (s < 0.0) s = 0.0;
        return -std::pow(s, e) / (block - 1);
    };
    const int n = 1 << bits;
    std::vector<double> c(n), t(n + 1);
    // start: evenly spaced over +-2.5 standard deviations, kept inside (-1, 1)
    // so that every cell has mass (the fixed point is unique)
    const double spread = std::fmin(0.9, 2.5 / std::sqrt((double)block));
    for (int i = 0; i < n; ++i) c[i] = spread * (2.0 * i + 1.0 - n) / n;
    for (int it = 0; it < 1000000; ++it) {
        t[0] = -1.0;
        t[n] = 1.0;
        for (int i = 1; i < n; ++i) t[i] = 0.5 * (c[i - 1] + c[i]);
        double moved = 0.0;
        for (int i = 0; i < n; ++i) {
            double mass = cdf_raw(t[i + 1]) - cdf_raw(t[i]);
            double mom = moment_raw(t[i + 1]) - moment_raw(t[i]);
            double ci = mom / mass;
            moved = std::fmax(moved, std::fabs(ci - c[i]));
            c[i] = ci;
        }
        if (moved < 1e-14) {
            // enforce exact symmetry of the fixed point
            for (int i = 0; i < n / 2; ++i) {
                double m = 0.5 * (c[n - 1 - i] - c[i]);
                c[i] = -m;
                c[n - 1 - i] = m;
            }
            *centroids = c;
            return true;
        }
    }
    *why = "Lloyd-Max iteration did not converge";
    return false;
}

bool build_search_table(int bits, const float * boundaries, SearchTable * out, std::string * why) {
    const int nt = (1 << bits) - 1;
    double gap = 2.0;
    for (int i = 0; i + 1 < nt; ++i) gap = std::fmin(gap, (double)boundaries[i + 1] - boundaries[i]);
    int k = 0;
    while (std::ldexp(1.0, -k) >= gap) ++k;
    const double w = std::ldexp(1.0, -k);
    const int half_cells = (int)(1.0 / w);
    const int K = half_cells + 1;              // u = 0 falls in cell K; u = -1 in cell 1
    const int top = 2 * half_cells + 2;        // u >= 1 + w/2
    uint32_t size = 1;
    while (size < (uint32_t)top + 1) size <<= 1;
    if (size > (uint32_t)kSearchMax) {
        *why = "codebook boundaries too close for the search table";
        return false;
    }
    // The kernels form y = fmaf(u, 128 / w, 2^23 + 128 K + 64): one rounding
    // to an integer (the offset keeps y in [2^23, 2^24)), so the fp32 bits of
    // y are 0x4B000000 + RN(128 (u / w + K) + 64) and bits & ((size - 1) << 7)
    // is 128 * cell -- the byte offset of the cell's entry in a table of
    // 128-byte rows.  RN(v) lands in [128 c, 128 c + 128) exactly when
    // v in [128 c - 1/2, 128 c + 127.5) (ties go to the even 128 c), so cell c
    // holds u in [(c - K - 1/2 - 1/256) w, (c - K + 1/2 - 1/256) w).
    out->scale = (float)(128.0 / w);                     // power of two: exact
    out->offset = (float)(8388608.0 + 128.0 * K + 64.0); // integer below 2^24: exact
    out->mask = (size - 1) << 7;
    out->size = size;
    const float inf = std::numeric_limits<float>::infinity();
    for (int c = 0; c < kSearchMax; ++c) {
        out->t[c] = inf;
        out->base[c] = 0;
    }
    out->base[top] = nt;
    for (int c = 1; c < top; ++c) {
        const double lo = (c - K - 0.5 - 1.0 / 256.0) * w, hi = lo + w;
        int base = 0, inside = 0;
        float tin = inf;
        for (int i = 0; i < nt; ++i) {
            const double ti = boundaries[i];
            if (ti <= lo) ++base;
            else if (ti < hi) { ++inside; tin = boundaries[i]; }
        }
        if (inside > 1) {
            *why = "search table cell holds two boundaries";
            return false;
        }
        out->t[c] = tin;
        out->base[c] = base;
    }
    return true;
}

int32_t decode_splits(int32_t batch, int32_t n_q_heads, int32_t n_kv_heads, int64_t ctx,
                      int32_t head_dim) {
    // CTAs of the split kernel: batch * kv heads * ceil(G / 4) units per split.
    // Pick the split count that fills whole waves of two resident CTAs per SM
    // best, with at least 256 tokens per split and the partials of all splits
    // within 4 MiB; ties go to the smaller count.
    const int64_t group = n_q_heads / (n_kv_heads > 0 ? n_kv_heads : 1);
    const int64_t units = (int64_t)batch * n_kv_heads * ((group + 3) / 4);
    const int64_t slots = 2LL * device_sm_count();
    const int64_t per_split = (int64_t)batch * n_q_heads * (head_dim + 2) * 4;
    int64_t s_max = ctx / 256;
    if (s_max > 64) s_max = 64;
    const int64_t by_ws = per_split > 0 ? (int64_t)(4u << 20) / per_split : 64;
    if (s_max > by_ws) s_max = by_ws;
    if (s_max < 1) s_max = 1;
    int64_t best = 1;
    double best_eff = -1.0;
    for (int64_t sp = 1; sp <= s_max; ++sp) {
        const int64_t ctas = units * sp;
        const int64_t waves = (ctas + slots - 1) / slots;
        const double eff = (double)ctas / (double)(waves * slots);
        if (eff > best_eff + 1e-9) { best_eff = eff; best = sp; }
    }
    return (int32_t)best;
}

}  // namespace tq

// ---------------------------------------------------------------------------
// Host-only C entry points.

extern "C" {

const char * tq_status_string(tq_status s) {
    switch (s) {
        case TQ_OK: return "ok";
        case TQ_ERR_INVALID_ARG: return "invalid argument";
        case TQ_ERR_UNSUPPORTED: return "unsupported configuration";
        case TQ_ERR_CUDA: return "CUDA error";
        case TQ_ERR_ALLOC: return "allocation failed";
    }
    return "unknown status";
}

const char * tq_last_error(void) { return tq::last_error_cstr(); }

tq_status tq_rotation_generate(tq_rot_kind kind, int32_t rows, int32_t cols, uint64_t seed,
                               double * out) {
    if (!out) return tq::fail(TQ_ERR_INVALID_ARG, "out is NULL");
    std::string why;
    if (!tq::generate_matrix((int32_t)kind, rows, cols, seed, out, &why))
        return tq::fail(TQ_ERR_INVALID_ARG, why);
    return TQ_OK;
}

namespace {

// Nearest binary16 value of x (ties to even), returned as a double; |x| is
// far below the fp16 range here, so only the normal / subnormal spacing
// matters: ulp = 2^(e - 10) for x in [2^e, 2^(e+1)), e >= -14, else 2^-24.
double round_to_half(double x) {
    if (x == 0.0 || !std::isfinite(x)) return x;
    int e2 = 0;
    std::frexp(std::fabs(x), &e2);           // |x| in [2^(e2-1), 2^e2)
    int e = e2 - 1;
    if (e < -14) e = -14;
    const double ulp = std::ldexp(1.0, e - 10);
    return std::copysign(std::nearbyint(std::fabs(x) / ulp) * ulp, x);
}

}  // namespace

tq_status tq_build_codebook(int32_t bits, int32_t block, float * centroids, float * boundaries) {
    if (!centroids || !boundaries) return tq::fail(TQ_ERR_INVALID_ARG, "null output pointer");
    std::vector<double> c;
    std::string why;
    if (!tq::lloyd_max(bits, block, &c, &why)) return tq::fail(TQ_ERR_INVALID_ARG, why);
    int n = 1 << bits;
    // reconstruction points are stored at fp16 precision (exact in fp32);
    // the decision boundaries stay the midpoints of the float64 fixed point
    for (int i = 0; i < n; ++i) centroids[i] = (float)round_to_half(c[i]);
    for (int i = 0; i + 1 < n; ++i) boundaries[i] = (float)(0.5 * (c[i] + c[i + 1]));
    return TQ_OK;
}

int64_t tq_code_words_per_row(int32_t bits, int32_t block, int32_t head_dim) {
    if (bits < 1 || block < 1 || head_dim < block || head_dim % block || (bits * block) % 32)
        return -1;
    return (int64_t)(head_dim / block) * (bits * block / 32);
}

}  // extern "C"
