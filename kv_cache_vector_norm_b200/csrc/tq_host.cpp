// Host-side parameter builders of libtq: the seeded Haar (or Walsh-Hadamard) rotation and the Lloyd-Max
// codebook.
//
// Rotation: "KV Cache API" (TurboQuant docs), compressors.py MSECompressor.__init__ -- a Gaussian d x d
// matrix G, its QR factorisation, Pi = Q * sign(diag R).  The Gaussian draws come from SplitMix64
// (Steele, Lea & Flood 2014) through the Box-Muller transform, both from their published definitions.
//
// Codebook: the page calls _solve_codebook(head_dim, bits) without showing it; "TurboQuant: A KV Cache
// Compression Technique" says the codebooks are Lloyd-Max levels pre-computed from a mathematical
// derivation.  Here the density of one rotated coordinate is the exact sphere marginal
// f(x) = (1 - x^2)^((d-3)/2) / B(1/2, (d-1)/2) on [-1, 1], and each Lloyd step integrates it with
// composite Gauss-Legendre quadrature (first moments in closed form).
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "tq_internal.h"

namespace tq {

static thread_local std::string g_last_error;

tq_status fail(tq_status status, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return status;
}

void clear_error() { g_last_error.clear(); }

// ----------------------------------------------------------------------------------- random numbers

static inline uint64_t splitmix64_at(uint64_t seed, uint64_t i) {
    // output i (0-based) of SplitMix64 seeded with `seed`: the state after i+1 golden-ratio increments,
    // passed through the two xor-shift-multiply rounds
    uint64_t z = seed + (i + 1) * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

void host_gaussians(uint64_t seed, size_t count, double* out) {
    const double two_pi = 6.283185307179586476925286766559;
    for (size_t p = 0; 2 * p < count; ++p) {
        double u1 = (static_cast<double>(splitmix64_at(seed, 2 * p) >> 11) + 0.5) * 0x1.0p-53;
        double u2 = static_cast<double>(splitmix64_at(seed, 2 * p + 1) >> 11) * 0x1.0p-53;
        double r = std::sqrt(-2.0 * std::log(u1));
        out[2 * p] = r * std::cos(two_pi * u2);
        if (2 * p + 1 < count) out[2 * p + 1] = r * std::sin(two_pi * u2);
    }
}

// ------------------------------------------------------------------------------------------ rotation

void host_rotation(int d, uint64_t seed, double* pi) {
    const size_t n = static_cast<size_t>(d);
    std::vector<double> a(n * n), vs(n * n, 0.0);   // a: working matrix (row-major); vs: reflectors
    host_gaussians(seed, n * n, a.data());
    std::vector<double> rdiag(n);
    // Householder QR: for column k, reflect a[k:, k] onto a multiple of e_k.
    for (size_t k = 0; k < n; ++k) {
        double norm2 = 0.0;
        for (size_t i = k; i < n; ++i) norm2 += a[i * n + k] * a[i * n + k];
        double norm = std::sqrt(norm2);
        double x0 = a[k * n + k];
        double alpha = (x0 >= 0.0) ? -norm : norm;      // avoids cancellation in v_0
        double* v = &vs[k * n];
        for (size_t i = k; i < n; ++i) v[i] = a[i * n + k];
        v[k] -= alpha;
        double vnorm2 = 0.0;
        for (size_t i = k; i < n; ++i) vnorm2 += v[i] * v[i];
        if (vnorm2 > 0.0) {
            double inv = 1.0 / std::sqrt(vnorm2);
            for (size_t i = k; i < n; ++i) v[i] *= inv;
            for (size_t j = k; j < n; ++j) {             // a[k:, j] -= 2 v (v . a[k:, j])
                double dot = 0.0;
                for (size_t i = k; i < n; ++i) dot += v[i] * a[i * n + j];
                for (size_t i = k; i < n; ++i) a[i * n + j] -= 2.0 * dot * v[i];
            }
        }
        rdiag[k] = a[k * n + k];
    }
    // Q = H_0 H_1 ... H_{n-1} I, accumulated right to left.
    std::vector<double> q(n * n, 0.0);
    for (size_t i = 0; i < n; ++i) q[i * n + i] = 1.0;
    for (size_t kk = n; kk-- > 0;) {
        const double* v = &vs[kk * n];
        for (size_t j = 0; j < n; ++j) {
            double dot = 0.0;
            for (size_t i = kk; i < n; ++i) dot += v[i] * q[i * n + j];
            if (dot != 0.0)
                for (size_t i = kk; i < n; ++i) q[i * n + j] -= 2.0 * dot * v[i];
        }
    }
    // Pi = Q diag(sign(R_jj)), sign(0) := +1
    for (size_t i = 0; i < n; ++i)
        for (size_t j = 0; j < n; ++j) pi[i * n + j] = (rdiag[j] < 0.0 ? -1.0 : 1.0) * q[i * n + j];
}

// "turbo-attn", The codec, "Hadamard rotation": a Walsh-Hadamard transform spreads outlier channels over the
// vector; queries are rotated the same way.  H by Sylvester's doubling (H_1 = [1], H_2m = [[H, H], [H, -H]]),
// i.e. H[i][j] = (-1)^popcount(i & j); columns scaled by the seeded signs and by 1/sqrt(d).
void host_hadamard(int d, uint64_t seed, double* pi) {
    const double inv = 1.0 / std::sqrt(static_cast<double>(d));
    for (int j = 0; j < d; ++j) {
        const double sj = (splitmix64_at(seed, static_cast<uint64_t>(j)) >> 63) ? -inv : inv;
        for (int i = 0; i < d; ++i) {
            const bool odd = __builtin_popcount(static_cast<unsigned>(i & j)) & 1;
            pi[static_cast<size_t>(i) * d + j] = odd ? -sj : sj;
        }
    }
}

bool host_rotation_of(int kind, int d, uint64_t seed, double* pi) {
    if (kind == TQ_ROT_HAAR) {
        host_rotation(d, seed, pi);
        return true;
    }
    if (kind == TQ_ROT_HADAMARD) {
        host_hadamard(d, seed, pi);
        return true;
    }
    return false;
}

// ------------------------------------------------------------------------------------------ codebook

namespace {

// Gauss-Legendre nodes/weights on [-1, 1] by Newton iteration on the three-term recurrence.
struct GaussLegendre {
    static constexpr int kN = 24;
    double x[kN], w[kN];
    GaussLegendre() {
        const double pi = 3.14159265358979323846264338327950288;
        for (int i = 0; i < kN; ++i) {
            double z = std::cos(pi * (i + 0.75) / (kN + 0.5));
            double dp = 1.0;
            for (int it = 0; it < 100; ++it) {
                double p0 = 1.0, p1 = z;
                for (int k = 2; k <= kN; ++k) {
                    double p2 = ((2.0 * k - 1.0) * z * p1 - (k - 1.0) * p0) / k;
                    p0 = p1;
                    p1 = p2;
                }
                dp = kN * (z * p1 - p0) / (z * z - 1.0);
                double dz = p1 / dp;
                z -= dz;
                if (std::fabs(dz) < 1e-17) break;
            }
            x[i] = z;
            w[i] = 2.0 / ((1.0 - z * z) * dp * dp);
        }
    }
};

const GaussLegendre& gl() {
    static const GaussLegendre g;
    return g;
}

struct Sphere {
    double a, log_norm;   // f(x) = exp(a log1p(-x^2) - log_norm)
    explicit Sphere(int d) {
        a = (d - 3) / 2.0;
        log_norm = std::lgamma(0.5) + std::lgamma(a + 1.0) - std::lgamma(a + 1.5);
    }
    double f(double x) const {
        if (x >= 1.0) return 0.0;
        return std::exp(a * std::log1p(-x * x) - log_norm);
    }
    // int_lo^hi x f = ((1-lo^2)^(a+1) - (1-hi^2)^(a+1)) / (2 (a+1)) / norm
    double m1(double lo, double hi) const {
        auto g = [&](double x) { return x >= 1.0 ? 0.0 : std::exp((a + 1.0) * std::log1p(-x * x) - log_norm); };
        return (g(lo) - g(hi)) / (2.0 * (a + 1.0));
    }
    // int_lo^hi x^p f(x) dx by composite Gauss-Legendre with panels sized to the density's spread
    double moment(double lo, double hi, int p, double spread) const {
        const GaussLegendre& q = gl();
        int panels = static_cast<int>(std::ceil((hi - lo) / (0.25 * spread)));
        if (panels < 4) panels = 4;
        if (panels > 4096) panels = 4096;
        double h = (hi - lo) / panels, sum = 0.0;
        for (int k = 0; k < panels; ++k) {
            double c = lo + (k + 0.5) * h, r = 0.5 * h, part = 0.0;
            for (int i = 0; i < GaussLegendre::kN; ++i) {
                double x = c + r * q.x[i];
                double v = f(x);
                if (p == 2) v *= x * x;
                part += q.w[i] * v;
            }
            sum += part * r;
        }
        return sum;
    }
};

}  // namespace

void host_codebook(int d, int bits, double* levels) {
    Sphere s(d);
    const int half = 1 << (bits - 1);
    const double spread = 1.0 / std::sqrt(static_cast<double>(d));
    // start: half-distribution quantiles (i + 1/2) / half, by bisection on the cumulative mass
    std::vector<double> c(half), t(half + 1);
    double total = s.moment(0.0, 1.0, 0, spread);
    for (int i = 0; i < half; ++i) {
        double target = (i + 0.5) / half * total, lo = 0.0, hi = 1.0;
        for (int it = 0; it < 100; ++it) {
            double mid = 0.5 * (lo + hi);
            (s.moment(0.0, mid, 0, spread) < target ? lo : hi) = mid;
        }
        c[i] = 0.5 * (lo + hi);
    }
    // Newton's method on the Lloyd fixed point c = g(c), g_i the centroid of cell i = [t_i, t_{i+1}] with
    // t_i = (c_{i-1} + c_i) / 2 (t_0 = 0, t_half = 1).  A centroid moves with its two boundaries,
    //   dg_i/dt_i = f(t_i) (g_i - t_i) / P_i,   dg_i/dt_{i+1} = f(t_{i+1}) (t_{i+1} - g_i) / P_i   (P_i the mass),
    // and each boundary with its two levels (1/2 each), so J = dg/dc is tridiagonal and each step solves
    // (J - I) dc = c - g(c) by the Thomas algorithm.  The plain iteration below converges linearly with a rate
    // near 1 - O(1 / half^2) (minutes at 8 bits); Newton's converges quadratically to the same fixed point.
    // A step that would break the ordering 0 < c_0 < ... < c_{half-1} < 1 is halved.
    bool newton_converged = false;
    {
        std::vector<double> g(half), lo_d(half), di(half), up(half), r(half), cp(half), dp(half), nc(half);
        double prev = INFINITY;
        for (int it = 0; it < 60; ++it) {
            t[0] = 0.0;
            t[half] = 1.0;
            for (int i = 1; i < half; ++i) t[i] = 0.5 * (c[i - 1] + c[i]);
            double rmax = 0.0, cmax = 0.0;
            for (int i = 0; i < half; ++i) {
                const double mass = s.moment(t[i], t[i + 1], 0, spread);
                g[i] = s.m1(t[i], t[i + 1]) / mass;
                const double a_lo = (i > 0) ? s.f(t[i]) * (g[i] - t[i]) / mass : 0.0;
                const double a_hi = (i < half - 1) ? s.f(t[i + 1]) * (t[i + 1] - g[i]) / mass : 0.0;
                lo_d[i] = 0.5 * a_lo;
                up[i] = 0.5 * a_hi;
                di[i] = 0.5 * (a_lo + a_hi) - 1.0;
                r[i] = c[i] - g[i];
                rmax = std::fmax(rmax, std::fabs(r[i]));
                cmax = std::fmax(cmax, std::fabs(c[i]));
            }
            // converged to the quadrature's noise floor (about 1e-15 relative): a further step cannot reduce it
            if (rmax <= 1e-13 * cmax) newton_converged = true;
            if (rmax <= 2e-16 * cmax || (newton_converged && rmax > 0.25 * prev)) break;
            prev = rmax;
            // Thomas algorithm for the tridiagonal system (lo_d, di, up) dc = r
            cp[0] = up[0] / di[0];
            dp[0] = r[0] / di[0];
            for (int i = 1; i < half; ++i) {
                const double m = di[i] - lo_d[i] * cp[i - 1];
                cp[i] = up[i] / m;
                dp[i] = (r[i] - lo_d[i] * dp[i - 1]) / m;
            }
            for (int i = half - 2; i >= 0; --i) dp[i] -= cp[i] * dp[i + 1];
            double lambda = 1.0;
            for (int tries = 0; tries < 40; ++tries, lambda *= 0.5) {
                bool ordered = true;
                for (int i = 0; i < half; ++i) {
                    nc[i] = c[i] + lambda * dp[i];
                    if (nc[i] <= (i ? nc[i - 1] : 0.0) || nc[i] >= 1.0) ordered = false;
                }
                if (ordered) break;
            }
            c.swap(nc);
        }
    }
    // Lloyd iteration on the positive half: boundaries = midpoints, levels = cell centroids.  After Newton's
    // solution it only polishes (at most 1000 steps, as the 2e-16 stop can lie below the quadrature's noise);
    // it is also the fallback, with the full iteration budget, if Newton's did not converge
    const int lloyd_iters = newton_converged ? 1000 : 200000;
    for (int it = 0; it < lloyd_iters; ++it) {
        t[0] = 0.0;
        t[half] = 1.0;
        for (int i = 1; i < half; ++i) t[i] = 0.5 * (c[i - 1] + c[i]);
        double step = 0.0, cmax = 0.0;
        for (int i = 0; i < half; ++i) {
            double nc = s.m1(t[i], t[i + 1]) / s.moment(t[i], t[i + 1], 0, spread);
            step = std::fmax(step, std::fabs(nc - c[i]));
            c[i] = nc;
            cmax = std::fmax(cmax, std::fabs(nc));
        }
        if (step <= 2e-16 * cmax) break;
    }
    for (int i = 0; i < half; ++i) {
        levels[half + i] = c[i];
        levels[half - 1 - i] = -c[i];
    }
}

double host_distortion(int d, int bits, const double* c, const double* t) {
    Sphere s(d);
    const int k = 1 << bits;
    const double spread = 1.0 / std::sqrt(static_cast<double>(d));
    double total = 0.0;
    // cells [e_i, e_{i+1}] with e_0 = -1, e_k = 1; integrate each cell piece on one side of 0 and use
    // the evenness of f (a piece [lo, hi] with hi <= 0 is mirrored to [-hi, -lo])
    for (int i = 0; i < k; ++i) {
        double lo = (i == 0) ? -1.0 : t[i - 1];
        double hi = (i == k - 1) ? 1.0 : t[i];
        double pieces[2][3];
        int np = 0;
        if (lo < 0.0) { pieces[np][0] = std::fmax(0.0, -hi); pieces[np][1] = -lo; pieces[np][2] = -1.0; ++np; }
        if (hi > 0.0) { pieces[np][0] = std::fmax(lo, 0.0); pieces[np][1] = hi; pieces[np][2] = 1.0; ++np; }
        for (int p = 0; p < np; ++p) {
            double a = pieces[p][0], b = pieces[p][1], sg = pieces[p][2];
            if (b <= a) continue;
            double m0 = s.moment(a, b, 0, spread), m1 = sg * s.m1(a, b), m2 = s.moment(a, b, 2, spread);
            total += m2 - 2.0 * c[i] * m1 + c[i] * c[i] * m0;
        }
    }
    return d * total;
}

// ---------------------------------------------------------------------------------- binary16 helpers

uint16_t f64_to_f16(double v) {
    // correctly rounded (nearest even) double -> binary16 via exact scaling
    uint16_t sign = std::signbit(v) ? 0x8000 : 0;
    double a = std::fabs(v);
    if (std::isnan(a)) return 0x7E00;
    if (a >= 65520.0) return sign | 0x7C00;                  // rounds to infinity
    if (a < 0x1.0p-14) {                                     // subnormal range: multiples of 2^-24
        double m = std::nearbyint(a * 0x1.0p24);             // FE_TONEAREST default
        return sign | static_cast<uint16_t>(m);
    }
    int e;
    double fr = std::frexp(a, &e);                           // a = fr * 2^e, fr in [0.5, 1)
    double m = std::nearbyint(fr * 2048.0);                  // 11 significant bits
    if (m >= 2048.0) { m = 1024.0; ++e; }
    int exp16 = e - 1 + 15;                                  // a = (m/1024) * 2^(e-1)
    if (exp16 >= 31) return sign | 0x7C00;
    return sign | static_cast<uint16_t>((exp16 << 10) | (static_cast<int>(m) - 1024));
}

double f16_to_f64(uint16_t h) {
    int e = (h >> 10) & 0x1F, m = h & 0x3FF;
    double v;
    if (e == 0) v = std::ldexp(static_cast<double>(m), -24);
    else if (e == 31) v = m ? NAN : INFINITY;
    else v = std::ldexp(static_cast<double>(m + 1024), e - 25);
    return (h & 0x8000) ? -v : v;
}

}  // namespace tq

// ------------------------------------------------------------------------------------- C entry points

extern "C" const char* tq_last_error(void) { return tq::g_last_error.c_str(); }

extern "C" int tq_version(void) { return 101; }

extern "C" tq_status tq_make_rotation_ex(int d, uint64_t seed, int rotation, double* pi, uint16_t* pi_f16) {
    tq::clear_error();
    if (d < 2 || d > 1024) return tq::fail(TQ_ERR_INVALID_ARG, "tq_make_rotation: d=%d outside [2, 1024]", d);
    if (!pi && !pi_f16) return tq::fail(TQ_ERR_INVALID_ARG, "tq_make_rotation: pi and pi_f16 are both NULL");
    if (rotation != TQ_ROT_HAAR && rotation != TQ_ROT_HADAMARD)
        return tq::fail(TQ_ERR_INVALID_ARG, "tq_make_rotation: rotation=%d (TQ_ROT_HAAR or TQ_ROT_HADAMARD)", rotation);
    if (rotation == TQ_ROT_HADAMARD && (d & (d - 1)))
        return tq::fail(TQ_ERR_INVALID_ARG, "tq_make_rotation: d=%d is not a power of two (Hadamard)", d);
    std::vector<double> m(static_cast<size_t>(d) * d);
    tq::host_rotation_of(rotation, d, seed, m.data());
    if (pi) std::memcpy(pi, m.data(), m.size() * sizeof(double));
    if (pi_f16)
        for (size_t i = 0; i < m.size(); ++i) pi_f16[i] = tq::f64_to_f16(m[i]);
    return TQ_OK;
}

extern "C" tq_status tq_make_qjl_matrix(int d, uint64_t seed, double* s, uint16_t* s_f16) {
    tq::clear_error();
    if (d < 1 || d > 4096) return tq::fail(TQ_ERR_INVALID_ARG, "tq_make_qjl_matrix: d=%d outside [1, 4096]", d);
    if (!s && !s_f16) return tq::fail(TQ_ERR_INVALID_ARG, "tq_make_qjl_matrix: both outputs are NULL");
    const size_t dd = static_cast<size_t>(d) * d;
    std::vector<double> g(dd);
    tq::host_gaussians(seed + 10000, dd, g.data());
    for (size_t i = 0; i < dd; ++i) {
        if (s) s[i] = g[i];
        if (s_f16) s_f16[i] = tq::f64_to_f16(g[i]);
    }
    return TQ_OK;
}

extern "C" tq_status tq_make_rotation(int d, uint64_t seed, double* pi, uint16_t* pi_f16) {
    return tq_make_rotation_ex(d, seed, TQ_ROT_HAAR, pi, pi_f16);
}

extern "C" tq_status tq_build_codebook(int d, int bits, double* centroids, uint16_t* centroids_f16,
                                       float* boundaries, double* distortion) {
    tq::clear_error();
    if (d < 2 || d > 65536) return tq::fail(TQ_ERR_INVALID_ARG, "tq_build_codebook: d=%d outside [2, 65536]", d);
    if (bits < 1 || bits > 8) return tq::fail(TQ_ERR_INVALID_ARG, "tq_build_codebook: bits=%d outside [1, 8]", bits);
    const int k = 1 << bits;
    std::vector<double> c(k), cop(k), t(k - 1);
    tq::host_codebook(d, bits, c.data());
    for (int i = 0; i < k; ++i) cop[i] = tq::f16_to_f64(tq::f64_to_f16(c[i]));
    for (int i = 0; i + 1 < k; ++i) t[i] = 0.5 * (cop[i] + cop[i + 1]);   // exact: few significant bits
    if (centroids) std::memcpy(centroids, c.data(), k * sizeof(double));
    if (centroids_f16)
        for (int i = 0; i < k; ++i) centroids_f16[i] = tq::f64_to_f16(c[i]);
    if (boundaries)
        for (int i = 0; i + 1 < k; ++i) boundaries[i] = static_cast<float>(t[i]);
    if (distortion) *distortion = tq::host_distortion(d, bits, cop.data(), t.data());
    return TQ_OK;
}
