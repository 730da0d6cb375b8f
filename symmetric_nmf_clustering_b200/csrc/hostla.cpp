// Small dense symmetric eigen-solvers on the host, used by the spectral
// probe's Rayleigh-Ritz step (matrices of at most a few hundred rows).
//
//  - cyclic Jacobi with eigenvectors (Golub & Van Loan, "Matrix
//    Computations", section 8.5) for the b x b Gram matrices of a block;
//  - reduction to tridiagonal form followed by Sturm-sequence bisection
//    (section 8.4.1) for the leading eigenvalues of the block-tridiagonal
//    Lanczos matrix: for a band matrix (the Lanczos matrix has half-bandwidth
//    b) by Givens rotations with bulge chasing (H. R. Schwarz,
//    "Tridiagonalization of a symmetric band matrix", Numerische Mathematik
//    12, 1968), O(m^2 b) instead of O(m^3); for a full matrix by Householder
//    reflections (section 8.3.1).
#include "hostla.h"

#include <algorithm>
#include <cmath>
#include <limits>
#include <vector>

namespace symnmf {

void jacobi_eig(int m, std::vector<double>& A, std::vector<double>& w,
                std::vector<double>& V) {
    V.assign((size_t)m * m, 0.0);
    for (int i = 0; i < m; ++i) V[(size_t)i * m + i] = 1.0;
    auto a = [&](int i, int j) -> double& { return A[(size_t)i * m + j]; };
    for (int sweep = 0; sweep < 100; ++sweep) {
        double off = 0.0, tot = 0.0;
        for (int i = 0; i < m; ++i)
            for (int j = 0; j < m; ++j) {
                tot += a(i, j) * a(i, j);
                if (i != j) off += a(i, j) * a(i, j);
            }
        if (off <= 1e-30 * tot || off == 0.0) break;
        for (int p = 0; p < m - 1; ++p) {
            for (int q = p + 1; q < m; ++q) {
                const double apq = a(p, q);
                if (apq == 0.0) continue;
                // rotation that zeroes a(p,q): tan(theta) from the 2x2 symmetric Schur step
                const double tau = (a(q, q) - a(p, p)) / (2.0 * apq);
                const double t = (tau >= 0 ? 1.0 : -1.0) / (std::fabs(tau) + std::sqrt(1.0 + tau * tau));
                const double c = 1.0 / std::sqrt(1.0 + t * t), s = t * c;
                for (int k = 0; k < m; ++k) {  // columns p, q
                    const double akp = a(k, p), akq = a(k, q);
                    a(k, p) = c * akp - s * akq;
                    a(k, q) = s * akp + c * akq;
                }
                for (int k = 0; k < m; ++k) {  // rows p, q
                    const double apk = a(p, k), aqk = a(q, k);
                    a(p, k) = c * apk - s * aqk;
                    a(q, k) = s * apk + c * aqk;
                }
                for (int k = 0; k < m; ++k) {
                    double& vkp = V[(size_t)k * m + p];
                    double& vkq = V[(size_t)k * m + q];
                    const double x = vkp, y = vkq;
                    vkp = c * x - s * y;
                    vkq = s * x + c * y;
                }
            }
        }
    }
    w.resize(m);
    for (int i = 0; i < m; ++i) w[i] = a(i, i);
}

// Householder tridiagonalisation of a symmetric m x m matrix (row-major,
// destroyed): diagonal d (m) and off-diagonal e (m-1).
static void householder_tridiag(int m, std::vector<double>& A, std::vector<double>& d,
                                std::vector<double>& e) {
    auto a = [&](int i, int j) -> double& { return A[(size_t)i * m + j]; };
    d.assign(m, 0.0);
    e.assign(m > 1 ? m - 1 : 0, 0.0);
    std::vector<double> v(m), p(m);
    for (int k = 0; k + 2 < m; ++k) {
        double norm = 0.0;
        for (int i = k + 1; i < m; ++i) norm += a(i, k) * a(i, k);
        norm = std::sqrt(norm);
        const double x0 = a(k + 1, k);
        const double alpha = x0 >= 0 ? -norm : norm;
        double vnorm2 = 0.0;
        for (int i = k + 1; i < m; ++i) {
            v[i] = a(i, k);
            if (i == k + 1) v[i] -= alpha;
            vnorm2 += v[i] * v[i];
        }
        d[k] = a(k, k);
        if (vnorm2 == 0.0) {  // column already reduced
            e[k] = x0;
            continue;
        }
        e[k] = alpha;
        const double beta = 2.0 / vnorm2;
        // trailing block B = A[k+1:, k+1:]: B <- (I - beta v v^T) B (I - beta v v^T)
        for (int i = k + 1; i < m; ++i) {
            // four independent partial sums (latency, not flops, bounds this loop)
            const double* ai = &a(i, 0);
            double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
            int j = k + 1;
            for (; j + 3 < m; j += 4) {
                s0 += ai[j] * v[j];
                s1 += ai[j + 1] * v[j + 1];
                s2 += ai[j + 2] * v[j + 2];
                s3 += ai[j + 3] * v[j + 3];
            }
            for (; j < m; ++j) s0 += ai[j] * v[j];
            p[i] = beta * ((s0 + s1) + (s2 + s3));
        }
        double K = 0.0;
        for (int i = k + 1; i < m; ++i) K += v[i] * p[i];
        K *= beta / 2.0;
        for (int i = k + 1; i < m; ++i) p[i] -= K * v[i];
        for (int i = k + 1; i < m; ++i)
            for (int j = k + 1; j < m; ++j) a(i, j) -= v[i] * p[j] + p[i] * v[j];
    }
    if (m >= 2) {
        d[m - 2] = a(m - 2, m - 2);
        e[m - 2] = a(m - 1, m - 2);
    }
    d[m - 1] = a(m - 1, m - 1);
}

// Largest |i - j| over the nonzero entries of an m x m matrix (row-major).
static int half_bandwidth(int m, const std::vector<double>& A) {
    int w = 0;
    for (int i = 0; i < m; ++i) {
        const double* ai = &A[(size_t)i * m];
        for (int j = m - 1; j > i + w; --j)
            if (ai[j] != 0.0 || A[(size_t)j * m + i] != 0.0) {
                w = j - i;
                break;
            }
    }
    return w;
}

// Tridiagonal form of a symmetric band matrix of half-bandwidth w (dense
// row-major A; only its lower band is read): the entries at distance
// dd = w, w - 1, ..., 2 below the diagonal are zeroed one width at a time,
// column by column, each by a rotation in the plane (c - 1, c) of its row c.
// Such a rotation mixes columns c - 1 and c, which fills entry (c + dd, c - 1)
// just outside the band; the next rotation, in plane (c + dd - 1, c + dd),
// zeroes that and moves the fill dd further down, until it leaves the matrix.
// The rotations are orthogonal similarities, so the eigenvalues are kept to
// rounding.  The lower band is held compactly, row i's entries at distances
// 0 .. w + 1 (the last for the fill) side by side, so that a rotation's
// updates stay within a few cache lines.
static void band_tridiag(int m, int w, const std::vector<double>& A, std::vector<double>& d,
                         std::vector<double>& e) {
    const int W = w + 2;
    std::vector<double> band((size_t)m * W, 0.0);
    // entry (i, j), j <= i <= j + w + 1
    auto a = [&](int i, int j) -> double& { return band[(size_t)i * W + (i - j)]; };
    for (int i = 0; i < m; ++i)
        for (int j = std::max(0, i - w); j <= i; ++j) a(i, j) = A[(size_t)i * m + j];
    for (int dd = w; dd >= 2; --dd) {
        for (int k = 0; k + dd < m; ++k) {
            int r = k, c = k + dd;   // the entry (c, r) to zero
            while (c < m) {
                const int p = c - 1;
                const double x = a(p, r), y = a(c, r);
                if (y == 0.0) break;   // nothing to zero: no fill either
                double h = std::sqrt(x * x + y * y);
                if (!(h > 0.0) || !std::isfinite(h)) h = std::hypot(x, y);   // under/overflow
                const double cs = x / h, sn = y / h;
                // rows p and c left of the 2 x 2 diagonal block: their nonzeros
                // start at column p - dd (row p's band edge)
                for (int j = std::max(0, p - dd); j < p; ++j) {
                    double& u = a(p, j);
                    double& v = a(c, j);
                    const double u0 = u, v0 = v;
                    u = cs * u0 + sn * v0;
                    v = cs * v0 - sn * u0;
                }
                // the diagonal block
                const double app = a(p, p), acp = a(c, p), acc = a(c, c);
                a(p, p) = cs * cs * app + 2.0 * cs * sn * acp + sn * sn * acc;
                a(c, c) = sn * sn * app - 2.0 * cs * sn * acp + cs * cs * acc;
                a(c, p) = cs * sn * (acc - app) + (cs * cs - sn * sn) * acp;
                // columns p and c below it: nonzeros down to row c + dd (column
                // c's band edge), where the fill appears in column p
                const int ihi = std::min(m - 1, c + dd);
                for (int i = c + 1; i <= ihi; ++i) {
                    double& u = a(i, p);
                    double& v = a(i, c);
                    const double u0 = u, v0 = v;
                    u = cs * u0 + sn * v0;
                    v = cs * v0 - sn * u0;
                }
                a(c, r) = 0.0;
                r = p;        // the fill entry (c + dd, c - 1)
                c += dd;
            }
        }
    }
    d.assign(m, 0.0);
    e.assign(m > 1 ? m - 1 : 0, 0.0);
    for (int i = 0; i < m; ++i) d[i] = a(i, i);
    for (int i = 0; i + 1 < m; ++i) e[i] = a(i + 1, i);
}

// Number of eigenvalues of the tridiagonal (d, e) below each of four shifts
// x[r] (Sturm counts through the pivots of the LDL^T factorisations of
// T - x[r] I), as four independent recurrences so that their divisions overlap.
static void sturm_below4(const std::vector<double>& d, const std::vector<double>& e,
                         const double x[4], int c[4]) {
    const int m = (int)d.size();
    const double tiny = std::numeric_limits<double>::min();
    double q[4] = {1.0, 1.0, 1.0, 1.0};
    int cnt[4] = {0, 0, 0, 0};
    for (int i = 0; i < m; ++i) {
        const double e2 = i > 0 ? e[i - 1] * e[i - 1] : 0.0;
        for (int r = 0; r < 4; ++r) {
            double v = (d[i] - x[r]) - (i > 0 ? e2 / q[r] : 0.0);
            if (v == 0.0) v = -tiny;
            cnt[r] += v < 0.0 ? 1 : 0;
            q[r] = v;
        }
    }
    for (int r = 0; r < 4; ++r) c[r] = cnt[r];
}

void sym_top_eigvals(int m, std::vector<double> A, int count, std::vector<double>& out) {
    // scale by a power of two (exact) so that the largest entry is about 1:
    // the rotations' squares and the Sturm recurrence's e^2 then neither
    // overflow nor underflow for any finite input scale
    double amax = 0.0;
    for (double v : A) amax = std::max(amax, std::fabs(v));
    const int ex = amax > 0.0 && std::isfinite(amax) ? std::ilogb(amax) : 0;
    if (ex != 0)
        for (double& v : A) v = std::ldexp(v, -ex);
    std::vector<double> d, e;
    const int w = half_bandwidth(m, A);
    if (w <= m / 8) band_tridiag(m, w, A, d, e);   // also w <= 1: read off d and e
    else householder_tridiag(m, A, d, e);
    // Gershgorin interval
    double lo = 0.0, hi = 0.0;
    for (int i = 0; i < m; ++i) {
        const double r = (i > 0 ? std::fabs(e[i - 1]) : 0.0) + (i + 1 < m ? std::fabs(e[i]) : 0.0);
        lo = std::min(lo, d[i] - r);
        hi = std::max(hi, d[i] + r);
    }
    const double span = std::max(hi - lo, 1e-300);
    lo -= 1e-6 * span;
    hi += 1e-6 * span;
    count = std::min(count, m);
    out.assign(count, 0.0);
    // brackets [blo, bhi] of every target; every Sturm count narrows the
    // brackets of all targets.  Four targets are bisected in lockstep so that
    // their Sturm recurrences (chains of dependent divisions) overlap.
    std::vector<double> blo(count, lo), bhi(count, hi);
    constexpr int G = 4;
    for (int j0 = 0; j0 < count; j0 += G) {
        const int g = std::min(G, count - j0);
        bool done[G] = {false, false, false, false};
        for (int it = 0; it < 200; ++it) {
            double mid[G];
            bool any = false;
            for (int q = 0; q < G; ++q) {
                mid[q] = 0.0;
                if (q >= g || done[q]) continue;
                const double a = blo[j0 + q], b = bhi[j0 + q];
                mid[q] = 0.5 * (a + b);
                if (mid[q] == a || mid[q] == b) done[q] = true;
                else any = true;
            }
            if (!any) break;
            int c[G];
            sturm_below4(d, e, mid, c);
            for (int q = 0; q < g; ++q) {
                if (done[q]) continue;
                // eigenvalues below mid[q]: c[q]; the target of ascending index
                // m-1-j lies at or above mid[q] iff c[q] <= m-1-j
                for (int j = j0; j < count; ++j) {
                    if (c[q] <= m - 1 - j) blo[j] = std::max(blo[j], mid[q]);
                    else bhi[j] = std::min(bhi[j], mid[q]);
                }
            }
        }
        for (int q = 0; q < g; ++q) out[j0 + q] = 0.5 * (blo[j0 + q] + bhi[j0 + q]);
    }
    if (ex != 0)
        for (double& v : out) v = std::ldexp(v, ex);
}

bool cholesky_upper(int m, const std::vector<double>& M, std::vector<double>& R) {
    R.assign((size_t)m * m, 0.0);
    for (int j = 0; j < m; ++j) {
        double s = M[(size_t)j * m + j];
        for (int k = 0; k < j; ++k) s -= R[(size_t)k * m + j] * R[(size_t)k * m + j];
        if (!(s > 0.0)) return false;
        const double rjj = std::sqrt(s);
        R[(size_t)j * m + j] = rjj;
        for (int i = j + 1; i < m; ++i) {
            double t = M[(size_t)j * m + i];
            for (int k = 0; k < j; ++k) t -= R[(size_t)k * m + j] * R[(size_t)k * m + i];
            R[(size_t)j * m + i] = t / rjj;
        }
    }
    return true;
}

}  // namespace symnmf
