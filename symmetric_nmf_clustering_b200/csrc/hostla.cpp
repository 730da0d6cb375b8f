// Small dense symmetric eigen-solvers on the host, used by the spectral
// probe's Rayleigh-Ritz step (matrices of at most a few hundred rows).
//
//  - cyclic Jacobi with eigenvectors (Golub & Van Loan, "Matrix
//    Computations", section 8.5) for the b x b Gram matrices of a block;
//  - Householder reduction to tridiagonal form (section 8.3.1) followed by
//    Sturm-sequence bisection (section 8.4.1) for the leading eigenvalues of
//    the block-tridiagonal Lanczos matrix.
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
    std::vector<double> d, e;
    householder_tridiag(m, A, d, e);
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
