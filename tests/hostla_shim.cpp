// C entry points over the host eigen-solvers of the spectral probe, compiled
// by the CPU tests only (the library itself calls the C++ functions).
#include <vector>

#include "hostla.h"

extern "C" {

int hl_top_eigvals(int m, const double* A, int count, double* out) {
    std::vector<double> a(A, A + (size_t)m * m), w;
    symnmf::sym_top_eigvals(m, a, count, w);
    for (size_t i = 0; i < w.size(); ++i) out[i] = w[i];
    return (int)w.size();
}

void hl_jacobi(int m, const double* A, double* w, double* V) {
    std::vector<double> a(A, A + (size_t)m * m), wv, Vv;
    symnmf::jacobi_eig(m, a, wv, Vv);
    for (int i = 0; i < m; ++i) w[i] = wv[i];
    for (size_t i = 0; i < Vv.size(); ++i) V[i] = Vv[i];
}

int hl_cholesky_upper(int m, const double* M, double* R) {
    std::vector<double> mv(M, M + (size_t)m * m), r;
    const bool ok = symnmf::cholesky_upper(m, mv, r);
    for (size_t i = 0; i < r.size(); ++i) R[i] = r[i];
    return ok ? 1 : 0;
}

}  // extern "C"
