// Host-side small symmetric eigen-solvers (see hostla.cpp).
#pragma once
#include <vector>

namespace symnmf {

// Eigen-decomposition of a symmetric m x m matrix A (row-major, destroyed):
// eigenvalues w (unsorted) and eigenvectors as the columns of V (row-major).
void jacobi_eig(int m, std::vector<double>& A, std::vector<double>& w, std::vector<double>& V);

// The `count` algebraically largest eigenvalues of a symmetric m x m matrix,
// descending.
void sym_top_eigvals(int m, std::vector<double> A, int count, std::vector<double>& out);

// Upper Cholesky factor R (M = R^T R) of a symmetric m x m matrix; false if
// M is not numerically positive definite.
bool cholesky_upper(int m, const std::vector<double>& M, std::vector<double>& R);

}  // namespace symnmf
