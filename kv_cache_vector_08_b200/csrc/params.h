// Host-side parameter generation for a TurboQuant context (float64).
#pragma once

#include <cstdint>
#include <vector>

namespace tq {

struct HostParams {
  int d = 0, bits = 0, k = 0, m = 0, mode = 0;
  uint64_t seed = 0;
  std::vector<double> Pi;          // [d*d] row-major, y = Pi x
  std::vector<double> S;           // [m*d] row-major (prod mode)
  std::vector<double> M;           // [m*d] row-major, M = S Pi^T (prod mode)
  std::vector<double> centroids;   // [2^k] ascending
  std::vector<double> boundaries;  // [2^k - 1]
};

// SplitMix64 outputs start .. start+count-1 for `seed`.
void splitmix64(uint64_t seed, uint64_t start, uint64_t count, uint64_t* out);
// First `count` standard normal draws (Box-Muller on SplitMix64 uniforms in (0,1]).
void gaussian_stream(uint64_t seed, uint64_t count, double* out);
// Q of the QR factorisation of the d x d row-major matrix G, with R_ii > 0 (Householder).
void haar_rotation(int d, const double* G, double* Pi);
// Regularised incomplete beta I_x(a, b).
double incomplete_beta(double a, double b, double x);
// Lloyd-Max codebook with `levels` cells on the coordinate density f_d.
void lloyd_max_beta(int d, int levels, double* centroids, double* boundaries);
// Everything above for one context.  Returns false on bad arguments.
bool build_params(int d, int bits, uint64_t seed, int mode, HostParams* p);

}  // namespace tq
