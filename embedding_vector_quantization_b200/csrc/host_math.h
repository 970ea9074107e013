// Host-side math of the library (see host_math.cpp for the method and readings).
#pragma once

#include <cstddef>
#include <cstdint>

namespace tqhost {

// First `count` N(0,1) values of the SplitMix64 + Box-Muller stream for `seed`.
void gaussian_stream(uint64_t seed, size_t count, double* out);

// Pi (d x d, row-major, y = Pi u) = sign-fixed Q of a Householder QR of G, and
// S (m x d, row-major) continuing the same Gaussian stream. S may be null.
void rotation(int d, int m, uint64_t seed, double* Pi, double* S);

// Lloyd-Max codebook (2^bits ascending centroids, 2^bits - 1 midpoint
// boundaries) for one coordinate of a uniform unit vector in R^d.
// Returns 0, or -1 for d < 3 or bits outside 1..8.
int codebook(int d, int bits, double* centroids, double* bounds);

// Lloyd-Max codebook of the level-`level` angle of the recursive polar transform of a
// uniform direction: level 1 is uniform on (-pi, pi] (uniform grid); level l >= 2 has
// density proportional to (sin psi cos psi)^(2^(l-1) - 1) on [0, pi/2].
// Returns 0, or -1 for level outside 1..16 or bits outside 1..8.
int polar_codebook(int level, int bits, double* centroids, double* bounds);

}  // namespace tqhost
