/* Counter-based random inputs for the synthetic workloads (no arithmetic of the
 * attention method lives here).  splitmix64 over a counter, Box-Muller normals,
 * and the per-workload transforms documented in workloads/__init__.py. */
#include <math.h>
#include <stdint.h>

static inline uint64_t mix(uint64_t z) {
  z ^= z >> 30;
  z *= 0xBF58476D1CE4E5B9ull;
  z ^= z >> 27;
  z *= 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

static inline double uni(uint64_t key, int64_t i) {
  return (double)(mix(key + (uint64_t)(i + 1) * 0x9E3779B97F4A7C15ull) >> 11) * 0x1.0p-53;
}

static inline double nrm(uint64_t key, int64_t i) {
  double u1 = uni(key, 2 * i), u2 = uni(key, 2 * i + 1);
  return sqrt(-2.0 * log1p(-u1)) * cos(2.0 * 3.14159265358979323846 * u2);
}

uint64_t wl_key(uint64_t seed, uint64_t stream) { return mix((seed << 20) + stream); }

void wl_uniform(uint64_t key, int64_t start, int64_t n, double* out) {
  for (int64_t t = 0; t < n; ++t) out[t] = uni(key, start + t);
}

void wl_normal(uint64_t key, int64_t start, int64_t n, double* out) {
  for (int64_t t = 0; t < n; ++t) out[t] = nrm(key, start + t);
}

/* dist 0: normal.  1: normal, x20 where uniform(key2) < 0.01, plus vec[(i / (N d)) * d + i % d]
 * when vec != 0.  2: Student-t nu = 3 from normals 4i..4i+3, clipped to |x| <= 60.
 * 3: normal times vec[i / d] (one factor per token row). */
void wl_fill(int dist, uint64_t key, uint64_t key2, int64_t start, int64_t n, const double* vec, int64_t N,
             int64_t d, double* out) {
  for (int64_t t = 0; t < n; ++t) {
    int64_t i = start + t;
    double x;
    if (dist == 0) {
      x = nrm(key, i);
    } else if (dist == 1) {
      x = nrm(key, i);
      if (uni(key2, i) < 0.01) x *= 20.0;
      if (vec) x += vec[(i / (N * d)) * d + i % d];
    } else if (dist == 2) {
      double z0 = nrm(key, 4 * i), z1 = nrm(key, 4 * i + 1), z2 = nrm(key, 4 * i + 2), z3 = nrm(key, 4 * i + 3);
      x = z0 / sqrt((z1 * z1 + z2 * z2 + z3 * z3) / 3.0);
      if (x > 60.0) x = 60.0;
      if (x < -60.0) x = -60.0;
    } else {
      x = nrm(key, i) * vec[i / d];
    }
    out[t] = x;
  }
}
