/*
 * Seeded synthetic input generator for the deformable-convolution core.
 *
 * This module holds NO arithmetic of the operator: it only turns
 * (seed, tensor id, flat index) into numbers.  Both the CPU oracle and the
 * CUDA path are fed from it, so that they see the same inputs.
 *
 * Counter-based: value i of tensor t under seed s is a pure function of
 * (s, t, i), computed from one SplitMix64 hash of  s ^ (t << 40) ^ i .
 * SplitMix64 is the finaliser published by Steele, Lea and Flood,
 * "Fast splittable pseudorandom number generators" (OOPSLA 2014).
 * Uniforms use the top 53 bits of the hash; normals use the Box-Muller
 * transform (Box and Muller, 1958) on the two 32-bit halves of the hash.
 * Because every value depends only on its own counter, generation order and
 * thread count do not change the output.
 */
#include <math.h>
#include <stdint.h>

static inline uint64_t splitmix64(uint64_t z) {
  z += 0x9E3779B97F4A7C15ULL;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static inline uint64_t hash_at(uint64_t seed, uint64_t tensor_id, uint64_t i) {
  return splitmix64(seed ^ (tensor_id << 40) ^ i);
}

/* Uniform in [0, 1) with 53 random bits. */
static inline double unit_uniform(uint64_t h) {
  return (double)(h >> 11) * (1.0 / 9007199254740992.0);
}

/* Standard normal from one hash: Box-Muller on its two 32-bit halves. */
static inline double unit_normal(uint64_t h) {
  const double two_pi = 6.283185307179586476925286766559;
  double u1 = ((double)(h >> 32) + 0.5) * (1.0 / 4294967296.0);          /* (0,1) */
  double u2 = (double)(h & 0xFFFFFFFFULL) * (1.0 / 4294967296.0);       /* [0,1) */
  return sqrt(-2.0 * log(u1)) * cos(two_pi * u2);
}

/* out[i] = (float)(lo + (hi - lo) * U_i),  i in [0, n). */
void gen_uniform_f32(uint64_t seed, uint64_t tensor_id, int64_t n, double lo,
                     double hi, float* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i)
    out[i] = (float)(lo + (hi - lo) * unit_uniform(hash_at(seed, tensor_id, (uint64_t)i)));
}

/* out[i] = (float)(mean + sd * Z_i),  i in [0, n). */
void gen_normal_f32(uint64_t seed, uint64_t tensor_id, int64_t n, double mean,
                    double sd, float* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i)
    out[i] = (float)(mean + sd * unit_normal(hash_at(seed, tensor_id, (uint64_t)i)));
}

/*
 * Redraw a fraction of (a, b) pairs: pair p (elements 2p and 2p+1 of `pairs`)
 * is selected when U(seed, select_id, p) < frac, and then both of its
 * elements are replaced by lo + (hi - lo) * U(seed, value_id, 2p + e).
 * Returns the number of pairs redrawn.
 */
int64_t gen_redraw_pairs_f32(uint64_t seed, uint64_t select_id,
                             uint64_t value_id, int64_t n_pairs, double frac,
                             double lo, double hi, float* pairs) {
  int64_t count = 0;
#pragma omp parallel for schedule(static) reduction(+ : count)
  for (int64_t p = 0; p < n_pairs; ++p) {
    if (unit_uniform(hash_at(seed, select_id, (uint64_t)p)) < frac) {
      for (int e = 0; e < 2; ++e)
        pairs[2 * p + e] = (float)(lo + (hi - lo) *
            unit_uniform(hash_at(seed, value_id, (uint64_t)(2 * p + e))));
      ++count;
    }
  }
  return count;
}

/* Raw hash, exposed so that tests can check the generator is counter-based. */
uint64_t gen_hash(uint64_t seed, uint64_t tensor_id, uint64_t i) {
  return hash_at(seed, tensor_id, i);
}
