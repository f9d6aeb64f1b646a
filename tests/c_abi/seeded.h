/* seeded.h -- the C ABI test's seeded input generator: xorshift64* words and Box-Muller normals.
 * Inputs only; nothing here knows about the quantizer. */
#ifndef SEEDED_H
#define SEEDED_H

#include <math.h>
#include <stdint.h>

typedef struct {
  uint64_t s;
} seeded_rng;

static uint64_t seeded_next(seeded_rng* r) {
  r->s ^= r->s >> 12;
  r->s ^= r->s << 25;
  r->s ^= r->s >> 27;
  return r->s * 2685821657736338717ull;
}

/* uniform in (0, 1): 24 random bits, offset by half a step */
static double seeded_uniform(seeded_rng* r) { return ((double)(seeded_next(r) >> 40) + 0.5) / 16777216.0; }

static float seeded_normal(seeded_rng* r) {
  const double u = seeded_uniform(r), v = seeded_uniform(r);
  return (float)(sqrt(-2.0 * log(u)) * cos(6.283185307179586 * v));
}

#endif
