/*
 * Seeded synthetic inputs for the fused residual / gate / norm / modulation row op.
 *
 * This module only draws numbers. It holds none of the op's arithmetic: no
 * residual add, no statistics, no normalisation, no modulation. Both the
 * fp64 oracle (tests) and the benchmark read its output, so the two sides see
 * the same bf16 inputs.
 *
 * Generator: counter-based. Every element has a 64-bit counter built from
 * (seed, tensor id, row, column pair); the counter is hashed with the SplitMix64
 * output function (Steele, Lea & Flood, "Fast splittable pseudorandom number
 * generators", OOPSLA 2014), which gives a 64-bit word per call. Two words make
 * two uniforms and the Box-Muller transform (Box & Muller, 1958) turns them into
 * two standard normals, one for the even and one for the odd column of the pair.
 * Because nothing is sequential, any row range can be generated on its own and in
 * parallel, and the result does not depend on the thread count.
 *
 * A value is mu + sigma * z, times an optional per-row factor (outlier rows),
 * rounded to the nearest float and then to the nearest bf16 (ties to even at
 * each step). The double step is part of the recipe, not an accuracy claim: the
 * bf16 values produced are simply the inputs.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define SYNTH_GOLDEN 0x9E3779B97F4A7C15ULL

static uint64_t splitmix64_out(uint64_t z) {
  z += SYNTH_GOLDEN;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

/* Key of one (seed, tensor, row) stream. */
static uint64_t stream_key(uint64_t seed, uint32_t tensor_id, int64_t row) {
  uint64_t k = splitmix64_out(seed);
  k = splitmix64_out(k ^ (0x100000001B3ULL * (uint64_t)(tensor_id + 1)));
  k = splitmix64_out(k ^ (uint64_t)row);
  return k;
}

/* Uniform in the open interval (0, 1) from the top 53 bits. */
static double u01_open(uint64_t w) { return ((double)(w >> 11) + 0.5) * (1.0 / 9007199254740992.0); }

static uint16_t float_to_bf16_bits(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x0040u);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

/* One standard normal for column c of the stream with key k. */
static double normal_at(uint64_t k, int64_t c) {
  int64_t pair = c >> 1;
  uint64_t a = splitmix64_out(k + (uint64_t)(2 * pair) * SYNTH_GOLDEN);
  uint64_t b = splitmix64_out(k + (uint64_t)(2 * pair + 1) * SYNTH_GOLDEN);
  double u1 = u01_open(a), u2 = u01_open(b);
  double rad = sqrt(-2.0 * log(u1));
  double ang = 6.283185307179586476925286766559 * u2;
  return (c & 1) ? rad * sin(ang) : rad * cos(ang);
}

/*
 * Fill rows [row0, row0 + nrows) of a (rows, D) bf16 tensor, row-major with row
 * pitch `pitch` elements (pitch >= D). `row_mult` is NULL or holds one factor per
 * generated row (index 0 is row0). Rows are keyed by their global index, so a
 * slice matches the same rows of a full fill.
 */
void synth_fill_bf16(uint16_t* out, int64_t pitch, int64_t row0, int64_t nrows, int64_t D,
                     uint64_t seed, uint32_t tensor_id, double mu, double sigma,
                     const double* row_mult) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < nrows; ++i) {
    int64_t row = row0 + i;
    uint64_t k = stream_key(seed, tensor_id, row);
    double m = row_mult ? row_mult[i] : 1.0;
    uint16_t* o = out + i * pitch;
    for (int64_t c = 0; c < D; c += 2) {
      int64_t pair = c >> 1;
      uint64_t a = splitmix64_out(k + (uint64_t)(2 * pair) * SYNTH_GOLDEN);
      uint64_t b = splitmix64_out(k + (uint64_t)(2 * pair + 1) * SYNTH_GOLDEN);
      double u1 = u01_open(a), u2 = u01_open(b);
      double rad = sqrt(-2.0 * log(u1));
      double ang = 6.283185307179586476925286766559 * u2;
      o[c] = float_to_bf16_bits((float)((mu + sigma * rad * cos(ang)) * m));
      if (c + 1 < D) o[c + 1] = float_to_bf16_bits((float)((mu + sigma * rad * sin(ang)) * m));
    }
  }
}

/* Like synth_fill_bf16, but out row i holds stream row rows[i]. */
void synth_fill_bf16_rows(uint16_t* out, int64_t pitch, const int64_t* rows, int64_t nrows,
                          int64_t D, uint64_t seed, uint32_t tensor_id, double mu, double sigma,
                          const double* row_mult) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < nrows; ++i) {
    synth_fill_bf16(out + i * pitch, pitch, rows[i], 1, D, seed, tensor_id, mu, sigma,
                    row_mult ? row_mult + i : NULL);
  }
}

/* Like synth_fill_bf16 for one (1, D) row, but the values are kept as binary32 (the
 * same draws, rounded to float only). For fp32 affine parameters. */
void synth_fill_f32_row(float* out, int64_t D, uint64_t seed, uint32_t tensor_id, double mu,
                        double sigma) {
  uint64_t k = stream_key(seed, tensor_id, 0);
  for (int64_t c = 0; c < D; ++c) out[c] = (float)(mu + sigma * normal_at(k, c));
}

/* Single element, for spot checks of the fill above. */
uint16_t synth_value_bf16(int64_t row, int64_t c, uint64_t seed, uint32_t tensor_id, double mu,
                          double sigma, double mult) {
  uint64_t k = stream_key(seed, tensor_id, row);
  return float_to_bf16_bits((float)((mu + sigma * normal_at(k, c)) * mult));
}

/*
 * The first `count` entries of a seeded uniform permutation of [0, n), by the
 * Fisher-Yates shuffle (Durstenfeld's in-place form) driven by a SplitMix64 counter
 * stream. Used to pick outlier rows. `perm` is scratch of n entries; the picked
 * rows are written to out[0..count) in permutation order.
 */
void synth_pick_rows(int64_t n, int64_t count, uint64_t seed, int64_t* perm, int64_t* out) {
  for (int64_t i = 0; i < n; ++i) perm[i] = i;
  uint64_t k = stream_key(seed, 0xFFFFu, -1);
  for (int64_t i = n - 1; i > 0; --i) {
    uint64_t w = splitmix64_out(k + (uint64_t)(n - 1 - i) * SYNTH_GOLDEN);
    /* unbiased enough for picking rows: 128-bit multiply-shift onto [0, i] */
    int64_t j = (int64_t)(((unsigned __int128)w * (unsigned __int128)(uint64_t)(i + 1)) >> 64);
    int64_t t = perm[i];
    perm[i] = perm[j];
    perm[j] = t;
  }
  /* Durstenfeld's loop fixes positions from the back; take the last `count`. */
  for (int64_t i = 0; i < count; ++i) out[i] = perm[n - 1 - i];
}
