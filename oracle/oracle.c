/*
 * fp64 CPU oracle for the fused residual / gate / norm / modulation row op.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's CPU
 * baseline may load this. The GPU library does not, and it shares no code with it.
 *
 * What it computes, per row (b, l) of a (B, L, D) problem, following the pages:
 *   - sglang PR #36349 "[AMD][Diffusion] Migrate FlyDSL fused norm kernels to the
 *     v0.3.0 stable API", section "Microbenchmark": the fused op takes
 *     (residual, x, gate, weight, bias, scale, shift, "layer" | "rms", eps) and
 *     returns the modulated output and the updated residual; the norm-only op
 *     takes (x, weight, bias, scale, shift, ...) and returns the output alone.
 *   - sglang PR #33144 (same title), section "Modifications" and "Accuracy Tests":
 *     LayerNorm and RMSNorm specialisations, gate-free and no-affine forms,
 *     broadcast (1, C) operands selecting row 0, per-row scale/shift and the 4D
 *     frame-gate layout; "Known gaps" lists the eps, weight-dtype, 2D broadcast
 *     and empty-tensor quirks this oracle does not reproduce.
 *
 *   1. operand rows: off = b*stride_b + (l / tokens_per_frame)*stride_f + l*stride_l
 *      (tokens_per_frame == 0: no frame axis, stride_f unused).
 *   2. r = residual + gate * x          (gate = 1 when absent)  -> rounded to bf16,
 *      returned; the norm acts on this rounded r.  Norm-only: r = x, nothing returned.
 *   3. LayerNorm: mu = sum(r)/D, var = sum((r - mu)^2)/D (biased, two passes),
 *      n = (r - mu) / sqrt(var + eps).   RMSNorm: ms = sum(r^2)/D, n = r / sqrt(ms + eps).
 *   4. affine: n = n * weight (if any), then n = n + bias (if any). weight and bias are
 *      bf16, or binary32 when given as float arrays (the pages' kernel takes fp32
 *      affine parameters and casts them to bf16; here they are used as given).
 *   5. modulation: y = n * (1 + scale) + shift, rounded to bf16.
 * Every step runs in fp64 on the bf16 input values; each bf16 rounding is a single
 * round-to-nearest-even of the fp64 value (bf16_rne below, written from the IEEE
 * 754 definition of rounding).
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* bf16 bit pattern -> double (exact: bf16 is the top half of a binary32). */
double oracle_bf16_to_double(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/*
 * double -> bf16 bit pattern, round to nearest, ties to even, in one step.
 * bf16: 8 significant bits, exponent range of binary32, subnormal quantum 2^-133,
 * largest finite (2 - 2^-7) * 2^127. NaN -> quiet NaN with the input's sign.
 */
uint16_t oracle_bf16_rne(double v) {
  uint16_t sign = signbit(v) ? 0x8000u : 0u;
  if (isnan(v)) return (uint16_t)(sign | 0x7FC0u);
  double a = fabs(v);
  if (isinf(a)) return (uint16_t)(sign | 0x7F80u);
  if (a == 0.0) return sign;
  int e;
  frexp(a, &e);                /* a = m * 2^e, 0.5 <= m < 1 */
  int qexp = e - 8;            /* spacing of 8-bit significands in [2^(e-1), 2^e) */
  if (qexp < -133) qexp = -133; /* subnormal range */
  double q = ldexp(1.0, qexp);
  double k = a / q;            /* exact: division by a power of two */
  double whole = floor(k);
  double frac = k - whole;
  if (frac > 0.5 || (frac == 0.5 && fmod(whole, 2.0) == 1.0)) whole += 1.0;
  double rounded = whole * q;
  if (rounded > 3.3895313892515355e38) return (uint16_t)(sign | 0x7F80u); /* overflow */
  float f = (float)rounded;    /* exact: at most 8 significant bits, in binary32 range */
  uint32_t u;
  memcpy(&u, &f, 4);
  return (uint16_t)(sign | (uint16_t)((u >> 16) & 0x7FFFu));
}

static int64_t row_offset(const int64_t* st, int64_t b, int64_t f, int64_t l) {
  return b * st[0] + f * st[1] + l * st[2];
}

/*
 * The whole op on host memory. Operand strides `*_st` are {stride_b, stride_f,
 * stride_l} in elements (0 = broadcast); output strides are {stride_b, stride_l}.
 * gate, weight, bias may be NULL (absent); weight_f32 / bias_f32 give the affine
 * parameters as binary32 instead (at most one of weight / weight_f32, and of bias /
 * bias_f32). norm_only != 0: residual, gate and r must be NULL, and x is normalised
 * directly.
 * Optional outputs: n_out (fp64 n after the norm, before the affine step, laid out
 * like y) and stats (3 doubles per row b*L + l: mean or 0, variance or mean-square,
 * 1/sqrt(. + eps)).
 * Returns 0, or -1 on an argument it cannot use.
 */
int oracle_fused_norm(int64_t B, int64_t L, int64_t D, int64_t tokens_per_frame, int is_rms,
                      int norm_only, double eps,
                      const uint16_t* x, const int64_t* x_st,
                      const uint16_t* res, const int64_t* res_st,
                      const uint16_t* gate, const int64_t* gate_st,
                      const uint16_t* weight, const uint16_t* bias,
                      const float* weight_f32, const float* bias_f32,
                      const uint16_t* scale, const int64_t* scale_st,
                      const uint16_t* shift, const int64_t* shift_st,
                      uint16_t* y, const int64_t* y_st,
                      uint16_t* r, const int64_t* r_st,
                      double* n_out, double* stats) {
  if (B < 0 || L < 0 || D <= 0 || tokens_per_frame < 0) return -1;
  if (tokens_per_frame > 0 && L % tokens_per_frame != 0) return -1;
  if (!x || !scale || !shift || !y) return -1;
  if (norm_only && (res || gate || r)) return -1;
  if (!norm_only && (!res || !r)) return -1;
  if ((weight && weight_f32) || (bias && bias_f32)) return -1;
  int64_t rows = B * L;
  int bad = 0;
#pragma omp parallel
  {
    double* v = (double*)malloc((size_t)D * sizeof(double));
    if (!v) {
#pragma omp atomic write
      bad = 1;
    }
#pragma omp for schedule(static)
    for (int64_t row = 0; row < rows; ++row) {
      if (!v) continue;
      int64_t b = row / L, l = row % L;
      int64_t f = tokens_per_frame > 0 ? l / tokens_per_frame : 0;
      const uint16_t* xr = x + row_offset(x_st, b, f, l);
      const uint16_t* sr = scale + row_offset(scale_st, b, f, l);
      const uint16_t* tr = shift + row_offset(shift_st, b, f, l);
      uint16_t* yr = y + b * y_st[0] + l * y_st[1];

      /* step 2: residual add with gate, rounded to bf16 */
      if (norm_only) {
        for (int64_t c = 0; c < D; ++c) v[c] = oracle_bf16_to_double(xr[c]);
      } else {
        const uint16_t* rr = res + row_offset(res_st, b, f, l);
        const uint16_t* gr = gate ? gate + row_offset(gate_st, b, f, l) : NULL;
        uint16_t* ro = r + b * r_st[0] + l * r_st[1];
        for (int64_t c = 0; c < D; ++c) {
          double g = gr ? oracle_bf16_to_double(gr[c]) : 1.0;
          double exact = oracle_bf16_to_double(rr[c]) + g * oracle_bf16_to_double(xr[c]);
          uint16_t rb = oracle_bf16_rne(exact);
          ro[c] = rb;
          v[c] = oracle_bf16_to_double(rb);
        }
      }

      /* steps 3-4 of the statistics: mean/variance or mean-square, then 1/sqrt */
      double mu = 0.0, second = 0.0;
      if (is_rms) {
        for (int64_t c = 0; c < D; ++c) second += v[c] * v[c];
        second /= (double)D;
      } else {
        for (int64_t c = 0; c < D; ++c) mu += v[c];
        mu /= (double)D;
        for (int64_t c = 0; c < D; ++c) second += (v[c] - mu) * (v[c] - mu);
        second /= (double)D;
      }
      double rho = 1.0 / sqrt(second + eps);
      if (stats) {
        stats[3 * row + 0] = mu;
        stats[3 * row + 1] = second;
        stats[3 * row + 2] = rho;
      }

      /* normalise, affine, modulate, round */
      for (int64_t c = 0; c < D; ++c) {
        double n = (v[c] - mu) * rho;
        if (n_out) n_out[b * y_st[0] + l * y_st[1] + c] = n;
        if (weight) n = n * oracle_bf16_to_double(weight[c]);
        if (weight_f32) n = n * (double)weight_f32[c];
        if (bias) n = n + oracle_bf16_to_double(bias[c]);
        if (bias_f32) n = n + (double)bias_f32[c];
        double yv = n * (1.0 + oracle_bf16_to_double(sr[c])) + oracle_bf16_to_double(tr[c]);
        yr[c] = oracle_bf16_rne(yv);
      }
    }
    free(v);
  }
  return bad ? -1 : 0;
}

/* Threads the oracle's row loop uses from now on (n >= 1). Not part of the arithmetic. */
void oracle_set_num_threads(int n) {
  if (n >= 1) omp_set_num_threads(n);
}

int oracle_num_threads(void) {
  int n = 1;
#pragma omp parallel
  {
#pragma omp single
    n = omp_get_num_threads();
  }
  return n;
}
