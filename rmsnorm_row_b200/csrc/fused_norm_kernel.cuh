// Row kernels for the fused residual / gate / norm / modulation op on sm_100a.
//
// Operation (sglang PR #36349 "[AMD][Diffusion] Migrate FlyDSL fused norm kernels to
// the v0.3.0 stable API", section "Microbenchmark"; sglang PR #33144, sections
// "Modifications" and "Accuracy Tests"), per row of D channels:
//   r = residual + gate * x (rounded once to bf16), n = LayerNorm/RMSNorm(r) with eps,
//   n = n * weight + bias (each optional), y = n * (1 + scale) + shift.
//
// Design (B200, memory-bound: ~1 flop per byte, no tensor-core work):
//   * One CTA per row, T = D / (8 * VPT) threads. Thread t owns the 16-byte vectors
//     t, t + T, ..., t + (VPT-1) T of each operand row, so every warp access is 512
//     contiguous bytes (fully coalesced 128-bit loads and stores).
//   * The row stays in registers as packed bf16 between the statistics and the
//     normalise pass; HBM sees each full tensor exactly once.
//   * Statistics: every bf16 value is exact in fp64, and so are its square and (for
//     all practical exponent ranges) the row sums, so each thread accumulates
//     sum(r) and sum(r^2) in fp64, warps add through xor-shuffles and warps combine
//     through shared memory in a fixed order after one barrier. LayerNorm takes
//     var = E[r^2] - mean^2; a row whose mean dwarfs its spread (mean^2 > 2^20 var)
//     is recomputed with a second, centred pass. The order of every sum is fixed, so
//     results are bitwise reproducible.
//   * Output rounding: y is evaluated in fp32 with the fp64 statistics rounded to
//     fp32, together with a bound on its error (8 units of fp32 roundoff times the
//     sum of the magnitudes that enter it). The value minus the bound, rounded down,
//     and plus the bound, rounded up, enclose the exact value; when both ends round to
//     the same bf16 value, so does the exact value (rounding is monotone), and that is
//     the result. Otherwise (a few in 10^4 elements) the element is recomputed in fp64
//     and rounded once (round-to-odd to fp32, then nearest-even to bf16). y is therefore
//     the bf16 rounding of the formula evaluated in fp64 with the fp64 statistics, within
//     one bf16 ulp of the exact value. The fp32 arithmetic runs two elements per
//     instruction where it can (sm_100 f32x2), with results identical to the scalar form.
//   * r is the correctly rounded bf16 of the exact residual + gate * x: one bf16x2
//     fused multiply-add per pair computes the exact value and rounds it once.
//   * Per-row (streamed-once) operands use evict-first loads and stores; broadcast
//     and per-frame operands use the read-only cached path (they are re-read by
//     every row and stay in L1/L2). When scale and shift are both of the second kind,
//     separate instances fetch them as each vector is used rather than holding them
//     across the statistics, and run one more CTA per SM on the registers saved.
//   * Norm-only rows with such scale and shift move 4 bytes per element, so their
//     instruction count and the latency of each row's statistics set the pace: they
//     hold 10 vectors per thread (fewer threads share each row's fixed work, more rows
//     are in flight per SM) and, where it measured faster, call one shared out-of-line
//     copy of the rare fp64 path instead of inlining it into every unrolled vector.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>

namespace fused_norm_impl {

// Division of 32-bit values by a divisor fixed for a launch, as a multiply-high and
// shifts (the branch-free round-up method of Granlund and Montgomery, "Division by
// invariant integers using multiplication", 1994): for d >= 2, with l = ceil(log2 d)
// and m = floor(2^32 (2^l - d) / d) + 1, t = mulhi(m, n) gives
// n / d = (t + ((n - t) >> 1)) >> (l - 1) for every 32-bit n. d == 1 is kept apart.
struct DivU32 {
  uint32_t d, m;
  int shift;  // l - 1
};
inline DivU32 make_div_u32(uint32_t d) {
  DivU32 v{d, 0u, 0};
  if (d <= 1) return v;
  int l = 0;
  while ((uint64_t(1) << l) < d) ++l;
  v.m = (uint32_t)((((uint64_t(1) << l) - d) << 32) / d + 1);
  v.shift = l - 1;
  return v;
}
__host__ __device__ __forceinline__ uint32_t div_u32(uint32_t n, const DivU32& v) {
  if (v.d == 1) return n;
#ifdef __CUDA_ARCH__
  const uint32_t t = __umulhi(v.m, n);
#else
  const uint32_t t = (uint32_t)(((uint64_t)v.m * n) >> 32);
#endif
  return (t + ((n - t) >> 1)) >> v.shift;
}

struct RowParams {
  const uint16_t* x;
  const uint16_t* res;
  const uint16_t* gate;
  const uint16_t* scale;
  const uint16_t* shift;
  const void* weight;  // (D) bf16, or fp32 when AFFINE_F32
  const void* bias;
  uint16_t* y;
  uint16_t* r;
  int64_t x_sb, x_sf, x_sl;
  int64_t res_sb, res_sf, res_sl;
  int64_t gate_sb, gate_sf, gate_sl;
  int64_t scale_sb, scale_sf, scale_sl;
  int64_t shift_sb, shift_sf, shift_sl;
  int64_t y_sb, y_sl, r_sb, r_sl;
  uint32_t rows, L, tpf;   // B * L < 2^31 (checked on the host); tpf = 0: no frame axis
  DivU32 div_L, div_tpf;   // division by L and by tpf (tpf > 0)
  double eps;
  uint32_t stream_mask;  // bit set: operand is per-row (read once) -> streaming load
};

enum : uint32_t { kX = 1u, kRes = 2u, kGate = 4u, kScale = 8u, kShift = 16u };

using LaunchFn = cudaError_t (*)(const RowParams&, int64_t grid, cudaStream_t);

__device__ __forceinline__ uint4 load_vec(const uint16_t* base, int j, bool streamed) {
  const uint4* p = reinterpret_cast<const uint4*>(base) + j;
  return streamed ? __ldcs(p) : __ldg(p);
}

__device__ __forceinline__ float lo_f(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float hi_f(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t word(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}
// element q (0..7) of a 16-byte vector of bf16, as fp32
__device__ __forceinline__ float elem(const uint4& v, int q) {
  return (q & 1) ? hi_f(word(v, q >> 1)) : lo_f(word(v, q >> 1));
}

// Element q's value from a 16-byte vector, for a runtime q (rare paths only).
__device__ __forceinline__ float elem_dyn(const uint4& v, int q) {
  const uint32_t w = q < 2 ? v.x : q < 4 ? v.y : q < 6 ? v.z : v.w;
  return (q & 1) ? hi_f(w) : lo_f(w);
}

// ---- bf16 arithmetic on packed pairs (sm_90+ bf16x2, sm_100 mixed precision) ----

// d = a * b + c per bf16 lane, the exact result rounded once to nearest-even bf16.
__device__ __forceinline__ uint32_t fma_bf16x2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
// bf16 half H (0: low, 1: high) of p, plus an fp32 value, rounded once to fp32.
template <int H>
__device__ __forceinline__ float add_bf16_f32(uint32_t p, float c) {
  float d;
  if (H == 0)
    asm("{.reg .b16 l, h; mov.b32 {l, h}, %1; add.rn.f32.bf16 %0, l, %2;}" : "=f"(d) : "r"(p), "f"(c));
  else
    asm("{.reg .b16 l, h; mov.b32 {l, h}, %1; add.rn.f32.bf16 %0, h, %2;}" : "=f"(d) : "r"(p), "f"(c));
  return d;
}
// bf16 half H of p, exactly, as fp64.
template <int H>
__device__ __forceinline__ double bf16_f64(uint32_t p) {
  double d;
  if (H == 0)
    asm("{.reg .b16 l, h; mov.b32 {l, h}, %1; cvt.f64.bf16 %0, l;}" : "=d"(d) : "r"(p));
  else
    asm("{.reg .b16 l, h; mov.b32 {l, h}, %1; cvt.f64.bf16 %0, h;}" : "=d"(d) : "r"(p));
  return d;
}

__device__ __forceinline__ uint32_t pack_rn(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  uint32_t u;
  memcpy(&u, &h, sizeof(u));
  return u;
}

__device__ __forceinline__ uint32_t bf16_rn(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// bf16 bits of an fp64 value rounded once to nearest even: round to odd into fp32
// (24 significant bits, at least two more than bf16 needs), then to nearest even.
__device__ __forceinline__ uint32_t bf16_from_double(double v) {
  float f = __double2float_rz(v);
  if ((double)f != v) f = __uint_as_float(__float_as_uint(f) | 1u);
  return bf16_rn(f);
}

// One 16-byte vector of r = residual + gate * x (gate = 1 when absent): one bf16x2
// fused multiply-add per pair gives the exact sum rounded once to bf16.
template <bool HAS_GATE>
__device__ __forceinline__ uint4 residual_vec(const uint4& res, const uint4& x, const uint4& g) {
  constexpr uint32_t kOnes = 0x3F803F80u;  // (1.0, 1.0) in bf16
  return make_uint4(fma_bf16x2(HAS_GATE ? g.x : kOnes, x.x, res.x),
                    fma_bf16x2(HAS_GATE ? g.y : kOnes, x.y, res.y),
                    fma_bf16x2(HAS_GATE ? g.z : kOnes, x.z, res.z),
                    fma_bf16x2(HAS_GATE ? g.w : kOnes, x.w, res.w));
}

// a / D rounded once to nearest, for D = 5 * 2^k. Markstein's correction: with
// y = RN(1/5) and q0 = RN(a y) (within one ulp of a/5), the residual r = a - 5 q0 is
// exact under fma, and RN(q0 + r y) is the correctly rounded a/5; the power-of-two
// scaling is then exact. Same result as an IEEE division, without its slow path.
template <int D>
__device__ __forceinline__ double div_by_row_length(double a) {
  static_assert(D == 5120 || D == 10240, "D must be 5 * 2^k");
  constexpr double kScale = D == 5120 ? 1.0 / 1024.0 : 1.0 / 2048.0;
  const double q0 = __dmul_rn(a, 0.2);
  if (!isfinite(q0)) return q0 * kScale;  // an infinite or NaN sum divides to itself
  const double r = fma(-5.0, q0, a);
  return fma(r, 0.2, q0) * kScale;
}

struct RowStats {
  double mu, rho;       // fp64 statistics (mu = 0 for RMSNorm)
  float neg_mu32, rho32;  // -mu and rho rounded to fp32, for the fast path
  float kappa;          // |mu32| * rho32: how much of n the mean's rounding can move
};

// y of one element, exactly rounded (see the header comment).
template <bool HAS_WEIGHT, bool HAS_BIAS>
__device__ __forceinline__ uint32_t y_exact(float v, float w, float b, float s, float t,
                                         double mu, double rho) {
  double n = __dmul_rn(__dsub_rn((double)v, mu), rho);
  if (HAS_WEIGHT) n = __dmul_rn(n, (double)w);
  if (HAS_BIAS) n = __dadd_rn(n, (double)b);
  const double y = __dadd_rn(__dmul_rn(n, __dadd_rn(1.0, (double)s)), (double)t);
  return bf16_from_double(y);
}

// fp32 evaluation of y for one element, widened to an interval [lo, hi] that holds
// the exact value of the formula with the fp64 statistics.
//
// Error of the fp32 evaluation, to first order in u = 2^-24 (mu and rho are exact to
// far better than u). With exact n* = (v - mu) rho, the eight roundings (-mu, rho,
// the subtraction, the product with rho, the weight product, the bias sum, 1 + scale,
// the final fma) give
//   |y - y*| <= u (|1+s| |w| kappa + 7 |1+s| |n* w| + 3 |1+s| |b| + |shift|) <= 7 u P,
//   P = |1+s| (|w| kappa + |n w| + |b|) + |shift|,  kappa = |mu| rho.
// The interval is y -/+ 8 u P with its ends rounded outward (down, up); 8 u instead of
// 7 u covers second-order terms and P's own rounding. If both ends round to the same
// bf16 value, the exact value rounds to it too (round to nearest is monotone, across
// binade edges included); otherwise the element takes the fp64 path.
constexpr float k8u = 4.76837158203125e-7f;  // 2^-21

template <int H, bool HAS_WEIGHT, bool HAS_BIAS>
__device__ __forceinline__ void y_enclose(uint32_t vw, uint32_t sw, uint32_t tw, float w, float b,
                                          const RowStats& st, float& lo, float& hi) {
  const float n = add_bf16_f32<H>(vw, st.neg_mu32) * st.rho32;
  const float nw = HAS_WEIGHT ? n * w : n;
  const float nb = HAS_BIAS ? nw + b : nw;
  const float a = add_bf16_f32<H>(sw, 1.0f);
  const float t = H ? hi_f(tw) : lo_f(tw);
  const float y = fmaf(nb, a, t);
  float inner = HAS_WEIGHT ? fmaf(fabsf(w), st.kappa, fabsf(nw)) : st.kappa + fabsf(nw);
  if (HAS_BIAS) inner += fabsf(b);
  const float p = fmaf(fabsf(a), inner, fabsf(t));
  lo = __fmaf_rd(p, -k8u, y);
  hi = __fmaf_ru(p, k8u, y);
}

// ---- paired fp32 arithmetic (sm_100: two fp32 lanes per instruction, each lane
// rounded as the scalar instruction would) ----------------------------------------
__device__ __forceinline__ uint64_t pk2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void upk2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fma2_rd(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rm.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fma2_ru(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rp.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

// y_enclose for both elements of one packed word (low half first): the same
// operations in the same order, two lanes per instruction where no operand needs its
// magnitude, so each y, interval and decision is bit-identical to the scalar path.
template <bool HAS_WEIGHT, bool HAS_BIAS>
__device__ __forceinline__ void y_enclose_pair(uint32_t vw, uint32_t sw, uint32_t tw, float w0, float w1,
                                               float b0, float b1, const RowStats& st, float& lo0,
                                               float& lo1, float& hi0, float& hi1) {
  // r - mu and 1 + scale: with a weight or bias, both halves widened exactly to fp32 and
  // added in one paired instruction (6% fewer instructions, 1% faster on the frame-gate
  // and broadcast affine shapes, measured on B200); without, one mixed-precision add per
  // element (1% faster on norm-only). The sums are the same either way.
  constexpr bool kUnpack = HAS_WEIGHT || HAS_BIAS;
  const uint64_t d = kUnpack ? add2(pk2(lo_f(vw), hi_f(vw)), pk2(st.neg_mu32, st.neg_mu32))
                             : pk2(add_bf16_f32<0>(vw, st.neg_mu32), add_bf16_f32<1>(vw, st.neg_mu32));
  const uint64_t n = mul2(d, pk2(st.rho32, st.rho32));
  const uint64_t nw = HAS_WEIGHT ? mul2(n, pk2(w0, w1)) : n;
  const uint64_t nb = HAS_BIAS ? add2(nw, pk2(b0, b1)) : nw;
  float a0, a1;
  if (kUnpack) {
    upk2(add2(pk2(lo_f(sw), hi_f(sw)), pk2(1.0f, 1.0f)), a0, a1);
  } else {
    a0 = add_bf16_f32<0>(sw, 1.0f);
    a1 = add_bf16_f32<1>(sw, 1.0f);
  }
  const float t0 = lo_f(tw), t1 = hi_f(tw);
  const uint64_t y = fma2(nb, pk2(a0, a1), pk2(t0, t1));
  float nw0, nw1;
  upk2(nw, nw0, nw1);
  float in0 = HAS_WEIGHT ? fmaf(fabsf(w0), st.kappa, fabsf(nw0)) : st.kappa + fabsf(nw0);
  float in1 = HAS_WEIGHT ? fmaf(fabsf(w1), st.kappa, fabsf(nw1)) : st.kappa + fabsf(nw1);
  if (HAS_BIAS) {
    in0 += fabsf(b0);
    in1 += fabsf(b1);
  }
  const uint64_t p = pk2(fmaf(fabsf(a0), in0, fabsf(t0)), fmaf(fabsf(a1), in1, fabsf(t1)));
  upk2(fma2_rd(p, pk2(-k8u, -k8u), y), lo0, lo1);
  upk2(fma2_ru(p, pk2(k8u, k8u), y), hi0, hi1);
}

// Affine parameters of 8 consecutive channels: fp32 as given (two 16-byte loads) or
// bf16 (one 16-byte load, each value widened exactly where it is used).
struct AffineF32 {
  float v[8];
  __device__ __forceinline__ float operator[](int q) const { return v[q]; }
  __device__ __forceinline__ float at(int q) const {  // runtime q (rare paths only)
    return q == 0 ? v[0] : q == 1 ? v[1] : q == 2 ? v[2] : q == 3 ? v[3]
         : q == 4 ? v[4] : q == 5 ? v[5] : q == 6 ? v[6] : v[7];
  }
  static __device__ __forceinline__ AffineF32 load(const void* p, int j) {
    const float4* f = reinterpret_cast<const float4*>(p) + 2 * j;
    const float4 a = __ldg(f), c = __ldg(f + 1);
    return AffineF32{{a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w}};
  }
  static __device__ __forceinline__ AffineF32 fill(float x) { return AffineF32{{x, x, x, x, x, x, x, x}}; }
};
struct AffineBF16 {
  uint4 u;
  __device__ __forceinline__ float operator[](int q) const { return elem(u, q); }
  __device__ __forceinline__ float at(int q) const { return elem_dyn(u, q); }
  static __device__ __forceinline__ AffineBF16 load(const void* p, int j) {
    return AffineBF16{__ldg(reinterpret_cast<const uint4*>(p) + j)};
  }
  static __device__ __forceinline__ AffineBF16 fill(float x) {
    const uint32_t h = __float_as_uint(x) >> 16;  // 0 and 1 are exact in bf16
    return AffineBF16{make_uint4(h * 0x10001u, h * 0x10001u, h * 0x10001u, h * 0x10001u)};
  }
};

// The elements of one output vector whose fp32 interval straddled a rounding boundary
// (bits of near_mask), recomputed in fp64.
template <bool HAS_WEIGHT, bool HAS_BIAS, class Affine>
__device__ __forceinline__ uint4 repair_vec(uint4 out, uint32_t near_mask, const uint4& v, const uint4& sv,
                                            const uint4& tv, const Affine& wf, const Affine& bf, double mu,
                                            double rho) {
#pragma unroll 1
  while (near_mask) {
    const int q = __ffs(near_mask) - 1;
    near_mask &= near_mask - 1;
    const uint32_t bits = y_exact<HAS_WEIGHT, HAS_BIAS>(elem_dyn(v, q), wf.at(q), bf.at(q),
                                                        elem_dyn(sv, q), elem_dyn(tv, q), mu, rho);
    const uint32_t put = (q & 1) ? (bits << 16) : bits;
    const uint32_t keep = (q & 1) ? 0x0000FFFFu : 0xFFFF0000u;
    const int i = q >> 1;
    out.x = i == 0 ? ((out.x & keep) | put) : out.x;
    out.y = i == 1 ? ((out.y & keep) | put) : out.y;
    out.z = i == 2 ? ((out.z & keep) | put) : out.z;
    out.w = i == 3 ? ((out.w & keep) | put) : out.w;
  }
  return out;
}
// The same as one shared out-of-line copy. It runs for a few vectors in 10^3; in the
// norm-only instances with 10 vectors per thread, one copy instead of one per unrolled
// vector keeps the row loop's code small (instruction-fetch stalls 0.88 -> 0.24 per issue,
// measured on B200: 2% faster without weight or bias; 3-7% with fp32 weight or bias at
// D = 10240). Where the kernel holds more live values (the fused instances, norm-only with
// bf16 weight or bias, fp32 ones at D = 5120), the call's register saves cost more (2-6%).
template <bool HAS_WEIGHT, bool HAS_BIAS, class Affine>
__device__ __noinline__ uint4 repair_vec_outlined(uint4 out, uint32_t near_mask, const uint4 v,
                                                  const uint4 sv, const uint4 tv, const Affine wf,
                                                  const Affine bf, double mu, double rho) {
  return repair_vec<HAS_WEIGHT, HAS_BIAS, Affine>(out, near_mask, v, sv, tv, wf, bf, mu, rho);
}

// One 16-byte vector of y: the fp32 interval for all eight elements, packed to bf16 at
// both ends; then (rarely) the fp64 path for the elements whose ends differ.
template <bool PAIRED, bool OUTLINED, bool HAS_WEIGHT, bool HAS_BIAS, class Affine>
__device__ __forceinline__ uint4 output_vec(const uint4& v, const uint4& sv, const uint4& tv,
                                            const Affine& wf, const Affine& bf, const RowStats& st) {
  uint32_t o[4], d[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t vw = word(v, i), sw = word(sv, i), tw = word(tv, i);
    const int e = 2 * i, f = 2 * i + 1;
    float lo0, lo1, hi0, hi1;
    if (PAIRED) {
      y_enclose_pair<HAS_WEIGHT, HAS_BIAS>(vw, sw, tw, wf[e], wf[f], bf[e], bf[f], st, lo0, lo1, hi0, hi1);
    } else {
      y_enclose<0, HAS_WEIGHT, HAS_BIAS>(vw, sw, tw, wf[e], bf[e], st, lo0, hi0);
      y_enclose<1, HAS_WEIGHT, HAS_BIAS>(vw, sw, tw, wf[f], bf[f], st, lo1, hi1);
    }
    o[i] = pack_rn(hi0, hi1);
    d[i] = pack_rn(lo0, lo1) ^ o[i];
  }
  uint4 out = make_uint4(o[0], o[1], o[2], o[3]);
  if ((d[0] | d[1]) | (d[2] | d[3])) {  // rare
    uint32_t near_mask = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      near_mask |= ((d[i] & 0xFFFFu) ? 1u : 0u) << (2 * i) | ((d[i] >> 16) ? 2u : 0u) << (2 * i);
    if constexpr (OUTLINED)
      out = repair_vec_outlined<HAS_WEIGHT, HAS_BIAS, Affine>(out, near_mask, v, sv, tv, wf, bf, st.mu, st.rho);
    else
      out = repair_vec<HAS_WEIGHT, HAS_BIAS, Affine>(out, near_mask, v, sv, tv, wf, bf, st.mu, st.rho);
  }
  return out;
}

// Launch shape per D: vectors per thread (threads = D / (8 VPT)) and the CTAs per SM
// the register budget is sized for (65536 / (threads * kMinBlocks) registers each),
// the same for every specialisation of a D (measured on B200 across all of them).
template <int D> struct RowShape;
#ifndef FN_VPT_5120
#define FN_VPT_5120 5
#endif
#ifndef FN_MINB_5120
#define FN_MINB_5120 5
#endif
#ifndef FN_VPT_10240
#define FN_VPT_10240 4
#endif
#ifndef FN_MINB_10240
#define FN_MINB_10240 2
#endif
// CTAs per SM for the instances whose scale and shift are broadcast or per frame: they
// fetch scale and shift from L1 as each vector is used instead of holding them across
// the statistics, which frees registers for more rows per SM (measured on B200: frame
// gate, broadcast fused and norm-only shapes 2-5% faster than with the streamed
// instances; 7 CTAs at D = 5120 is slower again for the fused ones).
#ifndef FN_VPT_CM_5120
#define FN_VPT_CM_5120 FN_VPT_5120
#endif
#ifndef FN_VPT_CM_10240
#define FN_VPT_CM_10240 FN_VPT_10240
#endif
#ifndef FN_MINB_CM_5120
#define FN_MINB_CM_5120 6
#endif
#ifndef FN_MINB_CM_10240
#define FN_MINB_CM_10240 3
#endif
// 1: y's fp32 arithmetic in paired (f32x2) instructions where no operand needs its
// magnitude. Bit-identical either way; it cuts the instructions per element. Measured on
// B200 with the interval check: 1-3% faster on the broadcast, frame-gate, norm-only
// and D = 10240 shapes, neutral on the WAN2.2 shape.
#ifndef FN_PAIRED_5120
#define FN_PAIRED_5120 1
#endif
#ifndef FN_PAIRED_10240
#define FN_PAIRED_10240 1
#endif
// 1: per-row scale/shift loads are issued with x and residual, before the r stores;
// 0: after them, where the statistics' reduction and barrier hide their latency (fewer
// live registers). Measured on B200: 0 is faster at D = 5120 (WAN2.2 shape), 1 at
// D = 10240, whose two CTAs per SM leave registers to spare (0.4-2% on all its per-row
// specialisations).
#ifndef FN_EARLY_MODULATION_LOADS_5120
#define FN_EARLY_MODULATION_LOADS_5120 0
#endif
#ifndef FN_EARLY_MODULATION_LOADS_10240
#define FN_EARLY_MODULATION_LOADS_10240 1
#endif
// Norm-only with broadcast / per-frame scale and shift reads one tensor and writes one
// per row, so its per-element arithmetic and the latency of each row's statistics, not
// HBM, set its pace. Without weight or bias those instances hold 10 vectors per thread:
// fewer threads per row share the per-thread fixed work (the reduction tail, the fp64
// division and square root, the row addressing), and more rows are in flight per SM.
// D = 5120: 64 threads, 12 CTAs per SM (80 registers, no spills); D = 10240: 128 threads,
// 6 CTAs per SM. Measured on B200 against 128 x 5 at 8 CTAs (D = 5120) and 256 x 5 at 4
// (D = 10240): broadcast LayerNorm 6% and 10% faster, per-frame 2% and 5%. One warp per
// row (20 vectors per lane, 16 warps per SM) was 24% slower at D = 5120: fewer
// instructions, but too few rows in flight.
// With weight or bias (more cached operands per vector) the 64 x 10 shape measured 10%
// slower at D = 5120 (LayerNorm, bf16 weight and bias), so those keep 128 x 5 at 8 CTAs;
// at D = 10240 they take 128 x 10 as well (RMSNorm with weight 4% faster than 256 x 5),
// fp32 affine values at one CTA fewer (2% faster; with 6 CTAs they spill and are slower).
#ifndef FN_VPT_NSS_5120
#define FN_VPT_NSS_5120 10
#endif
#ifndef FN_MINB_NSS_5120
#define FN_MINB_NSS_5120 12
#endif
#ifndef FN_VPT_NSS_AFFINE_5120
#define FN_VPT_NSS_AFFINE_5120 5
#endif
#ifndef FN_MINB_NSS_AFFINE_5120
#define FN_MINB_NSS_AFFINE_5120 8
#endif
#ifndef FN_VPT_NSS_10240
#define FN_VPT_NSS_10240 10
#endif
#ifndef FN_MINB_NSS_10240
#define FN_MINB_NSS_10240 6
#endif
#ifndef FN_VPT_NSS_AFFINE_10240
#define FN_VPT_NSS_AFFINE_10240 10
#endif
#ifndef FN_MINB_NSS_AFFINE_10240
#define FN_MINB_NSS_AFFINE_10240 6
#endif
template <> struct RowShape<5120> {
  static constexpr int VPT = FN_VPT_5120, kMinBlocks = FN_MINB_5120;
  static constexpr int kMinBlocksCachedMod = FN_MINB_CM_5120, kVptCachedMod = FN_VPT_CM_5120;
  static constexpr int kMinBlocksNss = FN_MINB_NSS_5120, kVptNss = FN_VPT_NSS_5120;
  static constexpr int kMinBlocksNssAffine = FN_MINB_NSS_AFFINE_5120, kVptNssAffine = FN_VPT_NSS_AFFINE_5120;
  static constexpr bool kPaired = FN_PAIRED_5120 != 0;
  static constexpr bool kEarlyModLoads = FN_EARLY_MODULATION_LOADS_5120 != 0;
};
template <> struct RowShape<10240> {
  static constexpr int VPT = FN_VPT_10240, kMinBlocks = FN_MINB_10240;
  static constexpr int kMinBlocksCachedMod = FN_MINB_CM_10240, kVptCachedMod = FN_VPT_CM_10240;
  static constexpr int kMinBlocksNss = FN_MINB_NSS_10240, kVptNss = FN_VPT_NSS_10240;
  static constexpr int kMinBlocksNssAffine = FN_MINB_NSS_AFFINE_10240, kVptNssAffine = FN_VPT_NSS_AFFINE_10240;
  static constexpr bool kPaired = FN_PAIRED_10240 != 0;
  static constexpr bool kEarlyModLoads = FN_EARLY_MODULATION_LOADS_10240 != 0;
};

// Vectors per thread of an instance (its CTA has D / (8 VPT) threads): by operand
// placement (norm-only, scale and shift cached) and whether it has a weight or bias.
// The launchers and the host's launch plan both take the shape from here.
template <int D>
__host__ __device__ constexpr int vpt_of(bool norm_only, bool cached_mod, bool affine) {
  return (norm_only && cached_mod) ? (affine ? RowShape<D>::kVptNssAffine : RowShape<D>::kVptNss)
         : cached_mod              ? RowShape<D>::kVptCachedMod
                                   : RowShape<D>::VPT;
}

// CTAs per SM an instance's register budget is sized for. The figure is per D and
// operand placement: instances that carry more live values (fp32 affine, bias, RMSNorm
// with weight at D = 10240) spill a few registers to L1 at these counts, and most measured
// faster so than with one CTA fewer (D = 10240, broadcast modulation: 1.15 ms with 3 CTAs
// per SM and spills, 1.30 ms with 2 and none). The exceptions are an fp32 bias with cached
// modulation, whose 16 fp32 affine values per vector spill ~90 bytes at 6 CTAs: one CTA
// fewer is 4% faster there (the pages' broadcast shape with fp32 w and b), while fp32
// weight alone is 2% slower with one CTA fewer; and norm-only fp32 affine at D = 10240
// (above).
template <int D, bool NORM_ONLY, bool CACHED_MOD, bool AFFINE_F32, bool HAS_WEIGHT, bool HAS_BIAS>
constexpr int min_blocks() {
  return (NORM_ONLY && CACHED_MOD)
             ? ((HAS_WEIGHT || HAS_BIAS)
                    ? RowShape<D>::kMinBlocksNssAffine - ((AFFINE_F32 && D == 10240) ? 1 : 0)
                    : RowShape<D>::kMinBlocksNss)
         : CACHED_MOD ? RowShape<D>::kMinBlocksCachedMod - ((AFFINE_F32 && HAS_BIAS && D == 5120) ? 1 : 0)
                      : RowShape<D>::kMinBlocks;
}

template <int D, int VPT, bool IS_RMS, bool NORM_ONLY, bool HAS_GATE, bool HAS_WEIGHT, bool HAS_BIAS,
          bool AFFINE_F32, bool CACHED_MOD>
__global__ void __launch_bounds__(D / (8 * VPT), (min_blocks<D, NORM_ONLY, CACHED_MOD, AFFINE_F32, HAS_WEIGHT, HAS_BIAS>()))
fused_norm_rows(const RowParams p) {
  constexpr int T = D / (8 * VPT);
  constexpr int W = T / 32;
  static_assert(T % 32 == 0 && T * 8 * VPT == D, "row must split evenly into warps");
  static_assert(!(NORM_ONLY && HAS_GATE), "norm-only has no gate");

  __shared__ double2 part[W];
  __shared__ double centred[W];
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;

  // One row per CTA: the grid is B * L (< 2^31, checked on the host).
  const uint32_t row = blockIdx.x;
  const uint32_t b = div_u32(row, p.div_L);
  const uint32_t l = row - b * p.L;
  const uint32_t f = p.tpf > 0 ? div_u32(l, p.div_tpf) : 0u;

  const uint16_t* xr = p.x + (b * p.x_sb + f * p.x_sf + l * p.x_sl);
  const uint16_t* sr = p.scale + (b * p.scale_sb + f * p.scale_sf + l * p.scale_sl);
  const uint16_t* tr = p.shift + (b * p.shift_sb + f * p.shift_sf + l * p.shift_sl);

  // ---- loads: x, residual and gate are requested together. scale and shift are
  // requested with them or right after the r stores (RowShape<D>::kEarlyModLoads);
  // a load written after a store waits for the store's issue, since the compiler
  // cannot rule out aliasing.
  uint4 xv[VPT], rv[VPT], gv[VPT], sv[VPT], tv[VPT];
#pragma unroll
  for (int k = 0; k < VPT; ++k) xv[k] = load_vec(xr, tid + k * T, p.stream_mask & kX);
  if (!NORM_ONLY) {
    const uint16_t* rr = p.res + (b * p.res_sb + f * p.res_sf + l * p.res_sl);
#pragma unroll
    for (int k = 0; k < VPT; ++k) rv[k] = load_vec(rr, tid + k * T, p.stream_mask & kRes);
  }
  if (HAS_GATE) {
    const uint16_t* gr = p.gate + (b * p.gate_sb + f * p.gate_sf + l * p.gate_sl);
#pragma unroll
    for (int k = 0; k < VPT; ++k) gv[k] = load_vec(gr, tid + k * T, p.stream_mask & kGate);
  }
  if (RowShape<D>::kEarlyModLoads && !CACHED_MOD) {
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      sv[k] = load_vec(sr, tid + k * T, p.stream_mask & kScale);
      tv[k] = load_vec(tr, tid + k * T, p.stream_mask & kShift);
    }
  }

  // ---- step 1: r = residual + gate * x, rounded to bf16, stored -------------
  uint4 v[VPT];  // the row (r, or x when norm-only), packed bf16 pairs
  if (NORM_ONLY) {
#pragma unroll
    for (int k = 0; k < VPT; ++k) v[k] = xv[k];
  } else {
    uint4* ro = reinterpret_cast<uint4*>(p.r + (b * p.r_sb + l * p.r_sl));
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      v[k] = residual_vec<HAS_GATE>(rv[k], xv[k], HAS_GATE ? gv[k] : rv[k]);
      __stcs(ro + tid + k * T, v[k]);
    }
  }

  if (!RowShape<D>::kEarlyModLoads && !CACHED_MOD) {
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      sv[k] = load_vec(sr, tid + k * T, p.stream_mask & kScale);
      tv[k] = load_vec(tr, tid + k * T, p.stream_mask & kShift);
    }
  }

  // ---- step 2: row statistics in fp64 ------------------------------------
  // Four independent accumulation chains per thread (one per word of a vector),
  // combined in a fixed order: short dependency chains, reproducible sums.
  double a1[4] = {0.0, 0.0, 0.0, 0.0}, a2[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
  for (int k = 0; k < VPT; ++k)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const double a = bf16_f64<0>(word(v[k], i)), c = bf16_f64<1>(word(v[k], i));
      if (!IS_RMS) a1[i] += a + c;                 // a + c exact: two bf16 values
      a2[i] = fma(c, c, fma(a, a, a2[i]));         // squares of bf16 values: exact
    }
  double s1 = (a1[0] + a1[1]) + (a1[2] + a1[3]);
  double s2 = (a2[0] + a2[1]) + (a2[2] + a2[3]);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    if (!IS_RMS) s1 += __shfl_xor_sync(0xFFFFFFFFu, s1, o);
    s2 += __shfl_xor_sync(0xFFFFFFFFu, s2, o);
  }
  if (lane == 0) part[warp] = make_double2(s1, s2);
  __syncthreads();
  double t1 = part[0].x, t2 = part[0].y;
#pragma unroll
  for (int w = 1; w < W; ++w) {
    t1 += part[w].x;
    t2 += part[w].y;
  }
  // Correctly rounded divisions by D (not products with 1/D): the mean is then the
  // rounded quotient of the exact sum, as defined, and a row whose mean dwarfs its
  // spread does not turn a last-bit difference of the mean into a different output.
  RowStats st;
  if (IS_RMS) {
    st.mu = 0.0;
    st.rho = rsqrt(div_by_row_length<D>(t2) + p.eps);
  } else {
    const double mu = div_by_row_length<D>(t1);
    double var = div_by_row_length<D>(t2) - mu * mu;
    if (var < 0.0) var = 0.0;  // rounding below zero; a NaN (non-finite row) stays NaN
    if (mu * mu > 1048576.0 * var && var > 0.0) {
      // The mean dwarfs the spread: take the variance around the mean instead
      // (uniform branch: every thread of the CTA has the same statistics). The row
      // is read back from memory (this thread's own r stores, or x) in a rolled
      // loop: unrolled over the register copy, this rare pass would set the
      // kernel's register allocation and force spills on the common path.
      const uint4* rowv = NORM_ONLY ? reinterpret_cast<const uint4*>(xr)
                                    : reinterpret_cast<const uint4*>(p.r + (b * p.r_sb + l * p.r_sl));
      double c2 = 0.0;
#pragma unroll 1
      for (int k = 0; k < VPT; ++k) {
        const uint4 vk = __ldcg(rowv + tid + k * T);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const double a = bf16_f64<0>(word(vk, i)) - mu, c = bf16_f64<1>(word(vk, i)) - mu;
          c2 = fma(a, a, c2);
          c2 = fma(c, c, c2);
        }
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) c2 += __shfl_xor_sync(0xFFFFFFFFu, c2, o);
      if (lane == 0) centred[warp] = c2;
      __syncthreads();
      double tc = centred[0];
#pragma unroll
      for (int w = 1; w < W; ++w) tc += centred[w];
      var = div_by_row_length<D>(tc);
    }
    st.mu = mu;
    st.rho = rsqrt(var + p.eps);
  }
  st.neg_mu32 = -(float)st.mu;
  st.rho32 = (float)st.rho;
  st.kappa = fabsf(st.neg_mu32) * st.rho32;

  // ---- step 3: normalise, affine, modulate, store y ------------------------
  uint4* yo = reinterpret_cast<uint4*>(p.y + (b * p.y_sb + l * p.y_sl));
#pragma unroll
  for (int k = 0; k < VPT; ++k) {
    const int j = tid + k * T;
    if (CACHED_MOD) {  // broadcast / per-frame rows: L1 hits, fetched as they are used
      sv[k] = __ldg(reinterpret_cast<const uint4*>(sr) + j);
      tv[k] = __ldg(reinterpret_cast<const uint4*>(tr) + j);
    }
    using Affine = typename std::conditional<AFFINE_F32, AffineF32, AffineBF16>::type;
    const Affine wf = HAS_WEIGHT ? Affine::load(p.weight, j) : Affine::fill(1.0f);
    const Affine bf = HAS_BIAS ? Affine::load(p.bias, j) : Affine::fill(0.0f);
    constexpr bool kOutlined = NORM_ONLY && CACHED_MOD && ((!HAS_WEIGHT && !HAS_BIAS) || (D == 10240 && AFFINE_F32));
    __stcs(yo + j, output_vec<RowShape<D>::kPaired, kOutlined, HAS_WEIGHT, HAS_BIAS>(v[k], sv[k], tv[k], wf,
                                                                                   bf, st));
  }
}

// Launches one instance and returns the status of this launch alone (the value the
// runtime returns for it; no earlier error is read or cleared).
template <int D, int VPT, bool IS_RMS, bool NORM_ONLY, bool HAS_GATE, bool HAS_WEIGHT, bool HAS_BIAS,
          bool AFFINE_F32, bool CACHED_MOD>
cudaError_t launch_rows(const RowParams& p, int64_t grid, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(D / (8 * VPT), 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  return cudaLaunchKernelEx(
      &cfg, fused_norm_rows<D, VPT, IS_RMS, NORM_ONLY, HAS_GATE, HAS_WEIGHT, HAS_BIAS, AFFINE_F32, CACHED_MOD>, p);
}

// Launcher for one (norm_only, gate, modulation caching) group: the affine combinations.
template <int D, bool RMS, bool NO, bool G, bool CM>
LaunchFn pick_affine(bool w, bool b, bool f32) {
  constexpr int V0 = vpt_of<D>(NO, CM, false);  // no weight or bias
  constexpr int V = vpt_of<D>(NO, CM, true);
  if (!w && !b) return &launch_rows<D, V0, RMS, NO, G, false, false, false, CM>;
  if (f32) {
    if (w && b) return &launch_rows<D, V, RMS, NO, G, true, true, true, CM>;
    return w ? &launch_rows<D, V, RMS, NO, G, true, false, true, CM>
             : &launch_rows<D, V, RMS, NO, G, false, true, true, CM>;
  }
  if (w && b) return &launch_rows<D, V, RMS, NO, G, true, true, false, CM>;
  return w ? &launch_rows<D, V, RMS, NO, G, true, false, false, CM>
           : &launch_rows<D, V, RMS, NO, G, false, true, false, CM>;
}

// Launcher for every specialisation of one (D, norm); instantiated in one translation
// unit per (D, norm) so the instances compile in parallel. cached_mod selects the
// instances for scale and shift that are broadcast or per frame (re-read by many rows).
template <int D, bool RMS>
LaunchFn pick_launcher(bool norm_only, bool has_gate, bool has_weight, bool has_bias, bool f32,
                       bool cached_mod) {
  if (cached_mod) {
    if (norm_only) return pick_affine<D, RMS, true, false, true>(has_weight, has_bias, f32);
    return has_gate ? pick_affine<D, RMS, false, true, true>(has_weight, has_bias, f32)
                    : pick_affine<D, RMS, false, false, true>(has_weight, has_bias, f32);
  }
  if (norm_only) return pick_affine<D, RMS, true, false, false>(has_weight, has_bias, f32);
  return has_gate ? pick_affine<D, RMS, false, true, false>(has_weight, has_bias, f32)
                  : pick_affine<D, RMS, false, false, false>(has_weight, has_bias, f32);
}

LaunchFn select_launcher(int D, bool is_rms, bool norm_only, bool has_gate, bool has_weight,
                         bool has_bias, bool affine_f32, bool cached_mod);
LaunchFn select_launcher_5120_ln(bool norm_only, bool has_gate, bool has_weight, bool has_bias, bool f32, bool cm);
LaunchFn select_launcher_5120_rms(bool norm_only, bool has_gate, bool has_weight, bool has_bias, bool f32, bool cm);
LaunchFn select_launcher_10240_ln(bool norm_only, bool has_gate, bool has_weight, bool has_bias, bool f32, bool cm);
LaunchFn select_launcher_10240_rms(bool norm_only, bool has_gate, bool has_weight, bool has_bias, bool f32, bool cm);

}  // namespace fused_norm_impl

// Defines the launcher selector of one (D, norm) translation unit.
#define FUSED_NORM_DEFINE_SELECTOR(NAME, D_, RMS_)                                              \
  namespace fused_norm_impl {                                                                   \
  LaunchFn NAME(bool norm_only, bool has_gate, bool has_weight, bool has_bias, bool f32, bool cm) { \
    return pick_launcher<D_, RMS_>(norm_only, has_gate, has_weight, has_bias, f32, cm);         \
  }                                                                                             \
  }
