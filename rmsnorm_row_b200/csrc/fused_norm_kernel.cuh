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
//     sum of the magnitudes that enter it). When that bound does not reach the
//     nearest bf16 rounding boundary the fp32 result rounds like the exact value;
//     otherwise (a few in 10^4 elements) the element is recomputed in fp64 and
//     rounded once (round-to-odd to fp32, then nearest-even to bf16). y is therefore
//     the correctly rounded bf16 of the formula evaluated with the fp64 statistics.
//     At D = 10240 the fp32 arithmetic runs two elements per instruction (sm_100
//     f32x2), with results identical to the scalar form.
//   * r is the correctly rounded bf16 of the exact residual + gate * x: one bf16x2
//     fused multiply-add per pair computes the exact value and rounds it once.
//   * Per-row (streamed-once) operands use evict-first loads and stores; broadcast
//     and per-frame operands use the read-only cached path (they are re-read by
//     every row and stay in L1/L2). When scale and shift are both of the second kind,
//     separate instances fetch them as each vector is used rather than holding them
//     across the statistics, and run one more CTA per SM on the registers saved.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace fused_norm_impl {

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
  int64_t L, tpf, rows;
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

// fp32 evaluation of y for one element, and whether it is far enough from every bf16
// rounding boundary to be rounded as is (otherwise `near` is set).
//
// Error of the fp32 evaluation, to first order in u = 2^-24 (mu and rho are exact to
// far better than u). With exact n* = (v - mu) rho, the eight roundings (-mu, rho,
// the subtraction, the product with rho, the weight product, the bias sum, 1 + scale,
// the final fma) give
//   |y - y*| <= u (|1+s| |w| kappa + 7 |1+s| |n* w| + 3 |1+s| |b| + |shift|) <= 7 u P,
//   P = |1+s| (|w| kappa + |n w| + |b|) + |shift|,  kappa = |mu| rho.
// The test uses B = 8 u P, which also covers second-order terms and P's own rounding.
// Rounding boundaries next to y: the midpoint D away in its bf16 interval, and, when y
// lies in the lowest interval of a binade, one at least ulp/4 below (ulp = bf16 spacing
// at y; |y| 2^-10 <= ulp/4). So y rounds correctly if B < min(D, |y| 2^-10).
template <int H, bool HAS_WEIGHT, bool HAS_BIAS>
__device__ __forceinline__ float y_fast_core(uint32_t vw, uint32_t sw, uint32_t tw, float w, float b,
                                             const RowStats& st, bool& near) {
  constexpr float k8u = 4.76837158203125e-7f;  // 2^-21
  const float n = add_bf16_f32<H>(vw, st.neg_mu32) * st.rho32;
  const float nw = HAS_WEIGHT ? n * w : n;
  const float nb = HAS_BIAS ? nw + b : nw;
  const float a = add_bf16_f32<H>(sw, 1.0f);
  const float t = H ? hi_f(tw) : lo_f(tw);
  const float y = fmaf(nb, a, t);
  float inner = HAS_WEIGHT ? fmaf(fabsf(w), st.kappa, fabsf(nw)) : st.kappa + fabsf(nw);
  if (HAS_BIAS) inner += fabsf(b);
  const float bound = fmaf(fabsf(a), inner, fabsf(t)) * k8u;
  // the bf16 rounding boundary next to y: same sign and exponent, low half 0x8000
  const float mid = __uint_as_float((__float_as_uint(y) & 0xFFFF0000u) | 0x8000u);
  const float room = fminf(fabsf(y - mid), fabsf(y) * 9.765625e-4f);  // 2^-10
  near |= !(room > bound);  // NaN/Inf also take the fp64 path
  return y;
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
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ float bf16_mid(float y) {
  return __uint_as_float((__float_as_uint(y) & 0xFFFF0000u) | 0x8000u);
}

// y_fast_core for both elements of one packed word (low half first): the same
// operations in the same order, two lanes per instruction where no operand needs its
// magnitude, so each y, bound and decision is bit-identical to the scalar path.
template <bool HAS_WEIGHT, bool HAS_BIAS>
__device__ __forceinline__ void y_fast_pair(uint32_t vw, uint32_t sw, uint32_t tw, float w0, float w1,
                                            float b0, float b1, const RowStats& st, float& y0,
                                            float& y1, bool& near0, bool& near1) {
  constexpr float k8u = 4.76837158203125e-7f;  // 2^-21
  constexpr float kEdge = 9.765625e-4f;        // 2^-10
  const uint64_t n = mul2(pk2(add_bf16_f32<0>(vw, st.neg_mu32), add_bf16_f32<1>(vw, st.neg_mu32)),
                          pk2(st.rho32, st.rho32));
  const uint64_t nw = HAS_WEIGHT ? mul2(n, pk2(w0, w1)) : n;
  const uint64_t nb = HAS_BIAS ? add2(nw, pk2(b0, b1)) : nw;
  const float a0 = add_bf16_f32<0>(sw, 1.0f), a1 = add_bf16_f32<1>(sw, 1.0f);
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
  const uint64_t bound = mul2(pk2(fmaf(fabsf(a0), in0, fabsf(t0)), fmaf(fabsf(a1), in1, fabsf(t1))),
                              pk2(k8u, k8u));
  upk2(y, y0, y1);
  const uint64_t dm = sub2(y, pk2(bf16_mid(y0), bf16_mid(y1)));
  const uint64_t ye = mul2(y, pk2(kEdge, kEdge));
  float d0, d1, e0, e1, q0, q1;
  upk2(dm, d0, d1);
  upk2(ye, e0, e1);
  upk2(bound, q0, q1);
  near0 |= !(fminf(fabsf(d0), fabsf(e0)) > q0);
  near1 |= !(fminf(fabsf(d1), fabsf(e1)) > q1);
}

// y_fast_core with bf16 weight / bias taken from packed words.
template <int H, bool HAS_WEIGHT, bool HAS_BIAS>
__device__ __forceinline__ float y_fast(uint32_t vw, uint32_t sw, uint32_t tw, uint32_t ww,
                                        uint32_t bw, const RowStats& st, bool& near) {
  return y_fast_core<H, HAS_WEIGHT, HAS_BIAS>(vw, sw, tw, H ? hi_f(ww) : lo_f(ww),
                                              H ? hi_f(bw) : lo_f(bw), st, near);
}

// Element q's value from a 16-byte vector, for a runtime q (rare paths only).
__device__ __forceinline__ float elem_dyn(const uint4& v, int q) {
  const uint32_t w = q < 2 ? v.x : q < 4 ? v.y : q < 6 ? v.z : v.w;
  return (q & 1) ? hi_f(w) : lo_f(w);
}

// One 16-byte vector of y: the fp32 fast path for all eight elements, then (rarely) the
// fp64 path for the elements whose fast value came near a rounding boundary.
template <bool PAIRED, bool HAS_WEIGHT, bool HAS_BIAS>
__device__ __forceinline__ uint4 output_vec(const uint4& v, const uint4& sv, const uint4& tv,
                                            const uint4& wv, const uint4& bv, const RowStats& st) {
  uint32_t o[4];
  uint32_t near_mask = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t vw = word(v, i), sw = word(sv, i), tw = word(tv, i);
    const uint32_t ww = word(wv, i), bw = word(bv, i);
    bool n0 = false, n1 = false;
    float y0, y1;
    if (PAIRED) {
      y_fast_pair<HAS_WEIGHT, HAS_BIAS>(vw, sw, tw, lo_f(ww), hi_f(ww), lo_f(bw), hi_f(bw), st, y0, y1,
                                        n0, n1);
    } else {
      y0 = y_fast<0, HAS_WEIGHT, HAS_BIAS>(vw, sw, tw, ww, bw, st, n0);
      y1 = y_fast<1, HAS_WEIGHT, HAS_BIAS>(vw, sw, tw, ww, bw, st, n1);
    }
    o[i] = pack_rn(y0, y1);
    near_mask |= (n0 ? 1u : 0u) << (2 * i);
    near_mask |= (n1 ? 2u : 0u) << (2 * i);
  }
  uint4 out = make_uint4(o[0], o[1], o[2], o[3]);
#pragma unroll 1
  while (near_mask) {  // rare
    const int q = __ffs(near_mask) - 1;
    near_mask &= near_mask - 1;
    const uint32_t bits = y_exact<HAS_WEIGHT, HAS_BIAS>(
        elem_dyn(v, q), HAS_WEIGHT ? elem_dyn(wv, q) : 1.0f, HAS_BIAS ? elem_dyn(bv, q) : 0.0f,
        elem_dyn(sv, q), elem_dyn(tv, q), st.mu, st.rho);
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

// fp32 affine parameters (w, b as given, 8 per vector: two 16-byte loads each).
struct Affine8 {
  float v[8];
};
__device__ __forceinline__ Affine8 load_affine_f32(const void* p, int j) {
  const float4* f = reinterpret_cast<const float4*>(p) + 2 * j;
  const float4 a = __ldg(f), c = __ldg(f + 1);
  return Affine8{{a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w}};
}
__device__ __forceinline__ float sel8(const Affine8& a, int q) {
  return q == 0 ? a.v[0] : q == 1 ? a.v[1] : q == 2 ? a.v[2] : q == 3 ? a.v[3]
       : q == 4 ? a.v[4] : q == 5 ? a.v[5] : q == 6 ? a.v[6] : a.v[7];
}

// As output_vec, with fp32 weight / bias.
template <bool PAIRED, bool HAS_WEIGHT, bool HAS_BIAS>
__device__ __forceinline__ uint4 output_vec_f32(const uint4& v, const uint4& sv, const uint4& tv,
                                                const Affine8& wf, const Affine8& bf,
                                                const RowStats& st) {
  uint32_t o[4];
  uint32_t near_mask = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t vw = word(v, i), sw = word(sv, i), tw = word(tv, i);
    bool n0 = false, n1 = false;
    float y0, y1;
    if (PAIRED) {
      y_fast_pair<HAS_WEIGHT, HAS_BIAS>(vw, sw, tw, wf.v[2 * i], wf.v[2 * i + 1], bf.v[2 * i],
                                        bf.v[2 * i + 1], st, y0, y1, n0, n1);
    } else {
      y0 = y_fast_core<0, HAS_WEIGHT, HAS_BIAS>(vw, sw, tw, wf.v[2 * i], bf.v[2 * i], st, n0);
      y1 = y_fast_core<1, HAS_WEIGHT, HAS_BIAS>(vw, sw, tw, wf.v[2 * i + 1], bf.v[2 * i + 1], st, n1);
    }
    o[i] = pack_rn(y0, y1);
    near_mask |= (n0 ? 1u : 0u) << (2 * i);
    near_mask |= (n1 ? 2u : 0u) << (2 * i);
  }
  uint4 out = make_uint4(o[0], o[1], o[2], o[3]);
#pragma unroll 1
  while (near_mask) {  // rare
    const int q = __ffs(near_mask) - 1;
    near_mask &= near_mask - 1;
    const uint32_t bits = y_exact<HAS_WEIGHT, HAS_BIAS>(elem_dyn(v, q), sel8(wf, q), sel8(bf, q),
                                                        elem_dyn(sv, q), elem_dyn(tv, q), st.mu, st.rho);
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
// 1: y's fp32 arithmetic in paired (f32x2) instructions. Bit-identical either way; it
// cuts ~6% of the instructions but lengthens each thread's dependency chains. Measured
// on B200: ~4% faster at D = 10240 (two CTAs per SM, issue-bound with weight), neutral
// to mixed at D = 5120 and slower there when launches run serialised.
// CTAs per SM for the instances whose scale and shift are broadcast or per frame: they
// fetch scale and shift from L1 as each vector is used instead of holding them across
// the statistics, which frees registers for more rows per SM (measured on B200: frame
// gate, broadcast fused and norm-only shapes 2-5% faster than with the streamed
// instances; 7 CTAs at D = 5120 is slower again).
#ifndef FN_MINB_CM_5120
#define FN_MINB_CM_5120 6
#endif
#ifndef FN_MINB_CM_10240
#define FN_MINB_CM_10240 3
#endif
#ifndef FN_PAIRED_5120
#define FN_PAIRED_5120 0
#endif
#ifndef FN_PAIRED_10240
#define FN_PAIRED_10240 1
#endif
// 1: scale/shift loads are issued with x and residual, before the r stores;
// 0: after them, where the statistics' reduction and barrier hide their latency
// (fewer live registers; measured faster on B200 for the WAN2.2 shape).
#ifndef FN_EARLY_MODULATION_LOADS
#define FN_EARLY_MODULATION_LOADS 0
#endif
template <> struct RowShape<5120> {
  static constexpr int VPT = FN_VPT_5120, kMinBlocks = FN_MINB_5120;
  static constexpr int kMinBlocksCachedMod = FN_MINB_CM_5120;
  static constexpr bool kPaired = FN_PAIRED_5120 != 0;
};
template <> struct RowShape<10240> {
  static constexpr int VPT = FN_VPT_10240, kMinBlocks = FN_MINB_10240;
  static constexpr int kMinBlocksCachedMod = FN_MINB_CM_10240;
  static constexpr bool kPaired = FN_PAIRED_10240 != 0;
};

template <int D, int VPT, bool IS_RMS, bool NORM_ONLY, bool HAS_GATE, bool HAS_WEIGHT, bool HAS_BIAS,
          bool AFFINE_F32, bool CACHED_MOD>
__global__ void __launch_bounds__(D / (8 * VPT), CACHED_MOD ? RowShape<D>::kMinBlocksCachedMod
                                                            : RowShape<D>::kMinBlocks)
fused_norm_rows(const RowParams p) {
  constexpr int T = D / (8 * VPT);
  constexpr int W = T / 32;
  static_assert(T % 32 == 0 && T * 8 * VPT == D, "row must split evenly into warps");
  static_assert(!(NORM_ONLY && HAS_GATE), "norm-only has no gate");

  __shared__ double2 part[2][W];
  __shared__ double centred[W];
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  int parity = 0;

  for (int64_t row = blockIdx.x; row < p.rows; row += gridDim.x, parity ^= 1) {
    const int64_t b = row / p.L;
    const int64_t l = row - b * p.L;
    const int64_t f = p.tpf > 0 ? l / p.tpf : 0;

    const uint16_t* xr = p.x + (b * p.x_sb + f * p.x_sf + l * p.x_sl);
    const uint16_t* sr = p.scale + (b * p.scale_sb + f * p.scale_sf + l * p.scale_sl);
    const uint16_t* tr = p.shift + (b * p.shift_sb + f * p.shift_sf + l * p.shift_sl);

    // ---- loads: x, residual and gate are requested together. scale and shift are
    // requested with them or right after the r stores (FN_EARLY_MODULATION_LOADS);
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
    if (FN_EARLY_MODULATION_LOADS && !CACHED_MOD) {
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

    if (!FN_EARLY_MODULATION_LOADS && !CACHED_MOD) {
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
        a2[i] += fma(a, a, c * c);                   // c * c exact (16-bit significand)
      }
    double s1 = (a1[0] + a1[1]) + (a1[2] + a1[3]);
    double s2 = (a2[0] + a2[1]) + (a2[2] + a2[3]);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      if (!IS_RMS) s1 += __shfl_xor_sync(0xFFFFFFFFu, s1, o);
      s2 += __shfl_xor_sync(0xFFFFFFFFu, s2, o);
    }
    if (lane == 0) part[parity][warp] = make_double2(s1, s2);
    __syncthreads();
    double t1 = part[parity][0].x, t2 = part[parity][0].y;
#pragma unroll
    for (int w = 1; w < W; ++w) {
      t1 += part[parity][w].x;
      t2 += part[parity][w].y;
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
      double var = fmax(div_by_row_length<D>(t2) - mu * mu, 0.0);
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
        __syncthreads();  // centred[] is reused by the next such row
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
      if (AFFINE_F32) {
        Affine8 wf{{1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f}}, bf{{0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}};
        if (HAS_WEIGHT) wf = load_affine_f32(p.weight, j);
        if (HAS_BIAS) bf = load_affine_f32(p.bias, j);
        __stcs(yo + j, output_vec_f32<RowShape<D>::kPaired, HAS_WEIGHT, HAS_BIAS>(v[k], sv[k], tv[k], wf, bf, st));
      } else {
        uint4 wv = make_uint4(0, 0, 0, 0), bv = make_uint4(0, 0, 0, 0);
        if (HAS_WEIGHT) wv = __ldg(reinterpret_cast<const uint4*>(p.weight) + j);
        if (HAS_BIAS) bv = __ldg(reinterpret_cast<const uint4*>(p.bias) + j);
        __stcs(yo + j, output_vec<RowShape<D>::kPaired, HAS_WEIGHT, HAS_BIAS>(v[k], sv[k], tv[k], wv, bv, st));
      }
    }
  }
}

template <int D, int VPT, bool IS_RMS, bool NORM_ONLY, bool HAS_GATE, bool HAS_WEIGHT, bool HAS_BIAS,
          bool AFFINE_F32, bool CACHED_MOD>
cudaError_t launch_rows(const RowParams& p, int64_t grid, cudaStream_t stream) {
  constexpr int T = D / (8 * VPT);
  fused_norm_rows<D, VPT, IS_RMS, NORM_ONLY, HAS_GATE, HAS_WEIGHT, HAS_BIAS, AFFINE_F32, CACHED_MOD>
      <<<(unsigned)grid, T, 0, stream>>>(p);
  return cudaGetLastError();
}

// Launcher for one (norm_only, gate, modulation caching) group: the affine combinations.
template <int D, bool RMS, bool NO, bool G, bool CM>
LaunchFn pick_affine(bool w, bool b, bool f32) {
  constexpr int V = RowShape<D>::VPT;
  if (!w && !b) return &launch_rows<D, V, RMS, NO, G, false, false, false, CM>;
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
