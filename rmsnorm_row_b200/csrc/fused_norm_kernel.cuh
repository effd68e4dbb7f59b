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
//   * Statistics in fp32: each thread reduces its VPT*8 values locally (two passes
//     for LayerNorm), warps merge with Chan et al.'s pairwise update through
//     xor-shuffles (all lanes end bitwise equal), and warps combine through shared
//     memory in a fixed order after a single barrier. The order never depends on
//     timing, so results are bitwise reproducible.
//   * Per-row (streamed-once) operands use evict-first loads and stores; broadcast
//     and per-frame operands use the read-only cached path (they are re-read by
//     every row and stay in L1/L2).
//   * r is the correctly rounded bf16 of the exact residual + gate * x: gate * x is
//     exact in fp32 (two 8-bit significands), TwoSum recovers the error of the fp32
//     sum, and a sum that lands exactly on a bf16 midpoint is resolved by the sign of
//     that error instead of ties-to-even.
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
  const uint16_t* weight;
  const uint16_t* bias;
  uint16_t* y;
  uint16_t* r;
  int64_t x_sb, x_sf, x_sl;
  int64_t res_sb, res_sf, res_sl;
  int64_t gate_sb, gate_sf, gate_sl;
  int64_t scale_sb, scale_sf, scale_sl;
  int64_t shift_sb, shift_sf, shift_sl;
  int64_t y_sb, y_sl, r_sb, r_sl;
  int64_t L, tpf, rows;
  float eps;
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

__device__ __forceinline__ uint32_t pack_rn(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  uint32_t u;
  memcpy(&u, &h, sizeof(u));
  return u;
}

// bf16 bits of (a + p) rounded once to nearest even, where a + p is the exact real
// sum of two fp32 values (Knuth's TwoSum gives s + e == a + p exactly).
__device__ __forceinline__ uint32_t round_sum_bf16(float a, float p) {
  const float s = __fadd_rn(a, p);
  const float bv = __fsub_rn(s, a);
  const float av = __fsub_rn(s, bv);
  const float e = __fadd_rn(__fsub_rn(a, av), __fsub_rn(p, bv));
  const uint32_t u = __float_as_uint(s);
  const uint32_t rn = __bfloat16_as_ushort(__float2bfloat16_rn(s));
  // s sits on a bf16 midpoint but the exact sum does not (e != 0, not NaN):
  // round towards the exact value.
  const bool tie = ((u & 0xFFFFu) == 0x8000u) && (fabsf(e) > 0.0f);
  const uint32_t toward = ((e > 0.0f) == (s > 0.0f)) ? ((u + 0x8000u) >> 16) : (u >> 16);
  return tie ? toward : rn;
}

// r pair = residual pair + gate pair * x pair
template <bool HAS_GATE>
__device__ __forceinline__ uint32_t residual_pair(uint32_t res, uint32_t x, uint32_t g) {
  float plo = lo_f(x), phi = hi_f(x);
  if (HAS_GATE) {
    plo = __fmul_rn(lo_f(g), plo);  // exact: 8-bit x 8-bit significands
    phi = __fmul_rn(hi_f(g), phi);
  }
  return round_sum_bf16(lo_f(res), plo) | (round_sum_bf16(hi_f(res), phi) << 16);
}

template <int D, int VPT, bool IS_RMS, bool NORM_ONLY, bool HAS_GATE, bool HAS_WEIGHT, bool HAS_BIAS>
__global__ void __launch_bounds__(D / (8 * VPT)) fused_norm_rows(const RowParams p) {
  constexpr int T = D / (8 * VPT);
  constexpr int W = T / 32;
  constexpr int PER_THREAD = VPT * 8;
  static_assert(T % 32 == 0 && T * 8 * VPT == D, "row must split evenly into warps");
  static_assert(!(NORM_ONLY && HAS_GATE), "norm-only has no gate");

  __shared__ float2 part[2][W];
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

    // ---- loads: every streamed operand is requested before the first store, so
    // the row's whole input is in flight at once (stores could alias loads as far
    // as the compiler knows, so loads written after them would wait for them).
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
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      sv[k] = load_vec(sr, tid + k * T, p.stream_mask & kScale);
      tv[k] = load_vec(tr, tid + k * T, p.stream_mask & kShift);
    }

    // ---- step 1: r = residual + gate * x, rounded to bf16, stored -------------
    uint32_t v[VPT][4];  // the row (r, or x when norm-only), packed bf16 pairs
    if (NORM_ONLY) {
#pragma unroll
      for (int k = 0; k < VPT; ++k) {
        v[k][0] = xv[k].x; v[k][1] = xv[k].y; v[k][2] = xv[k].z; v[k][3] = xv[k].w;
      }
    } else {
      uint4* ro = reinterpret_cast<uint4*>(p.r + (b * p.r_sb + l * p.r_sl));
#pragma unroll
      for (int k = 0; k < VPT; ++k) {
        const uint4 g = HAS_GATE ? gv[k] : make_uint4(0, 0, 0, 0);
        v[k][0] = residual_pair<HAS_GATE>(rv[k].x, xv[k].x, g.x);
        v[k][1] = residual_pair<HAS_GATE>(rv[k].y, xv[k].y, g.y);
        v[k][2] = residual_pair<HAS_GATE>(rv[k].z, xv[k].z, g.z);
        v[k][3] = residual_pair<HAS_GATE>(rv[k].w, xv[k].w, g.w);
        __stcs(ro + tid + k * T, make_uint4(v[k][0], v[k][1], v[k][2], v[k][3]));
      }
    }

    // ---- step 2: row statistics --------------------------------------------
    float mean = 0.0f, second;
    if (IS_RMS) {
      float ss = 0.0f;
#pragma unroll
      for (int k = 0; k < VPT; ++k)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float a = lo_f(v[k][q]), c = hi_f(v[k][q]);
          ss = fmaf(a, a, ss);
          ss = fmaf(c, c, ss);
        }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
      if (lane == 0) part[parity][warp] = make_float2(ss, 0.0f);
      __syncthreads();
      float tot = part[parity][0].x;
#pragma unroll
      for (int w = 1; w < W; ++w) tot += part[parity][w].x;
      second = tot / (float)D;
    } else {
      float sum = 0.0f;
#pragma unroll
      for (int k = 0; k < VPT; ++k)
#pragma unroll
        for (int q = 0; q < 4; ++q) sum += lo_f(v[k][q]) + hi_f(v[k][q]);
      float m = sum / (float)PER_THREAD;
      float m2 = 0.0f;
#pragma unroll
      for (int k = 0; k < VPT; ++k)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float a = lo_f(v[k][q]) - m, c = hi_f(v[k][q]) - m;
          m2 = fmaf(a, a, m2);
          m2 = fmaf(c, c, m2);
        }
      // Chan's pairwise merge of equal-count partials; symmetric in the two lanes.
      float half_cnt = 0.5f * (float)PER_THREAD;
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) {
        const float om = __shfl_xor_sync(0xFFFFFFFFu, m, o);
        const float om2 = __shfl_xor_sync(0xFFFFFFFFu, m2, o);
        const float d = om - m;
        m = (m + om) * 0.5f;
        m2 = (m2 + om2) + (d * d) * half_cnt;
        half_cnt *= 2.0f;
      }
      if (lane == 0) part[parity][warp] = make_float2(m, m2);
      __syncthreads();
      // Warps in a fixed order; every thread computes the same result.
      constexpr float kWarpCnt = 32.0f * PER_THREAD;
      float2 acc = part[parity][0];
#pragma unroll
      for (int w = 1; w < W; ++w) {
        const float2 o = part[parity][w];
        const float na = kWarpCnt * (float)w;
        const float frac = kWarpCnt / (na + kWarpCnt);
        const float d = o.x - acc.x;
        acc.x = acc.x + d * frac;
        acc.y = (acc.y + o.y) + (d * d) * (na * frac);
      }
      mean = acc.x;
      second = acc.y / (float)D;
    }
    const float rho = 1.0f / sqrtf(second + p.eps);

    // ---- step 3: normalise, affine, modulate, store y ------------------------
    uint4* yo = reinterpret_cast<uint4*>(p.y + (b * p.y_sb + l * p.y_sl));
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      const int j = tid + k * T;
      uint4 wv = make_uint4(0, 0, 0, 0), bv = make_uint4(0, 0, 0, 0);
      if (HAS_WEIGHT) wv = __ldg(reinterpret_cast<const uint4*>(p.weight) + j);
      if (HAS_BIAS) bv = __ldg(reinterpret_cast<const uint4*>(p.bias) + j);
      const uint32_t sw[4] = {sv[k].x, sv[k].y, sv[k].z, sv[k].w};
      const uint32_t tw[4] = {tv[k].x, tv[k].y, tv[k].z, tv[k].w};
      const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
      const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
      uint32_t out[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float n0 = (lo_f(v[k][q]) - mean) * rho;
        float n1 = (hi_f(v[k][q]) - mean) * rho;
        if (HAS_WEIGHT && HAS_BIAS) {
          n0 = fmaf(n0, lo_f(ww[q]), lo_f(bw[q]));
          n1 = fmaf(n1, hi_f(ww[q]), hi_f(bw[q]));
        } else if (HAS_WEIGHT) {
          n0 *= lo_f(ww[q]);
          n1 *= hi_f(ww[q]);
        } else if (HAS_BIAS) {
          n0 += lo_f(bw[q]);
          n1 += hi_f(bw[q]);
        }
        const float y0 = fmaf(n0, 1.0f + lo_f(sw[q]), lo_f(tw[q]));
        const float y1 = fmaf(n1, 1.0f + hi_f(sw[q]), hi_f(tw[q]));
        out[q] = pack_rn(y0, y1);
      }
      __stcs(yo + j, make_uint4(out[0], out[1], out[2], out[3]));
    }
  }
}

template <int D, int VPT, bool IS_RMS, bool NORM_ONLY, bool HAS_GATE, bool HAS_WEIGHT, bool HAS_BIAS>
cudaError_t launch_rows(const RowParams& p, int64_t grid, cudaStream_t stream) {
  constexpr int T = D / (8 * VPT);
  fused_norm_rows<D, VPT, IS_RMS, NORM_ONLY, HAS_GATE, HAS_WEIGHT, HAS_BIAS>
      <<<(unsigned)grid, T, 0, stream>>>(p);
  return cudaGetLastError();
}

// Threads per row and vectors per thread, per D.
template <int D> struct RowShape;
template <> struct RowShape<5120> { static constexpr int VPT = 4; };
template <> struct RowShape<10240> { static constexpr int VPT = 4; };

// Launcher for a specialisation, selected at create time. Defined in one
// translation unit per (D, norm type) so the instances compile in parallel.
LaunchFn select_launcher(int D, bool is_rms, bool norm_only, bool has_gate, bool has_weight,
                         bool has_bias);
LaunchFn select_launcher_5120_ln(bool norm_only, bool has_gate, bool has_weight, bool has_bias);
LaunchFn select_launcher_5120_rms(bool norm_only, bool has_gate, bool has_weight, bool has_bias);
LaunchFn select_launcher_10240_ln(bool norm_only, bool has_gate, bool has_weight, bool has_bias);
LaunchFn select_launcher_10240_rms(bool norm_only, bool has_gate, bool has_weight, bool has_bias);

}  // namespace fused_norm_impl

// Instantiates the 12 (norm_only, gate, weight, bias) launchers for one (D, norm).
#define FUSED_NORM_DEFINE_SELECTOR(NAME, D_, RMS_)                                              \
  namespace fused_norm_impl {                                                                   \
  LaunchFn NAME(bool norm_only, bool has_gate, bool has_weight, bool has_bias) {                \
    constexpr int V = RowShape<D_>::VPT;                                                        \
    if (norm_only) {                                                                            \
      if (has_weight)                                                                           \
        return has_bias ? &launch_rows<D_, V, RMS_, true, false, true, true>                    \
                        : &launch_rows<D_, V, RMS_, true, false, true, false>;                  \
      return has_bias ? &launch_rows<D_, V, RMS_, true, false, false, true>                     \
                      : &launch_rows<D_, V, RMS_, true, false, false, false>;                   \
    }                                                                                           \
    if (has_gate) {                                                                             \
      if (has_weight)                                                                           \
        return has_bias ? &launch_rows<D_, V, RMS_, false, true, true, true>                    \
                        : &launch_rows<D_, V, RMS_, false, true, true, false>;                  \
      return has_bias ? &launch_rows<D_, V, RMS_, false, true, false, true>                     \
                      : &launch_rows<D_, V, RMS_, false, true, false, false>;                   \
    }                                                                                           \
    if (has_weight)                                                                             \
      return has_bias ? &launch_rows<D_, V, RMS_, false, false, true, true>                     \
                      : &launch_rows<D_, V, RMS_, false, false, true, false>;                   \
    return has_bias ? &launch_rows<D_, V, RMS_, false, false, false, true>                      \
                    : &launch_rows<D_, V, RMS_, false, false, false, false>;                    \
  }                                                                                             \
  }
