// C ABI of libfused_norm.so: handle management, argument validation, operand
// resolution and kernel launch. Declarations and the contract: include/fused_norm.h.
//
// Operand resolution follows sglang PR #33144 "[Diffusion] Migrate FlyDSL fused
// norm kernels to the v0.3.0 stable API", section "Modifications" (a broadcast
// operand is a dense (1, C) row selected for every token) and "Accuracy Tests"
// (per-row scale/shift, 4D frame-gate layout): each operand is a pointer and three
// element strides, and stride 0 broadcasts along that axis. Unlike the pages'
// kernel, a (B, 1, D) per-batch operand works too (its "Known gaps" lists 2D
// [B, C] broadcasting as incorrect there), eps is honoured, and an empty problem is
// a valid no-op.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <new>

#include "../../include/fused_norm.h"
#include "fused_norm_kernel.cuh"

using namespace fused_norm_impl;

struct fused_norm_s {
  fn_config cfg;
  LaunchFn launch;            // scale or shift changes from token to token
  LaunchFn launch_cached_mod;  // scale and shift both broadcast, per batch or per frame
  int threads, threads_cached_mod;
};

namespace {

thread_local int g_last_cuda_error = 0;

constexpr int64_t kMaxExtent = (int64_t)1 << 46;  // elements; keeps byte math in int64
constexpr int64_t kMaxRows = 0x7FFFFFFFLL;       // B * L: one CTA per row, 32-bit row indices

bool is_flag(int v) { return v == 0 || v == 1; }

struct Span {
  uintptr_t lo, hi;  // [lo, hi) in bytes; empty when lo == hi
};

bool overlaps(const Span& a, const Span& b) { return a.lo < b.hi && b.lo < a.hi; }

// Largest element offset (exclusive end) an operand row set can touch, or -1 on overflow.
int64_t operand_extent(int64_t B, int64_t L, int64_t F, int64_t D, int64_t sb, int64_t sf,
                       int64_t sl) {
  __int128 end = (__int128)(B - 1) * sb + (__int128)(F - 1) * sf + (__int128)(L - 1) * sl + D;
  if (end > kMaxExtent) return -1;
  return (int64_t)end;
}

fn_status check_operand(const fn_operand& o, bool frame_axis) {
  if (o.stride_b < 0 || o.stride_f < 0 || o.stride_l < 0) return FN_ERR_INVALID_ARG;
  if (!frame_axis && o.stride_f != 0) return FN_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(o.ptr) % 16 != 0) return FN_ERR_MISALIGNED;
  if (o.stride_b % 8 || o.stride_f % 8 || o.stride_l % 8) return FN_ERR_MISALIGNED;
  return FN_OK;
}

fn_status check_output(const void* ptr, int64_t sb, int64_t sl, int64_t B, int64_t L, int64_t D) {
  if (sb < 0 || sl < 0) return FN_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(ptr) % 16 != 0) return FN_ERR_MISALIGNED;
  if (sb % 8 || sl % 8) return FN_ERR_MISALIGNED;
  // rows must not overlap one another (rows are written concurrently)
  if (L > 1 && sl < D) return FN_ERR_INVALID_ARG;
  if (B > 1 && (__int128)sb < (__int128)(L - 1) * sl + D) return FN_ERR_INVALID_ARG;
  return FN_OK;
}

#define FN_TRY(expr)                   \
  do {                                 \
    fn_status s_ = (expr);             \
    if (s_ != FN_OK) return s_;        \
  } while (0)

fn_status validate(const fused_norm_s* h, const fn_args* a) {
  if (!h || !a) return FN_ERR_INVALID_ARG;
  const fn_config& c = h->cfg;
  const int64_t D = c.D, B = a->B, L = a->L, tpf = a->tokens_per_frame;
  if (B < 0 || L < 0 || tpf < 0) return FN_ERR_INVALID_ARG;
  if (B == 0 || L == 0) return FN_OK;  // empty problem: nothing is read or written
  if (B > kMaxExtent || L > kMaxExtent || (__int128)B * L * D > kMaxExtent) return FN_ERR_INVALID_ARG;
  if ((__int128)B * L > (__int128)kMaxRows) return FN_ERR_INVALID_ARG;
  if (tpf > 0 && L % tpf != 0) return FN_ERR_INVALID_ARG;
  const bool frame_axis = tpf > 0;
  const int64_t F = frame_axis ? L / tpf : 1;

  // presence of pointers must match the specialisation
  if (!a->x.ptr || !a->scale.ptr || !a->shift.ptr || !a->y) return FN_ERR_INVALID_ARG;
  if (c.norm_only) {
    if (a->residual.ptr || a->gate.ptr || a->r) return FN_ERR_INVALID_ARG;
  } else {
    if (!a->residual.ptr || !a->r) return FN_ERR_INVALID_ARG;
    if ((a->gate.ptr != nullptr) != (c.has_gate != 0)) return FN_ERR_INVALID_ARG;
  }
  if ((a->weight != nullptr) != (c.has_weight != 0)) return FN_ERR_INVALID_ARG;
  if ((a->bias != nullptr) != (c.has_bias != 0)) return FN_ERR_INVALID_ARG;

  // strides, alignment: inputs. Negative values first (INVALID_ARG), then alignment.
  const fn_operand* ins[5] = {&a->x, &a->residual, &a->gate, &a->scale, &a->shift};
  fn_status worst = FN_OK;
  for (const fn_operand* o : ins) {
    if (!o->ptr) continue;
    fn_status s = check_operand(*o, frame_axis);
    if (s == FN_ERR_INVALID_ARG) return s;
    if (s != FN_OK) worst = s;
  }
  for (const void* v : {a->weight, a->bias})
    if (v && reinterpret_cast<uintptr_t>(v) % 16 != 0) worst = FN_ERR_MISALIGNED;
  fn_status sy = check_output(a->y, a->y_stride_b, a->y_stride_l, B, L, D);
  if (sy == FN_ERR_INVALID_ARG) return sy;
  if (sy != FN_OK) worst = sy;
  if (!c.norm_only) {
    fn_status sr = check_output(a->r, a->r_stride_b, a->r_stride_l, B, L, D);
    if (sr == FN_ERR_INVALID_ARG) return sr;
    if (sr != FN_OK) worst = sr;
  }
  if (worst != FN_OK) return worst;

  // byte spans of every buffer, for the overlap rules
  auto in_span = [&](const fn_operand& o, Span* out) -> bool {
    int64_t e = operand_extent(B, L, F, D, o.stride_b, o.stride_f, o.stride_l);
    if (e < 0) return false;
    uintptr_t lo = reinterpret_cast<uintptr_t>(o.ptr);
    *out = Span{lo, lo + (uintptr_t)e * 2};
    return true;
  };
  Span in[7];
  int n_in = 0;
  for (const fn_operand* o : ins) {
    if (!o->ptr) continue;
    if (!in_span(*o, &in[n_in++])) return FN_ERR_INVALID_ARG;
  }
  const uintptr_t affine_bytes = (uintptr_t)D * (c.affine_fp32 ? 4 : 2);
  for (const void* v : {a->weight, a->bias}) {
    if (!v) continue;
    uintptr_t lo = reinterpret_cast<uintptr_t>(v);
    in[n_in++] = Span{lo, lo + affine_bytes};
  }
  int64_t ye = operand_extent(B, L, 1, D, a->y_stride_b, 0, a->y_stride_l);
  if (ye < 0) return FN_ERR_INVALID_ARG;
  Span ys{reinterpret_cast<uintptr_t>(a->y), reinterpret_cast<uintptr_t>(a->y) + (uintptr_t)ye * 2};
  for (int i = 0; i < n_in; ++i)
    if (overlaps(ys, in[i])) return FN_ERR_INVALID_ARG;
  if (!c.norm_only) {
    int64_t re = operand_extent(B, L, 1, D, a->r_stride_b, 0, a->r_stride_l);
    if (re < 0) return FN_ERR_INVALID_ARG;
    Span rs{reinterpret_cast<uintptr_t>(a->r), reinterpret_cast<uintptr_t>(a->r) + (uintptr_t)re * 2};
    if (overlaps(rs, ys)) return FN_ERR_INVALID_ARG;
    // r may be the residual itself, element for element (in-place residual update):
    // each element is read and then written by the same thread.
    const bool in_place = a->r == a->residual.ptr && a->residual.stride_f == 0 &&
                          (a->residual.stride_b == a->r_stride_b || B == 1) &&
                          (a->residual.stride_l == a->r_stride_l || L == 1);
    int k = 0;
    for (const fn_operand* o : ins) {
      if (!o->ptr) continue;
      const Span& s = in[k++];
      if (o == &a->residual && in_place) continue;
      if (overlaps(rs, s)) return FN_ERR_INVALID_ARG;
    }
    for (; k < n_in; ++k)
      if (overlaps(rs, in[k])) return FN_ERR_INVALID_ARG;
  }
  return FN_OK;
}

RowParams make_params(const fused_norm_s* h, const fn_args* a) {
  RowParams p;
  std::memset(&p, 0, sizeof(p));
  auto u16 = [](const void* v) { return static_cast<const uint16_t*>(v); };
  auto raw = [](const void* v) { return v; };
  p.x = u16(a->x.ptr);
  p.res = u16(a->residual.ptr);
  p.gate = u16(a->gate.ptr);
  p.scale = u16(a->scale.ptr);
  p.shift = u16(a->shift.ptr);
  p.weight = raw(a->weight);
  p.bias = raw(a->bias);
  p.y = static_cast<uint16_t*>(a->y);
  p.r = static_cast<uint16_t*>(a->r);
  p.x_sb = a->x.stride_b; p.x_sf = a->x.stride_f; p.x_sl = a->x.stride_l;
  p.res_sb = a->residual.stride_b; p.res_sf = a->residual.stride_f; p.res_sl = a->residual.stride_l;
  p.gate_sb = a->gate.stride_b; p.gate_sf = a->gate.stride_f; p.gate_sl = a->gate.stride_l;
  p.scale_sb = a->scale.stride_b; p.scale_sf = a->scale.stride_f; p.scale_sl = a->scale.stride_l;
  p.shift_sb = a->shift.stride_b; p.shift_sf = a->shift.stride_f; p.shift_sl = a->shift.stride_l;
  p.y_sb = a->y_stride_b; p.y_sl = a->y_stride_l;
  p.r_sb = a->r_stride_b; p.r_sl = a->r_stride_l;
  p.L = (uint32_t)a->L;
  p.tpf = (uint32_t)a->tokens_per_frame;
  p.rows = (uint32_t)(a->B * a->L);
  p.div_L = make_div_u32(p.L);
  p.div_tpf = make_div_u32(p.tpf > 0 ? p.tpf : 1u);
  p.eps = h->cfg.eps;
  // An operand that changes from token to token (stride_l != 0) is read once per
  // call: stream it. Broadcast, per-batch and per-frame rows are re-read by many
  // tokens: keep them cached.
  uint32_t m = 0;
  if (a->x.stride_l) m |= kX;
  if (a->residual.stride_l) m |= kRes;
  if (a->gate.stride_l) m |= kGate;
  if (a->scale.stride_l) m |= kScale;
  if (a->shift.stride_l) m |= kShift;
  p.stream_mask = m;
  return p;
}

int64_t grid_for(int64_t rows) { return rows; }  // one CTA per row (B * L <= kMaxRows)

}  // namespace

namespace fused_norm_impl {
LaunchFn select_launcher(int D, bool is_rms, bool norm_only, bool has_gate, bool has_weight,
                         bool has_bias, bool f32, bool cm) {
  if (D == 5120)
    return is_rms ? select_launcher_5120_rms(norm_only, has_gate, has_weight, has_bias, f32, cm)
                  : select_launcher_5120_ln(norm_only, has_gate, has_weight, has_bias, f32, cm);
  if (D == 10240)
    return is_rms ? select_launcher_10240_rms(norm_only, has_gate, has_weight, has_bias, f32, cm)
                  : select_launcher_10240_ln(norm_only, has_gate, has_weight, has_bias, f32, cm);
  return nullptr;
}
}  // namespace fused_norm_impl

extern "C" {

fn_status fused_norm_create(fused_norm_t* out, const fn_config* cfg) {
  if (!out || !cfg) return FN_ERR_INVALID_ARG;
  const fn_config& c = *cfg;
  if (!is_flag(c.is_rms) || !is_flag(c.has_gate) || !is_flag(c.has_weight) ||
      !is_flag(c.has_bias) || !is_flag(c.norm_only) || !is_flag(c.affine_fp32))
    return FN_ERR_INVALID_ARG;
  if (c.affine_fp32 && !c.has_weight && !c.has_bias) return FN_ERR_INVALID_ARG;
  if (!std::isfinite(c.eps) || c.eps < 0.0) return FN_ERR_INVALID_ARG;
  if (c.norm_only && c.has_gate) return FN_ERR_INVALID_ARG;
  if (c.D != 5120 && c.D != 10240) return FN_ERR_UNSUPPORTED;
  LaunchFn fn = select_launcher(c.D, c.is_rms, c.norm_only, c.has_gate, c.has_weight, c.has_bias,
                                c.affine_fp32, false);
  LaunchFn fn_cm = select_launcher(c.D, c.is_rms, c.norm_only, c.has_gate, c.has_weight, c.has_bias,
                                   c.affine_fp32, true);
  if (!fn || !fn_cm) return FN_ERR_UNSUPPORTED;
  fused_norm_s* h = new (std::nothrow) fused_norm_s;
  if (!h) return FN_ERR_INVALID_ARG;
  h->cfg = c;
  h->launch = fn;
  h->launch_cached_mod = fn_cm;
  const bool affine = c.has_weight || c.has_bias;
  for (int cm = 0; cm < 2; ++cm) {
    const int vpt = c.D == 5120 ? vpt_of<5120>(c.norm_only, cm, affine) : vpt_of<10240>(c.norm_only, cm, affine);
    (cm ? h->threads_cached_mod : h->threads) = c.D / (8 * vpt);
  }
  *out = h;
  return FN_OK;
}

fn_status fused_norm_validate(fused_norm_t h, const fn_args* a) { return validate(h, a); }

fn_status fused_norm_plan(fused_norm_t h, const fn_args* a, int64_t* grid, int* block,
                          size_t* smem_bytes) {
  FN_TRY(validate(h, a));
  if (!grid || !block || !smem_bytes) return FN_ERR_INVALID_ARG;
  *grid = grid_for(a->B * a->L);
  *block = (a->scale.stride_l == 0 && a->shift.stride_l == 0) ? h->threads_cached_mod : h->threads;
  *smem_bytes = 0;
  return FN_OK;
}

fn_status fused_norm_launch(fused_norm_t h, const fn_args* a, fn_stream_t stream) {
  FN_TRY(validate(h, a));
  const int64_t rows = a->B * a->L;
  if (rows == 0) return FN_OK;
  RowParams p = make_params(h, a);
  const bool cached_mod = a->scale.stride_l == 0 && a->shift.stride_l == 0;
  cudaError_t e = (cached_mod ? h->launch_cached_mod : h->launch)(p, grid_for(a->B * a->L),
                                                                  reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    g_last_cuda_error = (int)e;
    return FN_ERR_CUDA;
  }
  return FN_OK;
}

fn_status fused_norm_destroy(fused_norm_t h) {
  delete h;
  return FN_OK;
}

fn_status fused_norm_get_config(fused_norm_t h, fn_config* out) {
  if (!h || !out) return FN_ERR_INVALID_ARG;
  *out = h->cfg;
  return FN_OK;
}

const char* fused_norm_status_string(fn_status s) {
  switch (s) {
    case FN_OK: return "ok";
    case FN_ERR_INVALID_ARG: return "invalid argument";
    case FN_ERR_UNSUPPORTED: return "unsupported configuration (D must be 5120 or 10240)";
    case FN_ERR_MISALIGNED: return "misaligned pointer or stride (16-byte rows required)";
    case FN_ERR_CUDA: return "CUDA launch error";
  }
  return "unknown status";
}

int fused_norm_last_cuda_error(void) { return g_last_cuda_error; }

int fused_norm_version(void) { return 10000; }

}  // extern "C"
