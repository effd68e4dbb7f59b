/*
 * fused_norm.h -- C ABI of the B200 (sm_100a) fused residual / gate / norm /
 * modulation row kernels (libfused_norm.so).
 *
 * The operation (sglang PR #36349 "[AMD][Diffusion] Migrate FlyDSL fused norm
 * kernels to the v0.3.0 stable API", section "Microbenchmark"; sglang PR #33144,
 * same title, sections "Modifications" and "Accuracy Tests"). For every row
 * (b, l) of a (B, L, D) problem, c in [0, D):
 *
 *   r[c] = residual[c] + gate[c] * x[c]          gate = 1 when has_gate == 0
 *   LayerNorm: mu = mean(r), var = mean((r - mu)^2), n = (r - mu) / sqrt(var + eps)
 *   RMSNorm:   ms = mean(r^2),                       n = r / sqrt(ms + eps)
 *   n = n * weight[c]  (has_weight),  n = n + bias[c]  (has_bias)
 *   y[c] = n * (1 + scale[c]) + shift[c]
 *
 * y and r are returned in bf16. r is rounded once, to nearest even, from the exact
 * residual + gate * x, and the norm statistics are taken over that rounded r (the
 * value the caller gets back). Norm-only mode (norm_only = 1, the pages' "norm
 * scale shift" op) has no residual, gate or r: the norm acts on x directly.
 *
 * Data types: every tensor is bf16 (IEEE binary32 truncated to its top 16 bits), except
 * that the affine weight and bias may be fp32 (affine_fp32; the pages' kernel takes fp32
 * affine parameters but casts them to bf16 -- PR 33144, "Known gaps" -- here they are used
 * at full precision).
 * Arithmetic: fp32 for the element-wise work, fp64 for the row statistics. r is the
 * correctly rounded bf16 of the exact residual + gate * x. y is the bf16 rounding of the
 * formula evaluated in fp64 with those statistics: the fp32 value is used where its error
 * bound proves that it rounds the same way, and the other elements (a few in 10^4) are
 * evaluated in fp64 and rounded once. Against the exact value of the formula y is within
 * one bf16 ulp (the fp64 evaluation's own last-bit error can only matter for a value
 * within about 2^-50 of a rounding boundary); on every tested workload it is bit-identical
 * to the fp64 CPU oracle. eps is a runtime value (the pages' kernel hardcodes 1e-6 and
 * ignores the argument; this library does not).
 *
 * Operand layouts (PR #33144, "Modifications": a broadcast operand is a dense
 * (1, C) row selected for every token; "Accuracy Tests": per-row scale/shift and the
 * 4D frame-gate layout). Each gate/scale/shift/x/residual operand is a pointer plus
 * three element strides; the row of token (b, l) starts at
 *
 *   ptr + b * stride_b + (l / tokens_per_frame) * stride_f + l * stride_l
 *
 * and its D channels are contiguous. Common layouts:
 *   broadcast (1, D)        {0, 0, 0}
 *   per-row (B, L, D)       {L*D, 0, D}
 *   per-frame (B, F, 1, D)  {F*D, D, 0}   with tokens_per_frame = L / F
 *   per-batch (B, 1, D)     {D, 0, 0}
 * weight and bias are contiguous (D) vectors.
 *
 * Ownership and threading: the caller owns every buffer and the stream. The
 * library never allocates device memory, never synchronises, and holds no device
 * state; a handle records the chosen specialisation and eps and is immutable after
 * fused_norm_create, so one handle may be used by several host threads and streams
 * at once. fused_norm_launch is asynchronous on the given stream.
 *
 * Errors: argument errors are detected on the host, before anything is launched,
 * and leave every output untouched. FN_ERR_CUDA means the CUDA runtime rejected this
 * call's kernel launch; the runtime's status for that launch is kept per host thread
 * (fused_norm_last_cuda_error). The library links its own copy of the CUDA runtime
 * and reads no error state: an error left pending by an earlier CUDA call, in this
 * library or in the caller's runtime, is neither reported as this launch's failure
 * nor cleared. Launches go to the calling thread's current device, which must be the
 * device that owns the stream and the buffers. There is no fallback path of any kind.
 */
#ifndef FUSED_NORM_H_
#define FUSED_NORM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as the CUDA runtime's cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* fn_stream_t;

typedef enum {
  FN_OK = 0,
  FN_ERR_INVALID_ARG = 1, /* null / inconsistent / negative / overlapping arguments */
  FN_ERR_UNSUPPORTED = 2, /* D not in {5120, 10240} */
  FN_ERR_MISALIGNED = 3,  /* pointer not 16-byte aligned, or stride not a multiple of 8 */
  FN_ERR_CUDA = 4         /* the CUDA runtime rejected this call's kernel launch */
} fn_status;

typedef struct fused_norm_s* fused_norm_t; /* opaque, host-only */

/* Specialisation chosen at create time (compile-time template instance). */
typedef struct {
  int D;          /* channels per row: 5120 or 10240 */
  int is_rms;     /* 0: LayerNorm (mean/variance), 1: RMSNorm */
  int has_gate;   /* 1: r = residual + gate * x; 0: gate-free, r = residual + x */
  int has_weight; /* 1: n *= weight (affine) */
  int has_bias;   /* 1: n += bias (after the weight) */
  int norm_only;  /* 1: no residual, gate or r; normalise x (requires has_gate == 0) */
  int affine_fp32; /* 1: weight and bias are fp32 (D floats each), used at full precision;
                      0: bf16. Needs has_weight or has_bias. */
  double eps;     /* added to the variance / mean-square inside the sqrt; finite, >= 0 */
} fn_config;

/* One row-addressed bf16 input operand (device pointer). Strides in elements. */
typedef struct {
  const void* ptr;
  int64_t stride_b, stride_f, stride_l; /* 0 = broadcast along that axis */
} fn_operand;

typedef struct {
  int64_t B, L;
  int64_t tokens_per_frame;  /* > 0: frame index = l / tokens_per_frame (must divide L);
                                0: no frame axis (every stride_f must then be 0) */
  fn_operand x;              /* required */
  fn_operand residual;       /* required unless norm_only; NULL when norm_only */
  fn_operand gate;           /* NULL iff has_gate == 0 */
  fn_operand scale, shift;   /* required */
  const void* weight;        /* (D) contiguous bf16 (fp32 if affine_fp32); NULL iff has_weight == 0 */
  const void* bias;          /* (D) contiguous bf16 (fp32 if affine_fp32); NULL iff has_bias == 0 */
  void* y;                   /* output (B, L, D) bf16: row (b, l) at y + b*y_stride_b + l*y_stride_l */
  int64_t y_stride_b, y_stride_l;
  void* r;                   /* output, same addressing; NULL when norm_only */
  int64_t r_stride_b, r_stride_l;
} fn_args;

/*
 * Create a handle for one specialisation.
 * Errors: FN_ERR_INVALID_ARG (null pointers, flags not 0/1, eps negative or not
 * finite, norm_only with has_gate, affine_fp32 without weight or bias),
 * FN_ERR_UNSUPPORTED (D not 5120 or 10240).
 * *out is set only on FN_OK. Host only; makes no CUDA call.
 */
fn_status fused_norm_create(fused_norm_t* out, const fn_config* cfg);

/*
 * Check a call without launching anything: every rule fused_norm_launch applies
 * before a launch. Host only; makes no CUDA call and dereferences no device pointer.
 *   FN_ERR_INVALID_ARG: a null handle or args; B, L, tokens_per_frame or a stride
 *     negative; tokens_per_frame not dividing L, or 0 while some stride_f != 0; a
 *     required pointer missing or a pointer present that the specialisation does not
 *     use; output rows that overlap one another (y/r stride_l < D when L > 1, or
 *     stride_b < (L-1)*stride_l + D when B > 1); y and r overlapping each other or
 *     any input, except r == residual exactly (same pointer and strides, stride_f 0),
 *     which updates the residual stream in place; sizes whose byte extents overflow;
 *     B * L of 2^31 rows or more (the kernel runs one thread block per row).
 *   FN_ERR_MISALIGNED: a pointer not 16-byte aligned, or a non-zero stride that is
 *     not a multiple of 8 elements (16 bytes).
 *   B * L == 0 is valid (FN_OK) and reads no pointer.
 */
fn_status fused_norm_validate(fused_norm_t h, const fn_args* a);

/*
 * Validate (as above), then launch the kernel on `stream`. Asynchronous: returns
 * once the launch is queued. B * L == 0 launches nothing. On FN_ERR_CUDA the CUDA
 * error code is kept per host thread (fused_norm_last_cuda_error).
 * One kernel launch per call. Which compiled instance runs depends on the strides as
 * well as on the handle: when scale and shift both have stride_l == 0 (broadcast, per
 * batch or per frame) an instance that re-reads them from cache runs with more rows per
 * SM; the results are the same bits either way.
 */
fn_status fused_norm_launch(fused_norm_t h, const fn_args* a, fn_stream_t stream);

/* Release a handle (NULL is accepted). Never blocks; launches in flight are unaffected. */
fn_status fused_norm_destroy(fused_norm_t h);

/* Copy a handle's configuration. FN_ERR_INVALID_ARG on null arguments. */
fn_status fused_norm_get_config(fused_norm_t h, fn_config* out);

/*
 * The launch the library would issue for these arguments (after validation):
 * grid and block size and dynamic shared memory bytes. For tests and profiling.
 */
fn_status fused_norm_plan(fused_norm_t h, const fn_args* a, int64_t* grid, int* block,
                          size_t* smem_bytes);

/* Static text for a status code; never NULL. */
const char* fused_norm_status_string(fn_status s);

/* cudaError_t (as int) that the runtime returned for the last launch that ended in
 * FN_ERR_CUDA on this host thread; 0 if none. Successful launches leave it as it is. */
int fused_norm_last_cuda_error(void);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int fused_norm_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FUSED_NORM_H_ */
