"""B200 (sm_100a) fused residual / gate / LayerNorm-RMSNorm / modulation row kernels.

The kernels live in libfused_norm.so behind the C ABI of include/fused_norm.h;
this package is a thin binding over it:

* the C entry points under their own names (``fused_norm_create``,
  ``fused_norm_validate``, ``fused_norm_launch``, ``fused_norm_destroy``, ...) and
  the ctypes structures ``fn_config`` / ``fn_operand`` / ``fn_args``;
* tensor-level ops ``fused_residual_norm_scale_shift`` and ``norm_scale_shift``.

The library is loaded on first use: every entry point raises ImportError if it has not
been built (``python -m rmsnorm_row_b200.build``); there is no fallback implementation.
Importing the package does not need it, so the build module can run from a clean tree.
"""
from ._abi import (FN_ERR_CUDA, FN_ERR_INVALID_ARG, FN_ERR_MISALIGNED, FN_ERR_UNSUPPORTED, FN_OK,
                   FusedNormError, fn_args, fn_config, fn_operand, fused_norm_create,
                   fused_norm_destroy, fused_norm_get_config, fused_norm_last_cuda_error,
                   fused_norm_launch, fused_norm_plan, fused_norm_status_string,
                   fused_norm_validate, fused_norm_version, load)
from .api import build_args, fused_residual_norm_scale_shift, norm_scale_shift

__all__ = [
    "FN_OK", "FN_ERR_INVALID_ARG", "FN_ERR_UNSUPPORTED", "FN_ERR_MISALIGNED", "FN_ERR_CUDA",
    "FusedNormError", "fn_args", "fn_config", "fn_operand", "fused_norm_create",
    "fused_norm_destroy", "fused_norm_get_config", "fused_norm_last_cuda_error",
    "fused_norm_launch", "fused_norm_plan", "fused_norm_status_string", "fused_norm_validate",
    "fused_norm_version", "build_args", "fused_residual_norm_scale_shift", "norm_scale_shift",
]
