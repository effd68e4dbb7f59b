// Template instances for D = 5120, LayerNorm: every (norm_only, gate, weight, bias)
// combination. One translation unit per (D, norm) so they compile in parallel.
#include "fused_norm_kernel.cuh"

FUSED_NORM_DEFINE_SELECTOR(select_launcher_5120_ln, 5120, false)
