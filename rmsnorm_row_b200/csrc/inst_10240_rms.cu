// Template instances for D = 10240, RMSNorm: every (norm_only, gate, weight, bias)
// combination. One translation unit per (D, norm) so they compile in parallel.
#include "fused_norm_kernel.cuh"

FUSED_NORM_DEFINE_SELECTOR(select_launcher_10240_rms, 10240, true)
