// residual.h -- launcher of the residual update between chained layers (residual.cu).
#pragma once

#include <cuda_runtime.h>

#include "coli_moe.h"

namespace coli {

// x_next = x + out for T rows of cfg.hidden: one float32 addition per element, rounded to bf16
// (round to nearest even) for bf16 activations.  x_next may be x.
cudaError_t launch_residual(const coli_moe_config &c, const void *x, const float *out, int T, void *x_next,
                            cudaStream_t st);

}  // namespace coli
