// Internal interface of the small-batch expert FFN kernels (batch.cu).
#pragma once

#include <cuda.h>

#include "coli_internal.cuh"

namespace coli {

// Tokens per call the small-batch kernels take (every expert list fits
// eight 8-token MMA column tiles).
constexpr int kBatchMaxTokens = 64;

// True when the small-batch kernels can run a call with T tokens.
bool batch_supported(int H, int I, int T);
// gate/up + SwiGLU (h rows), then down (y rows), over the union lists of a
// call; the activation operand (xp, fragment order) must be ready; the caller
// runs the combine.  wmaps: per-expert code tensor maps (3 per expert,
// 128-row boxes of 128 bytes, 128-byte swizzle).
cudaError_t launch_batch_ffn(const FfnArgs& a, const CUtensorMap* wmaps, int num_sms,
                             cudaStream_t st);

}  // namespace coli
