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
// runs the combine.  bmaps: build_batch_maps's tensor maps.
cudaError_t launch_batch_ffn(const FfnArgs& a, const CUtensorMap* bmaps, int num_sms,
                             cudaStream_t st);
// The small-batch kernels' tensor maps (device array, 6 per expert): gate,
// up and down codes in boxes of 128 rows x 128 bytes (four K-blocks, 128-byte
// swizzle); gate, up and down scales in boxes of 128 rows x 8 scales where a
// scale row is whole 16-byte chunks (gs64 with K / 64 a multiple of 8), else
// zeroed (those kernels then read scales from global memory).
cudaError_t build_batch_maps(const DevExpert* host_experts, int n, int H, int I, bool per_row,
                             CUtensorMap** d_maps);

}  // namespace coli
