// Internal interface of the tensor-core prefill path (prefill.cu).
#pragma once

#include <cuda.h>

#include "coli_internal.cuh"

namespace coli {

struct GemmArgs {
    const DevExpert* experts;
    int H, I, E, k, n_shared, T;
    const int* offsets;      // [E+1]
    const int* active;       // [E]
    const int* n_active;     // [1]
    const int* ntile_start;  // [n_slots+1] token tiles before each slot
    const CUtensorMap* wmaps;  // [experts][3] packed gate / up / down codes
    __half* hbuf;            // [S][I] SwiGLU output, operand order
    float* y;                // [S][H]
    int per_row;             // scales: one per row instead of one per 64 codes
    int* status;
};

struct GatherArgs {
    int T, k, E, H, n_shared;
    int bn;                  // token-tile width of the GEMM that follows
    const __nv_bfloat16* x;  // [T][H]
    const int* pairs;        // [T*k]
    const int* offsets;
    const int* active;
    const int* n_active;
    __half* xg;              // [T*k + T][H] expert-sorted activations, operand order
    int* ntile_start;
    int* status;
};

// Tensor maps of every expert's packed code matrices (device array, 3 per
// expert: gate, up, down), boxes of one 64-code K-block (32 bytes) x 128 rows.
// Returns an error if the driver lacks tensor maps.
cudaError_t build_weight_maps(const DevExpert* host_experts, int n, int H, int I,
                              CUtensorMap** d_maps);
// A 2-D map of a row-major byte matrix (rows of row_bytes), boxes of
// box_bytes x box_rows, optionally with the 128-byte swizzle.
bool encode_codes_2d(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows,
                     uint32_t box_bytes, uint32_t box_rows, bool swizzle128);
// gather -> gate/up GEMM -> down GEMM (writes y); the caller runs the combine.
cudaError_t launch_prefill(const FfnArgs& f, const CUtensorMap* wmaps, __half* xg,
                           int* ntile_start, int num_sms, cudaStream_t st);
bool prefill_available();

}  // namespace coli
