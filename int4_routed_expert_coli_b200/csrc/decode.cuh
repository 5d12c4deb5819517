// Internal interface of the fused decode kernel (decode.cu).
#pragma once

#include <cuda.h>

#include "coli_internal.cuh"

namespace coli {

constexpr int kMaxGW = 9;   // gate/up scale groups per consumer warp (H <= 6336)
constexpr int kMaxDW = 3;   // down scale groups per consumer warp (I <= 2112)

struct DecodeArgs {
    FfnArgs f;
    const CUtensorMap* maps;  // [experts][3]: gate, up (8-row boxes), down (32-row box)
};

// True when a call with T tokens can run the fused decode kernel.
bool decode_supported(int H, int I, int T);
// 3-D swizzled tensor maps of every expert's packed code matrices.
cudaError_t build_decode_maps(const DevExpert* host_experts, int n, int H, int I,
                              CUtensorMap** d_maps);
// gate/up + down + combine in one launch; the union, inverse map, operand
// copy of x and zeroed counters must be ready (prep kernel).
cudaError_t launch_decode_fused(const FfnArgs& f, const CUtensorMap* maps, int num_sms,
                                cudaStream_t st);
// Encode a 3-D uint8 tensor map over a [rows][row_bytes] matrix viewed as
// [rows][row_bytes / 128][128], box {128, segs, box_rows}, 128-byte swizzle;
// chunks past the row end read as zero.
bool encode_tma(CUtensorMap* m, const void* base, int rank, int rows, int row_bytes, int segs,
                int box_rows);

}  // namespace coli
