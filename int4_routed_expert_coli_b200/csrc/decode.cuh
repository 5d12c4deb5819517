// Internal interface of the fused decode kernel (decode.cu).
#pragma once

#include <cuda.h>

#include "coli_internal.cuh"

namespace coli {

constexpr int kMaxGW = 6;   // gate/up scale groups per consumer warp (H <= 6144)
constexpr int kMaxDW = 2;   // down scale groups per consumer warp (I <= 2048)

struct DecodeArgs {
    FfnArgs f;                // shapes, experts, x, the union (when logits is null), h rows,
                              // residual, out, status
    // [experts][6]: gate, up (8-row boxes), down (16-row box) codes; then
    // the same three scale matrices (rows padded to 8 x odd bf16 columns)
    const CUtensorMap* maps;
    const float* logits;      // [T][E]: route inside the kernel; null: f holds the union
    int32_t* idx_out;         // [T][k] nullable: the routing (with logits)
    float* w_out;             // [T][k] nullable
    int* sync;                // [0] finished CTAs, [1 + s] finished gate/up tiles of slot s;
                              // zero on entry, left zero on exit
    int max_slots;            // bound on shared + active experts (sizes the slot table)
};

// True when a call with T tokens can run the fused decode kernel on a GPU
// with num_sms SMs.
bool decode_supported(int H, int I, int T, int E, int k, int n_shared, int num_sms);
// Tensor maps of every expert's packed code matrices (3-D, swizzled) and,
// for gs64 (per_row == 0), scale matrices (2-D, padded rows).
cudaError_t build_decode_maps(const DevExpert* host_experts, int n, int H, int I, int per_row,
                              CUtensorMap** d_maps);
// True when at least one CTA of the kernel fits on an SM (so a grid of one
// CTA per SM can be resident at once).
bool decode_coresident(int H, int I, int E, int k, int n_shared, int num_sms);
// Routing (or the given union), gate/up, down and combine in one cooperative
// launch.  Returns cudaErrorCooperativeLaunchTooLarge, with nothing launched
// and the error cleared, when the grid cannot be resident at once (fewer
// usable SMs than the handle saw, e.g. a partitioned GPU): the caller then
// runs the call on another path.
cudaError_t launch_decode_fused(const DecodeArgs& d, int num_sms, cudaStream_t st);
// Test hook: with `on`, the next launch_decode_fused behaves as if the launch
// had been refused for lack of co-resident SMs; false clears it.
void decode_force_not_resident(bool on);
// Encode a 3-D uint8 tensor map over a [rows][row_bytes] matrix viewed as
// [rows][row_bytes / 128][128], box {128, segs, box_rows}, 128-byte swizzle;
// chunks past the row end read as zero.
bool encode_tma(CUtensorMap* m, const void* base, int rank, int rows, int row_bytes, int segs,
                int box_rows);
// Encode a 2-D 16-bit tensor map over a [rows][cols] matrix (cols a multiple
// of 8), box {box_cols, box_rows}; columns past cols read as zero.
bool encode_tma_rows_u16(CUtensorMap* m, const void* base, int rows, int cols, int box_cols,
                         int box_rows);

}  // namespace coli
