// Internal declarations shared by the CUDA translation units of libcoli_moe.
// Not part of the public ABI (include/coli_moe.h is).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "coli_moe.h"

namespace coli {

constexpr int kGroup = 64;        // codes per bf16 scale (gs64)
constexpr int kMaxExperts = 1024; // E limit (one union thread per expert)
constexpr int kMaxTopK = 32;      // k limit (one route lane per slot)
constexpr int kMaxShared = 4;
constexpr size_t kHeaderBytes = 16384; // status word + tile counters at the start of ws
constexpr size_t kSlotCntOffset = 1024; // int counters: finished gate/up items per expert slot
constexpr size_t kTileCntOffset = 8192; // int counters: finished down items per 32-row tile
constexpr size_t kBatchCntOffset = 64;  // 2 int counters: tiles handed out by the small-batch
                                        // gate/up and down kernels (zeroed by the preparation)
constexpr int kSmallT = 64;            // calls with T <= kSmallT use the fused prep kernel

// Device status codes live in the first word of the workspace.
struct WsHeader {
    int status;   // first device-detected error (coli_status), 0 = none
    int pad[31];
};

// One expert as the kernels see it (device table, routed then shared).
struct DevExpert {
    const uint8_t* gate_q;   // [I][H/2]
    const uint8_t* up_q;     // [I][H/2]
    const uint8_t* down_q;   // [H][I/2]
    const uint16_t* gate_s;  // [I][H/64] bf16 (per-row format: [I][1])
    const uint16_t* up_s;    // [I][H/64] bf16 (per-row format: [I][1])
    const uint16_t* down_s;  // [H][I/64] bf16 (per-row format: [H][1])
};

// Scale columns of a row of K codes: K / 64 (gs64) or 1 (per-row).
__host__ __device__ inline int scale_cols(int K, int per_row) { return per_row ? 1 : K / kGroup; }

// Byte offsets of the workspace regions for a call with T tokens.
struct WsLayout {
    size_t logits;   // [T][E] f32   (router GEMV output)
    size_t idx;      // [T][k] i32
    size_t w;        // [T][k] f32
    size_t counts;   // [E] i32
    size_t offsets;  // [E+1] i32
    size_t pairs;    // [T*k] i32
    size_t active;   // [E] i32
    size_t n_active; // [1] i32
    size_t inv;      // [T*k] i32: position of pair p in `pairs`
    size_t xp;       // [T][H] f16, fragment-permuted operand copy of x
    size_t corr;     // [T][H/64] f32, unpack-offset sums of each x group
    size_t hp;       // [S][I] f16, fragment-permuted SwiGLU output, S = T*k + T*n_shared
    size_t y;        // [S][H] f32, per-(pair) expert outputs
    size_t xg;       // [T*k + T][H] f16, expert-sorted activations (tensor-core path)
    size_t ntile;    // [E + n_shared + 1] i32, token-tile prefix (tensor-core path)
    size_t ucnt;     // [C][E] i32, per-CTA expert counts of the split batch-union
    size_t total;
};

// The batch-union of T*k >= kUnionSplitPairs pairs runs on C CTAs of
// union_chunk(P) pairs each (a multiple of 1024, at most kUnionMaxCtas CTAs).
constexpr int64_t kUnionSplitPairs = 4096;
constexpr int64_t kUnionMaxCtas = 256;
inline int64_t union_chunk(int64_t P) {
    int64_t c = (P + kUnionMaxCtas - 1) / kUnionMaxCtas;
    c = (c + 1023) / 1024 * 1024;
    return c < 1024 ? 1024 : c;
}
inline int union_ctas(int64_t P) { return (int)((P + union_chunk(P) - 1) / union_chunk(P)); }
inline size_t union_scratch_bytes(int64_t P, int E) {
    return P >= kUnionSplitPairs ? sizeof(int) * (size_t)union_ctas(P) * (size_t)E : 0;
}

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

inline WsLayout ws_layout(int64_t T, int E, int k, int H, int I, int n_shared) {
    WsLayout L;
    size_t o = kHeaderBytes;
    auto take = [&](size_t bytes) {
        size_t r = o;
        o = align_up(o + bytes, 256);
        return r;
    };
    const int64_t P = T * k, S = P + T * n_shared;
    L.logits = take(sizeof(float) * T * E);
    L.idx = take(sizeof(int) * P);
    L.w = take(sizeof(float) * P);
    L.counts = take(sizeof(int) * E);
    L.offsets = take(sizeof(int) * (E + 1));
    L.pairs = take(sizeof(int) * P);
    L.active = take(sizeof(int) * E);
    L.n_active = take(sizeof(int));
    L.inv = take(sizeof(int) * P);
    L.xp = take(sizeof(uint16_t) * T * H);
    L.corr = take(sizeof(float) * T * (H / 64));
    L.hp = take(sizeof(uint16_t) * S * I);
    L.y = take(sizeof(float) * S * H);
    L.xg = take(sizeof(uint16_t) * (P + T) * H);
    L.ntile = take(sizeof(int) * (E + n_shared + 2));
    L.ucnt = take(union_scratch_bytes(P, E));
    L.total = o;
    return L;
}

// Everything the FFN kernels need for one call.
struct FfnArgs {
    const DevExpert* experts;
    int H, I, E, k, n_shared, T;
    const int* offsets;        // [E+1]
    const int* pairs;          // [T*k]
    const int* active;         // [E]
    const int* n_active;       // [1]
    const float* topk_w;       // [T][k]
    const __nv_bfloat16* x;    // [T][H]
    __half* xp;                // [T][H] operand copy of x (fragment order)
    float* corr;               // [T][H/64] unpack-offset sums
    int* inv;                  // [T*k]
    __half* hp;                // [S][I] permuted
    float* y;                  // [S][H]
    const void* residual;      // [T][H] nullable
    void* out;                 // [T][H]
    int out_bf16;
    int per_row;               // scales: one per row instead of one per 64 codes
    int* status;
    int withhold_item;         // test hook: producer never fills this item (-1 = off)
};

// Arguments of the fused small-batch preparation kernel.
struct PrepArgs {
    int T, E, k, H, n_shared;
    const float* logits;      // [T][E]
    int* idx;                 // [T][k] out
    float* w;                 // [T][k] out
    int* counts;              // [E]
    int* offsets;             // [E+1]
    int* pairs;               // [T*k]
    int* active;              // [E]
    int* n_active;            // [1]
    int* inv;                 // [T*k]
    const __nv_bfloat16* x;   // [T][H]
    __half* xp;               // [T][H] operand copy of x
    float* corr;              // [T][H/64]
    int* status;
};

// ---- timing diagnostics (coli_moe_profile_*) ------------------------------
// Returns the event to record at phase boundary `i` (0..4) of the current
// call, or nullptr when profiling is off.
cudaEvent_t profile_event(int i);
inline void profile_mark(int i, cudaStream_t st) {
    if (cudaEvent_t ev = profile_event(i)) cudaEventRecord(ev, st);
}
// Test hook (coli_moe_debug_inject): item index the next FFN launch's producer
// withholds, or -1.  Reading it clears it.
int take_withhold_item();

// ---- launchers (each returns cudaGetLastError() of its launch) ----------
cudaError_t launch_router_logits(int T, int E, int H, const __nv_bfloat16* x, const float* wr,
                                 float* logits, cudaStream_t st);
cudaError_t launch_route(int T, int E, int k, const float* logits, int* idx, float* w,
                         cudaStream_t st);
// `scratch` (nullable, union_scratch_bytes): with it, T*k >= kUnionSplitPairs
// pairs are split over several CTAs (two launches); the lists are the same.
cudaError_t launch_union(int T, int E, int k, const int* idx, int* counts, int* offsets,
                         int* pairs, int* active, int* n_active, int* inv, int* status,
                         int* scratch, cudaStream_t st);
cudaError_t launch_prep_small(const PrepArgs& p, cudaStream_t st);
cudaError_t launch_ffn_stream(const FfnArgs& a, int num_sms, cudaStream_t st);
cudaError_t launch_prepare_x(int T, int H, const __nv_bfloat16* x, __half* xp, float* corr,
                             int* status, cudaStream_t st);
cudaError_t launch_inverse_pairs(int P, const int* pairs, int* inv, int* status, cudaStream_t st);
bool stream_shapes_fit(int H, int I);  // the streaming FFN's 2 stages fit in shared memory
cudaError_t launch_combine(const FfnArgs& a, int num_sms, cudaStream_t st);

// ---- device helpers --------------------------------------------------------
__device__ __forceinline__ void report(int* status, int code) {
    if (status) atomicCAS(status, 0, code);
}

}  // namespace coli
