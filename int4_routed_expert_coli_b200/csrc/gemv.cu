// Expert FFN for decode and small batches: int4 gs64 dequant-GEMV on tensor
// cores with the weights streamed from HBM exactly once per call
// ("batch-union", "yunpan.plus/t/30351-1-1", capability two).
//
// Work.  An item is (expert slot, row tile of a weight matrix).  The shared
// experts come first in slot order, so their weights stream while the
// routing of the call is still running (programmatic dependent launch); the
// active routed experts follow.  A gate/up item is 8 gate rows and the same
// 8 up rows (one m16 MMA tile), so each thread ends with g and u of one
// (token, n) and forms the SwiGLU output in registers.  A down item is 32
// consecutive rows of W_d (two m16 tiles sharing the activation fragments).
//
// Data movement.  One CTA per SM.  A producer warp copies each item's rows
// (one bulk copy per row, into rows padded by 32 bytes so fragment reads do
// not conflict on banks) and its scale rows into a ring of stages; an
// mbarrier per stage carries the byte count.  Sixteen consumer warps split
// the reduction dimension of the item.  HBM sees only whole, contiguous,
// read-once weight rows.
//
// Arithmetic.  Codes are exact in fp16, activations are fp16 operands,
// products are exact, accumulation is fp32 (m16n8k16 MMA), and the gs64
// scale multiplies each 64-group's fp32 partial sum:
//   g[n] = sum_groups s[n][grp] * (sum_{k in grp} q[n][k] x[k]).
// Unpack: 0x6400 | n is the fp16 value 1024 + n.  For down the codes are
// made exact (subtract 1032; the high nibble, placed as 1024 + 16 n, comes
// back with v / 16 - 72).  For gate/up the subtraction is skipped: even codes
// enter as 1032 + q and odd codes as 1152 + 16 q against x_odd / 16, so the
// MMA yields sum q x plus a per-(token, group) offset that the preparation
// step computed from the same fp16 operand values; it is subtracted before
// the scale.  This halves the unpack work of the dominant kernel.
//
// K order.  The 16 k-slots a lane feeds to one m16n8k16 MMA come from 16
// consecutive codes of its row (8 bytes) in the order the unpack produces
// them; the activation operands (xp, hp) are stored in that same order.
//
// The fp32 outputs y of every (token, slot) are combined per token by a
// small kernel chained to the down kernel:
//   out[t] = sum_j w[t][j] y[(t,j)] (j ascending) + y_shared[t] (+ residual[t])
// in fp32, in that fixed order, so results do not depend on timing.
#include <algorithm>

#include "moe_device.cuh"
#include "ptx.cuh"

namespace coli {
namespace {

constexpr int kConsumerWarps = 16;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;  // + producer warp
constexpr int kMaxStages = 16;
constexpr int kFixedSmem = 512;            // barriers, flags, token row map
constexpr int kSmemLimit = 227 * 1024;

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
    return __uint_as_float((uint32_t)b << 16);
}

// Raw unpack of one word (codes k = 0..7 of a slice) into four fp16 pairs
// (0,4) (1,5) (2,6) (3,7): even codes as 1032 + q, odd codes as 1152 + 16 q.
__device__ __forceinline__ void unpack_raw(uint32_t w, uint32_t o[4]) {
    const uint32_t w8 = w >> 8;
    o[0] = (w & 0x000F000Fu) ^ 0x64086408u;
    o[1] = (w & 0x00F000F0u) ^ 0x64806480u;
    o[2] = (w8 & 0x000F000Fu) ^ 0x64086408u;
    o[3] = (w8 & 0x00F000F0u) ^ 0x64806480u;
}

// Exact unpack: the same four pairs as the codes q themselves.
__device__ __forceinline__ void unpack_exact(uint32_t w, uint32_t o[4]) {
    const __half2 bias_lo = __floats2half2_rn(1032.f, 1032.f);
    const __half2 sixteenth = __floats2half2_rn(0.0625f, 0.0625f);
    const __half2 bias_hi = __floats2half2_rn(-72.f, -72.f);
    uint32_t t[4];
    unpack_raw(w, t);
    __half2 v0 = __hsub2(*reinterpret_cast<__half2*>(&t[0]), bias_lo);
    __half2 v1 = __hfma2(*reinterpret_cast<__half2*>(&t[1]), sixteenth, bias_hi);
    __half2 v2 = __hsub2(*reinterpret_cast<__half2*>(&t[2]), bias_lo);
    __half2 v3 = __hfma2(*reinterpret_cast<__half2*>(&t[3]), sixteenth, bias_hi);
    o[0] = *reinterpret_cast<uint32_t*>(&v0);
    o[1] = *reinterpret_cast<uint32_t*>(&v1);
    o[2] = *reinterpret_cast<uint32_t*>(&v2);
    o[3] = *reinterpret_cast<uint32_t*>(&v3);
}

// d = A B + c, m16n8k16, fp16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma16816(float d[4], const float c[4], uint32_t a0, uint32_t a1,
                                         uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, "
        "{%4,%5,%6,%7}, {%8,%9}, {%10,%11,%12,%13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(c[2]),
          "f"(c[3]));
}

// Partial sum of one 64-group for one m16 tile: 4 MMAs over the group's codes
// (rows r: words wa, rows r + 8: words wb) against B fragments bw[8].
template <bool kExact>
__device__ __forceinline__ void group_partial(float part[4], uint2 wa, uint2 wb,
                                              const uint32_t bw[8]) {
    uint32_t aa[8], ab[8];
    if constexpr (kExact) {
        unpack_exact(wa.x, aa);
        unpack_exact(wa.y, aa + 4);
        unpack_exact(wb.x, ab);
        unpack_exact(wb.y, ab + 4);
    } else {
        unpack_raw(wa.x, aa);
        unpack_raw(wa.y, aa + 4);
        unpack_raw(wb.x, ab);
        unpack_raw(wb.y, ab + 4);
    }
    const float zero[4] = {0.f, 0.f, 0.f, 0.f};
    float p0[4], p1[4];
    // two independent chains, then one add
    mma16816(p0, zero, aa[0], ab[0], aa[1], ab[1], bw[0], bw[1]);
    mma16816(p1, zero, aa[2], ab[2], aa[3], ab[3], bw[2], bw[3]);
    mma16816(p0, p0, aa[4], ab[4], aa[5], ab[5], bw[4], bw[5]);
    mma16816(p1, p1, aa[6], ab[6], aa[7], ab[7], bw[6], bw[7]);
#pragma unroll
    for (int q = 0; q < 4; ++q) part[q] = p0[q] + p1[q];
}

__device__ __forceinline__ void load_b(uint32_t bw[8], const __half* p) {
    const uint4 b0 = __ldg(reinterpret_cast<const uint4*>(p));
    const uint4 b1 = __ldg(reinterpret_cast<const uint4*>(p) + 1);
    bw[0] = b0.x; bw[1] = b0.y; bw[2] = b0.z; bw[3] = b0.w;
    bw[4] = b1.x; bw[5] = b1.y; bw[6] = b1.z; bw[7] = b1.w;
}

// Geometry of one kernel kind.
struct Geo {
    int K;           // reduction length (H for gate/up, I for down)
    int G;           // 64-groups per row, K / 64 (offset sums are per group)
    int SG;          // scale columns per row: G (gs64) or 1 (per-row format)
    int gs;          // scale column step per group: 1 (gs64) or 0 (per-row)
    int rows;        // staged rows per item: 16 * MT
    int row_stride;  // bytes per staged row: K/2 + 32
    int scale_off;   // offset of the scale block ([rows][SG] bf16) in a stage
    int stage_bytes;
    int tiles;       // items per expert
};

inline Geo make_geo(int K, int rows, int tiles, int per_row) {
    Geo g;
    g.K = K;
    g.G = K / kGroup;
    g.SG = scale_cols(K, per_row);
    g.gs = per_row ? 0 : 1;
    g.rows = rows;
    g.row_stride = K / 2 + 32;
    g.scale_off = rows * g.row_stride;
    g.stage_bytes = g.scale_off + (int)align_up((size_t)rows * g.SG * 2, 16);
    g.tiles = tiles;
    return g;
}

// Shared memory ahead of the stages: barriers and flags, the cross-warp
// reduction buffer, and (kAll) the offset sums of up to 8 tokens.
__host__ __device__ inline int fixed_smem_bytes(int MT, int NT, bool all, int G) {
    return kFixedSmem + kConsumerWarps * MT * NT * 4 * 32 * 4 + (all ? (8 * G * 4 + 127) / 128 * 128 : 0);
}

struct Slot {
    int e;           // expert row in the device table
    int list_begin;  // first output row (hp / y) of this expert
    int ntok;        // tokens on its list
    bool shared;
    bool valid;
};

// Slot order: shared experts first, then the active routed experts.
__device__ __forceinline__ Slot decode_slot(const FfnArgs& a, int slot, int n_act) {
    Slot s;
    const int P = a.T * a.k;
    s.valid = true;
    if (slot < a.n_shared) {
        s.e = a.E + slot;
        s.list_begin = P + slot * a.T;
        s.ntok = a.T;
        s.shared = true;
        return s;
    }
    s.shared = false;
    const int r = slot - a.n_shared;
    const int e = r < n_act ? a.active[r] : -1;
    int b = 0, en = 0;
    if (e >= 0 && e < a.E) {
        b = a.offsets[e];
        en = a.offsets[e + 1];
    }
    if (e < 0 || e >= a.E || b < 0 || en < b || en > P) {
        s.valid = false;
        s.e = 0;
        s.list_begin = 0;
        s.ntok = 0;
        return s;
    }
    s.e = e;
    s.list_begin = b;
    s.ntok = en - b;
    return s;
}

__device__ __forceinline__ int read_n_active(const FfnArgs& a) {
    const int n = *reinterpret_cast<const volatile int*>(a.n_active);
    if (n < 0 || n > a.E) {
        report(a.status, COLI_ERR_BAD_INDEX);
        return 0;
    }
    return n;
}

// ---------------------------------------------------------------------------
// The streaming FFN kernel.
//   kGU  : gate/up + SwiGLU (writes hp) / down (writes y)
//   MT   : m16 tiles per item (gate/up 1, down 2)
//   NT   : N-tiles of 8 tokens per pass (token-list path)
//   kAll : T <= 8: every item uses all T tokens as the 8 MMA columns, so the
//          activation fragments are loop-invariant and live in registers
//          (KW = groups per warp it can hold); outputs are written only for
//          the tokens on the item's list.
template <bool kGU, int MT, int NT, bool kAll, int KW>
__global__ void __launch_bounds__(kThreads, 1)
stream_ffn_kernel(const FfnArgs a, const Geo g, int stages) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kMaxStages;
    volatile int* flags = reinterpret_cast<volatile int*>(smem + 256);  // [0] abort
    int* rowmap = reinterpret_cast<int*>(smem + 320);                  // [8] token -> out row
    float* red = reinterpret_cast<float*>(smem + kFixedSmem);           // [16][MT][NT][4][32]
    float* corr_s = red + kConsumerWarps * MT * NT * 4 * 32;              // kAll: [8][G]
    uint8_t* stage0 = smem + fixed_smem_bytes(MT, NT, kAll, g.G);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        flags[0] = 0;
        fence_barrier_init();
    }
    __syncthreads();
    pdl_launch_dependents();

    const int shared_items = a.n_shared * g.tiles;

    if (warp == kConsumerWarps) {
        // ------------------------------ producer ------------------------------
        const uint64_t policy = policy_evict_first();
        const int row_bytes = g.K / 2;
        int64_t n_items = -1;  // unknown until the previous kernel has finished
        int n_act = 0;
        int j = 0;
        bool aborted = false;
        for (int64_t item = blockIdx.x;; item += gridDim.x, ++j) {
            if (n_items < 0 && item >= shared_items) {
                pdl_wait();
                n_act = read_n_active(a);
                n_items = (int64_t)(n_act + a.n_shared) * g.tiles;
            }
            if (n_items >= 0 && item >= n_items) break;
            const int stage = j % stages, use = j / stages;
            if (use > 0 && !mbar_wait(&empty[stage], (use - 1) & 1)) {
                if (lane == 0) report(a.status, COLI_ERR_TIMEOUT);
                aborted = true;
                break;
            }
            if (item == a.withhold_item) continue;  // test hook: this stage never fills
            const Slot sl = decode_slot(a, (int)(item / g.tiles), n_act);
            uint8_t* st = stage0 + (size_t)stage * g.stage_bytes;
            if (!sl.valid) {
                if (lane == 0) mbar_arrive(&full[stage]);  // nothing to copy
                continue;
            }
            const DevExpert ex = a.experts[sl.e];
            const int tile = (int)(item % g.tiles);
            if (lane == 0)
                mbar_arrive_expect_tx(&full[stage], g.rows * row_bytes + g.rows * g.SG * 2);
            __syncwarp();
            if constexpr (kGU) {
                // rows 0..7: gate rows n0.., rows 8..15: up rows n0..; scales likewise
                const int n0 = tile * 8;
                if (lane < 16) {
                    const uint8_t* src = (lane < 8 ? ex.gate_q : ex.up_q) +
                                         (int64_t)(n0 + (lane & 7)) * row_bytes;
                    bulk_g2s_evict_first(st + lane * g.row_stride, src, row_bytes, &full[stage],
                                         policy);
                } else if (lane < 18) {
                    const uint16_t* src = (lane == 16 ? ex.gate_s : ex.up_s) + (int64_t)n0 * g.SG;
                    bulk_g2s_evict_first(st + g.scale_off + (lane - 16) * 8 * g.SG * 2, src,
                                         8 * g.SG * 2, &full[stage], policy);
                }
            } else {
                const int m0 = tile * g.rows;
                for (int i = lane; i < g.rows; i += 32)
                    bulk_g2s_evict_first(st + i * g.row_stride,
                                         ex.down_q + (int64_t)(m0 + i) * row_bytes, row_bytes,
                                         &full[stage], policy);
                if (lane == 0)
                    bulk_g2s_evict_first(st + g.scale_off, ex.down_s + (int64_t)m0 * g.SG,
                                         g.rows * g.SG * 2, &full[stage], policy);
            }
        }
        if (aborted) {
            // let the copies already issued land before the CTA goes away
            for (int back = 1; back <= stages && back <= j; ++back) {
                const int jj = j - back;
                (void)mbar_wait(&full[jj % stages], (jj / stages) & 1);
            }
        }
        return;
    }

    // -------------------------------- consumers --------------------------------
    pdl_wait();
    const int n_act = read_n_active(a);
    const int n_slots = n_act + a.n_shared;
    const int64_t n_items = (int64_t)n_slots * g.tiles;
    const int r = lane >> 2, c = lane & 3;
    const int g_lo = (g.G * warp) / kConsumerWarps, g_hi = (g.G * (warp + 1)) / kConsumerWarps;
    const int tid = threadIdx.x;

    // kAll: activation fragments of all T tokens in registers, their offset
    // sums in shared memory (zero for padding columns), loaded once.
    uint32_t breg[kAll ? KW : 1][8];
    if constexpr (kAll) {
#pragma unroll
        for (int i = 0; i < KW; ++i) {
            const int grp = g_lo + i;
            if (grp < g_hi && r < a.T) {
                load_b(breg[i], a.xp + (int64_t)r * g.K + grp * kGroup + c * 16);
            } else {
#pragma unroll
                for (int q = 0; q < 8; ++q) breg[i][q] = 0u;
            }
        }
        for (int i = tid; i < 8 * g.G; i += kConsumers)
            corr_s[i] = (i / g.G) < a.T ? a.corr[i] : 0.f;
        named_barrier(1, kConsumers);
    }

    int j = 0;
    for (int64_t item = blockIdx.x; item < n_items; item += gridDim.x, ++j) {
        const int stage = j % stages, use = j / stages;
        const bool ok = mbar_wait(&full[stage], use & 1);
        if (!ok && lane == 0) {
            flags[0] = 1;
            report(a.status, COLI_ERR_TIMEOUT);
        }
        const int tile = (int)(item % g.tiles);
        const Slot sl = decode_slot(a, (int)(item / g.tiles), n_act);
        if (!sl.valid && tid == 0) report(a.status, COLI_ERR_BAD_INDEX);
        const uint8_t* st = stage0 + (size_t)stage * g.stage_bytes;
        const uint16_t* scales = reinterpret_cast<const uint16_t*>(st + g.scale_off);

        const int passes = kAll ? (sl.ntok > 0 ? 1 : 0) : (sl.ntok + NT * 8 - 1) / (NT * 8);
        for (int pass = 0; pass < passes; ++pass) {
            const int pass0 = pass * NT * 8;
            float acc[MT][NT][4];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int q = 0; q < 4; ++q) acc[mt][nt][q] = 0.f;

            if constexpr (kAll) {
                if (warp == 0 && lane < 8) {
                    // output row of each token column (-1: not on this list)
                    rowmap[lane] = -1;
                    __syncwarp(0xFFu);
                    if (sl.shared) {
                        if (lane < a.T) rowmap[lane] = sl.list_begin + lane;
                    } else if (lane < sl.ntok) {
                        const int t = a.pairs[sl.list_begin + lane] / a.k;
                        if (t >= 0 && t < a.T) rowmap[t] = sl.list_begin + lane;
                    }
                }
                if (ok) {
                    const uint8_t* rowA = st + r * g.row_stride + c * 8;
                    const uint8_t* rowB = st + (8 + r) * g.row_stride + c * 8;
                    const uint16_t* scA = scales + r * g.SG;
                    const uint16_t* scB = scales + (8 + r) * g.SG;
#pragma unroll
                    for (int i = 0; i < KW; ++i) {
                        const int grp = g_lo + i;
                        if (grp >= g_hi) break;
                        const uint2 wa = *reinterpret_cast<const uint2*>(rowA + grp * 32);
                        const uint2 wb = *reinterpret_cast<const uint2*>(rowB + grp * 32);
                        const float fa = bf16_bits_to_float(scA[grp * g.gs]);
                        const float fb = bf16_bits_to_float(scB[grp * g.gs]);
                        const float cr0 = corr_s[(2 * c) * g.G + grp];
                        const float cr1 = corr_s[(2 * c + 1) * g.G + grp];
                        float part[4];
                        group_partial<!kGU>(part, wa, wb, breg[i]);
                        acc[0][0][0] = fmaf(fa, part[0] - cr0, acc[0][0][0]);
                        acc[0][0][1] = fmaf(fa, part[1] - cr1, acc[0][0][1]);
                        acc[0][0][2] = fmaf(fb, part[2] - cr0, acc[0][0][2]);
                        acc[0][0][3] = fmaf(fb, part[3] - cr1, acc[0][0][3]);
                    }
                }
            } else {
                // B rows (N index = r) and offset-sum tokens (columns 2c, 2c+1)
                auto token_of = [&](int i) -> int {
                    if (i >= sl.ntok) return -1;
                    if (sl.shared) return i;
                    const int t = a.pairs[sl.list_begin + i] / a.k;
                    return (t >= 0 && t < a.T) ? t : -1;
                };
                const __half* brow[NT];
                int tc0[NT], tc1[NT];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int i = pass0 + nt * 8 + r;
                    brow[nt] = nullptr;
                    tc0[nt] = tc1[nt] = -1;
                    if constexpr (kGU) {
                        const int t = token_of(i);
                        if (t >= 0) brow[nt] = a.xp + (int64_t)t * g.K + c * 16;
                        tc0[nt] = token_of(pass0 + nt * 8 + 2 * c);
                        tc1[nt] = token_of(pass0 + nt * 8 + 2 * c + 1);
                    } else {
                        if (i < sl.ntok) brow[nt] = a.hp + (int64_t)(sl.list_begin + i) * g.K + c * 16;
                    }
                }
                if (ok) {
#pragma unroll 2
                    for (int grp = g_lo; grp < g_hi; ++grp) {
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            if (pass0 + nt * 8 >= sl.ntok) break;  // warp-uniform
                            uint32_t bw[8];
                            if (brow[nt]) {
                                load_b(bw, brow[nt] + grp * kGroup);
                            } else {
#pragma unroll
                                for (int q = 0; q < 8; ++q) bw[q] = 0u;
                            }
                            float c0 = 0.f, c1 = 0.f;
                            if constexpr (kGU) {
                                c0 = tc0[nt] >= 0 ? __ldg(a.corr + tc0[nt] * g.G + grp) : 0.f;
                                c1 = tc1[nt] >= 0 ? __ldg(a.corr + tc1[nt] * g.G + grp) : 0.f;
                            }
#pragma unroll
                            for (int mt = 0; mt < MT; ++mt) {
                                const uint8_t* rowA = st + (mt * 16 + r) * g.row_stride + c * 8;
                                const uint8_t* rowB = st + (mt * 16 + 8 + r) * g.row_stride + c * 8;
                                const uint2 wa = *reinterpret_cast<const uint2*>(rowA + grp * 32);
                                const uint2 wb = *reinterpret_cast<const uint2*>(rowB + grp * 32);
                                const float fa = bf16_bits_to_float(
                                    scales[(mt * 16 + r) * g.SG + grp * g.gs]);
                                const float fb = bf16_bits_to_float(
                                    scales[(mt * 16 + 8 + r) * g.SG + grp * g.gs]);
                                float part[4];
                                group_partial<!kGU>(part, wa, wb, bw);
                                acc[mt][nt][0] = fmaf(fa, part[0] - c0, acc[mt][nt][0]);
                                acc[mt][nt][1] = fmaf(fa, part[1] - c1, acc[mt][nt][1]);
                                acc[mt][nt][2] = fmaf(fb, part[2] - c0, acc[mt][nt][2]);
                                acc[mt][nt][3] = fmaf(fb, part[3] - c1, acc[mt][nt][3]);
                            }
                        }
                    }
                }
            }
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        red[(((warp * MT + mt) * NT + nt) * 4 + q) * 32 + lane] = acc[mt][nt][q];
            named_barrier(1, kConsumers);
            if (flags[0]) goto done;

            // Sum the K-splits in a fixed order and write this pass's outputs.
            for (int u = warp; u < MT * NT; u += kConsumerWarps) {
                const int mt = u / NT, nt = u % NT;
                if (!kAll && pass0 + nt * 8 >= sl.ntok) continue;
                float v[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float s = 0.f;
#pragma unroll
                    for (int w = 0; w < kConsumerWarps; ++w)
                        s += red[(((w * MT + mt) * NT + nt) * 4 + q) * 32 + lane];
                    v[q] = s;
                }
#pragma unroll
                for (int e2 = 0; e2 < 2; ++e2) {
                    const int col = nt * 8 + 2 * c + e2;  // MMA column of this value
                    int orow;                             // output row, -1 if none
                    if constexpr (kAll) {
                        orow = col < a.T ? rowmap[col] : -1;
                    } else {
                        orow = pass0 + col < sl.ntok ? sl.list_begin + pass0 + col : -1;
                    }
                    if (orow < 0) continue;
                    if constexpr (kGU) {
                        const int n = tile * 8 + r;
                        const int hcol = (n / kGroup) * kGroup + perm64(n % kGroup);
                        const float gv = v[e2], uv = v[2 + e2];
                        float h = gv / (1.f + expf(-gv)) * uv;
                        if (fabsf(h) > 65504.f) {
                            report(a.status, COLI_ERR_RANGE);
                            h = copysignf(65504.f, h);
                        }
                        a.hp[(int64_t)orow * a.I + hcol] = __float2half_rn(h);
                    } else {
                        float* yrow = a.y + (int64_t)orow * a.H + tile * g.rows + mt * 16;
                        yrow[r] = v[e2];
                        yrow[8 + r] = v[2 + e2];
                    }
                }
            }
            named_barrier(1, kConsumers);
        }
        // release the stage (all lanes' shared-memory reads are done)
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[stage]);
    }
done:
    return;
}

// ---------------------------------------------------------------------------
// out[t][m] = sum_j w[t][j] y[inv[t*k+j]][m] (j ascending) + sum_shared y
// (+ residual), fp32 in that fixed order.  One thread per output element.
// Launched as a programmatic dependent of the down kernel.
__global__ void combine_kernel(const FfnArgs a) {
    pdl_wait();
    const int H = a.H, k = a.k, P = a.T * a.k;
    const int64_t n = (int64_t)a.T * H;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < n;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int t = (int)(idx / H), m = (int)(idx % H);
        float acc = 0.f;
        for (int j = 0; j < k; ++j) {
            const int s = a.inv[t * k + j];
            if (s < 0 || s >= P) {
                report(a.status, COLI_ERR_BAD_INDEX);
                continue;
            }
            acc = fmaf(a.topk_w[t * k + j], a.y[(int64_t)s * H + m], acc);
        }
        for (int sh = 0; sh < a.n_shared; ++sh) acc += a.y[(int64_t)(P + sh * a.T + t) * H + m];
        const int64_t o = (int64_t)t * H + m;
        if (a.out_bf16) {
            if (a.residual)
                acc += __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(a.residual)[o]);
            reinterpret_cast<__nv_bfloat16*>(a.out)[o] = __float2bfloat16_rn(acc);
        } else {
            if (a.residual) acc += reinterpret_cast<const float*>(a.residual)[o];
            reinterpret_cast<float*>(a.out)[o] = acc;
        }
    }
}

// The same combine, four consecutive outputs per thread and one token per
// grid row at a time (no per-element division; 16-byte loads of y).  Same operations in
// the same order per element, so the result equals combine_kernel's bit for
// bit.  Needs H % 4 == 0 and 16-byte aligned y, out and residual (8-byte for
// bf16 out / residual).
__global__ void __launch_bounds__(256) combine_vec_kernel(const FfnArgs a) {
    pdl_wait();
    const int H = a.H, k = a.k, P = a.T * a.k;
    const int m = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
    if (m >= H) return;
    for (int t = blockIdx.y; t < a.T; t += gridDim.y) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int j = 0; j < k; ++j) {
            const int s = __ldg(a.inv + t * k + j);
            if (s < 0 || s >= P) {
                report(a.status, COLI_ERR_BAD_INDEX);
                continue;
            }
            const float w = __ldg(a.topk_w + t * k + j);
            const float4 v = __ldg(reinterpret_cast<const float4*>(a.y + (int64_t)s * H + m));
            acc[0] = fmaf(w, v.x, acc[0]);
            acc[1] = fmaf(w, v.y, acc[1]);
            acc[2] = fmaf(w, v.z, acc[2]);
            acc[3] = fmaf(w, v.w, acc[3]);
        }
        for (int sh = 0; sh < a.n_shared; ++sh) {
            const float4 v =
                __ldg(reinterpret_cast<const float4*>(a.y + (int64_t)(P + sh * a.T + t) * H + m));
            acc[0] += v.x;
            acc[1] += v.y;
            acc[2] += v.z;
            acc[3] += v.w;
        }
        const int64_t o = (int64_t)t * H + m;
        if (a.out_bf16) {
            if (a.residual) {
                const uint2 r = *reinterpret_cast<const uint2*>(
                    reinterpret_cast<const __nv_bfloat16*>(a.residual) + o);
                acc[0] += __uint_as_float(r.x << 16);
                acc[1] += __uint_as_float(r.x & 0xFFFF0000u);
                acc[2] += __uint_as_float(r.y << 16);
                acc[3] += __uint_as_float(r.y & 0xFFFF0000u);
            }
            const __nv_bfloat162 lo = __floats2bfloat162_rn(acc[0], acc[1]);
            const __nv_bfloat162 hi = __floats2bfloat162_rn(acc[2], acc[3]);
            uint2 w2;
            w2.x = *reinterpret_cast<const uint32_t*>(&lo);
            w2.y = *reinterpret_cast<const uint32_t*>(&hi);
            *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(a.out) + o) = w2;
        } else {
            if (a.residual) {
                const float4 r = *reinterpret_cast<const float4*>(
                    reinterpret_cast<const float*>(a.residual) + o);
                acc[0] += r.x;
                acc[1] += r.y;
                acc[2] += r.z;
                acc[3] += r.w;
            }
            *reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + o) =
                make_float4(acc[0], acc[1], acc[2], acc[3]);
        }
    }
}

// x [T][H] bf16 -> operand copy xp (fp16, fragment order) + offset sums.
__global__ void prepare_x_kernel(int T, int H, const __nv_bfloat16* __restrict__ x,
                                 __half* __restrict__ xp, float* __restrict__ corr, int* status) {
    const int64_t grp = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (grp == 0) {
        // the small-batch kernels' tile counters start at zero
        int* cnt = reinterpret_cast<int*>(reinterpret_cast<char*>(status) + kBatchCntOffset);
        cnt[0] = 0;
        cnt[1] = 0;
    }
    if (grp >= (int64_t)T * H / kGroup) return;
    corr[grp] = prepare_group64(reinterpret_cast<const uint16_t*>(x) + grp * kGroup,
                                xp + grp * kGroup, status);
}

// inv[p] = position of pair p in caller-supplied `pairs` (-1 if absent).
__global__ void inverse_pairs_kernel(int P, const int* __restrict__ pairs, int* __restrict__ inv,
                                     int* status) {
    for (int p = threadIdx.x; p < P; p += blockDim.x) inv[p] = -1;
    __syncthreads();
    for (int s = threadIdx.x; s < P; s += blockDim.x) {
        const int p = pairs[s];
        if (p < 0 || p >= P) report(status, COLI_ERR_BAD_INDEX);
        else inv[p] = s;
    }
}

void mark(int i, cudaStream_t st) { profile_mark(i, st); }

cudaLaunchConfig_t pdl_config(int blocks, int threads, int smem, cudaStream_t st,
                              cudaLaunchAttribute* attr) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(blocks);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
}


template <bool kGU, int MT, int NT, bool kAll, int KW>
cudaError_t launch_stream(const FfnArgs& a, const Geo& g, int num_sms, cudaStream_t st) {
    const int fixed = fixed_smem_bytes(MT, NT, kAll, g.G);
    const int stages = std::min(kMaxStages, (kSmemLimit - fixed) / g.stage_bytes);
    if (stages < 2) return cudaErrorInvalidValue;
    const int smem = fixed + stages * g.stage_bytes;
    auto kern = stream_ffn_kernel<kGU, MT, NT, kAll, KW>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    const int64_t max_slots = std::min<int64_t>(a.E, (int64_t)a.T * a.k) + a.n_shared;
    const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>(num_sms, max_slots * g.tiles));
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = pdl_config(blocks, kThreads, smem, st, attr);
    return cudaLaunchKernelEx(&cfg, kern, a, g, stages);
}

cudaError_t launch_combine_impl(const FfnArgs& a, int num_sms, cudaStream_t st) {
    const size_t oa = a.out_bf16 ? 8 : 16;
    auto al = [](const void* p, size_t n) { return reinterpret_cast<uintptr_t>(p) % n == 0; };
    if (a.H % 4 == 0 && a.T >= 1 && al(a.y, 16) && al(a.out, oa) &&
        (!a.residual || al(a.residual, oa))) {
        cudaLaunchAttribute attr[1];
        cudaLaunchConfig_t cfg = pdl_config(1, 256, 0, st, attr);
        cfg.gridDim = dim3((unsigned)((a.H / 4 + 255) / 256), (unsigned)std::min(a.T, 65535));
        return cudaLaunchKernelEx(&cfg, combine_vec_kernel, a);
    }
    const int64_t n = (int64_t)a.T * a.H;
    const int blocks =
        (int)std::max<int64_t>(1, std::min<int64_t>((n + 255) / 256, (int64_t)num_sms * 8));
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = pdl_config(blocks, 256, 0, st, attr);
    return cudaLaunchKernelEx(&cfg, combine_kernel, a);
}

// gate/up launch: T <= 8 uses the register-resident activation path when a
// warp's share of the groups fits KW.
cudaError_t launch_gateup(const FfnArgs& a, int num_sms, cudaStream_t st) {
    const Geo g = make_geo(a.H, 16, a.I / 8, a.per_row);
    const int per_warp = (g.G + kConsumerWarps - 1) / kConsumerWarps;
    if (a.T <= 8) {
        if (per_warp <= 2) return launch_stream<true, 1, 1, true, 2>(a, g, num_sms, st);
        if (per_warp <= 4) return launch_stream<true, 1, 1, true, 4>(a, g, num_sms, st);
        if (per_warp <= 6) return launch_stream<true, 1, 1, true, 6>(a, g, num_sms, st);
        if (per_warp <= 8) return launch_stream<true, 1, 1, true, 8>(a, g, num_sms, st);
    }
    if (a.T <= 8) return launch_stream<true, 1, 1, false, 1>(a, g, num_sms, st);
    return launch_stream<true, 1, 2, false, 1>(a, g, num_sms, st);
}

cudaError_t launch_down(const FfnArgs& a, int num_sms, cudaStream_t st) {
    if (a.T <= 8)
        return launch_stream<false, 2, 1, false, 1>(a, make_geo(a.I, 32, a.H / 32, a.per_row),
                                                   num_sms, st);
    return launch_stream<false, 1, 2, false, 1>(a, make_geo(a.I, 16, a.H / 16, a.per_row),
                                               num_sms, st);
}

}  // namespace

cudaError_t launch_combine(const FfnArgs& a, int num_sms, cudaStream_t st) {
    return launch_combine_impl(a, num_sms, st);
}

bool stream_shapes_fit(int H, int I) {
    const Geo g1 = make_geo(H, 16, I / 8, 0), g2 = make_geo(I, 32, H / 32, 0);
    return fixed_smem_bytes(1, 2, true, g1.G) + 2 * g1.stage_bytes <= kSmemLimit &&
           fixed_smem_bytes(2, 2, false, g2.G) + 2 * g2.stage_bytes <= kSmemLimit;
}

cudaError_t launch_ffn_stream(const FfnArgs& a_in, int num_sms, cudaStream_t st) {
    FfnArgs a = a_in;
    a.withhold_item = take_withhold_item();
    mark(1, st);
    cudaError_t err = launch_gateup(a, num_sms, st);
    if (err != cudaSuccess) return err;
    a.withhold_item = -1;
    mark(2, st);
    err = launch_down(a, num_sms, st);
    if (err != cudaSuccess) return err;
    mark(3, st);
    err = launch_combine_impl(a, num_sms, st);
    mark(4, st);
    return err;
}

cudaError_t launch_prepare_x(int T, int H, const __nv_bfloat16* x, __half* xp, float* corr,
                             int* status, cudaStream_t st) {
    const int64_t groups = (int64_t)T * H / kGroup;
    prepare_x_kernel<<<(unsigned)((groups + 127) / 128), 128, 0, st>>>(T, H, x, xp, corr, status);
    return cudaGetLastError();
}

cudaError_t launch_inverse_pairs(int P, const int* pairs, int* inv, int* status,
                                 cudaStream_t st) {
    inverse_pairs_kernel<<<1, 1024, 0, st>>>(P, pairs, inv, status);
    return cudaGetLastError();
}

}  // namespace coli
