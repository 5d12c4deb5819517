// Expert FFN for decode and small batches: int4 gs64 dequant-GEMV on tensor
// cores with the weights streamed from HBM exactly once per call
// ("batch-union", "yunpan.plus/t/30351-1-1", capability two).
//
// Work.  An item is (expert slot, 16-row tile of a weight matrix).  The
// shared experts come first in slot order, so their weights can stream while
// the routing of the call is still running (programmatic dependent launch);
// the active routed experts follow.  For gate/up the 16 MMA rows are 8 gate
// rows and the same 8 up rows, so each thread ends with g and u of one
// (token, n) and forms the SwiGLU output in registers.  For down the rows are
// 16 consecutive rows of W_d.
//
// Data movement.  One CTA per SM.  A producer warp copies each item's rows
// (one bulk copy per row, into rows padded by 32 bytes so the fragment reads
// are free of bank conflicts) and its scale rows into a ring of stages, with
// an mbarrier per stage carrying the byte count.  Eight consumer warps split
// the reduction dimension of the item and read fragments from shared memory.
// HBM sees only full, contiguous, streamed-once reads.
//
// Arithmetic.  A code q in [-8, 7] is exact in bf16 and fp16, so the MMA A
// operand holds raw codes (unpacked with a mask and a magic-number subtract:
// 0x4300 | n is the bf16 value 128 + n, 0x6400 | n the fp16 value 1024 + n);
// x (bf16) is exact as the bf16 B operand; products are exact and accumulate
// in fp32; the gs64 scale multiplies each group's fp32 partial sum:
//   g[n] = sum_groups s[n][grp] * (sum_{k in grp} q[n][k] x[k]).
// The SwiGLU output h is rounded once to fp16 (the down projection's B
// operand; |h| > 65504 is clamped and reported as COLI_ERR_RANGE).
//
// K order.  The 16 k-slots a lane feeds to one m16n8k16 MMA come from 16
// consecutive codes of its row (8 bytes) in the order the unpack produces
// them; the activation operand is stored in that same permuted order (xp,
// hp), so every dot product is unchanged.  One 64-code scale group is one
// 8-byte slice per lane of a quad, i.e. exactly four MMAs.
//
// Combine.  The down kernel writes each expert's rows of y (fp32); a small
// kernel chained to it by programmatic dependent launch forms
//   out[t][m] = sum_j w[t][j] y[(t,j)][m] (j ascending) + y_shared[t][m]
//               (+ residual[t][m])
// in fp32, in that fixed order, so the result does not depend on timing.
#include <algorithm>

#include "moe_device.cuh"
#include "ptx.cuh"

namespace coli {
namespace {

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;  // + producer warp
constexpr int kMaxStages = 16;
constexpr int kFixedSmem = 512;            // barriers + flags
constexpr int kSmemLimit = 227 * 1024;

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
    return __uint_as_float((uint32_t)b << 16);
}

// One word of 8 nibbles (codes k = 0..7 of a slice) -> four bf16x2 holding
// the code pairs (0,4), (1,5), (2,6), (3,7).
__device__ __forceinline__ void unpack_bf16(uint32_t w, uint32_t o[4]) {
    const uint32_t magic = 0x43084308u;  // (n ^ 8) | 0x4300 = 128 + q + 8
    const __nv_bfloat162 bias = __floats2bfloat162_rn(136.f, 136.f);
    uint32_t t[4];
    t[0] = (w & 0x000F000Fu) ^ magic;
    t[1] = ((w >> 4) & 0x000F000Fu) ^ magic;
    t[2] = ((w >> 8) & 0x000F000Fu) ^ magic;
    t[3] = ((w >> 12) & 0x000F000Fu) ^ magic;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&t[i]);
        v = __hsub2(v, bias);
        o[i] = *reinterpret_cast<uint32_t*>(&v);
    }
}

// Same for fp16.  For the nibble at bits 4..7, 0x6400 | n << 4 is
// 1024 + 16 n, brought back exactly with (v / 16) - 72.
__device__ __forceinline__ void unpack_f16(uint32_t w, uint32_t o[4]) {
    const __half2 bias_lo = __floats2half2_rn(1032.f, 1032.f);
    const __half2 sixteenth = __floats2half2_rn(0.0625f, 0.0625f);
    const __half2 bias_hi = __floats2half2_rn(-72.f, -72.f);
    const uint32_t w8 = w >> 8;
    uint32_t t[4];
    t[0] = (w & 0x000F000Fu) ^ 0x64086408u;
    t[1] = (w & 0x00F000F0u) ^ 0x64806480u;
    t[2] = (w8 & 0x000F000Fu) ^ 0x64086408u;
    t[3] = (w8 & 0x00F000F0u) ^ 0x64806480u;
    __half2 v0 = __hsub2(*reinterpret_cast<__half2*>(&t[0]), bias_lo);
    __half2 v1 = __hfma2(*reinterpret_cast<__half2*>(&t[1]), sixteenth, bias_hi);
    __half2 v2 = __hsub2(*reinterpret_cast<__half2*>(&t[2]), bias_lo);
    __half2 v3 = __hfma2(*reinterpret_cast<__half2*>(&t[3]), sixteenth, bias_hi);
    o[0] = *reinterpret_cast<uint32_t*>(&v0);
    o[1] = *reinterpret_cast<uint32_t*>(&v1);
    o[2] = *reinterpret_cast<uint32_t*>(&v2);
    o[3] = *reinterpret_cast<uint32_t*>(&v3);
}

template <bool kBf16>
__device__ __forceinline__ void mma16816(float d[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    if constexpr (kBf16) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, "
            "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    } else {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, "
            "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }
}

// Geometry of one kernel kind (gate/up or down).
struct Geo {
    int K;           // reduction length (H for gate/up, I for down)
    int G;           // scale groups per row, K / 64
    int row_stride;  // bytes per staged row: K/2 + 32
    int scale_blk;   // bytes of 8 rows of scales: K / 4
    int stage_bytes;
    int tiles;       // items per expert
};

inline Geo make_geo(int K, int tiles) {
    Geo g;
    g.K = K;
    g.G = K / kGroup;
    g.row_stride = K / 2 + 32;
    g.scale_blk = K / 4;
    g.stage_bytes = 16 * g.row_stride + 2 * g.scale_blk;
    g.tiles = tiles;
    return g;
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

// Sources of the 16 staged rows and two scale blocks of an item.
template <bool kGU>
__device__ __forceinline__ void item_sources(const DevExpert& ex, int tile, const Geo& g,
                                             const uint8_t*& a0, const uint8_t*& a1,
                                             const uint16_t*& s0, const uint16_t*& s1) {
    if constexpr (kGU) {
        const int n0 = tile * 8;
        a0 = ex.gate_q + (int64_t)n0 * (g.K / 2);
        a1 = ex.up_q + (int64_t)n0 * (g.K / 2);
        s0 = ex.gate_s + (int64_t)n0 * g.G;
        s1 = ex.up_s + (int64_t)n0 * g.G;
    } else {
        const int m0 = tile * 16;
        a0 = ex.down_q + (int64_t)m0 * (g.K / 2);
        a1 = ex.down_q + (int64_t)(m0 + 8) * (g.K / 2);
        s0 = ex.down_s + (int64_t)m0 * g.G;
        s1 = ex.down_s + (int64_t)(m0 + 8) * g.G;
    }
}

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

// ---------------------------------------------------------------------------
// The streaming FFN kernel.  kGU: gate/up + SwiGLU (bf16 MMA, writes hp);
// otherwise down (fp16 MMA, writes y).  NT = N-tiles of 8
// tokens per pass.
template <int NT, bool kGU>
__global__ void __launch_bounds__(kThreads, 1)
stream_ffn_kernel(const FfnArgs a, const Geo g, int stages) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kMaxStages;
    volatile int* flags = reinterpret_cast<volatile int*>(smem + 256);  // [0] abort
    float* red = reinterpret_cast<float*>(smem + kFixedSmem);            // [8][NT][4][32]
    uint8_t* stage0 = smem + kFixedSmem + kConsumerWarps * NT * 4 * 32 * 4;

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
            const Slot sl = decode_slot(a, (int)(item / g.tiles), n_act);
            uint8_t* st = stage0 + (size_t)stage * g.stage_bytes;
            if (item == a.withhold_item) continue;  // test hook: this stage never fills
            if (!sl.valid) {
                if (lane == 0) mbar_arrive(&full[stage]);  // nothing to copy
                continue;
            }
            const uint8_t *a0, *a1;
            const uint16_t *s0, *s1;
            item_sources<kGU>(a.experts[sl.e], (int)(item % g.tiles), g, a0, a1, s0, s1);
            if (lane == 0) mbar_arrive_expect_tx(&full[stage], 16 * (g.K / 2) + 2 * g.scale_blk);
            __syncwarp();
            if (lane < 16) {
                const uint8_t* src = (lane < 8 ? a0 : a1) + (int64_t)(lane & 7) * (g.K / 2);
                bulk_g2s_evict_first(st + lane * g.row_stride, src, g.K / 2, &full[stage], policy);
            } else if (lane == 16) {
                bulk_g2s_evict_first(st + 16 * g.row_stride, s0, g.scale_blk, &full[stage], policy);
            } else if (lane == 17) {
                bulk_g2s_evict_first(st + 16 * g.row_stride + g.scale_blk, s1, g.scale_blk,
                                     &full[stage], policy);
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
        const uint8_t* rowA = st + r * g.row_stride + c * 8;        // MMA row r
        const uint8_t* rowB = st + (8 + r) * g.row_stride + c * 8;  // MMA row r + 8
        const uint16_t* scA = reinterpret_cast<const uint16_t*>(st + 16 * g.row_stride) + r * g.G;
        const uint16_t* scB =
            reinterpret_cast<const uint16_t*>(st + 16 * g.row_stride + g.scale_blk) + r * g.G;

        for (int pass0 = 0; pass0 < sl.ntok; pass0 += NT * 8) {
            // B rows of this lane (N index = r) for every N-tile of the pass
            const uint16_t* brow[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int i = pass0 + nt * 8 + r;
                brow[nt] = nullptr;
                if (i < sl.ntok) {
                    if constexpr (kGU) {
                        const int t = sl.shared ? i : a.pairs[sl.list_begin + i] / a.k;
                        if (t >= 0 && t < a.T)
                            brow[nt] = reinterpret_cast<const uint16_t*>(a.xp) + (int64_t)t * g.K + c * 16;
                    } else {
                        brow[nt] = reinterpret_cast<const uint16_t*>(a.hp) +
                                   (int64_t)(sl.list_begin + i) * g.K + c * 16;
                    }
                }
            }
            float acc[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[nt][q] = 0.f;

            if (ok) {
#pragma unroll 2
                for (int grp = g_lo; grp < g_hi; ++grp) {
                    const uint2 wa = *reinterpret_cast<const uint2*>(rowA + grp * 32);
                    const uint2 wb = *reinterpret_cast<const uint2*>(rowB + grp * 32);
                    const float fa = bf16_bits_to_float(scA[grp]);
                    const float fb = bf16_bits_to_float(scB[grp]);
                    uint32_t aa[8], ab[8];
                    if constexpr (kGU) {
                        unpack_bf16(wa.x, aa);
                        unpack_bf16(wa.y, aa + 4);
                        unpack_bf16(wb.x, ab);
                        unpack_bf16(wb.y, ab + 4);
                    } else {
                        unpack_f16(wa.x, aa);
                        unpack_f16(wa.y, aa + 4);
                        unpack_f16(wb.x, ab);
                        unpack_f16(wb.y, ab + 4);
                    }
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        if (pass0 + nt * 8 >= sl.ntok) break;  // warp-uniform
                        uint32_t bw[8];
                        if (brow[nt]) {
                            const uint4 b0 = __ldg(reinterpret_cast<const uint4*>(brow[nt] + grp * kGroup));
                            const uint4 b1 = __ldg(reinterpret_cast<const uint4*>(brow[nt] + grp * kGroup + 8));
                            bw[0] = b0.x; bw[1] = b0.y; bw[2] = b0.z; bw[3] = b0.w;
                            bw[4] = b1.x; bw[5] = b1.y; bw[6] = b1.z; bw[7] = b1.w;
                        } else {
#pragma unroll
                            for (int q = 0; q < 8; ++q) bw[q] = 0u;
                        }
                        float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                        for (int m = 0; m < 4; ++m)
                            mma16816<kGU>(part, aa[2 * m], ab[2 * m], aa[2 * m + 1], ab[2 * m + 1],
                                          bw[2 * m], bw[2 * m + 1]);
                        acc[nt][0] = fmaf(fa, part[0], acc[nt][0]);
                        acc[nt][1] = fmaf(fa, part[1], acc[nt][1]);
                        acc[nt][2] = fmaf(fb, part[2], acc[nt][2]);
                        acc[nt][3] = fmaf(fb, part[3], acc[nt][3]);
                    }
                }
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) red[((warp * NT + nt) * 4 + q) * 32 + lane] = acc[nt][q];
            named_barrier(1, kConsumers);
            if (flags[0]) goto done;

            // Sum the K-splits in a fixed order and write this pass's outputs.
            for (int nt = warp; nt < NT; nt += kConsumerWarps) {
                if (pass0 + nt * 8 >= sl.ntok) continue;
                float v[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float s = 0.f;
#pragma unroll
                    for (int w = 0; w < kConsumerWarps; ++w) s += red[((w * NT + nt) * 4 + q) * 32 + lane];
                    v[q] = s;
                }
#pragma unroll
                for (int e2 = 0; e2 < 2; ++e2) {
                    const int i_tok = pass0 + nt * 8 + 2 * c + e2;
                    if (i_tok >= sl.ntok) continue;
                    if constexpr (kGU) {
                        const int n = tile * 8 + r;
                        const int hcol = (n / kGroup) * kGroup + perm64(n % kGroup);
                        const float gv = v[e2], uv = v[2 + e2];
                        float h = gv / (1.f + expf(-gv)) * uv;
                        if (fabsf(h) > 65504.f) {
                            report(a.status, COLI_ERR_RANGE);
                            h = copysignf(65504.f, h);
                        }
                        a.hp[(int64_t)(sl.list_begin + i_tok) * a.I + hcol] = __float2half_rn(h);
                    } else {
                        float* yrow = a.y + (int64_t)(sl.list_begin + i_tok) * a.H + tile * 16;
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
__global__ void permute_x_kernel(int T, int H, const __nv_bfloat16* __restrict__ x,
                                 __nv_bfloat16* __restrict__ xp) {
    const int64_t slice = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (slice >= (int64_t)T * H / 16) return;
    permute_slice16(reinterpret_cast<const uint16_t*>(x) + slice * 16,
                    reinterpret_cast<uint16_t*>(xp) + slice * 16);
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

void mark(int i, cudaStream_t st) {
    if (cudaEvent_t ev = profile_event(i)) cudaEventRecord(ev, st);
}

template <int NT>
int fixed_smem() {
    return kFixedSmem + kConsumerWarps * NT * 4 * 32 * 4;
}

template <int NT, bool kGU>
cudaError_t launch_stream(const FfnArgs& a, const Geo& g, int num_sms, cudaStream_t st) {
    const int fixed = fixed_smem<NT>();
    const int stages = std::min(kMaxStages, (kSmemLimit - fixed) / g.stage_bytes);
    if (stages < 2) return cudaErrorInvalidValue;
    const int smem = fixed + stages * g.stage_bytes;
    cudaError_t err = cudaFuncSetAttribute(stream_ffn_kernel<NT, kGU>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    const int64_t max_slots = std::min<int64_t>(a.E, (int64_t)a.T * a.k) + a.n_shared;
    const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>(num_sms, max_slots * g.tiles));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(blocks);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, stream_ffn_kernel<NT, kGU>, a, g, stages);
}

cudaError_t launch_combine(const FfnArgs& a, int num_sms, cudaStream_t st) {
    const int64_t n = (int64_t)a.T * a.H;
    const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>((n + 255) / 256, (int64_t)num_sms * 8));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(blocks);
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, combine_kernel, a);
}

template <int NT>
cudaError_t launch_pair(const FfnArgs& a_in, int num_sms, cudaStream_t st) {
    FfnArgs a = a_in;
    a.withhold_item = take_withhold_item();
    mark(1, st);
    cudaError_t err = launch_stream<NT, true>(a, make_geo(a.H, a.I / 8), num_sms, st);
    a.withhold_item = -1;
    if (err != cudaSuccess) return err;
    mark(2, st);
    err = launch_stream<NT, false>(a, make_geo(a.I, a.H / 16), num_sms, st);
    if (err != cudaSuccess) return err;
    mark(3, st);
    err = launch_combine(a, num_sms, st);
    mark(4, st);
    return err;
}

}  // namespace

bool stream_shapes_fit(int H, int I) {
    const int fixed = fixed_smem<4>();
    const Geo g1 = make_geo(H, I / 8), g2 = make_geo(I, H / 16);
    return fixed + 2 * std::max(g1.stage_bytes, g2.stage_bytes) <= kSmemLimit;
}

cudaError_t launch_ffn_stream(const FfnArgs& a, int num_sms, cudaStream_t st) {
    const int nt_needed = (a.T + 7) / 8;
    if (nt_needed <= 1) return launch_pair<1>(a, num_sms, st);
    if (nt_needed <= 2) return launch_pair<2>(a, num_sms, st);
    return launch_pair<4>(a, num_sms, st);
}

cudaError_t launch_permute_x(int T, int H, const __nv_bfloat16* x, __nv_bfloat16* xp,
                             cudaStream_t st) {
    const int64_t slices = (int64_t)T * H / 16;
    permute_x_kernel<<<(unsigned)((slices + 255) / 256), 256, 0, st>>>(T, H, x, xp);
    return cudaGetLastError();
}

cudaError_t launch_inverse_pairs(int P, const int* pairs, int* inv, int* status,
                                 cudaStream_t st) {
    inverse_pairs_kernel<<<1, 1024, 0, st>>>(P, pairs, inv, status);
    return cudaGetLastError();
}

}  // namespace coli
