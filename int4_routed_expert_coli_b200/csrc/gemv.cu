// Expert FFN for decode and small batches: int4 gs64 dequant-GEMV on
// tensor cores, weights streamed once per call ("batch-union",
// "yunpan.plus/t/30351-1-1", capability two).
//
// Shape of the work.  For every active expert (and the shared expert) the
// kernels stream its packed weights exactly once and multiply them against
// the (few) tokens on its list.  The weight matrix supplies the M = 16 rows of
// an m16n8k16 MMA; tokens are the N = 8 columns (padded with zeros).  This
// keeps the multiply-add off the CUDA cores: per 8 weights a thread spends
// one shift/mask/subtract chain on the unpack and one MMA, instead of a
// convert and an FMA per weight, which HBM3e bandwidth would outrun.
//
// Exactness.  A int4 code q in [-8, 7] is exact in bf16 and in fp16, so the
// MMA A operand holds the raw codes; x (bf16) is exact as a bf16 B operand;
// products are exact and accumulate in fp32.  The per-64 scale multiplies each
// group's fp32 partial sum:  g = sum_groups s[n][grp] * sum_{k in grp} q x.
// The SwiGLU output h is rounded to fp16 once before the down projection
// (whose A operand is then fp16 codes, exact as well); |h| above 65504 is
// clamped and reported as COLI_ERR_RANGE in the status word.
//
// K order.  The MMA's 16 k-slots of each thread are fed from 16 consecutive
// codes of one row (8 bytes), in the order the nibble-unpack produces them;
// the activation operand is stored in the same permuted order ("xp", "hp"),
// so the dot products are unchanged.  A 64-code scale group is one 8-byte
// slice per lane of a quad, i.e. exactly four MMAs.
#include <algorithm>

#include "coli_internal.cuh"

namespace coli {
namespace {

constexpr int kThreads = 128;  // 4 warps split K
constexpr int kU = 4;          // groups in flight per warp

// Position of element j (0..63) of a 64-group inside the permuted layout.
__host__ __device__ __forceinline__ int perm64(int j) {
    const int c = j >> 4, jj = j & 15;
    const int m = ((jj >> 3) << 1) + ((jj & 3) >> 1);
    const int e = (jj & 7) >> 2;
    const int odd = jj & 1;
    return c * 16 + 4 * m + 2 * odd + e;
}

__device__ __forceinline__ uint2 ldg_stream(const uint8_t* p) {
    uint2 r;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];"
                 : "=r"(r.x), "=r"(r.y)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
    return __uint_as_float((uint32_t)b << 16);
}

// One word of 8 nibbles (codes for k = 0..7 of a slice) -> four bf16x2 with
// pairs (0,4), (1,5), (2,6), (3,7) as exact codes.
__device__ __forceinline__ void unpack_bf16(uint32_t w, uint32_t o[4]) {
    // 0x4300 | n is the bf16 value 128 + n; n = nibble ^ 8 = q + 8.
    const uint32_t magic = 0x43084308u;
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

// Same for fp16: 0x6400 | n is 1024 + n; for the nibble at bits 4..7,
// 0x6400 | n << 4 is 1024 + 16 n, brought back with (v / 16) - 72.
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

// One 64-code group for a 16-row tile: rows r (word pair wa) and r + 8
// (word pair wb), B fragments bw[8] for one N-tile.  part = sum q * x.
template <bool kBf16>
__device__ __forceinline__ void group_mma(float part[4], const uint32_t ar[8], const uint32_t br[8],
                                          const uint32_t bw[8]) {
#pragma unroll
    for (int m = 0; m < 4; ++m)
        mma16816<kBf16>(part, ar[2 * m], br[2 * m], ar[2 * m + 1], br[2 * m + 1], bw[2 * m],
                        bw[2 * m + 1]);
}

// Work slot -> expert id and its token list.  Returns false for a bad slot.
struct Slot {
    int e;           // expert row in the device table
    int list_begin;  // first output row (hp/y) of this expert
    int ntok;        // tokens on the list
    bool shared;
};

__device__ __forceinline__ bool decode_slot(const FfnArgs& a, int slot, int n_act, Slot& s) {
    const int P = a.T * a.k;
    if (slot < n_act) {
        const int e = a.active[slot];
        if (e < 0 || e >= a.E) return false;
        const int b = a.offsets[e], en = a.offsets[e + 1];
        if (b < 0 || en < b || en > P) return false;
        s.e = e;
        s.list_begin = b;
        s.ntok = en - b;
        s.shared = false;
    } else {
        const int sh = slot - n_act;
        s.e = a.E + sh;
        s.list_begin = P + sh * a.T;
        s.ntok = a.T;
        s.shared = true;
    }
    return true;
}

__device__ __forceinline__ int read_n_active(const FfnArgs& a) {
    int n = *a.n_active;
    if (n < 0 || n > a.E) {
        report(a.status, COLI_ERR_BAD_INDEX);
        n = 0;
    }
    return n;
}

// ---------------------------------------------------------------------------
// x [T][H] bf16 -> xp [T][H] bf16 in the fragment order of perm64.
__global__ void permute_x_kernel(int T, int H, const __nv_bfloat16* __restrict__ x,
                                 __nv_bfloat16* __restrict__ xp) {
    const int64_t slice = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // 16 elements
    if (slice >= (int64_t)T * H / 16) return;
    const uint16_t* src = reinterpret_cast<const uint16_t*>(x) + slice * 16;
    uint16_t* dst = reinterpret_cast<uint16_t*>(xp) + slice * 16;
    uint4 in0 = *reinterpret_cast<const uint4*>(src);
    uint4 in1 = *reinterpret_cast<const uint4*>(src + 8);
    uint16_t v[16], o[16];
    *reinterpret_cast<uint4*>(&v[0]) = in0;
    *reinterpret_cast<uint4*>(&v[8]) = in1;
#pragma unroll
    for (int jj = 0; jj < 16; ++jj) o[perm64(jj) & 15] = v[jj];
    *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<uint4*>(&o[0]);
    *reinterpret_cast<uint4*>(dst + 8) = *reinterpret_cast<uint4*>(&o[8]);
}

// inv[p] = position of pair p in `pairs` (or -1), from caller-supplied lists.
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

// ---------------------------------------------------------------------------
// gate/up + SwiGLU.  Item = (slot, 8-row tile n0): rows 0..7 of the MMA tile
// are gate rows n0..n0+7, rows 8..15 the up rows n0..n0+7, so each thread
// ends with g and u of the same (token, n) and forms h in registers.
template <int NT>
__global__ void __launch_bounds__(kThreads) gateup_kernel(const FfnArgs a) {
    __shared__ float red[4][NT][4][32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int r = lane >> 2, c = lane & 3;
    const int H = a.H, I = a.I, G = H / kGroup;
    const int tiles = I / 8;
    const int n_act = read_n_active(a);
    const int64_t n_items = (int64_t)(n_act + a.n_shared) * tiles;
    const int g_lo = (G * warp) / 4, g_hi = (G * (warp + 1)) / 4;

    for (int64_t item = blockIdx.x; item < n_items; item += gridDim.x) {
        Slot sl;
        if (!decode_slot(a, (int)(item / tiles), n_act, sl)) {
            report(a.status, COLI_ERR_BAD_INDEX);
            continue;
        }
        const int n0 = (int)(item % tiles) * 8;
        const DevExpert ex = a.experts[sl.e];
        const uint8_t* grow = ex.gate_q + (int64_t)(n0 + r) * (H / 2) + c * 8;
        const uint8_t* urow = ex.up_q + (int64_t)(n0 + r) * (H / 2) + c * 8;
        const uint16_t* gs = ex.gate_s + (int64_t)(n0 + r) * G;
        const uint16_t* us = ex.up_s + (int64_t)(n0 + r) * G;

        for (int pass0 = 0; pass0 < sl.ntok; pass0 += NT * 8) {
            const uint16_t* brow[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int i = pass0 + nt * 8 + r;
                brow[nt] = nullptr;
                if (i < sl.ntok) {
                    const int t = sl.shared ? i : a.pairs[sl.list_begin + i] / a.k;
                    if (t >= 0 && t < a.T)
                        brow[nt] = reinterpret_cast<const uint16_t*>(a.xp) + (int64_t)t * H + c * 16;
                }
            }
            float acc[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;

            for (int gb = g_lo; gb < g_hi; gb += kU) {
                uint2 wg[kU], wu[kU];
                uint16_t sg[kU], su[kU];
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    if (gb + u < g_hi) {
                        wg[u] = ldg_stream(grow + (gb + u) * 32);
                        wu[u] = ldg_stream(urow + (gb + u) * 32);
                        sg[u] = __ldg(gs + gb + u);
                        su[u] = __ldg(us + gb + u);
                    }
                }
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    if (gb + u >= g_hi) break;
                    const int g = gb + u;
                    uint32_t ag[8], au[8];
                    unpack_bf16(wg[u].x, ag);
                    unpack_bf16(wg[u].y, ag + 4);
                    unpack_bf16(wu[u].x, au);
                    unpack_bf16(wu[u].y, au + 4);
                    const float fg = bf16_bits_to_float(sg[u]), fu = bf16_bits_to_float(su[u]);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        if (pass0 + nt * 8 >= sl.ntok) break;  // warp-uniform
                        uint32_t bw[8];
                        if (brow[nt]) {
                            const uint4 b0 = *reinterpret_cast<const uint4*>(brow[nt] + g * kGroup);
                            const uint4 b1 = *reinterpret_cast<const uint4*>(brow[nt] + g * kGroup + 8);
                            bw[0] = b0.x; bw[1] = b0.y; bw[2] = b0.z; bw[3] = b0.w;
                            bw[4] = b1.x; bw[5] = b1.y; bw[6] = b1.z; bw[7] = b1.w;
                        } else {
#pragma unroll
                            for (int i = 0; i < 8; ++i) bw[i] = 0u;
                        }
                        float part[4] = {0.f, 0.f, 0.f, 0.f};
                        group_mma<true>(part, ag, au, bw);
                        acc[nt][0] = fmaf(fg, part[0], acc[nt][0]);
                        acc[nt][1] = fmaf(fg, part[1], acc[nt][1]);
                        acc[nt][2] = fmaf(fu, part[2], acc[nt][2]);
                        acc[nt][3] = fmaf(fu, part[3], acc[nt][3]);
                    }
                }
            }

            // Sum the four K-quarters in a fixed order and form h.
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) red[warp][nt][i][lane] = acc[nt][i];
            __syncthreads();
            for (int nt = warp; nt < NT; nt += 4) {
                if (pass0 + nt * 8 >= sl.ntok) continue;
                float v[4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    v[i] = ((red[0][nt][i][lane] + red[1][nt][i][lane]) + red[2][nt][i][lane]) +
                           red[3][nt][i][lane];
                const int n = n0 + r;
                const int hcol = (n / kGroup) * kGroup + perm64(n % kGroup);
#pragma unroll
                for (int e2 = 0; e2 < 2; ++e2) {
                    const int i_tok = pass0 + nt * 8 + 2 * c + e2;
                    if (i_tok >= sl.ntok) continue;
                    const float gv = v[e2], uv = v[2 + e2];
                    float h = gv / (1.f + expf(-gv)) * uv;
                    if (fabsf(h) > 65504.f) {
                        report(a.status, COLI_ERR_RANGE);
                        h = copysignf(65504.f, h);
                    }
                    a.hp[(int64_t)(sl.list_begin + i_tok) * I + hcol] = __float2half_rn(h);
                }
            }
            __syncthreads();
        }
    }
}

// ---------------------------------------------------------------------------
// down projection.  Item = (slot, 16-row tile m0 of W_d); B = hp rows of the
// expert's list (contiguous); writes y[s][m] in fp32.
template <int NT>
__global__ void __launch_bounds__(kThreads) down_kernel(const FfnArgs a) {
    __shared__ float red[4][NT][4][32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int r = lane >> 2, c = lane & 3;
    const int H = a.H, I = a.I, G = I / kGroup;
    const int tiles = H / 16;
    const int n_act = read_n_active(a);
    const int64_t n_items = (int64_t)(n_act + a.n_shared) * tiles;
    const int g_lo = (G * warp) / 4, g_hi = (G * (warp + 1)) / 4;

    for (int64_t item = blockIdx.x; item < n_items; item += gridDim.x) {
        Slot sl;
        if (!decode_slot(a, (int)(item / tiles), n_act, sl)) {
            report(a.status, COLI_ERR_BAD_INDEX);
            continue;
        }
        const int m0 = (int)(item % tiles) * 16;
        const DevExpert ex = a.experts[sl.e];
        const uint8_t* row0 = ex.down_q + (int64_t)(m0 + r) * (I / 2) + c * 8;
        const uint8_t* row8 = ex.down_q + (int64_t)(m0 + 8 + r) * (I / 2) + c * 8;
        const uint16_t* s0 = ex.down_s + (int64_t)(m0 + r) * G;
        const uint16_t* s8 = ex.down_s + (int64_t)(m0 + 8 + r) * G;

        for (int pass0 = 0; pass0 < sl.ntok; pass0 += NT * 8) {
            const uint16_t* brow[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int i = pass0 + nt * 8 + r;
                brow[nt] = i < sl.ntok ? reinterpret_cast<const uint16_t*>(a.hp) +
                                             (int64_t)(sl.list_begin + i) * I + c * 16
                                       : nullptr;
            }
            float acc[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;

            for (int gb = g_lo; gb < g_hi; gb += kU) {
                uint2 w0[kU], w8[kU];
                uint16_t sc0[kU], sc8[kU];
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    if (gb + u < g_hi) {
                        w0[u] = ldg_stream(row0 + (gb + u) * 32);
                        w8[u] = ldg_stream(row8 + (gb + u) * 32);
                        sc0[u] = __ldg(s0 + gb + u);
                        sc8[u] = __ldg(s8 + gb + u);
                    }
                }
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    if (gb + u >= g_hi) break;
                    const int g = gb + u;
                    uint32_t a0[8], a8[8];
                    unpack_f16(w0[u].x, a0);
                    unpack_f16(w0[u].y, a0 + 4);
                    unpack_f16(w8[u].x, a8);
                    unpack_f16(w8[u].y, a8 + 4);
                    const float f0 = bf16_bits_to_float(sc0[u]), f8 = bf16_bits_to_float(sc8[u]);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        if (pass0 + nt * 8 >= sl.ntok) break;
                        uint32_t bw[8];
                        if (brow[nt]) {
                            const uint4 b0 = *reinterpret_cast<const uint4*>(brow[nt] + g * kGroup);
                            const uint4 b1 = *reinterpret_cast<const uint4*>(brow[nt] + g * kGroup + 8);
                            bw[0] = b0.x; bw[1] = b0.y; bw[2] = b0.z; bw[3] = b0.w;
                            bw[4] = b1.x; bw[5] = b1.y; bw[6] = b1.z; bw[7] = b1.w;
                        } else {
#pragma unroll
                            for (int i = 0; i < 8; ++i) bw[i] = 0u;
                        }
                        float part[4] = {0.f, 0.f, 0.f, 0.f};
                        group_mma<false>(part, a0, a8, bw);
                        acc[nt][0] = fmaf(f0, part[0], acc[nt][0]);
                        acc[nt][1] = fmaf(f0, part[1], acc[nt][1]);
                        acc[nt][2] = fmaf(f8, part[2], acc[nt][2]);
                        acc[nt][3] = fmaf(f8, part[3], acc[nt][3]);
                    }
                }
            }

#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) red[warp][nt][i][lane] = acc[nt][i];
            __syncthreads();
            for (int nt = warp; nt < NT; nt += 4) {
                if (pass0 + nt * 8 >= sl.ntok) continue;
                float v[4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    v[i] = ((red[0][nt][i][lane] + red[1][nt][i][lane]) + red[2][nt][i][lane]) +
                           red[3][nt][i][lane];
#pragma unroll
                for (int e2 = 0; e2 < 2; ++e2) {
                    const int i_tok = pass0 + nt * 8 + 2 * c + e2;
                    if (i_tok >= sl.ntok) continue;
                    float* yrow = a.y + (int64_t)(sl.list_begin + i_tok) * H;
                    yrow[m0 + r] = v[e2];
                    yrow[m0 + 8 + r] = v[2 + e2];
                }
            }
            __syncthreads();
        }
    }
}

// ---------------------------------------------------------------------------
// out[t] = sum_j w[t][j] * y[inv[t*k+j]] (j ascending) + sum_shared y + residual.
__global__ void combine_kernel(const FfnArgs a) {
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // 4 outputs each
    const int per_row = a.H / 4;
    if (gid >= (int64_t)a.T * per_row) return;
    const int t = (int)(gid / per_row);
    const int m = (int)(gid % per_row) * 4;
    const int H = a.H, k = a.k, P = a.T * a.k;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
        const int s = a.inv[t * k + j];
        if (s < 0 || s >= P) {
            report(a.status, COLI_ERR_BAD_INDEX);
            continue;
        }
        const float w = a.topk_w[t * k + j];
        const float4 y = *reinterpret_cast<const float4*>(a.y + (int64_t)s * H + m);
        acc.x = fmaf(w, y.x, acc.x);
        acc.y = fmaf(w, y.y, acc.y);
        acc.z = fmaf(w, y.z, acc.z);
        acc.w = fmaf(w, y.w, acc.w);
    }
    for (int sh = 0; sh < a.n_shared; ++sh) {
        const float4 y = *reinterpret_cast<const float4*>(a.y + (int64_t)(P + sh * a.T + t) * H + m);
        acc.x += y.x;
        acc.y += y.y;
        acc.z += y.z;
        acc.w += y.w;
    }
    const int64_t o = (int64_t)t * H + m;
    if (a.out_bf16) {
        if (a.residual) {
            const __nv_bfloat16* rb = reinterpret_cast<const __nv_bfloat16*>(a.residual) + o;
            acc.x += __bfloat162float(rb[0]);
            acc.y += __bfloat162float(rb[1]);
            acc.z += __bfloat162float(rb[2]);
            acc.w += __bfloat162float(rb[3]);
        }
        __nv_bfloat162* ob = reinterpret_cast<__nv_bfloat162*>(
            reinterpret_cast<__nv_bfloat16*>(a.out) + o);
        ob[0] = __floats2bfloat162_rn(acc.x, acc.y);
        ob[1] = __floats2bfloat162_rn(acc.z, acc.w);
    } else {
        if (a.residual) {
            const float4 rv = *reinterpret_cast<const float4*>(
                reinterpret_cast<const float*>(a.residual) + o);
            acc.x += rv.x;
            acc.y += rv.y;
            acc.z += rv.z;
            acc.w += rv.w;
        }
        *reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + o) = acc;
    }
}

void mark(int i, cudaStream_t st) {
    if (cudaEvent_t ev = profile_event(i)) cudaEventRecord(ev, st);
}

template <int NT>
cudaError_t launch_nt(const FfnArgs& a, int blocks_gu, int blocks_dn, cudaStream_t st) {
    mark(1, st);
    gateup_kernel<NT><<<blocks_gu, kThreads, 0, st>>>(a);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    mark(2, st);
    down_kernel<NT><<<blocks_dn, kThreads, 0, st>>>(a);
    mark(3, st);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ffn_gemv(const FfnArgs& a, int num_sms, cudaStream_t st) {
    const int64_t slice_count = (int64_t)a.T * a.H / 16;
    permute_x_kernel<<<(unsigned)((slice_count + 255) / 256), 256, 0, st>>>(a.T, a.H, a.x, a.xp);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;

    const int64_t max_slots = (int64_t)std::min<int64_t>(a.E, (int64_t)a.T * a.k) + a.n_shared;
    const int64_t items_gu = max_slots * (a.I / 8);
    const int64_t items_dn = max_slots * (a.H / 16);
    const int64_t cap = (int64_t)num_sms * 8;
    const int blocks_gu = (int)std::max<int64_t>(1, std::min(items_gu, cap));
    const int blocks_dn = (int)std::max<int64_t>(1, std::min(items_dn, cap));
    const int nt_needed = (a.T + 7) / 8;
    if (nt_needed <= 1) err = launch_nt<1>(a, blocks_gu, blocks_dn, st);
    else if (nt_needed <= 2) err = launch_nt<2>(a, blocks_gu, blocks_dn, st);
    else err = launch_nt<4>(a, blocks_gu, blocks_dn, st);
    if (err != cudaSuccess) return err;

    const int64_t quads = (int64_t)a.T * (a.H / 4);
    combine_kernel<<<(unsigned)((quads + 255) / 256), 256, 0, st>>>(a);
    mark(4, st);
    return cudaGetLastError();
}

cudaError_t launch_inverse_pairs(int P, const int* pairs, int* inv, int* status,
                                 cudaStream_t st) {
    inverse_pairs_kernel<<<1, 1024, 0, st>>>(P, pairs, inv, status);
    return cudaGetLastError();
}

}  // namespace coli
