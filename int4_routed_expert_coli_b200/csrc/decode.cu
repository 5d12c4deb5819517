// Fused decode step (T <= 8 tokens): gate/up + SwiGLU, down and the
// weighted combine in one persistent kernel, streaming every active
// expert's int4 gs64 weights from HBM exactly once per call ("batch-union",
// "yunpan.plus/t/30351-1-1", capability two).
//
// Items.  A CTA (one per SM) walks one list of items: first every gate/up
// item (8 gate rows + the same 8 up rows of one expert slot; shared experts
// first, so their weights stream while routing finishes), then every down
// item (32 rows of W_d).  A slot's down items read the h rows its gate/up
// items wrote; a per-slot counter (incremented after each gate/up item's h is
// written, read with acquire semantics) orders them, and because every CTA
// finishes all of its gate/up items before any down item, the waits cannot
// form a cycle.  The last down item of each 32-row output tile combines it:
//   out[t][m] = sum_j w[t][j] y[(t,j)][m] (j ascending) + y_shared[t][m] (+ residual)
// in fp32 in that fixed order.
//
// Data movement.  A producer warp loads each item with one 3-D TMA tensor
// copy per 8 (gate/up) or 32 (down) rows: the row is viewed as chunks of 128
// bytes plus one or two chunks past its end (zero-filled), 128-byte swizzle.
// The odd number of chunks per staged row makes the swizzle put the same
// column of different rows on different banks, so the consumers' fragment
// reads are conflict-free without per-row copies.  Scales come by bulk copy.
//
// Arithmetic as in the streaming GEMV (gemv.cu): raw fp16 unpack plus
// per-(token, group) offset sums for gate/up, exact unpack for down, m16n8k16
// MMA with fp32 accumulation, gs64 scale applied to each group's partial sum.
// For T <= 8 all tokens are the 8 MMA columns of every gate/up item, so those
// activation fragments stay in registers for the whole kernel.
//
// Reduction.  Eleven consumer warps split K; their partials go to one of two
// reduction buffers and one rotating warp per item sums them in a fixed order
// and writes the outputs, while the other warps go on to the next item.
// Every wait is bounded (COLI_ERR_TIMEOUT).
#include <algorithm>
#include <new>

#include "decode.cuh"
#include "moe_device.cuh"
#include "ptx.cuh"

namespace coli {
namespace {

constexpr int kCW = 11;                      // consumer warps (12 warps in all)
constexpr int kThreadsD = (kCW + 1) * 32;    // + producer warp
constexpr int kStagesD = 3;
constexpr int kRedBufs = 2;
constexpr int kSmemLimitD = 227 * 1024;
constexpr int kGuRows = 16, kDnRows = 32;

struct Layout {
    int gu_segs, dn_segs;       // 128-byte chunks per staged row (odd)
    int gu_op, dn_op;           // bytes of one TMA copy (8 or 32 rows)
    int gu_scale, dn_scale;     // offset of the scale block in a stage
    int gu_tx, dn_tx;           // bytes a stage receives
    int stage_bytes;
    int red_off, corr_off, stage_off, smem;
};

__host__ __device__ inline int odd_segs(int row_bytes) {
    const int chunks = row_bytes / 128;
    return chunks + ((chunks % 2 == 0) ? 1 : 2);
}

__host__ __device__ inline Layout make_layout(int H, int I) {
    Layout L;
    L.gu_segs = odd_segs(H / 2);
    L.dn_segs = odd_segs(I / 2);
    L.gu_op = 8 * L.gu_segs * 128;
    L.dn_op = kDnRows * L.dn_segs * 128;
    const int gG = H / kGroup, dG = I / kGroup;
    L.gu_scale = 2 * L.gu_op;
    L.dn_scale = L.dn_op;
    L.gu_tx = 2 * L.gu_op + kGuRows * gG * 2;
    L.dn_tx = L.dn_op + kDnRows * dG * 2;
    L.stage_bytes = ((L.gu_tx > L.dn_tx ? L.gu_tx : L.dn_tx) + 1023) / 1024 * 1024;
    L.red_off = 1024;
    L.corr_off = L.red_off + kRedBufs * kCW * 2 * 4 * 32 * 4;
    const int corr_bytes = 8 * gG * 4;
    L.stage_off = (L.corr_off + corr_bytes + 1023) / 1024 * 1024;
    L.smem = L.stage_off + kStagesD * L.stage_bytes + 1024;  // + alignment slack
    return L;
}

__device__ __forceinline__ float bf16f(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

__device__ __forceinline__ void unpack_raw(uint32_t w, uint32_t o[4]) {
    const uint32_t w8 = w >> 8;
    o[0] = (w & 0x000F000Fu) ^ 0x64086408u;
    o[1] = (w & 0x00F000F0u) ^ 0x64806480u;
    o[2] = (w8 & 0x000F000Fu) ^ 0x64086408u;
    o[3] = (w8 & 0x00F000F0u) ^ 0x64806480u;
}

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

__device__ __forceinline__ void mma16816(float d[4], const float c[4], uint32_t a0, uint32_t a1,
                                         uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, "
        "{%4,%5,%6,%7}, {%8,%9}, {%10,%11,%12,%13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(c[2]),
          "f"(c[3]));
}

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
    mma16816(p0, zero, aa[0], ab[0], aa[1], ab[1], bw[0], bw[1]);
    mma16816(p1, zero, aa[2], ab[2], aa[3], ab[3], bw[2], bw[3]);
    mma16816(p0, p0, aa[4], ab[4], aa[5], ab[5], bw[4], bw[5]);
    mma16816(p1, p1, aa[6], ab[6], aa[7], ab[7], bw[6], bw[7]);
#pragma unroll
    for (int q = 0; q < 4; ++q) part[q] = p0[q] + p1[q];
}

// 8 bytes of a staged row: codes [64 grp + 16 c, +16) of row `row`, in the
// padded, swizzled layout (segments of 128 bytes, segs per row, 16-byte
// chunk j of segment s stored at chunk j ^ (s & 7)).
__device__ __forceinline__ uint2 load_codes(const uint8_t* op_base, int row, int segs, int grp,
                                            int c) {
    const int kc = grp >> 2;                       // 128-byte segment of the row
    const int j = ((grp & 3) << 1) + (c >> 1);     // 16-byte chunk in the segment
    const int seg = row * segs + kc;
    const uint8_t* p = op_base + seg * 128 + ((j ^ (seg & 7)) << 4) + ((c & 1) << 3);
    return *reinterpret_cast<const uint2*>(p);
}

__device__ __forceinline__ void load_b(uint32_t bw[8], const __half* p) {
    const uint4 b0 = __ldcg(reinterpret_cast<const uint4*>(p));
    const uint4 b1 = __ldcg(reinterpret_cast<const uint4*>(p) + 1);
    bw[0] = b0.x; bw[1] = b0.y; bw[2] = b0.z; bw[3] = b0.w;
    bw[4] = b1.x; bw[5] = b1.y; bw[6] = b1.z; bw[7] = b1.w;
}

__device__ __forceinline__ int ld_acquire(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void tma_load_3d(void* dst, const void* tmap, int c0, int c1, int c2,
                                            uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
        "[%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_addr(dst)),
        "l"(tmap), "r"(c0), "r"(c1), "r"(c2), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

struct SlotD {
    int e, list_begin, ntok;
    bool shared, valid;
};

__device__ __forceinline__ SlotD slot_of(const FfnArgs& a, int slot, int n_act) {
    SlotD s;
    const int P = a.T * a.k;
    if (slot < a.n_shared) {
        s.e = a.E + slot;
        s.list_begin = P + slot * a.T;
        s.ntok = a.T;
        s.shared = true;
        s.valid = true;
        return s;
    }
    s.shared = false;
    const int r = slot - a.n_shared;
    const int e = r < n_act ? a.active[r] : -1;
    const int b = (e >= 0 && e < a.E) ? a.offsets[e] : 0;
    const int en = (e >= 0 && e < a.E) ? a.offsets[e + 1] : 0;
    s.valid = e >= 0 && e < a.E && b >= 0 && en >= b && en <= P && en - b <= 8;
    s.e = s.valid ? e : 0;
    s.list_begin = s.valid ? b : 0;
    s.ntok = s.valid ? en - b : 0;
    return s;
}

struct Ctx {
    const FfnArgs& a;
    const Layout& L;
    uint8_t* stage0;
    uint64_t* full;
    uint64_t* empty;
    uint64_t* red_full;
    uint64_t* red_empty;
    volatile int* abort_flag;
    float* red;
    const float* corr_s;
    int* slot_cnt;
    int* tile_cnt;
    int n_act, n_slots, gu_tiles, dn_tiles, gG, dG;
};

__device__ __forceinline__ void fail(const Ctx& x, int lane) {
    if (lane == 0) {
        report(x.a.status, COLI_ERR_TIMEOUT);
        *x.abort_flag = 1;
    }
}

// One item of the consumer walk (index `local` within its phase, `j` in the
// CTA's item sequence).  Returns false when the kernel must wind down.
template <bool kGU>
__device__ __forceinline__ bool consume_item(const Ctx& x, int64_t local, int j,
                                             const uint32_t (&breg)[kMaxGW][8], int& ready_slot) {
    const FfnArgs& a = x.a;
    const Layout& L = x.L;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = lane >> 2, c = lane & 3;
    if (*x.abort_flag) return false;
    const int stage = j % kStagesD, use = j / kStagesD;
    const int rb = j % kRedBufs, ruse = j / kRedBufs;
    const int tiles = kGU ? x.gu_tiles : x.dn_tiles;
    const int slot = (int)(local / tiles);
    const int tile = (int)(local % tiles);
    const SlotD sl = slot_of(a, slot, x.n_act);
    if (!sl.valid && threadIdx.x == 0) report(a.status, COLI_ERR_BAD_INDEX);
    const int G = kGU ? x.gG : x.dG;
    const int g_lo = (G * warp) / kCW, g_hi = (G * (warp + 1)) / kCW;

    float acc[2][4];
#pragma unroll
    for (int m = 0; m < 2; ++m)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[m][q] = 0.f;

    bool ok = true;
    uint32_t bdn[kGU ? 1 : kMaxDW][8];
    if constexpr (!kGU) {
        // this slot's h must be complete (every gate/up item counted)
        if (sl.valid && slot > ready_slot) {
            const uint64_t t0 = global_timer_ns();
            while (ld_acquire(x.slot_cnt + slot) < x.gu_tiles) {
                if (global_timer_ns() - t0 > kWaitLimitNs) {
                    ok = false;
                    break;
                }
            }
            if (ok) ready_slot = slot;
        }
        // B fragments: this expert's h rows, loaded before waiting on the stage
#pragma unroll
        for (int i = 0; i < kMaxDW; ++i) {
            const int grp = g_lo + i;
            if (ok && grp < g_hi && r < sl.ntok) {
                load_b(bdn[i], a.hp + (int64_t)(sl.list_begin + r) * a.I + grp * kGroup + c * 16);
            } else {
#pragma unroll
                for (int q = 0; q < 8; ++q) bdn[i][q] = 0u;
            }
        }
    }
    if (!ok || !mbar_wait(&x.full[stage], use & 1)) {
        fail(x, lane);
        return false;
    }
    const uint8_t* st = x.stage0 + (size_t)stage * L.stage_bytes;
    if (sl.valid) {
        if constexpr (kGU) {
            const uint16_t* scA = reinterpret_cast<const uint16_t*>(st + L.gu_scale) + r * G;
            const uint16_t* scB = reinterpret_cast<const uint16_t*>(st + L.gu_scale) + (8 + r) * G;
#pragma unroll
            for (int i = 0; i < kMaxGW; ++i) {
                const int grp = g_lo + i;
                if (grp >= g_hi) break;
                const uint2 wa = load_codes(st, r, L.gu_segs, grp, c);
                const uint2 wb = load_codes(st + L.gu_op, r, L.gu_segs, grp, c);
                const float fa = bf16f(scA[grp]), fb = bf16f(scB[grp]);
                const float cr0 = x.corr_s[(2 * c) * G + grp], cr1 = x.corr_s[(2 * c + 1) * G + grp];
                float part[4];
                group_partial<false>(part, wa, wb, breg[i]);
                acc[0][0] = fmaf(fa, part[0] - cr0, acc[0][0]);
                acc[0][1] = fmaf(fa, part[1] - cr1, acc[0][1]);
                acc[0][2] = fmaf(fb, part[2] - cr0, acc[0][2]);
                acc[0][3] = fmaf(fb, part[3] - cr1, acc[0][3]);
            }
        } else {
            const uint16_t* sc = reinterpret_cast<const uint16_t*>(st + L.dn_scale);
#pragma unroll
            for (int i = 0; i < kMaxDW; ++i) {
                const int grp = g_lo + i;
                if (grp >= g_hi) break;
#pragma unroll
                for (int m = 0; m < 2; ++m) {
                    const uint2 wa = load_codes(st, m * 16 + r, L.dn_segs, grp, c);
                    const uint2 wb = load_codes(st, m * 16 + 8 + r, L.dn_segs, grp, c);
                    const float fa = bf16f(sc[(m * 16 + r) * G + grp]);
                    const float fb = bf16f(sc[(m * 16 + 8 + r) * G + grp]);
                    float part[4];
                    group_partial<true>(part, wa, wb, bdn[i]);
                    acc[m][0] = fmaf(fa, part[0], acc[m][0]);
                    acc[m][1] = fmaf(fa, part[1], acc[m][1]);
                    acc[m][2] = fmaf(fb, part[2], acc[m][2]);
                    acc[m][3] = fmaf(fb, part[3], acc[m][3]);
                }
            }
        }
    }
    // the stage is no longer read by this warp
    __syncwarp();
    if (lane == 0) mbar_arrive(&x.empty[stage]);

    // partials -> reduction buffer rb (free once item j - 2's epilogue read it)
    if (ruse > 0 && !mbar_wait(&x.red_empty[rb], (ruse - 1) & 1)) {
        fail(x, lane);
        return false;
    }
    float* rbuf = x.red + rb * (kCW * 2 * 4 * 32);
#pragma unroll
    for (int m = 0; m < 2; ++m)
#pragma unroll
        for (int q = 0; q < 4; ++q) rbuf[((warp * 2 + m) * 4 + q) * 32 + lane] = acc[m][q];
    __syncwarp();
    if (lane == 0) mbar_arrive(&x.red_full[rb]);

    if (warp != j % kCW) return true;
    // --------------------- epilogue of this item (one warp) ---------------------
    if (!mbar_wait(&x.red_full[rb], ruse & 1)) {
        fail(x, lane);
        return false;
    }
    float v[2][4];
#pragma unroll
    for (int m = 0; m < 2; ++m)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float s = 0.f;
#pragma unroll
            for (int w = 0; w < kCW; ++w) s += rbuf[((w * 2 + m) * 4 + q) * 32 + lane];
            v[m][q] = s;
        }
    __syncwarp();
    if (lane == 0) mbar_arrive(&x.red_empty[rb]);
    const int P = a.T * a.k;
    if constexpr (kGU) {
        if (!sl.valid) return true;
        // columns are tokens 0..7: find each token's row on this expert's list
#pragma unroll
        for (int e2 = 0; e2 < 2; ++e2) {
            const int t = 2 * c + e2;
            int orow = -1;
            if (t < a.T) {
                if (sl.shared) {
                    orow = sl.list_begin + t;
                } else {
                    for (int i = 0; i < sl.ntok; ++i)
                        if (a.pairs[sl.list_begin + i] / a.k == t) orow = sl.list_begin + i;
                }
            }
            if (orow < 0) continue;
            const int n = tile * 8 + r;
            const int hcol = (n / kGroup) * kGroup + perm64(n % kGroup);
            const float gv = v[0][e2], uv = v[0][2 + e2];
            float h = gv / (1.f + expf(-gv)) * uv;
            if (fabsf(h) > 65504.f) {
                report(a.status, COLI_ERR_RANGE);
                h = copysignf(65504.f, h);
            }
            a.hp[(int64_t)orow * a.I + hcol] = __float2half_rn(h);
        }
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(x.slot_cnt + slot, 1);
    } else {
#pragma unroll
        for (int e2 = 0; e2 < 2; ++e2) {
            const int i_tok = 2 * c + e2;  // column = position on the expert's list
            if (!sl.valid || i_tok >= sl.ntok) continue;
            float* yrow = a.y + (int64_t)(sl.list_begin + i_tok) * a.H + tile * kDnRows;
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                yrow[m * 16 + r] = v[m][e2];
                yrow[m * 16 + 8 + r] = v[m][2 + e2];
            }
        }
        __threadfence();
        __syncwarp();
        int last = 0;
        if (lane == 0) last = atomicAdd(x.tile_cnt + tile, 1) == x.n_slots - 1;
        last = __shfl_sync(0xffffffffu, last, 0);
        if (last) {
            __threadfence();
            // combine rows [tile * 32, +32) of every token, fixed order
            for (int idx = lane; idx < a.T * kDnRows; idx += 32) {
                const int t = idx / kDnRows, m = tile * kDnRows + idx % kDnRows;
                float o = 0.f;
                for (int jj = 0; jj < a.k; ++jj) {
                    const int s = a.inv[t * a.k + jj];
                    if (s < 0 || s >= P) {
                        report(a.status, COLI_ERR_BAD_INDEX);
                        continue;
                    }
                    o = fmaf(a.topk_w[t * a.k + jj], __ldcg(a.y + (int64_t)s * a.H + m), o);
                }
                for (int sh = 0; sh < a.n_shared; ++sh)
                    o += __ldcg(a.y + (int64_t)(P + sh * a.T + t) * a.H + m);
                const int64_t oi = (int64_t)t * a.H + m;
                if (a.out_bf16) {
                    if (a.residual)
                        o += __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(a.residual)[oi]);
                    reinterpret_cast<__nv_bfloat16*>(a.out)[oi] = __float2bfloat16_rn(o);
                } else {
                    if (a.residual) o += reinterpret_cast<const float*>(a.residual)[oi];
                    reinterpret_cast<float*>(a.out)[oi] = o;
                }
            }
        }
    }
    return true;
}

__global__ void __launch_bounds__(kThreadsD, 1) decode_fused_kernel(const DecodeArgs d) {
    const FfnArgs& a = d.f;
    const Layout L = make_layout(a.H, a.I);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kStagesD;
    uint64_t* red_full = empty + kStagesD;
    uint64_t* red_empty = red_full + kRedBufs;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + 512);
    float* red = reinterpret_cast<float*>(smem + L.red_off);  // [2][8 warps][2 mt][4][32]
    float* corr_s = reinterpret_cast<float*>(smem + L.corr_off);  // [8 tokens][H/64]
    uint8_t* stage0 = smem + L.stage_off;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStagesD; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kCW);
        }
        for (int b = 0; b < kRedBufs; ++b) {
            mbar_init(&red_full[b], kCW);
            mbar_init(&red_empty[b], 1);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    pdl_launch_dependents();

    const int gG = a.H / kGroup, dG = a.I / kGroup;
    const int gu_tiles = a.I / 8, dn_tiles = a.H / kDnRows;
    int* slot_cnt = reinterpret_cast<int*>(reinterpret_cast<char*>(a.status) + kSlotCntOffset);
    int* tile_cnt = reinterpret_cast<int*>(reinterpret_cast<char*>(a.status) + kTileCntOffset);

    if (warp == kCW) {
        // ------------------------------ producer ------------------------------
        if (lane == 0) {
            const uint64_t policy = policy_evict_first();
            const int64_t shared_gu = (int64_t)a.n_shared * gu_tiles;
            int64_t n_gu = -1, n_all = -1;
            int n_act = 0;
            int j = 0;
            bool aborted = false;
            for (int64_t item = blockIdx.x;; item += gridDim.x, ++j) {
                if (n_all < 0 && item >= shared_gu) {
                    pdl_wait();
                    n_act = *reinterpret_cast<const volatile int*>(a.n_active);
                    if (n_act < 0 || n_act > a.E) n_act = 0;
                    n_gu = (int64_t)(n_act + a.n_shared) * gu_tiles;
                    n_all = n_gu + (int64_t)(n_act + a.n_shared) * dn_tiles;
                }
                if (n_all >= 0 && item >= n_all) break;
                if (*abort_flag) break;
                const int stage = j % kStagesD, use = j / kStagesD;
                if (use > 0 && !mbar_wait(&empty[stage], (use - 1) & 1)) {
                    report(a.status, COLI_ERR_TIMEOUT);
                    *abort_flag = 1;
                    aborted = true;
                    break;
                }
                if (item == a.withhold_item) continue;  // test hook: this stage never fills
                const bool gu = n_gu < 0 || item < n_gu;
                const int64_t local = gu ? item : item - n_gu;
                const int tiles = gu ? gu_tiles : dn_tiles;
                const SlotD sl = slot_of(a, (int)(local / tiles), n_act);
                uint8_t* st = stage0 + (size_t)stage * L.stage_bytes;
                if (!sl.valid) {
                    mbar_arrive(&full[stage]);
                    continue;
                }
                const int tile = (int)(local % tiles);
                const DevExpert ex = a.experts[sl.e];
                const CUtensorMap* maps = d.maps + (size_t)sl.e * 3;
                if (gu) {
                    mbar_arrive_expect_tx(&full[stage], L.gu_tx);
                    const int n0 = tile * 8;
                    tma_load_3d(st, maps + 0, 0, 0, n0, &full[stage], policy);
                    tma_load_3d(st + L.gu_op, maps + 1, 0, 0, n0, &full[stage], policy);
                    bulk_g2s_evict_first(st + L.gu_scale, ex.gate_s + (int64_t)n0 * gG, 8 * gG * 2,
                                         &full[stage], policy);
                    bulk_g2s_evict_first(st + L.gu_scale + 8 * gG * 2, ex.up_s + (int64_t)n0 * gG,
                                         8 * gG * 2, &full[stage], policy);
                } else {
                    mbar_arrive_expect_tx(&full[stage], L.dn_tx);
                    const int m0 = tile * kDnRows;
                    tma_load_3d(st, maps + 2, 0, 0, m0, &full[stage], policy);
                    bulk_g2s_evict_first(st + L.dn_scale, ex.down_s + (int64_t)m0 * dG,
                                         kDnRows * dG * 2, &full[stage], policy);
                }
            }
            if (aborted || *abort_flag) {
                // let the copies already issued land before the CTA goes away
                for (int back = 1; back <= kStagesD && back <= j; ++back) {
                    const int jj = j - back;
                    (void)mbar_wait(&full[jj % kStagesD], (jj / kStagesD) & 1);
                }
            }
        }
        return;
    }

    // -------------------------------- consumers --------------------------------
    pdl_wait();
    int n_act = *reinterpret_cast<const volatile int*>(a.n_active);
    if (n_act < 0 || n_act > a.E) {
        if (threadIdx.x == 0) report(a.status, COLI_ERR_BAD_INDEX);
        n_act = 0;
    }
    const int n_slots = n_act + a.n_shared;
    const int64_t n_gu = (int64_t)n_slots * gu_tiles;
    const int64_t n_all = n_gu + (int64_t)n_slots * dn_tiles;
    const int r = lane >> 2, c = lane & 3;

    // gate/up activation fragments of all T tokens (columns) and offset sums
    const int gg_lo = (gG * warp) / kCW, gg_hi = (gG * (warp + 1)) / kCW;
    uint32_t breg[kMaxGW][8];
#pragma unroll
    for (int i = 0; i < kMaxGW; ++i) {
        const int grp = gg_lo + i;
        if (grp < gg_hi && r < a.T) {
            load_b(breg[i], a.xp + (int64_t)r * a.H + grp * kGroup + c * 16);
        } else {
#pragma unroll
            for (int q = 0; q < 8; ++q) breg[i][q] = 0u;
        }
    }
    for (int i = threadIdx.x; i < 8 * gG; i += kCW * 32)
        corr_s[i] = (i / gG) < a.T ? a.corr[i] : 0.f;
    named_barrier(1, kCW * 32);

    int ready_slot = -1;  // down: highest slot whose h this warp has seen complete
    int j = 0;
    Ctx ctx{a, L, stage0, full, empty, red_full, red_empty, abort_flag, red, corr_s,
            slot_cnt, tile_cnt, n_act, n_slots, gu_tiles, dn_tiles, gG, dG};
    // phase 1: gate/up items (activation fragments live in registers)
    int64_t item = blockIdx.x;
    for (; item < n_gu; item += gridDim.x, ++j)
        if (!consume_item<true>(ctx, item, j, breg, ready_slot)) return;
    // phase 2: down items
    for (; item < n_all; item += gridDim.x, ++j)
        if (!consume_item<false>(ctx, item - n_gu, j, breg, ready_slot)) return;
}

}  // namespace

bool decode_supported(int H, int I, int T) {
    if (T < 1 || T > 8 || H % 256 || I % 256) return false;
    const Layout L = make_layout(H, I);
    if (L.smem > kSmemLimitD) return false;
    if ((H / kGroup + kCW - 1) / kCW > kMaxGW) return false;
    if ((I / kGroup + kCW - 1) / kCW > kMaxDW) return false;
    return L.gu_segs <= 256 && L.dn_segs <= 256;
}

cudaError_t build_decode_maps(const DevExpert* host_experts, int n, int H, int I,
                              CUtensorMap** d_maps) {
    *d_maps = nullptr;
    const Layout L = make_layout(H, I);
    CUtensorMap* maps = new (std::nothrow) CUtensorMap[(size_t)n * 3];
    if (!maps) return cudaErrorMemoryAllocation;
    bool ok = true;
    for (int e = 0; e < n && ok; ++e) {
        const DevExpert& x = host_experts[e];
        ok = encode_tma(&maps[e * 3 + 0], x.gate_q, 3, I, H / 2, L.gu_segs, 8) &&
             encode_tma(&maps[e * 3 + 1], x.up_q, 3, I, H / 2, L.gu_segs, 8) &&
             encode_tma(&maps[e * 3 + 2], x.down_q, 3, H, I / 2, L.dn_segs, kDnRows);
    }
    if (!ok) {
        delete[] maps;
        return cudaErrorInvalidValue;
    }
    cudaError_t err = cudaMalloc(d_maps, sizeof(CUtensorMap) * (size_t)n * 3);
    if (err == cudaSuccess)
        err = cudaMemcpy(*d_maps, maps, sizeof(CUtensorMap) * (size_t)n * 3, cudaMemcpyHostToDevice);
    delete[] maps;
    if (err != cudaSuccess && *d_maps) {
        cudaFree(*d_maps);
        *d_maps = nullptr;
    }
    return err;
}

cudaError_t launch_decode_fused(const FfnArgs& f, const CUtensorMap* maps, int num_sms,
                                cudaStream_t st) {
    DecodeArgs d;
    d.f = f;
    d.f.withhold_item = take_withhold_item();
    d.maps = maps;
    const Layout L = make_layout(f.H, f.I);
    cudaError_t err = cudaFuncSetAttribute(decode_fused_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, L.smem);
    if (err != cudaSuccess) return err;
    const int64_t max_slots = std::min<int64_t>(f.E, (int64_t)f.T * f.k) + f.n_shared;
    const int64_t items = max_slots * (f.I / 8 + f.H / kDnRows);
    const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>(num_sms, items));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(blocks);
    cfg.blockDim = dim3(kThreadsD);
    cfg.dynamicSmemBytes = L.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    profile_mark(1, st);
    err = cudaLaunchKernelEx(&cfg, decode_fused_kernel, d);
    profile_mark(2, st);
    profile_mark(3, st);
    profile_mark(4, st);
    return err;
}

}  // namespace coli
