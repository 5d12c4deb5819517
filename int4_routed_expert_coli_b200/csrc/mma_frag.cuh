// Register-operand pieces of the int4 kernels that run m16n8k16 MMAs on
// codes unpacked in registers (the fused decode kernel and the small-batch
// kernel): the raw fp16 unpack, the MMA, the activation-fragment load and the
// per-group offset sums that correct the unpack.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace coli {

// Unpack of a packed word (8 codes, two k16 steps of a lane's fragment) by
// the fp16 magic-number trick: step 0 takes bytes 0 and 2, step 1 bytes 1 and
// 3; e holds the even-k codes as 1032 + q, o the odd-k codes as 1152 + 16 q.
// (a & b) ^ c as one LOP3 with all operands in registers (a mask and a
// magic constant cannot both be immediates of one instruction).
__device__ __forceinline__ uint32_t and_xor(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0x6a;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

struct Magic {
    uint32_t lo_mask, lo_bias, hi_mask, hi_bias;
};
__device__ __forceinline__ Magic magic() { return {0x000F000Fu, 0x64086408u, 0x00F000F0u, 0x64806480u}; }

__device__ __forceinline__ void unpack_raw_step(uint32_t w, int step, uint32_t& e, uint32_t& o,
                                                const Magic& mg) {
    const uint32_t v = step ? (w >> 8) : w;
    e = and_xor(v, mg.lo_mask, mg.lo_bias);
    o = and_xor(v, mg.hi_mask, mg.hi_bias);
}

// A raw-unpacked pair less its offset: 1032 + q -> q (even k), 1152 + 16 q ->
// 16 q (odd k); fp16 represents both sides exactly, so the sum is exact.
__device__ __forceinline__ uint32_t strip_offset(uint32_t v, bool odd) {
    const uint32_t neg = odd ? 0xE480E480u : 0xE408E408u;  // (-1152, -1152), (-1032, -1032)
    uint32_t d;
    asm("add.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(v), "r"(neg));
    return d;
}

__device__ __forceinline__ void mma16816(float d[4], const float c[4], uint32_t a0, uint32_t a1,
                                         uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, "
        "{%4,%5,%6,%7}, {%8,%9}, {%10,%11,%12,%13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(c[2]),
          "f"(c[3]));
}

__device__ __forceinline__ void load_b_cg(uint32_t bw[8], const __half* p) {
    const uint4 b0 = __ldcg(reinterpret_cast<const uint4*>(p));
    const uint4 b1 = __ldcg(reinterpret_cast<const uint4*>(p) + 1);
    bw[0] = b0.x; bw[1] = b0.y; bw[2] = b0.z; bw[3] = b0.w;
    bw[4] = b1.x; bw[5] = b1.y; bw[6] = b1.z; bw[7] = b1.w;
}

// Offset sums of one group for this lane's two token columns: the MMA of the
// constant part of the raw unpack (1032 at even k, 1152 at odd k, every row)
// with the B fragment, i.e. 1032 * sum x_even + 1152 * sum (x_odd / 16).
__device__ __forceinline__ void offset_sums(const uint32_t bw[8], float c[4]) {
    const uint32_t ev = 0x64086408u, od = 0x64806480u;  // fp16 pairs (1032, 1032), (1152, 1152)
    const float zero[4] = {0.f, 0.f, 0.f, 0.f};
    mma16816(c, zero, ev, ev, od, od, bw[0], bw[1]);
    mma16816(c, c, ev, ev, od, od, bw[2], bw[3]);
    mma16816(c, c, ev, ev, od, od, bw[4], bw[5]);
    mma16816(c, c, ev, ev, od, od, bw[6], bw[7]);
}

}  // namespace coli
