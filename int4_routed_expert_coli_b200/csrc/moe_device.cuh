// Device bodies of the routing and batch-union steps, shared by their
// stand-alone kernels and by the fused small-batch preparation kernel.
#pragma once

#include "coli_internal.cuh"

namespace coli {

// ---------------------------------------------------------------------------
// Routing: the router picks k of the E routed experts for every token
// ("zhichai.net/topic/178503686", MoE-sparsity section).  Exact and
// deterministic: each logit becomes a 64-bit key that orders by value
// descending (NaN lowest, -0 == +0) and then by expert index ascending; k
// rounds of a warp-wide max pick the winners in slot order.

__device__ __forceinline__ uint64_t rank_key(float v, int e) {
    uint32_t k32;
    if (isnan(v)) {
        k32 = 0u;
    } else {
        const uint32_t b = __float_as_uint(v + 0.0f);  // -0 + 0 = +0
        k32 = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
    }
    return ((uint64_t)k32 << 32) | (uint32_t)(0xFFFFFFFFu - (uint32_t)e);
}

// One warp routes one token row.  NV = logits per lane (E <= 32 * NV).
// Weights: w_j = exp(l_j - m) / sum_i exp(l_i - m) over the chosen set in
// double, rounded to fp32 once; +inf entries share the weight when m = +inf;
// 1/k each when m is -inf or NaN; NaN entries contribute 0.
template <int NV>
__device__ __forceinline__ void route_row(const float* __restrict__ row, int E, int k, int lane,
                                          int* __restrict__ idx_out, float* __restrict__ w_out) {
    uint64_t key[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int e = lane + 32 * i;
        key[i] = e < E ? rank_key(row[e], e) : 0ull;  // padding never wins (k <= E)
    }
    int my_idx = -1;  // lane j keeps the j-th winner
    for (int j = 0; j < k; ++j) {
        uint64_t best = 0ull;
#pragma unroll
        for (int i = 0; i < NV; ++i) best = key[i] > best ? key[i] : best;
        // warp-wide max of the 64-bit keys: the high words, then the low words
        // of the lanes holding that high word (keys are unique)
        const uint32_t hi = __reduce_max_sync(0xffffffffu, (uint32_t)(best >> 32));
        const uint32_t lo =
            __reduce_max_sync(0xffffffffu, (uint32_t)(best >> 32) == hi ? (uint32_t)best : 0u);
        const uint64_t win = ((uint64_t)hi << 32) | lo;
#pragma unroll
        for (int i = 0; i < NV; ++i) key[i] = key[i] == win ? 0ull : key[i];
        if (lane == j) my_idx = (int)(0xFFFFFFFFu - lo);
    }
    const float v = (lane < k) ? row[my_idx] : 0.f;
    const float m = __shfl_sync(0xffffffffu, v, 0);
    double wj;
    if (isinf(m) && m > 0.f) {
        const bool pinf = lane < k && isinf(v) && v > 0.f;
        const unsigned inf_mask = __ballot_sync(0xffffffffu, pinf);
        wj = pinf ? 1.0 / (double)__popc(inf_mask) : 0.0;
    } else if (isnan(m) || (isinf(m) && m < 0.f)) {
        wj = 1.0 / (double)k;
    } else {
        const double ej = (lane < k && !isnan(v)) ? exp((double)v - (double)m) : 0.0;
        double z = ej;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
        wj = ej / z;
    }
    if (lane < k) {
        idx_out[lane] = my_idx;
        w_out[lane] = (float)wj;
    }
}

// ---------------------------------------------------------------------------
// Routing of one token row by one warp at low latency (the same selection
// and weights as route_row).  Top-k for E <= 256 and k in {1, 2, 4, 8}: each
// lane sorts its 8 keys (descending, a 19-comparator network), then five
// butterfly levels merge the lanes' lists: a lane keeps the 8 largest of its
// 16 keys and its partner's (the element-wise max of one list and the other
// reversed is a bitonic sequence holding them; three half-cleaner stages
// sort it), so after the last level every lane holds the row's 8 largest
// keys in order.  No warp-wide reduction sits on the critical path, which a
// round of the k-round selection needs twice.  The winners' logits come
// back from their keys, so no second read of the row is needed.  Other
// shapes use route_row.

__device__ __forceinline__ void cas_desc(uint64_t& a, uint64_t& b) {
    const bool sw = a < b;
    const uint64_t hi = sw ? b : a, lo = sw ? a : b;
    a = hi;
    b = lo;
}

__device__ __forceinline__ void sort8_desc(uint64_t (&v)[8]) {
    cas_desc(v[0], v[2]); cas_desc(v[1], v[3]); cas_desc(v[4], v[6]); cas_desc(v[5], v[7]);
    cas_desc(v[0], v[4]); cas_desc(v[1], v[5]); cas_desc(v[2], v[6]); cas_desc(v[3], v[7]);
    cas_desc(v[0], v[1]); cas_desc(v[2], v[3]); cas_desc(v[4], v[5]); cas_desc(v[6], v[7]);
    cas_desc(v[2], v[4]); cas_desc(v[3], v[5]);
    cas_desc(v[1], v[4]); cas_desc(v[3], v[6]);
    cas_desc(v[1], v[2]); cas_desc(v[3], v[4]); cas_desc(v[5], v[6]);
}

// v (sorted, descending) <- the 8 largest of v and lane ^ d's list, sorted.
__device__ __forceinline__ void merge8_xor(uint64_t (&v)[8], int d) {
    uint64_t o[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)v[i], d);
        const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(v[i] >> 32), d);
        o[i] = ((uint64_t)hi << 32) | lo;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = v[i] > o[7 - i] ? v[i] : o[7 - i];
#pragma unroll
    for (int s = 4; s >= 1; s >>= 1)
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if ((i & s) == 0) cas_desc(v[i], v[i + s]);
}

// The logit a key was made from (-0 comes back as +0, NaN as a NaN).
__device__ __forceinline__ float key_value(uint64_t key) {
    const uint32_t k32 = (uint32_t)(key >> 32);
    return __uint_as_float((k32 & 0x80000000u) ? (k32 & 0x7FFFFFFFu) : ~k32);
}

// True when route_row_fast handles the shape (else route_row).
template <int NV>
__device__ __forceinline__ bool route_fast_ok(int k) {
    return NV <= 8 && k <= 8 && (k & (k - 1)) == 0;
}

// This lane's logits of one row (e = lane + 32 i), loaded before the row is
// routed so the loads can be in flight with others.
template <int NV>
__device__ __forceinline__ void load_row8(const float* __restrict__ row, int E, int lane,
                                          float (&val)[8]) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int e = lane + 32 * i;
        val[i] = (i < NV && e < E) ? row[e] : 0.f;
    }
}

// Routes one row from the values load_row8 gave (route_fast_ok(k) holds).
template <int NV>
__device__ __forceinline__ void route_row_fast(const float (&val)[8], int E, int k, int lane,
                                               int* __restrict__ idx_out, float* __restrict__ w_out) {
    uint64_t v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int e = lane + 32 * i;
        v[i] = (i < NV && e < E) ? rank_key(val[i], e) : 0ull;  // padding never wins (k <= E)
    }
    sort8_desc(v);
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) merge8_xor(v, d);
    uint64_t mine = 0ull;
#pragma unroll
    for (int i = 0; i < 8; ++i) mine = lane == i ? v[i] : mine;
    const int my_idx = (int)(0xFFFFFFFFu - (uint32_t)mine);
    // weights: as route_row, over the k lanes holding the picks
    const float x = (lane < k) ? key_value(mine) : 0.f;
    const float m = __shfl_sync(0xffffffffu, x, 0);
    double wj;
    if (isinf(m) && m > 0.f) {
        const bool pinf = lane < k && isinf(x) && x > 0.f;
        const unsigned inf_mask = __ballot_sync(0xffffffffu, pinf);
        wj = pinf ? 1.0 / (double)__popc(inf_mask) : 0.0;
    } else if (isnan(m) || (isinf(m) && m < 0.f)) {
        wj = 1.0 / (double)k;
    } else {
        const double ej = (lane < k && !isnan(x)) ? exp((double)x - (double)m) : 0.0;
        double z = ej;
        for (int o = k >> 1; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
        wj = ej / z;
    }
    if (lane < k) {
        idx_out[lane] = my_idx;
        w_out[lane] = (float)wj;
    }
}

// ---------------------------------------------------------------------------
// Batch-union: all positions routed to one expert are listed together so the
// expert is read once for all of them ("yunpan.plus/t/30351-1-1",
// capability two, batch-union bullet).  A stable counting sort of the P
// pairs by expert in one CTA of kUnionThreads threads: per-warp histograms
// (one leader per distinct expert in a 32-pair slice), a scan over
// (expert, warp), then a second pass writing each pair at
// base + rank-among-equal-keys.  No position comes from an atomic ticket.

constexpr int kUnionThreads = 1024;
constexpr int kUnionWarps = kUnionThreads / 32;

__host__ __device__ constexpr size_t union_smem_bytes(int E) {
    return sizeof(int) * (size_t)kUnionWarps * E;
}

// Exclusive scan of one int per thread over a block of <= 1024 threads.
// `tmp` holds 32 ints.  Returns the prefix; *total gets the block sum.
__device__ __forceinline__ int block_exclusive_scan(int v, int* tmp, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) tmp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int nw = blockDim.x >> 5;
        int s = lane < nw ? tmp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += n;
        }
        tmp[lane] = s;
    }
    __syncthreads();
    const int base = warp > 0 ? tmp[warp - 1] : 0;
    *total = tmp[(blockDim.x >> 5) - 1];
    __syncthreads();
    return base + incl - v;
}

// Must be called by all kUnionThreads threads of the block.  `hist` is
// union_smem_bytes(E) of shared memory.  `inv` (nullable) receives, for each
// pair p, its position in `pairs` (-1 for a dropped pair).
__device__ __forceinline__ void union_block(int P, int E, const int* __restrict__ idx,
                                            int* __restrict__ counts, int* __restrict__ offsets,
                                            int* __restrict__ pairs, int* __restrict__ active,
                                            int* __restrict__ n_active, int* __restrict__ inv,
                                            int* status, int* hist, int* scan_tmp) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int i = threadIdx.x; i < kUnionWarps * E; i += blockDim.x) hist[i] = 0;
    __syncthreads();

    const int chunk = ((P + kUnionWarps - 1) / kUnionWarps + 31) / 32 * 32;
    const int p_begin = warp * chunk;
    const int p_end = min(P, p_begin + chunk);
    int* my_hist = hist + warp * E;

    for (int p0 = p_begin; p0 < p_end; p0 += 32) {
        const int p = p0 + lane;
        int e = p < p_end ? idx[p] : -1;
        if (p < p_end && (e < 0 || e >= E)) {
            report(status, COLI_ERR_BAD_INDEX);
            e = -1;
        }
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        if (e >= 0 && (peers & lt_mask) == 0) my_hist[e] += __popc(peers);
        __syncwarp();
    }
    __syncthreads();

    int cnt = 0;
    const int e_self = threadIdx.x;
    if (e_self < E) {
        for (int w = 0; w < kUnionWarps; ++w) {
            const int c = hist[w * E + e_self];
            hist[w * E + e_self] = cnt;
            cnt += c;
        }
    }
    int total;
    const int off = block_exclusive_scan(e_self < E ? cnt : 0, scan_tmp, &total);
    int act_total;
    const int act_pos =
        block_exclusive_scan((e_self < E && cnt > 0) ? 1 : 0, scan_tmp, &act_total);
    if (e_self < E) {
        counts[e_self] = cnt;
        offsets[e_self] = off;
        for (int w = 0; w < kUnionWarps; ++w) hist[w * E + e_self] += off;
        if (cnt > 0) active[act_pos] = e_self;
    }
    if (threadIdx.x == 0) {
        offsets[E] = total;
        *n_active = act_total;
    }
    for (int e = act_total + threadIdx.x; e < E; e += blockDim.x) active[e] = -1;
    __syncthreads();

    for (int p0 = p_begin; p0 < p_end; p0 += 32) {
        const int p = p0 + lane;
        int e = p < p_end ? idx[p] : -1;
        if (e >= E) e = -1;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        if (e >= 0) {
            const int pos = my_hist[e] + __popc(peers & lt_mask);
            pairs[pos] = p;
            if (inv) inv[p] = pos;
        } else if (p < p_end && inv) {
            inv[p] = -1;
        }
        __syncwarp();
        if (e >= 0 && (peers & lt_mask) == 0) my_hist[e] += __popc(peers);
        __syncwarp();
    }
}

// ---------------------------------------------------------------------------
// Activation operand of the streaming gate/up GEMV (see gemv.cu).
//
// Fragment order: position of element j (0..63) of a 64-element scale group
// in the permuted layout the m16n8k16 B fragments read.
__host__ __device__ __forceinline__ int perm64(int j) {
    const int c = j >> 4, jj = j & 15;
    const int m = ((jj >> 3) << 1) + ((jj & 3) >> 1);
    const int e = (jj & 7) >> 2;
    const int odd = jj & 1;
    return c * 16 + 4 * m + 2 * odd + e;
}

// One 64-element group of a bf16 activation row -> fp16 operand in fragment
// order, odd elements divided by 16 (they meet codes unpacked as 16 (q + 72)),
// and the group's offset sum
//   corr = 1032 * sum_{k even} x_k + 1152 * sum_{k odd} (x_k / 16),
// the part of the MMA result that the unpack offsets contribute (even codes
// are unpacked as 1032 + q, odd ones as 1152 + 16 q).  Values outside the
// fp16 range are clamped and reported as COLI_ERR_RANGE.
__device__ __forceinline__ float prepare_group64(const uint16_t* __restrict__ src,
                                                 __half* __restrict__ dst, int* status) {
    float se = 0.f, so = 0.f;
    uint16_t o[64];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const uint4 in = *reinterpret_cast<const uint4*>(src + q * 8);
        const uint16_t* v = reinterpret_cast<const uint16_t*>(&in);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int j = q * 8 + i;
            float f = __uint_as_float((uint32_t)v[i] << 16);
            if (fabsf(f) > 65504.f) {
                report(status, COLI_ERR_RANGE);
                f = copysignf(65504.f, f);
            }
            __half h = __float2half_rn((j & 1) ? f * 0.0625f : f);
            if (j & 1) so += __half2float(h);
            else se += __half2float(h);
            o[perm64(j)] = *reinterpret_cast<uint16_t*>(&h);
        }
    }
#pragma unroll
    for (int q = 0; q < 8; ++q)
        reinterpret_cast<uint4*>(dst)[q] = reinterpret_cast<const uint4*>(o)[q];
    return 1032.f * se + 1152.f * so;
}

}  // namespace coli
