// Router: logits GEMV and warp-per-token top-k with renormalised softmax.
//
// The router picks k of the E routed experts for every token
// ("zhichai.net/topic/178503686", MoE-sparsity section: 256 experts, 8 + 1
// active per layer).  Selection is exact and deterministic (the pages' rule
// that routing semantics never change silently, "yunpan.plus/t/30351-1-1",
// capability four): each logit becomes a 64-bit key that orders by value
// descending (NaN lowest, -0 == +0) and then by expert index ascending, and
// k rounds of a warp-wide max pick the winners.
#include "coli_internal.cuh"

namespace coli {
namespace {

// logits[t][e] = sum_h f32(x[t][h]) * wr[e][h], fp32; one warp per (t, e).
__global__ void router_logits_kernel(int T, int E, int H, const __nv_bfloat16* __restrict__ x,
                                     const float* __restrict__ wr, float* __restrict__ logits) {
    const int lane = threadIdx.x & 31;
    const int64_t item = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (item >= (int64_t)T * E) return;
    const int t = (int)(item / E), e = (int)(item % E);
    const __nv_bfloat16* xr = x + (int64_t)t * H;
    const float* wrow = wr + (int64_t)e * H;
    float acc = 0.f;
    for (int h = lane; h < H; h += 32) acc = fmaf(__bfloat162float(xr[h]), wrow[h], acc);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) logits[item] = acc;
}

// Order-preserving key: larger key = ranked first.  NaN -> 0 (lowest),
// -0 -> +0, other floats map monotonically above every NaN.
__device__ __forceinline__ uint64_t rank_key(float v, int e) {
    uint32_t k32;
    if (isnan(v)) {
        k32 = 0u;
    } else {
        uint32_t b = __float_as_uint(v + 0.0f);  // -0 + 0 = +0
        k32 = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
    }
    return ((uint64_t)k32 << 32) | (uint32_t)(0xFFFFFFFFu - (uint32_t)e);
}

__device__ __forceinline__ uint64_t warp_max_u64(uint64_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        uint64_t other = __shfl_xor_sync(0xffffffffu, v, o);
        v = other > v ? other : v;
    }
    return v;
}

// One warp per token.  NV = logits held per lane (E <= 32 * NV).
template <int NV>
__global__ void route_kernel(int T, int E, int k, const float* __restrict__ logits,
                             int* __restrict__ idx_out, float* __restrict__ w_out) {
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    const float* row = logits + (int64_t)t * E;

    uint64_t key[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int e = lane + 32 * i;
        key[i] = e < E ? rank_key(row[e], e) : 0ull;  // padding: never chosen (k <= E)
    }

    int my_idx = -1;  // lane j keeps the j-th winner
    for (int j = 0; j < k; ++j) {
        uint64_t best = 0ull;
#pragma unroll
        for (int i = 0; i < NV; ++i) best = key[i] > best ? key[i] : best;
        best = warp_max_u64(best);
        const int e = (int)(0xFFFFFFFFu - (uint32_t)(best & 0xFFFFFFFFull));
        if ((e & 31) == lane) {
#pragma unroll
            for (int i = 0; i < NV; ++i)
                if (i == (e >> 5)) key[i] = 0ull;
        }
        if (lane == j) my_idx = e;
    }

    // Weights in double, rounded to fp32 once.
    const float v = (lane < k) ? row[my_idx] : 0.f;
    const float m = __shfl_sync(0xffffffffu, v, 0);
    double wj;
    if (isinf(m) && m > 0.f) {
        const unsigned inf_mask = __ballot_sync(0xffffffffu, lane < k && isinf(v) && v > 0.f);
        wj = (lane < k && isinf(v) && v > 0.f) ? 1.0 / (double)__popc(inf_mask) : 0.0;
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
        idx_out[(int64_t)t * k + lane] = my_idx;
        w_out[(int64_t)t * k + lane] = (float)wj;
    }
}

}  // namespace

cudaError_t launch_router_logits(int T, int E, int H, const __nv_bfloat16* x, const float* wr,
                                 float* logits, cudaStream_t st) {
    const int64_t items = (int64_t)T * E;
    const int warps = 8;
    const int64_t blocks = (items + warps - 1) / warps;
    router_logits_kernel<<<(unsigned)blocks, warps * 32, 0, st>>>(T, E, H, x, wr, logits);
    return cudaGetLastError();
}

cudaError_t launch_route(int T, int E, int k, const float* logits, int* idx, float* w,
                         cudaStream_t st) {
    const int warps = 8;
    const unsigned blocks = (unsigned)((T + warps - 1) / warps);
    const int nv = (E + 31) / 32;
    if (nv <= 1) route_kernel<1><<<blocks, warps * 32, 0, st>>>(T, E, k, logits, idx, w);
    else if (nv <= 2) route_kernel<2><<<blocks, warps * 32, 0, st>>>(T, E, k, logits, idx, w);
    else if (nv <= 4) route_kernel<4><<<blocks, warps * 32, 0, st>>>(T, E, k, logits, idx, w);
    else if (nv <= 8) route_kernel<8><<<blocks, warps * 32, 0, st>>>(T, E, k, logits, idx, w);
    else if (nv <= 16) route_kernel<16><<<blocks, warps * 32, 0, st>>>(T, E, k, logits, idx, w);
    else route_kernel<32><<<blocks, warps * 32, 0, st>>>(T, E, k, logits, idx, w);
    return cudaGetLastError();
}

}  // namespace coli
