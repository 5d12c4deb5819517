// Router kernels: the fp32 logits GEMV (when the caller passes the router
// weight instead of logits) and the warp-per-token top-k (device body in
// moe_device.cuh).
#include "moe_device.cuh"

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

template <int NV>
__global__ void route_kernel(int T, int E, int k, const float* __restrict__ logits,
                             int* __restrict__ idx_out, float* __restrict__ w_out) {
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    route_row<NV>(logits + (int64_t)t * E, E, k, threadIdx.x & 31, idx_out + (int64_t)t * k,
                  w_out + (int64_t)t * k);
}

}  // namespace

cudaError_t launch_router_logits(int T, int E, int H, const __nv_bfloat16* x, const float* wr,
                                 float* logits, cudaStream_t st) {
    const int64_t items = (int64_t)T * E;
    const int warps = 8;
    router_logits_kernel<<<(unsigned)((items + warps - 1) / warps), warps * 32, 0, st>>>(
        T, E, H, x, wr, logits);
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
