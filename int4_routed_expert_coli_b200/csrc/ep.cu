// Combine step of the expert-parallel layer: the routed outputs of a token
// come back from the ranks that own its experts (already multiplied by the
// gate weight there), and the token's owner sums them with its shared-expert
// output and the residual.  The pages describe the split: a local-cluster
// worker receives one layer's routed batch-union and runs the FFN
// ("yunpan.plus/t/30351-1-1", capability three, local cluster paragraph).
//
// out[t] = ((sum_{j<k} rows[t*k + j]) + shared[t]) + residual[t], summed in
// fp32 in exactly that order, four consecutive outputs per thread.
#include "coli_internal.cuh"
#include "ptx.cuh"

namespace coli {
namespace {

__global__ void __launch_bounds__(256)
combine_rows_kernel(int T, int k, int H, const float* __restrict__ rows,
                    const float* __restrict__ shared, const void* __restrict__ residual, void* out,
                    int out_bf16) {
    const int m = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
    if (m >= H) return;
    for (int t = blockIdx.y; t < T; t += gridDim.y) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < k; ++j) {
            const float4 v =
                __ldg(reinterpret_cast<const float4*>(rows + ((int64_t)t * k + j) * H + m));
            acc.x += v.x;
            acc.y += v.y;
            acc.z += v.z;
            acc.w += v.w;
        }
        const int64_t o = (int64_t)t * H + m;
        if (shared) {
            const float4 v = __ldg(reinterpret_cast<const float4*>(shared + o));
            acc.x += v.x;
            acc.y += v.y;
            acc.z += v.z;
            acc.w += v.w;
        }
        if (out_bf16) {
            if (residual) {
                const uint2 r = *reinterpret_cast<const uint2*>(
                    reinterpret_cast<const __nv_bfloat16*>(residual) + o);
                acc.x += __uint_as_float(r.x << 16);
                acc.y += __uint_as_float(r.x & 0xFFFF0000u);
                acc.z += __uint_as_float(r.y << 16);
                acc.w += __uint_as_float(r.y & 0xFFFF0000u);
            }
            const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
            const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
            uint2 w2;
            w2.x = *reinterpret_cast<const uint32_t*>(&lo);
            w2.y = *reinterpret_cast<const uint32_t*>(&hi);
            *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(out) + o) = w2;
        } else {
            if (residual) {
                const float4 r = *reinterpret_cast<const float4*>(
                    reinterpret_cast<const float*>(residual) + o);
                acc.x += r.x;
                acc.y += r.y;
                acc.z += r.z;
                acc.w += r.w;
            }
            *reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + o) = acc;
        }
    }
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace
}  // namespace coli

extern "C" coli_status coli_moe_combine_rows(int32_t T, int32_t k, int32_t H, const float* rows,
                                             const float* shared, const void* residual,
                                             void* out, coli_out_dtype out_dtype, void* stream) {
    if (T < 0 || k < 0 || H <= 0) return COLI_ERR_INVALID_ARG;
    if (out_dtype != COLI_OUT_F32 && out_dtype != COLI_OUT_BF16) return COLI_ERR_INVALID_ARG;
    if (H % 4) return COLI_ERR_SHAPE;
    if (T == 0) return COLI_OK;
    if (!out || (k > 0 && !rows)) return COLI_ERR_INVALID_ARG;
    if ((rows && !coli::aligned(rows, 16)) || (shared && !coli::aligned(shared, 16)) ||
        !coli::aligned(out, 16) || (residual && !coli::aligned(residual, 16)))
        return COLI_ERR_ALIGN;
    const dim3 grid((unsigned)((H / 4 + 255) / 256), (unsigned)(T < 65535 ? T : 65535));
    coli::combine_rows_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        T, k, H, rows, shared, residual, out, out_dtype == COLI_OUT_BF16);
    return cudaGetLastError() == cudaSuccess ? COLI_OK : COLI_ERR_CUDA;
}
