// Router-lookahead prefetch into L2: while one layer runs, the weights of
// the experts the next layer is predicted to need are fetched from HBM into
// L2, so that layer's first tiles start from L2.  This is the on-GPU
// analogue of the pages' one-layer-ahead prefetch ("yunpan.plus/t/30351-1-1",
// capabilities one and two: PILOT=1 predicts the next layer's experts and
// prefetches them; the memory-tier section gives the next layer's routing as
// 71.6 % predictable), with HBM -> L2 in place of disk -> RAM.  The
// prediction is a routing the caller passes in, e.g. the previous step's
// routing of the next layer.
//
// One CTA: it marks the experts the routing names, then walks them in the
// order the layer's kernels take them (shared experts first, then routed
// experts by ascending index) and issues bulk L2 prefetches of each one's
// codes and scales until the byte budget is spent.  No shared-memory tiles
// and few registers, so it can run beside a persistent layer kernel.
#include "coli_internal.cuh"
#include "handle.cuh"
#include "ptx.cuh"

namespace coli {
namespace {

constexpr int kPfThreads = 256;
constexpr uint32_t kChunk = 64 * 1024;  // bytes per prefetch instruction

__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Prefetch `bytes` (a multiple of 16) at p, chunks spread over the CTA.
__device__ void prefetch_range(const void* p, uint64_t bytes) {
    const uint8_t* b = static_cast<const uint8_t*>(p);
    for (uint64_t off = (uint64_t)threadIdx.x * kChunk; off < bytes;
         off += (uint64_t)kPfThreads * kChunk) {
        const uint64_t n = bytes - off < kChunk ? bytes - off : kChunk;
        prefetch_l2(b + off, (uint32_t)n);
    }
}

__global__ void __launch_bounds__(kPfThreads)
prefetch_kernel(const DevExpert* __restrict__ experts, int E, int n_shared, int H, int I,
                int per_row, int T, int k, const int* __restrict__ idx, uint64_t max_bytes,
                int* status) {
    __shared__ uint32_t used[kMaxExperts / 32];
    for (int i = threadIdx.x; i < kMaxExperts / 32; i += kPfThreads) used[i] = 0u;
    __syncthreads();
    for (int p = threadIdx.x; p < T * k; p += kPfThreads) {
        const int e = idx[p];
        if (e >= 0 && e < E) atomicOr(&used[e >> 5], 1u << (e & 31));
        else report(status, COLI_ERR_BAD_INDEX);
    }
    __syncthreads();
    const uint64_t codes = (uint64_t)H * I / 2;              // bytes of one code matrix
    const uint64_t gsc = (uint64_t)I * scale_cols(H, per_row) * 2;  // gate (up) scales
    const uint64_t dsc = (uint64_t)H * scale_cols(I, per_row) * 2;  // down scales
    const uint64_t per_expert = 3 * codes + 2 * gsc + dsc;
    uint64_t spent = 0;
    for (int i = 0; i < n_shared + E; ++i) {
        const int e = i < n_shared ? E + i : i - n_shared;
        if (e < E && !((used[e >> 5] >> (e & 31)) & 1u)) continue;
        if (spent + per_expert > max_bytes) break;
        spent += per_expert;
        const DevExpert ex = experts[e];
        prefetch_range(ex.gate_q, codes);
        prefetch_range(ex.up_q, codes);
        prefetch_range(ex.down_q, codes);
        prefetch_range(ex.gate_s, gsc);
        prefetch_range(ex.up_s, gsc);
        prefetch_range(ex.down_s, dsc);
    }
}

}  // namespace
}  // namespace coli

extern "C" coli_status coli_moe_prefetch(const coli_moe* h, int32_t T, int32_t k,
                                         const int32_t* topk_idx, size_t max_bytes, void* ws,
                                         size_t ws_bytes, void* stream) {
    if (!h || T < 0 || k < 1 || k > h->E) return COLI_ERR_INVALID_ARG;
    if ((int64_t)T * k > (int64_t)1 << 24) return COLI_ERR_SHAPE;
    if (T > 0 && !topk_idx) return COLI_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(topk_idx) & 3) return COLI_ERR_ALIGN;
    if (ws && (ws_bytes < coli::kHeaderBytes || (reinterpret_cast<uintptr_t>(ws) & 255)))
        return COLI_ERR_WORKSPACE;
    coli::prefetch_kernel<<<1, coli::kPfThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        h->d_experts, h->E, h->n_shared, h->H, h->I, h->per_row, T, k, topk_idx,
        (uint64_t)max_bytes, static_cast<int*>(ws));
    return cudaGetLastError() == cudaSuccess ? COLI_OK : COLI_ERR_CUDA;
}
