// Batch-union kernel (device body in moe_device.cuh) and the fused
// preparation kernel for small batches: routing, batch-union, the inverse
// pair map and the activation permutation in a single launch.
#include "moe_device.cuh"
#include "ptx.cuh"

namespace coli {
namespace {

__global__ void __launch_bounds__(kUnionThreads)
union_kernel(int P, int E, const int* __restrict__ idx, int* __restrict__ counts,
             int* __restrict__ offsets, int* __restrict__ pairs, int* __restrict__ active,
             int* __restrict__ n_active, int* __restrict__ inv, int* status) {
    extern __shared__ int hist[];
    __shared__ int scan_tmp[32];
    union_block(P, E, idx, counts, offsets, pairs, active, n_active, inv, status, hist, scan_tmp);
}

// Block 0 routes every token (one warp per token), then builds the union
// lists and the inverse map; the other blocks build the fp16 operand copy of
// x and its per-group offset sums.
// Launched as a programmatic dependent: it waits for the previous kernel on
// the stream before touching the workspace, and lets the FFN kernel start
// streaming shared-expert weights as early as possible.
template <int NV>
__global__ void __launch_bounds__(kUnionThreads)
prep_small_kernel(PrepArgs p) {
    extern __shared__ int hist[];
    __shared__ int scan_tmp[32];
    pdl_wait();
    pdl_launch_dependents();
    if (blockIdx.x == 0) {
        // per-call counters of the fused decode kernel start at zero
        int* slot_cnt = reinterpret_cast<int*>(reinterpret_cast<char*>(p.status) + kSlotCntOffset);
        int* tile_cnt = reinterpret_cast<int*>(reinterpret_cast<char*>(p.status) + kTileCntOffset);
        for (int i = threadIdx.x; i < p.E + p.n_shared; i += blockDim.x) slot_cnt[i] = 0;
        for (int i = threadIdx.x; i < p.H / 32; i += blockDim.x) tile_cnt[i] = 0;
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
        for (int t = warp; t < p.T; t += kUnionWarps)
            route_row<NV>(p.logits + (int64_t)t * p.E, p.E, p.k, lane, p.idx + (int64_t)t * p.k,
                          p.w + (int64_t)t * p.k);
        __syncthreads();
        union_block(p.T * p.k, p.E, p.idx, p.counts, p.offsets, p.pairs, p.active, p.n_active,
                    p.inv, p.status, hist, scan_tmp);
    } else {
        const int64_t n_groups = (int64_t)p.T * p.H / kGroup;
        for (int64_t g = (int64_t)(blockIdx.x - 1) * blockDim.x + threadIdx.x; g < n_groups;
             g += (int64_t)(gridDim.x - 1) * blockDim.x)
            p.corr[g] = prepare_group64(reinterpret_cast<const uint16_t*>(p.x) + g * kGroup,
                                        p.xp + g * kGroup, p.status);
    }
}

}  // namespace

cudaError_t launch_union(int T, int E, int k, const int* idx, int* counts, int* offsets,
                         int* pairs, int* active, int* n_active, int* inv, int* status,
                         cudaStream_t st) {
    const int P = T * k;
    const size_t smem = union_smem_bytes(E);
    if (smem > 48 * 1024) {
        cudaError_t err = cudaFuncSetAttribute(union_kernel,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)smem);
        if (err != cudaSuccess) return err;
    }
    union_kernel<<<1, kUnionThreads, smem, st>>>(P, E, idx, counts, offsets, pairs, active,
                                                 n_active, inv, status);
    return cudaGetLastError();
}

template <int NV>
static cudaError_t launch_prep_nv(const PrepArgs& p, cudaStream_t st) {
    const size_t smem = union_smem_bytes(p.E);
    cudaError_t err = cudaSuccess;
    if (smem > 48 * 1024)
        err = cudaFuncSetAttribute(prep_small_kernel<NV>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    const int64_t n_groups = (int64_t)p.T * p.H / kGroup;
    const int perm_blocks = (int)std::min<int64_t>(64, (n_groups + 255) / 256);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1 + perm_blocks);
    cfg.blockDim = dim3(kUnionThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, prep_small_kernel<NV>, p);
}

cudaError_t launch_prep_small(const PrepArgs& p, cudaStream_t st) {
    const int nv = (p.E + 31) / 32;
    if (nv <= 1) return launch_prep_nv<1>(p, st);
    if (nv <= 2) return launch_prep_nv<2>(p, st);
    if (nv <= 4) return launch_prep_nv<4>(p, st);
    if (nv <= 8) return launch_prep_nv<8>(p, st);
    if (nv <= 16) return launch_prep_nv<16>(p, st);
    return launch_prep_nv<32>(p, st);
}

}  // namespace coli
