// Batch-union kernels (device body in moe_device.cuh) and the fused
// preparation kernel for small batches: routing, batch-union, the inverse
// pair map and the activation permutation in a single launch.
//
// Large batches (T*k >= kUnionSplitPairs) split the union over C CTAs of a
// contiguous pair range each, in two launches: every CTA counts its pairs
// per expert (per-warp histograms, one leader per distinct expert in a
// 32-pair slice); then every CTA reads all CTAs' counts, scans them
// (expert-major, then CTA, then warp) and writes its pairs at
// base + rank-among-equal-keys.  The lists are those of the one-CTA union:
// inside an expert, pairs ascend.
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
        int* batch_cnt = reinterpret_cast<int*>(reinterpret_cast<char*>(p.status) + kBatchCntOffset);
        if (threadIdx.x < 2) batch_cnt[threadIdx.x] = 0;  // the small-batch kernels' tile counters
        for (int i = threadIdx.x; i < p.E + p.n_shared; i += blockDim.x) slot_cnt[i] = 0;
        for (int i = threadIdx.x; i < p.H / 32; i += blockDim.x) tile_cnt[i] = 0;
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
        for (int t = warp; t < p.T; t += kUnionWarps) {
            const float* row = p.logits + (int64_t)t * p.E;
            if (route_fast_ok<NV>(p.k)) {
                float v[8];
                load_row8<NV>(row, p.E, lane, v);
                route_row_fast<NV>(v, p.E, p.k, lane, p.idx + (int64_t)t * p.k, p.w + (int64_t)t * p.k);
            } else {
                route_row<NV>(row, p.E, p.k, lane, p.idx + (int64_t)t * p.k, p.w + (int64_t)t * p.k);
            }
        }
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

// Per-warp histograms of pairs [lo, hi) of this warp (hist[warp][E], zeroed
// by the caller); invalid indices count nowhere and, with `status`, are
// reported.
__device__ __forceinline__ void warp_hist(int lo, int hi, int E, const int* __restrict__ idx,
                                          int* my_hist, int* status) {
    const int lane = threadIdx.x & 31;
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int p0 = lo; p0 < hi; p0 += 32) {
        const int p = p0 + lane;
        int e = p < hi ? idx[p] : -1;
        if (p < hi && (e < 0 || e >= E)) {
            if (status) report(status, COLI_ERR_BAD_INDEX);
            e = -1;
        }
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        if (e >= 0 && (peers & lt_mask) == 0) my_hist[e] += __popc(peers);
        __syncwarp();
    }
}

// Split union, launch 1: cta_cnt[c][e] = pairs of CTA c's range routed to e.
__global__ void __launch_bounds__(kUnionThreads)
union_count_kernel(int P, int E, int chunk, const int* __restrict__ idx, int* __restrict__ cta_cnt,
                   int* status) {
    extern __shared__ int hist[];
    const int warp = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < kUnionWarps * E; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    const int wchunk = chunk / kUnionWarps;
    const int lo = blockIdx.x * chunk + warp * wchunk;
    warp_hist(lo, min(P, lo + wchunk), E, idx, hist + warp * E, status);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int n = 0;
        for (int w = 0; w < kUnionWarps; ++w) n += hist[w * E + e];
        cta_cnt[(int64_t)blockIdx.x * E + e] = n;
    }
}

// Split union, launch 2: every CTA scans all CTAs' counts and writes its
// pairs; CTA 0 also writes counts, offsets, active and n_active.
__global__ void __launch_bounds__(kUnionThreads)
union_write_kernel(int P, int E, int chunk, int n_cta, const int* __restrict__ idx,
                   const int* __restrict__ cta_cnt, int* __restrict__ counts,
                   int* __restrict__ offsets, int* __restrict__ pairs, int* __restrict__ active,
                   int* __restrict__ n_active, int* __restrict__ inv) {
    extern __shared__ int hist[];
    __shared__ int scan_tmp[32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int i = threadIdx.x; i < kUnionWarps * E; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    const int wchunk = chunk / kUnionWarps;
    const int lo = blockIdx.x * chunk + warp * wchunk;
    const int hi = min(P, lo + wchunk);
    int* my_hist = hist + warp * E;
    warp_hist(lo, hi, E, idx, my_hist, nullptr);
    __syncthreads();

    const int e_self = threadIdx.x;  // E <= kUnionThreads
    int total = 0, before = 0;
    if (e_self < E) {
        for (int c = 0; c < n_cta; ++c) {
            const int n = cta_cnt[(int64_t)c * E + e_self];
            total += n;
            before += c < (int)blockIdx.x ? n : 0;
        }
    }
    int all;
    const int off = block_exclusive_scan(e_self < E ? total : 0, scan_tmp, &all);
    int act_total;
    const int act_pos =
        block_exclusive_scan((e_self < E && total > 0) ? 1 : 0, scan_tmp, &act_total);
    if (e_self < E) {
        int run = off + before;  // this CTA's first position of expert e_self
        for (int w = 0; w < kUnionWarps; ++w) {
            const int n = hist[w * E + e_self];
            hist[w * E + e_self] = run;
            run += n;
        }
        if (blockIdx.x == 0) {
            counts[e_self] = total;
            offsets[e_self] = off;
            if (total > 0) active[act_pos] = e_self;
        }
    }
    if (blockIdx.x == 0) {
        if (threadIdx.x == 0) {
            offsets[E] = all;
            *n_active = act_total;
        }
        for (int e = act_total + threadIdx.x; e < E; e += blockDim.x) active[e] = -1;
    }
    __syncthreads();

    for (int p0 = lo; p0 < hi; p0 += 32) {
        const int p = p0 + lane;
        int e = p < hi ? idx[p] : -1;
        if (e >= E) e = -1;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        if (e >= 0) {
            const int pos = my_hist[e] + __popc(peers & lt_mask);
            pairs[pos] = p;
            if (inv) inv[p] = pos;
        } else if (p < hi && inv) {
            inv[p] = -1;
        }
        __syncwarp();
        if (e >= 0 && (peers & lt_mask) == 0) my_hist[e] += __popc(peers);
        __syncwarp();
    }
}

}  // namespace

cudaError_t launch_union(int T, int E, int k, const int* idx, int* counts, int* offsets,
                         int* pairs, int* active, int* n_active, int* inv, int* status,
                         int* scratch, cudaStream_t st) {
    const int P = T * k;
    const size_t smem = union_smem_bytes(E);
    const bool split = scratch != nullptr && P >= kUnionSplitPairs && E <= kUnionThreads;
    if (smem > 48 * 1024) {
        cudaError_t err = split ? cudaFuncSetAttribute(union_count_kernel,
                                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                       (int)smem)
                                : cudaFuncSetAttribute(union_kernel,
                                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                       (int)smem);
        if (err == cudaSuccess && split)
            err = cudaFuncSetAttribute(union_write_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
    }
    if (!split) {
        union_kernel<<<1, kUnionThreads, smem, st>>>(P, E, idx, counts, offsets, pairs, active,
                                                     n_active, inv, status);
        return cudaGetLastError();
    }
    const int chunk = (int)union_chunk(P), n_cta = union_ctas(P);
    union_count_kernel<<<n_cta, kUnionThreads, smem, st>>>(P, E, chunk, idx, scratch, status);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    union_write_kernel<<<n_cta, kUnionThreads, smem, st>>>(P, E, chunk, n_cta, idx, scratch,
                                                           counts, offsets, pairs, active,
                                                           n_active, inv);
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
