// Batch-union: per-expert lists of (token, slot) pairs.
//
// Positions that route to the same expert are grouped so the expert is read
// once for all of them ("yunpan.plus/t/30351-1-1", capability two,
// batch-union bullet).  This is a stable counting sort of the T*k pairs by
// expert id in one CTA: per-warp histograms (one leader per distinct expert
// in each 32-pair slice, found with __match_any_sync), a scan over
// (expert, warp), and a second pass that writes every pair at
// base + rank-among-equal-keys.  No position comes from an atomic ticket,
// so the lists are identical on every run.
#include "coli_internal.cuh"

namespace coli {
namespace {

constexpr int kUnionThreads = 1024;
constexpr int kUnionWarps = kUnionThreads / 32;

// Exclusive scan of one int per thread over the whole block (<= 1024
// threads).  `tmp` holds 32 ints.  Returns the prefix; *total gets the sum.
__device__ int block_exclusive_scan(int v, int* tmp, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) tmp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int nw = blockDim.x >> 5;
        int s = lane < nw ? tmp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int n = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += n;
        }
        tmp[lane] = s;  // inclusive warp totals
    }
    __syncthreads();
    const int base = warp > 0 ? tmp[warp - 1] : 0;
    *total = tmp[(blockDim.x >> 5) - 1];
    __syncthreads();
    return base + incl - v;
}

// hist: [kUnionWarps][E] ints in dynamic shared memory.
__global__ void __launch_bounds__(kUnionThreads)
union_kernel(int P, int E, const int* __restrict__ idx, int* __restrict__ counts,
             int* __restrict__ offsets, int* __restrict__ pairs, int* __restrict__ active,
             int* __restrict__ n_active, int* status) {
    extern __shared__ int hist[];
    __shared__ int scan_tmp[32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned lt_mask = (1u << lane) - 1u;

    for (int i = threadIdx.x; i < kUnionWarps * E; i += blockDim.x) hist[i] = 0;
    __syncthreads();

    // Warp w owns pairs [w*chunk, (w+1)*chunk), chunk a multiple of 32.
    const int chunk = ((P + kUnionWarps - 1) / kUnionWarps + 31) / 32 * 32;
    const int p_begin = warp * chunk;
    const int p_end = min(P, p_begin + chunk);
    int* my_hist = hist + warp * E;

    // Pass 1: per-warp counts.
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

    // Per expert: running prefix over warps, then a scan over experts.
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
    const int act_pos = block_exclusive_scan((e_self < E && cnt > 0) ? 1 : 0, scan_tmp,
                                             &act_total);
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

    // Pass 2: scatter in pair order.
    for (int p0 = p_begin; p0 < p_end; p0 += 32) {
        const int p = p0 + lane;
        int e = p < p_end ? idx[p] : -1;
        if (e >= E) e = -1;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        if (e >= 0) {
            const int pos = my_hist[e] + __popc(peers & lt_mask);
            pairs[pos] = p;
        }
        __syncwarp();
        if (e >= 0 && (peers & lt_mask) == 0) my_hist[e] += __popc(peers);
        __syncwarp();
    }
}

}  // namespace

cudaError_t launch_union(int T, int E, int k, const int* idx, int* counts, int* offsets,
                         int* pairs, int* active, int* n_active, int* status, cudaStream_t st) {
    const int P = T * k;
    const size_t smem = sizeof(int) * (size_t)kUnionWarps * E;
    if (smem > 48 * 1024) {  // per device; cheap host call
        cudaError_t err = cudaFuncSetAttribute(union_kernel,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)smem);
        if (err != cudaSuccess) return err;
    }
    union_kernel<<<1, kUnionThreads, smem, st>>>(P, E, idx, counts, offsets, pairs, active,
                                                 n_active, status);
    return cudaGetLastError();
}

}  // namespace coli
