// Expert FFN for prefill-sized batches: a grouped GEMM per expert on the
// fifth-generation tensor cores (tcgen05, accumulators in tensor memory),
// used when the tokens routed to an expert make its FFN a dense contraction.
//
// Shapes.  For expert e with a token list of n_e rows (the batch-union lists,
// "yunpan.plus/t/30351-1-1", capability two), gate/up is
//   [2 x I rows of int4 codes] x [n_e tokens x H]  -> h [n_e][I]
// and down is [H rows] x [n_e x I] -> y [n_e][H].  The weight rows are the MMA
// M dimension (128 per MMA; a tile runs two MMAs on the same activation tile:
// gate and up of 128 features, or two 128-row blocks of W_d, so each
// activation tile is loaded from L2 once per 256 weight rows), the tokens the
// N dimension (tiles of up to 192,
// rounded to 16, so a routed expert of a 4096-token prefill is one tile and
// its weights are dequantised once per M tile), K is walked in 64-element
// blocks (one gs64 scale group).
//
// Pipeline (one CTA per SM, persistent over a flattened list of tiles):
//   warp 0      TMA producer: packed int4 codes of the tile rows (a 2-D tensor
//               map per expert matrix, 32 bytes x 128 rows per K-block) and the
//               activation rows the tile has (128-byte swizzled fp16, at most
//               two boxes of 128/64/32 rows);
//   warps 4-7   dequant: each thread owns one weight row of each block,
//               turns its 64 codes into fp16 q * s (exact: a 3-bit code
//               magnitude times an 8-bit bf16 scale fits fp16's 11 bits) and
//               stores them straight into tensor memory (tcgen05.st, lane =
//               weight row, two fp16 per column): the weight operand never
//               passes through shared memory;
//   warp 1      one thread issues tcgen05.mma (kind::f16, A from tensor
//               memory, B from shared memory, fp32 accumulate in tensor
//               memory) and commits stage / operand release and tile
//               completion;
//   warps 8-15  epilogue: tcgen05.ld of the accumulator (a warp reads the 32
//               lanes of its quarter, the two warps of a quarter alternate
//               32-token chunks), SwiGLU to fp16 h, or the fp32 y rows of the
//               down GEMM.
//   Tensor memory (512 columns): one accumulator of two 192-column blocks in
//   [0, 384), drained by the epilogue before the next tile's MMAs, and a ring
//   of weight operands in [384, 512) (2 K-blocks of 2 x 32 columns).
// Every wait is bounded (COLI_ERR_TIMEOUT) so nothing can hang the GPU.
//
// K order.  Within each group of 8 consecutive K elements the dequant unpack
// yields codes in the order 0,4,1,5,2,6,3,7; the activation operands (the
// gathered x and the h written by the gate/up epilogue) are stored in that
// same order, so every dot product is unchanged.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>
#include <new>

#include "moe_device.cuh"
#include "decode.cuh"
#include "prefill.cuh"
#include "ptx.cuh"

namespace coli {
namespace {

constexpr int BM = 128, BK = 64;
constexpr int kBRowQuant = 32;      // activation rows are loaded in multiples of 32
constexpr uint32_t kTmemColsP = 512;
constexpr int kHeaderP = 2048;
constexpr int kSmemLimitP = 227 * 1024;

// Two shapes of the same pipeline, both with 8 dequantising warps (two per
// lane quarter, one weight row of one block per thread).  Large token tiles
// (prefill: ~128 tokens per expert): 192-token tiles, one accumulator, a
// 2-deep operand ring and 8 epilogue warps (20 warps in all).  Small token
// tiles (a few tokens per expert, every call with T <= 64): 64-token tiles,
// a double-buffered accumulator, a 4-deep operand ring and 4 epilogue warps
// (16 warps).
template <bool kSmall>
struct Cfg {
    static constexpr int BN = kSmall ? 64 : 192;            // tokens per tile (max)
    static constexpr int kAccBufs = kSmall ? 2 : 1;
    static constexpr uint32_t kAccCols = 2 * BN * kAccBufs;  // accumulators, then the ring
    static constexpr int kACols = BK;                        // operand columns per K-block (2 blocks)
    static constexpr int kAStages = (int)(kTmemColsP - kAccCols) / kACols;
    static constexpr int kDqWarp0 = 4;                       // warps 4-11: two per lane
    static constexpr int kDqWarps = 8;                       // quarter, one block each
    static constexpr int kEpiWarp0 = 12;
    static constexpr int kEpiWarps = kSmall ? 4 : 8;
    static constexpr int kThreads = (kEpiWarp0 + kEpiWarps) * 32;  // 512 or 640
    static constexpr int kBBytes = BN * BK * 2;               // activation tile per stage
    static constexpr int kStage = kBBytes + 2 * BM * BK / 2;  // + two blocks of packed codes
};
static_assert(Cfg<false>::kAStages == 2 && Cfg<true>::kAStages == 4, "operand ring depth");

// Position of element k (0..7) of an 8-group in the operand order.
__host__ __device__ __forceinline__ int perm8(int k) { return (k & 3) * 2 + (k >> 2); }
__host__ __device__ __forceinline__ int perm_col(int n) { return (n & ~7) + perm8(n & 7); }

// ---- tcgen05 / TMA wrappers ------------------------------------------------
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);  // start address
    d |= (uint64_t)1 << 16;                    // leading byte offset (unused for SW128 K-major)
    d |= (uint64_t)(1024 >> 4) << 32;          // stride byte offset: 8 rows x 128 B
    d |= (uint64_t)1 << 46;                    // descriptor version for sm_100
    d |= (uint64_t)2 << 61;                    // 128-byte swizzle
    return d;
}

__device__ __forceinline__ uint32_t idesc_f16(int n) {
    return (1u << 4)                          // D: f32
           | ((uint32_t)(n >> 3) << 17)       // N
           | ((uint32_t)(BM >> 4) << 24);     // M = 128; A, B: f16, K-major
}

// The four K=16 MMAs of one 64-wide K-block: A columns a, a + 8, a + 16,
// a + 24; the B descriptor advanced by 32 bytes (two 16-byte units) each.
// The first accumulates into d unless `accumulate` is 0, the others always.
__device__ __forceinline__ void mma_kblock_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b,
                                              uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, t;\n\t.reg .b64 b1, b2, b3;\n\t.reg .b32 a1, a2, a3;\n\t"
        "setp.ne.u32 p, %4, 0;\n\tsetp.ne.u32 t, %5, 0;\n\t"
        "add.s64 b1, %2, 2;\n\tadd.s64 b2, %2, 4;\n\tadd.s64 b3, %2, 6;\n\t"
        "add.u32 a1, %1, 8;\n\tadd.u32 a2, %1, 16;\n\tadd.u32 a3, %1, 24;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], b1, %3, t;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [a2], b2, %3, t;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [a3], b3, %3, t;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b), "r"(idesc), "r"(accumulate), "r"(1u));
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t v[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
        "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
          "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]),
          "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]),
          "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 32 consecutive columns of this warp's 32 lanes <- v (lane i writes its own row).
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t v[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
        "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
        "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
        "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, int c0, int c1,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_addr(dst)),
        "l"(tmap), "r"(c0), "r"(c1), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void tma_load_2d_hint(void* dst, const void* tmap, int c0, int c1,
                                                 uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
        "[%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_addr(dst)),
        "l"(tmap), "r"(c0), "r"(c1), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

// Position in a ring of barriers: slot index and how many times it wrapped
// (the parity of the phase to wait for), advanced without a division.
struct Ring {
    int i = 0, pass = 0;
    __device__ __forceinline__ void next(int n) {
        if (++i == n) {
            i = 0;
            ++pass;
        }
    }
};

// ---- tile bookkeeping --------------------------------------------------------
struct TileInfo {
    int e;          // expert row in the table
    int out_row0;   // first output row (hp / y) of this tile's tokens
    int b_row0;     // first activation row of this tile's tokens
    int ntok;       // valid tokens in the tile (<= BN)
    int n_mma;      // MMA N (ntok rounded up to 16)
    int m_tile;
    bool valid;
};

template <int BN>
__device__ __forceinline__ TileInfo tile_info(const GemmArgs& a, bool gu, int64_t tile,
                                              int n_slots, int m_tiles) {
    TileInfo ti;
    // slot with ntile_start[slot] * m_tiles <= tile < ntile_start[slot + 1] * m_tiles
    int lo = 0, hi = n_slots;  // invariant: start(lo) <= tile < start(hi)
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if ((int64_t)__ldg(a.ntile_start + mid) * m_tiles <= tile) lo = mid;
        else hi = mid;
    }
    const int slot = lo;
    const int s0 = __ldg(a.ntile_start + slot), s1 = __ldg(a.ntile_start + slot + 1);
    const int nt = s1 - s0;
    const int64_t local = tile - (int64_t)s0 * m_tiles;
    ti.m_tile = (int)(local / nt);
    const int n_tile = (int)(local % nt);
    const int P = a.T * a.k;
    int list_begin, ntok_total;
    ti.valid = true;
    if (slot < a.n_shared) {
        ti.e = a.E + slot;
        list_begin = P + slot * a.T;
        ntok_total = a.T;
        ti.b_row0 = (gu ? P : list_begin) + n_tile * BN;
    } else {
        const int e = a.active[slot - a.n_shared];
        const int b = (e >= 0 && e < a.E) ? a.offsets[e] : 0;
        const int en = (e >= 0 && e < a.E) ? a.offsets[e + 1] : 0;
        ti.valid = e >= 0 && e < a.E && b >= 0 && en >= b && en <= P;
        ti.e = ti.valid ? e : 0;
        list_begin = ti.valid ? b : 0;
        ntok_total = ti.valid ? en - b : 0;
        ti.b_row0 = list_begin + n_tile * BN;
    }
    ti.out_row0 = list_begin + n_tile * BN;
    ti.ntok = min(BN, max(0, ntok_total - n_tile * BN));
    ti.n_mma = max(16, (ti.ntok + 15) & ~15);
    return ti;
}

// ---- the GEMM kernel -------------------------------------------------------
// Two MMAs per K step on one activation tile: kGU gate/up (the gate rows and
// the up rows of the same 128 features, K = H), otherwise down (two blocks of
// 128 rows of W_d, 256 output features, K = I).
template <bool kGU, bool kSmall>
__global__ void __launch_bounds__(Cfg<kSmall>::kThreads, 1)
prefill_gemm_kernel(const __grid_constant__ CUtensorMap bmap128,
                    const __grid_constant__ CUtensorMap bmap64,
                    const __grid_constant__ CUtensorMap bmap32, const GemmArgs a, int stages) {
    using C = Cfg<kSmall>;
    constexpr int BN = C::BN;
    constexpr int NA = 2;                                    // weight blocks per tile
    constexpr int kFeat = kGU ? BM : 2 * BM;                 // output features per tile
    constexpr int kPkBytes = BM * BK / 2;                    // 4 KB per block
    constexpr int kAStages = C::kAStages;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);        // TMA landed
    uint64_t* dq_full = full + 16;                             // operand written to TMEM
    uint64_t* empty = full + 32;                               // MMAs done reading the stage
    uint64_t* acc_full = full + 48;                            // [2] accumulator ready
    uint64_t* acc_empty = full + 50;                           // [2] accumulator drained
    uint64_t* a_empty = full + 52;                             // [kAStages] MMAs done with an operand
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + 512);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + 520);
    uint8_t* stage0 = smem + kHeaderP;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < kAStages; ++s) {
            mbar_init(&dq_full[s], C::kDqWarps);
            mbar_init(&a_empty[s], 1);
        }
        for (int b = 0; b < C::kAccBufs; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], C::kEpiWarps);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 2) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_addr((const void*)tmem_slot)),
                     "r"(kTmemColsP)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_launch_dependents();
    pdl_wait();

    int n_act = *reinterpret_cast<const volatile int*>(a.n_active);
    if (n_act < 0 || n_act > a.E) {
        if (threadIdx.x == 0) report(a.status, COLI_ERR_BAD_INDEX);
        n_act = 0;
    }
    const int n_slots = n_act + a.n_shared;
    const int m_tiles = kGU ? a.I / BM : (a.H + kFeat - 1) / kFeat;
    const int K = kGU ? a.H : a.I;
    const int KB = K / BK;
    const int G = K / kGroup;
    const int64_t n_tiles = (int64_t)__ldg(a.ntile_start + n_slots) * m_tiles;

    auto stage_ptr = [&](int s) { return stage0 + (size_t)s * C::kStage; };
    auto timeout = [&]() {
        report(a.status, COLI_ERR_TIMEOUT);
        *abort_flag = 1;
    };

    if (warp == 0) {
        // ------------------------------ producer ------------------------------
        if (lane == 0) {
            const uint64_t policy = policy_evict_first();
            Ring rs;
            for (int64_t tile = blockIdx.x; tile < n_tiles && !*abort_flag; tile += gridDim.x) {
                const TileInfo ti = tile_info<BN>(a, kGU, tile, n_slots, m_tiles);
                const CUtensorMap* wm = a.wmaps + (size_t)ti.e * 3;
                const int f0 = ti.m_tile * kFeat;
                // only the token rows the tile has, rounded up to 32, in at
                // most two boxes (128 + 64 / 128 + 32 / 64 + 32 / one)
                const int brows = (max(ti.ntok, 1) + kBRowQuant - 1) / kBRowQuant * kBRowQuant;
                for (int kb = 0; kb < KB; ++kb) {
                    const int s = rs.i;
                    if (rs.pass > 0 && !mbar_wait(&empty[s], (uint32_t)(rs.pass - 1) & 1)) {
                        timeout();
                        break;
                    }
                    rs.next(stages);
                    uint8_t* st = stage_ptr(s);
                    mbar_arrive_expect_tx(&full[s], NA * kPkBytes + brows * BK * 2);
                    uint8_t* pk = st + C::kBBytes;
                    if constexpr (kGU) {
                        tma_load_2d_hint(pk, wm + 0, kb * (BK / 2), f0, &full[s], policy);
                        tma_load_2d_hint(pk + kPkBytes, wm + 1, kb * (BK / 2), f0, &full[s],
                                         policy);
                    } else {
                        // the second block may lie past H (zero-filled codes)
                        tma_load_2d_hint(pk, wm + 2, kb * (BK / 2), f0, &full[s], policy);
                        tma_load_2d_hint(pk + kPkBytes, wm + 2, kb * (BK / 2), f0 + BM, &full[s],
                                         policy);
                    }
                    int r0 = 0;
                    if (brows - r0 >= 128) {
                        tma_load_2d(st, &bmap128, kb * BK, ti.b_row0, &full[s]);
                        r0 += 128;
                    }
                    if (brows - r0 >= 64) {
                        tma_load_2d(st + r0 * (BK * 2), &bmap64, kb * BK, ti.b_row0 + r0, &full[s]);
                        r0 += 64;
                    }
                    if (brows - r0 >= 32)
                        tma_load_2d(st + r0 * (BK * 2), &bmap32, kb * BK, ti.b_row0 + r0, &full[s]);
                }
            }
        }
    } else if (warp == 1) {
        // -------------------------------- MMA --------------------------------
        if (lane == 0) {
            Ring rs, ra;
            int64_t lt = 0;
            for (int64_t tile = blockIdx.x; tile < n_tiles && !*abort_flag;
                 tile += gridDim.x, ++lt) {
                const TileInfo ti = tile_info<BN>(a, kGU, tile, n_slots, m_tiles);
                // accumulator buffer lt % kAccBufs: wait for the epilogue of
                // the tile that used it before
                const int buf = (int)(lt % C::kAccBufs);
                const int64_t use = lt / C::kAccBufs;
                if (use > 0 && !mbar_wait(&acc_empty[buf], (uint32_t)(use - 1) & 1)) {
                    timeout();
                    break;
                }
                tc_fence_after();
                const uint32_t idesc = idesc_f16(ti.n_mma);
                const uint32_t d0 = tmem_base + (uint32_t)(buf * NA * BN);
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb) {
                    const int s = rs.i, as = ra.i;
                    if (!mbar_wait(&dq_full[as], (uint32_t)ra.pass & 1)) {
                        timeout();
                        ok = false;
                        break;
                    }
                    rs.next(stages);
                    ra.next(kAStages);
                    tc_fence_after();
                    const uint64_t bdesc = desc_sw128(smem_addr(stage_ptr(s)));
                    const uint32_t a0 = tmem_base + C::kAccCols + (uint32_t)(as * C::kACols);
#pragma unroll
                    for (int m = 0; m < NA; ++m)
                        mma_kblock_ts(d0 + m * BN, a0 + m * (BK / 2), bdesc, idesc, kb != 0);
                    mma_commit(&empty[s]);
                    mma_commit(&a_empty[as]);
                }
                if (!ok) break;
                mma_commit(&acc_full[buf]);
            }
        }
    } else if (warp >= C::kDqWarp0 && warp < C::kDqWarp0 + C::kDqWarps) {
        // ------------------------------- dequant -------------------------------
        // large tiles: one weight row of both blocks per thread; small tiles:
        // two warps per lane quarter, each one block
        const int q = warp & 3;
        const int row = q * 32 + lane;  // MMA row of the tile owned by this thread
        constexpr int kMyBlocks = 1;
        const int blk0 = (warp - C::kDqWarp0) >> 2;
        // this warp's 32 lanes of the operand ring
        const uint32_t ta = tmem_base + ((uint32_t)q << 21) + C::kAccCols;
        Ring rs, ra;
        for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
            const TileInfo ti = tile_info<BN>(a, kGU, tile, n_slots, m_tiles);
            const DevExpert ex = a.experts[ti.e];
            // gate/up: gate and up row of feature f0 + row; down: W_d rows
            // f0 + row and f0 + 128 + row (the latter past H in a ragged last
            // tile: scale 0, and its codes are zero-filled)
            const int f0 = ti.m_tile * kFeat;
            const int SG = scale_cols(K, a.per_row);  // scale columns per row
            const int gstep = a.per_row ? 0 : 1;      // scale column step per K-block
            const int64_t srow = (int64_t)(f0 + row) * SG;
            const bool has1 = kGU || f0 + BM < a.H;
            const uint16_t* sc_b0 = (kGU ? ex.gate_s : ex.down_s) + srow;
            const uint16_t* sc_b1 = kGU ? ex.up_s + srow : ex.down_s + srow + (int64_t)BM * SG;
            // Scales: a row's scales are contiguous, so where a row of them
            // is a whole number of 16-byte chunks (G % 8 == 0) a thread
            // loads 8 at a time, one chunk (8 K-blocks) ahead, and the load
            // latency hides behind 8 K-blocks of work; otherwise one scale
            // per K-block, one ahead; in the per-row format the row's one
            // scale, loaded once.
            const bool vec = !a.per_row && (G & 7) == 0;
            const uint16_t* scp[kMyBlocks];
            bool live[kMyBlocks];
            uint4 chunk[kMyBlocks], chunk_nxt[kMyBlocks];
            uint16_t nxt[kMyBlocks];
#pragma unroll
            for (int m = 0; m < kMyBlocks; ++m) {
                const int blk = blk0 + m;
                scp[m] = blk == 0 ? sc_b0 : sc_b1;
                live[m] = blk == 0 || has1;
                const uint4 z = make_uint4(0u, 0u, 0u, 0u);
                chunk[m] = z;
                chunk_nxt[m] = (vec && live[m]) ? __ldg(reinterpret_cast<const uint4*>(scp[m])) : z;
                nxt[m] = (!vec && live[m]) ? __ldg(scp[m]) : 0;
            }
            bool ok = true;
            for (int kb = 0; kb < KB; ++kb) {
                uint16_t cur[kMyBlocks];
                const int sub = kb & 7;
#pragma unroll
                for (int m = 0; m < kMyBlocks; ++m) {
                    if (vec) {
                        if (sub == 0) {
                            chunk[m] = chunk_nxt[m];
                            if (kb + 8 < KB && live[m])
                                chunk_nxt[m] =
                                    __ldg(reinterpret_cast<const uint4*>(scp[m] + kb + 8));
                        }
                        const uint32_t w2 = sub < 4 ? (sub < 2 ? chunk[m].x : chunk[m].y)
                                                    : (sub < 6 ? chunk[m].z : chunk[m].w);
                        cur[m] = (uint16_t)((sub & 1) ? (w2 >> 16) : (w2 & 0xFFFFu));
                    } else {
                        cur[m] = nxt[m];
                        if (kb + 1 < KB && live[m] && gstep) nxt[m] = __ldg(scp[m] + kb + 1);
                    }
                }
                const int s = rs.i, as = ra.i;
                if (!mbar_wait(&full[s], (uint32_t)rs.pass & 1) ||
                    (ra.pass > 0 && !mbar_wait(&a_empty[as], (uint32_t)(ra.pass - 1) & 1))) {
                    if (lane == 0) timeout();
                    ok = false;
                    break;
                }
                rs.next(stages);
                ra.next(kAStages);
                tc_fence_after();
#pragma unroll
                for (int m = 0; m < kMyBlocks; ++m) {
                    const int blk = blk0 + m;
                    const uint4* pk = reinterpret_cast<const uint4*>(stage_ptr(s) + C::kBBytes +
                                                                     blk * kPkBytes + row * 32);
                    const uint4 p0 = pk[0], p1 = pk[1];
                    const uint32_t words[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
                    // bf16 scale s -> fp16 s and s / 16 (exact for scales in
                    // fp16's normal range: 8 significant bits)
                    const float sf = __uint_as_float((uint32_t)cur[m] << 16);
                    const __half2 s2 = __float2half2_rn(sf);
                    const __half2 s16 = __float2half2_rn(sf * 0.0625f);
                    const __half2 lo = __floats2half2_rn(1032.f, 1032.f);
                    const __half2 hi = __floats2half2_rn(1152.f, 1152.f);
                    uint32_t cols[32];  // column 4c + i: elements i, i + 4 of 8-group c
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint32_t w = words[c], w8 = w >> 8;
                        // even codes (1032 + q) - 1032 = q, odd codes
                        // (1152 + 16 q) - 1152 = 16 q, both exact; times s and
                        // s / 16, exact (q s has at most 11 significant bits).
                        // A single fused multiply-add with a -72 s or -1032 s
                        // addend would not be exact: those products need up to
                        // 12 and 15 significant bits.
                        uint32_t t0 = (w & 0x000F000Fu) ^ 0x64086408u;
                        uint32_t t1 = (w & 0x00F000F0u) ^ 0x64806480u;
                        uint32_t t2 = (w8 & 0x000F000Fu) ^ 0x64086408u;
                        uint32_t t3 = (w8 & 0x00F000F0u) ^ 0x64806480u;
                        __half2 v0 = __hmul2(__hsub2(*reinterpret_cast<__half2*>(&t0), lo), s2);
                        __half2 v1 = __hmul2(__hsub2(*reinterpret_cast<__half2*>(&t1), hi), s16);
                        __half2 v2 = __hmul2(__hsub2(*reinterpret_cast<__half2*>(&t2), lo), s2);
                        __half2 v3 = __hmul2(__hsub2(*reinterpret_cast<__half2*>(&t3), hi), s16);
                        cols[4 * c + 0] = *reinterpret_cast<uint32_t*>(&v0);
                        cols[4 * c + 1] = *reinterpret_cast<uint32_t*>(&v1);
                        cols[4 * c + 2] = *reinterpret_cast<uint32_t*>(&v2);
                        cols[4 * c + 3] = *reinterpret_cast<uint32_t*>(&v3);
                    }
                    tmem_st32(ta + (uint32_t)(as * C::kACols + blk * (BK / 2)), cols);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&dq_full[as]);
            }
            if (!ok) break;
        }
    } else if (warp >= C::kEpiWarp0 && warp < C::kEpiWarp0 + C::kEpiWarps) {
        // ------------------------------- epilogue ------------------------------
        const int q = warp & 3;
        // large tiles: the two warps of a quarter take alternate 32-token chunks
        const int c_first = ((warp - C::kEpiWarp0) >> 2) * 32;
        constexpr int c_step = 32 * (C::kEpiWarps / 4);
        const int row = q * 32 + lane;  // accumulator lane = MMA row of the tile
        int64_t lt = 0;
        for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++lt) {
            const TileInfo ti = tile_info<BN>(a, kGU, tile, n_slots, m_tiles);
            const int buf = (int)(lt % C::kAccBufs);
            if (!mbar_wait(&acc_full[buf], (uint32_t)(lt / C::kAccBufs) & 1)) {
                if (lane == 0) timeout();
                break;
            }
            tc_fence_after();
            const uint32_t tq = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * NA * BN);
            const int feat = ti.m_tile * kFeat + row;
            if constexpr (kGU) {
                // gate and up of this lane's feature sit in the same lane; with
                // one accumulator buffer the next tile's MMAs wait for this,
                // so SiLU uses the fast exponential and division
                const int col = perm_col(feat);
                __half* hcol = a.hbuf + (int64_t)ti.out_row0 * a.I + col;
                for (int c0 = c_first; c0 < ti.ntok; c0 += c_step) {
                    uint32_t vg[32], vu[32];
                    tmem_ld32(tq + c0, vg);
                    tmem_ld32(tq + BN + c0, vu);
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        if (c0 + j < ti.ntok) {
                            const float g = __uint_as_float(vg[j]), u = __uint_as_float(vu[j]);
                            float hv = __fdividef(g, 1.f + __expf(-g)) * u;
                            if (!(fabsf(hv) <= 65504.f)) {
                                report(a.status, COLI_ERR_RANGE);
                                hv = copysignf(65504.f, hv);
                            }
                            hcol[(int64_t)(c0 + j) * a.I] = __float2half_rn(hv);
                        }
                    }
                }
            } else {
                const bool has1 = feat + BM < a.H;
                float* yrow = a.y + (int64_t)ti.out_row0 * a.H + feat;
                for (int c0 = c_first; c0 < ti.ntok; c0 += c_step) {
                    uint32_t v0[32], v1[32];
                    tmem_ld32(tq + c0, v0);
                    tmem_ld32(tq + BN + c0, v1);
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        if (c0 + j < ti.ntok) {
                            yrow[(int64_t)(c0 + j) * a.H] = __uint_as_float(v0[j]);
                            if (has1) yrow[(int64_t)(c0 + j) * a.H + BM] = __uint_as_float(v1[j]);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[buf]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(kTmemColsP)
                     : "memory");
    }
}

// ---- gather: expert-sorted fp16 activations ----------------------------------
// xg[s] = fp16(x[pairs[s] / k]) for s < P (the union's order), xg[P + t] =
// fp16(x[t]) (the shared experts' rows), columns in operand order.  Block 0
// also lays out the tile list: ntile_start[slot] = sum over earlier slots of
// ceil(tokens / bn), bn the GEMM's token-tile width.
__global__ void __launch_bounds__(1024) gather_kernel(GatherArgs g) {
    pdl_wait();
    pdl_launch_dependents();
    const int P = g.T * g.k;
    if (blockIdx.x == 0) {
        __shared__ int scan_tmp[32];
        int n_act = *reinterpret_cast<const volatile int*>(g.n_active);
        if (n_act < 0 || n_act > g.E) n_act = 0;
        const int n_slots = n_act + g.n_shared;
        int cnt[2];
        for (int u = 0; u < 2; ++u) {
            const int slot = threadIdx.x * 2 + u;
            int ntok = 0;
            if (slot < g.n_shared) {
                ntok = g.T;
            } else if (slot < n_slots) {
                // an expert id or token list the union could not have produced
                // is reported; its slot gets no tiles
                const int e = g.active[slot - g.n_shared];
                const int b = (e >= 0 && e < g.E) ? g.offsets[e] : 0;
                const int en = (e >= 0 && e < g.E) ? g.offsets[e + 1] : -1;
                if (e >= 0 && e < g.E && b >= 0 && en >= b && en <= P) ntok = en - b;
                else report(g.status, COLI_ERR_BAD_INDEX);
            }
            cnt[u] = slot < n_slots ? (max(ntok, 0) + g.bn - 1) / g.bn : 0;
        }
        int total;
        const int base = block_exclusive_scan(cnt[0] + cnt[1], scan_tmp, &total);
        const int s0 = threadIdx.x * 2;
        if (s0 <= n_slots) g.ntile_start[s0] = base;
        if (s0 + 1 <= n_slots) g.ntile_start[s0 + 1] = base + cnt[0];
        return;
    }
    // the other blocks: four rows per pass (256 threads per row), no
    // per-element division; a row's token index is one broadcast load
    const int chunks = g.H / 8;
    const int64_t rows = P + g.T;
    const int sub = threadIdx.x >> 8, lt = threadIdx.x & 255;
    for (int64_t s0 = (int64_t)(blockIdx.x - 1) * 4; s0 < rows; s0 += (int64_t)(gridDim.x - 1) * 4) {
        const int64_t s = s0 + sub;
        if (s >= rows) continue;
        int t;
        if (s < P) {
            const int p = g.pairs[s];
            t = (p >= 0 && p < P) ? p / g.k : -1;
        } else {
            t = (int)(s - P);
        }
        for (int c = lt; c < chunks; c += 256) {
            uint4 out = make_uint4(0, 0, 0, 0);
            if (t >= 0) {
                const uint4 in = *reinterpret_cast<const uint4*>(
                    reinterpret_cast<const uint16_t*>(g.x) + (int64_t)t * g.H + c * 8);
                const uint16_t* v = reinterpret_cast<const uint16_t*>(&in);
                uint16_t o[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    float f = __uint_as_float((uint32_t)v[j] << 16);
                    if (fabsf(f) > 65504.f) {
                        report(g.status, COLI_ERR_RANGE);
                        f = copysignf(65504.f, f);
                    }
                    const __half h = __float2half_rn(f);
                    o[perm8(j)] = *reinterpret_cast<const uint16_t*>(&h);
                }
                out = *reinterpret_cast<uint4*>(o);
            }
            *reinterpret_cast<uint4*>(g.xg + s * g.H + c * 8) = out;
        }
    }
}

// ---- host --------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

bool encode_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner,
               uint64_t rows, uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows,
               CUtensorMapSwizzle sw) {
    auto enc = get_encode();
    if (!enc) return false;
    const cuuint64_t dims[2] = {inner, rows};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_rows};
    const cuuint32_t es[2] = {1, 1};
    return enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool kSmall>
int gemm_stages() {
    return std::min(16, (kSmemLimitP - kHeaderP - 1024) / Cfg<kSmall>::kStage);
}

template <bool kGU, bool kSmall>
cudaError_t launch_gemm(const CUtensorMap (&bmap)[3], const GemmArgs& a, int num_sms,
                        cudaStream_t st) {
    const int stages = gemm_stages<kSmall>();
    const int smem = kHeaderP + 1024 + stages * Cfg<kSmall>::kStage;
    cudaError_t err = cudaFuncSetAttribute(prefill_gemm_kernel<kGU, kSmall>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(num_sms);
    cfg.blockDim = dim3(Cfg<kSmall>::kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, prefill_gemm_kernel<kGU, kSmall>, bmap[0], bmap[1], bmap[2],
                              a, stages);
}

}  // namespace

cudaError_t build_weight_maps(const DevExpert* host_experts, int n, int H, int I,
                              CUtensorMap** d_maps) {
    *d_maps = nullptr;
    CUtensorMap* maps = new (std::nothrow) CUtensorMap[(size_t)n * 3];
    if (!maps) return cudaErrorMemoryAllocation;
    for (int e = 0; e < n; ++e) {
        const DevExpert& x = host_experts[e];
        const bool ok =
            encode_2d(&maps[e * 3 + 0], CU_TENSOR_MAP_DATA_TYPE_UINT8, x.gate_q, H / 2, I, H / 2,
                      BK / 2, BM, CU_TENSOR_MAP_SWIZZLE_NONE) &&
            encode_2d(&maps[e * 3 + 1], CU_TENSOR_MAP_DATA_TYPE_UINT8, x.up_q, H / 2, I, H / 2,
                      BK / 2, BM, CU_TENSOR_MAP_SWIZZLE_NONE) &&
            encode_2d(&maps[e * 3 + 2], CU_TENSOR_MAP_DATA_TYPE_UINT8, x.down_q, I / 2, H, I / 2,
                      BK / 2, BM, CU_TENSOR_MAP_SWIZZLE_NONE);
        if (!ok) {
            delete[] maps;
            return cudaErrorInvalidValue;
        }
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

cudaError_t launch_prefill(const FfnArgs& f, const CUtensorMap* wmaps, __half* xg, int* ntile_start,
                           int num_sms, cudaStream_t st) {
    const int P = f.T * f.k;
    const int S = P + f.T * f.n_shared;
    // small token tiles when every list fits one (T <= 64) or the routed
    // experts average at most 8 tokens
    const bool small = f.T <= Cfg<true>::BN || (int64_t)P <= 8 * (int64_t)f.E;
    GatherArgs g;
    g.bn = small ? Cfg<true>::BN : Cfg<false>::BN;
    g.T = f.T;
    g.k = f.k;
    g.E = f.E;
    g.H = f.H;
    g.n_shared = f.n_shared;
    g.x = f.x;
    g.pairs = f.pairs;
    g.offsets = f.offsets;
    g.active = f.active;
    g.n_active = f.n_active;
    g.xg = xg;
    g.ntile_start = ntile_start;
    g.status = f.status;
    {
        const int64_t rows = P + f.T;
        const int blocks = 1 + (int)std::min<int64_t>((rows + 3) / 4, (int64_t)num_sms * 2);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(blocks);
        cfg.blockDim = dim3(1024);
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cudaError_t err = cudaLaunchKernelEx(&cfg, gather_kernel, g);
        if (err != cudaSuccess) return err;
    }
    GemmArgs a;
    a.experts = f.experts;
    a.H = f.H;
    a.I = f.I;
    a.E = f.E;
    a.k = f.k;
    a.n_shared = f.n_shared;
    a.T = f.T;
    a.offsets = f.offsets;
    a.active = f.active;
    a.n_active = f.n_active;
    a.ntile_start = ntile_start;
    a.wmaps = wmaps;
    a.hbuf = f.hp;
    a.y = f.y;
    a.per_row = f.per_row;
    a.status = f.status;
    // activation / h tiles as 128-, 64- and 32-row boxes
    CUtensorMap xmap[3], hmap[3];
    for (int b = 0; b < 3; ++b) {
        const uint32_t rows = 128u >> b;
        if (!encode_2d(&xmap[b], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, xg, f.H, (uint64_t)(P + f.T),
                       (uint64_t)f.H * 2, BK, rows, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !encode_2d(&hmap[b], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, f.hp, f.I, (uint64_t)S,
                       (uint64_t)f.I * 2, BK, rows, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    }
    profile_mark(1, st);
    cudaError_t err = small ? launch_gemm<true, true>(xmap, a, num_sms, st)
                            : launch_gemm<true, false>(xmap, a, num_sms, st);
    if (err != cudaSuccess) return err;
    profile_mark(2, st);
    err = small ? launch_gemm<false, true>(hmap, a, num_sms, st)
                : launch_gemm<false, false>(hmap, a, num_sms, st);
    profile_mark(3, st);
    return err;
}

bool prefill_available() { return get_encode() != nullptr; }

bool encode_codes_2d(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows,
                     uint32_t box_bytes, uint32_t box_rows, bool swizzle128) {
    return encode_2d(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, row_bytes, rows, row_bytes, box_bytes,
                     box_rows, swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE);
}

bool encode_tma(CUtensorMap* m, const void* base, int rank, int rows, int row_bytes, int segs,
                int box_rows) {
    auto enc = get_encode();
    if (!enc || rank != 3 || row_bytes % 128) return false;
    const cuuint64_t dims[3] = {128, (cuuint64_t)(row_bytes / 128), (cuuint64_t)rows};
    const cuuint64_t strides[2] = {128, (cuuint64_t)row_bytes};
    const cuuint32_t box[3] = {128, (cuuint32_t)segs, (cuuint32_t)box_rows};
    const cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box,
               es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_tma_rows_u16(CUtensorMap* m, const void* base, int rows, int cols, int box_cols,
                         int box_rows) {
    auto enc = get_encode();
    if (!enc || cols % 8 || box_cols % 8 || box_cols > 256 || box_rows > 256) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    const cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(base), dims, strides, box,
               es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace coli
