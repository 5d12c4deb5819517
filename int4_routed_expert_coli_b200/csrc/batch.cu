// Small-batch expert FFN: every call with up to 64 tokens that the fused
// decode kernel does not take (more than 8 tokens, T*k >= E, or a layer
// shape outside the fused kernel's).
//
// With a few tokens per expert, each active expert's weights are streamed
// once for its token list (the batch-union, "yunpan.plus/t/30351-1-1",
// capability two).  Codes are unpacked in registers by the fused decode
// kernel's raw unpack (1032 + q at even k, 1152 + 16 q at odd k, whose
// activations enter divided by 16) and one fp16 add takes the offsets off
// (q, 16 q: exact), so each group's chain of m16n8k16 MMAs (the activation
// fragments as 8-token column tiles) starts from zero; fp32 accumulation,
// each group's bf16 scale applied to the group's partial.  (Offset sums as
// the chains' initial values, loaded or from an MMA of the unpack's constant
// part, put a dependent load or four MMAs in front of every chain, and were
// slower.)
// The weights never pass through shared-memory operands of the tensor cores
// or tensor memory: at a few tokens per expert the grouped GEMM's fp16
// operand costs more on-chip traffic than HBM delivers.
//
// Tiles.  A tile is 256 weight rows of one expert over the whole reduction
// dimension and up to 32 entries of its token list: for gate/up the gate and
// the up rows of 128 features, for down 256 rows of W_d.  Each of 16
// consumer warps owns 16 rows (gate/up: 8 gate and the 8 up rows of the same
// features, so SwiGLU happens in registers) and runs the whole K loop: no
// partial sums cross warps.  A list of more than 32 tokens (calls with more
// than 32 tokens: the shared experts, popular routed ones) is split into two
// column chunks, each a tile of its own that reads the rows again.  Tiles are
// numbered slot-major (shared experts first) and handed out one at a time
// through a counter in the workspace to the CTAs (one per SM).
//
// Data movement.  A producer warp stages four 64-element K-blocks at a time
// in a ring of 4 stages of 53 KB: the codes of the tile's rows by two 2-D
// tensor copies (128 rows x 128 bytes each, 128-byte swizzle: a box of one
// K-block per row moves a quarter of the bytes per copied row, and the copy
// engine's row rate then limits the stream); each token's 256 activations
// (fragment order, 512 bytes) by a 1-D bulk copy into a row of 528 bytes (the
// padding spreads the fragment reads over the banks): for gate/up the
// prepared x rows of the list's tokens, for down the h' rows that the gate/up
// kernel wrote (odd features / 16); and, for gs64 rows of whole 16-byte scale
// chunks, the 8-scale chunk of each row holding the stage's four scales (two
// 128-row tensor copies).  Other scale layouts (per-row, or K / 64 not a
// multiple of 8) are read by the consumers from global memory.  With each
// stage the producer writes a record of its tile (row tile, list, K-block,
// whether it ends the tile), so the consumers run stage by stage without
// global loads; a record with no entries ends the sequence.
//
// Every wait is bounded (COLI_ERR_TIMEOUT).
#include <cuda.h>

#include <cstring>
#include <type_traits>
#include <new>

#include "batch.cuh"
#include "decode.cuh"
#include "prefill.cuh"
#include "mma_frag.cuh"
#include "moe_device.cuh"
#include "ptx.cuh"

namespace coli {
namespace {

constexpr int kBW = 16;                               // consumer warps
constexpr int kBThreads = (kBW + 1) * 32;             // + producer warp
constexpr int kTileRows = 16 * kBW;                   // weight rows per tile
constexpr int kBoxRows = 128;                         // rows per tensor copy
constexpr int kChunkTok = 32;                         // list entries per tile
constexpr int kMaxNT = kChunkTok / 8;                 // 8-token column tiles
constexpr int kChunks = kBatchMaxTokens / kChunkTok;  // column chunks of a list
constexpr int kKBS = 4;                               // K-blocks (scale groups) per stage
constexpr int kBoxBytes = kBoxRows * kKBS * 32;       // one tensor copy: 128 rows x 128 bytes
constexpr int kCodeBytes = 2 * kBoxBytes;             // a stage's codes (two copies)
constexpr int kActRow = kKBS * 128 + 16;              // staged activation row (bytes)
constexpr int kScaleOff = kCodeBytes + kChunkTok * kActRow;  // scale chunks (kVec)
constexpr int kScaleBox = kBoxRows * 16;                      // 128 rows x 8 scales
constexpr int kScaleBytes = 2 * kScaleBox;
constexpr int kStageB = (kScaleOff + kScaleBytes + 1023) / 1024 * 1024;
constexpr int kHdrB = 1024;
constexpr int kSmemLimitB = 227 * 1024;
constexpr int kStagesB = 4;
constexpr int kSmemB = kHdrB + kStagesB * kStageB + 1024;  // 1024: alignment slack
constexpr unsigned kAllB = 0xffffffffu;
static_assert(kSmemB <= kSmemLimitB, "stage ring");
static_assert(kChunkTok <= 32, "one activation row per producer lane");
static_assert(kActRow % 16 == 0 && kScaleOff % 128 == 0, "copy destinations");
// the 128-byte swizzle repeats every 8 rows of 128 bytes: stages stay 1 KB aligned
static_assert(kStageB % 1024 == 0 && kHdrB % 1024 == 0 && kBoxBytes % 1024 == 0, "swizzle atoms");
// a staged activation row of 33 16-byte units: the 8 lanes of a quarter-warp
// (rows r, r + 1; units 2c .. 2c + 1) fall on distinct bank groups
static_assert((kActRow / 16) % 8 == 1, "activation row stride");

__device__ __forceinline__ uint4 lds_u4(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(a));
    return v;
}

__device__ __forceinline__ void tma_2d_hint(void* dst, const void* tmap, int c0, int c1,
                                            uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
        "[%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_addr(dst)),
        "l"(tmap), "r"(c0), "r"(c1), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void tma_2d(void* dst, const void* tmap, int c0, int c1, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_addr(dst)),
        "l"(tmap), "r"(c0), "r"(c1), "r"(smem_addr(bar))
        : "memory");
}

// One expert slot of the call: shared experts first (every token, weight 1),
// then the active routed experts in the union's order.
struct BSlot {
    int e;           // expert row in the device table
    int list_begin;  // first h / y row of the slot's token list
    int ntok;        // tokens on the list
    bool shared;
    bool valid;      // false: an inconsistent union entry (reported, skipped)
};

__device__ __forceinline__ BSlot batch_slot(const FfnArgs& a, int slot) {
    BSlot s;
    const int P = a.T * a.k;
    if (slot < a.n_shared) {
        s.e = a.E + slot;
        s.list_begin = P + slot * a.T;
        s.ntok = a.T;
        s.shared = true;
        s.valid = a.T <= kBatchMaxTokens;
        return s;
    }
    s.shared = false;
    const int e = a.active[slot - a.n_shared];
    int b = 0, en = 0;
    if (e >= 0 && e < a.E) {
        b = a.offsets[e];
        en = a.offsets[e + 1];
    }
    s.valid = e >= 0 && e < a.E && b >= 0 && en > b && en <= P && en - b <= kBatchMaxTokens;
    s.e = s.valid ? e : 0;
    s.list_begin = s.valid ? b : 0;
    s.ntok = s.valid ? en - b : 0;
    return s;
}

// What a staged stage holds, written by the producer before it arms the
// stage (the arming arrive releases it to the consumers' waits).
struct StageMeta {
    int mt;          // row tile
    int row_begin;   // first h / y row of the tile's list entries (0 .. ntok - 1)
    int ntok;        // list entries; 0: the CTA's tile sequence is over
    int kb0;         // first K-block of the stage
    int last;        // the tile's last stage
    int e;           // expert row in the device table
};

// kGU: gate/up + SwiGLU -> h' rows; otherwise down -> y rows.  kVec: gs64
// scale rows of whole 16-byte chunks (K / 64 a multiple of 8), staged with
// the codes; otherwise read from global memory one per K-block (per-row: the
// row's one scale).
template <bool kGU, bool kVec>
__global__ void __launch_bounds__(kBThreads, 1)
batch_ffn_kernel(const FfnArgs a, const CUtensorMap* __restrict__ bmaps) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kStagesB;
    volatile StageMeta* meta = reinterpret_cast<volatile StageMeta*>(smem + 128);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + 512);
    uint8_t* stage0 = smem + kHdrB;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStagesB; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kBW);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    pdl_launch_dependents();
    pdl_wait();  // the union lists and the activation rows come from the previous kernels

    const int K = kGU ? a.H : a.I;
    const int KB = K / kGroup;

    if (warp == kBW) {
        // ------------------------------ producer ------------------------------
        int n_act = *reinterpret_cast<const volatile int*>(a.n_active);
        if (n_act < 0 || n_act > a.E) {
            if (lane == 0) report(a.status, COLI_ERR_BAD_INDEX);
            n_act = 0;
        }
        const int n_slots = n_act + a.n_shared;
        const int m_tiles = kGU ? a.I / kBoxRows : (a.H + kTileRows - 1) / kTileRows;
        const int n_chunks = a.T > kChunkTok ? kChunks : 1;  // column chunks per list
        const int64_t n_tiles = (int64_t)n_slots * n_chunks * m_tiles;
        const int P = a.T * a.k;
        const uint64_t policy = policy_evict_first();
        int j = 0;
        bool stop = false;
        // waits for stage j's slot to be free; false: wind down
        auto acquire = [&](int jj) {
            const int use = jj / kStagesB;
            int ok = 1;
            if (lane == 0) {
                if (*abort_flag) ok = 0;
                else if (use > 0) ok = (int)mbar_wait(&empty[jj & (kStagesB - 1)], (uint32_t)(use - 1) & 1);
                if (!ok && !*abort_flag) {
                    report(a.status, COLI_ERR_TIMEOUT);
                    *abort_flag = 1;
                }
            }
            return __shfl_sync(kAllB, ok, 0) != 0;
        };
        // tiles are handed out one at a time (the next one grabbed while the
        // current one streams): the shared experts' and the long lists'
        // column tiles cost more than one-token tiles, so a fixed deal leaves
        // the CTAs that drew them behind
        int* tile_cnt = reinterpret_cast<int*>(reinterpret_cast<char*>(a.status) + kBatchCntOffset) +
                        (kGU ? 0 : 1);
        int grabbed = lane == 0 ? atomicAdd(tile_cnt, 1) : 0;  // lane 0's claim, read late
        for (int64_t tile = __shfl_sync(kAllB, grabbed, 0); tile < n_tiles && !stop;
             tile = __shfl_sync(kAllB, grabbed, 0)) {
            if (lane == 0) grabbed = atomicAdd(tile_cnt, 1);
            // tile -> slot (shared experts first), column chunk, row tile
            const int slot = (int)(tile / (n_chunks * m_tiles));
            const int rem = (int)(tile - (int64_t)slot * n_chunks * m_tiles);
            const int ch = rem / m_tiles, mt = rem - ch * m_tiles;
            const BSlot sl = batch_slot(a, slot);
            if (!sl.valid) {
                if (lane == 0 && ch == 0 && mt == 0) report(a.status, COLI_ERR_BAD_INDEX);
                continue;
            }
            const int n_base = ch * kChunkTok;
            const int ntok = min(kChunkTok, sl.ntok - n_base);
            if (ntok <= 0) continue;
            // this lane's activation row: list entry n_base + lane (a pair id
            // out of range reads token 0's row and is reported; the combine
            // skips it)
            const __half* src = nullptr;
            if (lane < ntok) {
                const int n = n_base + lane;
                if constexpr (kGU) {
                    int t = n;
                    if (!sl.shared) {
                        const int p = a.pairs[sl.list_begin + n];
                        if (p < 0 || p >= P) report(a.status, COLI_ERR_BAD_INDEX);
                        t = (p >= 0 && p < P) ? p / a.k : 0;
                    }
                    src = a.xp + (int64_t)t * a.H;
                } else {
                    src = a.hp + (int64_t)(sl.list_begin + n) * a.I;
                }
            }
            const CUtensorMap* maps = bmaps + (size_t)sl.e * 6;
            const CUtensorMap* map0 = maps + (kGU ? 0 : 2);
            const CUtensorMap* map1 = maps + (kGU ? 1 : 2);
            const int row0 = kGU ? mt * kBoxRows : mt * kTileRows;
            const int row1 = kGU ? row0 : row0 + kBoxRows;  // down rows past H read as zeros
            for (int kb0 = 0; kb0 < KB; kb0 += kKBS) {
                const int nkb = min(kKBS, KB - kb0);
                // a box past the end of K (or of the rows) is filled with zeros
                // and counts whole
                const uint32_t tx = (uint32_t)(kCodeBytes + ntok * nkb * 128) +
                                    (kVec ? (uint32_t)kScaleBytes : 0u);
                if (!acquire(j)) {
                    stop = true;
                    break;
                }
                const int s = j & (kStagesB - 1);
                uint8_t* st = stage0 + (size_t)s * kStageB;
                if (lane == 0) {
                    meta[s].mt = mt;
                    meta[s].row_begin = sl.list_begin + n_base;
                    meta[s].ntok = ntok;
                    meta[s].kb0 = kb0;
                    meta[s].last = kb0 + kKBS >= KB;
                    meta[s].e = sl.e;
                    mbar_arrive_expect_tx(&full[s], tx);  // releases the record
                    const int xk = kb0 * (kGroup / 2);     // a multiple of 128 bytes
                    tma_2d_hint(st, map0, xk, row0, &full[s], policy);
                    tma_2d_hint(st + kBoxBytes, map1, xk, row1, &full[s], policy);
                    if constexpr (kVec) {
                        // the 8-scale chunk holding the stage's 4 (x: a multiple of 8 scales)
                        const int xs = kb0 & ~7;
                        tma_2d(st + kScaleOff, maps + (kGU ? 3 : 5), xs, row0, &full[s]);
                        tma_2d(st + kScaleOff + kScaleBox, maps + (kGU ? 4 : 5), xs, row1, &full[s]);
                    }
                }
                __syncwarp();
                if (lane < ntok)
                    bulk_g2s(st + kCodeBytes + lane * kActRow, src + kb0 * kGroup,
                             (uint32_t)nkb * 128u, &full[s]);
                ++j;
            }
        }
        if (!stop && acquire(j)) {
            // the end of the sequence: a stage with no entries, armed by a plain arrive
            const int s = j & (kStagesB - 1);
            if (lane == 0) {
                meta[s].ntok = 0;
                mbar_arrive(&full[s]);
            }
            ++j;
        } else {
            stop = true;
        }
        if (stop && lane == 0) {
            // let the copies already issued land before the CTA goes away
            for (int back = 1; back <= kStagesB && back <= j; ++back) {
                const int jj = j - back;
                (void)mbar_wait(&full[jj & (kStagesB - 1)], (uint32_t)(jj / kStagesB) & 1);
            }
        }
        return;
    }

    // -------------------------------- consumers --------------------------------
    const int r = lane >> 2, c = lane & 3;
    const Magic mg = magic();
    // staged rows of this warp's A fragment rows 0-7 and 8-15: gate/up, row
    // 8 warp + r of the gate box and of the up box; down, rows 16 warp + r and
    // + 8 of the tile (box warp / 8).  Every such row is r modulo 8, so the
    // swizzle puts logical 16-byte unit u of a row at u ^ r: K-block q's 8
    // bytes for this lane (unit 2q + c / 2, half c % 2) sit at
    // ((q ^ (r / 2)) * 32) + ((c / 2) ^ (r % 2)) * 16 + (c % 2) * 8.
    const int rtop = kGU ? 8 * warp + r : 16 * warp + r;
    const uint32_t off_a = (uint32_t)((rtop / kBoxRows) * kBoxBytes + (rtop % kBoxRows) * 128 +
                                      (((c >> 1) ^ (r & 1)) << 4) + ((c & 1) << 3));
    const uint32_t off_b = kGU ? off_a + (uint32_t)kBoxBytes : off_a + 8u * 128u;
    const uint32_t rq = (uint32_t)(r >> 1);
    // staged scale chunks of the two rows (16 bytes a row in 128-row boxes)
    const uint32_t soff_a = (uint32_t)(kScaleOff + (rtop / kBoxRows) * kScaleBox + (rtop % kBoxRows) * 16);
    const uint32_t soff_b = kGU ? soff_a + (uint32_t)kScaleBox : soff_a + 8u * 16u;
    const int SG = scale_cols(K, a.per_row);

    float acc[kMaxNT][4];
    int ra = 0, rb = 0, nt = 0;
    bool live_a = true, live_b = true;
    const uint16_t* sa = nullptr;  // global scale rows (not kVec)
    const uint16_t* sb = nullptr;
    uint16_t na = 0, nb = 0;
    for (int j = 0;; ++j) {
        const int s = j & (kStagesB - 1);
        if (*abort_flag || !mbar_wait(&full[s], (uint32_t)(j / kStagesB) & 1)) {
            if (lane == 0 && !*abort_flag) {
                report(a.status, COLI_ERR_TIMEOUT);
                *abort_flag = 1;
            }
            return;
        }
        const int ntok = meta[s].ntok;
        if (ntok <= 0) return;  // the sequence is over
        const int mt = meta[s].mt, kb0 = meta[s].kb0, row_begin = meta[s].row_begin;
        const bool last = meta[s].last != 0;
        if (kb0 == 0) {
            // a new tile: this lane's two weight rows
            nt = (ntok + 7) >> 3;
            if constexpr (kGU) {
                ra = rb = mt * kBoxRows + 8 * warp + r;  // gate row and up row of one feature
            } else {
                ra = mt * kTileRows + 16 * warp + r;
                rb = ra + 8;
                live_a = ra < a.H;
                live_b = rb < a.H;
            }
            if constexpr (!kVec) {
                const DevExpert ex = a.experts[meta[s].e];
                if constexpr (kGU) {
                    sa = ex.gate_s + (int64_t)ra * SG;
                    sb = ex.up_s + (int64_t)rb * SG;
                } else {
                    sa = ex.down_s + (int64_t)(live_a ? ra : 0) * SG;
                    sb = ex.down_s + (int64_t)(live_b ? rb : 0) * SG;
                }
                na = live_a ? __ldg(sa) : (uint16_t)0;
                nb = live_b ? __ldg(sb) : (uint16_t)0;
            }
#pragma unroll
            for (int jn = 0; jn < kMaxNT; ++jn)
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[jn][q] = 0.f;
        }
        const uint32_t st = smem_addr(stage0) + (uint32_t)(s * kStageB);
        // the stage's four scales of both rows, as bf16 pairs: the first or
        // the second half of the staged chunk
        uint32_t spa0 = 0u, spa1 = 0u, spb0 = 0u, spb1 = 0u;
        if constexpr (kVec) {
            const uint32_t half = (kb0 & 4) ? 8u : 0u;
            const uint2 va = lds_u2(st + soff_a + half), vb = lds_u2(st + soff_b + half);
            spa0 = va.x;
            spa1 = va.y;
            spb0 = vb.x;
            spb1 = vb.y;
        }
        // the stage's MMAs with the tile's column-tile count fixed
        auto stage_math = [&](auto ntc) {
            constexpr int NT = decltype(ntc)::value;
#pragma unroll
            for (int q = 0; q < kKBS; ++q) {
                const int kb = kb0 + q;
                if (kb >= KB) break;
                float fa, fb;
                if constexpr (kVec) {
                    const uint32_t wa2 = q < 2 ? spa0 : spa1, wb2 = q < 2 ? spb0 : spb1;
                    fa = __uint_as_float((q & 1) ? (wa2 & 0xFFFF0000u) : (wa2 << 16));
                    fb = __uint_as_float((q & 1) ? (wb2 & 0xFFFF0000u) : (wb2 << 16));
                } else {
                    fa = __uint_as_float((uint32_t)na << 16);
                    fb = __uint_as_float((uint32_t)nb << 16);
                    if (!a.per_row && kb + 1 < KB) {
                        if (live_a) na = __ldg(sa + kb + 1);
                        if (live_b) nb = __ldg(sb + kb + 1);
                    }
                }
                const uint32_t blk = st + ((((uint32_t)q) ^ rq) << 5);
                const uint2 wa = lds_u2(blk + off_a), wb = lds_u2(blk + off_b);
                // exact codes: q at even k, 16 q at odd k (the raw unpack less
                // its offsets, exact in fp16), so every chain starts from zero
                uint32_t A[4][4];
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    unpack_raw_step((ks >> 1) ? wa.y : wa.x, ks & 1, A[ks][0], A[ks][2], mg);
                    unpack_raw_step((ks >> 1) ? wb.y : wb.x, ks & 1, A[ks][1], A[ks][3], mg);
#pragma unroll
                    for (int u = 0; u < 4; ++u) A[ks][u] = strip_offset(A[ks][u], u >= 2);
                }
                const uint32_t bbase = st + (uint32_t)(kCodeBytes + r * kActRow + q * 128 + c * 32);
#pragma unroll
                for (int jn = 0; jn < NT; ++jn) {
                    const uint4 b0 = lds_u4(bbase + (uint32_t)(jn * 8 * kActRow));
                    const uint4 b1 = lds_u4(bbase + (uint32_t)(jn * 8 * kActRow) + 16u);
                    const uint32_t bw[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
                    float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma16816(part, part, A[ks][0], A[ks][1], A[ks][2], A[ks][3],
                                 bw[2 * ks], bw[2 * ks + 1]);
                    acc[jn][0] = fmaf(fa, part[0], acc[jn][0]);
                    acc[jn][1] = fmaf(fa, part[1], acc[jn][1]);
                    acc[jn][2] = fmaf(fb, part[2], acc[jn][2]);
                    acc[jn][3] = fmaf(fb, part[3], acc[jn][3]);
                }
            }
        };
        if (nt == 1) stage_math(std::integral_constant<int, 1>{});
        else if (nt == 2) stage_math(std::integral_constant<int, 2>{});
        else if (nt == 3) stage_math(std::integral_constant<int, 3>{});
        else stage_math(std::integral_constant<int, 4>{});
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        if (!last) continue;

        // epilogue: column 8 jn + 2c + e2 is list entry that of the tile; rows
        // ra (acc 0, 1) and rb (acc 2, 3)
#pragma unroll
        for (int jn = 0; jn < kMaxNT; ++jn) {
            if (jn >= nt) continue;
#pragma unroll
            for (int e2 = 0; e2 < 2; ++e2) {
                const int nl = 8 * jn + 2 * c + e2;
                if (nl >= ntok) continue;
                const int64_t orow = row_begin + nl;
                if constexpr (kGU) {
                    // h = silu(g) * u; the gate weight is applied by the combine
                    const float gv = acc[jn][e2], uv = acc[jn][2 + e2];
                    float h = gv / (1.f + expf(-gv)) * uv;
                    if (fabsf(h) > 65504.f) {
                        report(a.status, COLI_ERR_RANGE);
                        h = copysignf(65504.f, h);
                    }
                    // h' in the down operand's fragment order; odd features
                    // are the down projection's odd-K elements: stored / 16
                    const int fe = ra;
                    const int hcol = (fe / kGroup) * kGroup + perm64(fe % kGroup);
                    a.hp[orow * a.I + hcol] = __float2half_rn((fe & 1) ? h * 0.0625f : h);
                } else {
                    if (live_a) a.y[orow * a.H + ra] = acc[jn][e2];
                    if (live_b) a.y[orow * a.H + rb] = acc[jn][2 + e2];
                }
            }
        }
    }
}

template <bool kGU, bool kVec>
cudaError_t launch_one(const FfnArgs& a, const CUtensorMap* bmaps, int blocks, cudaStream_t st) {
    auto kern = batch_ffn_kernel<kGU, kVec>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemB);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(blocks);
    cfg.blockDim = dim3(kBThreads);
    cfg.dynamicSmemBytes = kSmemB;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a, bmaps);
}

}  // namespace

bool batch_supported(int H, int I, int T) {
    return T >= 1 && T <= kBatchMaxTokens && H >= kKBS * kGroup && H % (kKBS * kGroup) == 0 &&
           I >= kBoxRows && I % kBoxRows == 0;
}

cudaError_t launch_batch_ffn(const FfnArgs& a, const CUtensorMap* bmaps, int num_sms,
                             cudaStream_t st) {
    // gs64 rows of whole 16-byte chunks: scales staged with the codes
    const bool vec_gu = !a.per_row && (a.H / kGroup) % 8 == 0;
    const bool vec_dn = !a.per_row && (a.I / kGroup) % 8 == 0;
    profile_mark(1, st);
    cudaError_t err = vec_gu ? launch_one<true, true>(a, bmaps, num_sms, st)
                             : launch_one<true, false>(a, bmaps, num_sms, st);
    if (err != cudaSuccess) return err;
    profile_mark(2, st);
    err = vec_dn ? launch_one<false, true>(a, bmaps, num_sms, st)
                 : launch_one<false, false>(a, bmaps, num_sms, st);
    profile_mark(3, st);
    return err;
}

cudaError_t build_batch_maps(const DevExpert* host_experts, int n, int H, int I, bool per_row,
                             CUtensorMap** d_maps) {
    *d_maps = nullptr;
    CUtensorMap* maps = new (std::nothrow) CUtensorMap[(size_t)n * 6];
    if (!maps) return cudaErrorMemoryAllocation;
    std::memset(maps, 0, sizeof(CUtensorMap) * (size_t)n * 6);
    const int GH = H / kGroup, GI = I / kGroup;
    const bool vec_gu = !per_row && GH % 8 == 0, vec_dn = !per_row && GI % 8 == 0;
    bool ok = true;
    for (int e = 0; e < n && ok; ++e) {
        const DevExpert& x = host_experts[e];
        CUtensorMap* m = maps + (size_t)e * 6;
        const uint32_t box = kKBS * 32;  // four K-blocks of a row
        ok = encode_codes_2d(&m[0], x.gate_q, H / 2, I, box, kBoxRows, true) &&
             encode_codes_2d(&m[1], x.up_q, H / 2, I, box, kBoxRows, true) &&
             encode_codes_2d(&m[2], x.down_q, I / 2, H, box, kBoxRows, true);
        if (ok && vec_gu)
            ok = encode_tma_rows_u16(&m[3], x.gate_s, I, GH, 8, kBoxRows) &&
                 encode_tma_rows_u16(&m[4], x.up_s, I, GH, 8, kBoxRows);
        if (ok && vec_dn) ok = encode_tma_rows_u16(&m[5], x.down_s, H, GI, 8, kBoxRows);
    }
    if (!ok) {
        delete[] maps;
        return cudaErrorInvalidValue;
    }
    cudaError_t err = cudaMalloc(d_maps, sizeof(CUtensorMap) * (size_t)n * 6);
    if (err == cudaSuccess)
        err = cudaMemcpy(*d_maps, maps, sizeof(CUtensorMap) * (size_t)n * 6, cudaMemcpyHostToDevice);
    delete[] maps;
    if (err != cudaSuccess && *d_maps) {
        cudaFree(*d_maps);
        *d_maps = nullptr;
    }
    return err;
}

}  // namespace coli
