// Fused decode step (T <= 8 tokens): routing, batch-union, gate/up +
// SwiGLU, down and the weighted combine in one persistent kernel that streams
// every active expert's int4 gs64 weights from HBM exactly once per call
// ("batch-union", "yunpan.plus/t/30351-1-1", capability two).
//
// Routing.  In every CTA, consumer warp t routes token t from the logits
// (the exact rule of the routing step, with a butterfly top-k) while the
// activations load, and the producer warp builds the slot table in shared
// memory: shared experts first, then the active routed experts in ascending
// order, each with the positions and gate weights of its tokens.  Given a
// precomputed union instead (the FFN entry point), the table is read from
// it.  The shared experts' entries need no routing, so their gate/up tiles
// are staged and computed before the table is known.
//
// Gate/up.  An item is 8 gate rows + the same 8 up rows of one slot over the
// whole hidden dimension; items are dealt round-robin to the CTAs (one per
// SM), shared experts first, so their weights stream while routing runs.
// The gate weight is folded into the epilogue: h' = w * silu(g) * u (fp16).
// After writing an item's h' values a warp bumps the slot's counter.
//
// Down + combine.  A CTA owns a fixed set of 16-row tiles of the output and
// streams, slot after slot, those rows of W_d.  The MMA columns are the
// tokens, so y = sum over slots of W_d h' accumulates in registers: the
// combine is the accumulation itself, in a fixed order (slot order, then a
// fixed sum over the warps).  A slot's h' rows are read once it is below the
// frontier of complete slots, which the producer warp follows by polling the
// slots' counters and publishes in shared memory.
//
// Data movement.  A producer warp loads each stage with 3-D TMA tensor copies
// of the packed code rows (viewed as 128-byte chunks plus zero-filled padding
// chunks, 128-byte swizzle, so the consumers' fragment reads spread over the
// banks) and 2-D copies of the scale rows (padded to 8 x odd columns).
//
// Arithmetic: raw fp16 unpack of the codes (1032 + q for even K, 1152 + 16 q
// for odd K, whose activations enter divided by 16) with the per-(token,
// group) offset sum of the activation operand as the MMA chain's initial
// value: for gate/up the sums of x, for down the sums of the slot's h'
// (stored with its odd elements divided by 16), computed from the h'
// fragments with four MMAs per group; m16n8k16 MMA with fp32 accumulation,
// the group's scale applied to each group's partial.  Sixteen consumer warps split K; a gate/up item's
// partials are summed through four reduction buffers, item j by warp j mod 16
// two items later (in warp order, so the sum does not depend on timing).
//
// Every wait is bounded (COLI_ERR_TIMEOUT).  The counters are zero on entry;
// the last CTA to finish puts them back to zero.
#include <algorithm>
#include <climits>
#include <new>

#include "decode.cuh"
#include "mma_frag.cuh"
#include "moe_device.cuh"
#include "ptx.cuh"

namespace coli {
namespace {

constexpr int kCW = 16;                      // consumer warps (17 warps in all)
constexpr int kThreadsD = (kCW + 1) * 32;    // + producer warp
constexpr int kStagesD = 3;
constexpr int kRedBufs = 4;
constexpr int kRedLag = 2;  // item j is summed by warp j % kCW while it works on item j + 2
constexpr int kSmemLimitD = 227 * 1024;
constexpr int kGuRows = 8;                   // gate rows (and up rows) per gate/up item
constexpr int kDnRows = 16;                  // rows per down tile
constexpr int kMaxMT = 3;                    // down tiles per CTA
constexpr int kMaps = 6;                     // per expert: 3 code maps, 3 scale maps
constexpr int kMaxPairs = 256;               // T * k
constexpr int kRedFloats = kRedBufs * kCW * 4 * 32;
// Counters of a call (ints at the workspace's counter offset, zero between calls)
constexpr int kSyncDone = 0;   // CTAs finished
constexpr int kSyncItems = 1;  // gate/up items handed out beyond the first one per CTA
constexpr int kSyncSlots = 2;  // + s: gate/up tiles of slot s published
static_assert(kRedFloats >= kCW * kMaxMT * 4 * 32, "final reduction reuses the buffers");

struct SlotEntry {
    int e;           // expert index (E + i for shared expert i); -1: invalid slot
    int list_begin;  // h row of the first token on the slot's list
    int8_t pos[8];   // position of token t on the list; -1: not routed here
    float w[8];      // gate weight of token t (1 for a shared expert)
};
static_assert(sizeof(SlotEntry) == 48, "slot entry layout");

// A padded scale row: 8 * odd bf16 columns, so 8 rows fall on distinct banks.
__host__ __device__ inline int padded_groups(int G) {
    int p = (G + 1 + 7) / 8 * 8;
    if ((p / 8) % 2 == 0) p += 8;
    return p;
}

// Chunks per staged gate/up row: = 2 (mod 8), so rows r and r + 1 differ by
// two in the swizzle phase and a half-warp's 8-byte reads hit 32 banks.
__host__ __device__ inline int gu_segs_for(int row_bytes) {
    int s = row_bytes / 128;
    while (s % 8 != 2) ++s;
    return s;
}

// Chunks per staged down row: odd (costs less shared memory than the rule above).
__host__ __device__ inline int dn_segs_for(int row_bytes) {
    const int chunks = row_bytes / 128;
    return chunks + ((chunks % 2 == 0) ? 1 : 2);
}

struct Layout {
    int gu_segs, dn_segs;       // 128-byte chunks per staged code row
    int gGp, dGp;               // padded scale row lengths (bf16 elements)
    int gsr, gsg, dsr, dsg;     // staged scale (row, group) strides in bytes, gate/up and down
    int gu_op, gu_sc, gu_tx;    // gate/up item: code copy, scale copy, bytes per stage
    int dn_op, dn_sc;           // down tile: code copy, scale copy
    int stage_bytes;
    int red_off, corr_off, route_off, table_off, stage_off, smem;
};

// per_row: one scale per row (staged as the item's rows' scales, 2 bytes
// each, every group reading its row's one scale).
__host__ __device__ inline Layout make_layout(int H, int I, int max_slots, int per_row) {
    Layout L;
    L.gu_segs = gu_segs_for(H / 2);
    L.dn_segs = dn_segs_for(I / 2);
    // every consumer warp owns kMaxGW (kMaxDW) consecutive groups; the groups
    // past the end read zero scales from the padding columns (gs64), or the
    // row's scale times a zero activation fragment (per-row)
    L.gGp = padded_groups(kCW * kMaxGW > H / kGroup ? kCW * kMaxGW : H / kGroup);
    L.dGp = padded_groups(kCW * kMaxDW > I / kGroup ? kCW * kMaxDW : I / kGroup);
    L.gsr = per_row ? 2 : L.gGp * 2;
    L.gsg = per_row ? 0 : 2;
    L.dsr = per_row ? 2 : L.dGp * 2;
    L.dsg = per_row ? 0 : 2;
    L.gu_op = kGuRows * L.gu_segs * 128;
    L.gu_sc = kGuRows * L.gsr;
    L.gu_tx = 2 * L.gu_op + 2 * L.gu_sc;
    L.dn_op = kDnRows * L.dn_segs * 128;
    L.dn_sc = kDnRows * L.dsr;
    const int dn_stage = kMaxMT * (L.dn_op + L.dn_sc);
    L.stage_bytes = ((L.gu_tx > dn_stage ? L.gu_tx : dn_stage) + 1023) / 1024 * 1024;
    L.red_off = 1024;
    L.corr_off = L.red_off + kRedFloats * 4;
    L.route_off = L.corr_off + kCW * kMaxGW * 16 * 4;
    L.table_off = L.route_off + 3 * kMaxPairs * 4;
    L.stage_off = (L.table_off + max_slots * (int)sizeof(SlotEntry) + 1023) / 1024 * 1024;
    L.smem = L.stage_off + kStagesD * L.stage_bytes + 1024;  // + alignment slack
    return L;
}


// Byte offset (in a code copy) of the 8 bytes lane c of row `row` feeds to
// group grp: the padded, swizzled layout (segments of 128 bytes, segs per
// row, 16-byte chunk j of segment s stored at chunk j ^ (s & 7)).
__device__ __forceinline__ int code_offset(int row, int segs, int grp, int c) {
    const int kc = grp >> 2;
    const int j = ((grp & 3) << 1) + (c >> 1);
    const int seg = row * segs + kc;
    return seg * 128 + ((j ^ (seg & 7)) << 4) + ((c & 1) << 3);
}

// 16 consecutive bf16 activations (elements 16c .. 16c+15 of a group, as 8
// words in bw) -> in place, this lane's 8 fp16 pairs of the gate/up B
// fragment, in the fragment order of the streaming GEMV: pair q holds
// elements e and e + 4, e = (q & 3) + 8 (q >> 2), odd elements divided by 16.
// Out-of-range values are clamped (|x| <= 65504, |x / 16| <= 4094); amax
// collects |x| for the range report.
__device__ __forceinline__ void x_fragment(uint32_t bw[8], float& amax) {
    const uint32_t in[8] = {bw[0], bw[1], bw[2], bw[3], bw[4], bw[5], bw[6], bw[7]};
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const int e = (q & 3) + 8 * (q >> 2);
        const uint32_t wl = in[e >> 1], wh = in[(e >> 1) + 2];
        float lo = __uint_as_float((q & 1) ? (wl & 0xFFFF0000u) : (wl << 16));
        float hi = __uint_as_float((q & 1) ? (wh & 0xFFFF0000u) : (wh << 16));
        amax = fmaxf(amax, fmaxf(fabsf(lo), fabsf(hi)));
        if (q & 1) {
            lo = fminf(fmaxf(lo * 0.0625f, -4094.f), 4094.f);
            hi = fminf(fmaxf(hi * 0.0625f, -4094.f), 4094.f);
        }
        asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(bw[q]) : "f"(hi), "f"(lo));
    }
}

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void fence_acq_rel_gpu() {
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const void* tmap, int c0, int c1, int c2,
                                            uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
        "[%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_addr(dst)),
        "l"(tmap), "r"(c0), "r"(c1), "r"(c2), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, int c0, int c1,
                                            uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
        "[%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_addr(dst)),
        "l"(tmap), "r"(c0), "r"(c1), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

// Pointers into the dynamic shared memory.
struct Smem {
    uint64_t* full;
    uint64_t* empty;
    uint64_t* red_empty;
    uint64_t* tbl_ready;
    uint64_t* routed;          // one arrival per routing warp
    volatile int* abort_flag;
    volatile int* n_slots;
    volatile int* frontier;    // slots [0, frontier) complete GPU-wide (producer-written)
    volatile int* stage_item;  // [kStagesD] gate/up item in the stage; -1: a down stage
    int* red_cnt;      // [kRedBufs] partials written into each reduction buffer
    volatile int* red_item;  // [kRedBufs] the item whose partials a buffer holds
    float* red;        // reduction buffers; during the prologue, the logits
    float* corr;       // [groups][4 lanes][4]: negated offset sums, C-fragment order
    int* s_idx;        // [T*k] routing
    float* s_w;
    int* s_aux;
    SlotEntry* table;
    uint8_t* stage0;
};

__device__ __forceinline__ Smem carve(uint8_t* smem, const Layout& L, int max_slots) {
    Smem S;
    S.full = reinterpret_cast<uint64_t*>(smem);
    S.empty = S.full + kStagesD;
    S.red_empty = S.empty + kStagesD;
    S.tbl_ready = S.red_empty + kRedBufs;
    S.routed = S.tbl_ready + 1;
    S.abort_flag = reinterpret_cast<volatile int*>(smem + 512);
    S.n_slots = S.abort_flag + 1;
    S.red_cnt = reinterpret_cast<int*>(smem + 528);
    S.stage_item = reinterpret_cast<volatile int*>(smem + 560);
    S.red_item = reinterpret_cast<volatile int*>(smem + 576);
    S.frontier = reinterpret_cast<volatile int*>(smem + 600);
    S.red = reinterpret_cast<float*>(smem + L.red_off);
    S.corr = reinterpret_cast<float*>(smem + L.corr_off);
    S.s_idx = reinterpret_cast<int*>(smem + L.route_off);
    S.s_w = reinterpret_cast<float*>(S.s_idx + kMaxPairs);
    S.s_aux = S.s_idx + 2 * kMaxPairs;
    S.table = reinterpret_cast<SlotEntry*>(smem + L.table_off);
    S.stage0 = smem + L.stage_off;
    return S;
}

constexpr int kConsumerThreads = kCW * 32;

__device__ __forceinline__ void consumers_sync() { named_barrier(1, kConsumerThreads); }

__device__ __forceinline__ void clear_entry(SlotEntry& en) {
    en.e = -1;
    en.list_begin = 0;
#pragma unroll
    for (int t = 0; t < 8; ++t) {
        en.pos[t] = -1;
        en.w[t] = 0.f;
    }
}

// Slot i < n_shared: shared expert i, every token, weight 1 -- known without
// routing.  Lanes of one warp, each its own entries.
__device__ void table_shared(const FfnArgs& a, const Smem& S, int lane) {
    for (int i = lane; i < a.n_shared; i += 32) {
        SlotEntry& en = S.table[i];
        en.e = a.E + i;
        en.list_begin = a.T * a.k + i * a.T;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            en.pos[t] = (int8_t)(t < a.T ? t : -1);
            en.w[t] = t < a.T ? 1.f : 0.f;
        }
    }
}

// The routed slots of the table from the routing (s_idx / s_w): the union of
// the pairs p = t * k + j, experts ascending, tokens ascending inside an
// expert (the lists the batch-union step defines).  One warp.
__device__ void table_from_logits(const DecodeArgs& d, const Smem& S, int lane) {
    const FfnArgs& a = d.f;
    const int P = a.T * a.k;
    if (blockIdx.x == 0) {
        for (int p = lane; p < P; p += 32) {
            if (d.idx_out) d.idx_out[p] = S.s_idx[p];
            if (d.w_out) d.w_out[p] = S.s_w[p];
        }
    }
    for (int i = a.n_shared + lane; i < d.max_slots; i += 32) clear_entry(S.table[i]);
    __syncwarp();
    if (P <= 32) {
        // one pair per lane: leaders by match_any, ranks by shuffles
        const bool on = lane < P;
        const int e = on ? S.s_idx[lane] : INT_MAX;
        const float w = on ? S.s_w[lane] : 0.f;
        const unsigned below = (1u << lane) - 1u;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const bool lead = on && (peers & below) == 0u;
        const unsigned leads = __ballot_sync(0xffffffffu, lead);
        int before = 0, rank = 0;
        for (int q = 0; q < P; ++q) {
            const int eq = __shfl_sync(0xffffffffu, e, q);
            before += eq < e;
            rank += (eq < e) & (int)((leads >> q) & 1u);
        }
        if (on) {
            SlotEntry& en = S.table[a.n_shared + rank];
            if (lead) {
                en.e = e;
                en.list_begin = before;
            }
            const int t = lane / a.k;
            en.pos[t] = (int8_t)__popc(peers & below);
            en.w[t] = w;
        }
        if (lane == 0) *S.n_slots = a.n_shared + __popc(leads);
        __syncwarp();
        return;
    }
    // a pair is its expert's leader if no earlier pair has the same expert
    for (int p = lane; p < P; p += 32) {
        const int e = S.s_idx[p];
        int lead = 1;
        for (int q = 0; q < p; ++q) lead &= S.s_idx[q] != e;
        S.s_aux[p] = lead;
    }
    __syncwarp();
    int n = 0;
    for (int p = lane; p < P; p += 32) {
        const int e = S.s_idx[p];
        int before = 0, rank = 0, pos = 0;
        for (int q = 0; q < P; ++q) {
            const int eq = S.s_idx[q];
            before += eq < e;
            rank += (eq < e) & S.s_aux[q];
            pos += (q < p) & (eq == e);
        }
        SlotEntry& en = S.table[a.n_shared + rank];
        if (S.s_aux[p]) {
            en.e = e;
            en.list_begin = before;
        }
        const int t = p / a.k;
        en.pos[t] = (int8_t)pos;
        en.w[t] = S.s_w[p];
        n += S.s_aux[p];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
    if (lane == 0) *S.n_slots = a.n_shared + n;
    __syncwarp();
}

// The routed slots from a given union (counts / offsets / pairs / active /
// n_active and the gate weights); an inconsistent entry is reported as
// COLI_ERR_BAD_INDEX and its slot skipped.  One warp.
__device__ void table_from_union(const DecodeArgs& d, const Smem& S, int lane) {
    const FfnArgs& a = d.f;
    const int P = a.T * a.k;
    for (int i = a.n_shared + lane; i < d.max_slots; i += 32) clear_entry(S.table[i]);
    __syncwarp();
    int n_act = __shfl_sync(0xffffffffu, *reinterpret_cast<const volatile int*>(a.n_active), 0);
    const int cap = d.max_slots - a.n_shared;
    if (n_act < 0 || n_act > cap) {
        if (lane == 0) report(a.status, COLI_ERR_BAD_INDEX);
        n_act = n_act < 0 ? 0 : cap;
    }
    for (int i = lane; i < n_act; i += 32) {
        SlotEntry& en = S.table[a.n_shared + i];
        const int e = a.active[i];
        bool ok = e >= 0 && e < a.E;
        const int b = ok ? a.offsets[e] : 0;
        const int n = ok ? a.offsets[e + 1] - b : 0;
        ok = ok && b >= 0 && n >= 1 && n <= a.T && b + n <= P;
        for (int q = 0; ok && q < n; ++q) {
            const int p = a.pairs[b + q];
            ok = p >= 0 && p < P;
            if (!ok) break;
            const int t = p / a.k;
            ok = en.pos[t] < 0;  // a token appears once per expert
            en.pos[t] = (int8_t)q;
            en.w[t] = a.topk_w[p];
        }
        if (ok) {
            en.e = e;
            en.list_begin = b;
        } else {
            report(a.status, COLI_ERR_BAD_INDEX);
        }
    }
    if (lane == 0) *S.n_slots = a.n_shared + n_act;
    __syncwarp();
}

// Frontier of complete slots in shared memory: the producer warp publishes
// it with a release store after it has observed (and acquired) the slots'
// counters; a consumer that reads it with an acquire load may then read the
// h' rows of every slot below it.
__device__ __forceinline__ int ld_acquire_cta(const volatile int* p) {
    int v;
    asm volatile("ld.acquire.cta.shared::cta.b32 %0, [%1];" : "=r"(v) : "r"(smem_addr((const void*)p))
                 : "memory");
    return v;
}
__device__ __forceinline__ void st_release_cta(volatile int* p, int v) {
    asm volatile("st.release.cta.shared::cta.b32 [%0], %1;" ::"r"(smem_addr((const void*)p)), "r"(v)
                 : "memory");
}

struct Ctx {
    const FfnArgs& a;
    const Layout& L;
    const Smem& S;
    int* sync;
    int gu_tiles;
};

__device__ __forceinline__ void fail(const Ctx& x, int lane) {
    if (lane == 0) {
        report(x.a.status, COLI_ERR_TIMEOUT);
        *x.S.abort_flag = 1;
    }
}

// Partials of item j -> reduction buffer j % kRedBufs (once the sum of item
// j - kRedBufs has released it).  false: timeout.
__device__ __forceinline__ bool post_partial(const Ctx& x, int j, int item,
                                             const float (&acc)[4]) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rb = j % kRedBufs, ruse = j / kRedBufs;
    if (ruse > 0 && !mbar_wait(&x.S.red_empty[rb], (ruse - 1) & 1)) return false;
    // [warp][lane] float4 per buffer: one 16-byte store per lane
    const uint32_t rbuf = smem_addr(x.S.red) + (rb * (kCW * 4 * 32) + lane * 4) * 4;
    sts_f4(rbuf + warp * 512, make_float4(acc[0], acc[1], acc[2], acc[3]));
    if (lane == 0) x.S.red_item[rb] = item;
    __threadfence_block();
    __syncwarp();
    if (lane == 0) atomicAdd(x.S.red_cnt + rb, 1);
    return true;
}

// Publishes a gate/up tile this warp finished earlier (slot `pending`, -1:
// none): one GPU-scope fence, which makes the tile's h' stores (by this
// warp's lanes, ordered by the __syncwarp) visible first, then the slot's
// counter.  Called before the warp issues new h' stores, so the fence does
// not wait for them: the tile's own stores went out a round of items ago.
__device__ __forceinline__ void publish_tile(const Ctx& x, int pending) {
    if (pending < 0) return;
    __syncwarp();
    if ((threadIdx.x & 31) == 0) {
        fence_acq_rel_gpu();
        atomicAdd(x.sync + kSyncSlots + pending, 1);
    }
}

// Sum of item m (its kCW partials in warp order, so the result does not
// depend on timing) and its epilogue h' = w * silu(g) * u for the slot's
// tokens, by warp m % kCW kRedLag items later: off the critical path of the
// warp that finished item m last.  The tile this warp finished before is
// published first; this one becomes `pending`, stored at item `at`.
// false: timeout or abort.
__device__ bool finish_item(const Ctx& x, int m, int& pending, int& pending_at, int at) {
    const FfnArgs& a = x.a;
    const int lane = threadIdx.x & 31, r = lane >> 2, c = lane & 3;
    const int rb = m % kRedBufs;
    const volatile int* cnt = x.S.red_cnt + rb;
    if (*cnt != kCW) {
        const uint64_t t0 = global_timer_ns();
        while (*cnt != kCW) {
            if (*x.S.abort_flag) return false;
            __nanosleep(64);
            if (global_timer_ns() - t0 > kWaitLimitNs) {
                fail(x, lane);
                return false;
            }
        }
    }
    __threadfence_block();
    const uint32_t rbuf = smem_addr(x.S.red) + (rb * (kCW * 4 * 32) + lane * 4) * 4;
    float4 sum = lds_f4(rbuf);
#pragma unroll
    for (int w = 1; w < kCW; ++w) {
        const float4 p = lds_f4(rbuf + w * 512);
        sum.x += p.x;
        sum.y += p.y;
        sum.z += p.z;
        sum.w += p.w;
    }
    const int item = x.S.red_item[rb];
    __syncwarp();
    if (lane == 0) {
        x.S.red_cnt[rb] = 0;
        mbar_arrive(&x.S.red_empty[rb]);
    }
    const int slot = item / x.gu_tiles, tile = item - slot * x.gu_tiles;
    const SlotEntry* en = x.S.table + slot;
    if (en->e < 0) return true;
    publish_tile(x, pending);
    pending = slot;
    pending_at = at;
    const float v[4] = {sum.x, sum.y, sum.z, sum.w};
    const int n = tile * kGuRows + r;
    const int hcol = (n / kGroup) * kGroup + perm64(n % kGroup);
    const int list_begin = en->list_begin;
#pragma unroll
    for (int e2 = 0; e2 < 2; ++e2) {
        const int t = 2 * c + e2;
        if (t >= a.T) continue;
        const int p = en->pos[t];
        if (p < 0) continue;
        const float gv = v[e2], uv = v[2 + e2];
        float h = en->w[t] * (gv / (1.f + expf(-gv)) * uv);
        if (fabsf(h) > 65504.f) {
            report(a.status, COLI_ERR_RANGE);
            h = copysignf(65504.f, h);
        }
        // odd features are the down projection's odd-K elements: stored / 16
        // for its raw unpack (odd codes as 1152 + 16 q)
        a.hp[(int64_t)(list_begin + p) * a.I + hcol] = __float2half_rn((n & 1) ? h * 0.0625f : h);
    }
    return true;
}

// One gate/up item, staged in stage j % kStagesD (its full barrier already
// passed): this warp's partial sums, posted for the item's reducing warp;
// then, if this warp reduces item j - kRedLag, that item's sum and epilogue.
// Returns false when the kernel must wind down.
__device__ __forceinline__ bool gateup_item(const Ctx& x, int item, int j,
                                            const uint32_t (&breg)[kMaxGW][8],
                                            const int (&coff)[kMaxGW], int g_lo, int& pending,
                                            int& pending_at) {
    const int slot = item / x.gu_tiles;
    const Layout& L = x.L;
    const int lane = threadIdx.x & 31, r = lane >> 2, c = lane & 3;
    const int stage = j % kStagesD;
    const SlotEntry* en = x.S.table + slot;
    const bool valid = en->e >= 0;

    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const uint32_t st = smem_addr(x.S.stage0) + stage * L.stage_bytes;
    if (valid) {
        const uint32_t scA = st + 2 * L.gu_op + r * L.gsr;
        const uint32_t scB = scA + L.gu_sc;
        const uint32_t cor = smem_addr(x.S.corr) + c * 16;
        const Magic mg = magic();
        // kChains independent MMA chains at a time.  A group past the end of
        // H (the last warp's) has a zero B fragment, a zero offset sum and a
        // zero scale, and reads real staged codes.
        constexpr int kChains = 2;
        static_assert(kMaxGW % kChains == 0, "whole chain sets");
#pragma unroll
        for (int i0 = 0; i0 < kMaxGW; i0 += kChains) {
            uint2 wa[kChains], wb[kChains];
            float part[kChains][4], fa[kChains], fb[kChains];
#pragma unroll
            for (int u = 0; u < kChains; ++u) {
                const int i = i0 + u, grp = g_lo + i;
                wa[u] = lds_u2(st + coff[i]);
                wb[u] = lds_u2(st + L.gu_op + coff[i]);
                const float4 cr = lds_f4(cor + grp * 64);
                part[u][0] = cr.x;
                part[u][1] = cr.y;
                part[u][2] = cr.z;
                part[u][3] = cr.w;
                fa[u] = __uint_as_float(lds_u16(scA + grp * L.gsg) << 16);
                fb[u] = __uint_as_float(lds_u16(scB + grp * L.gsg) << 16);
            }
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {  // k16 steps of the group
                uint32_t ae[kChains], ao[kChains], be[kChains], bo[kChains];
#pragma unroll
                for (int u = 0; u < kChains; ++u) {
                    unpack_raw_step((ks >> 1) ? wa[u].y : wa[u].x, ks & 1, ae[u], ao[u], mg);
                    unpack_raw_step((ks >> 1) ? wb[u].y : wb[u].x, ks & 1, be[u], bo[u], mg);
                }
#pragma unroll
                for (int u = 0; u < kChains; ++u)
                    mma16816(part[u], part[u], ae[u], be[u], ao[u], bo[u],
                             breg[i0 + u][2 * ks], breg[i0 + u][2 * ks + 1]);
            }
#pragma unroll
            for (int u = 0; u < kChains; ++u) {
                acc[0] = fmaf(fa[u], part[u][0], acc[0]);
                acc[1] = fmaf(fa[u], part[u][1], acc[1]);
                acc[2] = fmaf(fb[u], part[u][2], acc[2]);
                acc[3] = fmaf(fb[u], part[u][3], acc[3]);
            }
        }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&x.S.empty[stage]);

    if (!post_partial(x, j, item, acc)) {
        fail(x, lane);
        return false;
    }
    const int m = j - kRedLag;
    if (m >= 0 && m % kCW == (int)(threadIdx.x >> 5))
        return finish_item(x, m, pending, pending_at, j);
    return true;
}

// h' fragments of one slot for this warp's down groups (columns = tokens;
// zero where a token is not on the slot's list or the group is past I).
__device__ __forceinline__ void load_down_b(const FfnArgs& a, const SlotEntry* en, int g_lo,
                                            uint32_t (&bdn)[kMaxDW][8]) {
    const int g_hi = a.I / kGroup;
    const int lane = threadIdx.x & 31, r = lane >> 2, c = lane & 3;
    const int p = (r < a.T && en->e >= 0) ? en->pos[r] : -1;
    const __half* row = a.hp + (int64_t)(en->list_begin + (p < 0 ? 0 : p)) * a.I;
#pragma unroll
    for (int i = 0; i < kMaxDW; ++i) {
        const int grp = g_lo + i;
        if (p >= 0 && grp < g_hi) {
            load_b_cg(bdn[i], row + grp * kGroup + c * 16);
        } else {
#pragma unroll
            for (int q = 0; q < 8; ++q) bdn[i][q] = 0u;
        }
    }
}

// Wait until slot `need` is below the frontier the producer warp publishes
// (every lane acquires it, so its later h' reads of those slots see the
// writers' stores).  Warp-uniform; bounded; false on timeout or abort.
__device__ __forceinline__ bool wait_frontier(const Ctx& x, int need) {
    if (__all_sync(0xffffffffu, ld_acquire_cta(x.S.frontier) > need)) return true;
    const int lane = threadIdx.x & 31;
    const uint64_t t0 = global_timer_ns();
    for (;;) {
        __nanosleep(64);
        if (__all_sync(0xffffffffu, ld_acquire_cta(x.S.frontier) > need)) return true;
        int stop = 0;
        if (lane == 0) stop = *x.S.abort_flag ? 1 : global_timer_ns() - t0 > kWaitLimitNs ? 2 : 0;
        stop = __shfl_sync(0xffffffffu, stop, 0);
        if (stop == 2) fail(x, lane);
        if (stop) return false;
    }
}

// One down stage: this CTA's tiles of slot s's W_d, accumulated into acc.
// The codes are unpacked raw (1032 + q even, 1152 + 16 q odd, against h'
// whose odd elements are stored / 16); each group's MMA chain starts from
// dcorr, the negated offset sums of the slot's h' for this lane's columns.
__device__ __forceinline__ bool down_stage(const Ctx& x, int s, int j, int my_mt,
                                           const uint32_t (&bcur)[kMaxDW][8],
                                           const float (&dcorr)[kMaxDW][2],
                                           const int (&dcoff)[kMaxDW], int g_lo,
                                           float (&acc)[kMaxMT][4]) {
    const Layout& L = x.L;
    const int lane = threadIdx.x & 31, r = lane >> 2;
    if (*x.S.abort_flag) return false;
    const int stage = j % kStagesD, use = j / kStagesD;
    if (!mbar_wait(&x.S.full[stage], use & 1)) {
        fail(x, lane);
        return false;
    }
    const uint32_t st = smem_addr(x.S.stage0) + stage * L.stage_bytes;
    if (x.S.table[s].e >= 0) {
        const Magic mg = magic();
        // per group, the three tiles' MMA chains run interleaved.  A group past
        // the end of I has a zero B fragment and a zero scale (padding
        // column) and reads real staged codes, so it adds zero; a tile this
        // CTA does not own (m >= my_mt) computes on stale stage bytes into an
        // accumulator that is never read.  Row r + 8 of a tile sits 8 staged
        // rows after row r.
        const int row8 = 8 * L.dn_segs * 128;
        const uint32_t sc0 = st + kMaxMT * L.dn_op + r * L.dsr;
#pragma unroll
        for (int i = 0; i < kMaxDW; ++i) {
            const int gs = g_lo + i;
            uint2 wa[kMaxMT], wb[kMaxMT];
            float part[kMaxMT][4];
#pragma unroll
            for (int m = 0; m < kMaxMT; ++m) {
                const uint32_t codes = st + m * L.dn_op + dcoff[i];
                wa[m] = lds_u2(codes);
                wb[m] = lds_u2(codes + row8);
                part[m][0] = dcorr[i][0];
                part[m][1] = dcorr[i][1];
                part[m][2] = dcorr[i][0];
                part[m][3] = dcorr[i][1];
            }
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                uint32_t ae[kMaxMT], ao[kMaxMT], be[kMaxMT], bo[kMaxMT];
#pragma unroll
                for (int m = 0; m < kMaxMT; ++m) {
                    unpack_raw_step((ks >> 1) ? wa[m].y : wa[m].x, ks & 1, ae[m], ao[m], mg);
                    unpack_raw_step((ks >> 1) ? wb[m].y : wb[m].x, ks & 1, be[m], bo[m], mg);
                }
#pragma unroll
                for (int m = 0; m < kMaxMT; ++m)
                    mma16816(part[m], part[m], ae[m], be[m], ao[m], bo[m], bcur[i][2 * ks],
                             bcur[i][2 * ks + 1]);
            }
#pragma unroll
            for (int m = 0; m < kMaxMT; ++m) {
                const uint32_t sc = sc0 + m * L.dn_sc + gs * L.dsg;
                const float fa = __uint_as_float(lds_u16(sc) << 16);
                const float fb = __uint_as_float(lds_u16(sc + 8 * L.dsr) << 16);
                acc[m][0] = fmaf(fa, part[m][0], acc[m][0]);
                acc[m][1] = fmaf(fa, part[m][1], acc[m][1]);
                acc[m][2] = fmaf(fb, part[m][2], acc[m][2]);
                acc[m][3] = fmaf(fb, part[m][3], acc[m][3]);
            }
        }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&x.S.empty[stage]);
    return true;
}

// NV: logits per routing lane.  HC, IC, PR > 0 (PR >= 0): the layer's H, I
// and scale format fixed at compile time (the GLM-5.2 shape), so every stride
// of the shared-memory layout is a constant and the address arithmetic of the
// inner loops folds into immediates; 0 (and PR = -1): taken from the call.
template <int NV, int HC, int IC, int PR>
__global__ void __launch_bounds__(kThreadsD, 1) decode_fused_kernel(const DecodeArgs d0) {
    DecodeArgs d = d0;
    if constexpr (HC > 0) {
        d.f.H = HC;
        d.f.I = IC;
    }
    if constexpr (PR >= 0) d.f.per_row = PR;
    const FfnArgs& a = d.f;
    const Layout L = make_layout(a.H, a.I, d.max_slots, a.per_row);
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned start, by pointer arithmetic on the shared array (so
    // the compiler keeps it a shared-memory pointer)
    uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    const Smem S = carve(smem, L, d.max_slots);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStagesD; ++s) {
            mbar_init(&S.full[s], 1);
            mbar_init(&S.empty[s], kCW);
        }
        for (int b = 0; b < kRedBufs; ++b) {
            mbar_init(&S.red_empty[b], 1);
            S.red_cnt[b] = 0;
        }
        mbar_init(S.tbl_ready, 1);
        mbar_init(S.routed, a.T > 0 ? a.T : 1);

        *S.abort_flag = 0;
        *S.frontier = 0;
    }
    if (threadIdx.x == 0) {
        fence_barrier_init();
    }
    __syncthreads();
    pdl_launch_dependents();

    const int G = gridDim.x, b = blockIdx.x;
    const int gu_tiles = a.I / kGuRows;
    const int n_gu_shared = a.n_shared * gu_tiles;
    const int n_mt = a.H / kDnRows;
    const int bm = G - 1 - b;  // this CTA's down tiles: bm, bm + G, ...
    const int my_mt = bm < n_mt ? (n_mt - 1 - bm) / G + 1 : 0;
    constexpr unsigned kAll = 0xffffffffu;

    if (warp == kCW) {
        // ---------------------------- producer warp ----------------------------
        // Control flow is warp-uniform; lane 0 arms the barriers and issues
        // the copies, the whole warp routes and polls the slot counters.
        const uint64_t policy = policy_evict_first();
        // the shared experts' slots need no routing: written before the
        // first stage is armed, so a consumer that sees a staged item of
        // theirs also sees their entries
        table_shared(a, S, lane);
        __syncwarp();
        int n_slots = -1;
        int j = 0;
        bool stop = false;
        bool pdl_done = false;
        int frontier = 0;       // slots [0, frontier) complete GPU-wide
        bool poll = false;  // the frontier matters once this CTA's gate/up items are out
        auto abort_set = [&]() -> bool { return __shfl_sync(kAll, (int)*S.abort_flag, 0) != 0; };
        auto give_up = [&]() {
            if (lane == 0) {
                report(a.status, COLI_ERR_TIMEOUT);
                *S.abort_flag = 1;
            }
            __syncwarp();
        };
        // For this CTA's down phase, the frontier of complete slots (their
        // counters, published by the consumer warps that finished the
        // tiles): the lanes read 32 slot counters at once with acquire
        // loads, and lane 0 publishes the new frontier in shared memory with
        // a release store.  Runs whenever the producer would otherwise wait,
        // once the gate/up items are out.
        auto pump = [&]() {
            if (!poll || n_slots < 0 || frontier >= n_slots || my_mt == 0) return;
            const int sl = frontier + lane;
            const bool ready = sl >= n_slots || S.table[sl].e < 0 ||
                               ld_acquire_gpu(d.sync + kSyncSlots + sl) >= gu_tiles;
            const unsigned done = __ballot_sync(kAll, ready);
            const int adv = done == kAll ? 32 : __ffs(~done) - 1;
            if (adv > 0) {
                frontier = min(frontier + adv, n_slots);
                __syncwarp();
                if (lane == 0) st_release_cta(S.frontier, frontier);
            }
        };
        auto next_stage = [&](uint8_t*& st) -> bool {
            const int stage = j % kStagesD, use = j / kStagesD;
            if (use > 0) {
                const uint32_t par = (use - 1) & 1;
                int ok = lane == 0 ? (int)mbar_test_wait(&S.empty[stage], par) : 0;
                if (!__shfl_sync(kAll, ok, 0)) {
                    const uint64_t t0 = global_timer_ns();
                    for (;;) {
                        pump();
                        ok = lane == 0 ? (int)mbar_try_wait_sleep(&S.empty[stage], par, 400u) : 0;
                        if (__shfl_sync(kAll, ok, 0)) break;
                        int late = lane == 0 && global_timer_ns() - t0 > kWaitLimitNs;
                        if (__shfl_sync(kAll, late, 0)) {
                            give_up();
                            return false;
                        }
                    }
                }
            }
            st = S.stage0 + (size_t)stage * L.stage_bytes;
            return true;
        };
        // The table of the routed slots, from the consumers' routing (or the
        // given union); the consumers wait for tbl_ready before their first
        // routed item.  The union may come from the previous kernel.
        auto build_table = [&]() -> bool {
            if (!pdl_done) {
                pdl_wait();
                pdl_done = true;
            }
            if (d.logits) {
                int ok = lane == 0 ? (int)mbar_wait(S.routed, 0) : 0;
                __syncwarp();
                if (!__shfl_sync(kAll, ok, 0)) {
                    give_up();
                    return false;
                }
                table_from_logits(d, S, lane);
            } else {
                table_from_union(d, S, lane);
            }
            n_slots = *S.n_slots;
            __threadfence_block();
            __syncwarp();
            if (lane == 0) mbar_arrive(S.tbl_ready);
            return true;
        };

        // gate/up: item b first, then items handed out by a counter (after
        // the previous grid has finished and zeroed it), so faster CTAs take
        // more.  The table is built before the first item that needs it, or
        // once every stage is armed.  A CTA with one more down tile
        // than others stops taking items R before the end, R = the extra
        // down work in items.
        int* item_ctr = d.sync + kSyncItems;
        int cur = b;
        int last_taken = INT_MAX;  // set once the table is known
        for (;;) {
            if (abort_set()) {
                stop = true;
                break;
            }
            if (n_slots < 0 && (cur >= n_gu_shared || j >= kStagesD) && !build_table()) {
                stop = true;
                break;
            }
            uint8_t* st;
            if (!next_stage(st)) {
                stop = true;
                break;
            }
            if (n_slots >= 0 && last_taken == INT_MAX) {
                const int t_hi = (n_mt + G - 1) / G;
                const int n_hi = n_mt - (t_hi - 1) * G;
                const int lo = G - n_hi;
                const float extra =
                    (float)lo * n_slots * (float)(L.dn_op + L.dn_sc) / (float)L.gu_tx;
                last_taken = n_slots * gu_tiles - ((my_mt == t_hi && lo > 0) ? (int)extra : 0);
            }
            if (n_slots >= 0 && cur >= n_slots * gu_tiles) break;  // stage j stays free
            // the next item first: its round trip to the counter also lets the
            // consumers' first loads (logits, activations) reach memory ahead
            // of the copies' burst
            int nxt = INT_MAX;
            if (cur < last_taken) {
                if (!pdl_done) {
                    pdl_wait();
                    pdl_done = true;
                }
                if (lane == 0) nxt = G + atomicAdd(item_ctr, 1);
                nxt = __shfl_sync(kAll, nxt, 0);
            }
            const int stage = j % kStagesD;
            uint64_t* bar = &S.full[stage];
            const int item = cur;
            ++j;
            if (lane == 0) {
                S.stage_item[stage] = item;
                if (item != a.withhold_item) {  // test hook: this stage never fills
                    const int slot = item / gu_tiles, tile = item - slot * gu_tiles;
                    const int e = S.table[slot].e;
                    if (e < 0) {
                        mbar_arrive(bar);
                    } else {
                        const CUtensorMap* maps = d.maps + (size_t)e * kMaps;
                        const int n0 = tile * kGuRows;
                        mbar_arrive_expect_tx(bar, L.gu_tx);
                        tma_load_3d(st, maps + 0, 0, 0, n0, bar, policy);
                        tma_load_3d(st + L.gu_op, maps + 1, 0, 0, n0, bar, policy);
                        if (a.per_row) {  // 8 rows' scales: 16 contiguous bytes per matrix
                            const DevExpert& ex = a.experts[e];
                            bulk_g2s_evict_first(st + 2 * L.gu_op, ex.gate_s + n0, L.gu_sc, bar,
                                                 policy);
                            bulk_g2s_evict_first(st + 2 * L.gu_op + L.gu_sc, ex.up_s + n0, L.gu_sc,
                                                 bar, policy);
                        } else {
                            tma_load_2d(st + 2 * L.gu_op, maps + 3, 0, n0, bar, policy);
                            tma_load_2d(st + 2 * L.gu_op + L.gu_sc, maps + 4, 0, n0, bar, policy);
                        }
                    }
                }
            }
            cur = nxt;
        }
        // down stages carry item -1, which tells the consumers that gate/up
        // is over; without down work a single empty stage does
        poll = true;
        if (!stop) {
            if (my_mt == 0) {
                if (lane == 0) {
                    S.stage_item[j % kStagesD] = -1;
                    mbar_arrive(&S.full[j % kStagesD]);
                }
                ++j;
            }
            for (int s = 0; s < n_slots && my_mt > 0; ++s) {
                uint8_t* st;
                if (abort_set() || !next_stage(st)) break;
                const int stage = j % kStagesD;
                uint64_t* bar = &S.full[stage];
                ++j;
                if (lane == 0) {
                    S.stage_item[stage] = -1;
                    const int e = S.table[s].e;
                    if (e < 0) {
                        mbar_arrive(bar);
                    } else {
                        const CUtensorMap* maps = d.maps + (size_t)e * kMaps;
                        mbar_arrive_expect_tx(bar, my_mt * (L.dn_op + L.dn_sc));
                        for (int m = 0; m < my_mt; ++m) {
                            const int m0 = (bm + m * G) * kDnRows;
                            tma_load_3d(st + m * L.dn_op, maps + 2, 0, 0, m0, bar, policy);
                            if (a.per_row)  // 16 rows' scales: 32 contiguous bytes
                                bulk_g2s_evict_first(st + kMaxMT * L.dn_op + m * L.dn_sc,
                                                     a.experts[e].down_s + m0, L.dn_sc, bar,
                                                     policy);
                            else
                                tma_load_2d(st + kMaxMT * L.dn_op + m * L.dn_sc, maps + 5, 0, m0,
                                            bar, policy);
                        }
                    }
                }
            }
            // follow the frontier to the last slot
            const uint64_t t0 = global_timer_ns();
            for (;;) {
                pump();
                const bool fin = frontier >= n_slots || my_mt == 0;
                if (fin || abort_set()) break;
                int late = lane == 0 && global_timer_ns() - t0 > kWaitLimitNs;
                if (__shfl_sync(kAll, late, 0)) {
                    give_up();
                    break;
                }
                __nanosleep(200);
            }
        }
        if (abort_set() && lane == 0) {
            // let the copies already issued land before the CTA goes away
            for (int back = 1; back <= kStagesD && back <= j; ++back) {
                const int jj = j - back;
                (void)mbar_wait(&S.full[jj % kStagesD], (jj / kStagesD) & 1);
            }
        }
        return;
    }

    // -------------------------------- consumers --------------------------------
    pdl_wait();
    const int r = lane >> 2, c = lane & 3;

    // gate/up operand: all T tokens as MMA columns, this warp's kMaxGW
    // groups, in registers for the whole kernel; offset sums to shared memory
    // (zero for the groups past the end of H), read by this warp only
    const int gG = a.H / kGroup;
    const int gg_lo = kMaxGW * warp;
    uint32_t breg[kMaxGW][8];
    int coff[kMaxGW];
    float amax = 0.f;
    // all loads first (they are in flight together), then the routing (warp
    // t < T routes token t) and the conversions
    const bool routing = d.logits && warp < a.T;
    float lv[8];
    if (routing && route_fast_ok<NV>(a.k)) load_row8<NV>(d.logits + (int64_t)warp * a.E, a.E, lane, lv);
#pragma unroll
    for (int i = 0; i < kMaxGW; ++i) {
        const int grp = gg_lo + i;
        uint4 v0 = make_uint4(0u, 0u, 0u, 0u), v1 = v0;
        if (grp < gG && r < a.T) {
            const uint4* src = reinterpret_cast<const uint4*>(
                reinterpret_cast<const uint16_t*>(a.x) + (int64_t)r * a.H + grp * kGroup + c * 16);
            v0 = __ldg(src);
            v1 = __ldg(src + 1);
        }
        breg[i][0] = v0.x; breg[i][1] = v0.y; breg[i][2] = v0.z; breg[i][3] = v0.w;
        breg[i][4] = v1.x; breg[i][5] = v1.y; breg[i][6] = v1.z; breg[i][7] = v1.w;
    }
    if (routing) {
        if (route_fast_ok<NV>(a.k))
            route_row_fast<NV>(lv, a.E, a.k, lane, S.s_idx + warp * a.k, S.s_w + warp * a.k);
        else
            route_row<NV>(d.logits + (int64_t)warp * a.E, a.E, a.k, lane, S.s_idx + warp * a.k,
                          S.s_w + warp * a.k);
        __syncwarp();
        if (lane == 0) mbar_arrive(S.routed);
    }
#pragma unroll
    for (int i = 0; i < kMaxGW; ++i) {
        const int grp = gg_lo + i;
        coff[i] = code_offset(r, L.gu_segs, grp < gG ? grp : gG - 1, c);
        x_fragment(breg[i], amax);
        float cs[4];
        offset_sums(breg[i], cs);
        if (r == 0)  // stored negated, as the MMA's initial C fragment of lane c
            reinterpret_cast<float4*>(S.corr)[grp * 4 + c] = make_float4(-cs[0], -cs[1], -cs[0], -cs[1]);
    }
    if (amax > 65504.f) report(a.status, COLI_ERR_RANGE);
    __syncwarp();
    const Ctx ctx{a, L, S, d.sync, gu_tiles};
    bool have_table = false;
    auto wait_table = [&]() -> bool {
        if (have_table) return true;
        if (!mbar_wait(S.tbl_ready, 0)) {
            fail(ctx, lane);
            return false;
        }
        have_table = true;
        return true;
    };

    // phase 1: gate/up items (the shared experts' first: they need no table)
    int j = 0;
    bool alive = true;
    int pending = -1;  // the slot of the last tile this warp finished, not yet published
    int pending_at = 0;  // the item this warp was at when it stored that tile
    for (;;) {  // the producer names each stage's item; -1 ends gate/up
        const int stage = j % kStagesD;
        if (*S.abort_flag) {
            alive = false;
            break;
        }
        if (!mbar_wait(&S.full[stage], (j / kStagesD) & 1)) {
            fail(ctx, lane);
            alive = false;
            break;
        }
        const int item = S.stage_item[stage];
        if (item < 0) break;
        if (item >= n_gu_shared && !wait_table()) {
            alive = false;
            break;
        }
        // a tile stored two items ago goes out now (its stores are complete)
        if (pending >= 0 && j >= pending_at + 2) {
            publish_tile(ctx, pending);
            pending = -1;
        }
        alive = gateup_item(ctx, item, j, breg, coff, gg_lo, pending, pending_at);
        ++j;
        if (!alive) break;
    }
    // the sums of the last kRedLag items
    for (int m = j - kRedLag; alive && m < j; ++m)
        if (m >= 0 && m % kCW == warp) alive = finish_item(ctx, m, pending, pending_at, j);
    if (alive) publish_tile(ctx, pending);
    if (alive) alive = wait_table();
    const int n_slots = alive ? *S.n_slots : 0;

    // phase 2: down + combine over this CTA's output tiles, slot by slot;
    // h' fragments of the next slot are loaded while this one is computed
    const int dG = a.I / kGroup;
    const int dg_lo = kMaxDW * warp;
    float acc[kMaxMT][4];
#pragma unroll
    for (int m = 0; m < kMaxMT; ++m)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[m][q] = 0.f;
    if (alive && my_mt > 0 && n_slots > 0) {
        int dcoff[kMaxDW];
#pragma unroll
        for (int i = 0; i < kMaxDW; ++i)
            dcoff[i] = code_offset(r, L.dn_segs, dg_lo + i < dG ? dg_lo + i : dG - 1, c);
        // h' fragments: b0 = this slot, b1 = the next one (loading)
        uint32_t b0[kMaxDW][8], b1[kMaxDW][8];
        alive = wait_frontier(ctx, 0);
        if (alive) load_down_b(a, S.table + 0, dg_lo, b1);
        float dcorr[kMaxDW][2];
        for (int s = 0; s < n_slots && alive; ++s, ++j) {
#pragma unroll
            for (int i = 0; i < kMaxDW; ++i) {
#pragma unroll
                for (int q = 0; q < 8; ++q) b0[i][q] = b1[i][q];
                float cs[4];
                offset_sums(b0[i], cs);  // zero fragments (absent tokens, groups past I) give 0
                dcorr[i][0] = -cs[0];
                dcorr[i][1] = -cs[1];
            }
            if (s + 1 < n_slots) {
                alive = wait_frontier(ctx, s + 1);
                if (alive) load_down_b(a, S.table + s + 1, dg_lo, b1);
            }
            if (alive) alive = down_stage(ctx, s, j, my_mt, b0, dcorr, dcoff, dg_lo, acc);
        }
    }

    // final: sum the warps' partials in a fixed order, add the residual
    consumers_sync();  // every gate/up reduction is done with the buffers
    if (my_mt > 0) {
#pragma unroll
        for (int m = 0; m < kMaxMT; ++m)
            if (m < my_mt)
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    S.red[((warp * kMaxMT + m) * 4 + q) * 32 + lane] = acc[m][q];
    }
    consumers_sync();
    if (my_mt > 0 && !*S.abort_flag) {
        const int per_t = my_mt * kDnRows;
        for (int o = threadIdx.x; o < a.T * per_t; o += kConsumerThreads) {
            const int t = o / per_t, rem = o - t * per_t;
            const int m = rem / kDnRows, row = rem - m * kDnRows;
            const int src_lane = (row & 7) * 4 + (t >> 1);
            const int q = (row >> 3) * 2 + (t & 1);
            float y = 0.f;
#pragma unroll
            for (int w = 0; w < kCW; ++w) y += S.red[((w * kMaxMT + m) * 4 + q) * 32 + src_lane];
            const int64_t oi = (int64_t)t * a.H + (bm + m * G) * kDnRows + row;
            if (a.out_bf16) {
                if (a.residual)
                    y += __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(a.residual)[oi]);
                reinterpret_cast<__nv_bfloat16*>(a.out)[oi] = __float2bfloat16_rn(y);
            } else {
                if (a.residual) y += reinterpret_cast<const float*>(a.residual)[oi];
                reinterpret_cast<float*>(a.out)[oi] = y;
            }
        }
    }
    // the last CTA to get here returns the counters to zero (every slot a
    // call can have: a CTA that gave up may not know the table)
    if (threadIdx.x == 0) {
        fence_acq_rel_gpu();
        if (atomicAdd(d.sync + kSyncDone, 1) == G - 1) {
            fence_acq_rel_gpu();
            for (int s = 0; s < d.max_slots; ++s) d.sync[kSyncSlots + s] = 0;
            d.sync[kSyncItems] = 0;
            d.sync[kSyncDone] = 0;
        }
    }
}

// False once the runtime refused the cooperative launch together with
// programmatic dependent launch; later launches are cooperative only.
bool g_coop_with_pdl = true;

// A cooperative launch: the runtime starts it only if every CTA of the grid
// can be resident at once (cudaErrorCooperativeLaunchTooLarge otherwise),
// which the CTAs' waits on one another need.
template <int NV, int HC = 0, int IC = 0, int PR = -1>
cudaError_t launch_nv(const DecodeArgs& d, int blocks, int smem, cudaStream_t st) {
    auto kern = decode_fused_kernel<NV, HC, IC, PR>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(blocks);
    cfg.blockDim = dim3(kThreadsD);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = g_coop_with_pdl ? 2 : 1;
    err = cudaLaunchKernelEx(&cfg, kern, d);
    if (err != cudaSuccess && err != cudaErrorCooperativeLaunchTooLarge && g_coop_with_pdl) {
        cudaGetLastError();  // a refused configuration launched nothing
        g_coop_with_pdl = false;
        cfg.numAttrs = 1;
        err = cudaLaunchKernelEx(&cfg, kern, d);
    }
    return err;
}

// Resident CTAs of the kernel instance per SM at `smem` bytes of shared memory.
template <int NV, int HC = 0, int IC = 0, int PR = -1>
int resident_per_sm(int smem) {
    auto kern = decode_fused_kernel<NV, HC, IC, PR>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return 0;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kThreadsD, smem) != cudaSuccess)
        return 0;
    return n;
}

// The shape with a compile-time instance: GLM-5.2 (H 6144, I 2048), gs64.
constexpr int kFixH = 6144, kFixI = 2048;
bool fixed_shape(int H, int I, int per_row) { return H == kFixH && I == kFixI && !per_row; }

int max_slots_for(int E, int k, int T, int n_shared) {
    return std::min(E, T * k) + n_shared;
}

// Template instance for E routed experts (logits per routing lane).
int nv_for(int E) {
    const int nv = (E + 31) / 32;
    return nv <= 1 ? 1 : nv <= 2 ? 2 : nv <= 4 ? 4 : nv <= 8 ? 8 : nv <= 16 ? 16 : 32;
}

bool g_force_not_resident = false;  // test hook (coli_moe_debug_inject)

}  // namespace

bool decode_supported(int H, int I, int T, int E, int k, int n_shared, int num_sms) {
    if (T < 1 || T > 8 || T * k > kMaxPairs || H % 512 || I % 512 || num_sms < 1) return false;
    // the slot counters live between the two counter offsets of the header
    const int counters = (int)((kTileCntOffset - kSlotCntOffset) / 4);
    if (kSyncSlots + max_slots_for(E, k, T, n_shared) > counters) return false;
    const Layout L = make_layout(H, I, max_slots_for(E, k, T, n_shared), 0);
    if (L.smem > kSmemLimitD) return false;
    if (H / kGroup > kCW * kMaxGW || I / kGroup > kCW * kMaxDW) return false;
    if (T * E > 5632) return false;  // the routing shapes the kernel is tested with
    if (H / kDnRows > kMaxMT * num_sms) return false;
    return L.gu_segs <= 256 && L.dn_segs <= 256 && L.gGp <= 256 && L.dGp <= 256;
}

cudaError_t build_decode_maps(const DevExpert* host_experts, int n, int H, int I, int per_row,
                              CUtensorMap** d_maps) {
    *d_maps = nullptr;
    const Layout L = make_layout(H, I, 0, 0);
    CUtensorMap* maps = new (std::nothrow) CUtensorMap[(size_t)n * kMaps];
    if (!maps) return cudaErrorMemoryAllocation;
    bool ok = true;
    const int gG = H / kGroup, dG = I / kGroup;
    for (int e = 0; e < n && ok; ++e) {
        const DevExpert& x = host_experts[e];
        CUtensorMap* m = maps + (size_t)e * kMaps;
        // per-row scales are copied with 1-D bulk copies (their rows are 2
        // bytes, below a tensor map's 16-byte stride): no scale maps
        ok = encode_tma(&m[0], x.gate_q, 3, I, H / 2, L.gu_segs, kGuRows) &&
             encode_tma(&m[1], x.up_q, 3, I, H / 2, L.gu_segs, kGuRows) &&
             encode_tma(&m[2], x.down_q, 3, H, I / 2, L.dn_segs, kDnRows) &&
             (per_row || (encode_tma_rows_u16(&m[3], x.gate_s, I, gG, L.gGp, kGuRows) &&
                          encode_tma_rows_u16(&m[4], x.up_s, I, gG, L.gGp, kGuRows) &&
                          encode_tma_rows_u16(&m[5], x.down_s, H, dG, L.dGp, kDnRows)));
    }
    if (!ok) {
        delete[] maps;
        return cudaErrorInvalidValue;
    }
    cudaError_t err = cudaMalloc(d_maps, sizeof(CUtensorMap) * (size_t)n * kMaps);
    if (err == cudaSuccess)
        err = cudaMemcpy(*d_maps, maps, sizeof(CUtensorMap) * (size_t)n * kMaps,
                         cudaMemcpyHostToDevice);
    delete[] maps;
    if (err != cudaSuccess && *d_maps) {
        cudaFree(*d_maps);
        *d_maps = nullptr;
    }
    return err;
}

bool decode_coresident(int H, int I, int E, int k, int n_shared, int num_sms) {
    // the largest shared-memory footprint (8 tokens) of either template
    // instance a handle can launch (routing from logits, or a given union)
    const Layout L = make_layout(H, I, max_slots_for(E, k, 8, n_shared), 0);
    int per_sm = resident_per_sm<1>(L.smem);
    if (fixed_shape(H, I, 0))
        per_sm = std::min(per_sm, std::min(resident_per_sm<1, kFixH, kFixI, 0>(L.smem),
                                           resident_per_sm<8, kFixH, kFixI, 0>(L.smem)));
    switch (nv_for(E)) {
        case 1: per_sm = std::min(per_sm, resident_per_sm<1>(L.smem)); break;
        case 2: per_sm = std::min(per_sm, resident_per_sm<2>(L.smem)); break;
        case 4: per_sm = std::min(per_sm, resident_per_sm<4>(L.smem)); break;
        case 8: per_sm = std::min(per_sm, resident_per_sm<8>(L.smem)); break;
        case 16: per_sm = std::min(per_sm, resident_per_sm<16>(L.smem)); break;
        default: per_sm = std::min(per_sm, resident_per_sm<32>(L.smem)); break;
    }
    cudaGetLastError();
    return per_sm >= 1 && num_sms >= 1;
}

void decode_force_not_resident(bool on) { g_force_not_resident = on; }

cudaError_t launch_decode_fused(const DecodeArgs& d0, int num_sms, cudaStream_t st) {
    DecodeArgs d = d0;
    if (g_force_not_resident) {  // test hook: behave as if the launch were refused
        g_force_not_resident = false;
        return cudaErrorCooperativeLaunchTooLarge;
    }
    d.max_slots = max_slots_for(d.f.E, d.f.k, d.f.T, d.f.n_shared);
    const Layout L = make_layout(d.f.H, d.f.I, d.max_slots, d.f.per_row);
    const int blocks = num_sms;  // persistent: one CTA per SM, all resident
    d.f.withhold_item = take_withhold_item();
    profile_mark(1, st);
    cudaError_t err;
    const bool fixed = fixed_shape(d.f.H, d.f.I, d.f.per_row);
    switch (d.logits ? nv_for(d.f.E) : 1) {
        case 1:
            err = fixed ? launch_nv<1, kFixH, kFixI, 0>(d, blocks, L.smem, st)
                        : launch_nv<1>(d, blocks, L.smem, st);
            break;
        case 2: err = launch_nv<2>(d, blocks, L.smem, st); break;
        case 4: err = launch_nv<4>(d, blocks, L.smem, st); break;
        case 8:
            err = fixed ? launch_nv<8, kFixH, kFixI, 0>(d, blocks, L.smem, st)
                        : launch_nv<8>(d, blocks, L.smem, st);
            break;
        case 16: err = launch_nv<16>(d, blocks, L.smem, st); break;
        default: err = launch_nv<32>(d, blocks, L.smem, st); break;
    }
    if (err == cudaErrorCooperativeLaunchTooLarge) {
        cudaGetLastError();  // nothing was launched: the caller takes another path
        return err;
    }
    profile_mark(2, st);
    profile_mark(3, st);
    profile_mark(4, st);
    return err;
}

}  // namespace coli
