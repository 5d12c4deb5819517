// Host side of the C ABI declared in include/coli_moe.h: argument checks,
// workspace carving and kernel launches.  Every check runs before anything is
// enqueued, so a call that returns an error has launched nothing.
#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

#include "coli_internal.cuh"
#include "batch.cuh"
#include "decode.cuh"
#include "handle.cuh"
#include "prefill.cuh"

// Which kernels a call runs.  Up to 8 tokens with fewer routed pairs than
// experts (T*k < E), the fused decode kernel; by default every other call the
// tensor-core grouped GEMM.  Measured on the GLM-5.2 shape (Zipf routing):
// at T = 16 the streaming dequant-GEMV takes 1.35 ms per call, at T = 32
// 1.51 ms against the grouped GEMM's 1.10 ms, at T = 64 2.32 ms against
// 1.54 ms.  A positive prefill_min_tokens keeps the older rule (grouped GEMM
// from T*k >= prefill_min * E, streaming below it).

namespace {

using coli::kGroup;

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

coli_status check_route_dims(int32_t T, int32_t E, int32_t k) {
    if (T < 0) return COLI_ERR_INVALID_ARG;
    if (E < 1 || E > coli::kMaxExperts || k < 1 || k > E || k > coli::kMaxTopK)
        return COLI_ERR_SHAPE;
    if ((int64_t)T * k > (int64_t)1 << 24) return COLI_ERR_SHAPE;
    return COLI_OK;
}

coli_status from_cuda(cudaError_t e) { return e == cudaSuccess ? COLI_OK : COLI_ERR_CUDA; }

template <typename T>
T* at(void* ws, size_t off) {
    return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

coli::WsLayout layout_for(const coli_moe* h, int64_t T) {
    return coli::ws_layout(T, h->E, h->k, h->H, h->I, h->n_shared);
}

// Shared validation of the FFN-side arguments.
coli_status check_ffn_common(const coli_moe* h, int32_t T, const void* x, const void* residual,
                             const void* out, int out_dtype, const void* ws, size_t ws_bytes) {
    if (!h || T < 0) return COLI_ERR_INVALID_ARG;
    if (out_dtype != COLI_OUT_F32 && out_dtype != COLI_OUT_BF16) return COLI_ERR_INVALID_ARG;
    if ((int64_t)T * h->k > (int64_t)1 << 24) return COLI_ERR_SHAPE;
    if (T == 0) return COLI_OK;
    if (!x || !out || !ws) return COLI_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(out, 16) || (residual && !aligned(residual, 16)))
        return COLI_ERR_ALIGN;
    if (!aligned(ws, 256)) return COLI_ERR_ALIGN;
    if (ws_bytes < layout_for(h, T).total) return COLI_ERR_WORKSPACE;
    return COLI_OK;
}

coli::FfnArgs make_args(const coli_moe* h, int32_t T, const void* x, const float* w,
                        const int32_t* offsets, const int32_t* pairs, const int32_t* active,
                        const int32_t* n_active, const void* residual, void* out,
                        coli_out_dtype od, void* ws) {
    const coli::WsLayout L = layout_for(h, T);
    coli::FfnArgs a;
    a.experts = h->d_experts;
    a.H = h->H;
    a.I = h->I;
    a.E = h->E;
    a.k = h->k;
    a.n_shared = h->n_shared;
    a.T = T;
    a.offsets = offsets;
    a.pairs = pairs;
    a.active = active;
    a.n_active = n_active;
    a.topk_w = w;
    a.x = static_cast<const __nv_bfloat16*>(x);
    a.xp = at<__half>(ws, L.xp);
    a.corr = at<float>(ws, L.corr);
    a.inv = at<int>(ws, L.inv);
    a.hp = at<__half>(ws, L.hp);
    a.y = at<float>(ws, L.y);
    a.residual = residual;
    a.out = out;
    a.out_bf16 = od == COLI_OUT_BF16;
    a.per_row = h->per_row;
    a.status = at<int>(ws, 0);
    a.withhold_item = -1;
    return a;
}

// Timing diagnostics: one set of 5 events per recorded call.
struct ProfileState {
    bool enabled = false;
    std::vector<cudaEvent_t> events;  // 5 per call
    int open_call = -1;               // index of the call being recorded
};
ProfileState g_prof;
int g_withhold_item = -1;

void profile_begin_call(cudaStream_t st) {
    if (!g_prof.enabled) return;
    const size_t base = g_prof.events.size();
    for (int i = 0; i < 5; ++i) {
        cudaEvent_t ev = nullptr;
        if (cudaEventCreate(&ev) != cudaSuccess) {
            g_prof.open_call = -1;
            return;
        }
        g_prof.events.push_back(ev);
    }
    g_prof.open_call = (int)(base / 5);
    cudaEventRecord(g_prof.events[base], st);
}

void profile_end_call() { g_prof.open_call = -1; }

// True when the fused decode kernel can take a call with T tokens.
bool fused_ok(const coli_moe* h, int64_t T) {
    return h->d_dmaps != nullptr && T * h->k < h->E &&
           coli::decode_supported(h->H, h->I, (int)T, h->E, h->k, h->n_shared, h->num_sms);
}

// True when a call with T tokens runs the small-batch kernels (the default
// for calls of up to 64 tokens the fused decode kernel does not take).
bool use_batch(const coli_moe* h, int64_t T) {
    return h->d_bmaps != nullptr && h->prefill_min == 0 && !fused_ok(h, T) &&
           coli::batch_supported(h->H, h->I, (int)T);
}

// True when a call with T tokens runs the tensor-core grouped GEMM.
bool use_prefill(const coli_moe* h, int64_t T) {
    if (h->d_wmaps == nullptr) return false;
    if (h->prefill_min > 0) return T * h->k >= (int64_t)h->prefill_min * h->E;
    return !fused_ok(h, T) && !use_batch(h, T);
}

// True when a call with T tokens runs the fused decode kernel.
bool use_fused(const coli_moe* h, int64_t T) { return fused_ok(h, T) && !use_prefill(h, T); }

// The fused decode kernel: routing from `logits` (or the union in `a` when
// logits is null), gate/up, down and combine in one launch.
cudaError_t run_fused(const coli_moe* h, const coli::FfnArgs& a, const float* logits,
                      int32_t* idx_out, float* w_out, void* ws, cudaStream_t st) {
    coli::DecodeArgs d;
    d.f = a;
    d.maps = h->d_dmaps;
    d.logits = logits;
    d.idx_out = idx_out;
    d.w_out = w_out;
    d.sync = at<int>(ws, coli::kSlotCntOffset);
    d.max_slots = 0;  // set by the launcher
    return coli::launch_decode_fused(d, h->num_sms, st);
}

// The FFN of a call whose union lists (and inverse map) are ready: tensor-core
// grouped GEMM for prefill-sized batches, the fused decode kernel for up to
// 8 tokens, streaming GEMV otherwise (also when the fused kernel's grid
// cannot be resident at once).
// `x_prepared`: the fused prep kernel already built the GEMV operand of x.
cudaError_t run_ffn(const coli_moe* h, int32_t T, const coli::FfnArgs& a, void* ws,
                    cudaStream_t st, bool x_prepared) {
    const coli::WsLayout L = layout_for(h, T);
    cudaError_t err = cudaSuccess;
    if (use_prefill(h, T)) {
        err = coli::launch_prefill(a, h->d_wmaps, at<__half>(ws, L.xg), at<int>(ws, L.ntile),
                                   h->num_sms, st);
        if (err == cudaSuccess) err = coli::launch_combine(a, h->num_sms, st);
        coli::profile_mark(4, st);
        return err;
    }
    if (use_batch(h, T)) {
        if (!x_prepared) err = coli::launch_prepare_x(T, h->H, a.x, a.xp, a.corr, a.status, st);
        if (err == cudaSuccess) err = coli::launch_batch_ffn(a, h->d_bmaps, h->num_sms, st);
        if (err == cudaSuccess) err = coli::launch_combine(a, h->num_sms, st);
        coli::profile_mark(4, st);
        return err;
    }
    if (!x_prepared && use_fused(h, T)) {
        err = run_fused(h, a, nullptr, nullptr, nullptr, ws, st);
        if (err != cudaErrorCooperativeLaunchTooLarge) return err;
        err = cudaSuccess;  // not launched: stream instead
    }
    if (!x_prepared) err = coli::launch_prepare_x(T, h->H, a.x, a.xp, a.corr, a.status, st);
    if (err != cudaSuccess) return err;
    return coli::launch_ffn_stream(a, h->num_sms, st);
}

}  // namespace

namespace coli {
int take_withhold_item() {
    const int v = g_withhold_item;
    g_withhold_item = -1;
    return v;
}

cudaEvent_t profile_event(int i) {
    if (!g_prof.enabled || g_prof.open_call < 0 || i < 0 || i > 4) return nullptr;
    return g_prof.events[(size_t)g_prof.open_call * 5 + i];
}
}  // namespace coli

extern "C" {

coli_status coli_moe_debug_inject(int32_t what) {
    if (what == 0) {
        g_withhold_item = -1;
        coli::decode_force_not_resident(false);
        return COLI_OK;
    }
    if (what == COLI_INJECT_WITHHOLD_STAGE) {
        g_withhold_item = 0;  // the first item of CTA 0: a shared-expert gate/up tile
        return COLI_OK;
    }
    if (what == COLI_INJECT_NOT_RESIDENT) {
        coli::decode_force_not_resident(true);
        return COLI_OK;
    }
    return COLI_ERR_INVALID_ARG;
}

coli_status coli_moe_profile_enable(int32_t enable) {
    g_prof.enabled = enable != 0;
    g_prof.open_call = -1;
    return COLI_OK;
}

coli_status coli_moe_profile_read(double* ms, int32_t* n_calls) {
    if (!ms || !n_calls) return COLI_ERR_INVALID_ARG;
    for (int i = 0; i < 4; ++i) ms[i] = 0.0;
    const size_t calls = g_prof.events.size() / 5;
    coli_status st = COLI_OK;
    for (size_t c = 0; c < calls; ++c) {
        cudaEvent_t* ev = &g_prof.events[c * 5];
        if (cudaEventSynchronize(ev[4]) != cudaSuccess) st = COLI_ERR_CUDA;
        for (int i = 0; i < 4; ++i) {
            float t = 0.f;
            if (cudaEventElapsedTime(&t, ev[i], ev[i + 1]) == cudaSuccess) ms[i] += t;
            else st = COLI_ERR_CUDA;
        }
    }
    for (cudaEvent_t ev : g_prof.events) cudaEventDestroy(ev);
    g_prof.events.clear();
    g_prof.open_call = -1;
    *n_calls = (int32_t)calls;
    return st;
}

coli_status coli_moe_create(const coli_moe_desc* d, coli_moe** out) {
    if (!out) return COLI_ERR_INVALID_ARG;
    *out = nullptr;
    if (!d || !d->experts) return COLI_ERR_INVALID_ARG;
    if (d->group_size != kGroup && d->group_size != COLI_GROUP_PER_ROW) return COLI_ERR_SHAPE;
    if (d->hidden <= 0 || d->inter <= 0 || d->hidden % 128 || d->inter % 128) return COLI_ERR_SHAPE;
    if (d->n_routed < 1 || d->n_routed > coli::kMaxExperts) return COLI_ERR_SHAPE;
    if (d->top_k < 1 || d->top_k > d->n_routed || d->top_k > coli::kMaxTopK) return COLI_ERR_SHAPE;
    if (d->n_shared < 0 || d->n_shared > coli::kMaxShared) return COLI_ERR_SHAPE;
    if (d->prefill_min_tokens < 0) return COLI_ERR_INVALID_ARG;
    if (d->hidden > 12288 || d->inter > 12288 || !coli::stream_shapes_fit(d->hidden, d->inter))
        return COLI_ERR_SHAPE;
    const int n = d->n_routed + d->n_shared;
    for (int e = 0; e < n; ++e) {
        const coli_expert& x = d->experts[e];
        const void* ptrs[6] = {x.gate_q, x.up_q, x.down_q, x.gate_s, x.up_s, x.down_s};
        for (const void* p : ptrs) {
            if (!p) return COLI_ERR_INVALID_ARG;
            if (!aligned(p, 16)) return COLI_ERR_ALIGN;
        }
    }
    int dev = 0, major = 0, minor = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return COLI_ERR_CUDA;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return COLI_ERR_CUDA;
    if (major != 10 || minor != 0) return COLI_ERR_UNSUPPORTED;  // built for sm_100a only

    coli_moe* h = new (std::nothrow) coli_moe;
    if (!h) return COLI_ERR_INVALID_ARG;
    h->device = dev;
    h->H = d->hidden;
    h->I = d->inter;
    h->E = d->n_routed;
    h->k = d->top_k;
    h->n_shared = d->n_shared;
    h->prefill_min = d->prefill_min_tokens;
    h->per_row = d->group_size == COLI_GROUP_PER_ROW;
    h->num_sms = sms;
    h->d_experts = nullptr;
    h->d_wmaps = nullptr;
    h->d_bmaps = nullptr;
    h->d_dmaps = nullptr;
    coli::DevExpert* host = static_cast<coli::DevExpert*>(std::malloc(sizeof(coli::DevExpert) * n));
    if (!host) {
        delete h;
        return COLI_ERR_INVALID_ARG;
    }
    for (int e = 0; e < n; ++e) {
        host[e].gate_q = d->experts[e].gate_q;
        host[e].up_q = d->experts[e].up_q;
        host[e].down_q = d->experts[e].down_q;
        host[e].gate_s = d->experts[e].gate_s;
        host[e].up_s = d->experts[e].up_s;
        host[e].down_s = d->experts[e].down_s;
    }
    cudaError_t err = cudaMalloc(&h->d_experts, sizeof(coli::DevExpert) * n);
    if (err == cudaSuccess)
        err = cudaMemcpy(h->d_experts, host, sizeof(coli::DevExpert) * n, cudaMemcpyHostToDevice);
    if (err == cudaSuccess && coli::prefill_available())
        err = coli::build_weight_maps(host, n, h->H, h->I, &h->d_wmaps);
    if (err == cudaSuccess && h->d_wmaps)
        err = coli::build_batch_maps(host, n, h->H, h->I, h->per_row, &h->d_bmaps);
    // the fused decode kernel only where one CTA per SM can be resident at once
    if (err == cudaSuccess && h->d_wmaps &&
        coli::decode_supported(h->H, h->I, 1, h->E, h->k, h->n_shared, h->num_sms) &&
        coli::decode_coresident(h->H, h->I, h->E, h->k, h->n_shared, h->num_sms) &&
        coli::build_decode_maps(host, n, h->H, h->I, h->per_row, &h->d_dmaps) != cudaSuccess) {
        h->d_dmaps = nullptr;  // the fused decode path is an optimisation: go without it
        cudaGetLastError();
    }
    std::free(host);
    if (err != cudaSuccess) {
        if (h->d_experts) cudaFree(h->d_experts);
        if (h->d_wmaps) cudaFree(h->d_wmaps);
        if (h->d_bmaps) cudaFree(h->d_bmaps);
        if (h->d_dmaps) cudaFree(h->d_dmaps);
        delete h;
        return COLI_ERR_CUDA;
    }
    *out = h;
    return COLI_OK;
}

void coli_moe_destroy(coli_moe* h) {
    if (!h) return;
    cudaFree(h->d_experts);
    if (h->d_wmaps) cudaFree(h->d_wmaps);
    if (h->d_bmaps) cudaFree(h->d_bmaps);
    if (h->d_dmaps) cudaFree(h->d_dmaps);
    delete h;
}

size_t coli_moe_workspace_size(const coli_moe* h, int32_t max_tokens) {
    if (!h || max_tokens < 0) return 0;
    return layout_for(h, max_tokens).total;
}

coli_status coli_moe_workspace_clear(void* ws, size_t ws_bytes, void* stream) {
    if (!ws || ws_bytes < coli::kHeaderBytes) return COLI_ERR_INVALID_ARG;
    if (!aligned(ws, 256)) return COLI_ERR_ALIGN;
    return from_cuda(cudaMemsetAsync(ws, 0, coli::kHeaderBytes, static_cast<cudaStream_t>(stream)));
}

size_t coli_moe_union_workspace_size(int32_t T, int32_t E, int32_t k) {
    if (T < 0 || E < 1 || k < 1) return 0;
    return coli::kHeaderBytes + coli::union_scratch_bytes((int64_t)T * k, E);
}

coli_status coli_moe_route(int32_t T, int32_t E, int32_t k, const float* logits,
                           int32_t* topk_idx, float* topk_w, void* stream) {
    coli_status s = check_route_dims(T, E, k);
    if (s != COLI_OK || T == 0) return s;
    if (!logits || !topk_idx || !topk_w) return COLI_ERR_INVALID_ARG;
    if (!aligned(logits, 4) || !aligned(topk_idx, 4) || !aligned(topk_w, 4)) return COLI_ERR_ALIGN;
    return from_cuda(coli::launch_route(T, E, k, logits, topk_idx, topk_w,
                                        static_cast<cudaStream_t>(stream)));
}

coli_status coli_moe_union(int32_t T, int32_t E, int32_t k, const int32_t* topk_idx,
                           int32_t* counts, int32_t* offsets, int32_t* pairs, int32_t* active,
                           int32_t* n_active, void* ws, size_t ws_bytes, void* stream) {
    coli_status s = check_route_dims(T, E, k);
    if (s != COLI_OK) return s;
    if (!counts || !offsets || !active || !n_active) return COLI_ERR_INVALID_ARG;
    if (T > 0 && (!topk_idx || !pairs)) return COLI_ERR_INVALID_ARG;
    const void* ptrs[6] = {topk_idx, counts, offsets, pairs, active, n_active};
    for (const void* p : ptrs)
        if (p && !aligned(p, 4)) return COLI_ERR_ALIGN;
    if (ws && (ws_bytes < coli::kHeaderBytes || !aligned(ws, 256))) return COLI_ERR_WORKSPACE;
    // a workspace with room for the per-CTA counts past its header lets a
    // large batch split over several CTAs
    const size_t need = coli::union_scratch_bytes((int64_t)T * k, E);
    int* scratch = (ws && need > 0 && ws_bytes >= coli::kHeaderBytes + need)
                       ? reinterpret_cast<int*>(static_cast<char*>(ws) + coli::kHeaderBytes)
                       : nullptr;
    // T == 0 still writes empty lists (counts 0, offsets 0, no active experts).
    return from_cuda(coli::launch_union(T, E, k, topk_idx, counts, offsets, pairs, active,
                                        n_active, nullptr, ws ? static_cast<int*>(ws) : nullptr,
                                        scratch, static_cast<cudaStream_t>(stream)));
}

coli_status coli_moe_ffn(const coli_moe* h, int32_t T, const void* x_bf16, const float* topk_w,
                         const int32_t* counts, const int32_t* offsets, const int32_t* pairs,
                         const int32_t* active, const int32_t* n_active, const void* residual,
                         void* out, coli_out_dtype out_dtype, void* ws, size_t ws_bytes,
                         void* stream) {
    coli_status s = check_ffn_common(h, T, x_bf16, residual, out, out_dtype, ws, ws_bytes);
    if (s != COLI_OK || T == 0) return s;
    if (!topk_w || !counts || !offsets || !pairs || !active || !n_active) return COLI_ERR_INVALID_ARG;
    const void* ptrs[6] = {topk_w, counts, offsets, pairs, active, n_active};
    for (const void* p : ptrs)
        if (!aligned(p, 4)) return COLI_ERR_ALIGN;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    coli::FfnArgs a = make_args(h, T, x_bf16, topk_w, offsets, pairs, active, n_active, residual,
                                out, out_dtype, ws);
    profile_begin_call(st);
    cudaError_t err = coli::launch_inverse_pairs(T * h->k, pairs, a.inv, a.status, st);
    if (err == cudaSuccess) err = run_ffn(h, T, a, ws, st, false);
    profile_end_call();
    return from_cuda(err);
}

coli_status coli_moe_layer(const coli_moe* h, int32_t T, const void* x_bf16, const float* logits,
                           const float* router_w, const void* residual, void* out,
                           coli_out_dtype out_dtype, int32_t* topk_idx_out, float* topk_w_out,
                           void* ws, size_t ws_bytes, void* stream) {
    coli_status s = check_ffn_common(h, T, x_bf16, residual, out, out_dtype, ws, ws_bytes);
    if (s != COLI_OK) return s;
    if ((logits == nullptr) == (router_w == nullptr)) return COLI_ERR_INVALID_ARG;
    if (T == 0) return COLI_OK;
    const void* ptrs[4] = {logits, router_w, topk_idx_out, topk_w_out};
    for (const void* p : ptrs)
        if (p && !aligned(p, 4)) return COLI_ERR_ALIGN;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const coli::WsLayout L = layout_for(h, T);
    const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(x_bf16);
    profile_begin_call(st);
    cudaError_t err = cudaSuccess;
    const float* lg = logits;
    if (router_w) {
        float* wl = at<float>(ws, L.logits);
        err = coli::launch_router_logits(T, h->E, h->H, x, router_w, wl, st);
        lg = wl;
    }
    int* idx = topk_idx_out ? topk_idx_out : at<int>(ws, L.idx);
    float* w = topk_w_out ? topk_w_out : at<float>(ws, L.w);
    int* counts = at<int>(ws, L.counts);
    int* offsets = at<int>(ws, L.offsets);
    int* pairs = at<int>(ws, L.pairs);
    int* active = at<int>(ws, L.active);
    int* n_active = at<int>(ws, L.n_active);
    coli::FfnArgs a = make_args(h, T, x_bf16, w, offsets, pairs, active, n_active, residual, out,
                                out_dtype, ws);
    const bool prefill = use_prefill(h, T);
    if (err == cudaSuccess && use_fused(h, T)) {
        // one launch: every CTA routes the tokens itself
        err = run_fused(h, a, lg, topk_idx_out, topk_w_out, ws, st);
        if (err != cudaErrorCooperativeLaunchTooLarge) {
            profile_end_call();
            return from_cuda(err);
        }
        err = cudaSuccess;  // the grid cannot be resident at once: the streaming path below
    }
    if (T <= coli::kSmallT && !prefill) {
        // one launch: route, union, inverse map and activation preparation
        coli::PrepArgs p;
        p.T = T; p.E = h->E; p.k = h->k; p.H = h->H; p.n_shared = h->n_shared;
        p.logits = lg; p.idx = idx; p.w = w; p.counts = counts; p.offsets = offsets;
        p.pairs = pairs; p.active = active; p.n_active = n_active; p.inv = a.inv;
        p.x = x; p.xp = a.xp; p.corr = a.corr; p.status = a.status;
        if (err == cudaSuccess) err = coli::launch_prep_small(p, st);
    } else {
        if (err == cudaSuccess) err = coli::launch_route(T, h->E, h->k, lg, idx, w, st);
        if (err == cudaSuccess)
            err = coli::launch_union(T, h->E, h->k, idx, counts, offsets, pairs, active, n_active,
                                     a.inv, a.status, at<int>(ws, L.ucnt), st);
    }
    if (err == cudaSuccess) err = run_ffn(h, T, a, ws, st, T <= coli::kSmallT && !prefill);
    profile_end_call();
    return from_cuda(err);
}

coli_status coli_moe_get_status(const void* ws, void* stream) {
    if (!ws) return COLI_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return COLI_ERR_CUDA;
    int word = 0;
    if (cudaMemcpy(&word, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return COLI_ERR_CUDA;
    return static_cast<coli_status>(word);
}

const char* coli_status_string(coli_status s) {
    switch (s) {
        case COLI_OK: return "ok";
        case COLI_ERR_INVALID_ARG: return "invalid argument";
        case COLI_ERR_SHAPE: return "unsupported shape";
        case COLI_ERR_ALIGN: return "misaligned pointer";
        case COLI_ERR_WORKSPACE: return "workspace too small";
        case COLI_ERR_CUDA: return "CUDA runtime error";
        case COLI_ERR_TIMEOUT: return "device wait timed out";
        case COLI_ERR_UNSUPPORTED: return "unsupported device or feature";
        case COLI_ERR_BAD_INDEX: return "expert index out of range";
        case COLI_ERR_RANGE: return "intermediate outside the fp16 range (clamped)";
    }
    return "unknown status";
}

}  // extern "C"
