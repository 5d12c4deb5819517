// coli_moe_layer_noalloc: the small-batch layer step for callers that cannot
// allocate device memory themselves.
//
// Who needs it: a caller whose device memory is owned and pre-planned by a
// host framework (a fixed-budget serving process that hands out every byte
// from its own pool and forbids side allocations), or a latency-critical
// decode loop that must not call cudaMalloc because it can synchronise the
// device and take unbounded time.  Such a caller can still pass its inputs and
// outputs, but not a workspace or a handle, both of which need an allocation.
//
// How: the workspace of the call and the device copy of the expert pointer
// table live in one file-scope __device__ array of fixed size, which every
// GPU that loads the library holds until the process exits.  Host code never
// passes the array's name to a kernel (on the host it is only a stand-in, not
// a device address); the first call on each device, with that device
// current, looks up the array's device address with cudaGetSymbolAddress and
// keeps it.  Every call copies the expert pointer table into the array from
// pageable host memory, a copy a stream capture cannot record: no call of
// this entry point may be made under stream capture.
//
// Sharing: every call (on a device) uses the same array, which keeps the last
// call's contents; the call clears the part that must start at zero (the
// status word) itself.  Calls whose work overlaps on the GPU race on the
// array: order them on one stream.
#include <cstring>
#include <mutex>

#include "coli_internal.cuh"
#include "handle.cuh"

namespace {

constexpr size_t kTableBytes = 64 * 1024;        // device copy of the expert table
constexpr size_t kScratchBytes = 4u << 20;        // workspace of one call (4 MiB)
constexpr int32_t kMaxTokens = 8;                 // tokens per call
constexpr int kMaxDevices = 64;

__device__ __align__(256) uint8_t g_noalloc_scratch[kTableBytes + kScratchBytes];

struct DeviceSetup {
    bool ready = false;
    void* base = nullptr;  // device address of g_noalloc_scratch on this device
    int num_sms = 0;
};
DeviceSetup g_setup[kMaxDevices];
std::mutex g_setup_mu;
coli::DevExpert g_host_table[kTableBytes / sizeof(coli::DevExpert)];

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Once per device, with that device current: the array's device address.
coli_status setup_device(int dev, DeviceSetup** out) {
    if (dev < 0 || dev >= kMaxDevices) return COLI_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_setup_mu);
    DeviceSetup& s = g_setup[dev];
    if (!s.ready) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return COLI_ERR_CUDA;
        if (major != 10 || minor != 0) return COLI_ERR_UNSUPPORTED;
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr)
            return COLI_ERR_CUDA;
        s.base = ptr;
        s.num_sms = sms;
        s.ready = true;
    }
    *out = &s;
    return COLI_OK;
}

}  // namespace

extern "C" coli_status coli_moe_layer_noalloc(const coli_moe_desc* d, int32_t T, const void* x_bf16,
                                              const float* logits, const void* residual,
                                              void* out, coli_out_dtype out_dtype,
                                              int32_t* status_out, void* stream) {
    // the descriptor checks coli_moe_create makes, without its allocations
    if (!d || !d->experts || T < 0) return COLI_ERR_INVALID_ARG;
    if (d->group_size != coli::kGroup && d->group_size != COLI_GROUP_PER_ROW) return COLI_ERR_SHAPE;
    if (d->hidden <= 0 || d->inter <= 0 || d->hidden % 128 || d->inter % 128) return COLI_ERR_SHAPE;
    if (d->hidden > 12288 || d->inter > 12288 || !coli::stream_shapes_fit(d->hidden, d->inter))
        return COLI_ERR_SHAPE;
    if (d->n_routed < 1 || d->n_routed > coli::kMaxExperts) return COLI_ERR_SHAPE;
    if (d->top_k < 1 || d->top_k > d->n_routed || d->top_k > coli::kMaxTopK) return COLI_ERR_SHAPE;
    if (d->n_shared < 0 || d->n_shared > coli::kMaxShared) return COLI_ERR_SHAPE;
    if (T > kMaxTokens) return COLI_ERR_WORKSPACE;  // beyond what the fixed scratch serves
    const int n = d->n_routed + d->n_shared;
    if ((size_t)n * sizeof(coli::DevExpert) > kTableBytes) return COLI_ERR_SHAPE;
    const coli::WsLayout L = coli::ws_layout(T, d->n_routed, d->top_k, d->hidden, d->inter,
                                             d->n_shared);
    if (L.total > kScratchBytes) return COLI_ERR_WORKSPACE;
    if (T == 0) return COLI_OK;
    if (!x_bf16 || !logits || !out) return COLI_ERR_INVALID_ARG;
    if (!aligned16(x_bf16) || !aligned16(out) || (residual && !aligned16(residual)) ||
        (reinterpret_cast<uintptr_t>(logits) & 3) || (reinterpret_cast<uintptr_t>(status_out) & 3))
        return COLI_ERR_ALIGN;
    for (int e = 0; e < n; ++e) {
        const coli_expert& x = d->experts[e];
        const void* ptrs[6] = {x.gate_q, x.up_q, x.down_q, x.gate_s, x.up_s, x.down_s};
        for (const void* p : ptrs) {
            if (!p) return COLI_ERR_INVALID_ARG;
            if (!aligned16(p)) return COLI_ERR_ALIGN;
        }
    }

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return COLI_ERR_CUDA;
    DeviceSetup* s = nullptr;
    coli_status st = setup_device(dev, &s);
    if (st != COLI_OK) return st;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    uint8_t* base = static_cast<uint8_t*>(s->base);
    void* ws = base + kTableBytes;

    // expert pointer table -> the array (staged by the runtime; no allocation here)
    std::lock_guard<std::mutex> lock(g_setup_mu);
    for (int e = 0; e < n; ++e) {
        g_host_table[e].gate_q = d->experts[e].gate_q;
        g_host_table[e].up_q = d->experts[e].up_q;
        g_host_table[e].down_q = d->experts[e].down_q;
        g_host_table[e].gate_s = d->experts[e].gate_s;
        g_host_table[e].up_s = d->experts[e].up_s;
        g_host_table[e].down_s = d->experts[e].down_s;
    }
    if (cudaMemcpyAsync(base, g_host_table, n * sizeof(coli::DevExpert), cudaMemcpyHostToDevice,
                        cs) != cudaSuccess)
        return COLI_ERR_CUDA;
    // the status word and counters must start at zero on every call
    if (cudaMemsetAsync(ws, 0, coli::kHeaderBytes, cs) != cudaSuccess) return COLI_ERR_CUDA;

    // a handle that lives on the stack and points into the array; the
    // tensor-core path stays off (it needs per-expert tensor maps)
    coli_moe h;
    h.device = dev;
    h.H = d->hidden;
    h.I = d->inter;
    h.E = d->n_routed;
    h.k = d->top_k;
    h.n_shared = d->n_shared;
    h.prefill_min = d->prefill_min_tokens;
    h.per_row = d->group_size == COLI_GROUP_PER_ROW;
    h.num_sms = s->num_sms;
    h.d_experts = reinterpret_cast<coli::DevExpert*>(base);
    h.d_wmaps = nullptr;
    h.d_bmaps = nullptr;
    h.d_dmaps = nullptr;
    st = coli_moe_layer(&h, T, x_bf16, logits, nullptr, residual, out, out_dtype, nullptr, nullptr,
                        ws, kScratchBytes, stream);
    if (st == COLI_OK && status_out &&
        cudaMemcpyAsync(status_out, ws, sizeof(int32_t), cudaMemcpyDeviceToDevice, cs) != cudaSuccess)
        return COLI_ERR_CUDA;
    return st;
}
