/*
 * coli_moe.h - C ABI of libcoli_moe.so: one step of a routed Mixture-of-Experts
 * FFN layer with int4 group-64 (gs64) expert weights, on an NVIDIA B200
 * (sm_100a).
 *
 * The operation (from the pages about the Colibri MoE engine):
 *   - a router picks k of E routed experts for every token; one shared expert
 *     runs for every token as well ("zhichai.net/topic/178503686", MoE
 *     sparsity section: 256 experts, "8+1" active per layer; three-tier
 *     storage section: the "+1" is the shared expert in every layer);
 *   - batch-union: all positions of a batch that route to the same expert are
 *     served by one read of that expert ("yunpan.plus/t/30351-1-1",
 *     capability two, batch-union bullet); a worker receives one layer's
 *     routed batch-union and runs the FFN (same page, capability three, local
 *     cluster paragraph) - coli_moe_union / coli_moe_ffn follow that split;
 *   - experts are int4 with one scale per 64 weights ("yunpan.plus/t/30351-1-1",
 *     capability four: gs64 vs per-row int4; "ssnai.com/JustVugg_colibri.html",
 *     decision guide: the gs64 int4 container);
 *   - routing and precision are never changed silently
 *     ("yunpan.plus/t/30351-1-1", capability four): routing here is exact and
 *     deterministic, and the tie rule is part of the contract.
 *
 * Readings this library fixes where the pages are silent:
 *   - routing selects on the fp32 logits: descending value, ties to the lower
 *     expert index, -0 == +0, NaN ranks below -inf; slot j of a token holds
 *     its j-th best expert;
 *   - gate weights are the softmax renormalised over the k chosen experts:
 *     w_j = exp(l_j - m) / sum_i exp(l_i - m), m = the best chosen logit, NaN
 *     contributing 0; if m = +inf the +inf entries share weight 1 equally;
 *     if m is -inf or NaN every slot gets 1/k;
 *   - the expert FFN is SwiGLU: y = W_d (silu(W_g x) * (W_u x)),
 *     silu(z) = z / (1 + e^-z); the shared expert enters with weight 1;
 *   - out[t] = sum_j w[t][j] y_(t,j) (j ascending) + y_shared[t] (+ residual[t]),
 *     summed in fp32 in exactly that order.
 *
 * Weight format of one expert (all device memory, 16-byte aligned):
 *   gate_q, up_q : uint8 [I][H/2]   two codes per byte along H
 *   down_q       : uint8 [H][I/2]   two codes per byte along I
 *   gate_s, up_s : bf16  [I][H/64]  one scale per 64 consecutive codes of a row
 *   down_s       : bf16  [H][I/64]
 *   A code is a two's-complement nibble q in [-8, 7]; the LOW nibble of byte b
 *   is element 2b, the HIGH nibble element 2b+1; W[n][k] = q[n][k] * s[n][k/64].
 * Per-row int4 (group_size COLI_GROUP_PER_ROW), the format of the older
 * GLM-5.2 mirror ("ssnai.com/JustVugg_colibri.html", decision guide;
 * "yunpan.plus/t/30351-1-1", capability four: gs64 against per-row int4):
 * the same codes, one scale per row, W[n][k] = q[n][k] * s[n]:
 *   gate_s, up_s : bf16  [I][1]     down_s : bf16  [H][1]
 *
 * Conventions for every call:
 *   - all tensor arguments are DEVICE pointers owned by the caller, row-major
 *     and contiguous; the library never frees caller memory;
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream); every call is asynchronous on it and does not synchronise,
 *     except coli_moe_get_status;
 *   - argument errors are detected on the host and returned before anything
 *     is launched; T == 0 is a no-op that returns COLI_OK;
 *   - errors seen on the device (an expert index outside [0, E) in
 *     caller-supplied lists, a bounded wait that timed out, an intermediate
 *     outside the fp16 range) are recorded in a
 *     status word at the start of the workspace; the kernels skip the bad item
 *     and return normally; coli_moe_get_status reports the first one;
 *   - the workspace `ws` is caller-owned device memory of at least
 *     coli_moe_workspace_size() bytes, 256-byte aligned, cleared once with
 *     coli_moe_workspace_clear before its first use; calls that share a
 *     workspace must be ordered on one stream.
 */
#ifndef COLI_MOE_H
#define COLI_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    COLI_OK = 0,
    COLI_ERR_INVALID_ARG = 1, /* NULL pointer, negative size, bad enum */
    COLI_ERR_SHAPE = 2,       /* unsupported dims: k > E, k > 32, E > 1024, H or I not a multiple of 128 */
    COLI_ERR_ALIGN = 3,       /* a pointer not 16-byte aligned (workspace: 256) */
    COLI_ERR_WORKSPACE = 4,   /* workspace smaller than coli_moe_workspace_size */
    COLI_ERR_CUDA = 5,        /* a CUDA runtime call failed (launch, copy, allocation) */
    COLI_ERR_TIMEOUT = 6,     /* a bounded device wait gave up (status word) */
    COLI_ERR_UNSUPPORTED = 7, /* no sm_100 device, or a feature the library lacks */
    COLI_ERR_BAD_INDEX = 8,   /* device saw an expert index outside [0, E) (status word) */
    COLI_ERR_RANGE = 9        /* a SwiGLU output exceeded the fp16 range and was clamped to
                                 +-65504 before the down projection (status word) */
} coli_status;

typedef enum { COLI_OUT_F32 = 0, COLI_OUT_BF16 = 1 } coli_out_dtype;

/* One expert's weights (device pointers, 16-byte aligned, caller-owned; they
 * must outlive the handle). Layout as in the header comment. */
typedef struct {
    const uint8_t *gate_q, *up_q, *down_q;
    const uint16_t *gate_s, *up_s, *down_s; /* bf16 bit patterns */
} coli_expert;

/* Layer description.  `experts` is a HOST array of n_routed + n_shared
 * entries, routed experts first, shared experts last; it is copied by
 * coli_moe_create. */
typedef struct {
    int32_t hidden;             /* H, multiple of 128, at most 12288 */
    int32_t inter;              /* I, multiple of 128, at most 12288 */
    int32_t n_routed;           /* E, 1..1024 */
    int32_t top_k;              /* k, 1..min(E, 32) */
    int32_t group_size;         /* 64 (gs64) or COLI_GROUP_PER_ROW */
    int32_t n_shared;           /* shared experts, 0..4 */
    const coli_expert *experts; /* host array, n_routed + n_shared entries */
    int32_t prefill_min_tokens; /* T*k/E at or above which the tensor-core
                                   grouped GEMM is used; 0 = library default:
                                   the fused decode kernel where it applies
                                   (T <= 8, T*k < E), the small-batch kernels
                                   for the other calls of up to 64 tokens, the
                                   grouped GEMM above; a positive value: calls
                                   with T*k >= value * E, the streaming kernels
                                   for the rest the fused kernel does not
                                   take */
} coli_moe_desc;

#define COLI_GROUP_PER_ROW 0 /* group_size of the per-row int4 format */

typedef struct coli_moe coli_moe; /* opaque: device copy of the expert table */

/* Validate `desc` and build a handle on the current device.  Allocates a
 * small device table (cudaMalloc).  On error *out is set to NULL. */
coli_status coli_moe_create(const coli_moe_desc *desc, coli_moe **out);

/* Free the handle's table.  NULL is ignored.  Work that uses the handle must
 * have completed. */
void coli_moe_destroy(coli_moe *h);

/* Bytes of workspace coli_moe_layer / coli_moe_ffn need for calls with up to
 * max_tokens tokens (0 for a NULL handle or negative max_tokens). */
size_t coli_moe_workspace_size(const coli_moe *h, int32_t max_tokens);

/* Zero the workspace's status word and counters (async on `stream`).  Needed
 * once for a new workspace; later calls leave the counters at zero.  The
 * first COLI_WS_HEADER_BYTES of a workspace are this header. */
#define COLI_WS_HEADER_BYTES 16384
coli_status coli_moe_workspace_clear(void *ws, size_t ws_bytes, void *stream);

/* Router top-k (step 1 of the layer).
 *   logits   [T][E] fp32 (device)
 *   topk_idx [T][k] int32 out: slot j = j-th best expert (tie rule above)
 *   topk_w   [T][k] fp32  out: renormalised softmax weights of those experts
 * Exact: the same logits always give the same indices, bit for bit; the
 * weights are computed in double and rounded to fp32 once.
 * Errors: INVALID_ARG (NULL, T < 0), SHAPE (E < 1, E > 1024, k < 1, k > E,
 * k > 32), ALIGN (pointer not 4-byte aligned). */
coli_status coli_moe_route(int32_t T, int32_t E, int32_t k, const float *logits,
                           int32_t *topk_idx, float *topk_w, void *stream);

/* Batch-union (step 2): per-expert lists of the T*k (token, slot) pairs,
 * pair p = t*k + j.
 *   topk_idx [T][k] int32 in
 *   counts   [E]    out: pairs routed to each expert
 *   offsets  [E+1]  out: exclusive scan of counts; offsets[E] = T*k
 *   pairs    [T*k]  out: pair ids, expert-major, ascending token inside an expert
 *   active   [E]    out: experts with counts > 0, ascending; the rest -1
 *   n_active [1]    out: number of active experts
 * Deterministic: positions come from scans, never from atomic tickets.
 * `ws` may be NULL; if given (at least COLI_WS_HEADER_BYTES), an index
 * outside [0, E) is recorded in its status word (the pair is dropped from
 * the lists).  With at least coli_moe_union_workspace_size(T, E, k) bytes,
 * a batch of 4096 or more pairs is split over several CTAs (per-CTA counts
 * past the header); the lists are the same, bit for bit.
 * Errors: INVALID_ARG, SHAPE (as coli_moe_route; T*k > 2^24). */
coli_status coli_moe_union(int32_t T, int32_t E, int32_t k, const int32_t *topk_idx,
                           int32_t *counts, int32_t *offsets, int32_t *pairs,
                           int32_t *active, int32_t *n_active, void *ws, size_t ws_bytes,
                           void *stream);

/* Workspace bytes with which coli_moe_union splits a large batch over
 * several CTAs (COLI_WS_HEADER_BYTES when the batch is not split); 0 for
 * T < 0, E < 1 or k < 1.  A library addition, not an operation of the
 * pages. */
size_t coli_moe_union_workspace_size(int32_t T, int32_t E, int32_t k);

/* Expert FFN over a prepared batch-union (steps 3-5): every active expert's
 * weights are streamed once for all tokens on its list; the shared experts
 * run for all tokens; the results are combined per token in fixed order.
 *   x_bf16   [T][H] bf16 in (16-byte aligned)
 *   topk_w   [T][k] fp32 gate weights (slot order as topk_idx)
 *   counts, offsets, pairs, active, n_active: as produced by coli_moe_union
 *   residual [T][H] nullable, same dtype as out, added last
 *   out      [T][H] fp32 or bf16 (round to nearest even) out
 * Errors: INVALID_ARG, ALIGN, WORKSPACE; BAD_INDEX in the status word. */
coli_status coli_moe_ffn(const coli_moe *h, int32_t T, const void *x_bf16, const float *topk_w,
                         const int32_t *counts, const int32_t *offsets, const int32_t *pairs,
                         const int32_t *active, const int32_t *n_active, const void *residual,
                         void *out, coli_out_dtype out_dtype, void *ws, size_t ws_bytes,
                         void *stream);

/* The whole layer step: [router GEMV] -> route -> union -> FFN -> combine.
 * Exactly one of `logits` ([T][E] fp32) and `router_w` ([E][H] fp32; logits =
 * fp32(x) W_r^T computed in fp32) must be non-NULL.  With `router_w`, the
 * logits the call computed are left in the workspace at byte offset
 * COLI_WS_LOGITS_OFFSET, [T][E] fp32, until the next call.  topk_idx_out /
 * topk_w_out ([T][k]) receive the routing when non-NULL.  Other arguments as
 * coli_moe_ffn. */
#define COLI_WS_LOGITS_OFFSET 16384
coli_status coli_moe_layer(const coli_moe *h, int32_t T, const void *x_bf16, const float *logits,
                           const float *router_w, const void *residual, void *out,
                           coli_out_dtype out_dtype, int32_t *topk_idx_out, float *topk_w_out,
                           void *ws, size_t ws_bytes, void *stream);

/* The layer step (coli_moe_layer with `logits`) for callers that cannot
 * allocate device memory: it takes no handle and no workspace and allocates
 * nothing.  The pages have no counterpart of this entry point; it serves
 * callers whose device memory is owned by a host framework that forbids side
 * allocations, or latency-critical loops that must not call cudaMalloc (it
 * can synchronise the device).
 *   desc       layer description as for coli_moe_create (host struct; the
 *              expert pointers are device pointers); prefill_min_tokens is
 *              ignored (the streaming path always runs)
 *   T          tokens, at most 8; the call's workspace must also fit the
 *              library's 4 MiB scratch (H 6144 / I 2048 / 257 experts needs
 *              about 3 MB at T = 8); larger calls return COLI_ERR_WORKSPACE
 *              before anything is launched
 *   x_bf16, logits, residual, out, out_dtype: as coli_moe_layer
 *   status_out nullable device int32: receives the call's device status word
 *              (as coli_moe_get_status would read it) at the end of the call;
 *              written only when the call returns COLI_OK with T > 0 (a call
 *              that returns an error, or T == 0, leaves it untouched)
 * The scratch is one fixed __device__ array per GPU that loads the library,
 * held until exit.  The first call on a device (with that device current)
 * looks up the array's device address.  Every call also copies the expert
 * pointer table from pageable host memory into the array, so no call of this
 * entry point may be made under stream capture.  Every call shares the array
 * and clears its status word itself; calls whose work overlaps on the GPU
 * race on it, so order them on one stream.  Other errors as coli_moe_create
 * and coli_moe_layer. */
coli_status coli_moe_layer_noalloc(const coli_moe_desc *desc, int32_t T, const void *x_bf16,
                                   const float *logits, const void *residual, void *out,
                                   coli_out_dtype out_dtype, int32_t *status_out, void *stream);

/* Combine step of the expert-parallel layer (experts partitioned over
 * ranks): a local-cluster worker receives one layer's routed batch-union and
 * runs the FFN ("yunpan.plus/t/30351-1-1", capability three, local cluster
 * paragraph); the owner of a token then sums what comes back:
 *   out[t] = ((sum_{j<k} rows[t*k + j]) + shared[t]) + residual[t]
 * in fp32, in exactly that order.
 *   rows     [T*k][H] fp32: the token's routed outputs, each already
 *            multiplied by its gate weight, in slot order (nullable if k == 0)
 *   shared   [T][H] fp32 nullable: the shared experts' output
 *   residual [T][H] nullable, same dtype as out
 *   out      [T][H] fp32 or bf16 (round to nearest even)
 * All device pointers, 16-byte aligned; H a multiple of 4.  Asynchronous on
 * `stream`.  Errors: INVALID_ARG (NULL, negative sizes, bad enum), SHAPE
 * (H % 4), ALIGN. */
coli_status coli_moe_combine_rows(int32_t T, int32_t k, int32_t H, const float *rows,
                                  const float *shared, const void *residual, void *out,
                                  coli_out_dtype out_dtype, void *stream);

/* Router-lookahead prefetch into L2 (the pages' one-layer-ahead prefetch,
 * "yunpan.plus/t/30351-1-1", capabilities one and two, PILOT=1, with HBM ->
 * L2 in place of disk -> RAM): issue L2 prefetches of the weights of the
 * experts a routing names, in the order a layer call of handle `h` streams
 * them (shared experts first, then routed experts by ascending index), whole
 * experts only, until `max_bytes` would be exceeded.  Meant to run on a
 * second stream while the previous layer computes, with the previous step's
 * routing of `h`'s layer as the prediction.  Nothing is written; the layer
 * call's results do not depend on it.
 *   topk_idx [T][k] int32 device: the predicted routing
 *   ws       nullable; if given (at least COLI_WS_HEADER_BYTES, 256-byte
 *            aligned), an index outside [0, E) is recorded in its status word
 * Errors: INVALID_ARG (NULL handle, T < 0, k outside [1, E]), SHAPE, ALIGN,
 * WORKSPACE. */
coli_status coli_moe_prefetch(const coli_moe *h, int32_t T, int32_t k, const int32_t *topk_idx,
                              size_t max_bytes, void *ws, size_t ws_bytes, void *stream);

/* Synchronise `stream` and return the workspace's device status word
 * (COLI_OK, COLI_ERR_BAD_INDEX or COLI_ERR_TIMEOUT), or COLI_ERR_CUDA if the
 * stream reports an error.  The word stays set until coli_moe_workspace_clear. */
coli_status coli_moe_get_status(const void *ws, void *stream);

/* Timing diagnostics (not needed for correct use).  While enabled, every
 * coli_moe_layer / coli_moe_ffn call records CUDA events on its stream around
 * its phases: [0] routing + union + preparation, [1] the gate/up kernel,
 * [2] the down kernel, [3] the combine.  coli_moe_profile_read synchronises
 * those events and writes the summed milliseconds per phase to ms[0..3] and
 * the number of recorded calls to *n_calls, then forgets them.  Enabling or
 * reading is host-global state: use it from one thread. */
coli_status coli_moe_profile_enable(int32_t enable);
coli_status coli_moe_profile_read(double *ms, int32_t *n_calls);

/* Fault injection for tests (host-global, one thread).  With
 * COLI_INJECT_WITHHOLD_STAGE the next coli_moe_layer / coli_moe_ffn call that
 * runs the fused decode kernel or the streaming kernels (not the grouped
 * GEMM) never fills one staged gate/up tile: its consumers' bounded wait
 * (about one second) runs out, the kernel winds down without hanging or
 * faulting, and the status word reads COLI_ERR_TIMEOUT; the output of that
 * call is undefined and the context stays usable.  0 switches every hook
 * off.
 * Returns COLI_ERR_INVALID_ARG for an unknown code. */
#define COLI_INJECT_WITHHOLD_STAGE 1
/* With COLI_INJECT_NOT_RESIDENT the next call that would run the fused
 * decode kernel (up to 8 tokens) behaves as if its cooperative launch had
 * been refused because the grid cannot be resident at once (a GPU with fewer
 * usable SMs than the handle saw): nothing is launched for it and the call
 * runs on the streaming kernels instead, with the same result. */
#define COLI_INJECT_NOT_RESIDENT 2
coli_status coli_moe_debug_inject(int32_t what);

/* Static English text for a status code (never NULL). */
const char *coli_status_string(coli_status s);

#ifdef __cplusplus
}
#endif

#endif /* COLI_MOE_H */
