/*
 * rawint4_moe.h - C ABI of the B200 (sm_100a) routed RAWINT4 MoE-LoRA layer.
 *
 * The layer (rawint4_sft_reference.py, routed_rawint4_lora): a routed top-k
 * mixture of SwiGLU experts. Expert e's gate/up/down base projections are
 * frozen signed group-32 RAWINT4 and carry trainable rank-r LoRA adapters.
 * For token t, slot s, e = expert_ids[t,s], w = route_weights[t,s],
 * c = alpha / rank, L = swiglu_limit:
 *     G = W_g x + c B_g A_g x,  U = W_u x + c B_u A_u x
 *     G' = L > 0 ? min(G, L) : G,  U' = L > 0 ? clamp(U, -L, L) : U
 *     h = silu(G') U',  y = W_d h + c B_d A_d h,  out[t] = sum_s w y
 *
 * RAWINT4 storage (rawint4_sft_reference.py module docstring, unpack_rawint4):
 * two 4-bit codes per byte, LOW nibble first; weight = (code - 8) * scale,
 * one bf16 scale per 32 consecutive input features, no zero point.
 *
 * Conventions for every entry point:
 *  - bf16 / fp16 values are passed as uint16_t bit patterns.
 *  - Pointers named in the tensor lists are DEVICE pointers unless the
 *    comment says "host". All tensors are dense, row-major, contiguous.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream). Calls only
 *    enqueue work on it and return; they never synchronise except
 *    rawint4_moe_lora_status().
 *  - The caller owns every buffer. The library allocates no device memory
 *    and keeps no pointer after a call returns; all per-call state lives in
 *    the caller's workspace.
 *  - Return value: a RAWINT4_* status code. Argument errors are detected on
 *    the host before anything is enqueued, and nothing is written then.
 *
 * Design note: matrix products run on the 5th-generation tensor cores with
 * FP16 operands and FP32 accumulation. (code - 8) * scale has at most 12
 * significant bits, so every decoded weight is exact in FP16 as long as
 * |scale| lies in [2^-14, 8188]; activations are rounded once to FP16
 * (relative error 2^-11) where they become MMA operands. An activation
 * beyond the FP16 range raises RAWINT4_DEV_FP16_OVERFLOW. The backward
 * scales grad_out by an exact power of two chosen from its largest
 * magnitude before its FP16 operands are formed and undoes it in FP32, so
 * small gradients (1e-9 and below) keep their precision.
 * The LoRA tensors are copied to FP16 per call: exact for magnitudes in
 * [2^-14, 65504] (a bf16 value has 8 significant bits, FP16 holds 11),
 * rounded to FP16 subnormals below 2^-14 (absolute error at most 2^-25) and
 * to infinity above 65504 (no status bit: LoRA factors of that size are
 * outside any training regime).
 */
#ifndef RAWINT4_MOE_H
#define RAWINT4_MOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define RAWINT4_API __attribute__((visibility("default")))
#else
#define RAWINT4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---------------------------------------------------------------- codes */
enum {
  RAWINT4_OK = 0,
  RAWINT4_INVALID_ARGUMENT = 1, /* null pointer, bad size, workspace too small, ... */
  RAWINT4_FROZEN_BASE = 2,      /* a base-weight gradient buffer was passed (see bwd) */
  RAWINT4_NO_SAVED_FORWARD = 3, /* reported through the device status word */
  RAWINT4_CUDA_ERROR = 4,       /* a CUDA runtime/driver call failed */
  RAWINT4_BAD_EXPERT_ID = 5,    /* reported through the device status word */
  RAWINT4_DEVICE_TIMEOUT = 6,   /* a bounded pipeline wait expired (device status) */
  RAWINT4_FP16_OVERFLOW = 7,    /* an operand overflowed FP16 (device status) */
  RAWINT4_UNSUPPORTED = 8,      /* no sm_100 device, or shape outside the kernels' limits */
  RAWINT4_STATIC_SCRATCH_TOO_SMALL = 9 /* rawint4_moe_permute_static: needs more than its fixed scratch */
};

/* Bits of the device status word (rawint4_moe_lora_status). */
enum {
  RAWINT4_DEV_BAD_EXPERT_ID = 1u << 0,    /* an id outside [0, E): that slot contributed 0 */
  RAWINT4_DEV_NO_SAVED_FORWARD = 1u << 1, /* bwd found no pending saved forward: it did nothing */
  RAWINT4_DEV_TIMEOUT = 1u << 2,          /* a kernel gave up on a bounded wait: results invalid */
  RAWINT4_DEV_FP16_OVERFLOW = 1u << 3     /* an activation exceeded the FP16 range: results invalid */
};

/* ------------------------------------------------------------- structs */

/* Layer configuration. Mirrors the fields of the contract test's
 * MOESFTConfig that the method uses (test_rawint4_sft_numerical.py,
 * _make_backend): expert count, top_k, hidden size H, intermediate size I,
 * LoRA rank r and alpha (scaling c = alpha / r), swiglu_limit L (0 disables
 * the clamp; must be finite and >= 0) and max_tokens (the largest qlen a
 * workspace is sized for; the reference's max_len).
 * weight_format selects the frozen base format: RAWINT4 (the method) or the
 * pages' sibling MXFP4 format (the ext_bindings.cpp commit log's MXFP4
 * routed-expert LoRA path: E2M1 codes with UE8M0 group scales; only the
 * dequantisation differs, the LoRA, clamp, transpose-free dX and gradient
 * window are the same).
 * Limits: H % 64 == 0, I % 64 == 0 (the kernels reduce in stages of 64 and
 * mask a partial last block of output features; MXFP4: H % 128 == 0 and
 * I % 128 == 0, its scale bytes are fetched four at a time),
 * 1 <= rank <= 64 (the gate and up rank blocks, each padded to a multiple
 * of 16, take one or two 64-wide reduction stages), 1 <= top_k <= experts. */
enum {
  RAWINT4_FORMAT_RAWINT4 = 0, /* codes 0..15 -> (code - 8) * bf16 scale */
  RAWINT4_FORMAT_MXFP4 = 1    /* E2M1 codes * 2^(e - 127), e a UE8M0 scale byte */
};
typedef struct rawint4_moe_cfg {
  int32_t experts;
  int32_t top_k;
  int32_t hidden;
  int32_t inter;
  int32_t rank;
  float alpha;
  float swiglu_limit;
  int32_t max_tokens;
  int32_t weight_format; /* RAWINT4_FORMAT_*; 0 = RAWINT4 */
} rawint4_moe_cfg;

/* Frozen base weights (device, read-only; never written).
 * gate_q, up_q: uint8 [E, I, H/2]; gate_s, up_s: [E, I, H/32]
 * down_q:       uint8 [E, H, I/2]; down_s:       [E, H, I/32]
 * Layout of one projection: rawint4_sft_reference.py, _validate_rawint4_layout
 * (packed uint8 [N_out, K_in/2], one scale per 32 inputs). Scales are bf16
 * for RAWINT4 and UE8M0 bytes (uint8) for MXFP4; both formats pack two codes
 * per byte, low nibble first. */
/* Every base and LoRA pointer must be 16-byte aligned (RAWINT4_INVALID_ARGUMENT
 * otherwise): the kernels read them with TMA and 16-byte vector loads. */
typedef struct rawint4_moe_base {
  const uint8_t *gate_q, *up_q, *down_q;
  const void *gate_s, *up_s, *down_s;
} rawint4_moe_base;

/* LoRA adapters (device, bf16), the six tensors of the contract test
 * (GRAD_SHAPES): gate_a [E, r, H], gate_b [E, I, r], up_a [E, r, H],
 * up_b [E, I, r], down_a [E, r, I], down_b [E, H, r]. */
typedef struct rawint4_moe_lora {
  const uint16_t *gate_a, *gate_b, *up_a, *up_b, *down_a, *down_b;
} rawint4_moe_lora;

/* LoRA gradient buffers (device, bf16), same shapes as rawint4_moe_lora;
 * 16-byte aligned (RAWINT4_INVALID_ARGUMENT otherwise). */
typedef struct rawint4_moe_lora_grads {
  uint16_t *gate_a, *gate_b, *up_a, *up_b, *down_a, *down_b;
} rawint4_moe_lora_grads;

/* --------------------------------------------------------- entry points */

/* Bytes of device workspace a layer with this configuration needs
 * (*bytes, host). The workspace holds the routing permutation, the saved
 * forward context and backward scratch; its size grows linearly with
 * max_tokens * top_k. Returns RAWINT4_INVALID_ARGUMENT for a bad cfg. */
RAWINT4_API int rawint4_moe_lora_workspace_size(const rawint4_moe_cfg* cfg, size_t* bytes);

/* Forward (the contract test's forward_sft(qlen, top_k, ids, weights, in,
 * out, save_for_backward)).
 *   qlen          number of tokens Q, 0 <= qlen <= cfg->max_tokens (0: no-op
 *                 that still records an empty saved context when saving)
 *   expert_ids    int64 [Q, k]; ids outside [0, E) contribute nothing and
 *                 raise RAWINT4_DEV_BAD_EXPERT_ID in the device status
 *   route_weights fp32 [Q, k], used as given (no renormalisation)
 *   x             bf16 [Q, H];  out  bf16 [Q, H] (overwritten)
 *   save_for_backward  nonzero: keep the context for one rawint4_moe_lora_bwd
 *                 on this workspace, replacing any pending one (checkpoint
 *                 recompute). zero: the workspace's pending context, if any,
 *                 is invalidated (the scratch is shared).
 *   workspace     device buffer of at least rawint4_moe_lora_workspace_size
 *                 bytes, 256-byte aligned; ws_bytes is its size.
 *   lora          may be NULL: frozen-base inference forward, out = the
 *                 base-only layer (the LoRA terms are absent, as with zero
 *                 LoRA B). It saves no context, so save_for_backward must be
 *                 0 (RAWINT4_INVALID_ARGUMENT otherwise). This is the
 *                 frozen-base inference kernel of the contract test
 *                 (test_rawint4_sft_numerical.py, _run_inference_regression:
 *                 checked against the routed reference with zero LoRA).
 * The base, LoRA and input buffers must stay valid until the enqueued work
 * completes. */
RAWINT4_API int rawint4_moe_lora_fwd(const rawint4_moe_cfg* cfg, const rawint4_moe_base* base,
                         const rawint4_moe_lora* lora, int32_t qlen, const int64_t* expert_ids,
                         const float* route_weights, const uint16_t* x, uint16_t* out,
                         int save_for_backward, void* workspace, size_t ws_bytes, void* stream);

/* Backward of the most recent saving forward on this workspace (the
 * contract test's backward(dY, dX, 6 LoRA grads, dRoute, 3 base grads,
 * accumulate, grad_scale)). It consumes the saved context: exactly one
 * backward per saving forward. cfg, base and lora must be the ones the
 * forward used; lora must not be NULL (RAWINT4_INVALID_ARGUMENT).
 *   grad_out    bf16 [Q, H] (Q of the saved forward)
 *   grad_in     bf16 [Q, H] (overwritten) = d(sum grad_out*out)/dx
 *   grad_route  fp32 [Q, k] (overwritten; may be NULL) = <grad_out[t], y_{t,s}>
 *   grads       six bf16 buffers: buf = (accumulate ? buf : 0)
 *               + grad_scale * dLoRA, rounded once to bf16. Rows of experts
 *               that no slot of this call reached are zeroed when
 *               accumulate == 0 and left as they are otherwise
 *               (authoritative gradient window of the contract test).
 *               grad_scale multiplies only these six.
 *   base_grad_gate/up/down  must be NULL: the base is frozen and no base
 *               gradient is ever formed. Any non-NULL pointer returns
 *               RAWINT4_FROZEN_BASE before anything is enqueued.
 * Without a pending saved forward the call enqueues nothing that writes the
 * outputs and sets RAWINT4_DEV_NO_SAVED_FORWARD in the device status. */
RAWINT4_API int rawint4_moe_lora_bwd(const rawint4_moe_cfg* cfg, const rawint4_moe_base* base,
                         const rawint4_moe_lora* lora, const uint16_t* grad_out, uint16_t* grad_in,
                         float* grad_route, const rawint4_moe_lora_grads* grads,
                         const void* base_grad_gate, const void* base_grad_up,
                         const void* base_grad_down, int accumulate, float grad_scale,
                         void* workspace, size_t ws_bytes, void* stream);

/* Synchronises `stream`, then reads and clears the device status word kept
 * in `workspace` (*device_status, host: OR of RAWINT4_DEV_* bits raised by
 * calls since the last read). */
RAWINT4_API int rawint4_moe_lora_status(void* workspace, void* stream, uint32_t* device_status);

/* Human-readable text of a RAWINT4_* code (static storage). */
RAWINT4_API const char* rawint4_moe_lora_strerror(int code);

/* Bit-exact check export: decode one packed projection with the same device
 * routine the GEMM producers use.
 *   q [N, K/2] uint8, s [N, K/32] bf16 (device); K % 32 == 0.
 *   out_f32 [N, K] fp32 (device, may be NULL): (code - 8) * scale in fp32.
 *   out_f16 [N, K] fp16 bits (device, may be NULL): the MMA operand, i.e.
 *   the fp16 rounding of the same product (exact for scales in range). */
RAWINT4_API int rawint4_decode(const uint8_t* q, const uint16_t* s, int64_t n, int64_t k, float* out_f32,
                   uint16_t* out_f16, void* stream);

/* Bit-exact check export for the MXFP4 base format (the pages' sibling
 * format, weight layout mxfp4-e2m1-ue8m0-g32): one E2M1 code per nibble, low
 * nibble first, one UE8M0 scale byte e per 32 input features whose value is
 * 2^(e - 127) (the bf16 bit-cast e << 7: e == 0 is 0, e == 255 is +inf).
 *   q [N, K/2] uint8, s [N, K/32] uint8 (device); K % 32 == 0.
 *   out_f32 [N, K] fp32 (device, may be NULL): E2M1 value * 2^(e - 127).
 *   out_f16 [N, K] fp16 bits (device, may be NULL): the tensor-core operand
 *   the MXFP4 GEMM producers decode, exact for e in [104, 140]. */
RAWINT4_API int rawint4_mxfp4_decode(const uint8_t* q, const uint8_t* s, int64_t n, int64_t k, float* out_f32,
                                     uint16_t* out_f16, void* stream);

/* Bit-exact check export: the token->expert permutation of the forward.
 * ids int64 [Q, k] (device). Outputs (device, int32):
 *   offsets [E+1]  offsets[e] = first permuted row of expert e (exclusive
 *                  prefix sum of the per-expert counts)
 *   perm    [Q*k]  permuted row p -> flat slot f = t*k + s; stable (rows of
 *                  one expert ascend in f); entries past offsets[E] are -1
 *   inv     [Q*k]  flat slot -> permuted row, -1 for ids outside [0, E)
 * workspace: device scratch of rawint4_moe_permute_workspace_size bytes. */
RAWINT4_API int rawint4_moe_permute_workspace_size(int32_t qlen, int32_t top_k, int32_t experts, size_t* bytes);
RAWINT4_API int rawint4_moe_permute(const int64_t* ids, int32_t qlen, int32_t top_k, int32_t experts,
                        int32_t* offsets, int32_t* perm, int32_t* inv, void* workspace,
                        size_t ws_bytes, void* stream);

/* Same permutation as rawint4_moe_permute, for callers that cannot call
 * cudaMalloc to provide its scratch buffer (for example code running while
 * another component owns all device memory, or code that must not risk the
 * device-wide synchronisation a cudaMalloc can cause). No counterpart in the
 * paper; it exists only to serve such callers.
 *   ids, qlen, top_k, experts, offsets, perm, inv: as rawint4_moe_permute
 *   (device pointers, caller-owned outputs).
 * The scratch (header, tile list, per-block histograms: about
 * 512 + 16*(E + ceil(Q*k/192)) + 4*E*ceil(Q*k/1024) bytes) lives in a fixed
 * device array of rawint4_moe_permute_static_max_bytes() bytes (1 MiB)
 * inside the library; every GPU that loads the library holds it until the
 * process exits. Larger problems are rejected with
 * RAWINT4_STATIC_SCRATCH_TOO_SMALL before anything is enqueued. The first
 * call on a device looks up the array's device address (once per device, on
 * the current device); make that first call before any stream capture. All
 * calls share the one array, so calls whose work overlaps on the GPU (other
 * streams, other host threads) race and must be serialised by the caller.
 * The call allocates nothing: no cudaMalloc, cudaFree or allocating library
 * routine. */
RAWINT4_API int rawint4_moe_permute_static(const int64_t* ids, int32_t qlen, int32_t top_k, int32_t experts,
                                           int32_t* offsets, int32_t* perm, int32_t* inv, void* stream);
RAWINT4_API size_t rawint4_moe_permute_static_max_bytes(void);

/* Row moves of expert parallelism (no counterpart in the method, which runs
 * one process per layer: the layer's experts are split over G processes,
 * each routed slot travels to the process that owns its expert and its
 * result travels back). With
 * rawint4_moe_permute run on the owning process index of every slot
 * (experts = G), the slots are grouped by destination:
 *   rawint4_moe_dispatch_rows  dst[p, :] = src[perm[p] / top_k, :] for
 *     p < n: the bf16 token rows of the n slots that leave, in permuted
 *     order (src [Q, width], dst [n, width], width % 8 == 0, every perm[p]
 *     for p < n a valid slot; device pointers).
 *   rawint4_moe_combine_slots  out[t, :] = bf16 of the fp32 sum, in slot
 *     order s = 0..top_k-1, of src[inv[t * top_k + s], :] over the slots
 *     with inv >= 0 (0 where none): the token rows from the per-slot result
 *     rows that came back (src [n, width] bf16, out [qlen, width] bf16).
 *   rawint4_moe_gather_slots   out[f] = inv[f] >= 0 ? src[inv[f]] : 0 for
 *     f < n_slots: per-slot fp32 values (dRoute) back in slot order.
 * INVALID_ARGUMENT for a null pointer with a positive size, a negative size
 * or width % 8 != 0; asynchronous on `stream`. */
RAWINT4_API int rawint4_moe_dispatch_rows(const uint16_t* src, const int32_t* perm, int32_t n, int32_t top_k,
                                          int32_t width, uint16_t* dst, void* stream);
RAWINT4_API int rawint4_moe_combine_slots(const uint16_t* src, const int32_t* inv, int32_t qlen, int32_t top_k,
                                          int32_t width, uint16_t* out, void* stream);
RAWINT4_API int rawint4_moe_gather_slots(const float* src, const int32_t* inv, int32_t n_slots, float* out,
                                         void* stream);

/* Timing hook for measurement (no counterpart in the method): while enabled,
 * every kernel launch of the library records a CUDA event pair on the
 * launch's stream (at most max_launches launches). profile_end synchronises
 * on the recorded events and returns, per launch in issue order, a static
 * kernel name and its duration in ms (names/ms: host arrays of max_out
 * entries, may be NULL; *n_out = number of launches recorded). Not meant for
 * concurrent use from several threads. */
RAWINT4_API int rawint4_moe_profile_begin(int max_launches);
RAWINT4_API int rawint4_moe_profile_end(int max_out, int* n_out, const char** names, float* ms);

/* Router hand-off (test_gemma4_moe.py, Gemma4TextRouter.forward: softmax
 * over all experts, top-k, renormalise over the k, times a per-expert scale).
 * rawint4_moe_router_topk turns expert scores into the layer's inputs:
 *   scores   fp32 [Q, E] (device), the router's expert scores
 *   escale   fp32 [E] per-expert scale (device, may be NULL: all 1)
 *   ids      int64 [Q, k] (device, out): the k experts of largest probability,
 *            largest first, equal probabilities to the lower index
 *   weights  fp32 [Q, k] (device, out): renormalised probabilities * escale
 * rawint4_moe_router_bwd hands the layer's grad_route (= dL/dweights, from
 * rawint4_moe_lora_bwd) back to the router:
 *   grad_scores  fp32 [Q, E] (device, out): dL/dscores; 0 outside each
 *                token's k experts (the renormalisation cancels the softmax's
 *                normalisation over all E)
 *   grad_escale  fp32 [E] (device, out, may be NULL): dL/descale, summed over
 *                the slots routed to each expert in token order
 * Limits: 1 <= k <= min(E, 32), E <= 4096, Q >= 0; RAWINT4_INVALID_ARGUMENT
 * otherwise. Both only enqueue work on `stream`. */
RAWINT4_API int rawint4_moe_router_topk(const float* scores, int32_t qlen, int32_t experts, int32_t top_k,
                                        const float* escale, int64_t* ids, float* weights, void* stream);
RAWINT4_API int rawint4_moe_router_bwd(const float* scores, int32_t qlen, int32_t experts, int32_t top_k,
                                       const int64_t* ids, const float* grad_route, const float* escale,
                                       float* grad_scores, float* grad_escale, void* stream);

/* Test export (no counterpart in the method): the saved forward context of
 * `workspace` (left by the most recent saving rawint4_moe_lora_fwd and not yet
 * consumed by a backward), copied into caller-owned device buffers:
 *   perm    int32 [max_tokens * top_k]  permuted row -> flat slot f = t*k + s
 *           (-1 past the routed rows)
 *   g, u    fp32 [max_tokens * top_k, I]  the gate and up pre-activations G, U
 *           of each permuted row, the fp32 values the backward decides the
 *           clamp masks on (rows past the routed ones are unspecified)
 *   routed  host int32: number of routed (permuted) rows
 * Synchronises `stream`; changes nothing in the workspace. Returns
 * RAWINT4_NO_SAVED_FORWARD when no saved context is pending. */
RAWINT4_API int rawint4_moe_lora_saved_preacts(const rawint4_moe_cfg* cfg, const void* workspace, size_t ws_bytes,
                                               int32_t* perm, float* g, float* u, int32_t* routed, void* stream);

/* Test export (no counterpart in the method): the bound, in nanoseconds, on
 * every pipeline wait of the dequant GEMM kernels launched after this call
 * (default 4e9 ns; ns = 0 restores it). When a wait runs past the bound, the
 * kernel raises RAWINT4_DEV_TIMEOUT in the device status, every warp of the
 * kernel leaves at its next wait once the copies and tensor-core operations
 * it issued have landed, the tensor memory is released, and that call's
 * outputs are invalid; the next call with a normal bound is unaffected. A
 * bound far below a normal wait (1 ns, say) sends a call down that path on
 * purpose, which is how the path is tested. Process-wide; do not change it
 * while another host thread launches layer calls. */
RAWINT4_API int rawint4_moe_set_wait_limit_ns(uint64_t ns);

/* Kernel selection (read from the environment at each call; for testing both
 * kernel paths on one shape, the results agree within the layer tolerances):
 *   RAWINT4_TILES=narrow|wide  token tiles of at most 64 rows with the GEMMs'
 *                              narrow configuration, or of up to 192 rows.
 *                              Default: narrow when max_tokens * top_k <=
 *                              32 * experts, else wide.
 *                              Must not change between a forward and its
 *                              backward.
 *   RAWINT4_GEMM=tm            the transpose-free backward GEMMs of a RAWINT4
 *                              base on the tensor-memory kernel instead of
 *                              the shared-memory one (read once per process). */

#ifdef __cplusplus
}
#endif
#endif /* RAWINT4_MOE_H */
