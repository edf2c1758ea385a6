/*
 * moe_fp4.h -- C ABI of the NVFP4 sparse mixture-of-experts layer forward
 * (libmoe_fp4.so, CUDA, sm_100a).
 *
 * The operation (one decoder layer's MoE block, forward only):
 *   for each token t with activation x[t] (bf16, width d):
 *     l[t,e]   = sum_i x[t,i] * Wr[e,i]                          fp32 router logits
 *     S_t      = the top_k experts by l[t,:], ties to the lower index
 *     w[t,j]   = softmax(l[t,:])[S_j] / sum_{S} softmax(l[t,:])  renormalised
 *     out[t]   = bf16( sum_j w[t,j] * Wd[S_j] (SiLU(Wg[S_j] x) * (Wu[S_j] x)) )
 *   with every expert matrix stored in NVFP4.
 * Sources: "Optimizing Muse Spark Open on TPU v7 with SGLang-TorchTPU"
 * (Background: 8 of 256 experts per token, NVFP4 experts with one scale per
 * 16 values; section 5: the expert loop chosen by per-expert row count;
 * section 8: gate/up, SwiGLU, down, a one-pass combine that writes every
 * output row once) and "Optimizing Models to Be Fast at Codegen" (section 2:
 * FP4 e2m1 weights with a per-16 block scale, unpacked in registers, a
 * grouped GEMM over only the active experts).
 *
 * NVFP4 (canonical layout accepted by moe_fp4_load_experts), per expert and
 * matrix, row-major:
 *   q  uint8 [rows][K/2]  two e2m1 codes per byte, element 2i in the LOW nibble
 *                         (bit 3 sign, bits 2-1 exponent with bias 1, bit 0 mantissa)
 *   sf uint8 [rows][K/16] e4m3fn block scales, block i covers K elements 16i..16i+15
 *   gs float              one fp32 tensor scale per (expert, matrix)
 *   value[n][k] = e2m1(q[n][k]) * e4m3(sf[n][k/16]) * gs
 *   gate, up: rows = f, K = d;   down: rows = d, K = f.
 *
 * Activation precision, chosen per expert by its row count n_e in the call:
 *   n_e <  dense_threshold : x (bf16) and h = SiLU(g)*u stay unquantised
 *                            (tensor-core inputs are fp16 after an exact
 *                            power-of-two rescale of each x row);
 *   n_e >= dense_threshold : x and h are quantised to NVFP4 along K with
 *                            tensor scale 1.0 (sf = e4m3_rn(amax/6),
 *                            q = e2m1_rn(v/sf), decisions in fp32) and the
 *                            expert runs on block-scaled FP4 tensor cores.
 *   The threshold defaults to 9 (environment MOE_FP4_DENSE_THRESHOLD at
 *   create time, or moe_fp4_set_dense_threshold): an expert with 9 or more
 *   rows streams its weights faster through the tensor-core class.  The dense class needs d
 *   and f to be multiples of 256 (one 256-element K stage of the tensor-core
 *   pipeline); for other shapes, or if the driver's tensor-map encoder is not
 *   available, every expert runs in the light class whatever its row count.
 *   The dense GEMMs run on single CTAs (128-row tiles); the environment
 *   variable MOE_FP4_DENSE_PAIRS set to "1" at create time selects CTA pairs
 *   (clusters of two SMs, tcgen05 cta_group::2, 256 x 256 tiles) when the
 *   device fits them.  Both give results within the same bounds.
 *
 * Conventions
 *   - Every call returns a moe_fp4_status and never aborts the process.
 *   - Device pointers are plain CUDA device addresses of the current device;
 *     the library never frees caller memory.  The handle owns all of its
 *     own device memory (repacked experts + workspace) and frees it in
 *     moe_fp4_destroy.
 *   - A handle is bound to the device current at create time, is not
 *     thread-safe, and must be used from one stream at a time.
 *   - moe_fp4_forward is asynchronous on `stream`, performs no host
 *     synchronisation, and allocates nothing once moe_fp4_reserve(max_T) has
 *     sized the workspace for T <= max_T; under those conditions it can be
 *     captured into a CUDA graph.  Results are deterministic: the same inputs
 *     give bit-identical outputs.
 *   - Kernel-side failures (an internal wait that exceeded its bound, a
 *     numeric overflow of an fp16 intermediate, an unsupported expert class)
 *     set a device error word; read it with moe_fp4_get_device_error after
 *     synchronising the stream.
 */
#ifndef MOE_FP4_H
#define MOE_FP4_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define MOE_FP4_API __attribute__((visibility("default")))
#else
#define MOE_FP4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct moe_fp4 moe_fp4_t;

typedef enum {
  MOE_FP4_OK = 0,
  MOE_FP4_ERR_INVALID_ARG = 1,    /* null pointer, negative T, aliasing, bad value */
  MOE_FP4_ERR_UNSUPPORTED = 2,    /* shape outside the supported limits */
  MOE_FP4_ERR_NOT_LOADED = 3,     /* forward before moe_fp4_load_experts */
  MOE_FP4_ERR_CUDA = 4,           /* a CUDA runtime call failed */
  MOE_FP4_ERR_OOM = 5,            /* device allocation failed */
  MOE_FP4_ERR_DEVICE_TIMEOUT = 6, /* (device error word) a bounded wait expired */
  MOE_FP4_ERR_NUMERIC = 7,        /* (device error word) fp16 intermediate overflowed */
  MOE_FP4_ERR_CAPTURE = 8         /* workspace growth needed while the stream is capturing */
} moe_fp4_status;

/* Create a layer handle on the current device.
 * Defines the layer's shape: E experts, top_k routed per token, model width
 * d, expert FFN width f ("Optimizing Muse Spark Open on TPU v7 with
 * SGLang-TorchTPU", Background: each token goes to 8 of 256 experts; the
 * "Mixture of Experts" topic page: 256 experts, 8 selected).
 *   E       experts, 1..1024
 *   top_k   experts per token, 1..min(E, 32)
 *   d, f    model width and expert FFN width; multiples of 128, 128..16384
 * On success *out receives the handle (caller destroys it). */
MOE_FP4_API int moe_fp4_create(int E, int top_k, int d, int f, moe_fp4_t** out);

/* Canonical NVFP4 expert weights (device pointers, caller-owned, read only
 * during the call).  Layout as described at the top of this file:
 *   gate_q, up_q   [E][f][d/2]     gate_sf, up_sf [E][f][d/16]   gate_gs, up_gs [E]
 *   down_q         [E][d][f/2]     down_sf        [E][d][f/16]   down_gs        [E] */
typedef struct {
  const uint8_t* gate_q;
  const uint8_t* gate_sf;
  const float*   gate_gs;
  const uint8_t* up_q;
  const uint8_t* up_sf;
  const float*   up_gs;
  const uint8_t* down_q;
  const uint8_t* down_sf;
  const float*   down_gs;
} moe_fp4_experts;

/* Copy and repack the experts into library-owned device buffers (the
 * register-dequant GEMV layout and the tensor-core block-scaled layout).
 * The weights are NVFP4 as defined on "Optimizing Models to Be Fast at
 * Codegen", section 2 (e2m1 values, one scale per 16 along K) and the Muse
 * Spark page's Background (4-bit experts with a per-16 block scale); each
 * (expert, matrix) carries one fp32 tensor scale.  Also derives, per expert,
 * the largest row L1 norm of the gate and up matrices, which bounds the
 * light class's intermediates.  Synchronous; may be called again to replace
 * the weights.  Errors: MOE_FP4_ERR_INVALID_ARG (null handle, struct or
 * member), MOE_FP4_ERR_OOM, MOE_FP4_ERR_CUDA. */
MOE_FP4_API int moe_fp4_load_experts(moe_fp4_t* h, const moe_fp4_experts* w);

/* Which resident weight copies the next moe_fp4_load_experts keeps (each
 * copy holds exactly the canonical NVFP4 bytes: E * 3 * f * d * (1/2 + 1/16)):
 *   light = 1, dense = 1  both (the default): few-row experts stream the
 *                         register-dequant copy, many-row experts the
 *                         tensor-core copy;
 *   light = 1, dense = 0  only the register-dequant copy: every expert runs
 *                         in the light class;
 *   light = 0, dense = 1  only the tensor-core copy: every expert runs in the
 *                         dense class (NVFP4 activations), whatever its row
 *                         count; needs d and f multiples of 256.
 * The weights stay 4-bit in every copy ("Optimizing Models to Be Fast at
 * Codegen", section 2).  The choice takes effect at the next load, which
 * frees copies no longer kept; until then forwards report
 * MOE_FP4_ERR_NOT_LOADED.  Errors: MOE_FP4_ERR_INVALID_ARG (null handle, a
 * value other than 0/1, both 0), MOE_FP4_ERR_UNSUPPORTED (dense only with d
 * or f not a multiple of 256). */
MOE_FP4_API int moe_fp4_set_resident_classes(moe_fp4_t* h, int light, int dense);

/* Device bytes the handle holds: *weights for the resident weight copies,
 * *workspace for the forward's workspace.  Errors: MOE_FP4_ERR_INVALID_ARG. */
MOE_FP4_API int moe_fp4_device_bytes(moe_fp4_t* h, size_t* weights, size_t* workspace);

/* Pre-size the workspace for up to max_T tokens per forward (allocates).
 * After this, moe_fp4_forward with T <= max_T allocates nothing. */
MOE_FP4_API int moe_fp4_reserve(moe_fp4_t* h, int max_T);

/* The layer forward: router logits, softmax and top-k, the token -> expert
 * permutation, gate/up + SwiGLU, down x routing weight and the combine, as
 * stated at the top of this file (Muse Spark page, Background and section 8:
 * gate/up, SwiGLU, down, a single combine pass writing each output row
 * once; "Day-0 Inference Adaptation for Ultra-Large Sparse Models", section
 * II: routing indexes built on the device without a host round trip).
 *   x_bf16    device, bf16 [T][d] row-major
 *   T         tokens, >= 0 (T = 0 is a no-op)
 *   router_w  device, fp32 [E][d] row-major
 *   out_bf16  device, bf16 [T][d]; written completely, must not overlap x
 *   stream    CUDA stream (0 = legacy default stream)
 * Asynchronous on `stream`.  Errors: MOE_FP4_ERR_INVALID_ARG (null handle or
 * pointer, T < 0, a pointer not 16-byte aligned, out overlapping x),
 * MOE_FP4_ERR_UNSUPPORTED (T * top_k >= 2^30), MOE_FP4_ERR_NOT_LOADED,
 * MOE_FP4_ERR_OOM / MOE_FP4_ERR_CAPTURE (workspace growth), MOE_FP4_ERR_CUDA. */
MOE_FP4_API int moe_fp4_forward(moe_fp4_t* h, const void* x_bf16, int T, const float* router_w,
                    void* out_bf16, cudaStream_t stream);

/* Intermediates of a forward, for layer-by-layer comparison (the steps of
 * the layer as moe_fp4_forward states them).  Every member
 * may be NULL; non-NULL members are device buffers the caller owns:
 *   logits   fp32  [T][E]
 *   topk_ids int32 [T][top_k]   listed by (logit desc, expert asc)
 *   topk_w   fp32  [T][top_k]
 *   counts   int32 [E]          pairs per expert
 *   offsets  int32 [E+1]        exclusive scan of counts
 *   perm     int32 [T*top_k]    perm[pos] = t*top_k + j, pairs sorted by (expert, t, j)
 *   h        fp32  [T*top_k][f] SiLU(g)*u per pair, rows in perm order
 *   partial  fp32  [T*top_k][d] w * (Wd h) per pair, rows in perm order
 *                               (Wd h, unweighted, while the per-expert norm
 *                               is on)
 * Copies are enqueued on `stream` after the forward. */
typedef struct {
  float*   logits;
  int32_t* topk_ids;
  float*   topk_w;
  int32_t* counts;
  int32_t* offsets;
  int32_t* perm;
  float*   h;
  float*   partial;
} moe_fp4_debug;

MOE_FP4_API int moe_fp4_forward_ex(moe_fp4_t* h, const void* x_bf16, int T, const float* router_w,
                       void* out_bf16, cudaStream_t stream, moe_fp4_debug* dbg);

/* End-to-end variant taking HOST buffers: copies x (host bf16 [T][d]) to the
 * device, runs the forward and copies the result back into out_host (host
 * bf16 [T][d]), all on `stream`, then synchronises the stream.  Pinned host
 * memory gives asynchronous copies; pageable memory works but is slower.
 * router_w is a device pointer as in moe_fp4_forward. */
MOE_FP4_API int moe_fp4_forward_host(moe_fp4_t* h, const void* x_host, int T, const float* router_w,
                         void* out_host, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Expert parallelism: the layer split over G ranks (one GPU each), rank r
 * owning the contiguous experts [r E/G, (r+1) E/G).  The pages run the MoE
 * layer with its experts sharded across devices and the token rows exchanged
 * through an all-to-all ("Optimizing Muse Spark Open on TPU v7 with
 * SGLang-TorchTPU", section 8, "Sequence-parallel prefill": routing ids and
 * weights travel with the tokens, the MoE output returns through an
 * all-to-all; "Day-0 Inference Adaptation for Ultra-Large Sparse Models":
 * expert-parallel deployment).  These calls are the device-side pieces; the
 * exchange between them is the caller's (NCCL all-to-all of device buffers).
 * Because the permutation orders pairs by expert, the rows bound for one rank
 * form one contiguous run of the permuted order.
 * ------------------------------------------------------------------------ */

/* Routing of a forward without the experts: fp32 logits, top-k, weights,
 * counts, offsets, the permutation and its inverse (layouts as in
 * moe_fp4_debug; inv[t*top_k + j] = position of pair (t, j) in perm).  Any
 * member may be NULL; non-NULL members are caller-owned device buffers.
 * Needs no moe_fp4_load_experts.  Asynchronous on `stream`.  Errors as
 * moe_fp4_forward (without MOE_FP4_ERR_NOT_LOADED). */
typedef struct {
  float*   logits;
  int32_t* topk_ids;
  float*   topk_w;
  int32_t* counts;
  int32_t* offsets;
  int32_t* perm;
  int32_t* inv;
} moe_fp4_routing;
MOE_FP4_API int moe_fp4_route(moe_fp4_t* h, const void* x_bf16, int T, const float* router_w,
                              moe_fp4_routing* r, cudaStream_t stream);

/* rows[i] = x[perm[i] / top_k] for i < P: the token row of every pair in
 * permutation order (bf16 [P][d]; x bf16 [T][d]).  No handle.  d a multiple
 * of 8, x and rows 16-byte aligned, P <= T * top_k, every perm[i] in
 * [0, T * top_k) (not checked).  Errors: MOE_FP4_ERR_INVALID_ARG,
 * MOE_FP4_ERR_CUDA. */
MOE_FP4_API int moe_fp4_gather_rows(const void* x_bf16, int T, int d, const int32_t* perm, int P,
                                    int top_k, void* rows_bf16, cudaStream_t stream);

/* The experts of this handle on rows the caller routed: row i (bf16 [n][d])
 * goes to expert expert_ids[i] (0 <= id < E of this handle) with weight 1,
 * and y_rows[i] (fp32 [n][d]) receives Wd (SiLU(Wg x) * (Wu x)) of that
 * expert, unweighted.  The expert classes follow each expert's row count in
 * the call, as in moe_fp4_forward.  The handle must have top_k = 1.  An id
 * out of range records MOE_FP4_ERR_INVALID_ARG in the device error word and
 * leaves that row's output undefined.  Errors: MOE_FP4_ERR_INVALID_ARG,
 * MOE_FP4_ERR_UNSUPPORTED (top_k != 1), MOE_FP4_ERR_NOT_LOADED, as
 * moe_fp4_forward otherwise. */
MOE_FP4_API int moe_fp4_forward_routed(moe_fp4_t* h, const void* rows_bf16, int n, const int32_t* expert_ids,
                                       float* y_rows, cudaStream_t stream);

/* out[t] = bf16_rn( sum_j fl(topk_w[t][j] * y_rows[inv[t*top_k + j]]) ),
 * slots j = 0..top_k-1 in order, fp32: the routing-weighted combine of
 * expert outputs that came back in permutation order (y_rows fp32 [P][d],
 * out bf16 [T][d]).  No handle.  Errors: MOE_FP4_ERR_INVALID_ARG,
 * MOE_FP4_ERR_CUDA. */
MOE_FP4_API int moe_fp4_combine_rows(const float* y_rows, const int32_t* inv, const float* topk_w, int T,
                                     int top_k, int d, void* out_bf16, cudaStream_t stream);

/* Activation-precision threshold (see the top of this file); thr >= 1.
 * The split of a step's experts into a loop for few-row experts and one for
 * many-row experts follows the Muse Spark page, section 5 (two expert loops
 * chosen by per-expert row count).  Errors: MOE_FP4_ERR_INVALID_ARG. */
MOE_FP4_API int moe_fp4_set_dense_threshold(moe_fp4_t* h, int thr);

/* Per-expert output normalisation before the weighted sum (Muse Spark page,
 * section 8: each expert's output is normalised before the routing-weighted
 * sum, in the one fused combine pass).  With enable = 1 every later forward
 * computes
 *   out[t] = bf16( sum_j w[t,j] * y_j / sqrt(mean_i y_j[i]^2 + eps) ),
 *   y_j = Wd[S_j] (SiLU(Wg[S_j] x) * (Wu[S_j] x)),
 * an RMS norm over the d outputs of each expert with no learned gain;
 * enable = 0 (the default) restores the plain weighted sum.  eps >= 0 and
 * finite (ignored when enable = 0).  Errors: MOE_FP4_ERR_INVALID_ARG. */
MOE_FP4_API int moe_fp4_set_expert_norm(moe_fp4_t* h, int enable, float eps);

/* Activation tensor scale of the dense class (NVFP4 activations).
 *   dynamic = 0 (default): tensor scale 1.0, as at the top of this file; a
 *       16-block whose amax is below about 6 * 2^-10 quantises to zeros.
 *   dynamic = 1: every forward scales x and h by powers of two chosen from
 *       the call's own data: gs = 2^e, e the smallest integer with
 *       max|a| <= 6 * 448 * 2^e, max over the whole tensor (x: all T tokens;
 *       h: every dense-class row); a is quantised as a * 2^-e with the rule at
 *       the top of this file and the results are multiplied by gs.  h's
 *       maximum is known only after every gate/up tile, so in this mode the
 *       gate/up GEMM writes h in fp32 and a separate pass quantises it.
 * "Mixture of Experts" topic page and the Muse Spark page (Fig. 1 caption):
 * low-precision activations beside NVFP4 experts; the scale rule is this
 * library's.  Errors: MOE_FP4_ERR_INVALID_ARG. */
MOE_FP4_API int moe_fp4_set_act_scale(moe_fp4_t* h, int dynamic);

/* Residual add: with enable = 1 every later forward of this handle returns
 * out[t] = bf16_rn( x[t] + sum_j ... ), the MoE block's output added to its
 * input in the combine's fp32 sum (one rounding), as a decoder layer adds its
 * MoE output to the residual stream.  enable = 0 (default): the plain layer.
 * Not applied by moe_fp4_forward_routed.  Errors: MOE_FP4_ERR_INVALID_ARG. */
MOE_FP4_API int moe_fp4_set_residual(moe_fp4_t* h, int enable);

/* A stack of L layers on one stream: x_0 = x, x_{l+1} = forward of
 * layers[l] on x_l with router_w[l] (each handle's own options: threshold,
 * norm, residual, activation scale), out = x_L.  While layer l streams its
 * experts, its expert kernel prefetches layer l+1's router weights into L2,
 * so the next routing starts from L2 ("Optimizing Muse Spark Open on TPU v7
 * with SGLang-TorchTPU", sections 1-2: one program over all layers, the next
 * layer's weights fetched while the current layer computes).  Layer l < L-1
 * writes into its own handle's staging buffer, so consecutive entries must be
 * different handles; all on the same device with the same d.  Every argument
 * and workspace is checked before anything runs.  Asynchronous on `stream`;
 * capturable into one CUDA graph once every handle has reserved T tokens.
 * Errors: as moe_fp4_forward, and MOE_FP4_ERR_INVALID_ARG for L < 1, a null
 * entry, equal consecutive handles, or x overlapping out. */
MOE_FP4_API int moe_fp4_forward_layers(moe_fp4_t* const* layers, int L, const void* x_bf16, int T,
                                       const float* const* router_w, void* out_bf16, cudaStream_t stream);

/* Bound of every device-side wait of this handle's kernels, in milliseconds
 * (default 2000, or MOE_FP4_WAIT_TIMEOUT_MS at create time); ms >= 1.  A
 * wait that exceeds it records MOE_FP4_ERR_DEVICE_TIMEOUT in the device error
 * word and the kernel returns.  Errors: MOE_FP4_ERR_INVALID_ARG. */
MOE_FP4_API int moe_fp4_set_wait_timeout_ms(moe_fp4_t* h, int ms);

/* Test hook for the failure path (no counterpart on the pages): with
 * enable = 1 the light-class down tiles wait for a completion count that is
 * never reached, so each such wait runs out after the wait bound, records
 * MOE_FP4_ERR_DEVICE_TIMEOUT and the kernel drains the copies it issued and
 * returns; the forward's output is then undefined.  enable = 0 (default)
 * restores normal operation.  After moe_fp4_get_device_error has read the
 * error, the handle is usable again.  Errors: MOE_FP4_ERR_INVALID_ARG. */
MOE_FP4_API int moe_fp4_set_unreachable_wait(moe_fp4_t* h, int enable);

/* Stage timing (profiling hook).  With n = 9, every later forward records,
 * on the forward's stream, events[0] before the router, events[1] after the
 * router (and x staging), events[2] after top-k, events[3] after the
 * permutation, events[4] after the dense-class activation quantiser,
 * events[5] after the dense gate/up + SwiGLU GEMM, events[6] after the dense
 * down GEMM (4-6 follow 3 directly when T < thr and no expert can be dense;
 * with at most 32 (token, expert) pairs the router kernel also runs top-k and
 * the permutation, so 2 and 3 follow 1 directly),
 * events[7] after the light-class expert kernels and events[8] after the
 * combine (as external event nodes when the stream is being captured into a
 * CUDA graph).  The events must be created with timing enabled; the caller
 * owns them.  n = 0 (events may be NULL) turns the hook off.  Any other n is
 * MOE_FP4_ERR_INVALID_ARG.  Recording between stages serialises kernels that
 * would otherwise overlap through programmatic dependent launch. */
MOE_FP4_API int moe_fp4_set_stage_events(moe_fp4_t* h, cudaEvent_t* events, int n);

/* Read and clear the device error word (synchronises the handle's whole
 * device, not only one stream, so it waits for other work on that device
 * too).  *code receives MOE_FP4_OK or the first MOE_FP4_ERR_* a kernel
 * recorded; after an error the handle's completion counters are reset so
 * the next forward runs normally.  Errors: MOE_FP4_ERR_INVALID_ARG,
 * MOE_FP4_ERR_CUDA. */
MOE_FP4_API int moe_fp4_get_device_error(moe_fp4_t* h, int* code);

/* Allocation-free routing: fp32 router logits, top-k (ties to the lower
 * expert index) and the renormalised weights of every token, exactly the
 * topk_ids / topk_w that moe_fp4_forward_ex reports, for callers that cannot
 * call cudaMalloc: code that runs inside stream capture, under an external
 * memory pool or allocator that owns all device memory, or in a process
 * whose device memory budget is fixed in advance.  It needs no handle (a
 * handle allocates) and allocates nothing: the logits live in a scratch
 * array of MOE_FP4_STATIC_MAX_LOGITS floats (256 KB) that the library defines
 * as a file-scope device array; every GPU that loads the library holds it
 * until the process exits.  The pages this library follows have no
 * counterpart of this call.
 *   x_bf16    device, bf16 [T][d];   router_w device, fp32 [E][d]
 *   topk_ids  device, int32 [T][top_k];   topk_w device, fp32 [T][top_k]
 *   T >= 0 (0 is a no-op), T*E <= MOE_FP4_STATIC_MAX_LOGITS (else
 *   MOE_FP4_ERR_UNSUPPORTED), E, top_k, d as in moe_fp4_create; pointers
 *   16-byte aligned (else MOE_FP4_ERR_INVALID_ARG).
 * The first call on each device looks the scratch array up on that device
 * (cudaGetSymbolAddress) and keeps the address for the life of the process;
 * make that first call before any stream capture.  The kept address does not
 * survive cudaDeviceReset: no call may follow a reset of that device.
 * Asynchronous on `stream`.  All calls share the one scratch array per
 * device: calls whose executions overlap on the GPU (different streams
 * without ordering) race and give undefined results. */
#define MOE_FP4_STATIC_MAX_LOGITS 65536
MOE_FP4_API int moe_fp4_route_topk_static(const void* x_bf16, int T, int d, const float* router_w,
                                          int E, int top_k, int32_t* topk_ids, float* topk_w,
                                          cudaStream_t stream);

/* The CUDA runtime error behind the last MOE_FP4_ERR_CUDA returned to the
 * calling thread (error name, text and the library source line), or "" if
 * there was none.  The string is owned by the library and stays valid until
 * the thread's next failing call. */
MOE_FP4_API const char* moe_fp4_last_error_detail(void);

/* Static text for a status code. */
MOE_FP4_API const char* moe_fp4_status_string(int status);

/* Release every device buffer the handle owns; NULL is allowed. */
MOE_FP4_API void moe_fp4_destroy(moe_fp4_t* h);

#ifdef __cplusplus
}
#endif
#endif /* MOE_FP4_H */
