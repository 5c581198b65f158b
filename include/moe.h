/*
 * moe.h — C ABI of the B200 (sm_100a) quantized MoE expert-forward library.
 *
 * The library computes the per-token MoE expert forward of the Flash-MoE
 * engine ("Flash-MoE: running a 397B parameter model on a laptop", summary
 * pages): a router picks K=4 active experts per token including one shared
 * expert ("Model architecture"); each expert's gate/up/down projections are
 * 4-bit or 2-bit group-affine dequantising matrix-vector products, w = q*s + b
 * ("Key technologies > FMA-optimised dequant kernel"); SwiGLU joins gate and
 * up; the expert outputs are combined with the router weights and the shared
 * expert's gate, added to the residual and RMS-normalised on the device before
 * the next layer ("Key technologies > Metal compute shaders" and "Deferred GPU
 * expert compute").
 *
 * Conventions for every entry point
 *  - Tensor pointers are CUDA device memory owned by the caller. The library
 *    never allocates, frees or synchronises on these calls (moe_poll_status is
 *    the one call that synchronises, by design).
 *  - bf16 values are passed as their uint16_t bit patterns; fp32 as float.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream). Every call is asynchronous on that stream.
 *  - Argument and shape errors are detected on the host before anything is
 *    launched and returned as MOE_ERR_INVALID_ARGUMENT / MOE_ERR_UNSUPPORTED /
 *    MOE_ERR_WORKSPACE; a failed launch returns MOE_ERR_CUDA. Device-side
 *    errors (an expert id out of range, a bounded wait that ran out) are
 *    latched in the workspace status word and read back with moe_poll_status.
 *  - Every device-side wait (a staged copy, a grid-wide barrier of the fused
 *    decode kernel) gives up after 100 ms, or MOE_WAIT_TIMEOUT_NS from the
 *    environment (read once, clamped to 1 ms .. 10 s), latches
 *    MOE_ERR_TIMEOUT and skips the remaining waits of the call: the outputs
 *    of a call that latched a timeout are invalid.
 *  - Supported shapes. A layer call is rejected with MOE_ERR_UNSUPPORTED,
 *    before any launch, when no kernel path fits the device:
 *      T <= 8    the digit-block decode kernels (the default): the down
 *                kernel holds every slot's SwiGLU output as digit blocks
 *                (112 bytes per 32 values) in one CTA's shared memory,
 *                (top_k + shared) * I <= 51,200 (227 KB per CTA);
 *      T > 8     the grouped prefill kernels (two stages of their ring of
 *                weight tiles must fit and their row tiles must divide the
 *                matrices), else the digit-block kernels token by token;
 *      MXFP4    (group 32), any T: the digit-block kernels, same rule;
 *    and H, I <= 8192 throughout. MOE_DECODE_KERNEL in the environment (read
 *    at every call) selects other decode kernels where they fit (the
 *    digit-block kernels otherwise): =chain the four-kernel chain, whose
 *    gate/up stages 3 experts x 8 rows x H and down up to 4 experts x 32 rows
 *    x I in one CTA (top_k 3 + shared: H <= 7552 and I <= 2688 at 4 bits,
 *    I <= 4352 at 2 bits); =fused, for single-token calls and stacks, the
 *    fused single-kernel layer: H <= 4096, top_k <= 3 (top_k + shared <= 4),
 *    E <= 4096, I <= 8 n and H <= 32 n with n = min(SMs, I, H) (148 SMs:
 *    I <= 1152), else the chain.
 *    moe_layer_forward_noalloc and moe_stack_forward apply the same rules
 *    (T = 1 for the stack), and moe_workspace_size applies the rule of
 *    T = max_tokens.
 *  - Device pointers must be 16-byte aligned; H, I must be multiples of 128
 *    (one 128-element k-span) and of the quantisation group; the group is 64.
 *  - No global state: calls on different streams with different workspaces
 *    may run concurrently.
 *
 * Packed matrix layout (the pages fix the affine form, not the packing; this
 * is the plain reading used throughout):
 *  - q: uint32 [R][K*bits/32], row-major; element k of row r sits in word
 *    k/(32/bits) at bit offset bits*(k % (32/bits)), least significant first.
 *  - scales, biases: bf16 [R][K/group]; group = `group` consecutive k of a row.
 *  - dequantised weight w[r][k] = q * scales[r][k/group] + biases[r][k/group].
 *  - gate and up are [I][H] (R = I, K = H); down is [H][I].
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARGUMENT = 1, /* NULL pointer, bad shape, misalignment   */
  MOE_ERR_UNSUPPORTED = 2,      /* bits not in {2,4}, group != 64, ...    */
  MOE_ERR_WORKSPACE = 3,        /* workspace missing or too small          */
  MOE_ERR_CUDA = 4,             /* a CUDA launch or runtime call failed    */
  MOE_ERR_TIMEOUT = 5,          /* a bounded device-side wait gave up      */
  MOE_ERR_DEVICE_FAULT = 6      /* a kernel saw an out-of-range expert id  */
} moe_status;

/* One packed matrix (device pointers). */
typedef struct {
  const uint32_t* q;
  const uint16_t* scales;
  const uint16_t* biases;
} moe_qmat;

/* One expert: gate [I][H], up [I][H], down [H][I]. */
typedef struct {
  moe_qmat gate, up, down;
} moe_expert;

/*
 * One MoE layer. Host struct; its pointers are device memory.
 *   hidden H, inter I, n_experts E (routed), top_k k (routed, k <= 8),
 *   bits in {2,4}, group = 64, has_shared in {0,1}, rms_eps > 0.
 *   bits = 4 with group = 32 selects MXFP4 experts (see moe_mxmat): each
 *   moe_qmat's q holds the E2M1 codes, its scales pointer the E8M0 bytes
 *   uint8 [R][K/32], its biases are not read (may be NULL); through
 *   moe_layer_forward and moe_layer_forward_timed (any T: above 8 tokens the
 *   router is the many-token one and the expert kernels run per token, each
 *   expert's rows read once per token that chooses it), and
 *   moe_layer_forward_noalloc and moe_stack_forward (T <= 8 / T = 1).
 *   router_w    bf16 [E][H]
 *   router_bias fp32 [E] or NULL: added to the logits before softmax/top-k
 *   experts     device array [E] of moe_expert
 *   shared      the shared expert (ignored when has_shared == 0)
 *   shared_gate_w bf16 [H] (required when has_shared): gate = sigmoid(g_s . x)
 *   rms_gamma   bf16 [H]
 */
typedef struct {
  int32_t hidden, inter, n_experts, top_k, bits, group, has_shared;
  float rms_eps;
  const uint16_t* router_w;
  const float* router_bias;
  const moe_expert* experts;
  moe_expert shared;
  const uint16_t* shared_gate_w;
  const uint16_t* rms_gamma;
} moe_layer;

/* Bytes of workspace that calls on `layer` need for up to max_tokens tokens.
 * The workspace is caller-owned device memory; it must be zeroed once
 * (moe_workspace_init) before its first use and may be reused by later calls
 * on the same stream. */
moe_status moe_workspace_size(const moe_layer* layer, int32_t max_tokens, size_t* bytes);

/* Clears the workspace header, the first 256 bytes (async on `stream`): the
 * status word, the recheck counter, and the words the decode kernels keep
 * there between calls (grid-barrier counters, per-token selection flags;
 * all 0 between calls). */
moe_status moe_workspace_init(void* ws, size_t ws_bytes, void* stream);

/*
 * Router ("Model architecture": K=4 active per token incl. one shared;
 * the router results select the experts to load — HN thread, Table 3 comment).
 *   logits = router_w . x (+ router_bias). The ranking is that of the plain
 *   fp64 definition (exact bf16 x bf16 products summed in index order from
 *   0, bias added last). The logits are computed faster, each with a
 *   rigorous bound on its distance to the definition: T <= 8 as fp64 sums
 *   in a summation tree per token (bound about 2^-39 of sum|w x| at
 *   H = 4096); T > 8 exactly, in integers on the tensor cores, on 22-bit
 *   fixed-point forms of every router row and token (one power-of-two
 *   scale each), the bound made of the rows' own rounding residuals
 *   sum|v - v~| and the fp64 rounding of the sums (about 1e-7 on unit-scale
 *   activations); the shared-gate logit is an fp64 sum of the exact
 *   products. The top-k is certified against the
 *   bounds, and when two candidates are closer than them, every candidate
 *   near the k-th is recomputed as the definition and ranked again, so the
 *   indices are those of the definition;
 *   topk_idx [T][k]: the k largest logits, descending, ties to the lower index;
 *   topk_w [T][k]: softmax over all E renormalised over the chosen k (fp32);
 *   shared_gate [T] (nullable): sigmoid(shared_gate_w . x), 0 if no shared expert.
 * x: bf16 [T][H]. The logits stay in the workspace after the call: double
 * [T][E+1] at byte offset 256, column E holding shared_gate_w . x. The
 * uint32 at byte offset 16 of the workspace counts the selections (by this
 * and the decode layer calls) that needed the exact recheck; it wraps, and
 * moe_workspace_init clears it.
 * Requires E <= 4096 and k <= 8; |w x| products must be finite in fp32.
 */
moe_status moe_route(const moe_layer* layer, const uint16_t* x, int32_t T, int32_t* topk_idx,
                     float* topk_w, float* shared_gate, void* ws, size_t ws_bytes, void* stream);

/*
 * Dequantising matrix-vector product y = W x for one packed matrix
 * ("FMA-optimised dequant kernel": (q*s + b)*x summed over k).
 *   W: host struct of device pointers, R rows (a multiple of 16), K columns
 *   (a multiple of 128), group 64.
 *   x: fp32 [K]; y: fp32 [R] (overwritten). 4-bit and 2-bit variants.
 */
moe_status moe_expert_gemv_q4(const moe_qmat* W, int32_t R, int32_t K, int32_t group,
                              const float* x, float* y, void* stream);
moe_status moe_expert_gemv_q2(const moe_qmat* W, int32_t R, int32_t K, int32_t group,
                              const float* x, float* y, void* stream);

/*
 * MXFP4 expert matrices (the experts' format on "300b on 32gb MoE-streaming
 * findings + optimisations"), read as the OCP Microscaling (MX) v1.0 format:
 * FP4 E2M1 elements (values 0, 0.5, 1, 1.5, 2, 3, 4, 6 and negatives), one
 * E8M0 scale 2^(byte - 127) per 32 consecutive k of a row (byte 0xFF: NaN);
 * weight = scale * element.
 *   q: uint32 [R][K/8], element k of a row in word k/8 at bits 4*(k%8), LSB
 *      first (the 4-bit packing); 16-byte aligned.
 *   scales: uint8 [R][K/32].
 */
typedef struct {
  const uint32_t* q;
  const uint8_t* scales;
} moe_mxmat;

/*
 * y = W x for one MXFP4 matrix (decode). R >= 1, K a multiple of 32 and at
 * most 8192 (MOE_ERR_UNSUPPORTED above); x fp32 [K] (16-byte aligned); y fp32
 * [R], overwritten. Element products and block sums in fp32, each block sum
 * times its scale. Asynchronous on `stream`; no workspace.
 */
moe_status moe_expert_gemv_mxfp4(const moe_mxmat* W, int32_t R, int32_t K, const float* x, float* y,
                                 void* stream);

/* Bytes of workspace moe_expert_gemm_mxfp4 needs for R x K and T tokens
 * (R and K multiples of 128, K <= 8192: else MOE_ERR_UNSUPPORTED). */
moe_status moe_mxfp4_workspace_size(int32_t R, int32_t K, int32_t T, size_t* bytes);

/*
 * Y[t][r] = sum_k W[r][k] x[t][k] for T tokens (prefill-shaped expert GEMM) on
 * the tcgen05 tensor cores with block scaling (kind::mxf4): the codes are used
 * as stored and the hardware applies the E8M0 scales. Each token's bf16 row is
 * written as a sum of five E2M1 terms, each with its own E8M0 scale per
 * 32-block, exact up to a residual below 4^-4/3 of the block's largest
 * |x| (about 5e-5 of the output's norm on unit-scale activations); fp32
 * accumulation in tensor memory.
 *   R, K multiples of 128, K <= 8192; x bf16 [T][K] (16-byte aligned); y fp32
 *   [T][R], overwritten; W.q 16-byte aligned, W.scales 4-byte aligned.
 *   ws: caller-owned device memory of moe_mxfp4_workspace_size bytes, 256-byte
 *   aligned, header cleared by moe_workspace_init; a bounded wait that runs out
 *   latches MOE_ERR_TIMEOUT there (moe_poll_status), and Y is then invalid.
 *   Errors before any launch: MOE_ERR_INVALID_ARGUMENT, MOE_ERR_UNSUPPORTED,
 *   MOE_ERR_WORKSPACE (ws_bytes too small).
 */
moe_status moe_expert_gemm_mxfp4(const moe_mxmat* W, int32_t R, int32_t K, const uint16_t* x, int32_t T,
                                 float* y, void* ws, size_t ws_bytes, void* stream);

/*
 * Combine + residual + RMSNorm ("MoE combine + residual + gate", "normalisation +
 * residual ... passed directly to the next layer"):
 *   h'[t] = h[t] + sum_i topk_w[t][i] * y_routed[t][i] + shared_gate[t] * y_shared[t]
 *   x_out[t] = h'[t] / sqrt(mean(h'[t]^2) + eps) * gamma
 *   y_routed fp32 [T][k][H]; topk_w fp32 [T][k]; y_shared fp32 [T][H] or NULL
 *   (then shared_gate is ignored and may be NULL); h fp32 [T][H] in/out (h');
 *   gamma bf16 [H]; x_out bf16 [T][H]; x_out_f32 fp32 [T][H] or NULL.
 *   H a multiple of 8, at most 8192 (else MOE_ERR_UNSUPPORTED).
 */
moe_status moe_combine_residual_norm(int32_t T, int32_t H, int32_t k, const float* y_routed,
                                     const float* topk_w, const float* y_shared,
                                     const float* shared_gate, float* h, const uint16_t* gamma,
                                     float eps, uint16_t* x_out, float* x_out_f32, void* stream);

/*
 * Prefill grouping of routed (token, rank) pairs by expert:
 *   counts [E], offsets [E+1] (exclusive scan of counts), perm [T*k] where
 *   perm[offsets[e] + n] is the n-th flattened index t*k + r routed to e, in
 *   increasing order (a stable sort by expert). topk_idx int32 [T][k].
 */
moe_status moe_group_tokens(int32_t T, int32_t k, int32_t E, const int32_t* topk_idx,
                            int32_t* counts, int32_t* offsets, int32_t* perm, void* ws,
                            size_t ws_bytes, void* stream);

/*
 * Whole MoE layer for T tokens: router, expert gate/up + SwiGLU, down, combine
 * with the shared-expert gate, residual and RMSNorm, all on the device with
 * no host round trip. T = 1..8 runs the digit-block decode kernels (router,
 * which also writes x as exact fixed-point digit planes; certified top-k;
 * gate/up + SwiGLU, which writes the SwiGLU outputs' digit planes; down +
 * combine + residual; RMSNorm; five launches linked by programmatic
 * dependent launch), or on request the four-kernel decode chain or, for
 * T = 1, the fused decode kernel (the whole layer in one persistent launch,
 * grid-wide barriers between its phases); larger T the prefill kernels
 * (grouping by expert, grouped dequant GEMM). See "Supported shapes" above.
 *   x_in bf16 [T][H]; h fp32 [T][H] residual in, h' out; x_out bf16 [T][H];
 *   x_out_f32 fp32 [T][H] or NULL; topk_idx int32 [T][k] or NULL;
 *   topk_w fp32 [T][k] or NULL.
 */
moe_status moe_layer_forward(const moe_layer* layer, const uint16_t* x_in, float* h, int32_t T,
                             uint16_t* x_out, float* x_out_f32, int32_t* topk_idx, float* topk_w,
                             void* ws, size_t ws_bytes, void* stream);

/*
 * L layers in sequence for one decode token: layer l's x_out feeds layer l+1
 * and h is carried in fp32 ("Deferred GPU expert compute"); each layer runs
 * the decode kernels of moe_layer_forward at T = 1. With the fused
 * kernel (MOE_DECODE_KERNEL=fused), up to 24 layers run in one launch: x and
 * h stay on the chip between layers, and the next layer's router rows and
 * shared expert are requested while the current layer finishes.
 *   layers: host array [L]; x_in bf16 [H]; h fp32 [H] in/out; x_out bf16 [H];
 *   topk_idx_all int32 [L][k] or NULL; layer_inputs bf16 [L][H] or NULL and
 *   layer_h fp32 [L][H] or NULL: each layer's input x and residual h (for
 *   teacher-forced checks). Every layer must have the same H, I, E, k, bits, group.
 */
moe_status moe_stack_forward(const moe_layer* layers, int32_t L, const uint16_t* x_in, float* h,
                             uint16_t* x_out, int32_t* topk_idx_all, uint16_t* layer_inputs,
                             float* layer_h, void* ws, size_t ws_bytes, void* stream);

/*
 * The kernel path that serves a call of T tokens on `layer` (host only,
 * launches nothing): MOE_PATH_DIGIT (decode of an affine layer, T <= 8, the
 * default: router, top-k, gate/up + SwiGLU and down + combine on digit
 * blocks of x and of the SwiGLU outputs, RMSNorm), MOE_PATH_CHAIN (the
 * four-kernel decode chain, T <= 8), MOE_PATH_FUSED (the fused decode
 * kernel, T = 1), MOE_PATH_PREFILL (T > 8) or MOE_PATH_MXFP4 (a layer of
 * MXFP4 experts, the kernels of MOE_PATH_DIGIT with E2M1 codes), and in
 * *n_events the number of events moe_layer_forward_timed records on that
 * path (its stages + 1). Either output may be NULL. For affine decode,
 * MOE_DECODE_KERNEL=chain in the environment (read at every call) selects
 * the chain and MOE_DECODE_KERNEL=fused the fused kernel where it fits.
 * Errors: those of moe_workspace_size's layer checks; MOE_ERR_UNSUPPORTED
 * when no path fits (see "Supported shapes").
 */
typedef enum {
  MOE_PATH_FUSED = 1,
  MOE_PATH_CHAIN = 2,
  MOE_PATH_PREFILL = 3,
  MOE_PATH_MXFP4 = 4,
  MOE_PATH_DIGIT = 5
} moe_path;
moe_status moe_layer_path(const moe_layer* layer, int32_t T, int32_t* path, int32_t* n_events);

/*
 * Profiling variant of moe_layer_forward: the same kernels with a CUDA event
 * recorded before the first and after each of the kernels of the layer, so a
 * caller can time them one by one. events: host array of n_events created
 * cudaEvent_t handles (passed as void*); n_events must be at least the number
 * of recorded stages + 1 (moe_layer_path reports it): digit-block decode
 * and MXFP4 5 (router, top-k, gate/up + down, norm); decode chain 5 (router,
 * gate/up, down, norm); fused decode 2 (the one kernel); prefill 6 (router,
 * top-k + grouping, gate/up, down, combine + norm). The kernels run without programmatic overlap between
 * them. Same arguments and errors otherwise.
 */
moe_status moe_layer_forward_timed(const moe_layer* layer, const uint16_t* x_in, float* h, int32_t T,
                                   uint16_t* x_out, float* x_out_f32, int32_t* topk_idx, float* topk_w,
                                   void* ws, size_t ws_bytes, void* const* events, int32_t n_events,
                                   void* stream);

/*
 * moe_layer_forward without a caller-provided workspace, for callers that
 * cannot allocate device memory themselves: for example a plug-in running
 * inside a host application that owns every device allocation and hands the
 * plug-in only its input and output buffers, or a latency-critical loop in
 * which cudaMalloc (and the device-wide synchronisation it can imply) is not
 * allowed. The Flash-MoE pages have no counterpart to this entry point; it is
 * a deployment convenience of this library.
 *
 * The scratch lives in one static device array of MOE_NOALLOC_SCRATCH_BYTES
 * inside the library; every GPU that loads the library holds it until the
 * process exits. The call allocates and frees nothing. The first call on a
 * device looks up that array's device address (once per device, with that
 * device current); make that first call before any stream capture.
 * It serves decode only: T = 1..8; T > 8 is rejected with
 * MOE_ERR_UNSUPPORTED. Layers and token counts whose workspace
 * (moe_workspace_size) exceeds MOE_NOALLOC_SCRATCH_BYTES are rejected with
 * MOE_ERR_WORKSPACE.
 * All calls share the array and it keeps the last call's contents; the
 * kernels clear what has to start at zero. The array starts zeroed, and a
 * device-side status latched by a call (MOE_ERR_TIMEOUT,
 * MOE_ERR_DEVICE_FAULT) stays in it until moe_noalloc_poll_status reads and
 * clears it. Calls whose kernels overlap on the GPU (different streams, or
 * different host threads) race on the array: order them on one stream.
 * Arguments and errors are otherwise those of moe_layer_forward.
 */
#define MOE_NOALLOC_SCRATCH_BYTES (8u << 20)
moe_status moe_layer_forward_noalloc(const moe_layer* layer, const uint16_t* x_in, float* h, int32_t T,
                                     uint16_t* x_out, float* x_out_f32, int32_t* topk_idx, float* topk_w,
                                     void* stream);

/* moe_poll_status for the static scratch of moe_layer_forward_noalloc on the
 * current device: synchronises `stream`, returns the status latched by
 * earlier no-alloc calls (MOE_OK if none) and clears it. */
moe_status moe_noalloc_poll_status(void* stream);

/*
 * Host-resident routed experts with an HBM expert cache ("Key technologies >
 * SSD expert streaming" and "Trust the OS" of the Flash-MoE write-up: the
 * experts live outside the GPU and the ones the router picks are loaded for
 * each token). Here the routed experts live in host memory and HBM holds
 * `slots` of them; a slot that has to be reused is the least recently used
 * one (free slots first, the lowest index on ties). All memory is
 * caller-owned:
 *   host_experts  host array [E] of moe_expert whose q / scales / biases point
 *                 to host memory (page-locked memory lets the copies overlap
 *                 other work); it must stay valid while the cache is used;
 *   dev           device memory of dev_bytes (256-byte aligned): the expert
 *                 table [E] the kernels read, then the slots;
 *   state         host memory of state_bytes (8-byte aligned): the
 *                 bookkeeping.
 * moe_cache_size: the two sizes for `layer` and `slots` (layer->experts is not
 * read). moe_cache_init: empties the cache (host only, no device access).
 */
moe_status moe_cache_size(const moe_layer* layer, int32_t slots, size_t* dev_bytes, size_t* state_bytes);
moe_status moe_cache_init(const moe_layer* layer, const moe_expert* host_experts, int32_t slots, void* dev,
                          size_t dev_bytes, void* state, size_t state_bytes);

/* The cache's bookkeeping for one call, host only (no copy, no device access):
 * makes the n expert ids (duplicates allowed) resident and writes, per id, its
 * slot and whether it had to be loaded (missed = 1 on the first id of each
 * loaded expert, 0 otherwise). MOE_ERR_UNSUPPORTED when the call names more
 * distinct experts than there are slots; MOE_ERR_INVALID_ARGUMENT for an id
 * outside [0, E) or a state that moe_cache_init did not set up. */
moe_status moe_cache_admit(void* state, const int32_t* ids, int32_t n, int32_t* slot, int32_t* missed);

/* moe_layer_forward with the routed experts served from the cache: routes the
 * T tokens on the GPU (moe_route), reads the chosen ids back (synchronises
 * `stream`), admits them, copies each missing expert's nine arrays host -> HBM
 * (one cudaMemcpyAsync per array) and its entry of the device expert table,
 * then runs the layer as moe_layer_forward does, with layer->experts replaced
 * by the cache's table. Arguments, workspace and errors otherwise those of
 * moe_layer_forward; T * top_k <= 4096. */
moe_status moe_layer_forward_cached(const moe_layer* layer, void* state, const uint16_t* x_in, float* h, int32_t T,
                                    uint16_t* x_out, float* x_out_f32, int32_t* topk_idx, float* topk_w, void* ws,
                                    size_t ws_bytes, void* stream);

/* Counters of the cache since moe_cache_init: distinct experts found resident
 * and loaded per call, and bytes copied host -> HBM. Pointers may be NULL. */
moe_status moe_cache_stats(const void* state, uint64_t* hits, uint64_t* misses, uint64_t* bytes_copied);

/* Synchronises `stream` and returns the status latched in the workspace by
 * earlier calls (MOE_OK if none). A latched status is cleared together with
 * the counters and flags of the workspace header (the first 256 bytes),
 * which a call that ran out of time may have left mid-round. */
moe_status moe_poll_status(void* ws, void* stream);

/* Diagnostics for the device-side failure path. Launches one warp that waits,
 * through the library's bounded wait, on a barrier phase that nothing
 * completes (no copy is issued, so nothing is in flight). After bound_ns
 * (1 ns .. 10 s) the wait gives up, MOE_ERR_TIMEOUT is latched in the
 * workspace status word, and the kernel returns normally. The timeout is
 * read back with moe_poll_status, and later calls on the same context work
 * as before. Asynchronous on `stream`.
 * Errors: MOE_ERR_WORKSPACE (ws NULL or under 256 bytes),
 * MOE_ERR_INVALID_ARGUMENT (ws not 256-byte aligned, bound out of range). */
moe_status moe_selftest_wait_timeout(void* ws, size_t ws_bytes, uint64_t bound_ns, void* stream);

/* Diagnostics for the grid-wide barrier of the fused decode kernel. One
 * thread arrives at a barrier of the workspace header as if the grid had two
 * CTAs, so the round never completes; after bound_ns (1 ns .. 10 s) its wait
 * gives up, MOE_ERR_TIMEOUT is latched and the kernel returns. The barrier's
 * arrival counter is left mid-round, as a real timeout can leave it: read the
 * status with moe_poll_status, which also clears the counters, before the
 * workspace serves another call. Errors as for moe_selftest_wait_timeout. */
moe_status moe_selftest_grid_timeout(void* ws, size_t ws_bytes, uint64_t bound_ns, void* stream);

/* Static string naming a status code. */
const char* moe_status_string(moe_status s);

/* Library ABI version (this header: 1). */
int32_t moe_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
