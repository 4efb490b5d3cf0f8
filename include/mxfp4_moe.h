/*
 * mxfp4_moe.h -- C ABI of the MXFP4 mixture-of-experts decode layer for
 * NVIDIA B200 (sm_100a).
 *
 * The layer (sources: "NVIDIA 在单台 DGX Spark 上叠加三项优化，Ling-3.0-flash 的
 * MoE 推理吞吐提升 42.5%" (tanhow.com), section "Ling 3.0 是什么" sparse-MoE
 * bullet: each MoE layer routes a token to 8 of 512 routed experts plus 1
 * shared expert; section "三项优化是什么？" item 1: experts of width 768;
 * item 2: LM head 157,184 x 2,560, hence hidden 2560; section
 * "为什么 DGX Spark 上的 MoE 解码是内存受限的？": decode is weight-read bound
 * and runs the W4A8 recipe; devotd.net retelling, section 2: MXFP4 is a
 * blocked 4-bit float format):
 *
 *   logits  l[t,e] = f32( sum_k x[t,k] W_r[e,k] ) (+ b[e])     float64 sum
 *   ids     top_k experts by descending logit, ties -> lower index
 *   w       softmax over the selected logits (= softmax, keep top_k, renormalise)
 *   xq, xs  FP8 E4M3 codes of x / xs, xs = amax(|x_t|) / 448 (one per token)
 *   g, u    MXFP4 gate / up GEMV on xq, times xs
 *   h       silu(g) * u, re-quantised to FP8 per (token, expert): qh, sh
 *   y[t]    bf16( sum_i w[t,i] Down_{ids[t,i]}(qh) sh + sum_s Down_shared_s(qh) sh )
 *
 * MXFP4 (OCP Microscaling Formats v1.0): 32 consecutive elements along K
 * (the input dimension of a matrix) share one E8M0 scale 2^(e-127); each
 * element is a 4-bit E2M1 code (bit 3 sign, 2 exponent bits, 1 mantissa
 * bit).  Two codes per byte, element 2j in the low nibble of byte j.
 *
 * Conventions of every entry point:
 *  - Pointers marked "device" are CUDA device pointers owned by the caller;
 *    the library never frees them and never copies weights.  Every device
 *    pointer must be 16-byte aligned.
 *  - Work is enqueued on the given stream; no call synchronises the host
 *    except moe_create, moe_destroy and moe_device_error.
 *  - Return value: MOE_OK (0) or a negative MOE_ERR_* code.  Nothing throws
 *    or aborts across the ABI.  moe_strerror() names a code.
 *  - A handle holds one workspace and is not safe for concurrent use from
 *    several streams or threads.
 */
#ifndef MXFP4_MOE_H
#define MXFP4_MOE_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_OK 0
#define MOE_ERR_ARG (-1)         /* null pointer, T <= 0, T > max_tokens, ...  */
#define MOE_ERR_SHAPE (-2)       /* hidden/inter not multiples of 32, top_k, E  */
#define MOE_ERR_ALIGN (-3)       /* a pointer is not 16-byte aligned           */
#define MOE_ERR_CUDA (-4)        /* a CUDA call or launch failed               */
#define MOE_ERR_TIMEOUT (-5)     /* a bounded device-side wait gave up          */
#define MOE_ERR_UNSUPPORTED (-6) /* size outside what this build implements    */
#define MOE_ERR_DEVICE (-7)      /* device-side input check failed (bad ids)   */

#define MOE_MAX_EXPERTS 512
#define MOE_MAX_TOPK 8
#define MOE_MAX_SHARED 2
#define MOE_GEMV_MAX_TOKENS 4    /* T above this takes the grouped-GEMM path  */

typedef struct moe_handle_s* moe_handle;

typedef struct {
  int32_t hidden;     /* H, multiple of 64, <= 16384 (2560)               */
  int32_t inter;      /* I, expert width, multiple of 64, <= 4096 (768)   */
  int32_t n_experts;  /* E routed experts, 1..512                          */
  int32_t top_k;      /* experts per token, 1..8 and <= E                  */
  int32_t n_shared;   /* shared experts, 0..2, added with weight 1         */
} moe_config;

/* MXFP4 expert weights in the plain (canonical) layout, device pointers.
 * Expert arrays hold the routed experts 0..E-1 followed by the shared
 * experts E..E+n_shared-1, each expert contiguous:
 *   w13_codes  [E+S][2I][H/2]  rows 0..I-1 gate, rows I..2I-1 up (uint8)
 *   w13_scales [E+S][2I][H/32] E8M0 exponents (uint8)
 *   w2_codes   [E+S][H][I/2]   down projection
 *   w2_scales  [E+S][H][I/32]
 * E8M0 exponent 255 (NaN) is not supported.  This is the input of
 * moe_pack_weights; the layer itself reads the packed layout below. */
typedef struct {
  const uint8_t* w13_codes;
  const uint8_t* w13_scales;
  const uint8_t* w2_codes;
  const uint8_t* w2_scales;
} moe_mxfp4_weights;

/* Weights of one layer as the kernels read them (device pointers, borrowed:
 * they must stay valid while the handle is used):
 *   router_w   [E][H]  bfloat16 bit patterns (uint16)
 *   router_bias[E]     float32, or NULL for no bias
 *   w13        [E+S][I/8][MOE_W13_TILE_BYTES(H)]  packed gate/up tiles
 *   w2         [E+S][H/16][MOE_W2_TILE_BYTES(I)]  packed down tiles
 * The packed arrays hold exactly the bytes of the canonical layout,
 * reordered by moe_pack_weights so that every 16-row tile of every 32-element
 * block is contiguous in the order the tensor-core fragments are loaded
 * (see moe_pack_weights). */
typedef struct {
  const uint16_t* router_w;
  const float* router_bias;
  const uint8_t* w13;
  const uint8_t* w2;
} moe_weights;

#define MOE_W13_TILE_BYTES(H) (272 * ((H) / 32))  /* 8 gate + 8 up rows */
#define MOE_W2_TILE_BYTES(I) (272 * ((I) / 32))   /* 16 down rows */

/* Optional debug outputs of moe_forward (device pointers, each may be NULL):
 *   xq [T][H] FP8 codes of x, xs [T] their scales,
 *   h  [T][top_k+n_shared][I] float32 SwiGLU outputs,
 *   qh [T][top_k+n_shared][I] FP8 codes of h, sh [T][top_k+n_shared] scales,
 * slots in ids order, shared experts last. */
typedef struct {
  uint8_t* xq;
  float* xs;
  float* h;
  uint8_t* qh;
  float* sh;
} moe_debug;

/* Create a handle for one layer (one MoE layer of the tanhow.com page,
 * section "Ling 3.0 是什么": 8 of 512 routed experts plus 1 shared expert,
 * MXFP4 weights).  Validates the configuration (MOE_ERR_SHAPE)
 * and pointer alignment (MOE_ERR_ALIGN), then allocates a workspace sized for
 * max_tokens tokens per call (MOE_ERR_CUDA if that fails).  The weights are
 * borrowed, not copied.  *out is set only on success. */
int moe_create(const moe_config* cfg, const moe_weights* weights, int max_tokens,
               moe_handle* out);

/* Route T tokens (the routing step of tanhow.com, "Ling 3.0 是什么": each
 * token picks top_k of the routed experts): x [T][H] bfloat16 (device) ->
 * topk_ids [T][top_k] int32
 * (descending logit, ties to the lower expert index), topk_w [T][top_k]
 * float32 (renormalised softmax weights, sum 1), expert_counts [E] int32
 * (tokens per routed expert; may be NULL).  One kernel launch.
 * Errors: MOE_ERR_ARG for null pointers or T outside 1..max_tokens. */
int moe_route(moe_handle h, const uint16_t* x, int T, int32_t* topk_ids, float* topk_w,
              int32_t* expert_counts, cudaStream_t stream);

/* Run the experts of T tokens and combine (the W4A8 expert step of
 * tanhow.com, "为什么 DGX Spark 上的 MoE 解码是内存受限的？": MXFP4 weights
 * against FP8 activations; plus the shared expert of "Ling 3.0 是什么"):
 * x [T][H] bfloat16 (device), the
 * routing from moe_route (or any ids in 0..E-1 and weights the caller
 * chooses), y [T][H] bfloat16 (device, written).  dbg may be NULL.
 * T <= MOE_GEMV_MAX_TOKENS runs the fused decode kernel (one launch: FP8
 * quantisation of x, gate/up + SwiGLU, FP8 re-quantisation of h, down and
 * the weighted combine with the shared experts); larger T runs the dispatch +
 * grouped-GEMM path (tcgen05 or mma.sync kernels, see moe_set_prefill_kernel).
 * Ids outside 0..E-1 are skipped and recorded (see
 * moe_device_error).  Errors: MOE_ERR_ARG, MOE_ERR_UNSUPPORTED. */
int moe_forward(moe_handle h, const uint16_t* x, int T, const int32_t* topk_ids,
                const float* topk_w, uint16_t* y, const moe_debug* dbg,
                cudaStream_t stream);

/* moe_route followed by moe_forward: the same ids, weights, counts and y as
 * the two calls (the routing step of "Ling 3.0 是什么" on the tanhow.com page
 * -- 8 of 512 routed experts plus the shared one -- followed by the experts).
 * For decode and speculative verification (T in 1..MOE_GEMV_MAX_TOKENS) it is
 * ONE kernel launch; larger T (up to the handle's max_tokens) runs moe_route
 * and then the many-token kernels.  topk_ids/topk_w [T][top_k] and
 * expert_counts [E] (may be NULL) are written; the other arguments as for
 * moe_forward.  The single launch requires the whole grid (one CTA per SM)
 * to be resident at once: a launch that shares the GPU with long-running
 * kernels on other streams waits for them, and gives up with
 * MOE_ERR_TIMEOUT (moe_device_error) after a second.
 * Errors: MOE_ERR_ARG, MOE_ERR_ALIGN, MOE_ERR_UNSUPPORTED (shapes whose
 * tiles do not fit in shared memory). */
int moe_decode(moe_handle h, const uint16_t* x, int T, int32_t* topk_ids, float* topk_w,
               int32_t* expert_counts, uint16_t* y, const moe_debug* dbg,
               cudaStream_t stream);

/* moe_forward without a handle and without allocating anything.  The pages
 * describe no such call; it exists for host code that cannot allocate device
 * memory -- a serving engine that has given all device memory to its own
 * pool, or a plugin that may not call cudaMalloc (which can also block the
 * device) -- and so cannot call moe_create, which allocates a workspace.
 * The experts run exactly as in moe_forward (same kernel and results), with
 * their scratch memory (SwiGLU outputs, per-expert amax, counters, the
 * shared-row-tile counters and float64 row sums: about 691 KB) in one fixed array inside
 * this library, which every GPU that loads the library keeps until the
 * process exits.
 *   - Limits: T in 1..MOE_GEMV_MAX_TOKENS, inter <= 1024 and hidden <= 4096;
 *     anything larger returns MOE_ERR_UNSUPPORTED.  Other arguments as for moe_forward
 *     (cfg/weights as for moe_create; packed weights), no debug outputs.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before capturing a stream into a graph.
 *   - Every call on a device shares the one array: calls that overlap on the
 *     GPU (other streams, other threads) race and give wrong results.  The
 *     first call clears the parts that must start at zero; every call that
 *     completes leaves them zero again, so a call issues only its kernel.
 *   - Device-side errors (an expert id outside 0..E-1, skipped; a bounded
 *     wait that gave up) are kept in the array and reported by
 *     moe_forward_static_device_error, which must be called after an error
 *     before the next moe_forward_static on that device.
 * Errors: MOE_ERR_ARG, MOE_ERR_SHAPE, MOE_ERR_ALIGN, MOE_ERR_UNSUPPORTED,
 * MOE_ERR_CUDA. */
int moe_forward_static(const moe_config* cfg, const moe_weights* weights, const uint16_t* x, int T,
                       const int32_t* topk_ids, const float* topk_w, uint16_t* y,
                       cudaStream_t stream);

/* Synchronise the stream and report (then clear) the device-side errors of
 * earlier moe_forward_static calls on the current device, as
 * moe_device_error does for a handle: MOE_ERR_DEVICE for out-of-range expert
 * ids, MOE_ERR_TIMEOUT if a bounded wait inside the kernel gave up.  After
 * an error it also clears the array's counters and accumulators.  Allocates
 * nothing.  Errors: MOE_ERR_CUDA. */
int moe_forward_static_device_error(cudaStream_t stream);

/* A chained stack of layers run by ONE persistent launch per call (decode
 * of a whole model's MoE layers for 1..MOE_GEMV_MAX_TOKENS tokens).  The
 * pages chain MoE layers through the rest of the model, which is not part of
 * this library; between layers the stack applies the harness step of
 * moe_residual_rmsnorm (residual add, RMS normalisation without a learned
 * weight):  for l in 0..L-1:  y = layer_l(x) (routing inside);
 *   r = bf16(r + y);  x = bf16(r / sqrt(mean(r^2) + eps)).
 * The next layer's router rows and shared-expert tiles stream into shared
 * memory while the current layer finishes.
 *
 * moe_stack_create: layers[0..n_layers-1] are existing handles with the same
 * moe_config (their weights are borrowed; the handles must outlive the
 * stack); allocates the stack's own workspace.  n_layers <= 128.
 * Errors: MOE_ERR_ARG, MOE_ERR_SHAPE (configs differ), MOE_ERR_UNSUPPORTED,
 * MOE_ERR_CUDA. */
typedef struct moe_stack_s* moe_stack;
int moe_stack_create(const moe_handle* layers, int n_layers, moe_stack* out);

/* Run the stack on T tokens: r [T][H] and x [T][H] bfloat16 (device) hold
 * the residual and the first layer's input on entry, the final residual and
 * normalised x on return (in place).  topk_ids/topk_w [L][T][top_k] receive
 * every layer's routing and x_layers [L][T][H] every layer's input x (each
 * may be NULL).  Requires the whole grid (one CTA per SM) to be resident at
 * once, as moe_decode.  Errors: MOE_ERR_ARG (T outside 1..max_tokens of the
 * layers, at most MOE_GEMV_MAX_TOKENS), MOE_ERR_ALIGN, MOE_ERR_UNSUPPORTED,
 * MOE_ERR_CUDA; device-side errors via moe_stack_device_error. */
int moe_stack_decode(moe_stack s, uint16_t* r, uint16_t* x, int T, float eps, int32_t* topk_ids,
                     float* topk_w, uint16_t* x_layers, cudaStream_t stream);

/* As moe_device_error, for a stack. */
int moe_stack_device_error(moe_stack s, cudaStream_t stream);

/* As moe_profile_begin / moe_profile_end, for a stack (kernel id 1). */
int moe_stack_profile_begin(moe_stack s, int max_launches);
int moe_stack_profile_end(moe_stack s, float* ms, int* launches);

/* Free the stack's workspace (synchronises the device first).  NULL is
 * accepted.  The layer handles are not touched. */
int moe_stack_destroy(moe_stack s);

/* Synchronise the stream and report (then clear) device-side errors
 * recorded by earlier calls: MOE_ERR_DEVICE for out-of-range expert ids,
 * MOE_ERR_TIMEOUT if a bounded wait inside a kernel gave up. */
int moe_device_error(moe_handle h, cudaStream_t stream);

/* Which kernel path the last moe_forward on this handle launched:
 * 1 = fused decode kernel (T <= MOE_GEMV_MAX_TOKENS), 2 = grouped GEMM on
 * mma.sync with exact block sums, 3 = grouped GEMM on tcgen05 (block-scaled
 * MMA, float32 accumulation in tensor memory), 0 = none yet. */
int moe_last_path(moe_handle h);

/* Kernels of the many-token path (T > MOE_GEMV_MAX_TOKENS).
 *   MOE_PREFILL_AUTO    tcgen05 grouped GEMMs when the shape allows them
 *                       (hidden a multiple of 128),
 *                       else the mma.sync kernels (the default);
 *   MOE_PREFILL_TCGEN05 always the tcgen05 kernels (MOE_ERR_UNSUPPORTED if
 *                       the shape does not allow them);
 *   MOE_PREFILL_EXACT   the mma.sync kernels, whose 32-element block sums are
 *                       exact and scaled and summed in float64 like the decode
 *                       kernel's (h then matches the float64 definition up to
 *                       its final rounding to float32).
 * The tcgen05 kernels sum the scaled block products in float32 inside the
 * tensor cores, so h carries float32 rounding of the K-long sum.
 * Errors: MOE_ERR_ARG (bad handle or kind), MOE_ERR_UNSUPPORTED. */
#define MOE_PREFILL_AUTO 0
#define MOE_PREFILL_TCGEN05 1
#define MOE_PREFILL_EXACT 2
int moe_set_prefill_kernel(moe_handle h, int kind);

/* Per-kernel timing.  moe_profile_begin(h, n) makes the following calls on
 * this handle record a CUDA event pair around each kernel they launch (up to
 * n launches; further launches are not timed).  moe_profile_end synchronises,
 * writes for each kernel id -- 0 router, 1 gate/up + SwiGLU, 2 down + combine,
 * 3 reserved -- the summed milliseconds to ms[id] and the timed launches to
 * launches[id] (arrays of MOE_PROFILE_KERNELS entries), and stops recording.
 * The events are recorded on the stream each kernel runs on.  Errors:
 * MOE_ERR_ARG, MOE_ERR_CUDA. */
#define MOE_PROFILE_KERNELS 4
int moe_profile_begin(moe_handle h, int max_launches);
int moe_profile_end(moe_handle h, float* ms, int* launches);

/* Free the workspace (synchronises the device first).  NULL is accepted. */
int moe_destroy(moe_handle h);

/* Static text for a return code. */
const char* moe_strerror(int code);

/* Reorder canonical MXFP4 expert weights into the packed layout the
 * kernels read, for experts expert0 .. expert0+n_experts-1 (shared experts
 * included by index).  No value changes: every byte of the input appears once
 * in the output.  Layout of one gate/up tile (features j0..j0+7, j0 = 8c):
 * for each 32-element block b: 256 code bytes, for lane L = 4g+t (g 0..7,
 * t 0..3) the 4 bytes 16b+4t.. of gate row j0+g then those of up row j0+g;
 * then for each block 16 scale bytes (gate row j0+g, up row j0+g) for
 * g = 0..7.  A down tile (rows n0..n0+15, n0 = 16p) is the same with row
 * n0+g in place of the gate row and n0+g+8 in place of the up row.  Output
 * buffers are caller-allocated ([E+S][I/8][MOE_W13_TILE_BYTES(H)] and
 * [E+S][H/16][MOE_W2_TILE_BYTES(I)]); the call only enqueues a kernel.
 * Errors: MOE_ERR_ARG, MOE_ERR_SHAPE, MOE_ERR_ALIGN. */
int moe_pack_weights(const moe_config* cfg, const moe_mxfp4_weights* src, int expert0,
                     int n_experts, uint8_t* w13_packed, uint8_t* w2_packed,
                     cudaStream_t stream);

/* Per-row FP8 E4M3 quantisation, the activation step of the W4A8 recipe
 * (tanhow.com retelling, "为什么 DGX Spark 上的 MoE 解码是内存受限的？";
 * devotd.net retelling, section 2: 8-bit activations) as a standalone call:
 * v [rows][cols] float32 (device) -> q [rows][cols] E4M3 codes (uint8) and
 * s [rows] float32 with s = amax/448 (IEEE division; 1 if the row is all
 * zero) and q = E4M3(v / s), round to nearest even, saturating to +-448.
 * The same encoder moe_forward applies to x and to the SwiGLU output.
 * Errors: MOE_ERR_ARG (null pointer, rows or cols < 1). */
int moe_quantize_fp8(const float* v, int rows, int cols, uint8_t* q, float* s,
                     cudaStream_t stream);

/* FP8 LM head (the output layer read in full every token; "三项优化是什么？"
 * item 2 on tanhow.com, "Online FP8 LM head" on aivibenews.ru).
 *
 * moe_lmhead_quantize: BF16 weights w [V][H] (device) -> q [V][H] FP8 E4M3
 * codes and s [V] float32, one scale per row: s = amax/448 (IEEE float32
 * division, 1 for an all-zero row), q = E4M3(w / s) with round to nearest
 * even and saturation (the activation quantiser of moe_quantize_fp8).  Run
 * once when the weights are loaded.
 *
 * moe_lmhead_logits: x [T][H] BF16 (device, T = 1..8) -> logits [T][V]
 * float32:  l[t][v] = s[v] * s_x[t] * sum_k e4m3(q[v][k]) * e4m3(qx[t][k]),
 * with x quantised per token like the MoE activations (s_x = amax/448).
 * Products are exact and summed in float32 by the tensor cores.  One
 * launch; the weights are read once for all T tokens.
 *
 * H must be a multiple of 64 (MOE_ERR_SHAPE); pointers 16-byte aligned
 * (MOE_ERR_ALIGN); null pointers, V < 1 or T outside 1..8: MOE_ERR_ARG. */
int moe_lmhead_quantize(const uint16_t* w, int V, int H, uint8_t* q, float* s, cudaStream_t stream);
int moe_lmhead_logits(const uint8_t* q, const float* s, int V, int H, const uint16_t* x, int T,
                      float* logits, cudaStream_t stream);

/* Expert parallelism: one layer's routed experts split over several GPUs.
 * The pages run the layer on one device; the layer shards naturally by
 * expert (each token uses 8 of 512 routed experts, tanhow.com "Ling 3.0
 * 是什么"), so a GPU can hold a contiguous range of the routed experts and
 * compute their part of y, with the router replicated and the parts summed
 * across GPUs (NCCL all-reduce or any other sum) before the one BF16
 * rounding.
 *
 * moe_create_ep: a handle for routed experts expert_lo .. expert_hi-1 of a
 * layer with cfg->n_experts routed experts.  local->w13 / local->w2 hold the
 * packed tiles of those experts ([expert_hi - expert_lo][...], same tile
 * layout as moe_weights), followed by the n_shared shared experts when
 * with_shared is non-zero (one GPU adds them); local->router_w and
 * router_bias are the whole router [E][H].  max_tokens <= MOE_GEMV_MAX_TOKENS.
 * moe_forward and moe_decode return MOE_ERR_UNSUPPORTED on such a handle.
 * Errors: MOE_ERR_ARG (range, max_tokens), those of moe_create.
 *
 * moe_decode_partial: routing of T <= MOE_GEMV_MAX_TOKENS tokens (every
 * GPU computes the same ids, weights and counts, as moe_decode) and this
 * handle's part of y: y_part [T][H] float32 (device) = sum over the token's
 * routed experts in the handle's range of w * FFN(x) (+ the shared experts
 * when the handle adds them), not rounded.  The sum of all parts, rounded
 * once to BF16 (moe_round_bf16), is moe_decode's y up to the float32
 * additions of the parts.  One launch.  Errors: MOE_ERR_ARG, MOE_ERR_ALIGN.
 *
 * moe_round_bf16: out[i] = BF16 bits of v[i], round to nearest even (n
 * elements, device pointers).  Errors: MOE_ERR_ARG. */
int moe_create_ep(const moe_config* cfg, const moe_weights* local, int max_tokens, int expert_lo,
                  int expert_hi, int with_shared, moe_handle* out);
int moe_decode_partial(moe_handle h, const uint16_t* x, int T, int32_t* topk_ids, float* topk_w,
                       int32_t* expert_counts, float* y_part, cudaStream_t stream);
int moe_round_bf16(const float* v, size_t n, uint16_t* out, cudaStream_t stream);

/* Harness step for chained layers (not part of the MoE layer):
 * r[t] = bf16(r[t] + y[t]) in place, then
 * x_next[t] = bf16( r[t] / sqrt(mean_k r[t,k]^2 + eps) ).  All [T][H]
 * bfloat16 device arrays.  Returns MOE_ERR_ARG on bad arguments. */
int moe_residual_rmsnorm(uint16_t* r, const uint16_t* y, uint16_t* x_next, int T, int H,
                         float eps, cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* MXFP4_MOE_H */
