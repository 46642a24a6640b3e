/*
 * moe.h -- C ABI of the routed Mixture-of-Experts feed-forward layer on B200 (sm_100a).
 *
 * The layer (page "Gemma 4 26B-A4B it QAT Q4_0 with MTP assistant and vision, NInfer v3
 * artifact", table "What is inside"): 128 routed experts per block, each with [gate; up]
 * of 2 x 704 rows and down of 2,816 rows over a 2,816-wide hidden state, stored as ggml
 * Q4_0 blocks that are multiplied in place (intro: "nothing is requantized"); router,
 * router scale and expert scales are FP32.
 *
 * For each token t (x_t, bf16, width d):
 *   l_e      = sum_i W_r[e, i] x_t[i]                                   (router, FP32)
 *   ids_t    = the k experts with the largest l_e, ties to the lower index
 *   w_tj     = router_scale * softmax over the k selected logits
 *   g, u     = rows 0..f-1 and f..2f-1 of gate_up[e] applied to x_t
 *   h        = gelu_tanh(g) * u
 *   out_t[r] = sum_j w_tj * expert_scale[e_tj] * (down[e_tj] h_tj)[r]     (j = 0..k-1)
 *
 * Q4_0 block (ggml block_q4_0, 18 bytes per 32 weights): fp16 scale d (little-endian),
 * then 16 code bytes; weight i (i < 16) = ((byte_i & 15) - 8) * d, weight i + 16 =
 * ((byte_i >> 4) - 8) * d.
 *
 * Conventions for every entry point:
 *  - pointers named as device pointers must be device memory of the device given to
 *    moe_init; the caller owns them; the library never frees or retains them;
 *  - `stream` is a cudaStream_t (0 = legacy default stream); work is enqueued on it and
 *    the call returns without synchronising;
 *  - the return value is MOE_OK (0) or a negative MOE_ERR_*; moe_last_error() then
 *    describes the failure. Argument errors are detected before anything is enqueued.
 *  - one process-wide context: calls are not thread-safe, and forwards that overlap on
 *    different streams race on the shared workspace.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_OK 0
#define MOE_ERR_NOT_INIT (-1)            /* moe_init has not succeeded */
#define MOE_ERR_BAD_ARG (-2)             /* null pointer, bad shape, limit exceeded */
#define MOE_ERR_BAD_ALIGN (-3)           /* a pointer is not 16-byte aligned */
#define MOE_ERR_CUDA (-4)                /* a CUDA runtime call or launch failed */
#define MOE_ERR_DEVICE_TIMEOUT (-5)      /* a bounded device-side wait expired */
#define MOE_ERR_UNSUPPORTED_DEVICE (-6)  /* not an sm_100 device */

/* Path selection for moe_layer_forward. */
#define MOE_PATH_AUTO 0   /* GEMV when T <= the GEMV token limit, else grouped GEMM */
#define MOE_PATH_GEMV 1   /* FP32-accumulate Q4_0 GEMV path (decode) */
#define MOE_PATH_GEMM 2   /* bf16 tcgen05 grouped-GEMM path (prefill) */
#define MOE_PATH_GEMV_SPLIT 3   /* GEMV path as separate routing / gate_up / down kernels
                                   (MOE_PATH_GEMV uses one fused kernel when T <= 8) */

/*
 * moe_init: select `device`, check it is sm_100, and allocate the workspace for passes of
 * up to max_tokens tokens (longer calls run in chunks of max_tokens) with d <= max_d,
 * f <= max_f, E <= max_E, k <= max_k. Calling it again releases the previous context first.
 * Limits: 1 <= max_E <= 512, 1 <= max_k <= max_E, max_d and max_f multiples of 32.
 */
int moe_init(int device, int max_tokens, int max_d, int max_f, int max_E, int max_k);

/*
 * moe_layer_forward: one routed-MoE layer for T tokens.
 *   x            device, bf16 [T, d] row-major (uint16 bit patterns)
 *   router_w     device, fp32 [E, d] row-major
 *   router_scale device, fp32 [1]; multiplies every combine weight
 *   gate_up_q4   device, Q4_0 [E][2f][d/32] blocks (18 B each), expert-major, rows 0..f-1
 *                gate and f..2f-1 up; 16-byte aligned
 *   down_q4      device, Q4_0 [E][d][f/32] blocks, expert-major; 16-byte aligned
 *   expert_scale device, fp32 [E]
 *   T            tokens, T >= 0 (T = 0 is a no-op). A call with T > max_tokens runs as
 *                consecutive chunks of max_tokens tokens on the path the whole call selects,
 *                so the workspace stays bounded by moe_init's limits whatever T is; the
 *                output equals one pass's bit for bit (a token's output depends only on its
 *                own x).
 *   d, f, E, k   hidden width, expert width, experts, experts per token; d % 32 == 0,
 *                f % 32 == 0, 1 <= k <= E, all within the moe_init limits
 *   out          device, fp32 [T, d] row-major; written, never read
 *   stream       cudaStream_t
 * Deterministic: the same inputs give bitwise identical outputs. NaN/Inf in the inputs
 * propagate to the outputs (expert selection among NaN logits is then unspecified).
 * A device-side wait that ran out of time is reported by the next call that checks the
 * error word (this one or moe_debug_check) as MOE_ERR_DEVICE_TIMEOUT.
 */
int moe_layer_forward(const void *x, const float *router_w, const float *router_scale,
                      const uint8_t *gate_up_q4, const uint8_t *down_q4,
                      const float *expert_scale, int T, int d, int f, int E, int k,
                      float *out, void *stream);

/*
 * moe_block_forward: the block's feed-forward output, the routed layer plus the block's dense
 * MLP (same page, table "What is inside": the dense MLP's gate and up rows are one Q4_0
 * parent; the page gives no width, so it is an argument, and the MLP is read as a GELU-tanh
 * GeGLU whose output is added to the routed combine):
 *   out_t = [moe_layer_forward]_t + Wd_dense (gelu_tanh(Wg_dense x_t) * (Wu_dense x_t))
 *   gate_up_dense_q4  device, Q4_0 [2 f_dense][d/32] blocks: gate rows 0..f_dense-1, then up
 *                     rows; 16-byte aligned
 *   down_dense_q4     device, Q4_0 [d][f_dense/32] blocks; 16-byte aligned
 *   f_dense           positive multiple of 32, <= max_f of moe_init
 * Other arguments as moe_layer_forward. The dense MLP runs through the layer's own kernels as
 * one more expert that every token selects with weight 1, in a pass of its own (after the
 * routed pass of each chunk) whose combine adds into out.
 */
int moe_block_forward(const void *x, const float *router_w, const float *router_scale,
                      const uint8_t *gate_up_q4, const uint8_t *down_q4, const float *expert_scale,
                      const uint8_t *gate_up_dense_q4, const uint8_t *down_dense_q4, int T, int d,
                      int f, int f_dense, int E, int k, float *out, void *stream);

/*
 * Pieces of the layer for an expert-parallel deployment (experts spread over several GPUs:
 * the routing and the final sum stay with the tokens, the expert rows travel to the GPU that
 * holds their experts and back).
 *
 * moe_route: the layer's selection alone, ids int32 [T, k] and w fp32 [T, k] (as
 *   moe_debug_get_routing describes them) for T tokens, written to the caller's device
 *   buffers; the same selection moe_layer_forward makes (the decode routing up to 16 tokens,
 *   the tiled router product above).
 * moe_experts_forward: experts on rows the caller has routed, one expert per row:
 *   out_rows[r] = row_weight[r] * expert_scale[e_r] * Wd_e (gelu_tanh(Wg_e x_r) * (Wu_e x_r)),
 *   e_r = row_expert[r] in [0, E) (an id outside it gives that row 0 and makes the next
 *   checking call return MOE_ERR_BAD_ARG); x_rows bf16 [R, d], out_rows fp32 [R, d]; the
 *   GEMV path up to the AUTO threshold, the grouped GEMM above; R > max_tokens in chunks.
 * moe_gather_rows: dst[i, :] = src[index[i], :] for i < n, rows of row_bytes (a multiple of
 *   16), 16-byte aligned bases; index int32 device [n].
 * moe_combine_slots: out[t, :] = sum_{j < k} y_slots[t k + j, :] in j order; fp32, d % 4 == 0.
 */
int moe_route(const void *x, const float *router_w, const float *router_scale, int T, int d, int E, int k,
              int32_t *ids, float *w, void *stream);
int moe_experts_forward(const void *x_rows, const int32_t *row_expert, const float *row_weight,
                        const uint8_t *gate_up_q4, const uint8_t *down_q4, const float *expert_scale,
                        int R, int d, int f, int E, float *out_rows, void *stream);
int moe_gather_rows(const void *src, const int32_t *index, int n, size_t row_bytes, void *dst, void *stream);
int moe_combine_slots(const float *y_slots, int T, int d, int k, float *out, void *stream);

/*
 * moe_rmsnorm_bf16: the fixed normalisation between stacked layers,
 *   x[t, i] = bf16_rne(y[t, i] / sqrt(mean_i y[t, i]^2 + eps))   (unit gain, FP32 math)
 *   y  device fp32 [T, d];  x_out device bf16 [T, d];  1 <= d, T >= 0.
 */
int moe_rmsnorm_bf16(const float *y, void *x_out, int T, int d, float eps, void *stream);

/*
 * moe_stack_forward: L routed-MoE layers, layer i+1 reading moe_rmsnorm_bf16(eps) of
 * layer i's output. Per-layer weights come as host arrays of L device pointers.
 *   x_in     device bf16 [T, d], input of layer 0
 *   out      device fp32 [T, d], output of layer L-1
 *   x_trace  optional device bf16 [L, T, d]: receives each layer's input (NULL to skip)
 * Same shape rules as moe_layer_forward (a call above max_tokens runs the whole stack on one
 * chunk of tokens after another). The inter-layer activations live in the workspace.
 * Layers that take the fused decode kernel apply the normalisation inside that kernel (the
 * same arithmetic and bits as moe_rmsnorm_bf16), so such a stack is one launch per layer.
 */
int moe_stack_forward(const void *x_in, int L, const float *const *router_w,
                      const float *const *router_scale, const uint8_t *const *gate_up_q4,
                      const uint8_t *const *down_q4, const float *const *expert_scale,
                      int T, int d, int f, int E, int k, float eps, float *out,
                      void *x_trace, void *stream);

/* moe_set_path: force a path (MOE_PATH_*); gemv_max_tokens sets the AUTO threshold
 * (default 16). Returns MOE_ERR_BAD_ARG for an unknown path. */
int moe_set_path(int path, int gemv_max_tokens);

/* moe_destroy: synchronise the device and free the workspace. Safe to call twice. */
void moe_destroy(void);

/* moe_last_error: text for the last non-zero return of this library (static storage). */
const char *moe_last_error(void);

/*
 * moe_debug_get_routing: copy the routing of the last pass (the last chunk of a chunked call) of
 * the last moe_layer_forward (device-to-device,
 * enqueued on `stream`): ids int32 [T, k] (per token, logit descending, ties by index),
 * w fp32 [T, k], counts int32 [E], offsets int32 [E + 1], perm int32 [T * k] (slot
 * s = t * k + j of the r-th row of expert e sits at perm[offsets[e] + r], in increasing s).
 * Any destination may be NULL. Intended for tests.
 */
int moe_debug_get_routing(int32_t *ids, float *w, int32_t *counts, int32_t *offsets,
                          int32_t *perm, void *stream);

/*
 * moe_debug_get_hidden: copy h = gelu_tanh(g) * u of the last forward, fp32 [T * k, f] in
 * slot order (slot s = t * k + j), device-to-device on `stream`. Intended for tests.
 */
int moe_debug_get_hidden(float *h, void *stream);

/* moe_debug_check: synchronise `stream` and report the device error word (timeouts). After a
 * reported timeout the next forward first zeroes the workspace's arrival counters. */
int moe_debug_check(void *stream);

/*
 * Failure detection, for tests. Every device-side wait (mbarrier phases, arrival counters,
 * polls of launch-tagged words) is bounded; a wait that runs out records
 * MOE_ERR_DEVICE_TIMEOUT in the error word, the kernel ends on its own (it waits, again
 * bounded, for its copies in flight first) and the context stays usable.
 *   moe_debug_set_wait_ns: bound of every device-side wait of later forwards, in
 *     nanoseconds (0 restores the default of 2 s).
 *   moe_debug_inject: make the next forward simulate a fault by skipping one step --
 *     MOE_INJECT_SKIP_ROUTER_ARRIVAL: in the fused decode kernel, CTA 0 never stores its
 *     router logits, so every CTA's wait for them runs out. Cleared by that forward.
 */
#define MOE_INJECT_NONE 0
#define MOE_INJECT_SKIP_ROUTER_ARRIVAL 1
int moe_debug_set_wait_ns(unsigned long long ns);
int moe_debug_inject(int fault);

/*
 * Per-kernel timing with CUDA events, for measurement. After moe_profile_begin, every
 * kernel-group launch of the following forwards is bracketed by two events recorded on the
 * launch stream. moe_profile_end synchronises on them and writes, per group, the summed
 * milliseconds and the number of launches (arrays of MOE_PROF_GROUPS entries, may be NULL).
 * Groups: 0 routing (router, top-k, permutation), 1 decode gate_up GEMV + GeGLU, 2 decode
 * down GEMV + combine, 3 prefill gate_up grouped GEMM + GeGLU, 4 prefill down grouped GEMM,
 * 5 prefill combine, 6 RMSNorm, 7 fused decode kernel (routing to combine in one launch). Recording events serialises nothing but does separate the
 * launches, so a timed forward can run slightly slower than an untimed one.
 */
#define MOE_PROF_GROUPS 8
int moe_profile_begin(void);
int moe_profile_end(float *ms_total, int *launches);
/* moe_profile_kernel_launches: kernels this library launched (or recorded into a stream
 * capture) since the last moe_profile_begin; a group above can hold several kernels. */
long long moe_profile_kernel_launches(void);

/*
 * moe_layer_forward_static: the decode (FP32-accumulate GEMV) path of moe_layer_forward, for
 * callers that cannot let a library allocate device memory -- serving engines that reserve
 * all device memory in their own pool, plugins inside a host that owns every allocation,
 * loops that cannot afford an allocation's implicit synchronisation. It needs no moe_init
 * and calls no cudaMalloc / cudaFree: its scratch is a fixed static device array of
 * MOE_STATIC_SCRATCH_BYTES that every GPU loading this library holds until the process
 * exits. The pages have no counterpart of this entry point; it exists for library users.
 *   Arguments, layouts and results as moe_layer_forward (same kernels, same bits), on the
 *   current device. Limits: T <= MOE_STATIC_MAX_TOKENS, T * k <= MOE_STATIC_MAX_SLOTS,
 *   d <= MOE_STATIC_MAX_D, f <= MOE_STATIC_MAX_F, E <= MOE_STATIC_MAX_E; larger shapes
 *   return MOE_ERR_BAD_ARG with the limits in moe_last_error().
 *   The first call on each device (with that device current) looks up the array's device
 *   address; make that first call before any stream capture.
 *   All calls share the array and leave their contents in it; the counters that must start
 *   at zero are cleared at the start of each call on `stream`. Calls whose work overlaps on
 *   the GPU (other streams, other host threads) race on the array. First calls made from
 *   several host threads at once are safe: the set-up runs once per device.
 *   A device-side wait that runs out of time (2 s) ends the kernels early, leaving `out` not
 *   fully written; it is recorded in a device error word inside the array, which stays set
 *   until moe_layer_forward_static_check reads it.
 */
#define MOE_STATIC_SCRATCH_BYTES (4u << 20)
#define MOE_STATIC_MAX_TOKENS 16
#define MOE_STATIC_MAX_SLOTS 128
#define MOE_STATIC_MAX_D 4096
#define MOE_STATIC_MAX_F 1024
#define MOE_STATIC_MAX_E 256
int moe_layer_forward_static(const void *x, const float *router_w, const float *router_scale,
                             const uint8_t *gate_up_q4, const uint8_t *down_q4,
                             const float *expert_scale, int T, int d, int f, int E, int k,
                             float *out, void *stream);
/* moe_layer_forward_static_check: synchronise `stream`, then read and clear the static entry's
 * device error word on the current device: MOE_ERR_DEVICE_TIMEOUT if a call since the last
 * check had a device-side wait run out (its output is then not valid), else MOE_OK.
 * Allocates nothing. */
int moe_layer_forward_static_check(void *stream);

/* moe_workspace_bytes: device bytes moe_init would allocate for the given limits. */
size_t moe_workspace_bytes(int max_tokens, int max_d, int max_f, int max_E, int max_k);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
