// moe_common.cuh -- shared definitions of the sm_100a routed-MoE kernels: workspace
// layout, device error word, bounded waits, and thin inline-PTX wrappers for mbarriers
// and bulk asynchronous copies (cp.async.bulk, no cluster multicast anywhere).
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/moe.h"

#define MOE_QK 32          // weights per Q4_0 block
#define MOE_QBYTES 18      // bytes per Q4_0 block
#define MOE_MAX_E 512
#define MOE_WAIT_NS 2000000000ull   // default bound on any device-side wait: 2 s

// Device error word: code in the low 16 bits, location in the high 16.
#define MOE_DEV_ERR_TIMEOUT 1u
#define MOE_DEV_ERR_BAD_EXPERT 2u   // an expert id given to the experts-only path is out of range

// Routing and scratch produced and consumed inside one forward. All device pointers.
// Decode layout shared by the fused decode kernel and the separate decode kernels, so that
// both give the same bits and a token's output does not depend on the batch it is decoded in:
// - router: the d axis of an expert is cut into P = moe_decode_router_parts(d) slices, slice q
//   = [q s, q s + s) with s = (d / 4) / P * 4 and the last one running to d; lane l of a slice
//   takes the float4 groups at 4 l + 128 j; lanes are summed by an xor butterfly, slices in
//   order. P is the fused kernel's warp count (its compute warps, clamped to [8, 12], + 2).
// - down: a row's blocks are split in MOE_DN_PARTS parts (block pairs first when the row has
//   an even number of blocks), each summed in block order, the parts summed in order.
constexpr int MOE_DECODE_MIN_COMPUTE = 8, MOE_DECODE_MAX_COMPUTE = 12;
constexpr int MOE_DN_PARTS = 5;
// Tokens and slots (T k, with the dense MLP's slots) per launch of the fused decode kernel.
constexpr int MOE_FUSED_MAX_T = 8, MOE_FUSED_MAX_SLOTS = 128;
__host__ __device__ inline int moe_decode_router_parts(int d) {
  const int g = (d / 32 + 7) / 8;   // 8-block granules of a gate_up row
  return (g < MOE_DECODE_MIN_COMPUTE ? MOE_DECODE_MIN_COMPUTE : (g > MOE_DECODE_MAX_COMPUTE ? MOE_DECODE_MAX_COMPUTE : g)) + 2;
}

// Rows per tile of the grouped-GEMM tile list (the routed rows of each expert are padded to
// whole tiles; tile i covers padded rows [128 i, 128 i + 128)).
constexpr int MOE_GEMM_TILE_ROWS = 128;

struct MoeWork {
  float *logits;      // [T, E]
  int32_t *ids;       // [T*k]
  float *w;           // [T*k]
  int32_t *counts;    // [E]
  int32_t *offsets;   // [E+1]
  int32_t *perm;      // [T*k]  sorted position -> slot
  int32_t *inv;       // [T*k]  slot -> sorted position
  int32_t *act;       // [E]    active experts, ascending; act[E-1..] unused
  int32_t *n_act;     // [1]
  int16_t *xq;        // [T, d] x as block-scaled int16 in the GEMV's word order
  struct ActBlk *xblk;   // [T, d/32] per block of xq: -8 * sum of the values, 2^sigma
  float *h;           // [T*k, f] fp32 hidden (GEMV path), slot order
  float *ybuf;        // [T*k, d] per-slot expert outputs (GEMV path)
  uint32_t *counters; // [n] zero-initialised arrival counters (reset by their users)
  volatile uint32_t *err;   // mapped host word: device error code
  // grouped-GEMM path
  __nv_bfloat16 *hb;  // [tiles*128, f] bf16 hidden, padded tile order
  float *yslot;       // [T*k, d] per-slot weighted down outputs (bf16 in the GEMM path)
  int32_t *tiles;     // [max tiles] (expert, m0) work list
  int32_t *toff;      // [E] index of each expert's first tile
  unsigned long long *gbar;   // launch counter of the fused decode kernel (monotonic)
  // Launch-tagged words of the fused decode kernel: high 32 bits a tag unique to the launch,
  // low 32 bits an FP32 value, stored and polled as one 64-bit word, so that a reader that
  // sees its launch's tag has the value (zeroed with the launch counter).
  unsigned long long *ltag;   // [MOE_FUSED_MAX_T, E] router logits
  unsigned long long *ytag;   // [MOE_FUSED_MAX_SLOTS, d] per-slot down outputs
  unsigned long long *htag;   // [MOE_FUSED_MAX_SLOTS, f] per-slot hidden vectors
  int32_t *n_tiles;   // [1]
  int32_t *pairs;     // [n_pairs][2]: first tile of up to two consecutive tiles of one expert, second present
  int32_t *n_pairs;   // [1]
  __nv_bfloat16 *wsplit;   // [3][128][d] the router weights as three bf16 planes (prefill router)
  unsigned long long wait_ns;   // bound on every device-side wait of this launch
  int inject;         // test-only fault (MOE_INJECT_*), 0 in normal operation
};

// Test-only faults a launch can be asked to simulate (MOE_INJECT_* of moe.h, set with
// moe_debug_inject): the failure is made by skipping a step, never by a bad address or an
// unbounded wait, so the kernel still ends on its own when its bounded waits run out.

// ---------------------------------------------------------------- small helpers

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void report_error(volatile uint32_t *err, uint32_t code, uint32_t where) {
  if (err) {
    uint32_t v = code | (where << 16);
    atomicCAS(const_cast<uint32_t *>(err), 0u, v);
    __threadfence_system();
  }
}

// ---------------------------------------------------------------- int16 activations
//
// The GEMV path multiplies Q4_0 codes by int16 activations. Each 32-wide block of an
// activation vector is scaled by a power of two 2^-sigma that puts its largest magnitude in
// [2^14, 2^15) and rounded to the nearest integer: exact for bf16 values within 2^7 of the
// block's largest, an error of at most 2^-15 of the largest otherwise. The block's results
// are multiplied back by 2^sigma. A block holding a NaN or an infinity gets sigma = NaN, so
// the non-finite value reaches the output.
struct BlockScale {
  float scale;   // 2^-sigma
  float inv;     // 2^sigma
};
__device__ __forceinline__ BlockScale block_scale_for_max(float m) {
  int eb = (int)((__float_as_uint(m) >> 23) & 0xffu);   // biased exponent of max |v|
  eb = eb < 15 ? 15 : eb;                                  // tiny / zero blocks: scale 2^126
  BlockScale r;
  r.scale = __uint_as_float((uint32_t)(268 - eb) << 23);   // 2^(141 - e): max in [2^14, 2^15)
  r.inv = __uint_as_float((uint32_t)(eb - 14) << 23);
  return r;
}
__device__ __forceinline__ int act_to_i16(float v, float scale) {
  return __float2int_rn(fminf(fmaxf(v * scale, -32768.f), 32767.f));
}
// Per block of an int16 activation vector: -8 * (sum of its 32 values) and 2^sigma.
struct ActBlk {
  int neg8sum;
  float scale;
};
// Position of element e (0..31) of a block in the GEMV's word order: code word i (bytes
// 4i..4i+3) pairs with activations 4i..4i+3 (low nibbles) then 16+4i..16+4i+3 (high).
__device__ __forceinline__ int gemv_pos(int e) { return (e < 16) ? ((e >> 2) * 8 + (e & 3)) : (((e - 16) >> 2) * 8 + 4 + (e & 3)); }

// ---------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete, at most limit_ns. Returns false
// (and records a timeout in *err) when the bound expires.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile uint32_t *err,
                                          uint32_t where, uint64_t limit_ns) {
  if (mbar_test(bar, parity)) return true;
  uint64_t t0 = globaltimer_ns();
  while (!mbar_test(bar, parity)) {
    if (globaltimer_ns() - t0 > limit_ns) {
      report_error(err, MOE_DEV_ERR_TIMEOUT, where);
      return false;
    }
  }
  return true;
}

// ---------------------------------------------------------------- bulk async copy

// 1-D bulk copy global -> shared, completion counted in bytes on `bar`. Both addresses
// 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// L2 policy for data read exactly once per call (the expert weights): its lines are the
// first evicted, so they do not push out what later calls read again (code, router weights,
// activations, workspace).
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
// bulk_g2s with an L2 cache policy.
__device__ __forceinline__ void bulk_g2s_hint(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                                              uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}

// Bulk prefetch of [src, src + bytes) into L2 (no shared memory involved, no completion to
// wait for). src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- programmatic dependent launch

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- host-side launch helpers

struct MoeLaunch {
  cudaStream_t stream;
  bool pdl;                 // launch with programmatic stream serialization
  bool accumulate = false;  // the combine adds into out (out += ...) instead of writing it
};

// Kernel groups for the optional per-kernel event timing (moe_profile_begin / _end).
enum MoeKernelId {
  MOE_K_ROUTE = 0,        // router + top-k + permutation (one or more launches)
  MOE_K_GATEUP = 1,       // decode gate_up GEMV + GeGLU
  MOE_K_DOWN = 2,         // decode down GEMV + combine
  MOE_K_GEMM_GATEUP = 3,  // prefill gate_up grouped GEMM + GeGLU
  MOE_K_GEMM_DOWN = 4,    // prefill down grouped GEMM
  MOE_K_COMBINE = 5,      // prefill ordered combine
  MOE_K_NORM = 6,         // inter-layer RMSNorm
  MOE_K_FUSED = 7,        // fused decode kernel (router .. combine in one launch)
  MOE_K_COUNT = 8
};
// Record a CUDA event on `s` before (begin) / after a launch of kernel group `id`; a no-op
// unless timing is active. Defined in moe_api.cu.
void moe_prof_mark(cudaStream_t s, int id, bool begin);
// Count n kernel launches made by this library while timing is active (moe_api.cu).
void moe_prof_count(int n);
// Let kernel `fn` use the device's whole opt-in shared memory on the current device. The
// attribute belongs to each device's context, so it is set once per device (bit `device` of
// *done_mask records it; setting the same value twice is harmless). Returns false on error.
bool moe_allow_dyn_smem(const void *fn, unsigned long long *done_mask);

// Host prototypes of the kernel launchers (defined in the .cu files).
int moe_launch_route_decode(const MoeLaunch &L, const MoeWork &W, const void *x, const float *router_w,
                            const float *router_scale, int T, int d, int E, int k, int num_sms);
// Bytes of the ybuf slot the prefill routing uses as scratch (range partials of the router
// product, then per-CTA expert counts of the permutation).
// the prefill router's d splits (partials kept in the route scratch, added in split order)
#define MOE_ROUTER_MAX_SPLIT 9
// the prefill router on the tensor cores (W_r as three exact bf16 planes in W.wsplit): E <= 128,
// d a multiple of 64; writes part[nsplit][T][E] and sets *nsplit; -2 when not supported
bool moe_router_tc_supported(int d, int E);
int moe_launch_router_tc(const MoeLaunch &L, const MoeWork &W, const void *x, const float *router_w, int T, int d,
                         int E, int num_sms, float *part, int *nsplit);
size_t moe_route_scratch_bytes(int max_tokens, int max_E, int max_k);
int moe_launch_route_prefill(const MoeLaunch &L, const MoeWork &W, const void *x, const float *router_w,
                             const float *router_scale, int T, int d, int E, int k, int num_sms,
                             bool want_xprep, int tile_m);
int moe_launch_gemv_experts(const MoeLaunch &L, const MoeWork &W, const uint8_t *gate_up_q4,
                            const uint8_t *down_q4, const float *expert_scale, int T, int d, int f,
                            int E, int k, float *out, int num_sms);
int moe_launch_gemm_experts(const MoeLaunch &L, const MoeWork &W, const void *x, const uint8_t *gate_up_q4,
                            const uint8_t *down_q4, const float *expert_scale, int T, int d, int f,
                            int E, int k, float *out, int num_sms, int max_tiles);
// dense: the block's dense MLP (same width f) rides along as expert E, one more slot per token.
bool moe_fused_decode_supported(int T, int d, int f, int E, int k, bool dense = false);
// The fused decode kernel: x (bf16 [T, d]) as the layer input, or, with y_prev not null, the
// previous layer's FP32 output normalised in the kernel (x_out, when not null, receives that
// bf16 x; y_prev must not overlap out).
int moe_launch_fused_decode(const MoeLaunch &L, const MoeWork &W, const void *x, const float *y_prev, float eps,
                            void *x_out, const float *router_w, const float *router_scale,
                            const uint8_t *gate_up_q4, const uint8_t *down_q4, const float *expert_scale, int T,
                            int d, int f, int E, int k, float *out, int num_sms, const uint8_t *dense_gu = nullptr,
                            const uint8_t *dense_dn = nullptr, const float *next_router_w = nullptr);
int moe_launch_rmsnorm(cudaStream_t s, const float *y, void *x_out, int T, int d, float eps);
// Routing given by the caller (one expert and weight per row, k = 1): ids and weights into the
// workspace, the stable permutation (with the tile lists when tile_m > 0) and, with
// want_xprep, the GEMV path's activations. Out-of-range ids record MOE_DEV_ERR_BAD_EXPERT and
// become expert 0 with weight 0.
int moe_launch_route_given(const MoeLaunch &L, const MoeWork &W, const void *x, const int32_t *row_expert,
                           const float *row_weight, int R, int d, int E, int num_sms, bool want_xprep, int tile_m);
// dst row i = src row index[i] (rows of row_bytes, a multiple of 16; 16-byte aligned bases).
int moe_launch_gather_rows(cudaStream_t s, const void *src, const int32_t *index, int n, size_t row_bytes,
                           void *dst);
// out[t, :] = sum_j y[t * k + j, :] in j order (FP32 rows of d).
int moe_launch_combine_slots(cudaStream_t s, const float *y, int T, int d, int k, float *out);
int moe_launch_hidden_to_slots(cudaStream_t s, const MoeWork &W, float *h, int T, int f, int k,
                               bool gemm_path);
