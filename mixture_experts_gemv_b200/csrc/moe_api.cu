// moe_api.cu -- the C ABI (include/moe.h): context, workspace, argument checks, path
// selection and the launches on the caller's stream. Nothing here computes the layer;
// every step runs in the kernels of moe_route.cu, moe_gemv.cu and moe_gemm_sm100.cu.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <vector>

#include "../../include/moe.h"
#include "moe_common.cuh"

namespace {

struct Ctx {
  bool init = false;
  int device = -1;
  int num_sms = 0;
  int max_tokens = 0, max_d = 0, max_f = 0, max_E = 0, max_k = 0;
  void *ws = nullptr;
  size_t ws_bytes = 0;
  uint32_t *err_host = nullptr;   // mapped pinned word
  MoeWork W{};
  __nv_bfloat16 *xbuf[2] = {nullptr, nullptr};   // stack: inter-layer activations
  float *ylayer[2] = {nullptr, nullptr};         // stack: intermediate layer outputs (alternating)
  int path = MOE_PATH_AUTO;
  int gemv_max_tokens = 16;   // AUTO: GEMV for T <= 16, grouped GEMM above
  int last_T = 0, last_k = 0, last_E = 0, last_f = 0;
  bool last_gemm = false;
  size_t counters_bytes = 0;
  bool reset_pending = false;      // a device wait expired: zero the launch counter, the arrival
                                   // counters and the tagged words before the next launch
  float *dense_router = nullptr;   // [max_d] zeros: the router of the dense MLP's one-expert pass
  float *one = nullptr;            // 1.0f: its router scale and expert scale
};

Ctx g;
char g_err[512] = "";

// Per-kernel event timing: pairs of events recorded around each launch of a kernel group.
struct Prof {
  bool active = false;
  std::vector<cudaEvent_t> pool;
  size_t used = 0;
  struct Rec { int id; cudaEvent_t a, b; };
  std::vector<Rec> recs;
  int open_id[MOE_K_COUNT];
  cudaEvent_t open_ev[MOE_K_COUNT];
  bool overflow = false;
  long long kernels = 0;   // kernel launches since moe_profile_begin
};
Prof g_prof;

cudaEvent_t prof_event() {
  if (g_prof.used == g_prof.pool.size()) {
    if (g_prof.pool.size() >= 65536) { g_prof.overflow = true; return nullptr; }
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) { g_prof.overflow = true; return nullptr; }
    g_prof.pool.push_back(e);
  }
  return g_prof.pool[g_prof.used++];
}

int fail(int code, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
int fail(int code, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return code;
}

int cuda_fail(cudaError_t e, const char *what) {
  return fail(MOE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

constexpr int kTileM = MOE_GEMM_TILE_ROWS;   // rows per grouped-GEMM tile

struct Layout {
  size_t off[27];
  size_t total;
};

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// The fused decode kernel's launch-tagged words: logits [MOE_FUSED_MAX_T, E], then per-slot
// outputs [MOE_FUSED_MAX_SLOTS, d], then per-slot hidden vectors [MOE_FUSED_MAX_SLOTS, f].
size_t tag_logit_words(int max_E) { return (size_t)MOE_FUSED_MAX_T * max_E; }
size_t tag_bytes(int max_d, int max_f, int max_E) {
  return (align_up(tag_logit_words(max_E), 32) + (size_t)MOE_FUSED_MAX_SLOTS * (max_d + max_f)) * 8;
}

Layout make_layout(int maxT, int max_d, int max_f, int max_E, int max_k) {
  // per-slot buffers hold k + 1 slots per token: the block's dense MLP takes one more slot per
  // token when it rides in the fused decode launch
  const size_t S = (size_t)maxT * (max_k + 1);
  const size_t prow = (S / kTileM + max_E + 1) * kTileM;   // padded tile rows
  const size_t ybuf_bytes = S * max_d * 4 > moe_route_scratch_bytes(maxT, max_E, max_k)
                                ? S * max_d * 4
                                : moe_route_scratch_bytes(maxT, max_E, max_k);
  const size_t sizes[] = {
      (size_t)maxT * max_E * 4,          // 0 logits
      S * 4,                             // 1 ids
      S * 4,                             // 2 w
      (size_t)max_E * 4,                 // 3 counts
      (size_t)(max_E + 1) * 4,           // 4 offsets
      S * 4,                             // 5 perm
      S * 4,                             // 6 inv
      (size_t)max_E * 4,                 // 7 act
      16,                                // 8 n_act, n_tiles, n_pairs
      (size_t)maxT * max_d * 2,          // 9 xq
      (size_t)maxT * (max_d / 32) * 8,   // 10 xblk
      S * max_f * 4,                     // 11 h
      16,                                // 12 (unused)
      ybuf_bytes,                        // 13 ybuf / yslot (and routing scratch)
      (size_t)(2 + max_d / 8 + 1024) * 4,   // 14 counters
      prow * max_f * 2,                  // 15 hb (bf16, padded tiles)
      (S / kTileM + max_E + 1) * 8,      // 16 tiles
      (size_t)maxT * max_d * 2,          // 17 xbuf0
      (size_t)maxT * max_d * 2,          // 18 xbuf1
      (size_t)maxT * max_d * 4,          // 19 ylayer
      (S / kTileM + max_E + 1) * 8,      // 20 tile pairs
      (size_t)max_E * 4,                 // 21 toff
      64,                                // 22 launch counter of the fused decode kernel
      (size_t)max_d * 4 + 16,            // 23 dense MLP pass: zero router row, then 1.0f
      (size_t)3 * 128 * max_d * 2,       // 24 the router weights as three bf16 planes (prefill)
      tag_bytes(max_d, max_f, max_E),    // 25 launch-tagged logits, per-slot outputs and hidden vectors
      (size_t)maxT * max_d * 4,          // 26 ylayer2 (stack: layers alternate between 19 and 26)
  };
  Layout L{};
  size_t o = 0;
  for (size_t i = 0; i < sizeof(sizes) / sizeof(sizes[0]); ++i) {
    L.off[i] = o;
    o = align_up(o + sizes[i], 256);
  }
  L.total = o;
  return L;
}

void release() {
  if (g.ws) cudaFree(g.ws);
  if (g.err_host) cudaFreeHost(g.err_host);
  g = Ctx{};
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_device_error() {
  if (g.err_host && *reinterpret_cast<volatile uint32_t *>(g.err_host) != 0) {
    const uint32_t v = *reinterpret_cast<volatile uint32_t *>(g.err_host);
    *reinterpret_cast<volatile uint32_t *>(g.err_host) = 0;
    // the kernels that gave up left their arrival counters mid-count
    g.reset_pending = true;
    if ((v & 0xffffu) == MOE_DEV_ERR_BAD_EXPERT)
      return fail(MOE_ERR_BAD_ARG, "an expert id given to moe_experts_forward was outside [0, E) (its row was "
                                   "computed with weight 0)");
    return fail(MOE_ERR_DEVICE_TIMEOUT, "device wait timed out (code %u at site %u)", v & 0xffffu, v >> 16);
  }
  return MOE_OK;
}

// After an expired wait: the launch counter and the arrival counters start again from
// zero (enqueued on the stream of the next launch).
int reset_counters_if_needed(cudaStream_t s) {
  if (!g.reset_pending) return MOE_OK;
  cudaError_t e = cudaMemsetAsync(g.W.gbar, 0, 64, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(g.W.counters, 0, g.counters_bytes, s);
  // the launch tags restart with the counter: no word may carry a tag a coming launch uses
  if (e == cudaSuccess) e = cudaMemsetAsync(g.W.ltag, 0, tag_bytes(g.max_d, g.max_f, g.max_E), s);
  if (e != cudaSuccess) return cuda_fail(e, "resetting the arrival counters");
  g.reset_pending = false;
  return MOE_OK;
}

int check_shapes(int T, int d, int f, int E, int k) {
  if (T < 0) return fail(MOE_ERR_BAD_ARG, "T = %d < 0", T);
  if (d <= 0 || d % 32) return fail(MOE_ERR_BAD_ARG, "d = %d must be a positive multiple of 32", d);
  if (f <= 0 || f % 32) return fail(MOE_ERR_BAD_ARG, "f = %d must be a positive multiple of 32", f);
  if (E < 1 || E > MOE_MAX_E) return fail(MOE_ERR_BAD_ARG, "E = %d outside [1, %d]", E, MOE_MAX_E);
  if (k < 1 || k > E) return fail(MOE_ERR_BAD_ARG, "k = %d outside [1, E = %d]", k, E);
  return MOE_OK;
}

int check_limits(int T, int d, int f, int E, int k) {
  if (!g.init) return fail(MOE_ERR_NOT_INIT, "moe_init has not succeeded");
  (void)T;   // any T: calls above max_tokens run in chunks of max_tokens tokens
  if (d > g.max_d || f > g.max_f || E > g.max_E || k > g.max_k)
    return fail(MOE_ERR_BAD_ARG, "shape (d=%d, f=%d, E=%d, k=%d) exceeds the moe_init limits (%d, %d, %d, %d)",
                d, f, E, k, g.max_d, g.max_f, g.max_E, g.max_k);
  return MOE_OK;
}

// The path a call of T_call tokens takes (every chunk of a chunked call takes the same one).
bool gemm_path_for(int T_call) {
  return (g.path == MOE_PATH_GEMM) || (g.path == MOE_PATH_AUTO && T_call > g.gemv_max_tokens);
}

// One pass of T <= max_tokens tokens; `gemm` chooses the path.
int forward_impl(const void *x, const float *router_w, const float *router_scale, const uint8_t *gate_up_q4,
                 const uint8_t *down_q4, const float *expert_scale, int T, int d, int f, int E, int k, float *out,
                 cudaStream_t stream, bool gemm, bool accumulate = false) {
  MoeLaunch L{stream, false, accumulate};
  int rc = reset_counters_if_needed(stream);
  if (rc) return rc;
  // MOE_PATH_GEMV and AUTO below the threshold take the fused decode kernel when the shape
  // fits it (T <= 8), else the separate routing / gate_up / down kernels (MOE_PATH_GEMV_SPLIT).
  if (gemm) {
    rc = moe_launch_route_prefill(L, g.W, x, router_w, router_scale, T, d, E, k, g.num_sms, false, kTileM);
    if (rc) return cuda_fail(cudaGetLastError(), "routing launch");
    const int max_tiles = (int)((size_t)g.max_tokens * g.max_k / kTileM + g.max_E + 1);
    rc = moe_launch_gemm_experts(L, g.W, x, gate_up_q4, down_q4, expert_scale, T, d, f, E, k, out, g.num_sms,
                                 max_tiles);
    if (rc == -2) return fail(MOE_ERR_BAD_ARG, "shape not supported by the grouped-GEMM path");
    if (rc) return cuda_fail(cudaGetLastError(), "grouped-GEMM launch");
  } else if (g.path != MOE_PATH_GEMV_SPLIT && moe_fused_decode_supported(T, d, f, E, k)) {
    rc = moe_launch_fused_decode(L, g.W, x, nullptr, 0.f, nullptr, router_w, router_scale, gate_up_q4, down_q4,
                                 expert_scale, T, d, f, E, k, out, g.num_sms);
    if (rc) return cuda_fail(cudaGetLastError(), "fused decode launch");
  } else {
    if (T <= 16)
      rc = moe_launch_route_decode(L, g.W, x, router_w, router_scale, T, d, E, k, g.num_sms);
    else
      rc = moe_launch_route_prefill(L, g.W, x, router_w, router_scale, T, d, E, k, g.num_sms, true, 0);
    if (rc) return cuda_fail(cudaGetLastError(), "routing launch");
    rc = moe_launch_gemv_experts(L, g.W, gate_up_q4, down_q4, expert_scale, T, d, f, E, k, out, g.num_sms);
    if (rc == -2) return fail(MOE_ERR_BAD_ARG, "shape not supported by the GEMV path (d, f too large)");
    if (rc) return cuda_fail(cudaGetLastError(), "GEMV launch");
  }
  g.W.inject = MOE_INJECT_NONE;   // a test fault applies to one forward only
  g.last_T = T;
  g.last_k = k;
  g.last_E = E;
  g.last_f = f;
  g.last_gemm = gemm;
  return MOE_OK;
}

}  // namespace

// Lets other translation units of the library set the moe_last_error() text.
int moe_report_error(int code, const char *msg) {
  snprintf(g_err, sizeof g_err, "%s", msg);
  return code;
}

void moe_prof_mark(cudaStream_t s, int id, bool begin) {
  if (!g_prof.active || id < 0 || id >= MOE_K_COUNT) return;
  cudaEvent_t e = prof_event();
  if (!e) return;
  // inside a stream capture the record must become an event-record node of the graph
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaStreamIsCapturing(s, &cs);
  if (cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(e, s, cudaEventRecordExternal);
  else
    cudaEventRecord(e, s);
  if (begin) {
    g_prof.open_ev[id] = e;
  } else if (g_prof.open_ev[id]) {
    g_prof.recs.push_back({id, g_prof.open_ev[id], e});
    g_prof.open_ev[id] = nullptr;
  }
}

void moe_prof_count(int n) {
  if (g_prof.active) g_prof.kernels += n;
}

bool moe_allow_dyn_smem(const void *fn, unsigned long long *done_mask) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  const unsigned long long bit = 1ull << dev;
  if (__atomic_load_n(done_mask, __ATOMIC_ACQUIRE) & bit) return true;
  int optin = 0;
  if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return false;
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, fn) != cudaSuccess) return false;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, optin - (int)fa.sharedSizeBytes) !=
      cudaSuccess)
    return false;
  __atomic_fetch_or(done_mask, bit, __ATOMIC_RELEASE);
  return true;
}

extern "C" {

long long moe_profile_kernel_launches(void) { return g_prof.kernels; }

int moe_profile_begin(void) {
  if (!g.init) return fail(MOE_ERR_NOT_INIT, "moe_init has not succeeded");
  g_prof.active = true;
  g_prof.used = 0;
  g_prof.recs.clear();
  g_prof.overflow = false;
  g_prof.kernels = 0;
  for (int i = 0; i < MOE_K_COUNT; ++i) g_prof.open_ev[i] = nullptr;
  return MOE_OK;
}

int moe_profile_end(float *ms_total, int *launches) {
  if (!g.init) return fail(MOE_ERR_NOT_INIT, "moe_init has not succeeded");
  g_prof.active = false;
  for (int i = 0; i < MOE_K_COUNT; ++i) {
    if (ms_total) ms_total[i] = 0.f;
    if (launches) launches[i] = 0;
  }
  for (auto &r : g_prof.recs) {
    cudaError_t e = cudaEventSynchronize(r.b);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventSynchronize");
    float ms = 0.f;
    e = cudaEventElapsedTime(&ms, r.a, r.b);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventElapsedTime");
    if (ms_total) ms_total[r.id] += ms;
    if (launches) launches[r.id] += 1;
  }
  g_prof.recs.clear();
  if (g_prof.overflow) return fail(MOE_ERR_BAD_ARG, "too many launches timed (limit 32768)");
  return MOE_OK;
}


size_t moe_workspace_bytes(int max_tokens, int max_d, int max_f, int max_E, int max_k) {
  if (max_tokens < 1 || max_d < 32 || max_f < 32 || max_E < 1 || max_k < 1) return 0;
  return make_layout(max_tokens, max_d, max_f, max_E, max_k).total;
}

int moe_init(int device, int max_tokens, int max_d, int max_f, int max_E, int max_k) {
  if (max_tokens < 1) return fail(MOE_ERR_BAD_ARG, "max_tokens = %d < 1", max_tokens);
  if (max_d < 32 || max_d % 32 || max_f < 32 || max_f % 32)
    return fail(MOE_ERR_BAD_ARG, "max_d = %d and max_f = %d must be positive multiples of 32", max_d, max_f);
  if (max_E < 1 || max_E > MOE_MAX_E) return fail(MOE_ERR_BAD_ARG, "max_E = %d outside [1, %d]", max_E, MOE_MAX_E);
  if (max_k < 1 || max_k > max_E) return fail(MOE_ERR_BAD_ARG, "max_k = %d outside [1, max_E]", max_k);
  if (g.init) {
    cudaSetDevice(g.device);
    cudaDeviceSynchronize();
    release();
  }
  cudaError_t e = cudaSetDevice(device);
  if (e != cudaSuccess) return cuda_fail(e, "cudaSetDevice");
  cudaDeviceProp prop;
  e = cudaGetDeviceProperties(&prop, device);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceProperties");
  if (prop.major != 10 || prop.minor != 0)
    return fail(MOE_ERR_UNSUPPORTED_DEVICE, "device %d is sm_%d%d; this library is built for sm_100a", device,
                prop.major, prop.minor);
  const Layout Lt = make_layout(max_tokens, max_d, max_f, max_E, max_k);
  void *ws = nullptr;
  e = cudaMalloc(&ws, Lt.total);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(workspace)");
  e = cudaMemset(ws, 0, Lt.total);
  if (e != cudaSuccess) { cudaFree(ws); return cuda_fail(e, "cudaMemset(workspace)"); }
  {
    const float one = 1.0f;
    e = cudaMemcpy(static_cast<char *>(ws) + Lt.off[23] + (size_t)max_d * 4, &one, sizeof one, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) { cudaFree(ws); return cuda_fail(e, "workspace constants"); }
  }
  uint32_t *eh = nullptr;
  e = cudaHostAlloc(reinterpret_cast<void **>(&eh), 64, cudaHostAllocMapped);
  if (e != cudaSuccess) { cudaFree(ws); return cuda_fail(e, "cudaHostAlloc(error word)"); }
  *eh = 0;
  uint32_t *ed = nullptr;
  e = cudaHostGetDevicePointer(reinterpret_cast<void **>(&ed), eh, 0);
  if (e != cudaSuccess) { cudaFree(ws); cudaFreeHost(eh); return cuda_fail(e, "cudaHostGetDevicePointer"); }

  char *b = static_cast<char *>(ws);
  MoeWork W{};
  W.logits = reinterpret_cast<float *>(b + Lt.off[0]);
  W.ids = reinterpret_cast<int32_t *>(b + Lt.off[1]);
  W.w = reinterpret_cast<float *>(b + Lt.off[2]);
  W.counts = reinterpret_cast<int32_t *>(b + Lt.off[3]);
  W.offsets = reinterpret_cast<int32_t *>(b + Lt.off[4]);
  W.perm = reinterpret_cast<int32_t *>(b + Lt.off[5]);
  W.inv = reinterpret_cast<int32_t *>(b + Lt.off[6]);
  W.act = reinterpret_cast<int32_t *>(b + Lt.off[7]);
  W.n_act = reinterpret_cast<int32_t *>(b + Lt.off[8]);
  W.n_tiles = reinterpret_cast<int32_t *>(b + Lt.off[8] + 4);
  W.n_pairs = reinterpret_cast<int32_t *>(b + Lt.off[8] + 8);
  W.pairs = reinterpret_cast<int32_t *>(b + Lt.off[20]);
  W.xq = reinterpret_cast<int16_t *>(b + Lt.off[9]);
  W.xblk = reinterpret_cast<ActBlk *>(b + Lt.off[10]);
  W.h = reinterpret_cast<float *>(b + Lt.off[11]);
  W.ybuf = reinterpret_cast<float *>(b + Lt.off[13]);
  W.yslot = W.ybuf;
  W.counters = reinterpret_cast<uint32_t *>(b + Lt.off[14]);
  W.hb = reinterpret_cast<__nv_bfloat16 *>(b + Lt.off[15]);
  W.tiles = reinterpret_cast<int32_t *>(b + Lt.off[16]);
  W.toff = reinterpret_cast<int32_t *>(b + Lt.off[21]);
  W.gbar = reinterpret_cast<unsigned long long *>(b + Lt.off[22]);
  W.wsplit = reinterpret_cast<__nv_bfloat16 *>(b + Lt.off[24]);
  W.ltag = reinterpret_cast<unsigned long long *>(b + Lt.off[25]);
  W.ytag = W.ltag + align_up(tag_logit_words(max_E), 32);
  W.htag = W.ytag + (size_t)MOE_FUSED_MAX_SLOTS * max_d;
  W.err = ed;
  W.wait_ns = MOE_WAIT_NS;
  W.inject = MOE_INJECT_NONE;

  g.init = true;
  g.device = device;
  g.num_sms = prop.multiProcessorCount;
  g.max_tokens = max_tokens;
  g.max_d = max_d;
  g.max_f = max_f;
  g.max_E = max_E;
  g.max_k = max_k;
  g.ws = ws;
  g.ws_bytes = Lt.total;
  g.counters_bytes = (size_t)(2 + max_d / 8 + 1024) * 4;
  g.dense_router = reinterpret_cast<float *>(b + Lt.off[23]);   // zeroed with the workspace
  g.one = g.dense_router + max_d;
  g.err_host = eh;
  g.W = W;
  g.xbuf[0] = reinterpret_cast<__nv_bfloat16 *>(b + Lt.off[17]);
  g.xbuf[1] = reinterpret_cast<__nv_bfloat16 *>(b + Lt.off[18]);
  g.ylayer[0] = reinterpret_cast<float *>(b + Lt.off[19]);
  g.ylayer[1] = reinterpret_cast<float *>(b + Lt.off[26]);
  return MOE_OK;
}

int moe_layer_forward(const void *x, const float *router_w, const float *router_scale, const uint8_t *gate_up_q4,
                      const uint8_t *down_q4, const float *expert_scale, int T, int d, int f, int E, int k, float *out,
                      void *stream) {
  int rc = check_shapes(T, d, f, E, k);
  if (rc) return rc;
  if (!x || !router_w || !router_scale || !gate_up_q4 || !down_q4 || !expert_scale || !out)
    return fail(MOE_ERR_BAD_ARG, "null pointer argument");
  if (!aligned16(gate_up_q4) || !aligned16(down_q4) || !aligned16(router_w) || !aligned16(x))
    return fail(MOE_ERR_BAD_ALIGN, "x, router_w, gate_up_q4 and down_q4 must be 16-byte aligned");
  rc = check_limits(T, d, f, E, k);
  if (rc) return rc;
  rc = check_device_error();
  if (rc) return rc;
  if (T == 0) return MOE_OK;
  // Calls above the workspace's token capacity run as consecutive chunks of max_tokens tokens
  // on the path the whole call selects; a token's output depends only on its own x, so the
  // result is the same as one pass.
  const bool gemm = gemm_path_for(T);
  for (int c0 = 0; c0 < T; c0 += g.max_tokens) {
    const int Tc = T - c0 < g.max_tokens ? T - c0 : g.max_tokens;
    rc = forward_impl(static_cast<const char *>(x) + (size_t)c0 * d * 2, router_w, router_scale, gate_up_q4, down_q4,
                      expert_scale, Tc, d, f, E, k, out + (size_t)c0 * d, static_cast<cudaStream_t>(stream), gemm);
    if (rc) return rc;
  }
  return MOE_OK;
}

int moe_block_forward(const void *x, const float *router_w, const float *router_scale, const uint8_t *gate_up_q4,
                      const uint8_t *down_q4, const float *expert_scale, const uint8_t *gate_up_dense_q4,
                      const uint8_t *down_dense_q4, int T, int d, int f, int f_dense, int E, int k, float *out,
                      void *stream) {
  int rc = check_shapes(T, d, f, E, k);
  if (rc) return rc;
  if (f_dense <= 0 || f_dense % 32)
    return fail(MOE_ERR_BAD_ARG, "f_dense = %d must be a positive multiple of 32", f_dense);
  if (!x || !router_w || !router_scale || !gate_up_q4 || !down_q4 || !expert_scale || !gate_up_dense_q4 ||
      !down_dense_q4 || !out)
    return fail(MOE_ERR_BAD_ARG, "null pointer argument");
  if (!aligned16(gate_up_q4) || !aligned16(down_q4) || !aligned16(router_w) || !aligned16(x) ||
      !aligned16(gate_up_dense_q4) || !aligned16(down_dense_q4))
    return fail(MOE_ERR_BAD_ALIGN, "x, router_w and the Q4_0 matrices must be 16-byte aligned");
  rc = check_limits(T, d, f, E, k);
  if (rc) return rc;
  if (f_dense > g.max_f) return fail(MOE_ERR_BAD_ARG, "f_dense = %d exceeds max_f = %d", f_dense, g.max_f);
  rc = check_device_error();
  if (rc) return rc;
  if (T == 0) return MOE_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool gemm = gemm_path_for(T);
  for (int c0 = 0; c0 < T; c0 += g.max_tokens) {
    const int Tc = T - c0 < g.max_tokens ? T - c0 : g.max_tokens;
    const void *xc = static_cast<const char *>(x) + (size_t)c0 * d * 2;
    float *oc = out + (size_t)c0 * d;
    // Decode with a dense MLP of the experts' width: one fused launch takes it as expert E,
    // one more slot per token with weight 1, its output added in the combine
    if (!gemm && g.path != MOE_PATH_GEMV_SPLIT && f_dense == f && moe_fused_decode_supported(Tc, d, f, E, k, true)) {
      rc = reset_counters_if_needed(s);
      if (rc) return rc;
      MoeLaunch L{s, false};
      rc = moe_launch_fused_decode(L, g.W, xc, nullptr, 0.f, nullptr, router_w, router_scale, gate_up_q4, down_q4,
                                   expert_scale, Tc, d, f, E, k, oc, g.num_sms, gate_up_dense_q4, down_dense_q4);
      if (rc) return cuda_fail(cudaGetLastError(), "fused decode launch");
      g.last_T = Tc;
      g.last_k = k;
      g.last_E = E;
      g.last_f = f;
      g.last_gemm = false;
      continue;
    }
    rc = forward_impl(xc, router_w, router_scale, gate_up_q4, down_q4, expert_scale, Tc, d, f, E, k, oc, s, gemm);
    if (rc) return rc;
    // the dense MLP: one expert every token selects with weight 1 (a zero router row, router
    // and expert scale 1.0), its combine adding into out
    rc = forward_impl(xc, g.dense_router, g.one, gate_up_dense_q4, down_dense_q4, g.one, Tc, d, f_dense, 1, 1, oc, s,
                      gemm, true);
    if (rc) return rc;
  }
  return MOE_OK;
}

int moe_route(const void *x, const float *router_w, const float *router_scale, int T, int d, int E, int k,
              int32_t *ids, float *w, void *stream) {
  int rc = check_shapes(T, d, 32, E, k);
  if (rc) return rc;
  if (!x || !router_w || !router_scale || !ids || !w) return fail(MOE_ERR_BAD_ARG, "null pointer argument");
  if (!aligned16(router_w) || !aligned16(x)) return fail(MOE_ERR_BAD_ALIGN, "x and router_w must be 16-byte aligned");
  rc = check_limits(T, d, 32, E, k);
  if (rc) return rc;
  rc = check_device_error();
  if (rc) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  rc = reset_counters_if_needed(s);
  if (rc) return rc;
  MoeLaunch L{s, false};
  for (int c0 = 0; c0 < T; c0 += g.max_tokens) {
    const int Tc = T - c0 < g.max_tokens ? T - c0 : g.max_tokens;
    const void *xc = static_cast<const char *>(x) + (size_t)c0 * d * 2;
    // the selection the layer itself makes: the decode routing (logits cut as the fused
    // kernel cuts them) up to 16 tokens, the tiled router product above
    rc = Tc <= 16 ? moe_launch_route_decode(L, g.W, xc, router_w, router_scale, Tc, d, E, k, g.num_sms)
                  : moe_launch_route_prefill(L, g.W, xc, router_w, router_scale, Tc, d, E, k, g.num_sms, false, 0);
    if (rc == -2) return fail(MOE_ERR_BAD_ARG, "shape not supported by the routing kernels");
    if (rc) return cuda_fail(cudaGetLastError(), "routing launch");
    cudaError_t e = cudaMemcpyAsync(ids + (size_t)c0 * k, g.W.ids, (size_t)Tc * k * 4, cudaMemcpyDeviceToDevice, s);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(w + (size_t)c0 * k, g.W.w, (size_t)Tc * k * 4, cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "routing copy");
  }
  return MOE_OK;
}

int moe_experts_forward(const void *x_rows, const int32_t *row_expert, const float *row_weight,
                        const uint8_t *gate_up_q4, const uint8_t *down_q4, const float *expert_scale, int R, int d,
                        int f, int E, float *out_rows, void *stream) {
  int rc = check_shapes(R, d, f, E, 1);
  if (rc) return rc;
  if (!x_rows || !row_expert || !row_weight || !gate_up_q4 || !down_q4 || !expert_scale || !out_rows)
    return fail(MOE_ERR_BAD_ARG, "null pointer argument");
  if (!aligned16(gate_up_q4) || !aligned16(down_q4) || !aligned16(x_rows))
    return fail(MOE_ERR_BAD_ALIGN, "x_rows, gate_up_q4 and down_q4 must be 16-byte aligned");
  rc = check_limits(R, d, f, E, 1);
  if (rc) return rc;
  rc = check_device_error();
  if (rc) return rc;
  if (R == 0) return MOE_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  rc = reset_counters_if_needed(s);
  if (rc) return rc;
  MoeLaunch L{s, false};
  const bool gemm = gemm_path_for(R);
  for (int c0 = 0; c0 < R; c0 += g.max_tokens) {
    const int Rc = R - c0 < g.max_tokens ? R - c0 : g.max_tokens;
    const void *xc = static_cast<const char *>(x_rows) + (size_t)c0 * d * 2;
    float *oc = out_rows + (size_t)c0 * d;
    rc = moe_launch_route_given(L, g.W, xc, row_expert + c0, row_weight + c0, Rc, d, E, g.num_sms, !gemm,
                                gemm ? kTileM : 0);
    if (rc == -2) return fail(MOE_ERR_BAD_ARG, "E = %d not supported by the permutation kernels", E);
    if (rc) return cuda_fail(cudaGetLastError(), "routing launch");
    if (gemm) {
      const int max_tiles = (int)((size_t)g.max_tokens * g.max_k / kTileM + g.max_E + 1);
      rc = moe_launch_gemm_experts(L, g.W, xc, gate_up_q4, down_q4, expert_scale, Rc, d, f, E, 1, oc, g.num_sms,
                                   max_tiles);
      if (rc == -2) return fail(MOE_ERR_BAD_ARG, "shape not supported by the grouped-GEMM path");
      if (rc) return cuda_fail(cudaGetLastError(), "grouped-GEMM launch");
    } else {
      rc = moe_launch_gemv_experts(L, g.W, gate_up_q4, down_q4, expert_scale, Rc, d, f, E, 1, oc, g.num_sms);
      if (rc == -2) return fail(MOE_ERR_BAD_ARG, "shape not supported by the GEMV path (d, f too large)");
      if (rc) return cuda_fail(cudaGetLastError(), "GEMV launch");
    }
  }
  return MOE_OK;
}

int moe_gather_rows(const void *src, const int32_t *index, int n, size_t row_bytes, void *dst, void *stream) {
  if (n < 0 || row_bytes == 0 || row_bytes % 16) return fail(MOE_ERR_BAD_ARG, "n >= 0 and row_bytes %% 16 == 0 needed");
  if (!src || !index || !dst) return fail(MOE_ERR_BAD_ARG, "null pointer argument");
  if (!aligned16(src) || !aligned16(dst)) return fail(MOE_ERR_BAD_ALIGN, "src and dst must be 16-byte aligned");
  if (n == 0) return MOE_OK;
  if (moe_launch_gather_rows(static_cast<cudaStream_t>(stream), src, index, n, row_bytes, dst))
    return cuda_fail(cudaGetLastError(), "gather launch");
  return MOE_OK;
}

int moe_combine_slots(const float *y_slots, int T, int d, int k, float *out, void *stream) {
  if (T < 0 || d <= 0 || d % 4 || k < 1) return fail(MOE_ERR_BAD_ARG, "T >= 0, d %% 4 == 0, k >= 1 needed");
  if (!y_slots || !out) return fail(MOE_ERR_BAD_ARG, "null pointer argument");
  if (!aligned16(y_slots) || !aligned16(out)) return fail(MOE_ERR_BAD_ALIGN, "y_slots and out must be 16-byte aligned");
  if (T == 0) return MOE_OK;
  if (moe_launch_combine_slots(static_cast<cudaStream_t>(stream), y_slots, T, d, k, out))
    return cuda_fail(cudaGetLastError(), "combine launch");
  return MOE_OK;
}

int moe_rmsnorm_bf16(const float *y, void *x_out, int T, int d, float eps, void *stream) {
  if (T < 0 || d < 1) return fail(MOE_ERR_BAD_ARG, "bad shape T = %d, d = %d", T, d);
  if (!y || !x_out) return fail(MOE_ERR_BAD_ARG, "null pointer argument");
  if (!g.init) return fail(MOE_ERR_NOT_INIT, "moe_init has not succeeded");
  if (T == 0) return MOE_OK;
  if (moe_launch_rmsnorm(static_cast<cudaStream_t>(stream), y, x_out, T, d, eps))
    return cuda_fail(cudaGetLastError(), "rmsnorm launch");
  return MOE_OK;
}

int moe_stack_forward(const void *x_in, int L, const float *const *router_w, const float *const *router_scale,
                      const uint8_t *const *gate_up_q4, const uint8_t *const *down_q4,
                      const float *const *expert_scale, int T, int d, int f, int E, int k, float eps, float *out,
                      void *x_trace, void *stream) {
  int rc = check_shapes(T, d, f, E, k);
  if (rc) return rc;
  if (L < 1) return fail(MOE_ERR_BAD_ARG, "L = %d < 1", L);
  if (!x_in || !router_w || !router_scale || !gate_up_q4 || !down_q4 || !expert_scale || !out)
    return fail(MOE_ERR_BAD_ARG, "null pointer argument");
  for (int i = 0; i < L; ++i) {
    if (!router_w[i] || !router_scale[i] || !gate_up_q4[i] || !down_q4[i] || !expert_scale[i])
      return fail(MOE_ERR_BAD_ARG, "null weight pointer for layer %d", i);
    if (!aligned16(gate_up_q4[i]) || !aligned16(down_q4[i]) || !aligned16(router_w[i]))
      return fail(MOE_ERR_BAD_ALIGN, "layer %d weights must be 16-byte aligned", i);
  }
  if (!aligned16(x_in)) return fail(MOE_ERR_BAD_ALIGN, "x_in must be 16-byte aligned");
  rc = check_limits(T, d, f, E, k);
  if (rc) return rc;
  rc = check_device_error();
  if (rc) return rc;
  if (T == 0) return MOE_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  rc = reset_counters_if_needed(s);
  if (rc) return rc;
  // Tokens are independent through every layer, so a call above max_tokens runs the whole
  // stack on one chunk of tokens after another.
  const bool gemm = gemm_path_for(T);
  // Layers that take the fused decode kernel normalise the previous layer's output inside
  // it (no separate norm launch); the others get moe_rmsnorm_bf16's x. Both give the same x.
  for (int c0 = 0; c0 < T; c0 += g.max_tokens) {
    const int Tc = T - c0 < g.max_tokens ? T - c0 : g.max_tokens;
    const bool fused = !gemm && g.path != MOE_PATH_GEMV_SPLIT && moe_fused_decode_supported(Tc, d, f, E, k);
    const void *xc = static_cast<const char *>(x_in) + (size_t)c0 * d * 2;
    float *out_c = out + (size_t)c0 * d;
    for (int i = 0; i < L; ++i) {
      char *trace_i = x_trace ? static_cast<char *>(x_trace) + ((size_t)i * T + c0) * d * 2 : nullptr;
      // layer i writes ylayer[i & 1] and the fused kernel of layer i + 1 reads it: the kernel has
      // no grid barrier, so its CTAs may write their output rows while others still read y_prev
      float *yo = (i == L - 1) ? out_c : g.ylayer[i & 1];
      if (i > 0 && fused) {
        MoeLaunch Lf{s, false};
        rc = moe_launch_fused_decode(Lf, g.W, nullptr, g.ylayer[(i - 1) & 1], eps, trace_i, router_w[i], router_scale[i],
                                     gate_up_q4[i], down_q4[i], expert_scale[i], Tc, d, f, E, k, yo, g.num_sms,
                                     nullptr, nullptr, i + 1 < L ? router_w[i + 1] : nullptr);
        if (rc) return cuda_fail(cudaGetLastError(), "fused decode launch");
        continue;
      }
      if (x_trace) {
        cudaError_t e = cudaMemcpyAsync(trace_i, xc, (size_t)Tc * d * 2, cudaMemcpyDeviceToDevice, s);
        if (e != cudaSuccess) return cuda_fail(e, "x_trace copy");
      }
      rc = forward_impl(xc, router_w[i], router_scale[i], gate_up_q4[i], down_q4[i], expert_scale[i], Tc, d, f, E,
                        k, yo, s, gemm);
      if (rc) return rc;
      if (i < L - 1 && !fused) {
        __nv_bfloat16 *xn = g.xbuf[i & 1];
        if (moe_launch_rmsnorm(s, yo, xn, Tc, d, eps)) return cuda_fail(cudaGetLastError(), "rmsnorm launch");
        xc = xn;
      }
    }
  }
  return MOE_OK;
}

int moe_set_path(int path, int gemv_max_tokens) {
  if (path != MOE_PATH_AUTO && path != MOE_PATH_GEMV && path != MOE_PATH_GEMM && path != MOE_PATH_GEMV_SPLIT)
    return fail(MOE_ERR_BAD_ARG, "unknown path %d", path);
  if (gemv_max_tokens < 0) return fail(MOE_ERR_BAD_ARG, "gemv_max_tokens = %d < 0", gemv_max_tokens);
  g.path = path;
  g.gemv_max_tokens = gemv_max_tokens;
  return MOE_OK;
}

void moe_destroy(void) {
  if (!g.init) return;
  cudaSetDevice(g.device);
  cudaDeviceSynchronize();
  release();
}

const char *moe_last_error(void) { return g_err; }

int moe_debug_get_routing(int32_t *ids, float *w, int32_t *counts, int32_t *offsets, int32_t *perm, void *stream) {
  if (!g.init) return fail(MOE_ERR_NOT_INIT, "moe_init has not succeeded");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t S = (size_t)g.last_T * g.last_k;
  struct Cp { void *dst; const void *src; size_t n; } cps[] = {
      {ids, g.W.ids, S * 4}, {w, g.W.w, S * 4}, {counts, g.W.counts, (size_t)g.last_E * 4},
      {offsets, g.W.offsets, (size_t)(g.last_E + 1) * 4}, {perm, g.W.perm, S * 4}};
  for (auto &c : cps) {
    if (!c.dst || c.n == 0) continue;
    cudaError_t e = cudaMemcpyAsync(c.dst, c.src, c.n, cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "routing copy");
  }
  return MOE_OK;
}

int moe_debug_get_hidden(float *h, void *stream) {
  if (!g.init) return fail(MOE_ERR_NOT_INIT, "moe_init has not succeeded");
  if (!h) return fail(MOE_ERR_BAD_ARG, "null pointer argument");
  if (g.last_T == 0) return MOE_OK;
  if (moe_launch_hidden_to_slots(static_cast<cudaStream_t>(stream), g.W, h, g.last_T, g.last_f, g.last_k,
                                 g.last_gemm))
    return cuda_fail(cudaGetLastError(), "hidden copy");
  return MOE_OK;
}

int moe_debug_check(void *stream) {
  if (!g.init) return fail(MOE_ERR_NOT_INIT, "moe_init has not succeeded");
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  return check_device_error();
}

int moe_debug_set_wait_ns(unsigned long long ns) {
  if (!g.init) return fail(MOE_ERR_NOT_INIT, "moe_init has not succeeded");
  g.W.wait_ns = ns ? ns : MOE_WAIT_NS;
  return MOE_OK;
}

int moe_debug_inject(int fault) {
  if (!g.init) return fail(MOE_ERR_NOT_INIT, "moe_init has not succeeded");
  if (fault != MOE_INJECT_NONE && fault != MOE_INJECT_SKIP_ROUTER_ARRIVAL)
    return fail(MOE_ERR_BAD_ARG, "unknown fault %d", fault);
  g.W.inject = fault;
  return MOE_OK;
}

}  // extern "C"
