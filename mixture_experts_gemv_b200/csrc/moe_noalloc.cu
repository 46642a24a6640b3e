// moe_noalloc.cu -- moe_layer_forward_static: the decode (GEMV) path of the routed-MoE
// layer for callers that cannot let a library allocate device memory.
//
// Who needs it: some host programs forbid cudaMalloc inside a library call -- serving
// engines that reserve all device memory up front in their own pool and account for every
// byte, plugins running inside a host process that owns every allocation, and loops with
// latency budgets where an allocation (and the device-wide synchronisation it can imply)
// would stall other work. moe_layer_forward needs moe_init's workspace; this entry point
// needs nothing but the caller's inputs and outputs.
//
// Its scratch (router logits, routing, reordered activations, h, per-slot outputs, arrival
// counters) is the file-scope array below, MOE_STATIC_SCRATCH_BYTES large. The array
// belongs to the loaded module: every GPU that loads this library holds it until the
// process exits, whether or not the entry point is called. Host code must not pass the
// array's name to a kernel (on the host it names a stand-in, not device memory); the device
// address is obtained once per device with cudaGetSymbolAddress, on the first call made
// while that device is current. That first call should therefore be made before any
// stream capture.
//
// All calls share the one array and leave their contents in it: the arrival counters that
// must start at zero are cleared at the start of every call (cudaMemsetAsync on the
// caller's stream), and two calls whose work overlaps on the GPU (different streams, or
// different host threads) race on the array.
//
// One word of the array is the device error word of these calls: a device-side wait that
// runs out of time records itself there (the kernels then end early and `out` is not fully
// written). It stays set until moe_layer_forward_static_check reads and clears it.
#include <atomic>
#include <cstdio>
#include <mutex>

#include "../../include/moe.h"
#include "moe_common.cuh"

namespace {

// Byte offsets of the scratch sub-buffers, sized for the limits in include/moe.h.
constexpr size_t kAlign = 256;
constexpr size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }
constexpr size_t kT = MOE_STATIC_MAX_TOKENS, kS = MOE_STATIC_MAX_SLOTS, kD = MOE_STATIC_MAX_D,
                 kF = MOE_STATIC_MAX_F, kE = MOE_STATIC_MAX_E;
constexpr size_t kOffLogits = 0;
constexpr size_t kOffIds = align_up(kOffLogits + kT * kE * 4);
constexpr size_t kOffW = align_up(kOffIds + kS * 4);
constexpr size_t kOffCounts = align_up(kOffW + kS * 4);
constexpr size_t kOffOffsets = align_up(kOffCounts + kE * 4);
constexpr size_t kOffPerm = align_up(kOffOffsets + (kE + 1) * 4);
constexpr size_t kOffInv = align_up(kOffPerm + kS * 4);
constexpr size_t kOffAct = align_up(kOffInv + kS * 4);
constexpr size_t kOffNAct = align_up(kOffAct + kE * 4);
constexpr size_t kOffXprep = align_up(kOffNAct + 16);
constexpr size_t kOffXblk = align_up(kOffXprep + kT * kD * 2);
constexpr size_t kOffH = align_up(kOffXblk + kT * (kD / 32) * 8);
constexpr size_t kOffYbuf = align_up(kOffH + kS * kF * 4);
constexpr size_t kCounterWords = 2 + kD / 8;
constexpr size_t kOffCounters = align_up(kOffYbuf + kS * kD * 4);
constexpr size_t kOffErr = align_up(kOffCounters + kCounterWords * 4);   // device error word
constexpr size_t kEnd = align_up(kOffErr + 16);
static_assert(kEnd <= MOE_STATIC_SCRATCH_BYTES, "static scratch layout exceeds MOE_STATIC_SCRATCH_BYTES");

static __device__ __align__(256) unsigned char g_moe_static_scratch[MOE_STATIC_SCRATCH_BYTES];

struct StaticDevice {
  std::atomic<bool> ready{false};     // set (release) after scratch and num_sms are stored
  unsigned char *scratch = nullptr;   // device address of g_moe_static_scratch
  int num_sms = 0;
};
constexpr int kMaxDevices = 64;
StaticDevice g_dev[kMaxDevices];
std::mutex g_setup;   // the one-time set-up of a device runs under it (first calls may race)

int current_device(int *dev, char *msg, size_t n) {
  const cudaError_t e = cudaGetDevice(dev);
  if (e != cudaSuccess || *dev < 0 || *dev >= kMaxDevices) {
    snprintf(msg, n, "moe_layer_forward_static: cudaGetDevice: %s", cudaGetErrorString(e));
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

}  // namespace

int moe_report_error(int code, const char *msg);   // moe_api.cu: sets moe_last_error()

extern "C" int moe_layer_forward_static(const void *x, const float *router_w, const float *router_scale,
                                        const uint8_t *gate_up_q4, const uint8_t *down_q4,
                                        const float *expert_scale, int T, int d, int f, int E, int k,
                                        float *out, void *stream) {
  char msg[256];
  if (T < 0 || d <= 0 || d % 32 || f <= 0 || f % 32 || E < 1 || k < 1 || k > E)
    return moe_report_error(MOE_ERR_BAD_ARG, "moe_layer_forward_static: bad shape (need d, f multiples of 32, "
                                             "1 <= k <= E, T >= 0)");
  if (T > MOE_STATIC_MAX_TOKENS || (long long)T * k > MOE_STATIC_MAX_SLOTS || d > MOE_STATIC_MAX_D ||
      f > MOE_STATIC_MAX_F || E > MOE_STATIC_MAX_E) {
    snprintf(msg, sizeof msg,
             "moe_layer_forward_static: shape (T=%d, d=%d, f=%d, E=%d, k=%d) exceeds the static scratch limits "
             "(T <= %d, T*k <= %d, d <= %d, f <= %d, E <= %d)",
             T, d, f, E, k, MOE_STATIC_MAX_TOKENS, MOE_STATIC_MAX_SLOTS, MOE_STATIC_MAX_D, MOE_STATIC_MAX_F,
             MOE_STATIC_MAX_E);
    return moe_report_error(MOE_ERR_BAD_ARG, msg);
  }
  if (!x || !router_w || !router_scale || !gate_up_q4 || !down_q4 || !expert_scale || !out)
    return moe_report_error(MOE_ERR_BAD_ARG, "moe_layer_forward_static: null pointer argument");
  auto al16 = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!al16(x) || !al16(router_w) || !al16(gate_up_q4) || !al16(down_q4))
    return moe_report_error(MOE_ERR_BAD_ALIGN, "moe_layer_forward_static: x, router_w, gate_up_q4 and down_q4 "
                                               "must be 16-byte aligned");
  if (T == 0) return MOE_OK;

  int dev = -1;
  if (current_device(&dev, msg, sizeof msg) != MOE_OK) return moe_report_error(MOE_ERR_CUDA, msg);
  cudaError_t e;
  StaticDevice &sd = g_dev[dev];
  if (!sd.ready.load(std::memory_order_acquire)) {
    // one-time set-up for this device, made while it is current; host threads making their
    // first call at the same time wait here for the one that does it
    std::lock_guard<std::mutex> lock(g_setup);
    if (!sd.ready.load(std::memory_order_relaxed)) {
      int major = 0, minor = 0, sms = 0;
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
      if (major != 10 || minor != 0) {
        snprintf(msg, sizeof msg, "moe_layer_forward_static: device %d is sm_%d%d, not sm_100", dev, major, minor);
        return moe_report_error(MOE_ERR_UNSUPPORTED_DEVICE, msg);
      }
      void *p = nullptr;
      e = cudaGetSymbolAddress(&p, g_moe_static_scratch);
      if (e != cudaSuccess || p == nullptr) {
        snprintf(msg, sizeof msg, "moe_layer_forward_static: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
        return moe_report_error(MOE_ERR_CUDA, msg);
      }
      sd.scratch = static_cast<unsigned char *>(p);
      sd.num_sms = sms;
      sd.ready.store(true, std::memory_order_release);
    }
  }

  unsigned char *b = sd.scratch;
  MoeWork W{};
  W.logits = reinterpret_cast<float *>(b + kOffLogits);
  W.ids = reinterpret_cast<int32_t *>(b + kOffIds);
  W.w = reinterpret_cast<float *>(b + kOffW);
  W.counts = reinterpret_cast<int32_t *>(b + kOffCounts);
  W.offsets = reinterpret_cast<int32_t *>(b + kOffOffsets);
  W.perm = reinterpret_cast<int32_t *>(b + kOffPerm);
  W.inv = reinterpret_cast<int32_t *>(b + kOffInv);
  W.act = reinterpret_cast<int32_t *>(b + kOffAct);
  W.n_act = reinterpret_cast<int32_t *>(b + kOffNAct);
  W.n_tiles = reinterpret_cast<int32_t *>(b + kOffNAct + 4);
  W.xq = reinterpret_cast<int16_t *>(b + kOffXprep);
  W.xblk = reinterpret_cast<ActBlk *>(b + kOffXblk);
  W.h = reinterpret_cast<float *>(b + kOffH);
  W.ybuf = reinterpret_cast<float *>(b + kOffYbuf);
  W.yslot = W.ybuf;
  W.counters = reinterpret_cast<uint32_t *>(b + kOffCounters);
  W.err = reinterpret_cast<volatile uint32_t *>(b + kOffErr);   // sticky until the check call clears it
  W.wait_ns = MOE_WAIT_NS;
  W.inject = MOE_INJECT_NONE;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  e = cudaMemsetAsync(W.counters, 0, kCounterWords * 4, s);
  if (e != cudaSuccess) {
    snprintf(msg, sizeof msg, "moe_layer_forward_static: clearing counters: %s", cudaGetErrorString(e));
    return moe_report_error(MOE_ERR_CUDA, msg);
  }
  MoeLaunch L{s, false};
  if (moe_launch_route_decode(L, W, x, router_w, router_scale, T, d, E, k, sd.num_sms) != 0) {
    snprintf(msg, sizeof msg, "moe_layer_forward_static: routing launch: %s", cudaGetErrorString(cudaGetLastError()));
    return moe_report_error(MOE_ERR_CUDA, msg);
  }
  const int rc = moe_launch_gemv_experts(L, W, gate_up_q4, down_q4, expert_scale, T, d, f, E, k, out, sd.num_sms);
  if (rc == -2) return moe_report_error(MOE_ERR_BAD_ARG, "moe_layer_forward_static: shape not supported by the GEMV path");
  if (rc != 0) {
    snprintf(msg, sizeof msg, "moe_layer_forward_static: GEMV launch: %s", cudaGetErrorString(cudaGetLastError()));
    return moe_report_error(MOE_ERR_CUDA, msg);
  }
  return MOE_OK;
}

extern "C" int moe_layer_forward_static_check(void *stream) {
  char msg[256];
  int dev = -1;
  if (current_device(&dev, msg, sizeof msg) != MOE_OK) return moe_report_error(MOE_ERR_CUDA, msg);
  StaticDevice &sd = g_dev[dev];
  if (!sd.ready.load(std::memory_order_acquire)) return MOE_OK;   // no call has run on this device
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  uint32_t v = 0;
  if (e == cudaSuccess) e = cudaMemcpy(&v, sd.scratch + kOffErr, sizeof v, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && v != 0) {
    const uint32_t zero = 0;
    e = cudaMemcpy(sd.scratch + kOffErr, &zero, sizeof zero, cudaMemcpyHostToDevice);
  }
  if (e != cudaSuccess) {
    snprintf(msg, sizeof msg, "moe_layer_forward_static_check: %s", cudaGetErrorString(e));
    return moe_report_error(MOE_ERR_CUDA, msg);
  }
  if (v != 0) {
    snprintf(msg, sizeof msg,
             "moe_layer_forward_static: a device wait timed out (code %u at site %u); the output of that call "
             "is not valid", v & 0xffffu, v >> 16);
    return moe_report_error(MOE_ERR_DEVICE_TIMEOUT, msg);
  }
  return MOE_OK;
}
