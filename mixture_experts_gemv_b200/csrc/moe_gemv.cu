// moe_gemv.cu -- decode path: Q4_0 GEMVs of the active experts with FP32 accumulation.
//
// Page "Gemma 4 26B-A4B it QAT Q4_0 ... NInfer v3 artifact", "What is inside": each routed
// expert is [gate; up] (2 x 704 rows) and down (2,816 rows) of ggml Q4_0 blocks, multiplied
// in place. For every active expert e and each slot (t, j) routed to it:
//   g = Wg_e x_t, u = Wu_e x_t, h = gelu_tanh(g) * u          (k_gateup_gemv)
//   y = Wd_e h                                                 (k_down_gemv_combine)
//   out[t, r] = sum_j w_tj * expert_scale[e_tj] * y_tj[r]      (same kernel, last arriver)
//
// Memory: every weight byte of an active expert is read once. The flat space of 8-row
// units of all active experts is split evenly over one CTA per SM; each CTA streams its
// units through a ring of shared-memory stages filled by 1-D bulk asynchronous copies
// (cp.async.bulk, mbarrier completion), so HBM reads stay in flight while the SM decodes.
//
// Arithmetic: a Q4_0 weight is (q - 8) * d. Per block and token the kernel forms
// sum_i q_i x_i exactly term by term (products of a 4-bit integer and a bf16 value are
// exact in FP32) from codes turned into floats by OR-ing them into the mantissa of 2^23,
// then adds d * (that sum - 8 * sum_i x_i) to the row's FP32 accumulator.
#include "moe_common.cuh"

namespace {

constexpr int kThreads = 256;
constexpr int kStagesMax = 4;
constexpr int kGuPairs = 16;   // row pairs (gate c, up f+c) per gate_up chunk
constexpr int kGuParts = 16;   // a row's blocks are split over 16 threads
constexpr int kDnRows = 128;   // rows per down chunk
constexpr int kDnParts = 2;
constexpr int kUnit = 8;       // rows (or row pairs) per scheduling unit
constexpr int kTG = 4;         // tokens per pass over a staged chunk
constexpr uint32_t kMagic = 0x4B000000u;   // 2^23
constexpr int kSmemBudget = 200 * 1024;   // dynamic ring; static smem comes on top

__device__ __forceinline__ float gelu_tanh_f(float z) {
  const float c = 0.7978845608028654f;   // sqrt(2/pi)
  return 0.5f * z * (1.0f + tanhf(c * (z + 0.044715f * z * z * z)));
}

// Element index inside a 32-wide block -> position in the (code word, nibble) order
// used by xprep / hprep, and that position's power-of-two scale.
__device__ __forceinline__ int nib_pos(int e) {
  if (e < 16) return 8 * (e >> 2) + 2 * (e & 3);
  const int e2 = e - 16;
  return 8 * (e2 >> 2) + 2 * (e2 & 3) + 1;
}
__device__ __forceinline__ float nib_scale_pos(int p) {
  const int j = p & 7;
  const int s = (j <= 4) ? 4 * j : 4 * (j - 3);
  return __int_as_float((127 - s) << 23);
}

// Read one 18-byte block at byte offset `o` of shared memory (2-byte aligned).
struct Blk {
  float d;
  uint32_t q[4];
};
__device__ __forceinline__ Blk load_blk(const uint8_t *smem, uint32_t o) {
  const uint32_t a = o & ~3u;
  const uint32_t sh = (o & 3u) * 8u;   // 0 or 16
  const uint32_t *wp = reinterpret_cast<const uint32_t *>(smem + a);
  uint32_t w0 = wp[0], w1 = wp[1], w2 = wp[2], w3 = wp[3], w4 = wp[4];
  Blk b;
  b.d = __half2float(__ushort_as_half((unsigned short)((w0 >> sh) & 0xffffu)));
  const uint32_t s2 = sh + 16u;
  b.q[0] = __funnelshift_rc(w0, w1, s2);
  b.q[1] = __funnelshift_rc(w1, w2, s2);
  b.q[2] = __funnelshift_rc(w2, w3, s2);
  b.q[3] = __funnelshift_rc(w3, w4, s2);
  return b;
}

// Eight codes of one word as exact floats q * 2^s_j, in nibble order j = 0..7.
__device__ __forceinline__ void codes8(uint32_t w, float2 &c01, float2 &c23, float2 &c45, float2 &c67) {
  const uint32_t w12 = w >> 12;
  const float2 m = make_float2(-8388608.f, -8388608.f);
  c01 = __fadd2_rn(make_float2(__uint_as_float((w & 0xFu) | kMagic), __uint_as_float((w & 0xF0u) | kMagic)), m);
  c23 = __fadd2_rn(make_float2(__uint_as_float((w & 0xF00u) | kMagic), __uint_as_float((w & 0xF000u) | kMagic)), m);
  c45 = __fadd2_rn(make_float2(__uint_as_float((w & 0xF0000u) | kMagic), __uint_as_float((w12 & 0xF00u) | kMagic)), m);
  c67 = __fadd2_rn(make_float2(__uint_as_float((w12 & 0xF000u) | kMagic), __uint_as_float((w12 & 0xF0000u) | kMagic)), m);
}

struct RingCtl {
  uint64_t full[kStagesMax];
};

// Flat split of n units over the grid.
__device__ __forceinline__ void my_units(int n, int &u0, int &u1) {
  u0 = (int)((long long)n * blockIdx.x / gridDim.x);
  u1 = (int)((long long)n * (blockIdx.x + 1) / gridDim.x);
}

// ---------------------------------------------------------------- gate_up + GeGLU

struct GuChunk {
  int a, c0, np;   // active-expert index, first row pair, row pairs (8 or 16)
};

__device__ __forceinline__ GuChunk gu_chunk(int u, int u1, int upe) {
  GuChunk c;
  c.a = u / upe;
  const int r = u % upe;
  c.c0 = r * kUnit;
  const int n = (u + 1 < u1 && (u + 1) / upe == c.a) ? 2 : 1;
  c.np = n * kUnit;
  return c;
}

__global__ void __launch_bounds__(kThreads, 1)
k_gateup_gemv(const uint8_t *__restrict__ gate_up_q4, int d, int f, int k, int nstages, MoeWork W) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((128u - (smem_u32(smem_raw) & 127u)) & 127u);
  __shared__ RingCtl ring;
  __shared__ float red[kGuParts][kGuPairs][kTG][2];

  const int nb = d / MOE_QK;
  const uint32_t rb = (uint32_t)nb * MOE_QBYTES;                // bytes per row
  const uint32_t stage_bytes = 2u * kGuPairs * rb + 16u;        // + slack for 20-byte block reads
  const int upe = f / kUnit;                                    // units per expert
  const int n_act = *W.n_act;
  int u0, u1;
  my_units(n_act * upe, u0, u1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < nstages; ++s) mbar_init(&ring.full[s], 1);
    fence_mbar_init();
  }
  __syncthreads();

  auto issue = [&](int u, int slot) {
    const GuChunk c = gu_chunk(u, u1, upe);
    const int e = W.act[c.a];
    const uint8_t *base = gate_up_q4 + (size_t)e * 2 * f * rb;
    uint8_t *dst = smem + (size_t)slot * stage_bytes;
    const uint32_t bytes = (uint32_t)c.np * rb;
    mbar_arrive_expect_tx(&ring.full[slot], 2u * bytes);
    bulk_g2s(dst, base + (size_t)c.c0 * rb, bytes, &ring.full[slot]);
    bulk_g2s(dst + kGuPairs * rb, base + (size_t)(f + c.c0) * rb, bytes, &ring.full[slot]);
  };

  int u_issue = u0;   // thread 0's cursor: next chunk to issue
  if (threadIdx.x == 0) {
    for (int s = 0; s < nstages && u_issue < u1; ++s) {
      issue(u_issue, s);
      u_issue += gu_chunk(u_issue, u1, upe).np / kUnit;
    }
  }

  const int p = threadIdx.x % kGuPairs;    // row pair inside the chunk
  const int q = threadIdx.x / kGuPairs;    // part of the row's blocks
  const int bpp = (nb + kGuParts - 1) / kGuParts;
  const int b0 = q * bpp, b1 = min(nb, b0 + bpp);

  int it = 0;
  for (int u = u0; u < u1; ++it) {
    const GuChunk c = gu_chunk(u, u1, upe);
    const int slot = it % nstages;
    const uint32_t par = (uint32_t)(it / nstages) & 1u;
    const bool ok = mbar_wait(&ring.full[slot], par, W.err, 1);
    if (__syncthreads_or(!ok)) return;

    const int e = W.act[c.a];
    const int cnt = W.counts[e];
    const int off = W.offsets[e];
    const uint8_t *st = smem + (size_t)slot * stage_bytes;
    const uint32_t og = (uint32_t)p * rb, ou = (uint32_t)(kGuPairs + p) * rb;

    for (int g0 = 0; g0 < cnt; g0 += kTG) {
      const int ng = min(kTG, cnt - g0);
      int tok[kTG];
#pragma unroll
      for (int i = 0; i < kTG; ++i) tok[i] = (i < ng) ? W.perm[off + g0 + i] / k : 0;
      float yg[kTG], yu[kTG];
#pragma unroll
      for (int i = 0; i < kTG; ++i) { yg[i] = 0.f; yu[i] = 0.f; }
      if (p < c.np) {
        for (int b = b0; b < b1; ++b) {
          const Blk bg = load_blk(st, og + (uint32_t)b * MOE_QBYTES);
          const Blk bu = load_blk(st, ou + (uint32_t)b * MOE_QBYTES);
          float2 ag[kTG], au[kTG];
#pragma unroll
          for (int i = 0; i < kTG; ++i) { ag[i] = make_float2(0.f, 0.f); au[i] = make_float2(0.f, 0.f); }
#pragma unroll
          for (int wi = 0; wi < 4; ++wi) {
            float2 g01, g23, g45, g67, v01, v23, v45, v67;
            codes8(bg.q[wi], g01, g23, g45, g67);
            codes8(bu.q[wi], v01, v23, v45, v67);
#pragma unroll
            for (int i = 0; i < kTG; ++i) {
              if (i < ng) {
                const float4 *xp = reinterpret_cast<const float4 *>(
                    W.xprep + (size_t)tok[i] * d + (size_t)b * MOE_QK + 8 * wi);
                const float4 xa = __ldg(xp), xb = __ldg(xp + 1);
                const float2 x01 = make_float2(xa.x, xa.y), x23 = make_float2(xa.z, xa.w);
                const float2 x45 = make_float2(xb.x, xb.y), x67 = make_float2(xb.z, xb.w);
                ag[i] = __ffma2_rn(g01, x01, ag[i]);
                ag[i] = __ffma2_rn(g23, x23, ag[i]);
                ag[i] = __ffma2_rn(g45, x45, ag[i]);
                ag[i] = __ffma2_rn(g67, x67, ag[i]);
                au[i] = __ffma2_rn(v01, x01, au[i]);
                au[i] = __ffma2_rn(v23, x23, au[i]);
                au[i] = __ffma2_rn(v45, x45, au[i]);
                au[i] = __ffma2_rn(v67, x67, au[i]);
              }
            }
          }
#pragma unroll
          for (int i = 0; i < kTG; ++i) {
            if (i < ng) {
              const float sx = __ldg(W.xsum + (size_t)tok[i] * nb + b);
              yg[i] = fmaf(bg.d, fmaf(-8.f, sx, ag[i].x + ag[i].y), yg[i]);
              yu[i] = fmaf(bu.d, fmaf(-8.f, sx, au[i].x + au[i].y), yu[i]);
            }
          }
        }
      }
#pragma unroll
      for (int i = 0; i < kTG; ++i) { red[q][p][i][0] = yg[i]; red[q][p][i][1] = yu[i]; }
      __syncthreads();
      if (threadIdx.x < kGuPairs * kTG) {
        const int pp = threadIdx.x % kGuPairs, i = threadIdx.x / kGuPairs;
        if (pp < c.np && i < ng) {
          float g = 0.f, uu = 0.f;
          for (int qq = 0; qq < kGuParts; ++qq) { g += red[qq][pp][i][0]; uu += red[qq][pp][i][1]; }
          const float hv = gelu_tanh_f(g) * uu;
          const int slotid = W.perm[off + g0 + i];
          const int cidx = c.c0 + pp;
          W.h[(size_t)slotid * f + cidx] = hv;
          const int cb = cidx / MOE_QK, ce = cidx % MOE_QK;
          const int pos = nib_pos(ce);
          W.hprep[(size_t)slotid * f + (size_t)cb * MOE_QK + pos] = hv * nib_scale_pos(pos);
        }
      }
      __syncthreads();
    }
    u += c.np / kUnit;
    // stage `slot` is free: refill it
    if (threadIdx.x == 0 && u_issue < u1) {
      issue(u_issue, slot);
      u_issue += gu_chunk(u_issue, u1, upe).np / kUnit;
    }
  }
}

// ---------------------------------------------------------------- down + combine

struct DnChunk {
  int a, r0, nr;
};

__device__ __forceinline__ DnChunk dn_chunk(int u, int u1, int upe) {
  DnChunk c;
  c.a = u / upe;
  const int r = u % upe;
  c.r0 = r * kUnit;
  int n = 1;
  while (n < kDnRows / kUnit && u + n < u1 && (u + n) / upe == c.a) ++n;
  c.nr = n * kUnit;
  return c;
}

__global__ void __launch_bounds__(kThreads, 1)
k_down_gemv_combine(const uint8_t *__restrict__ down_q4, const float *__restrict__ expert_scale, int T,
                    int d, int f, int k, int nstages, float *__restrict__ out, MoeWork W) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((128u - (smem_u32(smem_raw) & 127u)) & 127u);
  __shared__ RingCtl ring;
  __shared__ float red[kDnParts][kDnRows][kTG];
  __shared__ float hs[kTG][64];           // per-block sums of h for the token group (f/32 <= 64)
  __shared__ int done_units[kDnRows / kUnit];
  __shared__ int n_done;

  const int nbf = f / MOE_QK;
  const uint32_t rb = (uint32_t)nbf * MOE_QBYTES;
  const uint32_t stage_bytes = (uint32_t)kDnRows * rb + 16u;
  const int upe = d / kUnit;
  const int n_act = *W.n_act;
  int u0, u1;
  my_units(n_act * upe, u0, u1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < nstages; ++s) mbar_init(&ring.full[s], 1);
    fence_mbar_init();
  }
  __syncthreads();

  auto issue = [&](int u, int slot) {
    const DnChunk c = dn_chunk(u, u1, upe);
    const int e = W.act[c.a];
    const uint8_t *src = down_q4 + (size_t)e * d * rb + (size_t)c.r0 * rb;
    const uint32_t bytes = (uint32_t)c.nr * rb;
    mbar_arrive_expect_tx(&ring.full[slot], bytes);
    bulk_g2s(smem + (size_t)slot * stage_bytes, src, bytes, &ring.full[slot]);
  };
  int u_issue = u0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < nstages && u_issue < u1; ++s) {
      issue(u_issue, s);
      u_issue += dn_chunk(u_issue, u1, upe).nr / kUnit;
    }
  }

  const int p = threadIdx.x % kDnRows;
  const int q = threadIdx.x / kDnRows;
  const int bpp = (nbf + kDnParts - 1) / kDnParts;
  const int b0 = q * bpp, b1 = min(nbf, b0 + bpp);

  int it = 0;
  for (int u = u0; u < u1; ++it) {
    const DnChunk c = dn_chunk(u, u1, upe);
    const int slot = it % nstages;
    const uint32_t par = (uint32_t)(it / nstages) & 1u;
    const bool ok = mbar_wait(&ring.full[slot], par, W.err, 2);
    if (__syncthreads_or(!ok)) return;

    const int e = W.act[c.a];
    const int cnt = W.counts[e];
    const int off = W.offsets[e];
    const uint8_t *st = smem + (size_t)slot * stage_bytes;
    const uint32_t orow = (uint32_t)p * rb;

    for (int g0 = 0; g0 < cnt; g0 += kTG) {
      const int ng = min(kTG, cnt - g0);
      int sl[kTG];
#pragma unroll
      for (int i = 0; i < kTG; ++i) sl[i] = (i < ng) ? W.perm[off + g0 + i] : 0;
      // block sums of h for these slots
      for (int i2 = threadIdx.x; i2 < kTG * nbf; i2 += kThreads) {
        const int i = i2 / nbf, cb = i2 % nbf;
        float s = 0.f;
        if (i < ng) {
          const float *hp = W.h + (size_t)sl[i] * f + (size_t)cb * MOE_QK;
          for (int c2 = 0; c2 < MOE_QK; ++c2) s += hp[c2];
        }
        hs[i][cb] = s;
      }
      __syncthreads();
      float y[kTG];
#pragma unroll
      for (int i = 0; i < kTG; ++i) y[i] = 0.f;
      if (p < c.nr) {
        for (int b = b0; b < b1; ++b) {
          const Blk bk = load_blk(st, orow + (uint32_t)b * MOE_QBYTES);
          float2 acc[kTG];
#pragma unroll
          for (int i = 0; i < kTG; ++i) acc[i] = make_float2(0.f, 0.f);
#pragma unroll
          for (int wi = 0; wi < 4; ++wi) {
            float2 c01, c23, c45, c67;
            codes8(bk.q[wi], c01, c23, c45, c67);
#pragma unroll
            for (int i = 0; i < kTG; ++i) {
              if (i < ng) {
                const float4 *hp = reinterpret_cast<const float4 *>(
                    W.hprep + (size_t)sl[i] * f + (size_t)b * MOE_QK + 8 * wi);
                const float4 ha = hp[0], hb = hp[1];
                acc[i] = __ffma2_rn(c01, make_float2(ha.x, ha.y), acc[i]);
                acc[i] = __ffma2_rn(c23, make_float2(ha.z, ha.w), acc[i]);
                acc[i] = __ffma2_rn(c45, make_float2(hb.x, hb.y), acc[i]);
                acc[i] = __ffma2_rn(c67, make_float2(hb.z, hb.w), acc[i]);
              }
            }
          }
#pragma unroll
          for (int i = 0; i < kTG; ++i)
            if (i < ng) y[i] = fmaf(bk.d, fmaf(-8.f, hs[i][b], acc[i].x + acc[i].y), y[i]);
        }
      }
#pragma unroll
      for (int i = 0; i < kTG; ++i) red[q][p][i] = y[i];
      __syncthreads();
      for (int i2 = threadIdx.x; i2 < kDnRows * kTG; i2 += kThreads) {
        const int pp = i2 % kDnRows, i = i2 / kDnRows;
        if (pp < c.nr && i < ng) {
          float s = red[0][pp][i];
#pragma unroll
          for (int qq = 1; qq < kDnParts; ++qq) s += red[qq][pp][i];
          W.ybuf[(size_t)sl[i] * d + c.r0 + pp] = s;
        }
      }
      __syncthreads();
    }
    // this chunk's rows of expert e are final: count arrivals per 8-row unit
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
      int nd = 0;
      for (int uu = 0; uu < c.nr / kUnit; ++uu) {
        const int unit = c.r0 / kUnit + uu;
        const uint32_t prev = atomicAdd(&W.counters[1 + unit], 1u);
        if (prev == (uint32_t)n_act - 1u) done_units[nd++] = unit;
      }
      n_done = nd;
    }
    __syncthreads();
    if (n_done > 0) {
      __threadfence();
      for (int i2 = threadIdx.x; i2 < n_done * kUnit * T; i2 += kThreads) {
        const int un = i2 / (kUnit * T), rem = i2 % (kUnit * T);
        const int t = rem / kUnit, r = done_units[un] * kUnit + rem % kUnit;
        float s = 0.f;
        for (int j = 0; j < k; ++j) {
          const int slotid = t * k + j;
          s += W.w[slotid] * expert_scale[W.ids[slotid]] * __ldcg(W.ybuf + (size_t)slotid * d + r);
        }
        out[(size_t)t * d + r] = s;
      }
      __syncthreads();
      if (threadIdx.x < n_done) W.counters[1 + done_units[threadIdx.x]] = 0;
    }
    u += c.nr / kUnit;
    if (threadIdx.x == 0 && u_issue < u1) {
      issue(u_issue, slot);
      u_issue += dn_chunk(u_issue, u1, upe).nr / kUnit;
    }
    __syncthreads();
  }
}

// h of the grouped-GEMM path (bf16, padded tile rows) -> fp32 slot order.
__global__ void k_hidden_slots_from_bf16(const __nv_bfloat16 *hb, const int32_t *ids, const int32_t *inv,
                                         const int32_t *offsets, const int32_t *toff, int S, int f, float *h) {
  const long long n = (long long)S * f;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const int s = (int)(i / f), c = (int)(i % f);
    const int e = ids[s];
    const long long prow = (long long)toff[e] * 128 + (inv[s] - offsets[e]);
    h[i] = __bfloat162float(hb[prow * f + c]);
  }
}

}  // namespace

static int launch_err() { return cudaGetLastError() == cudaSuccess ? 0 : -1; }

int moe_launch_gemv_experts(const MoeLaunch &L, const MoeWork &W, const uint8_t *gate_up_q4,
                            const uint8_t *down_q4, const float *expert_scale, int T, int d, int f,
                            int E, int k, float *out, int num_sms) {
  (void)E;
  const uint32_t gu_stage = 2u * kGuPairs * (uint32_t)(d / MOE_QK) * MOE_QBYTES + 16u;
  const uint32_t dn_stage = (uint32_t)kDnRows * (uint32_t)(f / MOE_QK) * MOE_QBYTES + 16u;
  int gu_st = (int)(kSmemBudget / gu_stage);
  int dn_st = (int)(kSmemBudget / dn_stage);
  if (gu_st > kStagesMax) gu_st = kStagesMax;
  if (dn_st > kStagesMax) dn_st = kStagesMax;
  if (gu_st < 2 || dn_st < 2 || f / MOE_QK > 64) return -2;
  const size_t gu_smem = (size_t)gu_st * gu_stage + 128, dn_smem = (size_t)dn_st * dn_stage + 128;
  static size_t gu_set = 0, dn_set = 0;
  if (gu_smem > gu_set) {
    if (cudaFuncSetAttribute(k_gateup_gemv, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gu_smem) != cudaSuccess) return -1;
    gu_set = gu_smem;
  }
  if (dn_smem > dn_set) {
    if (cudaFuncSetAttribute(k_down_gemv_combine, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dn_smem) != cudaSuccess) return -1;
    dn_set = dn_smem;
  }
  moe_prof_mark(L.stream, MOE_K_GATEUP, true);
  k_gateup_gemv<<<num_sms, kThreads, gu_smem, L.stream>>>(gate_up_q4, d, f, k, gu_st, W);
  if (launch_err()) return -1;
  moe_prof_mark(L.stream, MOE_K_GATEUP, false);
  moe_prof_mark(L.stream, MOE_K_DOWN, true);
  k_down_gemv_combine<<<num_sms, kThreads, dn_smem, L.stream>>>(down_q4, expert_scale, T, d, f, k, dn_st, out, W);
  if (launch_err()) return -1;
  moe_prof_mark(L.stream, MOE_K_DOWN, false);
  return 0;
}

int moe_launch_hidden_to_slots(cudaStream_t s, const MoeWork &W, float *h, int T, int f, int k, bool gemm_path) {
  const int S = T * k;
  if (!gemm_path) {
    if (cudaMemcpyAsync(h, W.h, sizeof(float) * (size_t)S * f, cudaMemcpyDeviceToDevice, s) != cudaSuccess) return -1;
    return 0;
  }
  k_hidden_slots_from_bf16<<<256, 256, 0, s>>>(W.hb, W.ids, W.inv, W.offsets, W.toff, S, f, h);
  return launch_err();
}
