// moe_decode.cu -- the whole routed-MoE layer for small token counts (decode) in one
// persistent kernel: one CTA per SM, launched cooperatively so all CTAs are resident.
//
//   phase 0  router logits (one expert per CTA, warps split d) and the GEMV activations
//   barrier  (grid-wide, bounded wait)
//   phase 1  every CTA selects the top-k experts of every token and builds the stable
//            permutation in its own shared memory (T*k <= 128 slots: no global round trips)
//   phase 2  gate_up GEMV + GeGLU over this CTA's share of the active experts' rows; the
//            bulk-copy ring keeps streaming, so this CTA's down rows are already loading
//   barrier  (h complete)
//   phase 3  down GEMV over this CTA's share of the active experts' down rows
//   barrier  (per-slot outputs complete)
//   phase 4  combine: out[t, r] = sum_j w_tj * s_e * y_tj[r], j in order, rows split over CTAs
//
// Definitions as in moe_route.cu / moe_gemv.cu (page "Gemma 4 26B-A4B it QAT Q4_0 ... NInfer
// v3 artifact", "What is inside"). Results equal the separate-kernel path's up to the order
// of the router's FP32 partial sums.
#include "moe_gemv_core.cuh"
#include "moe_route_core.cuh"

namespace {

constexpr int kFMaxT = 8;          // tokens per call on the fused path
constexpr int kFMaxSlots = 128;    // T * k
constexpr int kFStages = 3;
constexpr int kFMaxWarps = 16;

struct FusedShared {
  uint64_t full[kFStages];
  int32_t ids[kFMaxSlots];
  float w[kFMaxSlots];
  int32_t perm[kFMaxSlots];
  int32_t inv[kFMaxSlots];
  int32_t counts[MOE_MAX_E];
  int32_t offsets[MOE_MAX_E + 1];
  int32_t act[MOE_MAX_E];
  int32_t cnt[MOE_MAX_E];
  int32_t pcost[2][MOE_MAX_E + 1];   // per active expert: cost prefix of its gate_up / down units
  int32_t scan_tmp[64];
  float part[kFMaxWarps][kFMaxT];
  int n_act;
  int st_key[kTX + 1];
  int ok;
};

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long *p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// Grid-wide barrier on a monotonically increasing 64-bit counter: arrival k of a phase
// waits for the counter to reach the end of its window of gridDim.x arrivals. Bounded.
__device__ bool grid_barrier(unsigned long long *ctr, volatile uint32_t *err, uint32_t where, int &ok_s) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned long long n = gridDim.x;
    const unsigned long long old = atomicAdd(ctr, 1ull);
    const unsigned long long target = (old / n + 1ull) * n;
    int ok = 1;
    if (ld_acquire_u64(ctr) < target) {
      const uint64_t t0 = globaltimer_ns();
      while (ld_acquire_u64(ctr) < target) {
        if (globaltimer_ns() - t0 > MOE_WAIT_NS) {
          report_error(err, MOE_DEV_ERR_TIMEOUT, where);
          ok = 0;
          break;
        }
      }
    }
    __threadfence();
    ok_s = ok;
  }
  __syncthreads();
  return ok_s != 0;
}

struct FChunk {
  int down;   // 0: gate_up chunk, 1: down chunk
  int a, r0, n;
};

// The CTA's chunk sequence: its gate_up units (grouped in chunks of up to 2 units of 8 row
// pairs inside one expert), then its down units (chunks of up to 16 units of 8 rows).
struct FSeq {
  int g0, g1, d0, d1, upe_g, upe_d;
  __device__ FChunk at(int u) const {   // u: position in the concatenated unit sequence
    FChunk c;
    if (u < g1 - g0) {
      const int v = g0 + u;
      c.down = 0;
      c.a = v / upe_g;
      c.r0 = (v % upe_g) * kUnit;
      c.n = (v + 1 < g1 && (v + 1) / upe_g == c.a) ? 2 : 1;
    } else {
      const int v = d0 + (u - (g1 - g0));
      c.down = 1;
      c.a = v / upe_d;
      c.r0 = (v % upe_d) * kUnit;
      int n = 1;
      while (n < kDnRows / kUnit && v + n < d1 && (v + n) / upe_d == c.a) ++n;
      c.n = n;
    }
    return c;
  }
  __device__ int total() const { return (g1 - g0) + (d1 - d0); }
};

__global__ void __launch_bounds__(kFMaxWarps * 32, 1)
k_moe_decode(const __nv_bfloat16 *__restrict__ x, const float *__restrict__ router_w,
             const float *__restrict__ router_scale, const uint8_t *__restrict__ gate_up_q4,
             const uint8_t *__restrict__ down_q4, const float *__restrict__ expert_scale, int T, int d, int f,
             int E, int k, float *__restrict__ out, uint32_t stage_bytes, MoeWork W) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  __shared__ FusedShared sh;
  const int lane = threadIdx.x & 31, wq = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int nb = d / MOE_QK, nbf = f / MOE_QK;
  const int G = (nb + kGran - 1) / kGran;
  const uint32_t rb_g = (uint32_t)nb * MOE_QBYTES, rb_d = (uint32_t)nbf * MOE_QBYTES;
  uint8_t *smem = align128(smem_raw);
  uint16_t *xs = reinterpret_cast<uint16_t *>(smem + (size_t)kFStages * stage_bytes);   // [kTX][d]
  float2 *ss = reinterpret_cast<float2 *>(xs + (size_t)kTX * d);                          // [kTX][nb]
  uint16_t *hs = reinterpret_cast<uint16_t *>(ss + (size_t)kTX * nb);                     // [kTX][f]
  float2 *hbk = reinterpret_cast<float2 *>(hs + (size_t)kTX * f);                         // [kTX][nbf]
  float *red = reinterpret_cast<float *>(hbk + (size_t)kTX * nbf);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kFStages; ++s) mbar_init(&sh.full[s], 1);
    fence_mbar_init();
    for (int i = 0; i <= kTX; ++i) sh.st_key[i] = -1;
  }

  // ---------------------------------------------------------------- phase 0: router
  for (int e = blockIdx.x; e < E; e += gridDim.x) {
    float acc[kFMaxT];
#pragma unroll
    for (int t = 0; t < kFMaxT; ++t) acc[t] = 0.f;
    const int seg = (d / 4) / nw * 4;   // float4-aligned slice per warp; the last warp takes the tail
    const int i0 = wq * seg, i1 = (wq == nw - 1) ? d : i0 + seg;
    const float *wr = router_w + (size_t)e * d;
    for (int i = i0 + lane * 4; i + 3 < i1; i += 128) {
      const float4 wv = __ldg(reinterpret_cast<const float4 *>(wr + i));
#pragma unroll
      for (int t = 0; t < kFMaxT; ++t) {
        if (t < T) {
          const uint2 xv = __ldg(reinterpret_cast<const uint2 *>(x + (size_t)t * d + i));
          float a = acc[t];
          a = fmaf(wv.x, __uint_as_float(xv.x << 16), a);
          a = fmaf(wv.y, __uint_as_float(xv.x & 0xffff0000u), a);
          a = fmaf(wv.z, __uint_as_float(xv.y << 16), a);
          a = fmaf(wv.w, __uint_as_float(xv.y & 0xffff0000u), a);
          acc[t] = a;
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kFMaxT; ++t) {
      float a = acc[t];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
      if (lane == 0) sh.part[wq][t] = a;
    }
    __syncthreads();
    if (threadIdx.x < T) {
      float s = 0.f;
      for (int q = 0; q < nw; ++q) s += sh.part[q][threadIdx.x];
      W.logits[(size_t)threadIdx.x * E + e] = s;
    }
    __syncthreads();
  }
  prep_x_range(x, W.x16, W.xblk, T, d, blockIdx.x * blockDim.x + threadIdx.x, gridDim.x * blockDim.x);
  if (!grid_barrier(W.gbar, W.err, 20, sh.ok)) return;

  // ---------------------------------------------------------------- phase 1: selection
  const float rs = *router_scale;
  for (int t = wq; t < T; t += nw)
    warp_topk_softmax(W.logits + (size_t)t * E, E, k, rs, sh.ids + t * k, sh.w + t * k);
  __syncthreads();
  const int S = T * k;
  block_permutation_direct(sh.ids, S, E, sh.counts, sh.offsets, sh.perm, sh.inv, sh.act, &sh.n_act, sh.cnt,
                           sh.scan_tmp);
  if (blockIdx.x == 0) {   // routing copies for the debug readers
    for (int i = threadIdx.x; i < S; i += blockDim.x) {
      W.ids[i] = sh.ids[i];
      W.w[i] = sh.w[i];
      W.perm[i] = sh.perm[i];
      W.inv[i] = sh.inv[i];
    }
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      W.counts[e] = sh.counts[e];
      W.offsets[e] = sh.offsets[e];
      W.act[e] = sh.act[e];
    }
    if (threadIdx.x == 0) {
      W.offsets[E] = sh.offsets[E];
      *W.n_act = sh.n_act;
    }
  }
  const int n_act = sh.n_act;

  // ---------------------------------------------------------------- chunk sequence + ring
  // Units (8 row pairs of gate_up, 8 rows of down) are split over the CTAs by cost, not by
  // bytes: a unit of an expert with T_e tokens costs kUnitDecode + kUnitToken * T_e (decoding
  // the codes is shared by the tokens, the multiply-adds are per token).
  constexpr int kUnitDecode = 5, kUnitToken = 4;
  FSeq seq;
  seq.upe_g = f / kUnit;
  seq.upe_d = d / kUnit;
  for (int a = threadIdx.x; a < n_act; a += blockDim.x) {
    const int c = kUnitDecode + kUnitToken * sh.counts[sh.act[a]];
    sh.pcost[0][a] = c * seq.upe_g;
    sh.pcost[1][a] = c * seq.upe_d;
  }
  __syncthreads();
  int32_t cg_tot, cd_tot;
  block_exclusive_scan2_smem(sh.pcost[0], sh.pcost[1], n_act, sh.scan_tmp, cg_tot, cd_tot);
  auto unit_at = [&](const int32_t *pc, int tot, int upe, int b) -> int {
    // first unit whose cost start is >= b * tot / G
    const long long x = (long long)tot * b / gridDim.x;
    int lo = 0, hi = n_act;   // largest a with pc[a] <= x
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (pc[mid] <= x) lo = mid; else hi = mid;
    }
    if (b >= (int)gridDim.x || n_act == 0) return n_act * upe;
    const int c = kUnitDecode + kUnitToken * sh.counts[sh.act[lo]];
    const long long inexp = (x - pc[lo] + c - 1) / c;   // units of expert lo starting before x
    return lo * upe + (int)(inexp < upe ? inexp : upe);
  };
  seq.g0 = unit_at(sh.pcost[0], cg_tot, seq.upe_g, blockIdx.x);
  seq.g1 = unit_at(sh.pcost[0], cg_tot, seq.upe_g, blockIdx.x + 1);
  seq.d0 = unit_at(sh.pcost[1], cd_tot, seq.upe_d, blockIdx.x);
  seq.d1 = unit_at(sh.pcost[1], cd_tot, seq.upe_d, blockIdx.x + 1);
  const int n_units = seq.total();
  auto issue = [&](int u, int slot) {
    const FChunk c = seq.at(u);
    const int e = sh.act[c.a];
    uint8_t *dst = smem + (size_t)slot * stage_bytes;
    if (!c.down) {
      const uint8_t *base = gate_up_q4 + (size_t)e * 2 * f * rb_g;
      const uint32_t bytes = (uint32_t)(c.n * kUnit) * rb_g;
      mbar_arrive_expect_tx(&sh.full[slot], 2u * bytes);
      bulk_g2s(dst, base + (size_t)c.r0 * rb_g, bytes, &sh.full[slot]);
      bulk_g2s(dst + kPairs * rb_g, base + (size_t)(f + c.r0) * rb_g, bytes, &sh.full[slot]);
    } else {
      const uint32_t bytes = (uint32_t)(c.n * kUnit) * rb_d;
      mbar_arrive_expect_tx(&sh.full[slot], bytes);
      bulk_g2s(dst, down_q4 + (size_t)e * d * rb_d + (size_t)c.r0 * rb_d, bytes, &sh.full[slot]);
    }
  };
  int u_issue = 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kFStages && u_issue < n_units; ++s) {
      issue(u_issue, s);
      u_issue += seq.at(u_issue).n;
    }
  }

  float *my_red_g = red + ((size_t)(wq * kPairs + (lane >> 1)) * kTX) * 2;
  float *my_red_d = red + (size_t)((wq >> 2) & 1) * kTX * kDnRows + (wq & 3) * 32 + lane;
  const bool aligned = (nb % kGran) == 0;
  bool down_phase = false;
  int it = 0;
  for (int u = 0; u < n_units; ++it) {
    const FChunk c = seq.at(u);
    if (c.down && !down_phase) {
      // all h written before any CTA reads it
      if (!grid_barrier(W.gbar, W.err, 21, sh.ok)) return;
      down_phase = true;
      if (threadIdx.x == 0) sh.st_key[0] = -1;
      __syncthreads();
    }
    const int slot = it % kFStages;
    const uint32_t par = (uint32_t)(it / kFStages) & 1u;
    const bool okw = mbar_wait(&sh.full[slot], par, W.err, 22);
    if (__syncthreads_or(!okw)) return;
    const int e = sh.act[c.a];
    const int cnt = sh.counts[e];
    const int off = sh.offsets[e];
    const uint8_t *st = smem + (size_t)slot * stage_bytes;
    for (int g0 = 0; g0 < cnt; g0 += kTX) {
      const int ng = min(kTX, cnt - g0);
      // staging key: the slots of this token group (gate_up needs their tokens' x)
      bool same = sh.st_key[kTX] == ng;
      for (int i = 0; i < ng; ++i) {
        const int want = c.down ? sh.perm[off + g0 + i] : sh.perm[off + g0 + i] / k;
        same = same && (sh.st_key[i] == want);
      }
      if (!same) {
        if (!c.down) {
          for (int i2 = threadIdx.x; i2 < ng * (d / 8); i2 += blockDim.x) {
            const int i = i2 / (d / 8), v = i2 % (d / 8);
            const int tok = sh.perm[off + g0 + i] / k;
            reinterpret_cast<uint4 *>(xs + (size_t)i * d)[v] =
                __ldcg(reinterpret_cast<const uint4 *>(W.x16 + (size_t)tok * d) + v);
          }
          for (int i2 = threadIdx.x; i2 < ng * nb; i2 += blockDim.x) {
            const int i = i2 / nb, b = i2 % nb;
            ss[i * nb + b] = __ldcg(W.xblk + (size_t)(sh.perm[off + g0 + i] / k) * nb + b);
          }
        } else {
          for (int it2 = wq; it2 < ng * nbf; it2 += nw) {
            const int i = it2 / nbf, cb = it2 % nbf;
            const float v = __ldcg(W.h + (size_t)sh.perm[off + g0 + i] * f + (size_t)cb * MOE_QK + lane);
            float m = fabsf(v);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            const BlockScale bs = block_scale_for_max(m);
            const __half hv = __float2half_rn(v * bs.scale);
            hs[(size_t)i * f + (size_t)cb * MOE_QK + gemv_pos(lane)] = __half_as_ushort(hv);
            float sm = __half2float(hv);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, o);
            if (lane == 0) hbk[i * nbf + cb] = make_float2(-8.f * sm, bs.inv);
          }
        }
        __syncthreads();
        if (threadIdx.x == 0) {
          for (int i = 0; i < ng; ++i) sh.st_key[i] = c.down ? sh.perm[off + g0 + i] : sh.perm[off + g0 + i] / k;
          sh.st_key[kTX] = ng;
        }
      }
      if (!c.down) {
        const int np = c.n * kUnit;
        if (wq < G) {
          if (aligned) {
            switch (ng) {
              case 1: gu_compute<1, true>(st, rb_g, nb, xs, ss, d, my_red_g); break;
              case 2: gu_compute<2, true>(st, rb_g, nb, xs, ss, d, my_red_g); break;
              case 3: gu_compute<3, true>(st, rb_g, nb, xs, ss, d, my_red_g); break;
              default: gu_compute<4, true>(st, rb_g, nb, xs, ss, d, my_red_g); break;
            }
          } else {
            switch (ng) {
              case 1: gu_compute<1, false>(st, rb_g, nb, xs, ss, d, my_red_g); break;
              case 2: gu_compute<2, false>(st, rb_g, nb, xs, ss, d, my_red_g); break;
              case 3: gu_compute<3, false>(st, rb_g, nb, xs, ss, d, my_red_g); break;
              default: gu_compute<4, false>(st, rb_g, nb, xs, ss, d, my_red_g); break;
            }
          }
        }
        __syncthreads();
        for (int i2 = threadIdx.x; i2 < kPairs * ng; i2 += blockDim.x) {
          const int pp = i2 % kPairs, i = i2 / kPairs;
          if (pp < np) {
            float g = 0.f, uu = 0.f;
            for (int q = 0; q < G; ++q) {
              const float *r = red + ((size_t)(q * kPairs + pp) * kTX + i) * 2;
              g += r[0];
              uu += r[1];
            }
            W.h[(size_t)sh.perm[off + g0 + i] * f + c.r0 + pp] = gelu_tanh_f(g) * uu;
          }
        }
        __syncthreads();
      } else {
        const int nr = c.n * kUnit;
        if (wq < 8 && (wq & 3) * 32 + lane < nr) {
          switch (ng) {
            case 1: dn_compute<1>(st, rb_d, nbf, hs, hbk, f, my_red_d); break;
            case 2: dn_compute<2>(st, rb_d, nbf, hs, hbk, f, my_red_d); break;
            case 3: dn_compute<3>(st, rb_d, nbf, hs, hbk, f, my_red_d); break;
            default: dn_compute<4>(st, rb_d, nbf, hs, hbk, f, my_red_d); break;
          }
        }
        __syncthreads();
        for (int i2 = threadIdx.x; i2 < kDnRows * ng; i2 += blockDim.x) {
          const int pp = i2 % kDnRows, i = i2 / kDnRows;
          if (pp < nr) {
            const float s = red[(size_t)i * kDnRows + pp] + red[(size_t)(kTX + i) * kDnRows + pp];
            W.ybuf[(size_t)sh.perm[off + g0 + i] * d + c.r0 + pp] = s;
          }
        }
        __syncthreads();
      }
    }
    u += c.n;
    if (threadIdx.x == 0 && u_issue < n_units) {   // every thread is done with stage `slot`
      issue(u_issue, slot);
      u_issue += seq.at(u_issue).n;
    }
  }
  if (!down_phase) {
    // this CTA had no down rows: it still takes part in the h barrier
    if (!grid_barrier(W.gbar, W.err, 21, sh.ok)) return;
  }
  // ---------------------------------------------------------------- phase 4: combine
  if (!grid_barrier(W.gbar, W.err, 23, sh.ok)) return;
  const int r0 = (int)((long long)d * blockIdx.x / gridDim.x), r1 = (int)((long long)d * (blockIdx.x + 1) / gridDim.x);
  const int nr = r1 - r0;
  for (int i2 = threadIdx.x; i2 < nr * T; i2 += blockDim.x) {
    const int t = i2 / nr, r = r0 + i2 % nr;
    float s = 0.f;
    for (int j = 0; j < k; ++j) {
      const int slotid = t * k + j;
      s += sh.w[slotid] * __ldg(expert_scale + sh.ids[slotid]) * __ldcg(W.ybuf + (size_t)slotid * d + r);
    }
    out[(size_t)t * d + r] = s;
  }
}

}  // namespace

// Dynamic shared memory of k_moe_decode for these shapes (0 if the shapes do not fit).
static size_t fused_smem(int d, int f, uint32_t &stage_bytes) {
  const int nb = d / MOE_QK, nbf = f / MOE_QK;
  const int G = (nb + kGran - 1) / kGran;
  const size_t sg = 2u * kPairs * (size_t)nb * MOE_QBYTES + 16u;
  const size_t sd = (size_t)kDnRows * nbf * MOE_QBYTES + 16u;
  stage_bytes = (uint32_t)(((sg > sd ? sg : sd) + 15u) & ~(size_t)15u);
  const size_t red_g = (size_t)G * 2 * kPairs * kTX * 2 * 4, red_d = (size_t)2 * kTX * kDnRows * 4;
  return (size_t)kFStages * stage_bytes + (size_t)kTX * d * 2 + (size_t)kTX * nb * 8 + (size_t)kTX * f * 2 +
         (size_t)kTX * nbf * 8 + (red_g > red_d ? red_g : red_d) + 128;
}

bool moe_fused_decode_supported(int T, int d, int f, int E, int k) {
  const int G = (d / MOE_QK + kGran - 1) / kGran;
  uint32_t sb;
  return T >= 1 && T <= kFMaxT && T * k <= kFMaxSlots && E <= MOE_MAX_E && G <= kFMaxWarps && f / MOE_QK <= 64 &&
         fused_smem(d, f, sb) + sizeof(FusedShared) <= 227 * 1024;
}

int moe_launch_fused_decode(const MoeLaunch &L, const MoeWork &W, const void *x, const float *router_w,
                            const float *router_scale, const uint8_t *gate_up_q4, const uint8_t *down_q4,
                            const float *expert_scale, int T, int d, int f, int E, int k, float *out,
                            int num_sms) {
  if (!moe_fused_decode_supported(T, d, f, E, k)) return -2;
  uint32_t stage_bytes;
  const size_t smem = fused_smem(d, f, stage_bytes);
  static size_t set = 0;
  if (smem > set) {
    if (cudaFuncSetAttribute(k_moe_decode, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return -1;
    set = smem;
  }
  const int G = (d / MOE_QK + kGran - 1) / kGran;
  const int warps = G > 8 ? G : 8;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(num_sms);
  cfg.blockDim = dim3(32 * warps);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = L.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  moe_prof_mark(L.stream, MOE_K_FUSED, true);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, k_moe_decode, static_cast<const __nv_bfloat16 *>(x), router_w,
                                           router_scale, gate_up_q4, down_q4, expert_scale, T, d, f, E, k, out,
                                           stage_bytes, W);
  if (e != cudaSuccess) return -1;
  moe_prof_mark(L.stream, MOE_K_FUSED, false);
  return 0;
}
