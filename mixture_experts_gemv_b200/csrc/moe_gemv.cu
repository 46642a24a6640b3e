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
// Arithmetic (moe_gemv_core.cuh): int16 block-scaled activations, dp2a integer dot
// products of codes and activations, exact per block; one FP32 rounding per block and row.

#include "moe_gemv_core.cuh"

namespace {

template <bool ALIGNED>
__global__ void __launch_bounds__(kMaxGran * 32, 1)
k_gateup_gemv(const uint8_t *__restrict__ gate_up_q4, int d, int f, int k, int nstages, MoeWork W) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  __shared__ RingCtl ring;
  __shared__ int st_key[2];

  const int nb = d / MOE_QK;
  const int G = (nb + kGran - 1) / kGran;
  const uint32_t rb = (uint32_t)nb * MOE_QBYTES;
  const uint32_t stage_bytes = (2u * kPairs * rb + 16u + 15u) & ~15u;
  uint8_t *smem = align128(smem_raw);
  uint16_t *xs = reinterpret_cast<uint16_t *>(smem + (size_t)nstages * stage_bytes);   // [kTX][d] int16
  ActBlk *ss = reinterpret_cast<ActBlk *>(xs + (size_t)kTX * d);                         // [kTX][nb]
  float *red = reinterpret_cast<float *>(ss + (size_t)kTX * nb);                         // [G*2][kPairs][kTX][2]
  const int upe = f / kUnit;
  const int n_act = *W.n_act;
  int u0, u1;
  my_units(n_act * upe, u0, u1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < nstages; ++s) mbar_init(&ring.full[s], 1);
    fence_mbar_init();
    st_key[0] = -1;
    st_key[1] = -1;
  }
  __syncthreads();

  const uint64_t pol = l2_evict_first_policy();   // expert weights are read once per call
  auto issue = [&](int u, int slot) {
    const GuChunk c = gu_chunk(u, u1, upe);
    const int e = W.act[c.a];
    const uint8_t *base = gate_up_q4 + (size_t)e * 2 * f * rb;
    uint8_t *dst = smem + (size_t)slot * stage_bytes;
    const uint32_t bytes = (uint32_t)c.np * rb;
    mbar_arrive_expect_tx(&ring.full[slot], 2u * bytes);
    bulk_g2s_hint(dst, base + (size_t)c.c0 * rb, bytes, &ring.full[slot], pol);
    bulk_g2s_hint(dst + kPairs * rb, base + (size_t)(f + c.c0) * rb, bytes, &ring.full[slot], pol);
  };
  int u_issue = u0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < nstages && u_issue < u1; ++s) {
      issue(u_issue, s);
      u_issue += gu_chunk(u_issue, u1, upe).np / kUnit;
    }
  }

  const int lane = threadIdx.x & 31, wq = threadIdx.x >> 5;
  float *my_red = red + ((size_t)(wq * kPairs + (lane >> 1)) * kTX) * 2;
  int it = 0;
  for (int u = u0; u < u1; ++it) {
    const GuChunk c = gu_chunk(u, u1, upe);
    const int slot = it % nstages;
    const uint32_t par = (uint32_t)(it / nstages) & 1u;
    const bool ok = mbar_wait(&ring.full[slot], par, W.err, 1, W.wait_ns);
    if (__syncthreads_or(!ok)) return;

    const int e = W.act[c.a];
    const int cnt = W.counts[e];
    const int off = W.offsets[e];
    const uint8_t *st = smem + (size_t)slot * stage_bytes;
    for (int g0 = 0; g0 < cnt; g0 += kTX) {
      const int ng = min(kTX, cnt - g0);
      if (st_key[0] != e || st_key[1] != g0) {
        // stage the activations of this token group (prepared x and block sums)
        for (int i2 = threadIdx.x; i2 < ng * (d / 8); i2 += blockDim.x) {
          const int i = i2 / (d / 8), v = i2 % (d / 8);
          const int tok = W.perm[off + g0 + i] / k;
          reinterpret_cast<uint4 *>(xs + (size_t)i * d)[v] =
              __ldcg(reinterpret_cast<const uint4 *>(W.xq + (size_t)tok * d) + v);
        }
        for (int i2 = threadIdx.x; i2 < ng * nb; i2 += blockDim.x) {
          const int i = i2 / nb, b = i2 % nb;
          const int2 v = __ldcg(reinterpret_cast<const int2 *>(W.xblk) + (size_t)(W.perm[off + g0 + i] / k) * nb + b);
          ss[i * nb + b] = ActBlk{v.x, __int_as_float(v.y)};
        }
        __syncthreads();
        if (threadIdx.x == 0) { st_key[0] = e; st_key[1] = g0; }
      }
      if (wq < G) {
        switch (ng) {
          case 1: gu_compute<1, ALIGNED>(st, rb, nb, xs, ss, d, my_red); break;
          case 2: gu_compute<2, ALIGNED>(st, rb, nb, xs, ss, d, my_red); break;
          case 3: gu_compute<3, ALIGNED>(st, rb, nb, xs, ss, d, my_red); break;
          default: gu_compute<4, ALIGNED>(st, rb, nb, xs, ss, d, my_red); break;
        }
      }
      __syncthreads();
      for (int i2 = threadIdx.x; i2 < kPairs * ng; i2 += blockDim.x) {
        const int pp = i2 % kPairs, i = i2 / kPairs;
        if (pp < c.np) {
          float g = 0.f, uu = 0.f;
          for (int q = 0; q < G; ++q) {
            const float *r = red + ((size_t)(q * kPairs + pp) * kTX + i) * 2;
            g += r[0];
            uu += r[1];
          }
          const float hv = gelu_tanh_f(g) * uu;
          W.h[(size_t)W.perm[off + g0 + i] * f + c.c0 + pp] = hv;
        }
      }
      __syncthreads();
    }
    u += c.np / kUnit;
    if (threadIdx.x == 0 && u_issue < u1) {   // stage `slot` has been read by every thread
      issue(u_issue, slot);
      u_issue += gu_chunk(u_issue, u1, upe).np / kUnit;
    }
  }
}

// ---------------------------------------------------------------- down + combine
//
// CTA = 8 warps over the work items (32-row group, part of the row's blocks) of a chunk, the
// parts as in the fused decode kernel (same block split, parts summed in order, so both paths
// give the same bits); lane = row. All lanes of a warp read the same hidden values
// (broadcast).

__global__ void __launch_bounds__(kDnThreads, 1)
k_down_gemv_combine(const uint8_t *__restrict__ down_q4, const float *__restrict__ expert_scale, int T,
                    int d, int f, int k, int nstages, float *__restrict__ out, MoeWork W, int accumulate) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  __shared__ RingCtl ring;
  __shared__ int done_units[kDnRows / kUnit];
  __shared__ int n_done;
  __shared__ int st_key[2];

  const int nbf = f / MOE_QK;
  const uint32_t rb = (uint32_t)nbf * MOE_QBYTES;
  const uint32_t stage_bytes = ((uint32_t)kDnRows * rb + 16u + 15u) & ~15u;
  uint8_t *smem = align128(smem_raw);
  uint16_t *hs = reinterpret_cast<uint16_t *>(smem + (size_t)nstages * stage_bytes);   // [kTX][f] int16 h
  ActBlk *hblk = reinterpret_cast<ActBlk *>(hs + (size_t)kTX * f);                      // [kTX][nbf]
  float *red = reinterpret_cast<float *>(hblk + (size_t)kTX * nbf);                     // [parts][kTX][kDnRows]
  const int upe = d / kUnit;
  const int n_act = *W.n_act;
  int u0, u1;
  my_units(n_act * upe, u0, u1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < nstages; ++s) mbar_init(&ring.full[s], 1);
    fence_mbar_init();
    st_key[0] = -1;
    st_key[1] = -1;
  }
  __syncthreads();

  const uint64_t pol = l2_evict_first_policy();
  auto issue = [&](int u, int slot) {
    const DnChunk c = dn_chunk(u, u1, upe);
    const int e = W.act[c.a];
    const uint8_t *src = down_q4 + (size_t)e * d * rb + (size_t)c.r0 * rb;
    const uint32_t bytes = (uint32_t)c.nr * rb;
    mbar_arrive_expect_tx(&ring.full[slot], bytes);
    bulk_g2s_hint(smem + (size_t)slot * stage_bytes, src, bytes, &ring.full[slot], pol);
  };
  int u_issue = u0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < nstages && u_issue < u1; ++s) {
      issue(u_issue, s);
      u_issue += dn_chunk(u_issue, u1, upe).nr / kUnit;
    }
  }

  const int lane = threadIdx.x & 31, wq = threadIdx.x >> 5;
  int it = 0;
  for (int u = u0; u < u1; ++it) {
    const DnChunk c = dn_chunk(u, u1, upe);
    const int slot = it % nstages;
    const uint32_t par = (uint32_t)(it / nstages) & 1u;
    const bool ok = mbar_wait(&ring.full[slot], par, W.err, 2, W.wait_ns);
    if (__syncthreads_or(!ok)) return;

    const int e = W.act[c.a];
    const int cnt = W.counts[e];
    const int off = W.offsets[e];
    const uint8_t *st = smem + (size_t)slot * stage_bytes;

    for (int g0 = 0; g0 < cnt; g0 += kTX) {
      const int ng = min(kTX, cnt - g0);
      if (st_key[0] != e || st_key[1] != g0) {
        // h of these slots -> block-scaled int16 in the word order; one warp per (slot,
        // block): lane = element
        for (int it2 = wq; it2 < ng * nbf; it2 += kDnThreads / 32) {
          const int i = it2 / nbf, cb = it2 % nbf;
          const float v = __ldcg(W.h + (size_t)W.perm[off + g0 + i] * f + (size_t)cb * MOE_QK + lane);
          float m = fabsf(v);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
          const bool finite = __all_sync(0xffffffffu, isfinite(v));
          const BlockScale bs = block_scale_for_max(m);
          const int a = act_to_i16(v, bs.scale);
          hs[(size_t)i * f + (size_t)cb * MOE_QK + gemv_pos(lane)] = (uint16_t)(a & 0xffff);
          int sm = a;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, o);
          if (lane == 0) hblk[i * nbf + cb] = ActBlk{-8 * sm, finite ? bs.inv : __int_as_float(0x7fffffff)};
        }
        __syncthreads();
        if (threadIdx.x == 0) { st_key[0] = e; st_key[1] = g0; }
      }
      switch (ng) {
        case 1: dn_compute<1>(st, rb, nbf, c.nr, hs, hblk, f, red); break;
        case 2: dn_compute<2>(st, rb, nbf, c.nr, hs, hblk, f, red); break;
        case 3: dn_compute<3>(st, rb, nbf, c.nr, hs, hblk, f, red); break;
        default: dn_compute<4>(st, rb, nbf, c.nr, hs, hblk, f, red); break;
      }
      __syncthreads();
      for (int i2 = threadIdx.x; i2 < kDnRows * ng; i2 += kDnThreads) {
        const int pp = i2 % kDnRows, i = i2 / kDnRows;
        if (pp < c.nr) {
          float s = 0.f;   // the parts in order
          for (int pt = 0; pt < MOE_DN_PARTS; ++pt) s += red[((size_t)pt * kTX + i) * kDnRows + pp];
          W.ybuf[(size_t)W.perm[off + g0 + i] * d + c.r0 + pp] = s;
        }
      }
      __syncthreads();
    }
    // this chunk's rows of expert e are final: count arrivals per 8-row unit; the CTA
    // bringing a unit to n_act combines it (sum over j in order, deterministic)
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
      for (int i2 = threadIdx.x; i2 < n_done * kUnit * T; i2 += kDnThreads) {
        const int un = i2 / (kUnit * T), rem = i2 % (kUnit * T);
        const int t = rem / kUnit, r = done_units[un] * kUnit + rem % kUnit;
        float s = 0.f;
        for (int j = 0; j < k; ++j) {
          const int slotid = t * k + j;
          s += W.w[slotid] * expert_scale[W.ids[slotid]] * __ldcg(W.ybuf + (size_t)slotid * d + r);
        }
        out[(size_t)t * d + r] = accumulate ? out[(size_t)t * d + r] + s : s;
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
    const long long prow = (long long)toff[e] * MOE_GEMM_TILE_ROWS + (inv[s] - offsets[e]);
    h[i] = __bfloat162float(hb[prow * f + c]);
  }
}

}  // namespace

static int launch_err() { return cudaGetLastError() == cudaSuccess ? 0 : -1; }

int moe_launch_gemv_experts(const MoeLaunch &L, const MoeWork &W, const uint8_t *gate_up_q4,
                            const uint8_t *down_q4, const float *expert_scale, int T, int d, int f,
                            int E, int k, float *out, int num_sms) {
  (void)E;
  const int nb = d / MOE_QK, nbf = f / MOE_QK;
  const int G = (nb + kGran - 1) / kGran;
  if (G > kMaxGran || nbf > 64) return -2;
  const size_t gu_stage = (2u * kPairs * (size_t)nb * MOE_QBYTES + 16u + 15u) & ~(size_t)15u;
  const size_t gu_extra = (size_t)kTX * d * 2 + (size_t)kTX * nb * 8 + (size_t)G * 2 * kPairs * kTX * 2 * 4 + 128;
  const size_t dn_stage = ((size_t)kDnRows * nbf * MOE_QBYTES + 16u + 15u) & ~(size_t)15u;
  const size_t dn_extra =
      (size_t)kTX * f * 2 + (size_t)kTX * nbf * 8 + (size_t)MOE_DN_PARTS * kTX * kDnRows * 4 + 128;
  int gu_st = (int)((kSmemBudget - (long long)gu_extra) / (long long)gu_stage);
  int dn_st = (int)((kSmemBudget - (long long)dn_extra) / (long long)dn_stage);
  if (gu_st > kGuStagesMax) gu_st = kGuStagesMax;
  if (dn_st > kDnStagesMax) dn_st = kDnStagesMax;
  if (gu_st < 2 || dn_st < 2) return -2;
  const size_t gu_smem = (size_t)gu_st * gu_stage + gu_extra, dn_smem = (size_t)dn_st * dn_stage + dn_extra;
  const bool aligned = (nb % kGran) == 0;
  static unsigned long long smem_ok[3] = {0ull, 0ull, 0ull};   // per device, per kernel
  auto gu_kernel = aligned ? k_gateup_gemv<true> : k_gateup_gemv<false>;
  if (!moe_allow_dyn_smem(reinterpret_cast<const void *>(gu_kernel), &smem_ok[aligned]) ||
      !moe_allow_dyn_smem(reinterpret_cast<const void *>(k_down_gemv_combine), &smem_ok[2]))
    return -1;
  moe_prof_mark(L.stream, MOE_K_GATEUP, true);
  gu_kernel<<<num_sms, 32 * G, gu_smem, L.stream>>>(gate_up_q4, d, f, k, gu_st, W);
  if (launch_err()) return -1;
  moe_prof_count(1);
  moe_prof_mark(L.stream, MOE_K_GATEUP, false);
  moe_prof_mark(L.stream, MOE_K_DOWN, true);
  k_down_gemv_combine<<<num_sms, kDnThreads, dn_smem, L.stream>>>(down_q4, expert_scale, T, d, f, k, dn_st, out, W,
                                                                      L.accumulate ? 1 : 0);
  if (launch_err()) return -1;
  moe_prof_count(1);
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
