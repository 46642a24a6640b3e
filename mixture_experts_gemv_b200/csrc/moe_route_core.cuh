// moe_route_core.cuh -- device building blocks of routing shared by the routing kernels
// (moe_route.cu) and the fused decode kernel (moe_decode.cu): activation preparation for
// the GEMV, warp-level top-k + softmax over the selected logits, and the one-warp stable
// permutation for small slot counts.
//
// Definition (page "Gemma 4 26B-A4B it QAT Q4_0 ... NInfer v3 artifact", "What is inside":
// FP32 router and router scale): the k largest logits are selected, equal logits going to
// the lower expert index; w_j = router_scale * exp(l_j - l_1) / sum_m exp(l_m - l_1) over the
// selected ones. The permutation is the stable counting sort of slots s = t*k + j by id.
#pragma once

#include "moe_common.cuh"

namespace {

// ---------------------------------------------------------------- x preparation
//
// For the Q4_0 GEMV: each 32-wide block of x becomes block-scaled int16 (moe_common.cuh),
// stored in the GEMV's word order, with the block's ActBlk. One (token, block) per thread,
// grid-stride.
__device__ void prep_x_range(const __nv_bfloat16 *x, int16_t *xq, ActBlk *xblk, int T, int d, int tid,
                             int nthreads) {
  const int nb = d / MOE_QK;
  for (int it = tid; it < T * nb; it += nthreads) {
    const int t = it / nb, b = it % nb;
    const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)t * d + (size_t)b * MOE_QK);
    float v[MOE_QK];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 q = __ldg(src + i);
      const uint32_t qq[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        v[8 * i + 2 * h] = __uint_as_float(qq[h] << 16);
        v[8 * i + 2 * h + 1] = __uint_as_float(qq[h] & 0xffff0000u);
      }
    }
    float m = 0.f;
    bool finite = true;
#pragma unroll
    for (int i = 0; i < MOE_QK; ++i) {
      m = fmaxf(m, fabsf(v[i]));
      finite = finite && isfinite(v[i]);
    }
    const BlockScale bs = block_scale_for_max(m);
    // output position p = 8 i + r holds element 4 i + r (r < 4) or 16 + 4 i + r - 4
    uint32_t pk[MOE_QK / 2];
    int s = 0;
#pragma unroll
    for (int p = 0; p < MOE_QK; ++p) {
      const int i = p >> 3, r = p & 7;
      const int e = (r < 4) ? (4 * i + r) : (16 + 4 * i + r - 4);
      const int a = act_to_i16(v[e], bs.scale);
      s += a;
      const uint32_t bits = (uint32_t)a & 0xffffu;
      if (p & 1) pk[p >> 1] |= bits << 16; else pk[p >> 1] = bits;
    }
    uint4 *dst = reinterpret_cast<uint4 *>(xq + (size_t)t * d + (size_t)b * MOE_QK);
#pragma unroll
    for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
    xblk[(size_t)t * nb + b] = ActBlk{-8 * s, finite ? bs.inv : __int_as_float(0x7fffffff)};
  }
}

// ---------------------------------------------------------------- top-k + softmax

// Warp-level selection for one token. Each logit becomes a 64-bit key (order-preserving
// float bits << 32 | ~index), so one maximum finds the largest logit and, among equal ones,
// the lower expert index; NaN logits rank as -inf. k rounds of a warp maximum pick the
// experts in order; lane 0 records each pick (the selected logits are parked in w[] until
// the softmax overwrites them).
__device__ __forceinline__ uint64_t topk_key(float v, int e) {
  uint32_t u = __float_as_uint(v);
  if (v != v) u = 0xff800000u;                       // NaN -> -inf
  const uint32_t ord = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((uint64_t)ord << 32) | (uint32_t)(0xffffffffu - (uint32_t)e);
}
__device__ __forceinline__ float topk_key_value(uint64_t key) {
  const uint32_t ord = (uint32_t)(key >> 32);
  const uint32_t u = (ord & 0x80000000u) ? (ord & 0x7fffffffu) : ~ord;
  return __uint_as_float(u);
}

template <int kMaxPer>
__device__ void warp_topk_softmax_t(const float *lg, int E, int k, float rscale, int32_t *ids, float *w) {
  const int lane = threadIdx.x & 31;
  uint64_t key[kMaxPer];
#pragma unroll
  for (int i = 0; i < kMaxPer; ++i) {
    const int e = lane + 32 * i;
    key[i] = (e < E) ? topk_key(__ldcg(lg + e), e) : 0ull;
  }
  for (int j = 0; j < k; ++j) {
    uint64_t best = key[0];
#pragma unroll
    for (int i = 1; i < kMaxPer; ++i) best = key[i] > best ? key[i] : best;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const uint64_t other = __shfl_xor_sync(0xffffffffu, best, o);
      best = other > best ? other : best;
    }
    const int e = (int)(0xffffffffu - (uint32_t)best);
    if ((e & 31) == lane) {
#pragma unroll
      for (int i = 0; i < kMaxPer; ++i)
        if (i == (e >> 5)) key[i] = 0ull;   // taken
    }
    if (lane == 0) {
      ids[j] = e;
      w[j] = topk_key_value(best);
    }
  }
  __syncwarp();
  // softmax over the selected logits, relative to the largest (j = 0)
  const float l1 = w[0];
  float part = 0.f;
  for (int j = lane; j < k; j += 32) part += expf(w[j] - l1);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  const float inv = rscale / part;
  __syncwarp();
  for (int j = lane; j < k; j += 32) w[j] = expf(w[j] - l1) * inv;
  __syncwarp();
}

// k <= 8: every lane sorts its keys, then five butterfly steps merge sorted top-8 lists
// (exchange with the partner lane, keep the 8 largest of the 16 by a bitonic merge), so
// every lane ends with the token's sorted top 8 after 5 shuffle rounds instead of k
// dependent warp maxima.
template <int kMaxPer>
__device__ void warp_top8_softmax_t(const float *lg, int E, int k, float rscale, int32_t *ids, float *w) {
  const int lane = threadIdx.x & 31;
  uint64_t t[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) t[i] = 0ull;
  // insert this lane's keys into a sorted (descending) list of 8
#pragma unroll
  for (int i = 0; i < kMaxPer; ++i) {
    const int e = lane + 32 * i;
    uint64_t v = (e < E) ? topk_key(__ldcg(lg + e), e) : 0ull;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint64_t hi = t[j] > v ? t[j] : v, lo = t[j] > v ? v : t[j];
      t[j] = hi;
      v = lo;
    }
  }
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint64_t u[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) u[j] = __shfl_xor_sync(0xffffffffu, t[j], o);
    // top 8 of two descending lists: pairwise max against the reversed partner list is a
    // bitonic sequence holding the 8 largest; sort it descending
#pragma unroll
    for (int j = 0; j < 8; ++j) t[j] = t[j] > u[7 - j] ? t[j] : u[7 - j];
#pragma unroll
    for (int s2 = 4; s2 > 0; s2 >>= 1) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if ((j & s2) == 0) {
          const uint64_t a2 = t[j], b2 = t[j + s2];
          t[j] = a2 > b2 ? a2 : b2;
          t[j + s2] = a2 > b2 ? b2 : a2;
        }
      }
    }
  }
  // every lane holds the sorted top 8; lanes j < k publish pick j
  const float l1 = topk_key_value(t[0]);
  float part = 0.f;
  float mine_v = 0.f;
  int mine_e = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j < k) {
      const float v = topk_key_value(t[j]);
      const float ev = expf(v - l1);
      part += ev;
      if (j == lane) { mine_v = ev; mine_e = (int)(0xffffffffu - (uint32_t)t[j]); }
    }
  }
  if (lane < k) {
    ids[lane] = mine_e;
    w[lane] = mine_v * (rscale / part);
  }
  __syncwarp();
}

// E <= 32 * kMaxPer logits per lane-strided register file.
// kMaxE: the largest E the caller supports (the register file of the selection grows with it).
template <int kMaxE = MOE_MAX_E>
__device__ __forceinline__ void warp_topk_softmax(const float *lg, int E, int k, float rscale, int32_t *ids,
                                                  float *w) {
  if (k <= 8 && E <= 128) {
    warp_top8_softmax_t<4>(lg, E, k, rscale, ids, w);
    return;
  }
  if (k <= 8 && E <= 256) {
    warp_top8_softmax_t<8>(lg, E, k, rscale, ids, w);
    return;
  }
  if (E <= 128) {
    warp_topk_softmax_t<4>(lg, E, k, rscale, ids, w);
    return;
  }
  if constexpr (kMaxE > 128) {
    if (E <= 256) {
      warp_topk_softmax_t<8>(lg, E, k, rscale, ids, w);
      return;
    }
  }
  if constexpr (kMaxE > 256) warp_topk_softmax_t<MOE_MAX_E / 32>(lg, E, k, rscale, ids, w);
}

// Stable counting sort of S <= 1024 slots by expert id in one warp: ranks from
// __match_any_sync in slot order, a warp scan of the counts, then placement.
constexpr int kSmallPermMax = 1024;
__device__ void warp_permutation_small(const int32_t *ids, int S, int E, int32_t *counts, int32_t *offsets,
                                       int32_t *perm, int32_t *inv, int32_t *act, int32_t *n_act,
                                       int32_t *cnt /* smem [E] */) {
  const int lane = threadIdx.x & 31;
  const uint32_t lt = (1u << lane) - 1u;
  for (int e = lane; e < E; e += 32) cnt[e] = 0;
  __syncwarp();
  int rk[kSmallPermMax / 32], idr[kSmallPermMax / 32];
#pragma unroll
  for (int r = 0; r < kSmallPermMax / 32; ++r) {
    const int s = r * 32 + lane;
    if (r * 32 < S) {
      const int id = (s < S) ? ids[s] : -1 - lane;   // written earlier by this CTA
      const uint32_t peers = __match_any_sync(0xffffffffu, id);
      rk[r] = (s < S) ? cnt[id] + __popc(peers & lt) : 0;
      idr[r] = id;
      __syncwarp();
      if (s < S && lane == 31 - __clz(peers)) cnt[id] += __popc(peers);
      __syncwarp();
    }
  }
  // exclusive scans of counts and of (count > 0), lane-chunked
  const int per = (E + 31) / 32;
  const int e0 = lane * per, e1 = min(E, e0 + per);
  int c_sum = 0, a_sum = 0;
  for (int e = e0; e < e1; ++e) { c_sum += cnt[e]; a_sum += cnt[e] > 0; }
  int c_inc = c_sum, a_inc = a_sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int nc = __shfl_up_sync(0xffffffffu, c_inc, o), na = __shfl_up_sync(0xffffffffu, a_inc, o);
    if (lane >= o) { c_inc += nc; a_inc += na; }
  }
  int c_run = c_inc - c_sum, a_run = a_inc - a_sum;
  const int c_tot = __shfl_sync(0xffffffffu, c_inc, 31), a_tot = __shfl_sync(0xffffffffu, a_inc, 31);
  __syncwarp();
  for (int e = e0; e < e1; ++e) {
    const int c = cnt[e];
    counts[e] = c;
    offsets[e] = c_run;
    if (c > 0) act[a_run++] = e;
    cnt[e] = c_run;   // becomes the expert's base
    c_run += c;
  }
  if (lane == 0) { offsets[E] = c_tot; *n_act = a_tot; }
  __syncwarp();
#pragma unroll
  for (int r = 0; r < kSmallPermMax / 32; ++r) {
    const int s = r * 32 + lane;
    if (r * 32 < S && s < S) {
      const int pos = cnt[idr[r]] + rk[r];
      perm[pos] = s;
      inv[s] = pos;
    }
  }
}

}  // namespace
