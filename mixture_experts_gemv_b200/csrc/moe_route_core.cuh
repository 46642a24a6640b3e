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

// The selection and softmax from the lane's keys key[i] = topk_key(logit, e) of experts
// e = lane + 32 i (0 past E).
template <int kMaxPer>
__device__ void warp_topk_softmax_keys64(uint64_t (&key)[kMaxPer], int k, float rscale, int32_t *ids, float *w) {
  const int lane = threadIdx.x & 31;
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

template <int kMaxPer>
__device__ void warp_topk_softmax_t(const float *lg, int E, int k, float rscale, int32_t *ids, float *w) {
  const int lane = threadIdx.x & 31;
  uint64_t key[kMaxPer];
#pragma unroll
  for (int i = 0; i < kMaxPer; ++i) {
    const int e = lane + 32 * i;
    key[i] = (e < E) ? topk_key(__ldcg(lg + e), e) : 0ull;
  }
  warp_topk_softmax_keys64<kMaxPer>(key, k, rscale, ids, w);
}

// Order-preserving 32-bit image of a logit (larger float -> larger unsigned; NaN ranks as
// -inf). Every value maps above 0, which marks a taken or absent entry.
__device__ __forceinline__ uint32_t logit_ord(float v) {
  uint32_t u = __float_as_uint(v);
  if (v != v) u = 0xff800000u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float logit_from_ord(uint32_t o) {
  return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}

// k <= 8: k rounds of a warp maximum, each as two 32-bit warp reductions (redux.sync): the
// largest logit, then, among the lanes holding it, the lowest expert index. A lane keeps its
// kMaxPer logits (experts lane + 32 i) and clears the one picked. Picks come out in the
// order (logit descending, index ascending), the same picks as a sort of the 64-bit keys.
// The selection and softmax of warp_top8_softmax_t from the lane's order keys o[i] of logits
// lane + 32 i (0 past E).
template <int kMaxPer>
__device__ void warp_top8_softmax_keys(uint32_t (&o)[kMaxPer], int k, float rscale, int32_t *ids, float *w) {
  const int lane = threadIdx.x & 31;
  uint32_t pick_o[8];
  int pick_e[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    pick_o[j] = 0u;
    pick_e[j] = 0;
    if (j < k) {
      uint32_t bo = o[0];
      int bi = 0;
#pragma unroll
      for (int i = 1; i < kMaxPer; ++i)
        if (o[i] > bo) { bo = o[i]; bi = i; }   // strict: the lower index among equal logits
      const uint32_t mo = __reduce_max_sync(0xffffffffu, bo);
      const uint32_t cand = (bo == mo) ? (uint32_t)(lane + 32 * bi) : 0xffffffffu;
      const uint32_t me = __reduce_min_sync(0xffffffffu, cand);
#pragma unroll
      for (int i = 0; i < kMaxPer; ++i)
        if (cand == me && i == bi) o[i] = 0u;   // taken
      pick_o[j] = mo;
      pick_e[j] = (int)me;
    }
  }
  // softmax over the selected logits, relative to the largest, summed in pick order
  const float l1 = logit_from_ord(pick_o[0]);
  float part = 0.f;
  float mine_v = 0.f;
  int mine_e = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j < k) {
      const float ev = expf(logit_from_ord(pick_o[j]) - l1);
      part += ev;
      if (j == lane) { mine_v = ev; mine_e = pick_e[j]; }
    }
  }
  if (lane < k) {
    ids[lane] = mine_e;
    w[lane] = mine_v * (rscale / part);
  }
  __syncwarp();
}

template <int kMaxPer>
__device__ void warp_top8_softmax_t(const float *lg, int E, int k, float rscale, int32_t *ids, float *w) {
  const int lane = threadIdx.x & 31;
  uint32_t o[kMaxPer];
#pragma unroll
  for (int i = 0; i < kMaxPer; ++i) {
    const int e = lane + 32 * i;
    o[i] = (e < E) ? logit_ord(__ldcg(lg + e)) : 0u;
  }
  warp_top8_softmax_keys<kMaxPer>(o, k, rscale, ids, w);
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

// Stable counting sort of S <= kMaxS slots by expert id in one warp: ranks from
// __match_any_sync in slot order, a warp scan of the counts, then placement.
constexpr int kSmallPermMax = 1024;
template <int kMaxS = kSmallPermMax>
__device__ void warp_permutation_small(const int32_t *ids, int S, int E, int32_t *counts, int32_t *offsets,
                                       int32_t *perm, int32_t *inv, int32_t *act, int32_t *n_act,
                                       int32_t *cnt /* smem [E] */) {
  const int lane = threadIdx.x & 31;
  const uint32_t lt = (1u << lane) - 1u;
  for (int e = lane; e < E; e += 32) cnt[e] = 0;
  __syncwarp();
  int rk[kMaxS / 32], idr[kMaxS / 32];
#pragma unroll
  for (int r = 0; r < kMaxS / 32; ++r) {
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
  for (int r = 0; r < kMaxS / 32; ++r) {
    const int s = r * 32 + lane;
    if (r * 32 < S && s < S) {
      const int pos = cnt[idr[r]] + rk[r];
      perm[pos] = s;
      inv[s] = pos;
    }
  }
}

// Stable counting sort of S <= 32 * kSlotWarps slots by expert id (E <= 32 * kExpWarps) by
// the calling CTA (every thread calls it; the block has at least max(kSlotWarps, kExpWarps)
// warps): warp w < kSlotWarps ranks its slots s = 32 w + lane among equal ids with
// __match_any_sync and records its per-expert counts; thread e < E sums the warps' counts
// of expert e in warp order (giving each warp's base inside the expert), and an exclusive
// scan over the experts gives the offsets and the active list; each slot's position is then
// its expert's offset + its warp's base + its rank in the warp.
// scratch: shared memory of kSlotWarps * E + 2 * kExpWarps ints.
template <int kSlotWarps, int kExpWarps>
__device__ void cta_permutation_small(const int32_t *ids, int S, int E, int32_t *counts, int32_t *offsets,
                                      int32_t *perm, int32_t *inv, int32_t *act, int32_t *n_act,
                                      int32_t *scratch) {
  const int tid = threadIdx.x, lane = tid & 31, wq = tid >> 5;
  int32_t *wc = scratch;                        // [kSlotWarps][E]: slots of expert e in warp w
  int32_t *tot = scratch + kSlotWarps * E;      // [kExpWarps] count totals, [kExpWarps] active totals
  for (int i = tid; i < kSlotWarps * E; i += blockDim.x) wc[i] = 0;
  __syncthreads();
  int id = -1, rank = 0;
  if (wq < kSlotWarps) {
    const int s = wq * 32 + lane;
    id = s < S ? ids[s] : -1 - lane;            // unique negative keys past the end
    const uint32_t peers = __match_any_sync(0xffffffffu, id);
    rank = __popc(peers & ((1u << lane) - 1u));
    if (s < S && lane == 31 - __clz(peers)) wc[wq * E + id] = __popc(peers);
  }
  __syncthreads();
  // thread e: count of expert e, and the bases of the slot warps inside it
  int c = 0, ic = 0, ia = 0;
  if (wq < kExpWarps) {
    if (tid < E) {
      for (int w = 0; w < kSlotWarps; ++w) {
        const int v = wc[w * E + tid];
        wc[w * E + tid] = c;
        c += v;
      }
    }
    ic = c;
    ia = c > 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {          // inclusive warp scans of count and active
      const int nc = __shfl_up_sync(0xffffffffu, ic, o), na = __shfl_up_sync(0xffffffffu, ia, o);
      if (lane >= o) { ic += nc; ia += na; }
    }
    if (lane == 31) { tot[wq] = ic; tot[kExpWarps + wq] = ia; }
  }
  __syncthreads();
  if (wq < kExpWarps) {
    int bc = 0, ba = 0, tc = 0, ta = 0;
    for (int w = 0; w < kExpWarps; ++w) {
      if (w < wq) { bc += tot[w]; ba += tot[kExpWarps + w]; }
      tc += tot[w];
      ta += tot[kExpWarps + w];
    }
    if (tid < E) {
      counts[tid] = c;
      offsets[tid] = bc + ic - c;
      if (c > 0) act[ba + ia - 1] = tid;
    }
    if (tid == 0) {
      offsets[E] = tc;
      *n_act = ta;
    }
  }
  __syncthreads();
  if (wq < kSlotWarps) {
    const int s = wq * 32 + lane;
    if (s < S) {
      const int pos = offsets[id] + wc[wq * E + id] + rank;
      perm[pos] = s;
      inv[s] = pos;
    }
  }
  __syncthreads();
}

}  // namespace
