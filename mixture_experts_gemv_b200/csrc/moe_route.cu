// moe_route.cu -- router logits, top-k + softmax over the selected logits, and the
// per-expert histogram / prefix sum / stable token permutation.
//
// Definition (page "Gemma 4 26B-A4B it QAT Q4_0 ... NInfer v3 artifact", "What is inside":
// FP32 router and router scale, 128 routed experts): l[t,e] = sum_i W_r[e,i] x[t,i] in FP32;
// the k largest logits are selected, equal logits going to the lower expert index;
// w[t,j] = router_scale * exp(l_j - l_1) / sum_m exp(l_m - l_1) over the selected ones.
// The permutation is the stable counting sort of slots s = t*k + j by expert id.
#include "moe_route_core.cuh"

namespace {

constexpr int kRouteThreads = 512;             // 16 warps
constexpr int kRouteWarps = kRouteThreads / 32;
constexpr int kDecodeMaxT = 16;

// ---------------------------------------------------------------- permutation (one CTA)
//
// Stable counting sort of S slots by expert id, all in one CTA of kRouteThreads threads.
// Warp w owns the contiguous slot range [w*S/NW, (w+1)*S/NW). Pass 1 counts, per warp and
// expert, using __match_any_sync to rank equal ids inside each 32-slot round; the counts
// are turned into per-(warp, expert) output bases; pass 2 repeats the ranking and places
// each slot. Also writes the active-expert list and, if tiles != nullptr, the list of
// (expert, first row) tiles of tile_m rows for the grouped GEMM.
struct PermSmem {
  int32_t cnt[kRouteWarps][MOE_MAX_E];
  int32_t tot[MOE_MAX_E];
  int32_t scan_tmp[kRouteWarps * 3];
};

__device__ void block_exclusive_scan3(int32_t a, int32_t b, int32_t c, int32_t &ea, int32_t &eb,
                                      int32_t &ec, int32_t *tmp, int32_t &ta, int32_t &tb, int32_t &tc) {
  // exclusive scan of three values over the CTA (thread order), plus totals
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int32_t ia = a, ib = b, ic = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t na = __shfl_up_sync(0xffffffffu, ia, o);
    const int32_t nb = __shfl_up_sync(0xffffffffu, ib, o);
    const int32_t nc = __shfl_up_sync(0xffffffffu, ic, o);
    if (lane >= o) { ia += na; ib += nb; ic += nc; }
  }
  if (lane == 31) { tmp[wid] = ia; tmp[kRouteWarps + wid] = ib; tmp[2 * kRouteWarps + wid] = ic; }
  __syncthreads();
  int32_t pa = 0, pb = 0, pc = 0;
  ta = tb = tc = 0;
  for (int i = 0; i < kRouteWarps; ++i) {
    const int32_t xa = tmp[i], xb = tmp[kRouteWarps + i], xc = tmp[2 * kRouteWarps + i];
    if (i < wid) { pa += xa; pb += xb; pc += xc; }
    ta += xa; tb += xb; tc += xc;
  }
  ea = pa + ia - a;
  eb = pb + ib - b;
  ec = pc + ic - c;
  __syncthreads();
}

__device__ void block_permutation(const int32_t *ids, int S, int E, int32_t *counts, int32_t *offsets,
                                  int32_t *perm, int32_t *inv, int32_t *act, int32_t *n_act,
                                  int32_t *tiles, int32_t *n_tiles, int32_t *toffs, int tile_m, PermSmem &sm) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < kRouteWarps * MOE_MAX_E; i += blockDim.x) (&sm.cnt[0][0])[i] = 0;
  __syncthreads();
  const int s0 = (int)((long long)S * wid / kRouteWarps);
  const int s1 = (int)((long long)S * (wid + 1) / kRouteWarps);
  const uint32_t lt = (1u << lane) - 1u;
  // pass 1: per-warp counts
  for (int base = s0; base < s1; base += 32) {
    const int s = base + lane;
    const int id = (s < s1) ? ids[s] : -1 - lane;   // unique negative keys for the tail
    const uint32_t peers = __match_any_sync(0xffffffffu, id);
    const int leader = 31 - __clz(peers);
    if (s < s1 && lane == leader) sm.cnt[wid][id] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // per-expert totals, then offsets, active list and tile counts by a CTA scan
  int32_t cnt = 0, a = 0, nt = 0;
  const int e = threadIdx.x;   // requires E <= blockDim.x
  if (e < E) {
    for (int w = 0; w < kRouteWarps; ++w) cnt += sm.cnt[w][e];
    a = cnt > 0;
    nt = tiles ? (cnt + tile_m - 1) / tile_m : 0;
  }
  int32_t off, aoff, toff, tot, atot, ttot;
  block_exclusive_scan3(cnt, a, nt, off, aoff, toff, sm.scan_tmp, tot, atot, ttot);
  if (e < E) {
    counts[e] = cnt;
    offsets[e] = off;
    if (a) act[aoff] = e;
    int32_t run = off;   // per-warp output bases for this expert
    for (int w = 0; w < kRouteWarps; ++w) {
      const int32_t c = sm.cnt[w][e];
      sm.cnt[w][e] = run;
      run += c;
    }
    if (tiles) {
      toffs[e] = toff;
      for (int i = 0; i < nt; ++i) {
        tiles[2 * (toff + i)] = e;
        tiles[2 * (toff + i) + 1] = i * tile_m;
      }
    }
  }
  if (threadIdx.x == 0) {
    offsets[E] = tot;
    *n_act = atot;
    if (n_tiles) *n_tiles = ttot;
  }
  __syncthreads();
  // pass 2: placement
  for (int base = s0; base < s1; base += 32) {
    const int s = base + lane;
    const int id = (s < s1) ? ids[s] : -1 - lane;
    const uint32_t peers = __match_any_sync(0xffffffffu, id);
    const int leader = 31 - __clz(peers);
    if (s < s1) {
      const int pos = sm.cnt[wid][id] + __popc(peers & lt);
      perm[pos] = s;
      inv[s] = pos;
    }
    __syncwarp();
    if (s < s1 && lane == leader) sm.cnt[wid][id] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
}

// ---------------------------------------------------------------- decode routing kernel
//
// T <= 16. CTA b handles epc = kRouteWarps / P experts, each cut in the P slices of d that the
// fused decode kernel uses (moe_common.cuh): warp (expert, slice) accumulates lane-strided
// float4 chunks of W_r against every token, reduces across the warp by a fixed xor tree, and
// the slices are summed in order, so the logits are the fused kernel's bit for bit. The last
// CTA to finish (arrival counter) runs top-k + softmax for all tokens and the permutation.
struct RouteDecodeSmem {
  float part[kRouteWarps][kDecodeMaxT];
  union {
    PermSmem perm;
    int32_t cnt[MOE_MAX_E];
  } u;
  int last;
};

__global__ void __launch_bounds__(kRouteThreads, 1)
k_route_decode(const __nv_bfloat16 *__restrict__ x, const float *__restrict__ router_w,
               const float *__restrict__ router_scale, int T, int d, int E, int k, MoeWork W) {
  __shared__ RouteDecodeSmem sm;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int P = moe_decode_router_parts(d), epc = kRouteWarps / P;
  const int el = wid / P, part = wid % P;
  const int e = blockIdx.x * epc + el;
  const int seg = (d / 4) / P * 4;   // float4-aligned slice; the last slice takes the tail
  const int i0 = part * seg, i1 = (part == P - 1) ? d : i0 + seg;
  if (el < epc && e < E) {
    float acc[kDecodeMaxT];
#pragma unroll
    for (int t = 0; t < kDecodeMaxT; ++t) acc[t] = 0.f;
    const float *wr = router_w + (size_t)e * d;
    for (int i = i0 + lane * 4; i + 3 < i1; i += 128) {
      const float4 wv = __ldg(reinterpret_cast<const float4 *>(wr + i));
#pragma unroll
      for (int t = 0; t < kDecodeMaxT; ++t) {
        if (t < T) {
          const uint2 xv = __ldg(reinterpret_cast<const uint2 *>(x + (size_t)t * d + i));
          const float x0 = __uint_as_float(xv.x << 16), x1 = __uint_as_float(xv.x & 0xffff0000u);
          const float x2 = __uint_as_float(xv.y << 16), x3 = __uint_as_float(xv.y & 0xffff0000u);
          float a = acc[t];
          a = fmaf(wv.x, x0, a);
          a = fmaf(wv.y, x1, a);
          a = fmaf(wv.z, x2, a);
          a = fmaf(wv.w, x3, a);
          acc[t] = a;
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kDecodeMaxT; ++t) {
      float a = acc[t];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
      if (lane == 0) sm.part[wid][t] = a;
    }
  }
  prep_x_range(x, W.xq, W.xblk, T, d, blockIdx.x * blockDim.x + threadIdx.x,
               gridDim.x * blockDim.x);
  __syncthreads();
  if (threadIdx.x < epc * kDecodeMaxT) {
    const int le = threadIdx.x / kDecodeMaxT, t = threadIdx.x % kDecodeMaxT;
    const int ee = blockIdx.x * epc + le;
    if (ee < E && t < T) {
      float s = 0.f;
      for (int p = 0; p < P; ++p) s += sm.part[le * P + p][t];
      W.logits[(size_t)t * E + ee] = s;
    }
  }
  // arrival: the last CTA selects experts for every token and builds the permutation
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t prev = atomicAdd(&W.counters[0], 1u);
    sm.last = (prev == gridDim.x - 1);
  }
  __syncthreads();
  if (!sm.last) return;
  __threadfence();
  const float rs = *router_scale;
  for (int t = wid; t < T; t += kRouteWarps)
    warp_topk_softmax(W.logits + (size_t)t * E, E, k, rs, W.ids + (size_t)t * k, W.w + (size_t)t * k);
  __threadfence_block();
  __syncthreads();
  if (T * k <= kSmallPermMax) {
    if (wid == 0)
      warp_permutation_small(W.ids, T * k, E, W.counts, W.offsets, W.perm, W.inv, W.act, W.n_act, sm.u.cnt);
  } else {
    block_permutation(W.ids, T * k, E, W.counts, W.offsets, W.perm, W.inv, W.act, W.n_act, nullptr, nullptr,
                      nullptr, 1, sm.u.perm);
  }
  if (threadIdx.x == 0) W.counters[0] = 0;
}

// ---------------------------------------------------------------- prefill routing
//
// Router logits as a tiled FP32 product: 128 tokens x 128 experts per CTA, 256 threads each
// owning an 8 x 8 patch, K steps of 16 staged in shared memory (double-buffered: the next
// step's global loads are in flight during this step's FMAs), the d axis split in kRgSplit
// ranges for parallelism (32 token tiles x 9 ranges = 288 CTAs, two per SM). Each output's
// terms are summed in K order inside its range; k_topk adds the range partials in range order.
constexpr int kRgM = 128, kRgN = 128, kRgK = 16, kRgSplit = MOE_ROUTER_MAX_SPLIT;

__global__ void __launch_bounds__(256)
k_router_gemm(const __nv_bfloat16 *__restrict__ x, const float *__restrict__ router_w, int T, int d, int E,
              float *__restrict__ part /* [kRgSplit][T][E] */) {
  __shared__ __align__(16) float xs[2][kRgK][kRgM];
  __shared__ __align__(16) float ws[2][kRgK][kRgN];
  const int tid = threadIdx.x;
  const int t0 = blockIdx.x * kRgM, e0 = blockIdx.y * kRgN, split = blockIdx.z;
  const int nk = d / kRgK;                       // K steps in total (d % 32 == 0)
  const int k0 = (int)((long long)nk * split / kRgSplit), k1 = (int)((long long)nk * (split + 1) / kRgSplit);
  const int ty = tid >> 4, tx = tid & 15;        // tokens ty*4 + {0..3}, 64 + ty*4 + {0..3}; experts alike
  // loaders: x row (tid >> 1), 8 elements at (tid & 1) * 8; W row (tid >> 1), 8 floats
  const int lr = tid >> 1, lc = (tid & 1) * 8;
  const int lt = t0 + lr, le = e0 + lr;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  float xv[8], wv[8];
  auto gload = [&](int ks) {   // this thread's share of K step ks, into registers
    const int kc = ks * kRgK + lc;
    if (lt < T) {
      const uint4 q = __ldg(reinterpret_cast<const uint4 *>(x + (size_t)lt * d + kc));
      const uint32_t qq[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        xv[2 * h] = __uint_as_float(qq[h] << 16);
        xv[2 * h + 1] = __uint_as_float(qq[h] & 0xffff0000u);
      }
    } else {
#pragma unroll
      for (int h = 0; h < 8; ++h) xv[h] = 0.f;
    }
    if (le < E) {
      const float4 a = __ldg(reinterpret_cast<const float4 *>(router_w + (size_t)le * d + kc));
      const float4 b = __ldg(reinterpret_cast<const float4 *>(router_w + (size_t)le * d + kc + 4));
      wv[0] = a.x; wv[1] = a.y; wv[2] = a.z; wv[3] = a.w; wv[4] = b.x; wv[5] = b.y; wv[6] = b.z; wv[7] = b.w;
    } else {
#pragma unroll
      for (int h = 0; h < 8; ++h) wv[h] = 0.f;
    }
  };
  auto sstore = [&](int buf) {
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      xs[buf][lc + h][lr] = xv[h];
      ws[buf][lc + h][lr] = wv[h];
    }
  };
  if (k0 < k1) {
    gload(k0);
    sstore(0);
  }
  __syncthreads();
  for (int ks = k0; ks < k1; ++ks) {
    const int buf = (ks - k0) & 1;
    if (ks + 1 < k1) gload(ks + 1);   // lands while this step computes
#pragma unroll
    for (int kk = 0; kk < kRgK; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4 *>(&xs[buf][kk][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4 *>(&xs[buf][kk][64 + ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4 *>(&ws[buf][kk][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4 *>(&ws[buf][kk][64 + tx * 4]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
    }
    // buffer buf ^ 1 was last read in the previous step, which every thread has left
    if (ks + 1 < k1) sstore(buf ^ 1);
    __syncthreads();
  }
  float *dst = part + (size_t)split * T * E;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int t = t0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + i - 4);
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = e0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + j - 4);
      if (e < E) dst[(size_t)t * E + e] = acc[i][j];
    }
  }
}

// logits = the nsplit range partials added in range order; then top-k + softmax per token
// (one warp per token).
__global__ void __launch_bounds__(256)
k_topk(const float *__restrict__ part, float *__restrict__ logits, const float *__restrict__ router_scale, int T,
       int E, int k, int32_t *ids, float *w, int nsplit) {
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + wid;
  if (t >= T) return;
  if (E <= 128 && k <= 8) {
    // every partial load of the lane's four logits in flight at once; the sums stay in
    // registers for the selection (the same additions, in split order, as below)
    float v[4][MOE_ROUTER_MAX_SPLIT];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int sp = 0; sp < MOE_ROUTER_MAX_SPLIT; ++sp) {
        const int e = lane + 32 * i;
        v[i][sp] = (e < E && sp < nsplit) ? __ldg(part + ((size_t)sp * T + t) * E + e) : 0.f;
      }
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = lane + 32 * i;
      float s = v[i][0];
#pragma unroll
      for (int sp = 1; sp < MOE_ROUTER_MAX_SPLIT; ++sp)
        if (sp < nsplit) s += v[i][sp];
      if (e < E) logits[(size_t)t * E + e] = s;
      o[i] = e < E ? logit_ord(s) : 0u;
    }
    warp_top8_softmax_keys<4>(o, k, *router_scale, ids + (size_t)t * k, w + (size_t)t * k);
    return;
  }
  for (int e = lane; e < E; e += 32) {
    float v = part[(size_t)t * E + e];
#pragma unroll
    for (int sp = 1; sp < nsplit; ++sp) v += part[((size_t)sp * T + t) * E + e];
    logits[(size_t)t * E + e] = v;
  }
  __syncwarp();
  warp_topk_softmax(logits + (size_t)t * E, E, k, *router_scale, ids + (size_t)t * k, w + (size_t)t * k);
}

// Stable permutation over many CTAs: CTA c owns slots [c * kPermSlots, (c + 1) * kPermSlots).
// count: per-CTA per-expert counts; scan: expert offsets, active list, tiles and each CTA's
// output base per expert; place: each slot's position = its CTA's base for its expert + the
// slots of that expert before it inside the CTA (warps in order, lanes ranked by match_any).
constexpr int kPermSlots = kRouteThreads;   // one slot per thread

__device__ void cta_warp_counts(const int32_t *ids, int S, int s0, int32_t (*cnt)[MOE_MAX_E]) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int s = s0 + wid * 32 + lane;
  const int id = s < S ? ids[s] : -1 - lane;
  const uint32_t peers = __match_any_sync(0xffffffffu, id);
  if (s < S && lane == 31 - __clz(peers)) cnt[wid][id] = __popc(peers);
}

__global__ void __launch_bounds__(kRouteThreads) k_perm_count(const int32_t *__restrict__ ids, int S, int E,
                                                              int32_t *__restrict__ ccnt /* [nc][E] */) {
  __shared__ int32_t cnt[kRouteWarps][MOE_MAX_E];
  for (int i = threadIdx.x; i < kRouteWarps * E; i += blockDim.x) cnt[i / E][i % E] = 0;
  __syncthreads();
  cta_warp_counts(ids, S, blockIdx.x * kPermSlots, cnt);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int c = 0;
    for (int w = 0; w < kRouteWarps; ++w) c += cnt[w][e];
    ccnt[(size_t)blockIdx.x * E + e] = c;
  }
}

__global__ void __launch_bounds__(kRouteThreads) k_perm_scan(int nc, int E, int tile_m, bool want_tiles,
                                                             int32_t *__restrict__ ccnt, MoeWork W) {
  __shared__ int32_t scan_tmp[kRouteWarps * 3];
  const int e = threadIdx.x;   // E <= blockDim.x
  int32_t cnt = 0;
  if (e < E)
    for (int c = 0; c < nc; ++c) cnt += ccnt[(size_t)c * E + e];
  const int32_t a = (e < E) && cnt > 0;
  const int32_t nt = (e < E && want_tiles) ? (cnt + tile_m - 1) / tile_m : 0;
  int32_t off, aoff, toff, tot, atot, ttot;
  block_exclusive_scan3(e < E ? cnt : 0, a, nt, off, aoff, toff, scan_tmp, tot, atot, ttot);
  if (e < E) {
    W.counts[e] = cnt;
    W.offsets[e] = off;
    if (a) W.act[aoff] = e;
    int32_t run = off;   // per-CTA output bases for this expert
    for (int c = 0; c < nc; ++c) {
      const int32_t v = ccnt[(size_t)c * E + e];
      ccnt[(size_t)c * E + e] = run;
      run += v;
    }
    if (want_tiles) {
      W.toff[e] = toff;
      for (int i = 0; i < nt; ++i) {
        W.tiles[2 * (toff + i)] = e;
        W.tiles[2 * (toff + i) + 1] = i * tile_m;
      }
    }
  }
  // the down GEMM's work list: consecutive tiles of one expert in pairs (the last may be alone)
  const int32_t np = (nt + 1) / 2;
  int32_t poff, u0, u1, ptot, v0, v1;
  block_exclusive_scan3(np, 0, 0, poff, u0, u1, scan_tmp, ptot, v0, v1);
  if (e < E && want_tiles) {
    for (int i = 0; i < np; ++i) {
      W.pairs[2 * (poff + i)] = toff + 2 * i;
      W.pairs[2 * (poff + i) + 1] = 2 * i + 1 < nt ? 1 : 0;
    }
  }
  if (threadIdx.x == 0) {
    W.offsets[E] = tot;
    *W.n_act = atot;
    if (want_tiles) {
      *W.n_tiles = ttot;
      *W.n_pairs = ptot;
    }
  }
}

__global__ void __launch_bounds__(kRouteThreads) k_perm_place(int S, int E, const int32_t *__restrict__ cbase,
                                                              MoeWork W) {
  __shared__ int32_t cnt[kRouteWarps][MOE_MAX_E];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < kRouteWarps * E; i += blockDim.x) cnt[i / E][i % E] = 0;
  __syncthreads();
  const int s0 = blockIdx.x * kPermSlots;
  cta_warp_counts(W.ids, S, s0, cnt);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {   // per-warp bases inside the CTA
    int32_t run = cbase[(size_t)blockIdx.x * E + e];
    for (int w = 0; w < kRouteWarps; ++w) {
      const int32_t c = cnt[w][e];
      cnt[w][e] = run;
      run += c;
    }
  }
  __syncthreads();
  const int s = s0 + wid * 32 + lane;
  const int id = s < S ? W.ids[s] : -1 - lane;
  const uint32_t peers = __match_any_sync(0xffffffffu, id);
  if (s < S) {
    const int pos = cnt[wid][id] + __popc(peers & ((1u << lane) - 1u));
    W.perm[pos] = s;
    W.inv[s] = pos;
  }
}

__global__ void __launch_bounds__(256)
k_prep_x(const __nv_bfloat16 *__restrict__ x, int T, int d, MoeWork W) {
  prep_x_range(x, W.xq, W.xblk, T, d, blockIdx.x * blockDim.x + threadIdx.x, gridDim.x * blockDim.x);
}

// ---------------------------------------------------------------- routing given by the caller

__global__ void __launch_bounds__(256)
k_route_given(const int32_t *__restrict__ row_expert, const float *__restrict__ row_weight, int R, int E, MoeWork W) {
  for (int r = blockIdx.x * blockDim.x + threadIdx.x; r < R; r += gridDim.x * blockDim.x) {
    int e = row_expert[r];
    float w = row_weight[r];
    if (e < 0 || e >= E) {
      report_error(W.err, MOE_DEV_ERR_BAD_EXPERT, 30);
      e = 0;
      w = 0.f;
    }
    W.ids[r] = e;
    W.w[r] = w;
  }
}

// dst row i = src row index[i], in 16-byte words.
__global__ void __launch_bounds__(256)
k_gather_rows(const uint4 *__restrict__ src, const int32_t *__restrict__ index, int n, int words, uint4 *__restrict__ dst) {
  const long long total = (long long)n * words;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total; i += (long long)gridDim.x * blockDim.x) {
    const int row = (int)(i / words), w = (int)(i - (long long)row * words);
    dst[i] = __ldg(src + (size_t)index[row] * words + w);
  }
}

// out[t, c] = sum_{j < k} y[t k + j, c], j ascending (FP32).
__global__ void __launch_bounds__(256)
k_combine_slots(const float4 *__restrict__ y, int T, int d4, int k, float4 *__restrict__ out) {
  const long long total = (long long)T * d4;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total; i += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(i / d4), c = (int)(i - (long long)t * d4);
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
      const float4 v = __ldg(y + ((size_t)t * k + j) * d4 + c);
      s.x += v.x;
      s.y += v.y;
      s.z += v.z;
      s.w += v.w;
    }
    out[i] = s;
  }
}

}  // namespace

// ---------------------------------------------------------------- launchers

static int launch_err() { return cudaGetLastError() == cudaSuccess ? 0 : -1; }

int moe_launch_route_decode(const MoeLaunch &L, const MoeWork &W, const void *x, const float *router_w,
                            const float *router_scale, int T, int d, int E, int k, int num_sms) {
  (void)num_sms;
  if (T > kDecodeMaxT) return -2;
  const int P = moe_decode_router_parts(d), epc = kRouteWarps / P;
  if (d % 32 || epc < 1) return -2;
  const int grid = (E + epc - 1) / epc;
  moe_prof_mark(L.stream, MOE_K_ROUTE, true);
  k_route_decode<<<grid, kRouteThreads, 0, L.stream>>>(static_cast<const __nv_bfloat16 *>(x), router_w,
                                                        router_scale, T, d, E, k, W);
  if (launch_err()) return -1;
  moe_prof_count(1);
  moe_prof_mark(L.stream, MOE_K_ROUTE, false);
  return 0;
}

size_t moe_route_scratch_bytes(int max_tokens, int max_E, int max_k) {
  const size_t S = (size_t)max_tokens * max_k;
  const size_t nc = (S + kPermSlots - 1) / kPermSlots;
  return ((size_t)kRgSplit * max_tokens * max_E + nc * max_E) * 4;
}

int moe_launch_route_prefill(const MoeLaunch &L, const MoeWork &W, const void *x, const float *router_w,
                             const float *router_scale, int T, int d, int E, int k, int num_sms,
                             bool want_xprep, int tile_m) {
  const __nv_bfloat16 *xb = static_cast<const __nv_bfloat16 *>(x);
  if (E > kRouteThreads) return -2;
  // scratch of the forward's per-slot outputs, free until the expert GEMMs run: the router's
  // range partials, then the per-CTA expert counts of the permutation
  float *part = W.ybuf;
  const int S = T * k;
  const int nc = (S + kPermSlots - 1) / kPermSlots;
  int32_t *ccnt = reinterpret_cast<int32_t *>(W.ybuf + (size_t)kRgSplit * T * E);
  moe_prof_mark(L.stream, MOE_K_ROUTE, true);
  // the router product on the tensor cores where the shape allows, else in FP32 on the CUDA cores
  int nsplit = kRgSplit;
  const int rc = moe_launch_router_tc(L, W, x, router_w, T, d, E, num_sms, part, &nsplit);
  if (rc == -2) {
    dim3 g1((T + kRgM - 1) / kRgM, (E + kRgN - 1) / kRgN, kRgSplit);
    k_router_gemm<<<g1, 256, 0, L.stream>>>(xb, router_w, T, d, E, part);
    if (launch_err()) return -1;
    moe_prof_count(1);
  } else if (rc) {
    return -1;
  }
  k_topk<<<(T + 7) / 8, 256, 0, L.stream>>>(part, W.logits, router_scale, T, E, k, W.ids, W.w, nsplit);
  if (launch_err()) return -1;
  k_perm_count<<<nc, kRouteThreads, 0, L.stream>>>(W.ids, S, E, ccnt);
  if (launch_err()) return -1;
  k_perm_scan<<<1, kRouteThreads, 0, L.stream>>>(nc, E, tile_m, tile_m > 0, ccnt, W);
  if (launch_err()) return -1;
  k_perm_place<<<nc, kRouteThreads, 0, L.stream>>>(S, E, ccnt, W);
  if (launch_err()) return -1;
  moe_prof_count(4);   // top-k, count, scan, place
  if (want_xprep) {
    const int nb = d / MOE_QK;
    const int items = T * nb;
    int grid = (items + 255) / 256;
    if (grid > 4 * num_sms) grid = 4 * num_sms;
    k_prep_x<<<grid, 256, 0, L.stream>>>(xb, T, d, W);
    if (launch_err()) return -1;
    moe_prof_count(1);
  }
  moe_prof_mark(L.stream, MOE_K_ROUTE, false);
  return 0;
}

int moe_launch_route_given(const MoeLaunch &L, const MoeWork &W, const void *x, const int32_t *row_expert,
                           const float *row_weight, int R, int d, int E, int num_sms, bool want_xprep, int tile_m) {
  if (E > kRouteThreads) return -2;
  const int nc = (R + kPermSlots - 1) / kPermSlots;
  int32_t *ccnt = reinterpret_cast<int32_t *>(W.ybuf);   // per-CTA expert counts (free until the experts run)
  moe_prof_mark(L.stream, MOE_K_ROUTE, true);
  int grid = (R + 255) / 256;
  if (grid > 4 * num_sms) grid = 4 * num_sms;
  k_route_given<<<grid, 256, 0, L.stream>>>(row_expert, row_weight, R, E, W);
  if (launch_err()) return -1;
  k_perm_count<<<nc, kRouteThreads, 0, L.stream>>>(W.ids, R, E, ccnt);
  if (launch_err()) return -1;
  k_perm_scan<<<1, kRouteThreads, 0, L.stream>>>(nc, E, tile_m, tile_m > 0, ccnt, W);
  if (launch_err()) return -1;
  k_perm_place<<<nc, kRouteThreads, 0, L.stream>>>(R, E, ccnt, W);
  if (launch_err()) return -1;
  moe_prof_count(4);
  if (want_xprep) {
    const int items = R * (d / MOE_QK);
    int g2 = (items + 255) / 256;
    if (g2 > 4 * num_sms) g2 = 4 * num_sms;
    k_prep_x<<<g2, 256, 0, L.stream>>>(static_cast<const __nv_bfloat16 *>(x), R, d, W);
    if (launch_err()) return -1;
    moe_prof_count(1);
  }
  moe_prof_mark(L.stream, MOE_K_ROUTE, false);
  return 0;
}

int moe_launch_gather_rows(cudaStream_t s, const void *src, const int32_t *index, int n, size_t row_bytes,
                           void *dst) {
  const int words = (int)(row_bytes / 16);
  long long total = (long long)n * words;
  int grid = (int)((total + 255) / 256);
  if (grid > 2048) grid = 2048;
  if (grid < 1) grid = 1;
  k_gather_rows<<<grid, 256, 0, s>>>(static_cast<const uint4 *>(src), index, n, words, static_cast<uint4 *>(dst));
  if (launch_err()) return -1;
  moe_prof_count(1);
  return 0;
}

int moe_launch_combine_slots(cudaStream_t s, const float *y, int T, int d, int k, float *out) {
  const long long total = (long long)T * (d / 4);
  int grid = (int)((total + 255) / 256);
  if (grid > 2048) grid = 2048;
  if (grid < 1) grid = 1;
  k_combine_slots<<<grid, 256, 0, s>>>(reinterpret_cast<const float4 *>(y), T, d / 4, k, reinterpret_cast<float4 *>(out));
  if (launch_err()) return -1;
  moe_prof_count(1);
  return 0;
}
