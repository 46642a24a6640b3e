// moe_decode.cu -- the whole routed-MoE layer for small token counts (decode) in one
// persistent kernel: one CTA per SM, launched cooperatively so all CTAs are resident.
//
//   phase 0  router logits (one expert per CTA, warps split d); arrive at the grid barrier,
//            stage every token's GEMV activations in shared memory, then wait (bounded)
//   phase 1  every CTA selects the top-k experts of every token, builds the stable
//            permutation and its cost-weighted share of the work in its own shared memory
//   phase 2  gate_up GEMV + GeGLU over this CTA's share of the active experts' rows
//   barrier  (h complete)
//   phase 3  down GEMV over this CTA's share of the active experts' down rows
//   barrier  (per-slot outputs complete)
//   phase 4  combine: out[t, r] = sum_j w_tj * s_e * y_tj[r], j in order, rows split over CTAs
//
// One producer warp streams the CTA's weight chunks (gate_up, then down) through a ring of
// shared-memory stages with 1-D bulk copies from the moment the routing is known, so the
// down rows are loading while the gate_up rows are multiplied; the compute warps release a
// stage through an mbarrier and synchronise among themselves with a named barrier.
//
// Definitions as in moe_route.cu / moe_gemv.cu (page "Gemma 4 26B-A4B it QAT Q4_0 ... NInfer
// v3 artifact", "What is inside"). Results equal the separate-kernel path's up to the order
// of the router's FP32 partial sums.
#include "moe_gemv_core.cuh"
#include "moe_route_core.cuh"

namespace {

constexpr int kFMaxT = 8;          // tokens per call on the fused path
constexpr int kFMaxSlots = 128;    // T * k
constexpr int kFMaxE = 256;
constexpr int kFStages = 3;
constexpr int kFMaxCompute = 22;   // compute warps (one more warp produces)
constexpr int kFMinCompute = 8;
constexpr int kDnGroups = kDnRows / 32;   // 32-row groups of a down chunk
constexpr int kBarCompute = 1;            // named barrier of the compute warps
// Cost of a scheduling unit of an expert with T_e tokens: reading the codes is shared by
// the tokens, the multiply-adds are per token.
constexpr int kUnitDecode = 5, kUnitToken = 4;

// Compute warps per CTA: two gate_up work items (gate rows, up rows) per granule, at least
// enough for the down row groups.
__host__ __device__ inline int fused_compute_warps(int G) {
  const int w = 2 * G;
  return w < kFMinCompute ? kFMinCompute : (w > kFMaxCompute ? kFMaxCompute : w);
}

struct FusedShared {
  uint64_t full[kFStages];
  uint64_t empty[kFStages];
  int32_t ids[kFMaxSlots];
  float w[kFMaxSlots];
  int32_t perm[kFMaxSlots];
  int32_t inv[kFMaxSlots];
  int32_t ptok[kFMaxSlots];   // token of each sorted position
  int32_t counts[kFMaxE];
  int32_t offsets[kFMaxE + 1];
  int32_t act[kFMaxE];
  int32_t pc[kFMaxE + 1];     // exclusive prefix of the per-unit costs over the active experts
  int32_t wcnt[kFMaxE / 32];  // active experts per 32-expert group
  uint32_t xb[4];             // cost positions of this CTA's unit boundaries
  float part[kFMaxCompute + 1][kFMaxT];
  int n_act;
  int seq[4];                 // this CTA's unit ranges: gate_up [0, 1), down [2, 3)
  int ok;
};

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long *p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// Named barrier that also returns whether any participating thread passed pred != 0.
__device__ __forceinline__ int named_sync_or(int id, int n, int pred) {
  int r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.s32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\tselp.s32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(pred), "r"(id), "r"(n)
      : "memory");
  return r;
}

// Grid-wide barrier on a monotonically increasing 64-bit counter, split in two: arrival k of
// a phase returns the end of its window of gridDim.x arrivals; the wait spins (bounded) until
// the counter reaches it. One thread per CTA, after the CTA's writes are ordered before it.
__device__ __forceinline__ unsigned long long grid_arrive(unsigned long long *ctr) {
  __threadfence();
  const unsigned long long n = gridDim.x;
  const unsigned long long old = atomicAdd(ctr, 1ull);
  return (old / n + 1ull) * n;
}
__device__ bool grid_wait(const unsigned long long *ctr, unsigned long long target, volatile uint32_t *err,
                          uint32_t where) {
  bool ok = true;
  if (ld_acquire_u64(ctr) < target) {
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire_u64(ctr) < target) {
      if (globaltimer_ns() - t0 > MOE_WAIT_NS) {
        report_error(err, MOE_DEV_ERR_TIMEOUT, where);
        ok = false;
        break;
      }
    }
  }
  __threadfence();
  return ok;
}
// The compute warps' grid barrier (named barrier inside the CTA).
__device__ bool grid_barrier_c(unsigned long long *ctr, volatile uint32_t *err, uint32_t where, int nct, int &ok_s) {
  named_sync(kBarCompute, nct);
  if (threadIdx.x == 0) ok_s = grid_wait(ctr, grid_arrive(ctr), err, where) ? 1 : 0;
  named_sync(kBarCompute, nct);
  return ok_s != 0;
}

struct FChunk {
  int down;   // 0: gate_up chunk, 1: down chunk
  int a, r0, n;
};

// The CTA's chunk sequence: its gate_up units (chunks of up to 2 units of 8 row pairs inside
// one expert), then its down units (chunks of up to 16 units of 8 rows inside one expert).
struct FSeq {
  int g0, g1, d0, d1, upe_g, upe_d;
  __device__ FChunk at(int u) const {   // u: position in the concatenated unit sequence
    FChunk c;
    if (u < g1 - g0) {
      const int v = g0 + u;
      c.down = 0;
      c.a = v / upe_g;
      const int r = v - c.a * upe_g;
      c.r0 = r * kUnit;
      c.n = (v + 1 < g1 && r + 1 < upe_g) ? 2 : 1;
    } else {
      const int v = d0 + (u - (g1 - g0));
      c.down = 1;
      c.a = v / upe_d;
      const int r = v - c.a * upe_d;
      c.r0 = r * kUnit;
      c.n = min(kDnRows / kUnit, min(d1 - v, upe_d - r));
    }
    return c;
  }
  __device__ int total() const { return (g1 - g0) + (d1 - d0); }
};

// Four consecutive lanes turn one 32-wide block into block-scaled int16 in the GEMV word
// order (moe_common.cuh): lane q = lane & 3 holds elements 8q .. 8q+7 in v[], which go to
// positions p1 .. p1+3 and p1+8 .. p1+11, p1 = 16 (q & 1) + 4 (q >> 1). The block's ActBlk
// goes to *blk_s. Every lane of the warp calls.
__device__ __forceinline__ void stage_block_q(const float (&v)[8], bool valid, uint16_t *blk16, ActBlk *blk_s) {
  const int q = threadIdx.x & 3;
  float m = 0.f;
  bool finite = true;
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    m = fmaxf(m, fabsf(v[r]));
    finite = finite && isfinite(v[r]);
  }
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
  int fin = finite ? 1 : 0;
  fin &= __shfl_xor_sync(0xffffffffu, fin, 1);
  fin &= __shfl_xor_sync(0xffffffffu, fin, 2);
  const BlockScale bs = block_scale_for_max(m);
  uint32_t pk[4];
  int s = 0;
#pragma unroll
  for (int r = 0; r < 8; r += 2) {
    const int a0 = act_to_i16(v[r], bs.scale), a1 = act_to_i16(v[r + 1], bs.scale);
    s += a0 + a1;
    pk[r >> 1] = ((uint32_t)a0 & 0xffffu) | ((uint32_t)a1 << 16);
  }
  s += __shfl_xor_sync(0xffffffffu, s, 1);
  s += __shfl_xor_sync(0xffffffffu, s, 2);
  if (valid) {
    const int p1 = 16 * (q & 1) + 4 * (q >> 1);
    *reinterpret_cast<uint2 *>(blk16 + p1) = make_uint2(pk[0], pk[1]);
    *reinterpret_cast<uint2 *>(blk16 + p1 + 8) = make_uint2(pk[2], pk[3]);
    if (q == 0) *blk_s = ActBlk{-8 * s, fin ? bs.inv : __int_as_float(0x7fffffff)};
  }
}

// One gate or up row block against NT tokens' staged activations.
template <int NT>
__device__ __forceinline__ void gu_row_block(const Blk &bk, int b, const uint16_t *xs, const ActBlk *ss,
                                             const uint32_t (&xo)[NT], const uint32_t (&so)[NT], float (&y)[NT]) {
  int al[NT], ah[NT];
  float sc[NT];
#pragma unroll
  for (int i = 0; i < NT; ++i) {
    const ActBlk ab = ss[so[i] + b];
    al[i] = ab.neg8sum;
    ah[i] = 0;
    sc[i] = ab.scale;
  }
#pragma unroll
  for (int wi = 0; wi < 4; ++wi) {
    const uint32_t lo = bk.q[wi] & 0x0F0F0F0Fu, hi = bk.q[wi] & 0xF0F0F0F0u;
#pragma unroll
    for (int i = 0; i < NT; ++i)
      dot8i(lo, hi, *reinterpret_cast<const uint4 *>(xs + xo[i] + b * MOE_QK + 8 * wi), al[i], ah[i]);
  }
#pragma unroll
  for (int i = 0; i < NT; ++i) y[i] = block_finish(y[i], bk.d, sc[i], al[i], ah[i]);
}

// gate_up pass over one staged chunk (kPairs row pairs) for NT tokens, by the compute warps.
// Work item = (granule, gate or up); lane = (row pair p, half h) covering blocks
// 8 granule + 4 h .. + 3. The halves are combined by a shuffle;
// red_b[(item * kPairs + p) * kTX + i] gets the partial.
template <int NT, bool ALIGNED>
__device__ __forceinline__ void gu_pass(const uint8_t *st, uint32_t rb, int nb, int n_items, int nwc, int d,
                                        const uint16_t *xs, const ActBlk *ss, const int32_t *ptok, float *red_b) {
  const int lane = threadIdx.x & 31;
  const int p = lane >> 1, h = lane & 1;
  uint32_t xo[NT], so[NT];
#pragma unroll
  for (int i = 0; i < NT; ++i) {
    const int t = ptok[i];
    xo[i] = (uint32_t)(t * d);
    so[i] = (uint32_t)(t * nb);
  }
  for (int item = threadIdx.x >> 5; item < n_items; item += nwc) {
    const int gran = item >> 1, type = item & 1;
    const int b0 = gran * kGran + h * 4;
    const uint32_t o = (uint32_t)(type * kPairs + p) * rb + (uint32_t)b0 * MOE_QBYTES;
    float y[NT];
#pragma unroll
    for (int i = 0; i < NT; ++i) y[i] = 0.f;
    if (ALIGNED) {
      {
        Blk k0, k1;
        load_blk2_lo(st, o, k0, k1);
        gu_row_block<NT>(k0, b0, xs, ss, xo, so, y);
        gu_row_block<NT>(k1, b0 + 1, xs, ss, xo, so, y);
      }
      {
        Blk k2, k3;
        load_blk2_hi(st, o, k2, k3);
        gu_row_block<NT>(k2, b0 + 2, xs, ss, xo, so, y);
        gu_row_block<NT>(k3, b0 + 3, xs, ss, xo, so, y);
      }
    } else {
      int nbl = nb - b0;
      nbl = nbl < 0 ? 0 : (nbl > 4 ? 4 : nbl);
      for (int j = 0; j < nbl; ++j) {
        const Blk kb = load_blk(st, o + (uint32_t)j * MOE_QBYTES);
        gu_row_block<NT>(kb, b0 + j, xs, ss, xo, so, y);
      }
    }
#pragma unroll
    for (int i = 0; i < NT; ++i) {
      const float yy = y[i] + __shfl_xor_sync(0xffffffffu, y[i], 1);
      if (h == 0) red_b[((size_t)item * kPairs + p) * kTX + i] = yy;
    }
  }
}

// down pass over one staged chunk (up to kDnRows rows) for NT slots: warp = (32-row group,
// part of the row's blocks), lane = row; red_b[(part * kTX + i) * kDnRows + row].
template <int NT>
__device__ __forceinline__ void dn_pass(const uint8_t *st, uint32_t rb, int nbf, int P, int nr, int f,
                                        const uint16_t *hs, const ActBlk *hbk, int rel0, float *red_b) {
  const int lane = threadIdx.x & 31, wq = threadIdx.x >> 5;
  if (wq >= kDnGroups * P) return;
  const int grp = wq % kDnGroups, part = wq / kDnGroups;
  const int row = grp * 32 + lane;
  if (row >= nr) return;
  uint32_t ho[NT], bo[NT];
#pragma unroll
  for (int i = 0; i < NT; ++i) {
    ho[i] = (uint32_t)((rel0 + i) * f);
    bo[i] = (uint32_t)((rel0 + i) * nbf);
  }
  const int b0 = part * nbf / P, b1 = (part + 1) * nbf / P;
  float y[NT];
#pragma unroll
  for (int i = 0; i < NT; ++i) y[i] = 0.f;
  const uint32_t orow = (uint32_t)row * rb;
  for (int b = b0; b < b1; ++b) {
    const Blk bk = load_blk(st, orow + (uint32_t)b * MOE_QBYTES);
    int al[NT], ah[NT];
    float sc[NT];
#pragma unroll
    for (int i = 0; i < NT; ++i) {
      const ActBlk ab = hbk[bo[i] + b];
      al[i] = ab.neg8sum;
      ah[i] = 0;
      sc[i] = ab.scale;
    }
#pragma unroll
    for (int wi = 0; wi < 4; ++wi) {
      const uint32_t lo = bk.q[wi] & 0x0F0F0F0Fu, hi = bk.q[wi] & 0xF0F0F0F0u;
#pragma unroll
      for (int i = 0; i < NT; ++i)
        dot8i(lo, hi, *reinterpret_cast<const uint4 *>(hs + ho[i] + b * MOE_QK + 8 * wi), al[i], ah[i]);
    }
#pragma unroll
    for (int i = 0; i < NT; ++i) y[i] = block_finish(y[i], bk.d, sc[i], al[i], ah[i]);
  }
#pragma unroll
  for (int i = 0; i < NT; ++i) red_b[((size_t)part * kTX + i) * kDnRows + row] = y[i];
}

__global__ void __launch_bounds__((kFMaxCompute + 1) * 32, 1)
k_moe_decode(const __nv_bfloat16 *__restrict__ x, const float *__restrict__ router_w,
             const float *__restrict__ router_scale, const uint8_t *__restrict__ gate_up_q4,
             const uint8_t *__restrict__ down_q4, const float *__restrict__ expert_scale, int T, int d, int f,
             int E, int k, float *__restrict__ out, uint32_t stage_bytes, uint32_t x_bytes, uint32_t red_half,
             MoeWork W) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  __shared__ FusedShared sh;
  const int tid = threadIdx.x, lane = tid & 31, wq = tid >> 5, nw = blockDim.x >> 5;
  const int nwc = nw - 1, nct = nwc * 32;   // compute warps 0 .. nwc-1; warp nwc produces
  const int nb = d / MOE_QK, nbf = f / MOE_QK;
  const int G = (nb + kGran - 1) / kGran;
  const int P = nwc / kDnGroups;
  const uint32_t rb_g = (uint32_t)nb * MOE_QBYTES, rb_d = (uint32_t)nbf * MOE_QBYTES;
  uint8_t *smem = align128(smem_raw);
  uint8_t *xreg = smem + (size_t)kFStages * stage_bytes;
  // gate_up phase: every token's activations; down phase: a window of slots' hidden vectors
  uint16_t *xs = reinterpret_cast<uint16_t *>(xreg);                          // [T][d]
  ActBlk *ss = reinterpret_cast<ActBlk *>(xreg + (size_t)T * d * 2);          // [T][nb]
  const int hcap = (int)(x_bytes / (uint32_t)(2 * f + 8 * nbf));
  uint16_t *hs = reinterpret_cast<uint16_t *>(xreg);                          // [hcap][f]
  ActBlk *hbk = reinterpret_cast<ActBlk *>(xreg + (size_t)hcap * f * 2);      // [hcap][nbf]
  float *red = reinterpret_cast<float *>(xreg + x_bytes);                      // 2 x red_half

  if (tid == 0) {
    for (int s = 0; s < kFStages; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.empty[s], 1);
    }
    fence_mbar_init();
  }
  const float rs = __ldg(router_scale);

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
    if (tid < T) {
      float s = 0.f;
      for (int q = 0; q < nw; ++q) s += sh.part[q][tid];
      W.logits[(size_t)tid * E + e] = s;
    }
    __syncthreads();
  }
  // arrive; stage every token's activations while the other CTAs finish their logits
  unsigned long long target = 0;
  if (tid == 0) target = grid_arrive(W.gbar);
  {
    const int ntask = T * nb * 4;
    for (int base = wq * 32; base < ntask; base += nw * 32) {
      const int task = base + lane;
      const bool valid = task < ntask;
      const int blk = valid ? task >> 2 : 0, q = task & 3;
      const int t = blk / nb, b = blk - t * nb;
      float v[8];
      if (valid) {
        const uint4 u = __ldg(reinterpret_cast<const uint4 *>(x + (size_t)t * d + (size_t)b * MOE_QK + 8 * q));
        const uint32_t uu[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          v[2 * r] = __uint_as_float(uu[r] << 16);
          v[2 * r + 1] = __uint_as_float(uu[r] & 0xffff0000u);
        }
      } else {
#pragma unroll
        for (int r = 0; r < 8; ++r) v[r] = 0.f;
      }
      stage_block_q(v, valid, xs + (size_t)t * d + (size_t)b * MOE_QK, ss + (size_t)t * nb + b);
    }
  }
  if (tid == 0) sh.ok = grid_wait(W.gbar, target, W.err, 20) ? 1 : 0;
  __syncthreads();
  if (!sh.ok) return;

  // ---------------------------------------------------------------- phase 1: selection
  for (int t = wq; t < T; t += nw)
    warp_topk_softmax<kFMaxE>(W.logits + (size_t)t * E, E, k, rs, sh.ids + t * k, sh.w + t * k);
  __syncthreads();
  const int S = T * k;
  const int Ew = (E + 31) & ~31;
  // per expert (threads e < E): slots routed to it and slots routed to lower experts; per
  // slot (threads Ew + s): its sorted position = slots of lower experts + earlier slots of
  // its own expert (the stable counting sort, written out)
  int my_c = 0;
  uint32_t my_bal = 0;
  if (tid < Ew) {
    int lt = 0;
    if (tid < E) {
      for (int s = 0; s < S; ++s) {
        const int id = sh.ids[s];
        my_c += id == tid;
        lt += id < tid;
      }
      sh.counts[tid] = my_c;
      sh.offsets[tid] = lt;
    }
    my_bal = __ballot_sync(0xffffffffu, my_c > 0);
    if (lane == 0) sh.wcnt[wq] = __popc(my_bal);
  }
  for (int s = tid - Ew; s < S; s += (int)blockDim.x - Ew) {
    if (s < 0) break;
    const int id = sh.ids[s];
    int p = 0;
    for (int q = 0; q < S; ++q) {
      const int iq = sh.ids[q];
      p += (iq < id) | ((iq == id) & (q < s));
    }
    sh.inv[s] = p;
    sh.perm[p] = s;
    sh.ptok[p] = s / k;
  }
  const int upe_g = f / kUnit, upe_d = d / kUnit;
  __syncthreads();
  // active experts in ascending order; unit-cost prefix in closed form:
  // pc[a] = sum over earlier active experts of (kUnitDecode + kUnitToken * T_e)
  if (tid < E && my_c > 0) {
    int a = __popc(my_bal & ((1u << lane) - 1u));
    for (int q = 0; q < wq; ++q) a += sh.wcnt[q];
    sh.act[a] = tid;
    sh.pc[a] = kUnitDecode * a + kUnitToken * sh.offsets[tid];
  }
  if (tid < 4) {
    int n_act = 0;
    for (int q = 0; q < Ew / 32; ++q) n_act += sh.wcnt[q];
    const uint32_t ptot = (uint32_t)(kUnitDecode * n_act + kUnitToken * S);
    const uint32_t upe = tid < 2 ? upe_g : upe_d;
    const uint32_t bb = blockIdx.x + (tid & 1);
    sh.xb[tid] = (uint32_t)((unsigned long long)upe * ptot * bb / gridDim.x);
    if (bb >= gridDim.x) sh.seq[tid] = n_act * (int)upe;
    if (tid == 0) {
      sh.n_act = n_act;
      sh.pc[n_act] = (int)ptot;
      sh.offsets[E] = S;
    }
  }
  __syncthreads();
  const int n_act = sh.n_act;
  // this CTA's unit ranges: boundary j lies in the cost interval of exactly one active expert
  for (int a = tid; a < n_act; a += blockDim.x) {
    const int c = kUnitDecode + kUnitToken * sh.counts[sh.act[a]];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t upe = j < 2 ? upe_g : upe_d;
      const uint32_t lo = upe * (uint32_t)sh.pc[a], hi = upe * (uint32_t)sh.pc[a + 1];
      const uint32_t xj = sh.xb[j];
      if (xj >= lo && xj < hi) {
        const uint32_t inexp = (xj - lo + (uint32_t)c - 1u) / (uint32_t)c;
        sh.seq[j] = a * (int)upe + (int)(inexp < upe ? inexp : upe);
      }
    }
  }
  __syncthreads();
  FSeq seq;
  seq.upe_g = upe_g;
  seq.upe_d = upe_d;
  seq.g0 = sh.seq[0];
  seq.g1 = sh.seq[1];
  seq.d0 = sh.seq[2];
  seq.d1 = sh.seq[3];
  const int n_units = seq.total();

  // ---------------------------------------------------------------- producer warp
  if (wq == nwc) {
    if (lane == 0) {
      int u = 0;
      for (int it = 0; u < n_units; ++it) {
        const int slot = it % kFStages;
        if (it >= kFStages &&
            !mbar_wait(&sh.empty[slot], (uint32_t)(it / kFStages - 1) & 1u, W.err, 24))
          break;
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
        u += c.n;
      }
    }
    return;
  }

  if (blockIdx.x == 0) {   // routing copies for the debug readers
    for (int i = tid; i < S; i += nct) {
      W.ids[i] = sh.ids[i];
      W.w[i] = sh.w[i];
      W.perm[i] = sh.perm[i];
      W.inv[i] = sh.inv[i];
    }
    for (int e = tid; e < E; e += nct) {
      W.counts[e] = sh.counts[e];
      W.offsets[e] = sh.offsets[e];
      W.act[e] = sh.act[e];
    }
    if (tid == 0) {
      W.offsets[E] = sh.offsets[E];
      *W.n_act = n_act;
    }
  }

  // ---------------------------------------------------------------- phases 2, 3: the GEMVs
  const bool aligned = (nb % kGran) == 0;
  const int n_items = 2 * G;
  const int lg = G <= 1 ? 1 : (G <= 2 ? 2 : (G <= 4 ? 4 : (G <= 8 ? 8 : 16)));   // lanes per epilogue item
  bool down_phase = false;
  int hw0 = 0, hw1 = 0;   // sorted positions whose hidden vectors are staged in hs
  int pass = 0;
  for (int u = 0, it = 0; u < n_units; ++it) {
    const FChunk c = seq.at(u);
    if (c.down && !down_phase) {
      // all h written before any CTA reads it
      if (!grid_barrier_c(W.gbar, W.err, 21, nct, sh.ok)) return;
      down_phase = true;
    }
    const int slot = it % kFStages;
    const uint32_t par = (uint32_t)(it / kFStages) & 1u;
    const bool okw = mbar_wait(&sh.full[slot], par, W.err, 22);
    if (named_sync_or(kBarCompute, nct, !okw)) return;
    const int e = sh.act[c.a];
    const int cnt = sh.counts[e];
    const int off = sh.offsets[e];
    const uint8_t *st = smem + (size_t)slot * stage_bytes;
    if (!c.down) {
      const int np = c.n * kUnit;
      for (int g0 = 0; g0 < cnt; g0 += kTX) {
        const int ng = min(kTX, cnt - g0);
        float *red_b = red + (size_t)(pass & 1) * red_half;
        ++pass;
        const int32_t *pt = sh.ptok + off + g0;
        if (aligned) {
          switch (ng) {
            case 1: gu_pass<1, true>(st, rb_g, nb, n_items, nwc, d, xs, ss, pt, red_b); break;
            case 2: gu_pass<2, true>(st, rb_g, nb, n_items, nwc, d, xs, ss, pt, red_b); break;
            case 3: gu_pass<3, true>(st, rb_g, nb, n_items, nwc, d, xs, ss, pt, red_b); break;
            default: gu_pass<4, true>(st, rb_g, nb, n_items, nwc, d, xs, ss, pt, red_b); break;
          }
        } else {
          switch (ng) {
            case 1: gu_pass<1, false>(st, rb_g, nb, n_items, nwc, d, xs, ss, pt, red_b); break;
            case 2: gu_pass<2, false>(st, rb_g, nb, n_items, nwc, d, xs, ss, pt, red_b); break;
            case 3: gu_pass<3, false>(st, rb_g, nb, n_items, nwc, d, xs, ss, pt, red_b); break;
            default: gu_pass<4, false>(st, rb_g, nb, n_items, nwc, d, xs, ss, pt, red_b); break;
          }
        }
        named_sync(kBarCompute, nct);
        if (g0 + kTX >= cnt && tid == 0) mbar_arrive(&sh.empty[slot]);   // last read of the stage
        // h = gelu(gate) * up: lg lanes per (row pair, token), partials summed by a shuffle tree
        const int per_warp = 32 / lg, n_it = np * ng;
        for (int base = wq * per_warp; base < n_it; base += nwc * per_warp) {
          const int itm = base + lane / lg, q = lane % lg;
          const int i = itm / np, pp = itm - i * np;
          float g = 0.f, uu = 0.f;
          if (itm < n_it && q < G) {
            g = red_b[((size_t)(2 * q) * kPairs + pp) * kTX + i];
            uu = red_b[((size_t)(2 * q + 1) * kPairs + pp) * kTX + i];
          }
          for (int o = lg >> 1; o > 0; o >>= 1) {
            g += __shfl_xor_sync(0xffffffffu, g, o);
            uu += __shfl_xor_sync(0xffffffffu, uu, o);
          }
          if (q == 0 && itm < n_it)
            W.h[(size_t)sh.perm[off + g0 + i] * f + c.r0 + pp] = gelu_tanh_f(g) * uu;
        }
        // no barrier: the next pass writes the other half of red
      }
    } else {
      if (off < hw0 || off + cnt > hw1) {
        // stage the hidden vectors of the slots from this expert on, up to the end of this
        // CTA's last expert or the window's capacity
        const int a_last = (seq.d1 - 1) / seq.upe_d;
        const int e_last = sh.act[a_last];
        hw0 = off;
        hw1 = min(sh.offsets[e_last] + sh.counts[e_last], off + hcap);
        const int ntask = (hw1 - hw0) * nbf * 4;
        for (int base = wq * 32; base < ntask; base += nwc * 32) {
          const int task = base + lane;
          const bool valid = task < ntask;
          const int blk = valid ? task >> 2 : 0, q = task & 3;
          const int i = blk / nbf, cb = blk - i * nbf;
          float v[8];
          if (valid) {
            const float4 *src =
                reinterpret_cast<const float4 *>(W.h + (size_t)sh.perm[hw0 + i] * f + (size_t)cb * MOE_QK + 8 * q);
            const float4 v0 = __ldcg(src), v1 = __ldcg(src + 1);
            v[0] = v0.x; v[1] = v0.y; v[2] = v0.z; v[3] = v0.w;
            v[4] = v1.x; v[5] = v1.y; v[6] = v1.z; v[7] = v1.w;
          } else {
#pragma unroll
            for (int r = 0; r < 8; ++r) v[r] = 0.f;
          }
          stage_block_q(v, valid, hs + (size_t)i * f + (size_t)cb * MOE_QK, hbk + (size_t)i * nbf + cb);
        }
        named_sync(kBarCompute, nct);
      }
      const int nr = c.n * kUnit;
      for (int g0 = 0; g0 < cnt; g0 += kTX) {
        const int ng = min(kTX, cnt - g0);
        float *red_b = red + (size_t)(pass & 1) * red_half;
        ++pass;
        const int rel0 = off + g0 - hw0;
        switch (ng) {
          case 1: dn_pass<1>(st, rb_d, nbf, P, nr, f, hs, hbk, rel0, red_b); break;
          case 2: dn_pass<2>(st, rb_d, nbf, P, nr, f, hs, hbk, rel0, red_b); break;
          case 3: dn_pass<3>(st, rb_d, nbf, P, nr, f, hs, hbk, rel0, red_b); break;
          default: dn_pass<4>(st, rb_d, nbf, P, nr, f, hs, hbk, rel0, red_b); break;
        }
        named_sync(kBarCompute, nct);
        if (g0 + kTX >= cnt && tid == 0) mbar_arrive(&sh.empty[slot]);   // last read of the stage
        for (int i2 = tid; i2 < nr * ng; i2 += nct) {
          const int i = i2 / nr, row = i2 - i * nr;
          float s = 0.f;
          for (int pt = 0; pt < P; ++pt) s += red_b[((size_t)pt * kTX + i) * kDnRows + row];
          W.ybuf[(size_t)sh.perm[off + g0 + i] * d + c.r0 + row] = s;
        }
      }
    }
    u += c.n;
  }
  if (!down_phase) {
    // this CTA had no down rows: it still takes part in the h barrier
    if (!grid_barrier_c(W.gbar, W.err, 21, nct, sh.ok)) return;
  }
  // ---------------------------------------------------------------- phase 4: combine
  if (!grid_barrier_c(W.gbar, W.err, 23, nct, sh.ok)) return;
  const int r0 = (int)((long long)d * blockIdx.x / gridDim.x), r1 = (int)((long long)d * (blockIdx.x + 1) / gridDim.x);
  const int nr = r1 - r0;
  for (int i2 = tid; i2 < nr * T; i2 += nct) {
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

// Dynamic shared memory of k_moe_decode for these shapes, with the sizes of its regions.
struct FusedSmem {
  uint32_t stage_bytes, x_bytes, red_half;   // red_half in floats
  size_t total;
};
static FusedSmem fused_smem(int T, int d, int f) {
  const int nb = d / MOE_QK, nbf = f / MOE_QK;
  const int G = (nb + kGran - 1) / kGran;
  const int P = fused_compute_warps(G) / kDnGroups;
  FusedSmem r;
  const size_t sg = 2u * kPairs * (size_t)nb * MOE_QBYTES + 16u;
  const size_t sd = (size_t)kDnRows * nbf * MOE_QBYTES + 16u;
  r.stage_bytes = (uint32_t)(((sg > sd ? sg : sd) + 15u) & ~(size_t)15u);
  const size_t xg = (size_t)T * (2 * d + 8 * nb), xh = (size_t)T * (2 * f + 8 * nbf);
  r.x_bytes = (uint32_t)(((xg > xh ? xg : xh) + 15u) & ~(size_t)15u);
  const size_t rg = (size_t)2 * G * kPairs * kTX, rd = (size_t)P * kTX * kDnRows;
  r.red_half = (uint32_t)(rg > rd ? rg : rd);
  r.total = (size_t)kFStages * r.stage_bytes + r.x_bytes + (size_t)2 * r.red_half * 4 + 128;
  return r;
}

bool moe_fused_decode_supported(int T, int d, int f, int E, int k) {
  const int G = (d / MOE_QK + kGran - 1) / kGran;
  return T >= 1 && T <= kFMaxT && T * k <= kFMaxSlots && E <= kFMaxE && G <= kMaxGran &&
         fused_smem(T, d, f).total + sizeof(FusedShared) <= 227 * 1024;
}

int moe_launch_fused_decode(const MoeLaunch &L, const MoeWork &W, const void *x, const float *router_w,
                            const float *router_scale, const uint8_t *gate_up_q4, const uint8_t *down_q4,
                            const float *expert_scale, int T, int d, int f, int E, int k, float *out,
                            int num_sms) {
  if (!moe_fused_decode_supported(T, d, f, E, k)) return -2;
  const FusedSmem fs = fused_smem(T, d, f);
  static size_t set = 0;
  if (fs.total > set) {
    if (cudaFuncSetAttribute(k_moe_decode, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fs.total) !=
        cudaSuccess)
      return -1;
    set = fs.total;
  }
  const int G = (d / MOE_QK + kGran - 1) / kGran;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(num_sms);
  cfg.blockDim = dim3(32 * (fused_compute_warps(G) + 1));
  cfg.dynamicSmemBytes = fs.total;
  cfg.stream = L.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  moe_prof_mark(L.stream, MOE_K_FUSED, true);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, k_moe_decode, static_cast<const __nv_bfloat16 *>(x), router_w,
                                           router_scale, gate_up_q4, down_q4, expert_scale, T, d, f, E, k, out,
                                           fs.stage_bytes, fs.x_bytes, fs.red_half, W);
  if (e != cudaSuccess) return -1;
  moe_prof_mark(L.stream, MOE_K_FUSED, false);
  return 0;
}
