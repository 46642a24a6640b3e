// moe_decode.cu -- the whole routed-MoE layer for small token counts (decode) in one
// persistent kernel: one CTA per SM, launched cooperatively so all CTAs are resident.
//
//   phase 0  x into shared memory (a bulk copy of the bf16 input, or, in a layer stack, the
//            previous layer's FP32 output normalised in place: NORM_IN); router logits (one
//            expert per CTA, warps split d), stored as launch-tagged words
//   phase 1  every CTA selects the top-k experts of every token as soon as that token's
//            tagged logits are all in (bounded polls; the other warps stage every token's
//            GEMV activations in shared memory meanwhile), then builds the stable
//            permutation and its cost-weighted share of the work in its own shared memory
//   phase 2  gate_up GEMV + GeGLU over this CTA's share of the active experts' rows, h stored
//            as launch-tagged words
//   phase 3  down GEMV over this CTA's share of the active experts' down rows (the hidden
//            vectors it needs polled, bounded, until they are in), stored as launch-tagged words
//   phase 4  combine: out[t, r] = sum_j w_tj * s_e * y_tj[r], j in order, rows split over CTAs,
//            each term polled (bounded) until its tagged word is in
//
// One producer warp streams the CTA's weight chunks (gate_up, then down) through a ring of
// shared-memory stages with 1-D bulk copies from the moment the routing is known, so the
// down rows are loading while the gate_up rows are multiplied; the compute warps release a
// stage through an mbarrier and synchronise among themselves with a named barrier.
//
// Definitions as in moe_route.cu / moe_gemv.cu (page "Gemma 4 26B-A4B it QAT Q4_0 ... NInfer
// v3 artifact", "What is inside"). Results equal the separate-kernel path's bit for bit: both
// cut the router's d axis and the down rows the same way and sum in the same orders
// (moe_common.cuh), so a token's output does not depend on the batch it is decoded in.
#include "moe_gemv_core.cuh"
#include "moe_route_core.cuh"

namespace {

constexpr int kFMaxT = 8;          // tokens per call on the fused path
constexpr int kFMaxSlots = 128;    // T * k
constexpr int kFMaxE = 256;
constexpr int kFStages = 3;
constexpr int kFMaxCompute = 12;   // compute warps (128 registers a thread)
constexpr int kFMinCompute = 8;
constexpr int kDnParts = 5;               // parts of a down row's blocks (work items: groups x parts)
static_assert(kFMaxE / 32 <= kFMinCompute + 2 && kFMaxSlots / 32 <= kFMinCompute + 2,
              "the permutation needs a warp per 32 experts and per 32 slots");
static_assert(2 * kDnParts * kTX * kDnRows >= (kFMaxSlots / 32) * kFMaxE + 2 * (kFMaxE / 32),
              "the reduction buffers hold the permutation scratch");
static_assert(kFMaxT == MOE_FUSED_MAX_T && kFMaxSlots == MOE_FUSED_MAX_SLOTS,
              "the workspace's launch-tagged words are sized for these limits");
static_assert(kDnParts == MOE_DN_PARTS && kFMinCompute == MOE_DECODE_MIN_COMPUTE &&
                  kFMaxCompute == MOE_DECODE_MAX_COMPUTE && kGran == 8,
              "the separate decode kernels reproduce this kernel's router slices and down parts");
// Named barriers (0 is __syncthreads): compute warps only; FULL / EMPTY of the two reduction
// buffers between the compute warps and the epilogue warp.
constexpr int kBarCompute = 1;
constexpr int kBarFull0 = 2;
constexpr int kBarEmpty0 = 4;
constexpr int kTXg = 3;                   // tokens per gate_up pass (register budget)
// Cost of a scheduling unit of an expert with T_e tokens: reading the codes is shared by
// the tokens, the multiply-adds are per token.
constexpr int kUnitDecode = 5, kUnitToken = 4;

// Compute warps per CTA: one per gate_up work item (a granule), at least kFMinCompute. Two
// more warps: the producer and the epilogue warp.
__host__ __device__ inline int fused_compute_warps(int G) {
  const int w = G;
  return w < kFMinCompute ? kFMinCompute : (w > kFMaxCompute ? kFMaxCompute : w);
}

struct FusedShared {
  uint64_t full[kFStages];
  uint64_t empty[kFStages];
  uint64_t xbar;              // x copied into shared memory
  int32_t ids[kFMaxSlots];
  float w[kFMaxSlots];
  int32_t perm[kFMaxSlots];
  int32_t inv[kFMaxSlots];
  int32_t ptok[kFMaxSlots];   // token of each sorted position
  int32_t counts[kFMaxE];
  int32_t offsets[kFMaxE + 1];
  int32_t act[kFMaxE];
  union {
    float part[kFMaxCompute + 2][kFMaxT];   // router partial sums (phase 0)
    int32_t pc[kFMaxE + 1];   // exclusive prefix of the per-unit costs over the active experts
  };
  int n_act;
  int seq[4];                 // this CTA's unit ranges: gate_up [0, 1), down [2, 3)
  int cnext;                  // next activation block to convert (phase 1)
  int abort;                  // set by any expired wait: the warps keep their barrier sequence, skip work
  uint32_t tag;               // this launch's tag (launch-tagged words)
};

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long *p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ void ld_relaxed_v2_u64(const unsigned long long *p, unsigned long long &a,
                                                  unsigned long long &b) {
  asm volatile("ld.relaxed.gpu.global.v2.u64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "l"(p));
}
__device__ __forceinline__ void st_relaxed_u64(unsigned long long *p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long tag_word(uint32_t tag, float v) {
  return ((unsigned long long)tag << 32) | __float_as_uint(v);
}
__device__ __forceinline__ bool has_tag(unsigned long long v, uint32_t tag) { return (uint32_t)(v >> 32) == tag; }
__device__ __forceinline__ float tag_value(unsigned long long v) { return __uint_as_float((uint32_t)v); }

__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// No grid barrier: every value one CTA hands to another -- the router logits, the hidden
// vectors h and the per-slot down outputs -- is stored as a launch-tagged 64-bit word, tag <<
// 32 | the FP32 bits, with one relaxed store, and the reader polls the word with relaxed loads
// (bounded) until it carries its launch's tag; it then holds the value, with no counter or
// fence in between, and a CTA goes on as soon as the values it needs are in.
//
// The tag comes from a launch counter: every CTA adds 1 to it once, as it starts, so the
// counter is a multiple of gridDim.x when a launch starts, and the value a CTA's add returns
// rounds down to that start value (the adds before it come from CTAs of its own launch). tag =
// start / gridDim.x + 1 differs for any two consecutive launches and is never 0, the value of
// zeroed words. A word a reader polls is always written by the reader's own launch, so a stale
// word carries an older launch's tag; the 32-bit tag repeats only every 2^32 launches (about a
// day of back-to-back single-token layers), so a stale word could pass only if it was last
// written a multiple of 2^32 launches earlier and is read before its new value lands. (After
// an expired wait the host zeroes the counter and the tagged words before the next launch.)
__device__ __forceinline__ void named_arrive(int id, int n) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// Wait for an mbarrier phase, at most limit_ns; gives up at once when *abort is set and sets
// it when the bound expires.
__device__ bool wait_phase(uint64_t *bar, uint32_t parity, volatile int *abort, volatile uint32_t *err,
                           uint32_t where, uint64_t limit_ns) {
  if (mbar_test(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_test(bar, parity)) {
    if (*abort) return false;
    if (globaltimer_ns() - t0 > limit_ns) {
      report_error(err, MOE_DEV_ERR_TIMEOUT, where);
      *abort = 1;
      return false;
    }
  }
  return true;
}

// The selection of one token by one warp from its launch-tagged logit words lt[0, E): each
// lane polls its experts' words (lane + 32 i) until every word of the token carries the
// launch's tag, then the warp selects as warp_topk_softmax does from the same values. A
// bound that runs out (decided by the warp as one) reports a timeout, sets *abort and
// returns false.
template <int kMaxPer>
__device__ bool warp_select_tagged(const unsigned long long *lt, uint32_t tag, int E, int k, float rscale,
                                   int32_t *ids, float *w, volatile int *abort, volatile uint32_t *err,
                                   uint64_t limit_ns) {
  const int lane = threadIdx.x & 31;
  unsigned long long v[kMaxPer];
#pragma unroll
  for (int i = 0; i < kMaxPer; ++i) {
    const int e = lane + 32 * i;
    v[i] = e < E ? ld_relaxed_u64(lt + e) : tag_word(tag, 0.f);
  }
  uint64_t t0 = 0;
  for (int round = 0;; ++round) {
    bool mine = true;
#pragma unroll
    for (int i = 0; i < kMaxPer; ++i) mine = mine && has_tag(v[i], tag);
    if (__all_sync(0xffffffffu, mine)) break;
    if (round == 0) {
      t0 = globaltimer_ns();
    } else if (__any_sync(0xffffffffu, globaltimer_ns() - t0 > limit_ns)) {
      if (lane == 0) {
        report_error(err, MOE_DEV_ERR_TIMEOUT, 20);
        *abort = 1;
      }
      return false;
    }
#pragma unroll
    for (int i = 0; i < kMaxPer; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !has_tag(v[i], tag)) v[i] = ld_relaxed_u64(lt + e);
    }
  }
  if (k <= 8) {
    uint32_t o[kMaxPer];
#pragma unroll
    for (int i = 0; i < kMaxPer; ++i) o[i] = lane + 32 * i < E ? logit_ord(tag_value(v[i])) : 0u;
    warp_top8_softmax_keys<kMaxPer>(o, k, rscale, ids, w);
  } else {
    uint64_t key[kMaxPer];
#pragma unroll
    for (int i = 0; i < kMaxPer; ++i) {
      const int e = lane + 32 * i;
      key[i] = e < E ? topk_key(tag_value(v[i]), e) : 0ull;
    }
    warp_topk_softmax_keys64<kMaxPer>(key, k, rscale, ids, w);
  }
  return true;
}

// Polls the n <= 8 launch-tagged words p[j * stride] (issued together) until each carries
// the tag; their values go to y[]. False when the bound ran out (reported, *abort set).
__device__ bool poll_tagged(const unsigned long long *p, size_t stride, int n, uint32_t tag, float (&y)[8],
                            volatile int *abort, volatile uint32_t *err, uint64_t limit_ns) {
  unsigned long long v[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) v[j] = j < n ? ld_relaxed_u64(p + (size_t)j * stride) : tag_word(tag, 0.f);
  bool all = true;
#pragma unroll
  for (int j = 0; j < 8; ++j) all = all && has_tag(v[j], tag);
  if (!all) {
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
      all = true;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (!has_tag(v[j], tag)) v[j] = ld_relaxed_u64(p + (size_t)j * stride);
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) all = all && has_tag(v[j], tag);
      if (all) break;
      if (*abort) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        report_error(err, MOE_DEV_ERR_TIMEOUT, 23);
        *abort = 1;
        return false;
      }
    }
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) y[j] = tag_value(v[j]);
  return true;
}

// Polls the 32 launch-tagged words p[0, 32) (16-byte aligned, all loads in flight at once)
// until each carries the tag; their values go to v[]. False when *abort is set or the bound
// ran out (reported, *abort set).
__device__ bool poll_tagged32(const unsigned long long *p, uint32_t tag, float (&v)[MOE_QK], volatile int *abort,
                              volatile uint32_t *err, uint64_t limit_ns) {
  unsigned long long w[MOE_QK];
#pragma unroll
  for (int i = 0; i < MOE_QK / 2; ++i) ld_relaxed_v2_u64(p + 2 * i, w[2 * i], w[2 * i + 1]);
  bool all = true;
#pragma unroll
  for (int i = 0; i < MOE_QK; ++i) all = all && has_tag(w[i], tag);
  if (!all) {
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
#pragma unroll
      for (int i = 0; i < MOE_QK / 2; ++i)
        if (!has_tag(w[2 * i], tag) || !has_tag(w[2 * i + 1], tag)) ld_relaxed_v2_u64(p + 2 * i, w[2 * i], w[2 * i + 1]);
      all = true;
#pragma unroll
      for (int i = 0; i < MOE_QK; ++i) all = all && has_tag(w[i], tag);
      if (all) break;
      if (*abort) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        report_error(err, MOE_DEV_ERR_TIMEOUT, 21);
        *abort = 1;
        return false;
      }
    }
  }
#pragma unroll
  for (int i = 0; i < MOE_QK; ++i) v[i] = tag_value(w[i]);
  return true;
}

struct FChunk {
  int down;   // 0: gate_up chunk, 1: down chunk
  int a, r0, n;
};

// The CTA's chunk sequence: its gate_up units [seq[0], seq[1]) (chunks of up to 2 units of 8
// row pairs inside one expert), then its down units [seq[2], seq[3]) (chunks of up to 16 units
// of 8 rows inside one expert), walked without a division per chunk.
struct FWalk {
  int down, a, r, left;    // phase, active-expert index, unit within the expert, units left in the phase
  __device__ void start(int u0, int u1, int upe, int dn) {
    down = dn;
    a = u0 / upe;
    r = u0 - a * upe;
    left = u1 - u0;
  }
  __device__ void init(const int *seq, int upe_g, int upe_d) {
    start(seq[0], seq[1], upe_g, 0);
    if (left == 0) start(seq[2], seq[3], upe_d, 1);
  }
  __device__ bool done() const { return down && left == 0; }
  __device__ FChunk cur(int upe_g, int upe_d) const {
    FChunk c;
    c.down = down;
    c.a = a;
    c.r0 = r * kUnit;
    c.n = down ? min(kDnRows / kUnit, min(left, upe_d - r)) : ((left >= 2 && r + 1 < upe_g) ? 2 : 1);
    return c;
  }
  __device__ void advance(int n, const int *seq, int upe_g, int upe_d) {
    left -= n;
    r += n;
    if (r == (down ? upe_d : upe_g)) {
      ++a;
      r = 0;
    }
    if (!down && left == 0) start(seq[2], seq[3], upe_d, 1);
  }
};

// One thread turns one 32-wide block v[] into block-scaled int16 in the GEMV word order
// (moe_common.cuh); with sw = 1 the block's 16-byte words are stored swapped in pairs (word w
// at w ^ 1). The block's ActBlk goes to *blk_s.
__device__ __forceinline__ void stage_block_t(const float (&v)[MOE_QK], int sw, uint16_t *blk16, ActBlk *blk_s) {
  float m = 0.f;
  bool finite = true;
#pragma unroll
  for (int i = 0; i < MOE_QK; ++i) {
    m = fmaxf(m, fabsf(v[i]));
    finite = finite && isfinite(v[i]);
  }
  const BlockScale bs = block_scale_for_max(m);
  int s = 0;
#pragma unroll
  for (int wi = 0; wi < 4; ++wi) {
    // word wi: elements 4wi..4wi+3 (low nibbles), then 16+4wi..16+4wi+3 (high nibbles)
    uint32_t pk[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const int e0 = h < 2 ? 4 * wi + 2 * h : 16 + 4 * wi + 2 * (h - 2);
      const int a0 = act_to_i16(v[e0], bs.scale), a1 = act_to_i16(v[e0 + 1], bs.scale);
      s += a0 + a1;
      pk[h] = ((uint32_t)a0 & 0xffffu) | ((uint32_t)a1 << 16);
    }
    *reinterpret_cast<uint4 *>(blk16 + 8 * (wi ^ sw)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  }
  *blk_s = ActBlk{-8 * s, finite ? bs.inv : __int_as_float(0x7fffffff)};
}

// Two consecutive Q4_0 blocks (36 bytes) of a row at a shared-memory byte offset o that is
// 8-byte aligned (ODD = false) or 4 bytes past it (ODD = true).
template <bool ODD>
__device__ __forceinline__ void load_span2(const uint8_t *smem, uint32_t o, Blk &b0, Blk &b1) {
  uint32_t w[10];
  if (!ODD) {
    const uint2 *wp = reinterpret_cast<const uint2 *>(smem + o);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint2 v = wp[i];
      w[2 * i] = v.x;
      w[2 * i + 1] = v.y;
    }
    w[8] = *reinterpret_cast<const uint32_t *>(smem + o + 32);
  } else {
    w[0] = *reinterpret_cast<const uint32_t *>(smem + o);
    const uint2 *wp = reinterpret_cast<const uint2 *>(smem + o + 4);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint2 v = wp[i];
      w[1 + 2 * i] = v.x;
      w[2 + 2 * i] = v.y;
    }
  }
  w[9] = 0u;
  split_blk2(w, b0, b1);
}

// One block of a gate row and its up row against NT tokens' staged activations (the
// activation words of block b are swizzled by sw).
template <int NT>
__device__ __forceinline__ void gu_pair_block(const Blk &bg, const Blk &bu, int b, int sw, const uint16_t *xs,
                                              const ActBlk *ss, const uint32_t (&xo)[NT], const uint32_t (&so)[NT],
                                              float (&yg)[NT], float (&yu)[NT]) {
  int gl[NT], gh[NT], ul[NT], uh[NT];
  float sc[NT];
#pragma unroll
  for (int i = 0; i < NT; ++i) {
    const ActBlk ab = ss[so[i] + b];
    gl[i] = ab.neg8sum;
    ul[i] = ab.neg8sum;
    gh[i] = 0;
    uh[i] = 0;
    sc[i] = ab.scale;
  }
#pragma unroll
  for (int wi = 0; wi < 4; ++wi) {
    const uint32_t glo = bg.q[wi] & 0x0F0F0F0Fu, ghi = bg.q[wi] & 0xF0F0F0F0u;
    const uint32_t ulo = bu.q[wi] & 0x0F0F0F0Fu, uhi = bu.q[wi] & 0xF0F0F0F0u;
#pragma unroll
    for (int i = 0; i < NT; ++i) {
      const uint4 xv = *reinterpret_cast<const uint4 *>(xs + xo[i] + b * MOE_QK + 8 * (wi ^ sw));
      dot8i(glo, ghi, xv, gl[i], gh[i]);
      dot8i(ulo, uhi, xv, ul[i], uh[i]);
    }
  }
#pragma unroll
  for (int i = 0; i < NT; ++i) {
    yg[i] = block_finish(yg[i], bg.d, sc[i], gl[i], gh[i]);
    yu[i] = block_finish(yu[i], bu.d, sc[i], ul[i], uh[i]);
  }
}

// gate_up pass over one staged chunk (kPairs row pairs) for NT tokens, by the compute warps:
// items first, first + nwc, ... Work item = granule g (G items); lane = (row pair p, s): the
// lane multiplies the gate and the up row of pair p over blocks 8 g + 4 s .. + 3, read as two
// 2-block spans (the first 8-byte aligned, the second 4 bytes past). The two lanes of a pair
// are combined by a shuffle; red_b[((g * kTX + i) * kPairs + p) * 2 + {0, 1}] gets the gate
// and up partials. Activation words of blocks with (b >> 2) & 1 = 1 are stored swapped in
// pairs, so the two halves of the warp read different banks.
template <int NT, bool ALIGNED>
__device__ __forceinline__ void gu_pass(const uint8_t *st, uint32_t rb, int nb, int n_items, int nwc, int first,
                                        int d, const uint16_t *xs, const ActBlk *ss, const int32_t *ptok,
                                        float *red_b) {
  const int lane = threadIdx.x & 31;
  const int p = lane >> 1, sl = lane & 1;
  uint32_t xo[NT], so[NT];
#pragma unroll
  for (int i = 0; i < NT; ++i) {
    const int t = ptok[i];
    xo[i] = (uint32_t)(t * d);
    so[i] = (uint32_t)(t * nb);
  }
  for (int item = first; item < n_items; item += nwc) {
    const int b0 = item * kGran + sl * 4;
    const uint32_t og = (uint32_t)p * rb + (uint32_t)b0 * MOE_QBYTES;
    const uint32_t ou = og + (uint32_t)kPairs * rb;
    float yg[NT], yu[NT];
#pragma unroll
    for (int i = 0; i < NT; ++i) { yg[i] = 0.f; yu[i] = 0.f; }
    if (ALIGNED) {
      Blk g0, g1, u0, u1, g2, g3, u2, u3;
      load_span2<false>(st, og, g0, g1);
      load_span2<false>(st, ou, u0, u1);
      load_span2<true>(st, og + 2 * MOE_QBYTES, g2, g3);
      load_span2<true>(st, ou + 2 * MOE_QBYTES, u2, u3);
      gu_pair_block<NT>(g0, u0, b0, sl, xs, ss, xo, so, yg, yu);
      gu_pair_block<NT>(g1, u1, b0 + 1, sl, xs, ss, xo, so, yg, yu);
      gu_pair_block<NT>(g2, u2, b0 + 2, sl, xs, ss, xo, so, yg, yu);
      gu_pair_block<NT>(g3, u3, b0 + 3, sl, xs, ss, xo, so, yg, yu);
    } else {
      for (int j = 0; j < 4 && b0 + j < nb; ++j) {
        const Blk bg = load_blk(st, og + (uint32_t)j * MOE_QBYTES);
        const Blk bu = load_blk(st, ou + (uint32_t)j * MOE_QBYTES);
        gu_pair_block<NT>(bg, bu, b0 + j, sl, xs, ss, xo, so, yg, yu);
      }
    }
#pragma unroll
    for (int i = 0; i < NT; ++i) {
      const float g = yg[i] + __shfl_xor_sync(0xffffffffu, yg[i], 1);
      const float u = yu[i] + __shfl_xor_sync(0xffffffffu, yu[i], 1);
      if (sl == 0) *reinterpret_cast<float2 *>(red_b + (((size_t)item * kTX + i) * kPairs + p) * 2) = make_float2(g, u);
    }
  }
}

// Blocks b, b + 1 (b even) of a row whose byte offset o is 4-byte aligned: nine 32-bit loads.
__device__ __forceinline__ void load_pair_w(const uint8_t *smem, uint32_t o, Blk &b0, Blk &b1) {
  const uint32_t *wp = reinterpret_cast<const uint32_t *>(smem + o);
  uint32_t w[10];
#pragma unroll
  for (int i = 0; i < 9; ++i) w[i] = wp[i];
  w[9] = 0u;
  split_blk2(w, b0, b1);
}

// One block of two down rows (k0, k1) against NT slots' staged hidden vectors (the block's
// integer dot products, then one rounding into y per row and slot), one activation load
// serving both rows.
template <int NT>
__device__ __forceinline__ void dn_block2(const Blk &k0, const Blk &k1, int b, const uint16_t *hs, const ActBlk *hbk,
                                          const uint32_t (&ho)[NT], const uint32_t (&bo)[NT], float (&y0)[NT],
                                          float (&y1)[NT]) {
  int al0[NT], ah0[NT], al1[NT], ah1[NT];
  float sc[NT];
#pragma unroll
  for (int i = 0; i < NT; ++i) {
    const ActBlk ab = hbk[bo[i] + b];
    al0[i] = ab.neg8sum;
    al1[i] = ab.neg8sum;
    ah0[i] = 0;
    ah1[i] = 0;
    sc[i] = ab.scale;
  }
#pragma unroll
  for (int wi = 0; wi < 4; ++wi) {
    const uint32_t lo0 = k0.q[wi] & 0x0F0F0F0Fu, hi0 = k0.q[wi] & 0xF0F0F0F0u;
    const uint32_t lo1 = k1.q[wi] & 0x0F0F0F0Fu, hi1 = k1.q[wi] & 0xF0F0F0F0u;
#pragma unroll
    for (int i = 0; i < NT; ++i) {
      const uint4 xv = *reinterpret_cast<const uint4 *>(hs + ho[i] + b * MOE_QK + 8 * wi);
      dot8i(lo0, hi0, xv, al0[i], ah0[i]);
      dot8i(lo1, hi1, xv, al1[i], ah1[i]);
    }
  }
#pragma unroll
  for (int i = 0; i < NT; ++i) {
    y0[i] = block_finish(y0[i], k0.d, sc[i], al0[i], ah0[i]);
    y1[i] = block_finish(y1[i], k1.d, sc[i], al1[i], ah1[i]);
  }
}

// down pass over one staged chunk (up to kDnRows rows) for NT slots, by the compute warps:
// items first, first + nwc, ... Work item = (pair of 32-row groups g2 and g2 + 2, part of the
// row's blocks); the lane takes one row of each group (an activation load serves both);
// red_b[(part * kTX + i) * kDnRows + row]. With PAIRED
// (an even number of blocks per row, so every row starts 4-byte aligned) a part takes whole
// block pairs and the blocks left over go one each to the first parts; otherwise parts are
// contiguous block ranges read block by block.
template <int NT, bool PAIRED>
__device__ __forceinline__ void dn_pass(const uint8_t *st, uint32_t rb, int nbf, int P, int nwc, int first, int nr,
                                        int f, const uint16_t *hs, const ActBlk *hbk, int rel0, float *red_b) {
  const int lane = threadIdx.x & 31;
  uint32_t ho[NT], bo[NT];
#pragma unroll
  for (int i = 0; i < NT; ++i) {
    ho[i] = (uint32_t)((rel0 + i) * f);
    bo[i] = (uint32_t)((rel0 + i) * nbf);
  }
  // work item = (row-group pair g2, part): the lane takes rows g2 * 32 + lane and that + 64
  for (int item = first; item < 2 * P; item += nwc) {
    const int g2 = item & 1, part = item >> 1;
    if (g2 * 32 >= nr) continue;   // warp-uniform: these rows are past the chunk
    const int r0 = g2 * 32 + lane, r1 = r0 + 64;
    const bool v0 = r0 < nr, v1 = r1 < nr;
    float y0[NT], y1[NT];
#pragma unroll
    for (int i = 0; i < NT; ++i) { y0[i] = 0.f; y1[i] = 0.f; }
    const uint32_t o0 = (uint32_t)(v0 ? r0 : 0) * rb, o1 = (uint32_t)(v1 ? r1 : 0) * rb;   // in the stage
    if (PAIRED) {
      const int per = nbf / (2 * P);   // pairs per part
      for (int pr = part * per; pr < (part + 1) * per; ++pr) {
        Blk a0, a1, c0, c1;
        load_pair_w(st, o0 + (uint32_t)(2 * pr) * MOE_QBYTES, a0, a1);
        load_pair_w(st, o1 + (uint32_t)(2 * pr) * MOE_QBYTES, c0, c1);
        dn_block2<NT>(a0, c0, 2 * pr, hs, hbk, ho, bo, y0, y1);
        dn_block2<NT>(a1, c1, 2 * pr + 1, hs, hbk, ho, bo, y0, y1);
      }
      for (int b = 2 * P * per + part; b < nbf; b += P) {
        const Blk a = load_blk(st, o0 + (uint32_t)b * MOE_QBYTES), c = load_blk(st, o1 + (uint32_t)b * MOE_QBYTES);
        dn_block2<NT>(a, c, b, hs, hbk, ho, bo, y0, y1);
      }
    } else {
      for (int b = part * nbf / P; b < (part + 1) * nbf / P; ++b) {
        const Blk a = load_blk(st, o0 + (uint32_t)b * MOE_QBYTES), c = load_blk(st, o1 + (uint32_t)b * MOE_QBYTES);
        dn_block2<NT>(a, c, b, hs, hbk, ho, bo, y0, y1);
      }
    }
#pragma unroll
    for (int i = 0; i < NT; ++i) {
      if (v0) red_b[((size_t)part * kTX + i) * kDnRows + r0] = y0[i];
      if (v1) red_b[((size_t)part * kTX + i) * kDnRows + r1] = y1[i];
    }
  }
}

// NORM_IN: the layer input is the previous layer's FP32 output y_prev, normalised here
// (unit-gain RMSNorm + bf16 cast, as moe_norm.cu) instead of a bf16 x; CTA 0 also writes the
// bf16 x to x_out when it is not null. y_prev must not overlap `out`: with no grid barrier, a
// CTA may write its output rows while another still reads y_prev.
template <bool NORM_IN>
__global__ void __launch_bounds__((kFMaxCompute + 2) * 32, 1)
k_moe_decode(const __nv_bfloat16 *__restrict__ x, const float *y_prev, float eps, __nv_bfloat16 *x_out,
             const float *__restrict__ router_w, const float *__restrict__ router_scale,
             const uint8_t *__restrict__ gate_up_q4, const uint8_t *__restrict__ down_q4,
             const float *__restrict__ expert_scale, int T, int d, int f, int E, int k, float *out,
             uint32_t stage_bytes, uint32_t x_bytes, uint32_t red_half, MoeWork W, int accumulate,
             const uint8_t *__restrict__ dense_gu, const uint8_t *__restrict__ dense_dn,
             const float *__restrict__ next_router_w) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  __shared__ FusedShared sh;
  const int tid = threadIdx.x, lane = tid & 31, wq = tid >> 5, nw = blockDim.x >> 5;
  // this CTA's add to the launch counter, which names the launch (its latency hides behind
  // the router)
  const int bar_tid = (int)blockDim.x - 32;
  const unsigned long long gstart = tid == bar_tid ? atomicAdd(W.gbar, 1ull) : 0ull;
  const int nwc = nw - 2, nct = nwc * 32;   // compute warps 0 .. nwc-1; warp nwc produces, nwc+1 epilogues
  const int nteam = nct + 32;   // compute + epilogue warps
  const int nb = d / MOE_QK, nbf = f / MOE_QK;
  const int G = (nb + kGran - 1) / kGran;
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
      mbar_init(&sh.empty[s], nwc);
    }
    mbar_init(&sh.xbar, 1);
    fence_mbar_init();
    sh.abort = 0;
    sh.cnext = 0;
    if constexpr (!NORM_IN) {
      // x (bf16) into the activation region now; it is converted in place before the first barrier
      mbar_arrive_expect_tx(&sh.xbar, (uint32_t)(T * d * 2));
      bulk_g2s(xreg, x, (uint32_t)(T * d * 2), &sh.xbar);
    }
  }
  if constexpr (NORM_IN) {
    // x = bf16(y / sqrt(mean(y^2) + eps)) per token with moe_norm.cu's arithmetic (256 lanes,
    // the same summation order), written straight into the activation region
    __syncthreads();   // the mbarriers are initialised
    __nv_bfloat16 *xb = reinterpret_cast<__nv_bfloat16 *>(xreg);
    for (int t = 0; t < T; ++t) {
      const float *yr = y_prev + (size_t)t * d;
      if (tid < 256) {
        float s = 0.f;
        for (int i = tid; i < d; i += 256) s = fmaf(yr[i], yr[i], s);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) sh.part[wq][0] = s;
      }
      __syncthreads();
      float tot = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) tot += sh.part[w][0];
      const float inv = 1.0f / sqrtf(tot / (float)d + eps);
      for (int i = tid; i < d; i += blockDim.x) xb[(size_t)t * d + i] = __float2bfloat16_rn(yr[i] * inv);
      __syncthreads();   // sh.part is reused for the next token
    }
    if (blockIdx.x == 0 && x_out != nullptr)
      for (int i = tid; i < T * d; i += blockDim.x) x_out[i] = xb[i];
    if (tid == 0) mbar_arrive(&sh.xbar);   // the activation region holds x (no copy to wait for)
  }
  const float rs = __ldg(router_scale);
  // test-only fault: CTA 0 never stores its router logits, so every CTA's bounded wait for
  // them runs out and reports a timeout
  const bool skip_logits = W.inject == MOE_INJECT_SKIP_ROUTER_ARRIVAL && blockIdx.x == 0;
  // the launch's tag into shared memory (gstart / gridDim.x rounds down to the launch's start)
  auto publish_base = [&]() {
    if (tid == bar_tid) {
      sh.tag = (uint32_t)(gstart / gridDim.x) + 1u;
    }
  };

  // ---------------------------------------------------------------- phase 0: router
  // A lane loads its router weights first (up to kRtrW float4 groups at once: their HBM
  // latency overlaps), then multiplies them with x from the shared-memory copy; the terms are
  // summed in the same order as a one-group-at-a-time loop (the separate router's order).
  constexpr int kRtrW = 4;
  for (int e = blockIdx.x; e < E; e += gridDim.x) {
    const int seg = (d / 4) / nw * 4;   // float4-aligned slice per warp; the last warp takes the tail
    const int i0 = wq * seg, i1 = (wq == nw - 1) ? d : i0 + seg;
    const float *wr = router_w + (size_t)e * d;
    float4 wv[kRtrW];
#pragma unroll
    for (int j = 0; j < kRtrW; ++j) {
      const int i = i0 + lane * 4 + 128 * j;
      wv[j] = (i + 3 < i1) ? __ldg(reinterpret_cast<const float4 *>(wr + i)) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();   // the x copy's mbarrier is initialised; sh.part is free
    wait_phase(&sh.xbar, 0u, &sh.abort, W.err, 26, W.wait_ns);
    if (e == (int)blockIdx.x) publish_base();
    float acc[kFMaxT];
#pragma unroll
    for (int t = 0; t < kFMaxT; ++t) acc[t] = 0.f;
    auto mac = [&](const float4 &w4, int i) {
#pragma unroll
      for (int t = 0; t < kFMaxT; ++t) {
        if (t < T) {
          const uint2 xv = *reinterpret_cast<const uint2 *>(xs + (size_t)t * d + i);
          float a = acc[t];
          a = fmaf(w4.x, __uint_as_float(xv.x << 16), a);
          a = fmaf(w4.y, __uint_as_float(xv.x & 0xffff0000u), a);
          a = fmaf(w4.z, __uint_as_float(xv.y << 16), a);
          a = fmaf(w4.w, __uint_as_float(xv.y & 0xffff0000u), a);
          acc[t] = a;
        }
      }
    };
#pragma unroll
    for (int j = 0; j < kRtrW; ++j) {
      const int i = i0 + lane * 4 + 128 * j;
      if (i + 3 < i1) mac(wv[j], i);
    }
    for (int i = i0 + lane * 4 + 128 * kRtrW; i + 3 < i1; i += 128)
      mac(__ldg(reinterpret_cast<const float4 *>(wr + i)), i);
#pragma unroll
    for (int t = 0; t < kFMaxT; ++t) {
      float a = acc[t];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
      if (lane == 0) sh.part[wq][t] = a;
    }
    __syncthreads();
    if (tid < T && !skip_logits) {
      float s = 0.f;
      for (int q = 0; q < nw; ++q) s += sh.part[q][tid];
      st_relaxed_u64(W.ltag + (size_t)tid * E + e, tag_word(sh.tag, s));
    }
    __syncthreads();
  }
  if ((int)blockIdx.x >= E) publish_base();
  // ---------------------------------------------------------------- phase 1: selection
  // warp t selects token t as soon as its tagged logits are in; the other warps convert every
  // token's activations in place meanwhile (x was copied into the activation region at the
  // start), a thread a (token, block), 32 blocks a warp at a time from a shared counter, and
  // the selecting warps join them when done
  __syncthreads();   // the router is done with x; sh.tag is published
  if (wq < T) {
    if (E <= 128)
      warp_select_tagged<4>(W.ltag + (size_t)wq * E, sh.tag, E, k, rs, sh.ids + wq * k, sh.w + wq * k, &sh.abort,
                            W.err, W.wait_ns);
    else
      warp_select_tagged<kFMaxE / 32>(W.ltag + (size_t)wq * E, sh.tag, E, k, rs, sh.ids + wq * k, sh.w + wq * k,
                                      &sh.abort, W.err, W.wait_ns);
  }
  if (wait_phase(&sh.xbar, 0u, &sh.abort, W.err, 26, W.wait_ns)) {
    const int nblk = T * nb;
    for (;;) {
      int b0 = 0;
      if (lane == 0) b0 = atomicAdd(&sh.cnext, 32);
      b0 = __shfl_sync(0xffffffffu, b0, 0);
      if (b0 >= nblk) break;
      const int blk = b0 + lane;
      if (blk < nblk) {
        const int t = blk / nb, b = blk - t * nb;
        const uint4 *src = reinterpret_cast<const uint4 *>(xs + (size_t)t * d + (size_t)b * MOE_QK);
        uint4 raw[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) raw[i] = src[i];
        float v[MOE_QK];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t uu[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            v[8 * i + 2 * h] = __uint_as_float(uu[h] << 16);
            v[8 * i + 2 * h + 1] = __uint_as_float(uu[h] & 0xffff0000u);
          }
        }
        stage_block_t(v, (b >> 2) & 1, xs + (size_t)t * d + (size_t)b * MOE_QK, ss + (size_t)t * nb + b);
      }
    }
  }
  __syncthreads();
  if (sh.abort) {
    if (tid == 0) mbar_wait(&sh.xbar, 0u, W.err, 27, W.wait_ns);   // no copy may land after the CTA exits
    return;
  }

  // with the block's dense MLP: expert index E, one more slot per token (s = T k + t), weight 1
  const int Sr = T * k;
  const bool dense = dense_gu != nullptr;
  if (dense)
    for (int t = tid; t < T; t += blockDim.x) {
      sh.ids[Sr + t] = E;
      sh.w[Sr + t] = 1.f;
    }
  __syncthreads();
  const int S = Sr + (dense ? T : 0);
  const int upe_g = f / kUnit, upe_d = d / kUnit;
  // the stable counting sort of the slots by expert, over the whole CTA (its scratch: the
  // reduction buffers, unused until the GEMVs)
  cta_permutation_small<kFMaxSlots / 32, kFMaxE / 32>(sh.ids, S, E + (dense ? 1 : 0), sh.counts, sh.offsets, sh.perm,
                                                     sh.inv, sh.act, &sh.n_act,
                                         reinterpret_cast<int32_t *>(red));
  const int n_act = sh.n_act;
  // each sorted position's token, and the unit-cost prefix over the active experts in closed
  // form: pc[a] = sum over earlier active experts of (kUnitDecode + kUnitToken * T_e)
  for (int p = tid; p < S; p += blockDim.x) {
    const int s = sh.perm[p];
    sh.ptok[p] = s < Sr ? s / k : s - Sr;
  }
  for (int a = tid; a < n_act; a += blockDim.x) sh.pc[a] = kUnitDecode * a + kUnitToken * sh.offsets[sh.act[a]];
  const uint32_t ptot = (uint32_t)(kUnitDecode * n_act + kUnitToken * S);
  if (tid < 4) {
    const uint32_t upe = tid < 2 ? upe_g : upe_d;
    const uint32_t bb = blockIdx.x + (tid & 1);
    if (bb >= gridDim.x) sh.seq[tid] = n_act * (int)upe;
    if (tid == 0) sh.pc[n_act] = (int)ptot;
  }
  __syncthreads();
  // this CTA's unit ranges: boundary j lies in the cost interval of exactly one active expert
  for (int a = tid; a < n_act; a += blockDim.x) {
    const int c = kUnitDecode + kUnitToken * sh.counts[sh.act[a]];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t upe = j < 2 ? upe_g : upe_d;
      const uint32_t xb = upe * ptot * (blockIdx.x + (j & 1)) / gridDim.x;   // < 2^32 for d <= 4096
      const uint32_t lo = upe * (uint32_t)sh.pc[a], hi = upe * (uint32_t)sh.pc[a + 1];
      if (xb >= lo && xb < hi) {
        const uint32_t inexp = (xb - lo + (uint32_t)c - 1u) / (uint32_t)c;
        sh.seq[j] = a * (int)upe + (int)(inexp < upe ? inexp : upe);
      }
    }
  }
  __syncthreads();

  // ---------------------------------------------------------------- producer warp
  if (wq == nwc) {
    // in a layer stack, this CTA's row of the next layer's router moves into L2 while this
    // layer runs (rows are 16-byte aligned: d is a multiple of 32)
    if (next_router_w != nullptr && lane == 1)
      for (int e = blockIdx.x; e < E; e += gridDim.x) bulk_prefetch_l2(next_router_w + (size_t)e * d, (uint32_t)d * 4u);
    if (lane == 0) {
      const uint64_t pol = l2_evict_first_policy();   // expert weights are read once per call
      FWalk wk;
      wk.init(sh.seq, upe_g, upe_d);
      int it = 0;
      for (; !wk.done(); ++it) {
        const int slot = it % kFStages;
        if (it >= kFStages &&
            !wait_phase(&sh.empty[slot], (uint32_t)(it / kFStages - 1) & 1u, &sh.abort, W.err, 24, W.wait_ns))
          break;
        const FChunk c = wk.cur(upe_g, upe_d);
        const int e = sh.act[c.a];
        uint8_t *dst = smem + (size_t)slot * stage_bytes;
        if (!c.down) {
          const uint8_t *base = e < E ? gate_up_q4 + (size_t)e * 2 * f * rb_g : dense_gu;
          const uint32_t bytes = (uint32_t)(c.n * kUnit) * rb_g;
          mbar_arrive_expect_tx(&sh.full[slot], 2u * bytes);
          bulk_g2s_hint(dst, base + (size_t)c.r0 * rb_g, bytes, &sh.full[slot], pol);
          bulk_g2s_hint(dst + kPairs * rb_g, base + (size_t)(f + c.r0) * rb_g, bytes, &sh.full[slot], pol);
        } else {
          const uint32_t bytes = (uint32_t)(c.n * kUnit) * rb_d;
          mbar_arrive_expect_tx(&sh.full[slot], bytes);
          const uint8_t *dbase = e < E ? down_q4 + (size_t)e * d * rb_d : dense_dn;
          bulk_g2s_hint(dst, dbase + (size_t)c.r0 * rb_d, bytes, &sh.full[slot], pol);
        }
        wk.advance(c.n, sh.seq, upe_g, upe_d);
      }
      // every copy issued has landed before this warp leaves (at once unless the call aborted)
      for (int q = it - 1; q >= 0 && q >= it - kFStages; --q)
        mbar_wait(&sh.full[q % kFStages], (uint32_t)(q / kFStages) & 1u, W.err, 28, W.wait_ns);
    }
    return;
  }

  if (blockIdx.x == 0 && wq < nwc) {   // routing copies for the debug readers
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
  // Compute warps multiply a staged chunk into one of two reduction buffers and move on; the
  // epilogue warp turns a full buffer into h (GeGLU) or per-slot outputs and hands it back.
  const bool aligned = (nb % kGran) == 0;
  const int n_items = G;
  const int P = kDnParts;
  int pass = 0;
  if (wq < nwc) {
    int hw0 = 0, hw1 = 0;   // sorted positions whose hidden vectors are staged in hs
    FWalk wk;
    wk.init(sh.seq, upe_g, upe_d);
    for (int it = 0; !wk.done(); ++it) {
      const FChunk c = wk.cur(upe_g, upe_d);
      const int slot = it % kFStages;
      const bool okw = wait_phase(&sh.full[slot], (uint32_t)(it / kFStages) & 1u, &sh.abort, W.err, 22, W.wait_ns);
      const int e = sh.act[c.a];
      const int cnt = sh.counts[e];
      const int off = sh.offsets[e];
      const uint8_t *st = smem + (size_t)slot * stage_bytes;
      if (!c.down) {
        for (int g0 = 0; g0 < cnt; g0 += kTXg, ++pass) {
          const int ng = min(kTXg, cnt - g0);
          const int b = pass & 1;
          if (pass >= 2) named_sync(kBarEmpty0 + b, nteam);
          float *red_b = red + (size_t)b * red_half;
          const int32_t *pt = sh.ptok + off + g0;
          const int first = wq;
          if (okw) {
            if (aligned) {
              switch (ng) {
                case 1: gu_pass<1, true>(st, rb_g, nb, n_items, nwc, first, d, xs, ss, pt, red_b); break;
                case 2: gu_pass<2, true>(st, rb_g, nb, n_items, nwc, first, d, xs, ss, pt, red_b); break;
                case 3: gu_pass<3, true>(st, rb_g, nb, n_items, nwc, first, d, xs, ss, pt, red_b); break;
                default: gu_pass<4, true>(st, rb_g, nb, n_items, nwc, first, d, xs, ss, pt, red_b); break;
              }
            } else {
              switch (ng) {
                case 1: gu_pass<1, false>(st, rb_g, nb, n_items, nwc, first, d, xs, ss, pt, red_b); break;
                case 2: gu_pass<2, false>(st, rb_g, nb, n_items, nwc, first, d, xs, ss, pt, red_b); break;
                case 3: gu_pass<3, false>(st, rb_g, nb, n_items, nwc, first, d, xs, ss, pt, red_b); break;
                default: gu_pass<4, false>(st, rb_g, nb, n_items, nwc, first, d, xs, ss, pt, red_b); break;
              }
            }
          }
          named_arrive(kBarFull0 + b, nteam);
        }
      } else {
        if (off < hw0 || off + cnt > hw1) {
          // stage the hidden vectors of the slots from this expert on, up to the end of this
          // CTA's last expert or the window's capacity
          named_sync(kBarCompute, nct);   // every compute warp is done with the previous window
          const int a_last = (sh.seq[3] - 1) / upe_d;
          const int e_last = sh.act[a_last];
          hw0 = off;
          hw1 = min(sh.offsets[e_last] + sh.counts[e_last], off + hcap);
          const int nblk = okw ? (hw1 - hw0) * nbf : 0;
          for (int blk = tid; blk < nblk; blk += nct) {
            const int i = blk / nbf, cb = blk - i * nbf;
            float v[MOE_QK];
            // the block's values as other CTAs' epilogues (or this one's) store them
            if (!poll_tagged32(W.htag + (size_t)sh.perm[hw0 + i] * f + (size_t)cb * MOE_QK, sh.tag, v, &sh.abort,
                               W.err, W.wait_ns))
              break;
            stage_block_t(v, 0, hs + (size_t)i * f + (size_t)cb * MOE_QK, hbk + (size_t)i * nbf + cb);
          }
          named_sync(kBarCompute, nct);
        }
        const int nr = c.n * kUnit;
        for (int g0 = 0; g0 < cnt; g0 += kTX, ++pass) {
          const int ng = min(kTX, cnt - g0);
          const int b = pass & 1;
          if (pass >= 2) named_sync(kBarEmpty0 + b, nteam);
          float *red_b = red + (size_t)b * red_half;
          const int rel0 = off + g0 - hw0;
          const int first = wq;
          if (okw) {
            if ((nbf & 1) == 0) {
              switch (ng) {
                case 1: dn_pass<1, true>(st, rb_d, nbf, P, nwc, first, nr, f, hs, hbk, rel0, red_b); break;
                case 2: dn_pass<2, true>(st, rb_d, nbf, P, nwc, first, nr, f, hs, hbk, rel0, red_b); break;
                case 3: dn_pass<3, true>(st, rb_d, nbf, P, nwc, first, nr, f, hs, hbk, rel0, red_b); break;
                default: dn_pass<4, true>(st, rb_d, nbf, P, nwc, first, nr, f, hs, hbk, rel0, red_b); break;
              }
            } else {
              switch (ng) {
                case 1: dn_pass<1, false>(st, rb_d, nbf, P, nwc, first, nr, f, hs, hbk, rel0, red_b); break;
                case 2: dn_pass<2, false>(st, rb_d, nbf, P, nwc, first, nr, f, hs, hbk, rel0, red_b); break;
                case 3: dn_pass<3, false>(st, rb_d, nbf, P, nwc, first, nr, f, hs, hbk, rel0, red_b); break;
                default: dn_pass<4, false>(st, rb_d, nbf, P, nwc, first, nr, f, hs, hbk, rel0, red_b); break;
              }
            }
          }
          named_arrive(kBarFull0 + b, nteam);
        }
      }
      if (lane == 0) mbar_arrive(&sh.empty[slot]);   // this warp's last read of the stage
      wk.advance(c.n, sh.seq, upe_g, upe_d);
    }
    for (int q = pass < 2 ? 0 : pass - 2; q < pass; ++q) named_sync(kBarEmpty0 + (q & 1), nteam);
  } else {
    // the epilogue warp: the same sequence of chunks and passes
    FWalk wk;
    wk.init(sh.seq, upe_g, upe_d);
    while (!wk.done()) {
      const FChunk c = wk.cur(upe_g, upe_d);
      const int e = sh.act[c.a];
      const int cnt = sh.counts[e];
      const int off = sh.offsets[e];
      const int step = c.down ? kTX : kTXg;
      for (int g0 = 0; g0 < cnt; g0 += step, ++pass) {
        const int ng = min(step, cnt - g0);
        const int b = pass & 1;
        named_sync(kBarFull0 + b, nteam);
        const float *red_b = red + (size_t)b * red_half;
        if (!sh.abort) {
          if (!c.down) {
            // h = gelu(gate) * up; the partials of the G work items summed in order
            const int np = c.n * kUnit, sh_np = np == 16 ? 4 : 3;
            for (int itm = lane; itm < np * ng; itm += 32) {
              const int i = itm >> sh_np, pp = itm & (np - 1);
              float g = 0.f, uu = 0.f;
              for (int q = 0; q < n_items; ++q) {
                const float2 v = *reinterpret_cast<const float2 *>(red_b + (((size_t)q * kTX + i) * kPairs + pp) * 2);
                g += v.x;
                uu += v.y;
              }
              const float hv = gelu_tanh_f(g) * uu;
              const size_t hi = (size_t)sh.perm[off + g0 + i] * f + c.r0 + pp;
              st_relaxed_u64(W.htag + hi, tag_word(sh.tag, hv));
              W.h[hi] = hv;   // the plain copy for the debug reader
            }
          } else {
            const int nr = c.n * kUnit;
            for (int i2 = lane; i2 < nr * ng; i2 += 32) {
              const int i = i2 / nr, row = i2 - i * nr;
              float s = 0.f;
              for (int pt = 0; pt < P; ++pt) s += red_b[((size_t)pt * kTX + i) * kDnRows + row];
              st_relaxed_u64(W.ytag + (size_t)sh.perm[off + g0 + i] * d + c.r0 + row, tag_word(sh.tag, s));
            }
          }
        }
        named_arrive(kBarEmpty0 + b, nteam);
      }
      wk.advance(c.n, sh.seq, upe_g, upe_d);
    }
  }
  // ---------------------------------------------------------------- phase 4: combine
  // no grid barrier: every term is polled (bounded) from its launch-tagged word, eight slots'
  // words in flight at once, and summed in j order
  if (sh.abort) return;
  const int ti = wq < nwc ? tid : nct + lane;
  const int r0 = (int)((long long)d * blockIdx.x / gridDim.x), r1 = (int)((long long)d * (blockIdx.x + 1) / gridDim.x);
  const int nr = r1 - r0;
  const uint32_t tag = sh.tag;
  for (int i2 = ti; i2 < nr * T; i2 += nteam) {
    const int t = i2 / nr, r = r0 + i2 % nr;
    float s = 0.f;
    float y[8];
    for (int j0 = 0; j0 < k; j0 += 8) {
      const int n = min(8, k - j0);
      if (!poll_tagged(W.ytag + (size_t)(t * k + j0) * d + r, (size_t)d, n, tag, y, &sh.abort, W.err, W.wait_ns))
        return;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (q < n) {
          const int slotid = t * k + j0 + q;
          s += sh.w[slotid] * __ldg(expert_scale + sh.ids[slotid]) * y[q];
        }
      }
    }
    if (dense) {   // the dense MLP's output, weight 1
      if (!poll_tagged(W.ytag + (size_t)(Sr + t) * d + r, (size_t)d, 1, tag, y, &sh.abort, W.err, W.wait_ns)) return;
      s += y[0];
    }
    out[(size_t)t * d + r] = accumulate ? out[(size_t)t * d + r] + s : s;
  }
}

}  // namespace

// Dynamic shared memory of k_moe_decode for these shapes, with the sizes of its regions.
// (the reduction buffers also hold the permutation's scratch in phase 1)
struct FusedSmem {
  uint32_t stage_bytes, x_bytes, red_half;   // red_half in floats
  size_t total;
};
static FusedSmem fused_smem(int T, int d, int f) {
  const int nb = d / MOE_QK, nbf = f / MOE_QK;
  const int G = (nb + kGran - 1) / kGran;
  FusedSmem r;
  const size_t sg = 2u * kPairs * (size_t)nb * MOE_QBYTES + 16u;
  const size_t sd = (size_t)kDnRows * nbf * MOE_QBYTES + 16u;
  r.stage_bytes = (uint32_t)(((sg > sd ? sg : sd) + 15u) & ~(size_t)15u);
  const size_t xg = (size_t)T * (2 * d + 8 * nb), xh = (size_t)T * (2 * f + 8 * nbf);
  r.x_bytes = (uint32_t)(((xg > xh ? xg : xh) + 15u) & ~(size_t)15u);
  const size_t rg = (size_t)G * kPairs * kTX * 2, rd = (size_t)kDnParts * kTX * kDnRows;
  r.red_half = (uint32_t)(rg > rd ? rg : rd);
  r.total = (size_t)kFStages * r.stage_bytes + r.x_bytes + (size_t)2 * r.red_half * 4 + 128;
  return r;
}

bool moe_fused_decode_supported(int T, int d, int f, int E, int k, bool dense) {
  const int G = (d / MOE_QK + kGran - 1) / kGran;
  const int S = T * k + (dense ? T : 0), Eall = E + (dense ? 1 : 0);
  return T >= 1 && T <= kFMaxT && S <= kFMaxSlots && Eall <= kFMaxE && G <= kMaxGran &&
         fused_smem(T, d, f).total + sizeof(FusedShared) <= 227 * 1024;
}

int moe_launch_fused_decode(const MoeLaunch &L, const MoeWork &W, const void *x, const float *y_prev, float eps,
                            void *x_out, const float *router_w, const float *router_scale,
                            const uint8_t *gate_up_q4, const uint8_t *down_q4, const float *expert_scale, int T,
                            int d, int f, int E, int k, float *out, int num_sms, const uint8_t *dense_gu,
                            const uint8_t *dense_dn, const float *next_router_w) {
  if (!moe_fused_decode_supported(T, d, f, E, k, dense_gu != nullptr)) return -2;
  const FusedSmem fs = fused_smem(T, d, f);
  static unsigned long long smem_ok[2] = {0ull, 0ull};   // per device, per kernel
  const bool norm_in = y_prev != nullptr;
  if (!moe_allow_dyn_smem(reinterpret_cast<const void *>(norm_in ? k_moe_decode<true> : k_moe_decode<false>),
                          &smem_ok[norm_in]))
    return -1;
  const int G = (d / MOE_QK + kGran - 1) / kGran;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(num_sms);
  cfg.blockDim = dim3(32 * (fused_compute_warps(G) + 2));
  cfg.dynamicSmemBytes = fs.total;
  cfg.stream = L.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  moe_prof_mark(L.stream, MOE_K_FUSED, true);
  const cudaError_t e =
      cudaLaunchKernelEx(&cfg, norm_in ? k_moe_decode<true> : k_moe_decode<false>,
                         static_cast<const __nv_bfloat16 *>(x), y_prev, eps, static_cast<__nv_bfloat16 *>(x_out),
                         router_w, router_scale, gate_up_q4, down_q4, expert_scale, T, d, f, E, k, out,
                         fs.stage_bytes, fs.x_bytes, fs.red_half, W, L.accumulate ? 1 : 0, dense_gu, dense_dn,
                         next_router_w);
  if (e != cudaSuccess) return -1;
  moe_prof_count(1);
  moe_prof_mark(L.stream, MOE_K_FUSED, false);
  return 0;
}
