// moe_gemv_core.cuh -- device building blocks of the Q4_0 decode GEMVs, shared by the
// separate-kernel path (moe_gemv.cu) and the fused decode kernel (moe_decode.cu).
//
// Arithmetic: a Q4_0 weight is (q - 8) * d. Activations are int16, block-scaled by a power
// of two (moe_common.cuh). The low nibbles of a 4-byte code word, masked in place, are four
// bytes q; the high nibbles, masked in place, are four bytes 16 q. The integer dot-product
// instruction dp2a multiplies two int16 activations by two code bytes and adds both to an
// int32 accumulator, exactly. Per block and token: r = sum(q a) - 8 sum(a), an exact
// integer with |r| < 2^23, and the row accumulator gets d * 2^sigma * r (one FP32 rounding).
#pragma once

#include "moe_common.cuh"

namespace {

constexpr int kGran = 8;        // blocks per granule: 144 bytes, 16-byte aligned in aligned rows
constexpr int kMaxGran = 16;    // gate_up: one warp per granule, d <= 4096
constexpr int kPairs = 16;      // row pairs (gate c, up f + c) per gate_up chunk
constexpr int kUnit = 8;        // rows (or row pairs) per scheduling unit
constexpr int kTX = 4;          // tokens per pass over a staged chunk
constexpr int kGuStagesMax = 3;
constexpr int kDnRows = 128;    // rows per down chunk
constexpr int kDnThreads = 256; // 4 warps x 32 rows, 2 parts of the row's blocks
constexpr int kDnStagesMax = 4;
constexpr int kSmemBudget = 222 * 1024;

__device__ __forceinline__ float gelu_tanh_f(float z) {
  const float c = 0.7978845608028654f;   // sqrt(2/pi)
  return 0.5f * z * (1.0f + tanhf(c * (z + 0.044715f * z * z * z)));
}

// c + a.h0 * b.byte0 + a.h1 * b.byte1 (lo) or bytes 2, 3 (hi): a two signed 16-bit values,
// b four unsigned bytes.
__device__ __forceinline__ int dp2a_lo(uint32_t a, uint32_t b, int c) {
  int r;
  asm("dp2a.lo.s32.u32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}
__device__ __forceinline__ int dp2a_hi(uint32_t a, uint32_t b, int c) {
  int r;
  asm("dp2a.hi.s32.u32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}
// One code word against 8 activations in the word order: lo = w & 0x0F0F0F0F (codes of
// elements 4i..4i+3), hi = w & 0xF0F0F0F0 (16 x codes of 16+4i..16+4i+3).
__device__ __forceinline__ void dot8i(uint32_t lo, uint32_t hi, const uint4 &xv, int &al, int &ah) {
  al = dp2a_lo(xv.x, lo, al);
  al = dp2a_hi(xv.y, lo, al);
  ah = dp2a_lo(xv.z, hi, ah);
  ah = dp2a_hi(xv.w, hi, ah);
}
// y += d * 2^sigma * (al + ah / 16) where al started at -8 sum(a): exact integer, one rounding
__device__ __forceinline__ float block_finish(float y, float d, float scale, int al, int ah) {
  return fmaf(d * scale, (float)(al + (ah >> 4)), y);
}

struct Blk {
  float d;
  uint32_t q[4];
};

// One 18-byte block at a 2-byte aligned shared-memory byte offset (five 32-bit loads).
__device__ __forceinline__ Blk load_blk(const uint8_t *smem, uint32_t o) {
  const uint32_t a = o & ~3u;
  const uint32_t sh = (o & 3u) * 8u;   // 0 or 16
  const uint32_t *wp = reinterpret_cast<const uint32_t *>(smem + a);
  const uint32_t w0 = wp[0], w1 = wp[1], w2 = wp[2], w3 = wp[3], w4 = wp[4];
  Blk b;
  b.d = __half2float(__ushort_as_half((unsigned short)((w0 >> sh) & 0xffffu)));
  const uint32_t s2 = sh + 16u;
  b.q[0] = __funnelshift_rc(w0, w1, s2);
  b.q[1] = __funnelshift_rc(w1, w2, s2);
  b.q[2] = __funnelshift_rc(w2, w3, s2);
  b.q[3] = __funnelshift_rc(w3, w4, s2);
  return b;
}

// Two consecutive blocks from nine words w[0..8]: the first starts on word 0 (scale in its
// low half, codes shifted by 16 bits), the second at byte 18 (scale in the high half of
// word 4, codes in words 5..8).
__device__ __forceinline__ void split_blk2(const uint32_t (&w)[10], Blk &b0, Blk &b1) {
  b0.d = __half2float(__ushort_as_half((unsigned short)(w[0] & 0xffffu)));
#pragma unroll
  for (int i = 0; i < 4; ++i) b0.q[i] = __funnelshift_r(w[i], w[i + 1], 16);
  b1.d = __half2float(__ushort_as_half((unsigned short)(w[4] >> 16)));
#pragma unroll
  for (int i = 0; i < 4; ++i) b1.q[i] = w[5 + i];
}

// Blocks 0, 1 of a 72-byte, 8-byte aligned four-block span: five 64-bit loads at o.
__device__ __forceinline__ void load_blk2_lo(const uint8_t *smem, uint32_t o, Blk &b0, Blk &b1) {
  const uint2 *wp = reinterpret_cast<const uint2 *>(smem + o);
  uint32_t w[10];
#pragma unroll
  for (int i = 0; i < 5; ++i) {
    const uint2 v = wp[i];
    w[2 * i] = v.x;
    w[2 * i + 1] = v.y;
  }
  split_blk2(w, b0, b1);
}

// Blocks 2, 3 of the same span: they start at byte 36 (4-byte aligned): one 32-bit load at
// o + 36 and four 64-bit loads from the 8-byte aligned o + 40.
__device__ __forceinline__ void load_blk2_hi(const uint8_t *smem, uint32_t o, Blk &b0, Blk &b1) {
  uint32_t w[10];
  w[0] = *reinterpret_cast<const uint32_t *>(smem + o + 36);
  const uint2 *wp = reinterpret_cast<const uint2 *>(smem + o + 40);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint2 v = wp[i];
    w[1 + 2 * i] = v.x;
    w[2 + 2 * i] = v.y;
  }
  w[9] = 0u;
  split_blk2(w, b0, b1);
}

struct RingCtl {
  uint64_t full[kDnStagesMax];
};

// Flat split of n units over the grid.
__device__ __forceinline__ void my_units(int n, int &u0, int &u1) {
  u0 = (int)((long long)n * blockIdx.x / gridDim.x);
  u1 = (int)((long long)n * (blockIdx.x + 1) / gridDim.x);
}

__device__ __forceinline__ uint8_t *align128(uint8_t *p) {
  return p + ((128u - (smem_u32(p) & 127u)) & 127u);
}

// ---------------------------------------------------------------- gate_up + GeGLU
//
// CTA = one warp per 144-byte granule of a row (11 warps for d = 2816). Lane = (row pair p,
// half h): rows c0 + p (gate) and f + c0 + p (up), blocks 8 w + 4 h .. + 3. All lanes of a
// warp read the same activations (shared-memory broadcast); the 2 G partials of each row
// are summed in a fixed order at the end of the chunk, where the GeGLU is applied.

struct GuChunk {
  int a, c0, np;   // active-expert index, first row pair, row pairs (8 or 16)
};

__device__ __forceinline__ GuChunk gu_chunk(int u, int u1, int upe) {
  GuChunk c;
  c.a = u / upe;
  c.c0 = (u % upe) * kUnit;
  const int n = (u + 1 < u1 && (u + 1) / upe == c.a) ? 2 : 1;
  c.np = n * kUnit;
  return c;
}

template <int NT>
__device__ __forceinline__ void gu_block(const Blk &bg, const Blk &bu, int b, int nb, const uint16_t *xs,
                                         const ActBlk *ss, int d, float (&yg)[NT], float (&yu)[NT]) {
  int gl[NT], gh[NT], ul[NT], uh[NT];
  float sc[NT];
#pragma unroll
  for (int i = 0; i < NT; ++i) {
    const ActBlk ab = ss[i * nb + b];
    gl[i] = ab.neg8sum; ul[i] = ab.neg8sum; gh[i] = 0; uh[i] = 0; sc[i] = ab.scale;
  }
#pragma unroll
  for (int wi = 0; wi < 4; ++wi) {
    const uint32_t glo = bg.q[wi] & 0x0F0F0F0Fu, ghi = bg.q[wi] & 0xF0F0F0F0u;
    const uint32_t ulo = bu.q[wi] & 0x0F0F0F0Fu, uhi = bu.q[wi] & 0xF0F0F0F0u;
#pragma unroll
    for (int i = 0; i < NT; ++i) {
      const uint4 xv = *reinterpret_cast<const uint4 *>(xs + (size_t)i * d + b * MOE_QK + 8 * wi);
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

template <int NT, bool ALIGNED>
__device__ __forceinline__ void gu_compute(const uint8_t *st, uint32_t rb, int nb, const uint16_t *xs,
                                           const ActBlk *ss, int d, float *red_out /* [NT][2] */) {
  // called by every lane of the warp (rows past the chunk read stale shared memory and are
  // not stored by the caller)
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int p = lane >> 1, h = lane & 1;
  float yg[NT], yu[NT];
#pragma unroll
  for (int i = 0; i < NT; ++i) { yg[i] = 0.f; yu[i] = 0.f; }
  const int b0 = w * kGran + h * 4;
  const uint32_t og = (uint32_t)p * rb + (uint32_t)b0 * MOE_QBYTES;
  const uint32_t ou = (uint32_t)(kPairs + p) * rb + (uint32_t)b0 * MOE_QBYTES;
  int nbl = nb - b0;
  nbl = nbl < 0 ? 0 : (nbl > 4 ? 4 : nbl);
  if (ALIGNED) {
    {
      Blk g0, g1, v0, v1;
      load_blk2_lo(st, og, g0, g1);
      load_blk2_lo(st, ou, v0, v1);
      gu_block<NT>(g0, v0, b0, nb, xs, ss, d, yg, yu);
      gu_block<NT>(g1, v1, b0 + 1, nb, xs, ss, d, yg, yu);
    }
    {
      Blk g2, g3, v2, v3;
      load_blk2_hi(st, og, g2, g3);
      load_blk2_hi(st, ou, v2, v3);
      gu_block<NT>(g2, v2, b0 + 2, nb, xs, ss, d, yg, yu);
      gu_block<NT>(g3, v3, b0 + 3, nb, xs, ss, d, yg, yu);
    }
  } else {
    for (int j = 0; j < nbl; ++j) {
      const Blk g = load_blk(st, og + j * MOE_QBYTES);
      const Blk v = load_blk(st, ou + j * MOE_QBYTES);
      gu_block<NT>(g, v, b0 + j, nb, xs, ss, d, yg, yu);
    }
  }
  // the two halves of a granule sit in adjacent lanes: combine them, even lanes store
#pragma unroll
  for (int i = 0; i < NT; ++i) {
    const float g = yg[i] + __shfl_xor_sync(0xffffffffu, yg[i], 1);
    const float u = yu[i] + __shfl_xor_sync(0xffffffffu, yu[i], 1);
    if (h == 0) {
      red_out[2 * i] = g;
      red_out[2 * i + 1] = u;
    }
  }
}

struct DnChunk {
  int a, r0, nr;
};

__device__ __forceinline__ DnChunk dn_chunk(int u, int u1, int upe) {
  DnChunk c;
  c.a = u / upe;
  c.r0 = (u % upe) * kUnit;
  int n = 1;
  while (n < kDnRows / kUnit && u + n < u1 && (u + n) / upe == c.a) ++n;
  c.nr = n * kUnit;
  return c;
}

// One down-row block against NT slots' staged hidden vectors, accumulated into y[].
template <int NT>
__device__ __forceinline__ void dn_block_acc(const Blk &bk, int b, int nbf, const uint16_t *hs, const ActBlk *hb,
                                             int f, float (&y)[NT]) {
  int al[NT], ah[NT];
  float sc[NT];
#pragma unroll
  for (int i = 0; i < NT; ++i) {
    const ActBlk ab = hb[i * nbf + b];
    al[i] = ab.neg8sum; ah[i] = 0; sc[i] = ab.scale;
  }
#pragma unroll
  for (int wi = 0; wi < 4; ++wi) {
    const uint32_t lo = bk.q[wi] & 0x0F0F0F0Fu, hi = bk.q[wi] & 0xF0F0F0F0u;
#pragma unroll
    for (int i = 0; i < NT; ++i)
      dot8i(lo, hi, *reinterpret_cast<const uint4 *>(hs + (size_t)i * f + b * MOE_QK + 8 * wi), al[i], ah[i]);
  }
#pragma unroll
  for (int i = 0; i < NT; ++i) y[i] = block_finish(y[i], bk.d, sc[i], al[i], ah[i]);
}

// Down rows of a staged chunk (nr rows) for NT slots, by every warp of the CTA: work items
// (32-row group, part) with the row's blocks split in MOE_DN_PARTS parts exactly as the fused
// decode kernel splits them (block pairs first when the row has an even number of blocks,
// leftovers one each to the first parts; otherwise contiguous ranges); lane = row.
// red_out[(part * kTX + i) * kDnRows + row].
template <int NT>
__device__ __forceinline__ void dn_compute(const uint8_t *st, uint32_t rb, int nbf, int nr, const uint16_t *hs,
                                           const ActBlk *hb, int f, float *red_out) {
  constexpr int P = MOE_DN_PARTS;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int item = w; item < (kDnRows / 32) * P; item += nw) {
    const int grp = item % (kDnRows / 32), part = item / (kDnRows / 32);
    const int row = grp * 32 + lane;
    if (row >= nr) continue;
    float y[NT];
#pragma unroll
    for (int i = 0; i < NT; ++i) y[i] = 0.f;
    const uint32_t orow = (uint32_t)row * rb;
    if ((nbf & 1) == 0) {
      const int per = nbf / (2 * P);   // block pairs per part
      for (int b = 2 * part * per; b < 2 * (part + 1) * per; ++b)
        dn_block_acc<NT>(load_blk(st, orow + (uint32_t)b * MOE_QBYTES), b, nbf, hs, hb, f, y);
      for (int b = 2 * P * per + part; b < nbf; b += P)
        dn_block_acc<NT>(load_blk(st, orow + (uint32_t)b * MOE_QBYTES), b, nbf, hs, hb, f, y);
    } else {
      for (int b = part * nbf / P; b < (part + 1) * nbf / P; ++b)
        dn_block_acc<NT>(load_blk(st, orow + (uint32_t)b * MOE_QBYTES), b, nbf, hs, hb, f, y);
    }
#pragma unroll
    for (int i = 0; i < NT; ++i) red_out[((size_t)part * kTX + i) * kDnRows + row] = y[i];
  }
}

}  // namespace
