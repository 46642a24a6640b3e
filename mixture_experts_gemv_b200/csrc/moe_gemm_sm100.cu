// moe_gemm_sm100.cu -- prefill path: grouped GEMMs of the routed experts on the sm_100
// tensor cores (tcgen05.mma, accumulators in TMEM), with the Q4_0 weights dequantised to
// bf16 in shared memory and GELU-tanh gating fused into the gate_up epilogue.
//
// Page "Gemma 4 26B-A4B it QAT Q4_0 ... NInfer v3 artifact", "What is inside": expert-major
// Q4_0 [gate; up] (2 x 704 rows) and down (2,816 rows) multiplied in place. With the slots
// of expert e sorted together (stable permutation) the layer is, per expert, two GEMMs:
//   H_e = gelu_tanh(X_e Wg_e^T) * (X_e Wu_e^T)      [M_e x f]
//   Y_e = H_e Wd_e^T                                [M_e x d]
// followed by out[t] = sum_j w_tj * s_e * Y[slot(t, j)] in j order.
//
// Layout: the routed rows of each expert are padded to whole 128-row tiles; tile i of the
// tile list covers padded rows [128 i, 128 i + 128). A work item is one n-tile of either one
// row tile (M = 128) or a pair of consecutive tiles of one expert (M = 256 as two 128-row MMA
// halves sharing the B tile, so the decode work per flop halves); the shapes per call are
// chosen by the launcher (GemmCfg below).
// The A tile of a K step lands in the 128-byte swizzled K-major layout: gate_up's producers
// gather the tokens' rows of x with 16-byte asynchronous copies, eight lanes per 128-byte row
// segment (zero-filled past the expert's rows); down's 128 x 64 tiles of the padded h come by
// 2-D TMA copies. The raw Q4_0 bytes of the B rows come by TMA too: the weight matrix is seen
// as lines of 4 consecutive rows (a line's length, 4 x 18 K / 32 bytes, is a multiple of 16
// for every K that is a multiple of 64), and one box of 48 bytes x 32 lines fetches, for one
// residue r of the row index mod 4, the K step's two blocks (36 bytes, which start at most 12
// bytes past a 16-byte boundary) of 32 rows. The weights never exist in bf16 in global
// memory: the producers decode (q - 8) * d from the staged bytes and write the swizzled
// K-major B tile that tcgen05.mma reads. B tile row 32 r + i holds weight row 4 i + r of the
// item (so a warp's lanes read and write shared memory without bank conflicts); the
// epilogue puts the columns back in weight-row order.
//
// One CTA per SM, persistent over work items, warp-specialised:
//   warps 0-3  epilogue: tcgen05.ld of the FP32 accumulators (lane = row)
//   warp  4    TMEM allocation; lane 0 issues tcgen05.mma (M = 128, N = 256 or 128, K = 16,
//              one per 16-wide K slice and item half)
//   warps 5-20 producers in two groups taking alternate K steps: A copies (gate_up) or the
//              TMA issue (down), the raw-weight TMA issue, Q4_0 -> bf16 dequantisation for B
// Shared-memory stages are handed over with mbarriers (every wait is time-bounded); where two
// accumulators fit in TMEM's 512 columns the epilogue of one item overlaps the next item's MMAs.
// The prefill router product runs in this file too (k_split_router, k_router_tc below).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "moe_common.cuh"

namespace {

constexpr int BM = 128, BK = 64;
static_assert(BM == MOE_GEMM_TILE_ROWS, "the tile list is built with this tile height");
constexpr int kMaxStages = 5;
constexpr int kMaxRawSlots = 3;
constexpr int kEpiWarps = 4;
constexpr int kMmaWarp = 4;
constexpr int kProdGroups = 2;                                // producer groups take alternate K steps
constexpr int kProdWarps = 8 * kProdGroups;
constexpr int kProdThreads = kProdWarps * 32;
constexpr int kGroupThreads = kProdThreads / kProdGroups;     // one (row, block) of the B tile each
constexpr int kThreads = (kEpiWarps + 1 + kProdWarps) * 32;
constexpr uint32_t kTileBytes = BM * BK * 2;                  // 16 KB: one 128-row A half
constexpr int kSubRows = 32;                                   // lines of one raw box (one residue mod 4)
constexpr int kRawBoxes = 8;                                   // raw boxes per K step: one per producer warp

// UMMA instruction descriptor, kind::f16: D FP32 (bits 4-5 = 1), A and B bf16 (bits 7-9,
// 10-12 = 1), both K-major (bits 15, 16 = 0), N >> 3 in bits 17-22, M >> 4 in bits 24-28.
constexpr uint32_t umma_idesc(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

// Per GEMM:
//  gate_up: N = 256 columns, the 128 gate rows c0 .. c0+127 and the matching 128 up rows (rows
//    past f are zero); measured: one tcgen05.mma of N = 256 does twice the work of an N = 128
//    one in about the same pipeline time. A rows are gathered by the producers.
//  down: N = 256 (or 128) output columns; A, the padded h, comes by TMA.
//  Each GEMM comes in shapes BN x HALVES (MMA N, and M = 128 HALVES): an item is one row tile
//    (HALVES = 1) or a tile pair of one expert (HALVES = 2, the halves sharing the decoded B
//    tile, so the decode work per flop halves); BN = 256 decodes one B row a producer thread
//    (down: d a multiple of 256), BN = 128 one block of a B row. TMEM holds two accumulator
//    buffers where 2 x HALVES x BN <= 512 columns (the epilogue of an item overlaps the next
//    item's MMAs), else one.
template <bool GATEUP, int BN, int HALVES>
struct GemmCfg {
  static constexpr bool kRowDec = BN == 256;                      // one B row (both blocks) a thread
  static constexpr int kBN = BN;                                  // MMA N
  static constexpr int kHalves = HALVES;                          // M = 128 kHalves
  static constexpr int kAccBufs = 2 * HALVES * BN <= 512 ? 2 : 1;  // accumulator buffers in TMEM
  static constexpr int kStages = (HALVES == 2 && BN == 128) ? 4 : 3;
  // group steps the copies run ahead of the decode
  static constexpr int kAhead = 1;
  static constexpr uint32_t kBBytes = (uint32_t)kBN * BK * 2;
  static constexpr uint32_t kBOff = kHalves * kTileBytes;        // B tile after the A halves
  static constexpr uint32_t kStageBytes = kBOff + kBBytes;
  // raw box width: gate_up, a row's whole 48-byte window (box w = part w / 4, residue w % 4);
  // down, 32 bytes holding one block (box w = residue w % 4, block w / 4: bytes 0-31 of the
  // window hold block 0, bytes 16-47 block 1)
  static constexpr uint32_t kBoxW = kRowDec ? 48 : 32;
  static constexpr uint32_t kSubBytes = kSubRows * kBoxW;
  static constexpr uint32_t kRawSlotBytes = kRawBoxes * kSubBytes;
  // raw ring slots per producer group (shared memory: 216-225 KB with the stages)
  static constexpr int kRawSlots = (HALVES == 2 && BN == 256) ? 1 : (BN == 256 ? 3 : 2);
  static constexpr uint32_t kTmemCols = kAccBufs * kHalves * kBN;
  static constexpr int kSmemBytes = kStages * kStageBytes + kProdGroups * kRawSlots * kRawSlotBytes + 1024;
  static constexpr uint32_t kIdesc = umma_idesc(kBN);
  static_assert(kAhead * kProdGroups <= kStages, "the prologue's stages must be free");
  static_assert(kStages <= kMaxStages && kRawSlots <= kMaxRawSlots && kTmemCols <= 512, "limits");
  static_assert(kSmemBytes <= 231 * 1024, "one CTA per SM, with the static barriers");
  // the producer group's threads: one B row each (gate_up), or one block of a B row (down)
  static_assert(kBN * (kRowDec ? 1 : 2) == kGroupThreads, "producer threads cover the B tile");
};

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle (layout type 2),
// rows of 128 bytes in 8-row atoms of 1024 bytes (stride byte offset 1024), version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}

struct GemmBars {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t raw[kProdGroups][kMaxRawSlots];   // a producer group's raw ring slot has landed (TMA bytes)
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint32_t tmem_base;
  int abort_flag;
};

// ---------------------------------------------------------------- PTX wrappers

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
// 2-D tiled TMA load (no multicast), completion on `bar` in bytes.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int c0, int c1, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// 16-byte asynchronous copy global -> shared; bytes past src_bytes (0 or 16) are zero-filled.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld4(uint32_t taddr, uint32_t (&r)[4]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// GELU, tanh form, with the hardware tanh approximation (`tanh.approx.f32`, absolute error
// about 2^-11): h is rounded to bf16 right after (relative step 2^-8), and this path's outputs
// are held to 2e-2 relative to an FP64 evaluation of the layer; it frees the epilogue's issue
// slots for the producer warps that share the SM's schedulers.
__device__ __forceinline__ float gelu_tanh_f(float z) {
  const float c = 0.7978845608028654f;   // sqrt(2/pi)
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(c * (z + 0.044715f * z * z * z)));
  return 0.5f * z * (1.0f + t);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t *>(&h);
}

// ---------------------------------------------------------------- Q4_0 -> bf16

// Four consecutive code bytes (one word) -> the bf16 pairs (q - 8) * d of their low nibbles
// (lo01: bytes 0,1; lo23: bytes 2,3) and high nibbles (hi01, hi23). A code q is first made
// the bf16 value 128 + q by OR-ing it into the mantissa of 128 (exact), then 136 is
// subtracted (exact) and the result is multiplied by d (one rounding).
// The four code bytes may straddle two words: bytes 0, 1 are sel01 of wa and bytes 2, 3 are
// sel23 of wb (aligned: wa = wb = w, 0x4140 / 0x4342; two bytes past: bytes 2, 3 of w[i] and
// 0, 1 of w[i + 1], 0x4342 / 0x4140).
__device__ __forceinline__ void dq_word2(uint32_t wa, uint32_t wb, uint32_t sel01, uint32_t sel23,
                                         __nv_bfloat162 d2, uint32_t &lo01, uint32_t &lo23, uint32_t &hi01,
                                         uint32_t &hi23) {
  const uint32_t v01 = __byte_perm(wa, 0u, sel01);    // [b0, 0, b1, 0]
  const uint32_t v23 = __byte_perm(wb, 0u, sel23);    // [b2, 0, b3, 0]
  const uint32_t kMag = 0x43004300u;                  // bf16 (128, 128)
  const uint32_t l01 = (v01 & 0x000F000Fu) | kMag;
  const uint32_t l23 = (v23 & 0x000F000Fu) | kMag;
  const uint32_t h01 = ((v01 >> 4) & 0x000F000Fu) | kMag;
  const uint32_t h23 = ((v23 >> 4) & 0x000F000Fu) | kMag;
  const __nv_bfloat162 c136 = __halves2bfloat162(__ushort_as_bfloat16((unsigned short)0x4308),
                                                 __ushort_as_bfloat16((unsigned short)0x4308));
  auto cv = [&](uint32_t x) -> uint32_t {
    __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162 *>(&x);
    v = __hmul2(__hsub2(v, c136), d2);
    return *reinterpret_cast<const uint32_t *>(&v);
  };
  lo01 = cv(l01);
  lo23 = cv(l23);
  hi01 = cv(h01);
  hi23 = cv(h23);
}

__device__ __forceinline__ void dq_word(uint32_t w, __nv_bfloat162 d2, uint32_t &lo01, uint32_t &lo23,
                                        uint32_t &hi01, uint32_t &hi23) {
  dq_word2(w, w, 0x4140u, 0x4342u, d2, lo01, lo23, hi01, hi23);
}

// One block -- fp16 scale bits and its four code words -- into its 4 swizzled 16-byte chunks
// (cbase .. cbase + 3) of the B tile row at rowbase (x = the row's swizzle phase). With SHIFT
// the block's code word i is bytes 2, 3 of q[i] and 0, 1 of q[i + 1] (q[0 .. 4]).
template <bool SHIFT>
__device__ __forceinline__ void store_blk_bf16(uint32_t dbits, const uint32_t *q, uint32_t rowbase, uint32_t x,
                                               int cbase) {
  const __nv_bfloat162 d2 = __float2bfloat162_rn(__half2float(__ushort_as_half((unsigned short)(dbits & 0xffffu))));
  uint32_t lo[8], hi[8];   // element pairs (0,1),(2,3),...,(14,15) and (16,17),...,(30,31)
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (SHIFT) dq_word2(q[i], q[i + 1], 0x4342u, 0x4140u, d2, lo[2 * i], lo[2 * i + 1], hi[2 * i], hi[2 * i + 1]);
    else dq_word(q[i], d2, lo[2 * i], lo[2 * i + 1], hi[2 * i], hi[2 * i + 1]);
  }
  st_shared_v4(rowbase + (((uint32_t)(cbase + 0) ^ x) << 4), lo[0], lo[1], lo[2], lo[3]);   // elements 0-7
  st_shared_v4(rowbase + (((uint32_t)(cbase + 1) ^ x) << 4), lo[4], lo[5], lo[6], lo[7]);   // 8-15
  st_shared_v4(rowbase + (((uint32_t)(cbase + 2) ^ x) << 4), hi[0], hi[1], hi[2], hi[3]);   // 16-23
  st_shared_v4(rowbase + (((uint32_t)(cbase + 3) ^ x) << 4), hi[4], hi[5], hi[6], hi[7]);   // 24-31
}

// A row's 48-byte window w[12] of a K step whose two blocks start at word WB (byte 4 WB):
// block 0 = scale in the low half of word WB, codes two bytes further (each code word spans
// two window words); block 1 = scale in the high half of word WB + 4, codes in words
// WB + 5 .. WB + 8. BLK selects the blocks decoded: 1, 2 or 3 (both).
template <int WB, int BLK>
__device__ __forceinline__ void dec_window(const uint32_t (&w)[12], uint32_t rowbase, uint32_t x) {
  if (BLK & 1) store_blk_bf16<true>(w[WB], w + WB, rowbase, x, 0);    // codes from byte 2 of word WB
  if (BLK & 2) store_blk_bf16<false>(w[WB + 4] >> 16, w + WB + 5, rowbase, x, 4);
}
template <int BLK>
__device__ __forceinline__ void dec_window_at(int wb, const uint32_t (&w)[12], uint32_t rowbase, uint32_t x) {
  switch (wb) {   // warp-uniform: the window offset depends on the K step and the row residue only
    case 0: dec_window<0, BLK>(w, rowbase, x); break;
    case 1: dec_window<1, BLK>(w, rowbase, x); break;
    case 2: dec_window<2, BLK>(w, rowbase, x); break;
    default: dec_window<3, BLK>(w, rowbase, x); break;
  }
}

// Zeros into the 4 swizzled 16-byte chunks cbase .. cbase + 3 of the B tile row at rowbase.
__device__ __forceinline__ void store_blk_zero(uint32_t rowbase, uint32_t x, int cbase) {
#pragma unroll
  for (int c = 0; c < 4; ++c) st_shared_v4(rowbase + (((uint32_t)(cbase + c) ^ x) << 4), 0u, 0u, 0u, 0u);
}

// ---------------------------------------------------------------- the grouped GEMM

// GATEUP: A = the tokens' rows of x [T, d] (a_src = x), B = gate rows c0..c0+127 and up
//         rows f+c0..f+c0+127 (zero past f), K = d; epilogue h = gelu(gate) * up -> hb (bf16,
//         padded order).
// DOWN:   A = hb [padded rows, f] (tmap_h: 2-D tiles of 128 rows x 64 columns by TMA), B =
//         down rows n0..n0+127, K = f; epilogue y * w * s -> yslot (bf16, slot order).
// tmap_w: the weight matrix (gate_up or down) as lines of 4 rows, boxes of 48 bytes x 32 lines.
template <bool GATEUP, int BN, int HALVES>
__global__ void __launch_bounds__(kThreads, 1)
k_moe_gemm(const __grid_constant__ CUtensorMap tmap_h, const __grid_constant__ CUtensorMap tmap_w,
           const __nv_bfloat16 *__restrict__ a_src, const float *__restrict__ expert_scale, int d, int f, int k,
           MoeWork W) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ GemmBars bars;
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = GATEUP ? d : f;
  const int ksteps = K / BK;
  using C = GemmCfg<GATEUP, BN, HALVES>;
  constexpr bool kRowDec = C::kRowDec;
  constexpr int kAccBufs = C::kAccBufs;
  constexpr int kBN = C::kBN;
  const int n_ntiles = GATEUP ? (f + kBN / 2 - 1) / (kBN / 2) : d / kBN;
  const int rb = (K / MOE_QK) * MOE_QBYTES;            // bytes per weight row
  constexpr int kHalves = C::kHalves, kStages = C::kStages, kAhead = C::kAhead;
  constexpr uint32_t kBOff = C::kBOff, kStageBytes = C::kStageBytes, kTmemCols = C::kTmemCols;
  const int n_items = (HALVES == 1 ? *W.n_tiles : *W.n_pairs) * n_ntiles;
  // Work order: the n-tiles of one row tile (gate_up) or tile pair (down) follow each other,
  // so its A rows are read while in L2.
  auto item_nt = [&](int item) -> int { return item % n_ntiles; };
  // work item -> its first tile, and whether a second tile (rows 128 .. 255 past the first
  // tile's start) belongs to it (down only)
  auto item_tile = [&](int item, int &tile, bool &h1) {
    const int q = item / n_ntiles;
    if (HALVES == 1) {
      tile = q;
      h1 = false;
    } else {
      tile = W.pairs[2 * q];
      h1 = W.pairs[2 * q + 1] != 0;
    }
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars.full[s], kGroupThreads / 32);   // the step's producer group's warps arrive
      mbar_init(&bars.empty[s], 1);
    }
    for (int q = 0; q < kProdGroups * kMaxRawSlots; ++q)
      mbar_init(&bars.raw[q / kMaxRawSlots][q % kMaxRawSlots], kRawBoxes);   // one arrival per box
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars.acc_full[b], 1);
      mbar_init(&bars.acc_empty[b], kEpiWarps * 32);
    }
    bars.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&bars.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;

  if (warp >= kMmaWarp + 1) {
    // ------------------------------------------------------------ producers
    // Producer group pg takes the K steps g with g % kProdGroups == pg (its local steps li:
    // g = pg + kProdGroups li). Thread pt of a group:
    //  A (gate_up): 16-byte chunk pt % 8 of A rows pt / 8 + 32 q (q < 4);
    //  B: warp wg = pt / 32 of the group and lane i decode weight row 4 i + r of the item into
    //    B tile row j * 128 + 32 r + i, where (gate_up) j = wg / 4 is gate (0) or up (1), both
    //    blocks of the K step; (down) j = 0 and the thread decodes block h = wg / 4 only;
    //    r = wg % 4 in both;
    //  raw: the group has a ring of kRawSlots slots of its own; warp wg alone reads box wg of a
    //    slot, and refills it (for the step kRawSlots local steps ahead) once its lanes have
    //    used the bytes they read. The warps of a group share no other wait.
    const int pq = threadIdx.x - (kMmaWarp + 1) * 32;
    const int pg = pq / kGroupThreads, pt = pq - pg * kGroupThreads;   // pt 0..255
    const int wg = pt >> 5, res = wg & 3, jh = wg >> 2;
    const int cb = pt & 7;                                              // A chunk
    constexpr uint32_t kSubBytes = C::kSubBytes;
    constexpr int kRawSlots = C::kRawSlots;
    constexpr uint32_t kRawSlotBytes = C::kRawSlotBytes;
    const uint32_t raw_base = sbase + (uint32_t)kStages * kStageBytes + (uint32_t)pg * kRawSlots * kRawSlotBytes;
    const int my_items = blockIdx.x < n_items ? (n_items - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    const int total = my_items * ksteps;
    const int n_local = total > pg ? (total - pg + kProdGroups - 1) / kProdGroups : 0;
    // the first line of the CTA's jj-th item's B rows in the weight map (gate rows for gate_up;
    // the up rows are f / 4 lines on)
    auto item_line0 = [&](int jj) -> int {
      const int item = (int)blockIdx.x + jj * (int)gridDim.x;
      const int nt = item_nt(item);
      int tile;
      bool h1;
      item_tile(item, tile, h1);
      const int e = W.tiles[2 * tile];
      return GATEUP ? (e * 2 * f + nt * (kBN / 2)) >> 2 : (int)(((long long)e * d + (long long)nt * kBN) >> 2);
    };
    // sources for the CTA's jj-th work item: this thread's A rows (null past the expert's rows;
    // gate_up only), whether this thread's B row is one of the expert's (gate_up: gate and up
    // rows c < f), the tile, and whether the second half holds any of the expert's rows
    struct RowSrc {
      const __nv_bfloat16 *arow[GATEUP ? 4 * kHalves : 1];
      bool wvalid;
      int tile, h1;
    };
    auto item_src = [&](int jj) -> RowSrc {
      const int item = (int)blockIdx.x + jj * (int)gridDim.x;
      const int nt = item_nt(item);
      int tile;
      bool h1;
      item_tile(item, tile, h1);
      const int e = W.tiles[2 * tile], m0 = W.tiles[2 * tile + 1];
      const int cnt = W.counts[e];
      RowSrc rs;
      rs.tile = tile;
      rs.h1 = h1;
      if (GATEUP) {
        // A row ra (0 .. 128 kHalves - 1) is row m0 + ra of the expert (a pair's second tile
        // follows its first)
#pragma unroll
        for (int q = 0; q < 4 * kHalves; ++q) {
          const int r = m0 + (pt >> 3) + 32 * q;
          rs.arow[q] = r < cnt ? a_src + (size_t)(W.perm[W.offsets[e] + r] / k) * d : nullptr;
        }
        rs.wvalid = nt * (kBN / 2) + 4 * (pt & 31) + res < f;
      } else {
        rs.arow[0] = nullptr;
        rs.wvalid = true;
      }
      return rs;
    };
    // A of step (rs, ks) into stage s: gathered rows (gate_up), or the h tiles by TMA (down)
    auto issue_a = [&](const RowSrc &rs, int ks, int s) {
      const uint32_t a_saddr = sbase + (uint32_t)s * kStageBytes;
      if (GATEUP) {
#pragma unroll
        for (int q = 0; q < 4 * kHalves; ++q) {
          const int ra = (pt >> 3) + 32 * q;
          if (ra >= BM && !rs.h1) break;   // the MMA skips an empty second half
          const __nv_bfloat16 *ap = rs.arow[q] ? rs.arow[q] + (size_t)ks * BK + 8 * cb : a_src;
          cp_async16(a_saddr + (uint32_t)(ra >> 7) * kTileBytes + (uint32_t)(ra & 127) * 128u +
                         (((uint32_t)cb ^ (uint32_t)(ra & 7)) << 4),
                     ap, rs.arow[q] ? 16u : 0u);
        }
      } else if (pt == 0) {
        // the 128 x 64 tiles of h by TMA: their bytes join the stage's full barrier, whose
        // phase cannot complete before this thread's warp arrives for the step (after this call)
        mbar_expect_tx(&bars.full[s], kTileBytes * (rs.h1 ? 2u : 1u));
        tma_load_2d(a_saddr, &tmap_h, ks * BK, rs.tile * BM, &bars.full[s]);
        if (rs.h1) tma_load_2d(a_saddr + kTileBytes, &tmap_h, ks * BK, rs.tile * BM + BM, &bars.full[s]);
      }
    };
    // this warp's raw box of step (line0, ks) into ring slot q (lane 0): residue r = wg % 4;
    // it starts at the K step's window rounded down to 16 bytes (gate_up: of part wg / 4;
    // down: plus 16 bytes for block 1)
    auto issue_raw = [&](int line0, int ks, int q) {
      if (lane == 0) {
        const uint32_t xb = (((uint32_t)res * (uint32_t)rb + (uint32_t)ks * 2u * MOE_QBYTES) & ~15u) +
                            (kRowDec ? 0u : 16u * (uint32_t)jh);
        mbar_arrive_expect_tx(&bars.raw[pg][q], kSubBytes);
        tma_load_2d(raw_base + (uint32_t)q * kRawSlotBytes + (uint32_t)wg * kSubBytes, &tmap_w, (int)xb,
                    line0 + (GATEUP ? jh * (f >> 2) : (kRowDec ? jh * 32 : 0)), &bars.raw[pg][q]);
      }
    };
    bool ok = true;
    // three walks over this group's steps: the raw issue (kRawSlots steps ahead), the A issue
    // (kAhead steps ahead) and the decode
    int rjj = 0, rks = pg, ijj = 0, iks = pg, cjj = 0, cks = pg;
    while (rks >= ksteps && rjj < my_items) { rks -= ksteps; ++rjj; }
    ijj = cjj = rjj;
    iks = cks = rks;
    int rline = rjj < my_items ? item_line0(rjj) : 0;
    RowSrc isrc{}, csrc{};
    if (ijj < my_items) { isrc = item_src(ijj); csrc = isrc; }
    auto step = [&](int &jj, int &ks) -> bool {   // to the group's next step; true on a new item
      ks += kProdGroups;
      bool moved = false;
      while (ks >= ksteps) { ks -= ksteps; ++jj; moved = true; }
      return moved && jj < my_items;
    };
    int raw_issued = 0;
    for (int q = 0; q < kRawSlots && q < n_local; ++q, ++raw_issued) {   // the ring's first fill
      issue_raw(rline, rks, q);
      if (step(rjj, rks)) rline = item_line0(rjj);
    }
    for (int a = 0; a < kAhead && a < n_local; ++a) {   // the first stages are free
      issue_a(isrc, iks, (pg + kProdGroups * a) % kStages);
      if (step(ijj, iks)) isrc = item_src(ijj);
      cp_async_commit();
    }
    // this thread's B row in the tile and its raw window in a ring slot (box wg, line lane)
    const int brow = (kRowDec ? jh * 128 : 0) + res * 32 + lane;
    const uint32_t win_off = (uint32_t)wg * kSubBytes + (uint32_t)lane * C::kBoxW;
    int li = 0;
    for (; li < n_local; ++li) {
      const int g = pg + kProdGroups * li;
      const int s = g % kStages, q = li % kRawSlots;
      // step g: its A copies (this thread's, issued kAhead steps ago) and its raw boxes have landed
      cp_async_wait<kAhead - 1>();
      if (!__all_sync(0xffffffffu, mbar_wait(&bars.raw[pg][q], (uint32_t)(li / kRawSlots) & 1u, W.err, 14,
                                             W.wait_ns)))
        ok = false;
      const uint32_t rowbase = sbase + (uint32_t)s * kStageBytes + kBOff + (uint32_t)brow * 128u;
      const uint32_t x = (uint32_t)(brow & 7);
      if (ok && csrc.wvalid) {
        const uint4 *wp = reinterpret_cast<const uint4 *>(smem_raw + (raw_base - smem_u32(smem_raw)) +
                                                          (size_t)q * kRawSlotBytes + win_off);
        const int wb = (int)((((uint32_t)res * (uint32_t)rb + (uint32_t)cks * 2u * MOE_QBYTES) & 15u) >> 2);
        if (kRowDec) {
          const uint4 v0 = wp[0], v1 = wp[1], v2 = wp[2];
          const uint32_t w[12] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w, v2.x, v2.y, v2.z, v2.w};
          dec_window_at<3>(wb, w, rowbase, x);
        } else {
          // the 32-byte box is window bytes 0-31 (block 0) or 16-47 (block 1): placed at its
          // words of the 48-byte window
          const uint4 v0 = wp[0], v1 = wp[1];
          if (jh == 0) {
            const uint32_t w[12] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w, 0u, 0u, 0u, 0u};
            dec_window_at<1>(wb, w, rowbase, x);
          } else {
            const uint32_t w[12] = {0u, 0u, 0u, 0u, v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
            dec_window_at<2>(wb, w, rowbase, x);
          }
        }
      } else {
        store_blk_zero(rowbase, x, 0);
        store_blk_zero(rowbase, x, 4);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.full[s]);
      if (!ok) break;   // warp-uniform
      // The warp's box of slot q is refilled by TMA (the async proxy) only once every lane has
      // used the bytes it read from it (the decode's stores depend on them, and the stores come
      // before the __syncwarp): a shared-memory load still in flight is not ordered before a
      // later TMA write by a barrier alone.
      if (li + kRawSlots < n_local) {
        issue_raw(rline, rks, q);
        ++raw_issued;
        if (step(rjj, rks)) rline = item_line0(rjj);
      }
      if (step(cjj, cks)) csrc = item_src(cjj);
      // then the A copies of local step li + kAhead, once the MMA has released its stage
      if (li + kAhead < n_local) {
        const int gi = g + kProdGroups * kAhead, si = gi % kStages;
        const uint32_t par = ((uint32_t)(gi / kStages) & 1u) ^ 1u;
        if (__all_sync(0xffffffffu, mbar_wait(&bars.empty[si], par, W.err, 10, W.wait_ns))) {
          issue_a(isrc, iks, si);
          if (step(ijj, iks)) isrc = item_src(ijj);
        } else {
          ok = false;   // the warp stops at its next step
        }
      }
      cp_async_commit();
    }
    cp_async_wait<0>();   // no copy lands after this thread leaves
    // after an early stop, the raw boxes still in flight land before the group leaves (each
    // wait bounded; a completed phase returns at once)
    for (int lq = li; lq < raw_issued; ++lq)
      mbar_wait(&bars.raw[pg][lq % kRawSlots], (uint32_t)(lq / kRawSlots) & 1u, W.err, 15, W.wait_ns);
    if (!ok) atomicExch(&bars.abort_flag, 1);
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issue (one thread)
    if (lane == 0) {
      int it = 0, j = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x, ++j) {
        const int b = kAccBufs == 2 ? (j & 1) : 0;
        const uint32_t upar = ((uint32_t)(kAccBufs == 2 ? (j >> 1) : j) & 1u) ^ 1u;
        if (!mbar_wait(&bars.acc_empty[b], upar, W.err, 11, W.wait_ns)) { ok = false; break; }
        tc_fence_after();
        // the second half only where the item holds a second tile
        int tile;
        bool h1;
        item_tile(item, tile, h1);
        const uint32_t dtm = tmem + (uint32_t)(b * kHalves * kBN);
        for (int ks = 0; ks < ksteps; ++ks, ++it) {
          const int s = it % kStages;
          const uint32_t par = (uint32_t)(it / kStages) & 1u;
          if (!mbar_wait(&bars.full[s], par, W.err, 12, W.wait_ns)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_saddr = sbase + (uint32_t)s * kStageBytes;
          const uint32_t b_saddr = a_saddr + kBOff;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t bdesc = sw128_desc(b_saddr + kk * 32);
            const uint32_t acc = (ks > 0 || kk > 0) ? 1u : 0u;
            umma_bf16(dtm, sw128_desc(a_saddr + kk * 32), bdesc, C::kIdesc, acc);
            if (h1) umma_bf16(dtm + kBN, sw128_desc(a_saddr + kTileBytes + kk * 32), bdesc, C::kIdesc, acc);
          }
          umma_commit(&bars.empty[s]);
        }
        if (!ok) break;
        umma_commit(&bars.acc_full[b]);
      }
      if (!ok) atomicExch(&bars.abort_flag, 1);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (lane = row)
    const int r = warp * 32 + lane;   // row inside a 128-row half == TMEM lane
    int j = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++j) {
      const int b = kAccBufs == 2 ? (j & 1) : 0;
      const uint32_t par = (uint32_t)(kAccBufs == 2 ? (j >> 1) : j) & 1u;
      const bool ok = mbar_wait(&bars.acc_full[b], par, W.err, 13, W.wait_ns);
      if (__any_sync(0xffffffffu, !ok)) { atomicExch(&bars.abort_flag, 1); break; }
      tc_fence_after();
      const int nt = item_nt(item);
      int tile;
      bool h1;
      item_tile(item, tile, h1);
      const int e = W.tiles[2 * tile], m0 = W.tiles[2 * tile + 1];
      const int cnt = W.counts[e];
      const int nh = h1 ? 2 : 1;   // halves of this item (warp-uniform)
      for (int h = 0; h < nh; ++h) {
        const int mr = m0 + h * BM + r;        // row of the expert
        const bool valid = mr < cnt;
        const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)((b * kHalves + h) * kBN);
        // accumulator column 32 r + i holds weight row 4 i + r of the item (of each part): the
        // 16 output columns 16 u .. 16 u + 15 are columns 32 r + 4 u + a (r, a < 4), output
        // column 4 a + r
        if (GATEUP) {
          const int c0 = nt * (kBN / 2);   // first h column of this item
          __nv_bfloat16 *dst = W.hb + (size_t)((tile + h) * BM + r) * f + (size_t)c0;
#pragma unroll
          for (int u16 = 0; u16 < kBN / 32; ++u16) {
            const int c = 16 * u16;
            if (c0 + c >= f) break;   // warp-uniform: the item's columns past f are zero rows
            uint32_t g[4][4], u[4][4];
#pragma unroll
            for (int rr = 0; rr < 4; ++rr) {
              tmem_ld4(taddr + (uint32_t)(32 * rr + 4 * u16), g[rr]);
              tmem_ld4(taddr + (uint32_t)(kBN / 2 + 32 * rr + 4 * u16), u[rr]);
            }
            tmem_ld_wait();
            uint32_t o[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {   // output columns 2 i, 2 i + 1 = 4 a + r, 4 a + r + 1
              const int a = i >> 1, r0 = 2 * (i & 1);
              const float h0 = gelu_tanh_f(__uint_as_float(g[r0][a])) * __uint_as_float(u[r0][a]);
              const float hv1 = gelu_tanh_f(__uint_as_float(g[r0 + 1][a])) * __uint_as_float(u[r0 + 1][a]);
              o[i] = pack_bf16(h0, hv1);
            }
            if (valid) {
              uint4 *dp = reinterpret_cast<uint4 *>(dst + c);
              dp[0] = make_uint4(o[0], o[1], o[2], o[3]);
              dp[1] = make_uint4(o[4], o[5], o[6], o[7]);
            }
          }
        } else {
          int slot = 0;
          float scale = 0.f;
          if (valid) {
            slot = W.perm[W.offsets[e] + mr];
            scale = W.w[slot] * expert_scale[e];
          }
          __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(W.yslot) + (size_t)slot * d + (size_t)nt * kBN;
#pragma unroll
          for (int u16 = 0; u16 < kBN / 16; ++u16) {
            const int c = 16 * u16;
            uint32_t y[4][4];
#pragma unroll
            for (int rr = 0; rr < 4; ++rr)   // part u16 / 8 of 128 columns, as in gate_up's parts
              tmem_ld4(taddr + (uint32_t)(128 * (u16 >> 3) + 32 * rr + 4 * (u16 & 7)), y[rr]);
            tmem_ld_wait();
            uint32_t o[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int a = i >> 1, r0 = 2 * (i & 1);
              o[i] = pack_bf16(__uint_as_float(y[r0][a]) * scale, __uint_as_float(y[r0 + 1][a]) * scale);
            }
            if (valid) {
              uint4 *dp = reinterpret_cast<uint4 *>(dst + c);
              dp[0] = make_uint4(o[0], o[1], o[2], o[3]);
              dp[1] = make_uint4(o[4], o[5], o[6], o[7]);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bars.acc_empty[b]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// out[t, c] = sum_{j < k} yslot[t k + j, c] (already weighted), j ascending.
__global__ void __launch_bounds__(256) k_combine(const __nv_bfloat16 *__restrict__ yslot, int T, int d, int k,
                                                 float *__restrict__ out, int accumulate) {
  const int vpr = d / 8;
  const long long total = (long long)T * vpr;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(i / vpr), v = (int)(i % vpr);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j0 = 0; j0 < k; j0 += 8) {   // eight slots' loads in flight, then the sums in j order
      uint4 q[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        q[u] = j0 + u < k ? __ldg(reinterpret_cast<const uint4 *>(yslot + (size_t)(t * k + j0 + u) * d) + v)
                          : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (j0 + u >= k) break;
        const uint32_t qq[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          acc[2 * h] += __uint_as_float(qq[h] << 16);
          acc[2 * h + 1] += __uint_as_float(qq[h] & 0xffff0000u);
        }
      }
    }
    float4 *op = reinterpret_cast<float4 *>(out + (size_t)t * d) + 2 * v;
    if (accumulate) {   // out += the sum (one FP32 addition per element)
      const float4 o0 = op[0], o1 = op[1];
      acc[0] = o0.x + acc[0]; acc[1] = o0.y + acc[1]; acc[2] = o0.z + acc[2]; acc[3] = o0.w + acc[3];
      acc[4] = o1.x + acc[4]; acc[5] = o1.y + acc[5]; acc[6] = o1.z + acc[6]; acc[7] = o1.w + acc[7];
    }
    op[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    op[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
}

// ---------------------------------------------------------------- router on the tensor cores
//
// The prefill router product logits[t, e] = sum_i x[t, i] W_r[e, i] (x bf16, W_r FP32) as a
// bf16 tensor-core GEMM with no loss: W_r = hi + mid + lo, three bf16 planes (each rounds
// what the planes before it left: 24 significand bits in three of 8), exact for |w| >= 2^-110
// and within 2^-133 below that (bf16's subnormal step); every product of a bf16 x with a bf16
// plane is exact, and the three products of a term accumulate in FP32 in the same accumulator. d is split over CTAs (the partials are added in split order by the
// top-k kernel, as for the FP32 SIMT router).

// wsplit [3][128][d]: planes hi, mid, lo of W_r, rows E..127 zero. Four weights a thread
// (d is a multiple of 4, so a group never straddles rows; 16-byte loads, 8-byte stores).
__global__ void __launch_bounds__(256) k_split_router(const float *__restrict__ w, int E, int d,
                                                      __nv_bfloat16 *__restrict__ ws) {
  const long long n = 128LL * d, ng = n / 4, nw = (long long)E * d;
  for (long long g = blockIdx.x * (long long)blockDim.x + threadIdx.x; g < ng; g += (long long)gridDim.x * blockDim.x) {
    const long long i = 4 * g;
    const float4 v4 = i < nw ? __ldg(reinterpret_cast<const float4 *>(w + i)) : make_float4(0.f, 0.f, 0.f, 0.f);
    const float v[4] = {v4.x, v4.y, v4.z, v4.w};
    __nv_bfloat16 p[3][4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const __nv_bfloat16 hi = __float2bfloat16_rn(v[q]);
      const float r1 = v[q] - __bfloat162float(hi);    // exact: v and hi are within a factor of two
      const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
      const float r2 = r1 - __bfloat162float(mid);     // exact, and at most 8 significant bits
      p[0][q] = hi;
      p[1][q] = mid;
      p[2][q] = __float2bfloat16_rn(r2);
    }
#pragma unroll
    for (int j = 0; j < 3; ++j) *reinterpret_cast<uint2 *>(ws + (size_t)j * n + i) = *reinterpret_cast<const uint2 *>(p[j]);
  }
}

constexpr int kRtStages = 3;
constexpr uint32_t kRtA = BM * BK * 2;           // 16 KB: 128 tokens x 64 of d
constexpr uint32_t kRtB = 128 * BK * 2;          // 16 KB: one plane, 128 experts x 64 of d
constexpr uint32_t kRtStage = kRtA + 3 * kRtB;   // 64 KB
constexpr int kRtSmem = kRtStages * (int)kRtStage + 1024;
constexpr uint32_t kRtIdesc = umma_idesc(128);   // M = 128, N = 128
constexpr int kRtSplit = 4;                        // d splits (<= MOE_ROUTER_MAX_SPLIT)
static_assert(kRtSplit <= MOE_ROUTER_MAX_SPLIT, "the route scratch holds that many partials");

struct RtBars {
  uint64_t full[kRtStages];
  uint64_t empty[kRtStages];
  uint64_t acc;
  uint32_t tmem_base;
};

// CTA (m, s): tokens 128 m .. 128 m + 127, K steps [s nk / S, (s + 1) nk / S) of the nk = d / 64;
// 4 warps: warp 0 lane 0 issues the TMA copies (x tile and the three plane tiles of a K step
// into one stage), warp 1 holds the TMEM accumulator (128 columns) and its lane 0 issues
// tcgen05.mma (M = 128, N = 128, K = 16; per K step 4 x 3, all into one accumulator); then every
// warp reads its 32 rows (lane = token) and writes part[s][t][e] for e < E.
__global__ void __launch_bounds__(128, 1)
k_router_tc(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w, int T, int d,
            int E, int nsplit, float *__restrict__ part, MoeWork W) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ RtBars bars;
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * BM, split = blockIdx.y;
  const int nk = d / BK;
  const int k0 = (int)((long long)nk * split / nsplit), k1 = (int)((long long)nk * (split + 1) / nsplit);
  if (threadIdx.x == 0) {
    for (int s = 0; s < kRtStages; ++s) {
      mbar_init(&bars.full[s], 1);
      mbar_init(&bars.empty[s], 1);
    }
    mbar_init(&bars.acc, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars.tmem_base, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;
  if (warp == 0 && lane == 0) {
    for (int ks = k0, i = 0; ks < k1; ++ks, ++i) {
      const int s = i % kRtStages;
      if (i >= kRtStages &&
          !mbar_wait(&bars.empty[s], (uint32_t)(i / kRtStages - 1) & 1u, W.err, 16, W.wait_ns))
        break;
      const uint32_t st = sbase + (uint32_t)s * kRtStage;
      mbar_arrive_expect_tx(&bars.full[s], kRtStage);
      tma_load_2d(st, &tmap_x, ks * BK, t0, &bars.full[s]);
#pragma unroll
      for (int j = 0; j < 3; ++j) tma_load_2d(st + kRtA + (uint32_t)j * kRtB, &tmap_w, ks * BK, j * 128, &bars.full[s]);
    }
  } else if (warp == 1 && lane == 0) {
    for (int ks = k0, i = 0; ks < k1; ++ks, ++i) {
      const int s = i % kRtStages;
      if (!mbar_wait(&bars.full[s], (uint32_t)(i / kRtStages) & 1u, W.err, 17, W.wait_ns)) break;
      tc_fence_after();
      const uint32_t st = sbase + (uint32_t)s * kRtStage;
#pragma unroll
      for (int kk = 0; kk < BK / 16; ++kk)
#pragma unroll
        for (int j = 0; j < 3; ++j)
          umma_bf16(tmem, sw128_desc(st + (uint32_t)kk * 32u), sw128_desc(st + kRtA + (uint32_t)j * kRtB + (uint32_t)kk * 32u),
                    kRtIdesc, (i > 0 || kk > 0 || j > 0) ? 1u : 0u);
      umma_commit(&bars.empty[s]);
    }
    umma_commit(&bars.acc);   // arrives once every MMA issued above has completed
  }
  __syncwarp();
  const bool ok = mbar_wait(&bars.acc, 0u, W.err, 18, W.wait_ns);
  if (__all_sync(0xffffffffu, ok)) {
    tc_fence_after();
    const int t = t0 + warp * 32 + lane;
    float *dst = part + ((size_t)split * T + (size_t)(t < T ? t : 0)) * E;
    const bool vec = (E & 3) == 0;   // 16-byte stores when every row starts 16-byte aligned
#pragma unroll
    for (int c = 0; c < 128; c += 4) {
      uint32_t v[4];
      tmem_ld4(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c, v);
      tmem_ld_wait();
      if (t < T && c < E) {
        if (vec) {
          *reinterpret_cast<float4 *>(dst + c) =
              make_float4(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2]), __uint_as_float(v[3]));
        } else {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (c + q < E) dst[c + q] = __uint_as_float(v[q]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

}  // namespace

static int launch_err() { return cudaGetLastError() == cudaSuccess ? 0 : -1; }

// Tensor map (driver entry point) of the padded h [rows, f] bf16 for the down GEMM's A tiles:
// box 64 columns x 128 rows, 128-byte swizzle (the layout the MMA descriptors expect).
static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void *p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

static bool make_tmap_h(CUtensorMap *m, const void *base, int cols, long long rows) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)BM};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Tensor map of a Q4_0 weight matrix of `rows` rows of rb bytes (rows a multiple of 4, 4 rb a
// multiple of 16) seen as rows / 4 lines of 4 rb bytes: boxes of box_w bytes x 32 lines, no
// swizzle; bytes past a line's end or past the last line read as zeros.
static bool make_tmap_w(CUtensorMap *m, const void *base, int rb, long long rows, uint32_t box_w) {
  auto enc = get_encode();
  if (!enc || rows % 4 || (4 * rb) % 16) return false;
  cuuint64_t dims[2] = {(cuuint64_t)(4 * rb), (cuuint64_t)(rows / 4)};
  cuuint64_t strides[1] = {(cuuint64_t)(4 * rb)};
  cuuint32_t box[2] = {box_w, (cuuint32_t)kSubRows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool moe_router_tc_supported(int d, int E) { return E >= 1 && E <= 128 && d % BK == 0; }
// (router_w must be 16-byte aligned for the split's 16-byte loads: the layer's entry points check it)

int moe_launch_router_tc(const MoeLaunch &L, const MoeWork &W, const void *x, const float *router_w, int T, int d,
                         int E, int num_sms, float *part, int *nsplit) {
  if (!moe_router_tc_supported(d, E) || W.wsplit == nullptr) return -2;
  static unsigned long long smem_ok = 0ull;   // per device
  if (!moe_allow_dyn_smem(reinterpret_cast<const void *>(k_router_tc), &smem_ok)) return -1;
  // a fixed number of d splits, whatever T: a token's logits are then the same bits in a call
  // of any size (a chunked call gives the bits of one pass); 32 row tiles x 4 splits = 128 CTAs
  // at 4,096 tokens
  const int nk = d / BK, mt = (T + BM - 1) / BM;
  const int ns = kRtSplit < nk ? kRtSplit : nk;
  (void)num_sms;
  CUtensorMap tx, tw;
  if (!make_tmap_h(&tx, x, d, T) || !make_tmap_h(&tw, W.wsplit, d, 3 * 128)) return -1;
  int grid = (int)((32LL * d + 255) / 256);   // 128 d / 4 groups
  if (grid > 4 * num_sms) grid = 4 * num_sms;
  k_split_router<<<grid, 256, 0, L.stream>>>(router_w, E, d, W.wsplit);
  if (launch_err()) return -1;
  moe_prof_count(1);
  k_router_tc<<<dim3(mt, ns), 128, kRtSmem, L.stream>>>(tx, tw, T, d, E, ns, part, W);
  if (launch_err()) return -1;
  moe_prof_count(1);
  *nsplit = ns;
  return 0;
}

constexpr int kDownWideHalves = 1;   // down with N = 256: single tiles (1) or tile pairs (2)

int moe_launch_gemm_experts(const MoeLaunch &L, const MoeWork &W, const void *x, const uint8_t *gate_up_q4,
                            const uint8_t *down_q4, const float *expert_scale, int T, int d, int f, int E, int k,
                            float *out, int num_sms, int max_tiles) {
  // K of both GEMMs in whole 64-wide steps; down's output in whole 128-column tiles
  if (d % BK || d % 128 || f % BK) return -2;
  // gate_up: tile pairs (M = 256 sharing one decoded B tile, one accumulator buffer) when the
  // experts hold 1.5 tiles of rows on average, else single tiles (two accumulator buffers, the
  // epilogue overlapping the next item); both give the same bits
  const bool gu_pairs = (long long)T * k >= 3LL * BM / 2 * E;
  // down: N = 256 over single tiles (two accumulator buffers) where d is a multiple of 256,
  // else N = 128 over tile pairs
  const bool wide = d % 256 == 0;
  using CG1 = GemmCfg<true, 256, 1>;
  using CG2 = GemmCfg<true, 256, 2>;
  using CDN = GemmCfg<false, 128, 2>;
  using CDW = GemmCfg<false, 256, kDownWideHalves>;
  static unsigned long long smem_ok[4] = {0ull, 0ull, 0ull, 0ull};   // per device, per kernel
  if (!moe_allow_dyn_smem(gu_pairs ? reinterpret_cast<const void *>(k_moe_gemm<true, 256, 2>)
                                   : reinterpret_cast<const void *>(k_moe_gemm<true, 256, 1>),
                          &smem_ok[gu_pairs ? 1 : 0]) ||
      !moe_allow_dyn_smem(wide ? reinterpret_cast<const void *>(k_moe_gemm<false, 256, kDownWideHalves>)
                               : reinterpret_cast<const void *>(k_moe_gemm<false, 128, 2>),
                          &smem_ok[wide ? 3 : 2]))
    return -1;
  moe_prof_mark(L.stream, MOE_K_GEMM_GATEUP, true);
  CUtensorMap th, twg, twd;
  if (!make_tmap_h(&th, W.hb, f, (long long)max_tiles * BM)) return -1;
  static_assert(CG1::kBoxW == CG2::kBoxW, "one gate_up weight map for both");
  if (!make_tmap_w(&twg, gate_up_q4, (d / MOE_QK) * MOE_QBYTES, (long long)E * 2 * f, CG1::kBoxW) ||
      !make_tmap_w(&twd, down_q4, (f / MOE_QK) * MOE_QBYTES, (long long)E * d, wide ? CDW::kBoxW : CDN::kBoxW))
    return -1;
  const __nv_bfloat16 *xb = static_cast<const __nv_bfloat16 *>(x);
  if (gu_pairs)
    k_moe_gemm<true, 256, 2><<<num_sms, kThreads, CG2::kSmemBytes, L.stream>>>(th, twg, xb, expert_scale, d, f, k, W);
  else
    k_moe_gemm<true, 256, 1><<<num_sms, kThreads, CG1::kSmemBytes, L.stream>>>(th, twg, xb, expert_scale, d, f, k, W);
  if (launch_err()) return -1;
  moe_prof_count(1);
  moe_prof_mark(L.stream, MOE_K_GEMM_GATEUP, false);
  moe_prof_mark(L.stream, MOE_K_GEMM_DOWN, true);
  if (wide)
    k_moe_gemm<false, 256, kDownWideHalves><<<num_sms, kThreads, CDW::kSmemBytes, L.stream>>>(th, twd, W.hb, expert_scale,
                                                                                             d, f, k, W);
  else
    k_moe_gemm<false, 128, 2><<<num_sms, kThreads, CDN::kSmemBytes, L.stream>>>(th, twd, W.hb, expert_scale, d, f, k, W);
  if (launch_err()) return -1;
  moe_prof_count(1);
  moe_prof_mark(L.stream, MOE_K_GEMM_DOWN, false);
  moe_prof_mark(L.stream, MOE_K_COMBINE, true);
  k_combine<<<4 * num_sms, 256, 0, L.stream>>>(reinterpret_cast<const __nv_bfloat16 *>(W.yslot), T, d, k, out,
                                               L.accumulate ? 1 : 0);
  if (launch_err()) return -1;
  moe_prof_count(1);
  moe_prof_mark(L.stream, MOE_K_COMBINE, false);
  return 0;
}
