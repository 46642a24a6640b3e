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
// tile list covers padded rows [128 i, 128 i + 128). A gate_up work item is one tile and one
// n-tile; a down work item is up to two consecutive tiles of one expert (M = 256 as two
// 128-row MMA halves sharing the B tile, so the decode work per MMA halves) and one n-tile.
// The A tile of a K step lands in the 128-byte swizzled K-major layout: gate_up's producers
// gather the tokens' rows of x with 16-byte asynchronous copies (zero-filled past the
// expert's rows); down's 128 x 64 tiles of the padded h come by 2-D TMA copies. The raw
// Q4_0 bytes of the B rows are copied (16-byte asynchronous copies of a 64-byte window per
// row) into a staging buffer of the stage. The weights never exist in bf16 in global memory:
// the producers decode (q - 8) * d from the staged bytes and write the swizzled K-major B
// tile that tcgen05.mma reads.
//
// One CTA per SM, persistent over work items, warp-specialised:
//   warps 0-3  epilogue: tcgen05.ld of the 128 x 128 FP32 accumulators (lane = row)
//   warp  4    TMEM allocation; lane 0 issues tcgen05.mma (M = 128, N = 128, K = 16, one
//              per 16-wide K slice and item half)
//   warps 5-20 producers in two groups taking alternate K steps: A copies (gate_up) or the
//              TMA issue (down), raw-window copies, Q4_0 -> bf16 dequantisation for B
// Shared-memory stages are handed over with mbarriers (every wait is time-bounded); the
// accumulators are double-buffered in TMEM so the epilogue of one item overlaps the next.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "moe_common.cuh"

namespace {

constexpr int BM = 128, BK = 64;
static_assert(BM == MOE_GEMM_TILE_ROWS, "the tile list is built with this tile height");
constexpr int kMaxStages = 5;
constexpr int kEpiWarps = 4;
constexpr int kMmaWarp = 4;
constexpr int kProdGroups = 2;                                // producer groups take alternate K steps
constexpr int kProdWarps = 8 * kProdGroups;
constexpr int kProdThreads = kProdWarps * 32;
constexpr int kGroupThreads = kProdThreads / kProdGroups;     // one (row, block) of the B tile each
constexpr int kThreads = (kEpiWarps + 1 + kProdWarps) * 32;
constexpr uint32_t kTileBytes = BM * BK * 2;                  // 16 KB: one 128-row A half
constexpr uint32_t kRawRowBytes = 64;                          // 16-byte-aligned window over a row's 36 bytes

// UMMA instruction descriptor, kind::f16: D FP32 (bits 4-5 = 1), A and B bf16 (bits 7-9,
// 10-12 = 1), both K-major (bits 15, 16 = 0), N >> 3 in bits 17-22, M >> 4 in bits 24-28.
constexpr uint32_t umma_idesc(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

// Per GEMM:
//  gate_up: an item is one 128-row tile and N = 256 columns, the 128 gate rows c0 .. c0+127 and
//    the matching 128 up rows (rows past f are zero); measured: one tcgen05.mma of N = 256 does
//    twice the work of an N = 128 one in about the same pipeline time. A rows are gathered by
//    the producers.
//  down: an item is up to two consecutive tiles of one expert, M = 256 as two 128-row halves
//    that share the dequantised N = 128 B tile (A comes by TMA), so the decode work per MMA
//    halves.
template <bool GATEUP>
struct GemmCfg {
  static constexpr int kBN = GATEUP ? 256 : 128;                 // MMA N
  static constexpr int kHalves = GATEUP ? 1 : 2;
  static constexpr int kStages = GATEUP ? 3 : 4;
  // group steps the copies run ahead of the decode
  static constexpr int kAhead = 1;
  static constexpr uint32_t kBBytes = (uint32_t)kBN * BK * 2;
  static constexpr uint32_t kBOff = kHalves * kTileBytes;        // B tile after the A halves
  static constexpr uint32_t kStageBytes = kBOff + kBBytes;
  static constexpr uint32_t kRawStageBytes = (uint32_t)kBN * kRawRowBytes;
  static constexpr uint32_t kTmemCols = 2 * kHalves * kBN;       // two accumulator buffers
  static constexpr int kSmemBytes = kStages * (kStageBytes + kRawStageBytes) + 1024;
  static constexpr int kRowsPerThread = kBN / (kGroupThreads / 2);   // B rows a producer thread decodes
  static constexpr uint32_t kIdesc = umma_idesc(kBN);
  static_assert(kAhead * kProdGroups <= kStages, "the prologue's stages must be free");
  static_assert(kStages <= kMaxStages && kTmemCols <= 512, "limits");
  static_assert(kRowsPerThread * (kGroupThreads / 2) == kBN, "producer threads cover the B rows");
};

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle (layout type 2),
// rows of 128 bytes in 8-row atoms of 1024 bytes (stride byte offset 1024), version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}

struct GemmBars {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
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

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ float gelu_tanh_f(float z) {
  const float c = 0.7978845608028654f;   // sqrt(2/pi)
  return 0.5f * z * (1.0f + tanhf(c * (z + 0.044715f * z * z * z)));
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
__device__ __forceinline__ void dq_word(uint32_t w, __nv_bfloat162 d2, uint32_t &lo01, uint32_t &lo23,
                                        uint32_t &hi01, uint32_t &hi23) {
  const uint32_t v01 = __byte_perm(w, 0u, 0x4140u);   // [b0, 0, b1, 0]
  const uint32_t v23 = __byte_perm(w, 0u, 0x4342u);   // [b2, 0, b3, 0]
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

// The 20-byte window holding one 18-byte Q4_0 block (starting at the block's address rounded
// down to 4 bytes; never past the end of a Q4_0 matrix whose rows are whole blocks, since
// the last block of a matrix starts at 2 mod 4) and the block's offset in it, in bits.
struct RawBlk {
  uint32_t w[5];
  uint32_t sh;
};

// Decode one block into its 4 swizzled 16-byte chunks of row `row` (chunks cbase..cbase+3).
__device__ __forceinline__ void store_blk_bf16(const RawBlk &r, uint32_t tile_saddr, int row, int cbase) {
  const float d = __half2float(__ushort_as_half((unsigned short)((r.w[0] >> r.sh) & 0xffffu)));
  const __nv_bfloat162 d2 = __float2bfloat162_rn(d);
  const uint32_t s2 = r.sh + 16u;
  uint32_t q[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) q[i] = __funnelshift_rc(r.w[i], r.w[i + 1], s2);
  uint32_t lo[8], hi[8];   // element pairs (0,1),(2,3),...,(14,15) and (16,17),...,(30,31)
#pragma unroll
  for (int i = 0; i < 4; ++i) dq_word(q[i], d2, lo[2 * i], lo[2 * i + 1], hi[2 * i], hi[2 * i + 1]);
  const uint32_t rowbase = tile_saddr + (uint32_t)row * 128u;
  const uint32_t x = (uint32_t)(row & 7);
  st_shared_v4(rowbase + (((uint32_t)(cbase + 0) ^ x) << 4), lo[0], lo[1], lo[2], lo[3]);   // elements 0-7
  st_shared_v4(rowbase + (((uint32_t)(cbase + 1) ^ x) << 4), lo[4], lo[5], lo[6], lo[7]);   // 8-15
  st_shared_v4(rowbase + (((uint32_t)(cbase + 2) ^ x) << 4), hi[0], hi[1], hi[2], hi[3]);   // 16-23
  st_shared_v4(rowbase + (((uint32_t)(cbase + 3) ^ x) << 4), hi[4], hi[5], hi[6], hi[7]);   // 24-31
}

// Zeros into the 4 swizzled 16-byte chunks of row `row` (chunks cbase..cbase+3).
__device__ __forceinline__ void store_blk_zero(uint32_t tile_saddr, int row, int cbase) {
  const uint32_t rowbase = tile_saddr + (uint32_t)row * 128u;
  const uint32_t x = (uint32_t)(row & 7);
#pragma unroll
  for (int c = 0; c < 4; ++c) st_shared_v4(rowbase + (((uint32_t)(cbase + c) ^ x) << 4), 0u, 0u, 0u, 0u);
}

// ---------------------------------------------------------------- the grouped GEMM

// GATEUP: A = the tokens' rows of x [T, d] (a_src = x), B = gate rows c0..c0+127 and up
//         rows f+c0..f+c0+127 (zero past f), K = d; epilogue h = gelu(gate) * up -> hb (bf16,
//         padded order).
// DOWN:   A = hb [padded rows, f] (tmap_h: 2-D tiles of 128 rows x 64 columns by TMA), B =
//         down rows n0..n0+127, K = f; epilogue y * w * s -> yslot (bf16, slot order).
template <bool GATEUP>
__global__ void __launch_bounds__(kThreads, 1)
k_moe_gemm(const __grid_constant__ CUtensorMap tmap_h, const __nv_bfloat16 *__restrict__ a_src,
           const uint8_t *__restrict__ wq, const uint8_t *wq_end,
           const float *__restrict__ expert_scale, int d, int f, int k, MoeWork W) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ GemmBars bars;
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = GATEUP ? d : f;
  const int ksteps = K / BK;
  using C = GemmCfg<GATEUP>;
  constexpr int kBN = C::kBN, kRows = C::kRowsPerThread;
  const int n_ntiles = GATEUP ? (f + kBN / 2 - 1) / (kBN / 2) : d / kBN;
  const int nb_row = K / MOE_QK;                       // Q4_0 blocks per weight row
  const size_t rb = (size_t)nb_row * MOE_QBYTES;       // bytes per weight row
  const size_t expert_bytes = (size_t)(GATEUP ? 2 * f : d) * rb;
  constexpr int kHalves = C::kHalves, kStages = C::kStages, kAhead = C::kAhead;
  constexpr uint32_t kBOff = C::kBOff, kStageBytes = C::kStageBytes, kTmemCols = C::kTmemCols;
  constexpr uint32_t kRawStageBytes = C::kRawStageBytes;
  const int n_items = (GATEUP ? *W.n_tiles : *W.n_pairs) * n_ntiles;
  // work item -> its first tile, and whether a second tile (rows 128 .. 255 past the first
  // tile's start) belongs to it (down only)
  auto item_tile = [&](int item, int &tile, bool &h1) {
    const int q = item / n_ntiles;
    if (GATEUP) {
      tile = q;
      h1 = false;
    } else {
      tile = W.pairs[2 * q];
      h1 = W.pairs[2 * q + 1] != 0;
    }
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars.full[s], kGroupThreads);   // the step's producer group arrives
      mbar_init(&bars.empty[s], 1);
    }
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
    // Producer group pg takes the K steps g with g % kProdGroups == pg. Thread pt of a group
    // owns A row r = pt / 2 (of each half): chunks 4 h .. 4 h + 3 (h = pt & 1) of the row's
    // 128-byte K-step segment; and B rows r + 128 j (j < kRows): Q4_0 block h of each row's two
    // blocks per K step.
    const int pq = threadIdx.x - (kMmaWarp + 1) * 32;
    const int pg = pq / kGroupThreads, pt = pq - pg * kGroupThreads;   // pt 0..255
    const int row = pt >> 1, hsel = pt & 1;
    // the raw Q4_0 bytes of B row n for a K step (two blocks, 36 bytes) arrive in a 64-byte
    // window starting at their address rounded down to 16; hsel copies its half of it
    const uint32_t raw_base = sbase + (uint32_t)kStages * kStageBytes;
    const int my_items = blockIdx.x < n_items ? (n_items - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    const int total = my_items * ksteps;
    // sources of this thread's rows for the CTA's jj-th work item: the A rows of both halves
    // (null past the expert's rows; gate_up only), the B rows (null past the expert's f gate
    // or up rows: decoded as zeros), the tile, and whether the second half holds any of the
    // expert's rows
    struct RowSrc {
      const __nv_bfloat16 *arow[kHalves];
      const uint8_t *wrow[kRows];
      uint32_t wlo[kRows];    // low 4 bits of the row's address
      bool wtail[kRows];      // the row's last windows can reach past the end of the matrix
      int tile, h1;
    };
    auto item_src = [&](int jj) -> RowSrc {
      const int item = (int)blockIdx.x + jj * (int)gridDim.x;
      const int nt = item % n_ntiles;
      int tile;
      bool h1;
      item_tile(item, tile, h1);
      const int e = W.tiles[2 * tile], m0 = W.tiles[2 * tile + 1];
      const int cnt = W.counts[e];
      RowSrc rs;
      rs.tile = tile;
      rs.h1 = h1;
#pragma unroll
      for (int h = 0; h < kHalves; ++h) {
        const int r = m0 + h * BM + row;
        rs.arow[h] = (GATEUP && r < cnt) ? a_src + (size_t)(W.perm[W.offsets[e] + r] / k) * d : nullptr;
      }
      const uint8_t *ebase = wq + (size_t)e * expert_bytes;
#pragma unroll
      for (int j = 0; j < kRows; ++j) {
        if (GATEUP) {
          // B row j * 128 + row: gate row c0 + row (j = 0) or up row f + c0 + row (j = 1)
          const int c = nt * (kBN / 2) + row;
          rs.wrow[j] = c < f ? ebase + (size_t)(j * f + c) * rb : nullptr;
        } else {
          rs.wrow[j] = ebase + (size_t)(nt * kBN + j * 128 + row) * rb;
        }
        // a K step's 64-byte window starts at most 15 bytes before its blocks and ends at most
        // 28 bytes past the row's last block
        rs.wlo[j] = (uint32_t)(reinterpret_cast<uintptr_t>(rs.wrow[j]) & 15u);
        rs.wtail[j] = rs.wrow[j] != nullptr && rs.wrow[j] + rb + 28 > wq_end;
      }
      return rs;
    };
    auto issue = [&](const RowSrc &rs, int ks, int s) {
      const uint32_t a_saddr = sbase + (uint32_t)s * kStageBytes;
      if (GATEUP) {
#pragma unroll
        for (int h = 0; h < kHalves; ++h) {
          if (h > 0 && !rs.h1) break;   // the MMA skips an empty second half
          const __nv_bfloat16 *ap = rs.arow[h] ? rs.arow[h] + (size_t)ks * BK + (size_t)hsel * (BK / 2) : a_src;
          const uint32_t tile_a = a_saddr + (uint32_t)h * kTileBytes;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint32_t chunk = (uint32_t)(hsel * 4 + c);
            cp_async16(tile_a + (uint32_t)row * 128u + ((chunk ^ (uint32_t)(row & 7)) << 4),
                       ap + (rs.arow[h] ? 8 * c : 0), rs.arow[h] ? 16u : 0u);
          }
        }
      } else if (pt == 0) {
        // the 128 x 64 tiles of h by TMA: their bytes join the stage's full barrier, whose
        // phase cannot complete before this thread's own arrival for the step (after this call)
        mbar_expect_tx(&bars.full[s], kTileBytes * (rs.h1 ? 2u : 1u));
        tma_load_2d(a_saddr, &tmap_h, ks * BK, rs.tile * BM, &bars.full[s]);
        if (rs.h1) tma_load_2d(a_saddr + kTileBytes, &tmap_h, ks * BK, rs.tile * BM + BM, &bars.full[s]);
      }
#pragma unroll
      for (int j = 0; j < kRows; ++j) {
        if (!rs.wrow[j]) continue;   // a zero row: nothing to copy
        const uint32_t kb = (uint32_t)ks * 2u * MOE_QBYTES;
        const uint8_t *wa = rs.wrow[j] + kb - ((rs.wlo[j] + kb) & 15u);   // 16-byte aligned window start
        const uint32_t rdst = raw_base + (uint32_t)s * kRawStageBytes + (uint32_t)(j * 128 + row) * kRawRowBytes +
                              (uint32_t)hsel * 32u;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const uint8_t *src = wa + hsel * 32 + c * 16;
          if (!rs.wtail[j]) {
            cp_async16(rdst + 16u * c, src, 16u);
          } else {   // the matrix's last rows: never read past its end
            const uintptr_t e = reinterpret_cast<uintptr_t>(wq_end), a = reinterpret_cast<uintptr_t>(src);
            const uint32_t nbytes = a >= e ? 0u : (e - a >= 16 ? 16u : (uint32_t)(e - a));
            cp_async16(rdst + 16u * c, nbytes ? static_cast<const void *>(src) : static_cast<const void *>(wq), nbytes);
          }
        }
      }
    };
    bool ok = true;
    // issue side and consume side walk this group's steps g = pg, pg + G, ... (G groups);
    // copies run kAhead group steps ahead of the decode
    RowSrc isrc{}, csrc{};
    int ijj = 0, iks = pg, cjj = 0, cks = pg;
    while (iks >= ksteps && ijj < my_items) { iks -= ksteps; ++ijj; }
    cjj = ijj;
    cks = iks;
    if (ijj < my_items) { isrc = item_src(ijj); csrc = isrc; }
    auto adv = [&](int &jj, int &ks, RowSrc &src) {
      ks += kProdGroups;
      bool moved = false;
      while (ks >= ksteps) { ks -= ksteps; ++jj; moved = true; }
      if (moved && jj < my_items) src = item_src(jj);
    };
    int gi = pg;
    for (int a = 0; a < kAhead; ++a, gi += kProdGroups) {   // the first stages are free
      if (gi < total) {
        issue(isrc, iks, gi % kStages);
        adv(ijj, iks, isrc);
      }
      cp_async_commit();
    }
    for (int g = pg; g < total; g += kProdGroups, gi += kProdGroups) {
      // step g: its copies have landed (issued kAhead group steps ago); decode B, hand over
      cp_async_wait<kAhead - 1>();
      __syncwarp();   // a row's window is copied by two lanes
      const int s = g % kStages;
      const uint32_t b_saddr = sbase + (uint32_t)s * kStageBytes + kBOff;
#pragma unroll
      for (int j = 0; j < kRows; ++j) {
        const int n = j * 128 + row;   // B row
        if (csrc.wrow[j]) {
          // this thread's block inside the row's window: 20 bytes from its offset rounded down to 4
          RawBlk cur;
          const uint32_t off = ((csrc.wlo[j] + (uint32_t)cks * 2u * MOE_QBYTES) & 15u) + (uint32_t)hsel * MOE_QBYTES;   // < 48
          const uint32_t *rp = reinterpret_cast<const uint32_t *>(
              smem_raw + (raw_base - smem_u32(smem_raw)) + (size_t)s * kRawStageBytes + (size_t)n * kRawRowBytes +
              (off & ~3u));
#pragma unroll
          for (int i = 0; i < 5; ++i) cur.w[i] = rp[i];
          cur.sh = (off & 3u) * 8u;
          store_blk_bf16(cur, b_saddr, n, hsel * 4);
        } else {
          store_blk_zero(b_saddr, n, hsel * 4);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&bars.full[s]);
      adv(cjj, cks, csrc);
      // then refill the stage that step gi uses, once the MMA has released it
      if (gi < total) {
        const int si = gi % kStages;
        const uint32_t par = ((uint32_t)(gi / kStages) & 1u) ^ 1u;
        if (!mbar_wait(&bars.empty[si], par, W.err, 10, W.wait_ns)) { ok = false; break; }
        issue(isrc, iks, si);
        adv(ijj, iks, isrc);
      }
      cp_async_commit();
    }
    cp_async_wait<0>();   // no copy lands after this thread leaves
    if (!ok) atomicExch(&bars.abort_flag, 1);
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issue (one thread)
    if (lane == 0) {
      int it = 0, j = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x, ++j) {
        const int b = j & 1;
        const uint32_t upar = ((uint32_t)(j >> 1) & 1u) ^ 1u;
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
      const int b = j & 1;
      const uint32_t par = (uint32_t)(j >> 1) & 1u;
      const bool ok = mbar_wait(&bars.acc_full[b], par, W.err, 13, W.wait_ns);
      if (__any_sync(0xffffffffu, !ok)) { atomicExch(&bars.abort_flag, 1); break; }
      tc_fence_after();
      const int nt = item % n_ntiles;
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
        if (GATEUP) {
          const int c0 = nt * (kBN / 2);   // first h column of this item
          __nv_bfloat16 *dst = W.hb + (size_t)((tile + h) * BM + r) * f + (size_t)c0;
#pragma unroll
          for (int c = 0; c < kBN / 2; c += 16) {
            if (c0 + c >= f) break;   // warp-uniform: the item's columns past f are zero rows
            uint32_t g[16], u[16];
            tmem_ld16(taddr + (uint32_t)c, g);
            tmem_ld16(taddr + (uint32_t)(kBN / 2 + c), u);
            tmem_ld_wait();
            uint32_t o[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float h0 = gelu_tanh_f(__uint_as_float(g[2 * i])) * __uint_as_float(u[2 * i]);
              const float hv1 = gelu_tanh_f(__uint_as_float(g[2 * i + 1])) * __uint_as_float(u[2 * i + 1]);
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
          for (int c = 0; c < kBN; c += 16) {
            uint32_t y[16];
            tmem_ld16(taddr + (uint32_t)c, y);
            tmem_ld_wait();
            uint32_t o[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
              o[i] = pack_bf16(__uint_as_float(y[2 * i]) * scale, __uint_as_float(y[2 * i + 1]) * scale);
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

int moe_launch_gemm_experts(const MoeLaunch &L, const MoeWork &W, const void *x, const uint8_t *gate_up_q4,
                            const uint8_t *down_q4, const float *expert_scale, int T, int d, int f, int E, int k,
                            float *out, int num_sms, int max_tiles) {
  // K of both GEMMs in whole 64-wide steps; down's output in whole 128-column tiles
  if (d % BK || d % GemmCfg<false>::kBN || f % BK) return -2;
  static unsigned long long smem_ok[2] = {0ull, 0ull};   // per device, per kernel
  if (!moe_allow_dyn_smem(reinterpret_cast<const void *>(k_moe_gemm<true>), &smem_ok[0]) ||
      !moe_allow_dyn_smem(reinterpret_cast<const void *>(k_moe_gemm<false>), &smem_ok[1]))
    return -1;
  moe_prof_mark(L.stream, MOE_K_GEMM_GATEUP, true);
  const uint8_t *gu_end = gate_up_q4 + (size_t)E * 2 * f * (d / MOE_QK) * MOE_QBYTES;
  const uint8_t *dn_end = down_q4 + (size_t)E * d * (f / MOE_QK) * MOE_QBYTES;
  CUtensorMap th;
  if (!make_tmap_h(&th, W.hb, f, (long long)max_tiles * BM)) return -1;
  constexpr int kSmemG = GemmCfg<true>::kSmemBytes, kSmemD = GemmCfg<false>::kSmemBytes;
  k_moe_gemm<true><<<num_sms, kThreads, kSmemG, L.stream>>>(th, static_cast<const __nv_bfloat16 *>(x), gate_up_q4,
                                                            gu_end, expert_scale, d, f, k, W);
  if (launch_err()) return -1;
  moe_prof_count(1);
  moe_prof_mark(L.stream, MOE_K_GEMM_GATEUP, false);
  moe_prof_mark(L.stream, MOE_K_GEMM_DOWN, true);
  k_moe_gemm<false><<<num_sms, kThreads, kSmemD, L.stream>>>(th, W.hb, down_q4, dn_end, expert_scale, d, f, k, W);
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
