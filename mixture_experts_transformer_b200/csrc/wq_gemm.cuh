// Grouped GEMM with the weights in a weight-only format, SFP8 or Q4_0 (the
// formats the pages name by their footprint; readings below), activations in
// bf16. The tensor cores take bf16 operands, so converter warps decode each
// stage's weight codes into bf16 and write them straight into tensor memory,
// where the MMA reads them as its A operand: the product is computed
// transposed, D^T = W^T X^T, with the tile's 128 weight columns as M (TMEM
// lanes) and its token rows as N (rounded up to 16). The decoded weights never
// pass through shared memory, which at small batches would otherwise carry
// three times the code bytes (codes in, bf16 out, bf16 read by the MMA).
//
//   GATEUP: h[row, n] = gelu_tanh(X Wg^)[row, n] * (X Wu^)[row, n]   (bf16 out)
//   DOWN:   y[row, n] = (X Wd^)[row, n]                              (bf16 or fp32 out)
//
// Formats (one [K, N] Linear; weights quantised along K, their input axis):
//   SFP8 - sign bit and a 7-bit magnitude code m: 0 is zero; m in [1, 63] is
//          (1 + (m & 3) / 4) 2^((m >> 2) - 23); m in [64, 127] is
//          (1 + (m & 7) / 8) 2^(((m >> 3) & 7) - 7); one fp32 scale S per
//          matrix (amax / 1.875), W^ = value * S. Every value is a bf16
//          number, so the decoded weights are exact and S multiplies the fp32
//          sums in the epilogue.
//   Q4_0 - blocks of 32 along K, fp16 scale d and 4-bit codes q, W^ = (q - 8) d;
//          (q - 8) d has up to 15 significant bits, so the decoded weight is
//          rounded to bf16 (nearest even) before the MMA.
//
// Storage (built by wq_quant_kernel): the transposed weight (row n = output
// column n) in 128-row blocks and 64-deep K blocks, each piece contiguous so
// that a stage brings it with one bulk copy:
//   SFP8: [G][ceil(N/128)][K/64][128 rows x 64 B codes]                     8192 B
//   Q4_0: [G][ceil(N/128)][K/64][128 rows x 32 B codes | 128 rows x 2 fp16]  4608 B
// A row's codes are 16-byte pieces in K order, piece j stored at position
// j ^ ((r >> 1) & 3) (SFP8) or j ^ ((r >> 2) & 1) (Q4_0) of row r, so that the
// 32 rows a converter warp reads at once spread over all shared-memory banks.
// (Q4_0: element 2i of a piece in the low nibble of its byte i; a row's two
// scales cover K 0-31 and 32-63 of the block.) Rows past N hold zeros.
//
// Roles (512 threads, one CTA per SM; 16 warps, so 4 per SM sub-partition):
//   warp 0        producer: tiles from the work counter into the tile ring,
//                 and the token rows of every stage into the X ring (TMA)
//   warp 1        MMA issuer: waits for a stage's token rows and decoded
//                 weights, 4 x (one or two) tcgen05.mma (K = 16, A in TMEM)
//   warps 2..5    epilogue, one per TMEM lane quarter (32 weight columns)
//   warps 6..13   converters: warp 6 + 4 b + q decodes rows 32 q .. 32 q + 31
//                 of weight block b of a stage (one row per thread) into TMEM
//                 lanes 32 q .. (tcgen05.st), then arrives
//   warps 14, 15  the weight blocks of every stage (block 0 and block 1) into
//                 the code ring by bulk copy
// Each ring is freed by its reader: X slots and TMEM weight stages by the MMAs'
// commits, code slots by the converters once they have read them, so the
// weight stream runs as far ahead as the code ring is deep.
// Shared memory: X ring 4 x 16 KB, code ring 128 KB. TMEM: the two
// accumulators D0, D1 (128 columns each: block 0 and block 1 of the tile)
// and 4 stages of decoded weights (32 columns per block).
#pragma once

#include <cuda_fp16.h>

#include "grouped_gemm.cuh"

namespace moe {

constexpr int kWfSfp8 = 1;
constexpr int kWfQ4 = 2;

template <int FMT>
__host__ __device__ constexpr int wq_block_bytes() {
  return FMT == kWfSfp8 ? 8192 : 4608;
}

constexpr int kWqXStages = 4;     // token-row stages (shared memory)
constexpr int kWqTStages = 4;     // decoded-weight stages (TMEM)
constexpr int kWqEpiWarps = 4;
constexpr int kWqConvWarps = 8;
constexpr int kWqCopyWarps = 2;  // the two weight-block issuers
constexpr int kWqThreads = 32 * (2 + kWqEpiWarps + kWqConvWarps + kWqCopyWarps);
constexpr int kWqCodeRing = 128 * 1024;         // code ring bytes
constexpr int kWqMaxCStages = 16;
constexpr uint32_t kWqDCols = 128;               // one accumulator: 128 lanes x up to 128 token columns
constexpr uint32_t kWqTCol0 = 2 * kWqDCols;      // first TMEM column of the weight stages
constexpr uint32_t kWqTStageCols = 64;           // a stage: block 0 at +0, block 1 at +32 (64 bf16 of K each)
static_assert(kWqTCol0 + kWqTStages * kWqTStageCols <= 512, "TMEM columns");
template <int FMT>
__host__ __device__ constexpr int wq_code_stage() {  // two 128-row weight blocks
  return 2 * wq_block_bytes<FMT>();
}
template <int FMT>
__host__ __device__ constexpr int wq_cstages() {
  return kWqCodeRing / wq_code_stage<FMT>() < kWqMaxCStages ? kWqCodeRing / wq_code_stage<FMT>() : kWqMaxCStages;
}
constexpr int kWqSmemBytes = kWqXStages * kAStageBytes + kWqCodeRing + kWqEpiWarps * kStgWarpBytes +
                             1024 /*align*/ + 1024 /*barriers*/;
static_assert(kWqSmemBytes <= 232448, "shared memory per CTA");

struct WqProblem {
  int K;         // reduction length, multiple of 64
  int N;         // output columns, multiple of 64
  int groups;    // number of weight matrices (range check)
  int a_rows;    // rows of the tiles' row space (range check)
  const uint8_t* w0;  // blocks of B0 (gate, or the only weight)
  const uint8_t* w1;  // blocks of B1 (up; GATEUP only)
  const float* s0;    // SFP8 matrix scales [groups] of B0, B1 (Q4_0: unused)
  const float* s1;
  void* out;     // [a_rows, ldo] bf16 or fp32
  int ldo;
  int out_f32;
};

struct WqParams {
  CUtensorMap tmA[2];   // activations [a_rows, K] bf16, box 64 x 128, 128-byte swizzle
  CUtensorMap tmAs[2];  // the same, box 64 x 32 (tiles of at most 32 rows)
  WqProblem prob[2];
  int nprob;
  int a_small;
  const Tile* tiles;
  const int32_t* num_tiles;
  int32_t* next_tile;
  uint32_t* err;
};

// Output columns of a tile: GATEUP 128 per projection, DOWN 256 (fewer at the end).
template <bool GATEUP>
__device__ __forceinline__ int wq_tile_cols(const WqProblem& pr, int n0) {
  const int cap = GATEUP ? 128 : 256;
  const int rem = pr.N - n0;
  return rem < cap ? rem : cap;
}

// bf16 bit pattern of an SFP8 code (sign included).
__host__ __device__ inline uint16_t sfp8_bf16_bits(uint32_t code) {
  const uint32_t m = code & 0x7Fu;
  uint32_t bits = 0;
  if (m >= 64)
    bits = ((((m >> 3) & 7u) + 120u) << 7) | ((m & 7u) << 4);  // 2^(e - 7), 3 mantissa bits
  else if (m > 0)
    bits = (((m >> 2) + 104u) << 7) | ((m & 3u) << 5);  // 2^(e - 23), 2 mantissa bits
  return static_cast<uint16_t>(bits | ((code & 0x80u) << 8));
}

// Per 16-bit half, the smaller of a and b (unsigned).
__device__ __forceinline__ uint32_t min_u16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("min.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// Two SFP8 codes, in bytes 0 and 2 of v (bytes 1 and 3 are ignored), to two
// bf16 bit patterns, in packed 16-bit lanes: m >= 64 -> 0x3800 + 16 m,
// 1 <= m < 64 -> 0x3400 + 32 m, m = 0 -> 0, sign to bit 15. The two linear
// pieces meet at m = 64 (0x3C00); below it 0x3400 + 32 m is the smaller, above
// it 0x3800 + 16 m, so their minimum is the value, and a third term, 0 for
// m = 0 and 0x7FFF otherwise, makes the minimum 0 for the zero code. Mostly
// multiply-adds; equal to sfp8_bf16_bits for all 2^16 code pairs.
__device__ __forceinline__ uint32_t sfp8x2_to_bf16x2(uint32_t v) {
  const uint32_t m = v & 0x007F007Fu;
  const uint32_t lg = m * 16u + 0x38003800u;
  const uint32_t sm = m * 32u + 0x34003400u;
  const uint32_t z = min_u16x2(m, 0x00010001u) * 0x7FFFu;
  return (v & 0x00800080u) * 256u + min_u16x2(min_u16x2(lg, sm), z);
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Bulk copy of `bytes` (a multiple of 16, both addresses 16-byte aligned) into
// this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// 32 consecutive 32-bit TMEM columns of this warp's 32 lanes from registers.
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
      "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
      "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait_all() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// tcgen05.mma kind::f16 with A in tensor memory (M = 128 lanes, 16 bf16 of K
// packed in 8 columns) and B from a shared-memory descriptor.
__device__ __forceinline__ void umma_f16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                                uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Epilogue stores of a transposed accumulator: thread `lane` holds column
// `lane` of 32 output rows (a[i] = row i). The values go through the warp's
// 4 KB staging buffer as fp32 [32 rows][32 columns] (16-byte pieces XOR-
// swizzled by row, conflict-free both ways), then the warp stores 16 bytes
// per lane along the rows. Rows at or past rows_valid are not stored.
__device__ __forceinline__ void stage_cols_f32x32(uint8_t* stg, const uint32_t (&a)[32], int lane) {
#pragma unroll
  for (int i = 0; i < 32; ++i)
    *reinterpret_cast<uint32_t*>(stg + i * 128 + (((lane >> 2) ^ (i & 7)) << 4) + (lane & 3) * 4) = a[i];
  __syncwarp();
}

__device__ __forceinline__ void store_cols_f32x32(uint8_t* stg, const uint32_t (&a)[32], int lane, float* base,
                                                  size_t ldo, int rows_valid) {
  stage_cols_f32x32(stg, a, lane);
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int row = it * 4 + (lane >> 3), c = lane & 7;  // 8 pieces of 16 B per row
    const uint4 v = *reinterpret_cast<const uint4*>(stg + row * 128 + ((c ^ (row & 7)) << 4));
    if (row < rows_valid) *reinterpret_cast<uint4*>(base + static_cast<size_t>(row) * ldo + c * 4) = v;
  }
  __syncwarp();
}

__device__ __forceinline__ void store_cols_bf16x32(uint8_t* stg, const uint32_t (&a)[32], int lane,
                                                   __nv_bfloat16* base, size_t ldo, int rows_valid) {
  stage_cols_f32x32(stg, a, lane);
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int row = it * 8 + (lane >> 2), v = lane & 3;  // 4 pieces of 8 bf16 per row
    const uint4 lo = *reinterpret_cast<const uint4*>(stg + row * 128 + (((2 * v) ^ (row & 7)) << 4));
    const uint4 hi = *reinterpret_cast<const uint4*>(stg + row * 128 + (((2 * v + 1) ^ (row & 7)) << 4));
    const uint4 pk = make_uint4(pack_bf16x2(__uint_as_float(lo.x), __uint_as_float(lo.y)),
                                pack_bf16x2(__uint_as_float(lo.z), __uint_as_float(lo.w)),
                                pack_bf16x2(__uint_as_float(hi.x), __uint_as_float(hi.y)),
                                pack_bf16x2(__uint_as_float(hi.z), __uint_as_float(hi.w)));
    if (row < rows_valid) *reinterpret_cast<uint4*>(base + static_cast<size_t>(row) * ldo + v * 8) = pk;
  }
  __syncwarp();
}

// Decoded row of one weight block for one stage: the 64 K of row r (codes at
// `blk`, swizzled as stored) as 32 packed bf16x2 words, word c = K 2c, 2c + 1.
template <int FMT>
__device__ __forceinline__ void wq_decode_row(const uint8_t* blk, int r, uint32_t (&out)[32]) {
  if (FMT == kWfSfp8) {
    const uint8_t* row = blk + r * 64;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint4 w = *reinterpret_cast<const uint4*>(row + ((j ^ ((r >> 1) & 3)) << 4));  // K 16 j .. 16 j + 15
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        out[8 * j + 2 * i] = sfp8x2_to_bf16x2(__byte_perm(ws[i], 0u, 0x4140));
        out[8 * j + 2 * i + 1] = sfp8x2_to_bf16x2(__byte_perm(ws[i], 0u, 0x4342));
      }
    }
  } else {
    const uint8_t* row = blk + r * 32;
    const __half2 dd = *reinterpret_cast<const __half2*>(blk + 4096 + r * 4);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      // A nibble q at bit 8 (12) of a word, or'ed into the mantissa of 1.0, is
      // the float f = 1 + q 2^-15 (1 + q 2^-11); one fma f A + B with
      // A = d 2^15, B = -d (2^15 + 8) (2^11 for bit 12) gives (q - 8) d: A and
      // B are exact (at most 13 x 11 significant bits), and so is (q - 8) d
      // (4 x 11), so the fma's one rounding leaves it exact; then one
      // rounding to bf16.
      const float d = __half2float(j ? dd.y : dd.x);
      const float a8 = __fmul_rn(d, 32768.0f), b8 = __fmul_rn(d, -32776.0f);
      const float a12 = __fmul_rn(d, 2048.0f), b12 = __fmul_rn(d, -2056.0f);
      const uint4 w = *reinterpret_cast<const uint4*>(row + ((j ^ ((r >> 2) & 1)) << 4));  // K 32 j .. 32 j + 31
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t x[4] = {ws[i] << 8, ws[i], ws[i] >> 8, ws[i] >> 16};  // elements 2qq, 2qq + 1 at bits 8, 12
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          const float lo = __uint_as_float((x[qq] & 0x00000F00u) | 0x3F800000u);
          const float hi = __uint_as_float((x[qq] & 0x0000F000u) | 0x3F800000u);
          out[16 * j + 4 * i + qq] = pack_bf16x2(__fmaf_rn(lo, a8, b8), __fmaf_rn(hi, a12, b12));
        }
      }
    }
  }
}

template <int FMT, bool GATEUP>
__global__ void __launch_bounds__(kWqThreads, 1) wq_gemm_kernel(const __grid_constant__ WqParams P) {
  constexpr int kBlk = wq_block_bytes<FMT>();
  constexpr int kCS = wq_code_stage<FMT>();
  constexpr int kCStages = wq_cstages<FMT>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sX = smem;
  uint8_t* sC = sX + kWqXStages * kAStageBytes;
  uint8_t* sStg = sC + kWqCodeRing;
  uint64_t* xfull = reinterpret_cast<uint64_t*>(sStg + kWqEpiWarps * kStgWarpBytes);
  uint64_t* xempty = xfull + kWqXStages;
  uint64_t* cfull = xempty + kWqXStages;
  uint64_t* cempty = cfull + kWqMaxCStages;
  uint64_t* tfull = cempty + kWqMaxCStages;
  uint64_t* tempty = tfull + kWqTStages;
  uint64_t* acc_full = tempty + kWqTStages;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint64_t* tile_full = drain + 1;
  uint64_t* tile_empty = tile_full + kTileRing;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tile_empty + kTileRing);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* tile_ring = abort_flag + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr int kConv0 = 2 + kWqEpiWarps;          // first converter warp
  constexpr int kCopy0 = kConv0 + kWqConvWarps;    // first weight-block issuer warp

  if (threadIdx.x == 0) {
    for (int s = 0; s < kWqXStages; ++s) {
      mbar_init(&xfull[s], 1);
      mbar_init(&xempty[s], 1);  // the MMAs have read the token rows
    }
    for (int s = 0; s < kCStages; ++s) {
      mbar_init(&cfull[s], kWqCopyWarps);   // one arrival (with its bytes) per block issuer
      mbar_init(&cempty[s], kWqConvWarps);  // every converter warp has read the codes
    }
    for (int t = 0; t < kWqTStages; ++t) {
      mbar_init(&tfull[t], kWqConvWarps);   // the stage's weights are in TMEM
      mbar_init(&tempty[t], 1);             // the MMAs have read them
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kWqEpiWarps);
    mbar_init(drain, 1);
    for (int r = 0; r < kTileRing; ++r) {
      mbar_init(&tile_full[r], 1);
      mbar_init(&tile_empty[r], 1 + kWqEpiWarps + kWqConvWarps + kWqCopyWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int p = 0; p < P.nprob; ++p) {
      tma_prefetch_desc(&P.tmA[p]);
      if (P.a_small) tma_prefetch_desc(&P.tmAs[p]);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait_then_release();
  const int num_tiles = *P.num_tiles;

  auto tile_ok = [&](const Tile& tile) -> bool {
    const int p = tile.pg >> 16, g = tile.pg & 0xFFFF;
    if (p >= P.nprob) return false;
    const WqProblem& pr = P.prob[p];
    return !(g >= pr.groups || tile.row0 < 0 || tile.row0 >= pr.a_rows || tile.rows < 1 || tile.rows > kBM ||
             tile.n0 < 0 || tile.n0 >= pr.N || (tile.n0 & 127) || tile.kb0 != 0 || tile.kbn != 0 ||
             tile.rows1 != 0);
  };
  // after an abort: let an issuer's copies in flight land before the CTA's memory goes away
  auto drain_ring = [&](uint64_t* full_bars, int nst, int s_now, uint32_t ph_now, int issued) {
    int st = s_now;
    uint32_t sp = ph_now;
    const int pending = issued < nst ? issued : nst;
    for (int i = 0; i < pending; ++i) {
      if (--st < 0) {
        st = nst - 1;
        sp ^= 1;
      }
      uint32_t dummy = 0;
      mbar_wait(&full_bars[st], sp, reinterpret_cast<volatile int*>(&dummy), P.err, 100000000ull);
    }
  };
  // A reader of the tile ring (MMA, epilogue, converter and block-issuer
  // warps): the next tile index, or -1 at the end / on abort.
  auto next_from_ring = [&](int& rs, uint32_t& rph, bool warp_wide) -> int {
    const bool got = mbar_wait(&tile_full[rs], rph, abort_flag, P.err);
    int ti = got ? tile_ring[rs] : -1;
    if (warp_wide) __syncwarp();
    if ((!warp_wide || lane == 0) && got) mbar_arrive(&tile_empty[rs]);
    if (++rs == kTileRing) {
      rs = 0;
      rph ^= 1;
    }
    return warp_wide ? __shfl_sync(0xffffffffu, ti, 0) : ti;
  };
  // Weight block b of a tile exists: GATEUP always two (gate, up); DOWN the
  // second only past the tile's first 128 columns.
  auto has_block = [&](int b, int wn) -> bool { return GATEUP || b == 0 || wn > kBM; };

  if (warp == 0) {
    // --------------------------------------- producer (tiles, token rows)
    int s = 0, issued = 0;
    uint32_t ph = 0;
    int rs = 0;
    uint32_t rph = 0;
    int ti = 0;
    if (lane == 0) ti = atomicAdd(P.next_tile, 1);
    ti = __shfl_sync(0xffffffffu, ti, 0);
    while (true) {
      int pub = 1;
      if (lane == 0) {
        pub = mbar_wait(&tile_empty[rs], rph ^ 1, abort_flag, P.err);
        if (pub) {
          tile_ring[rs] = ti < num_tiles ? ti : -1;
          mbar_arrive(&tile_full[rs]);
        }
      }
      if (!__shfl_sync(0xffffffffu, pub, 0)) break;
      if (++rs == kTileRing) {
        rs = 0;
        rph ^= 1;
      }
      if (ti >= num_tiles) break;
      int next = 0;
      if (lane == 0) next = atomicAdd(P.next_tile, 1);
      const Tile tile = P.tiles[ti];
      if (!tile_ok(tile)) {
        if (lane == 0) {
          atomicOr(P.err, kErrBadTile);
          *abort_flag = 1;
        }
        break;
      }
      const int p = tile.pg >> 16;
      const bool a_small = P.a_small && tile.rows <= kASmallRows;
      const int kb_end = P.prob[p].K / kBK;
      bool ok = true;
      for (int kb = 0; kb < kb_end; ++kb) {
        int waited = 1;
        if (lane == 0) {
          waited = mbar_wait(&xempty[s], ph ^ 1, abort_flag, P.err);
          if (waited) {
            mbar_arrive_expect_tx(&xfull[s], a_small ? kASmallBytes : kAStageBytes);
            tma_load_2d(sX + s * kAStageBytes, a_small ? &P.tmAs[p] : &P.tmA[p], &xfull[s], kb * kBK, tile.row0);
          }
        }
        if (!__shfl_sync(0xffffffffu, waited, 0)) {
          ok = false;
          break;
        }
        ++issued;
        if (++s == kWqXStages) {
          s = 0;
          ph ^= 1;
        }
      }
      if (!ok) break;
      ti = __shfl_sync(0xffffffffu, next, 0);
    }
    __syncwarp();
    if (lane == 0 && *abort_flag) drain_ring(xfull, kWqXStages, s, ph, issued);
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------- MMA issuer
      int s = 0, t = 0;
      uint32_t ph = 0, tph = 0, acc_ph = 0;
      bool any = false;
      int rs = 0;
      uint32_t rph = 0;
      while (true) {
        const int ti = next_from_ring(rs, rph, false);
        if (ti < 0) break;
        const Tile tile = P.tiles[ti];
        const int p = tile.pg >> 16;
        if (p >= P.nprob) break;
        const WqProblem& pr = P.prob[p];
        const bool two = has_block(1, wq_tile_cols<GATEUP>(pr, tile.n0));
        const uint32_t idesc = idesc_bf16_m128((tile.rows + 15) & ~15, 0);  // N = the rows; B K-major
        const int kb_end = pr.K / kBK;
        if (!mbar_wait(acc_empty, acc_ph ^ 1, abort_flag, P.err)) break;
        tc_fence_after_sync();
        bool ok = true;
        for (int kb = 0; kb < kb_end; ++kb) {
          if (!mbar_wait(&xfull[s], ph, abort_flag, P.err) || !mbar_wait(&tfull[t], tph, abort_flag, P.err)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t x_addr = smem_u32(sX + s * kAStageBytes);
          const uint32_t a0 = tmem_base + kWqTCol0 + t * kWqTStageCols;
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            // token rows: K-major, rows of 128 B, 8-row groups 1024 B apart; +32 B per 16 K;
            // weights in TMEM: 16 bf16 of K in 8 columns
            const uint64_t bd = sdesc_sw128(x_addr + k * 32, 16, 1024);
            umma_f16_tmem_a(tmem_base, a0 + 8 * k, bd, idesc, (kb | k) != 0);
            if (two) umma_f16_tmem_a(tmem_base + kWqDCols, a0 + 32 + 8 * k, bd, idesc, (kb | k) != 0);
          }
          any = true;
          umma_commit(&xempty[s]);  // token rows of this stage read
          umma_commit(&tempty[t]);  // decoded weights read
          if (++s == kWqXStages) {
            s = 0;
            ph ^= 1;
          }
          if (++t == kWqTStages) {
            t = 0;
            tph ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(acc_full);
        acc_ph ^= 1;
      }
      if (any) {
        umma_commit(drain);
        uint32_t dummy = 0;
        mbar_wait(drain, 0, reinterpret_cast<volatile int*>(&dummy), P.err);
      }
    }
  } else if (warp >= kCopy0) {
    // ------------------------------------------------- weight-block issuers
    // Warp kCopy0 + q copies block q of every stage (GATEUP: q = 0 gate, 1 up;
    // DOWN: the tile's first and, past 128 columns, second 128-row block).
    const int q = warp - kCopy0;
    if (lane == 0) {
      int s = 0, issued = 0;
      uint32_t ph = 0;
      int rs = 0;
      uint32_t rph = 0;
      while (true) {
        const int ti = next_from_ring(rs, rph, false);
        if (ti < 0) break;
        const Tile tile = P.tiles[ti];
        if (!tile_ok(tile)) break;  // the producer reports it
        const int p = tile.pg >> 16, g = tile.pg & 0xFFFF;
        const WqProblem& pr = P.prob[p];
        const bool mine = has_block(q, wq_tile_cols<GATEUP>(pr, tile.n0));
        const int nb = (pr.N + 127) / 128, kbs = pr.K / kBK;
        const uint8_t* w = (GATEUP && q) ? pr.w1 : pr.w0;
        const int row_blk = (tile.n0 >> 7) + (GATEUP ? 0 : q);
        const uint8_t* src = w + (static_cast<size_t>(g) * nb + row_blk) * kbs * kBlk;
        bool ok = true;
        for (int kb = 0; kb < kbs; ++kb) {
          if (!mbar_wait(&cempty[s], ph ^ 1, abort_flag, P.err)) {
            ok = false;
            break;
          }
          if (mine) {
            mbar_arrive_expect_tx(&cfull[s], kBlk);
            bulk_copy_g2s(sC + s * kCS + q * kBlk, src + static_cast<size_t>(kb) * kBlk, kBlk, &cfull[s]);
          } else {
            mbar_arrive(&cfull[s]);
          }
          ++issued;
          if (++s == kCStages) {
            s = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
      }
      if (*abort_flag) drain_ring(cfull, kCStages, s, ph, issued);
    }
  } else if (warp >= kConv0) {
    // ------------------------------------------------------- converters
    // Warp kConv0 + 4 b + j: weight block b, rows 32 q .. 32 q + 31 with
    // q = warp % 4 (the TMEM lane quarter this warp may write), one row per
    // thread: its 64 codes -> 32 bf16x2 columns of TMEM lane 32 q + lane.
    const int cb = (warp - kConv0) >> 2;  // the block
    const int r = (warp & 3) * 32 + lane;  // the row within it
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    int s = 0, t = 0;
    uint32_t ph = 0, tph = 0;
    int rs = 0;
    uint32_t rph = 0;
    while (true) {
      const int ti = next_from_ring(rs, rph, true);
      if (ti < 0) break;
      const Tile tile = P.tiles[ti];
      if (!tile_ok(tile)) break;
      const WqProblem& pr = P.prob[tile.pg >> 16];
      const bool mine = has_block(cb, wq_tile_cols<GATEUP>(pr, tile.n0));
      const int kb_end = pr.K / kBK;
      bool ok = true;
      for (int kb = 0; kb < kb_end; ++kb) {
        const bool got =
            mbar_wait(&cfull[s], ph, abort_flag, P.err) && mbar_wait(&tempty[t], tph ^ 1, abort_flag, P.err);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        uint32_t v[32];
        if (mine) wq_decode_row<FMT>(sC + s * kCS + cb * kBlk, r, v);
        __syncwarp();
        if (lane == 0) mbar_arrive(&cempty[s]);  // this warp is done with the stage's codes
        if (mine) {
          tc_fence_after_sync();
          tmem_st_32x32b_x32(tmem_base + lane_off + kWqTCol0 + t * kWqTStageCols + 32 * cb, v);
          tmem_st_wait_all();
        }
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tfull[t]);
        if (++s == kCStages) {
          s = 0;
          ph ^= 1;
        }
        if (++t == kWqTStages) {
          t = 0;
          tph ^= 1;
        }
      }
      if (!ok) break;
    }
  } else {
    // ----------------------------------------------------------- epilogue
    // lane = weight column 32 quarter + lane of D0 (block 0) and D1 (block 1);
    // TMEM column j = the tile's row j. Stores transposed through the warp's
    // staging buffer.
    const int quarter = warp & 3;
    uint32_t acc_ph = 0;
    int rs = 0;
    uint32_t rph = 0;
    uint8_t* stg = sStg + (warp - 2) * kStgWarpBytes;
    while (true) {
      const int ti = next_from_ring(rs, rph, true);
      if (ti < 0) break;
      const Tile tile = P.tiles[ti];
      const int p = tile.pg >> 16, g = tile.pg & 0xFFFF;
      if (p >= P.nprob) break;
      const WqProblem& pr = P.prob[p];
      const int wn = wq_tile_cols<GATEUP>(pr, tile.n0);
      const bool ready = mbar_wait(acc_full, acc_ph, abort_flag, P.err);
      __syncwarp();
      if (!ready) break;
      acc_ph ^= 1;
      tc_fence_after_sync();
      const uint32_t t0 = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
      const float sc0 = (FMT == kWfSfp8 && pr.s0) ? pr.s0[g] : 1.0f;
      const float sc1 = (FMT == kWfSfp8 && pr.s1) ? pr.s1[g] : 1.0f;
      const int n_tok = tile.rows;
      if (GATEUP) {
        // gate in D0, up in D1, both for columns n0 + 32 quarter + lane
        if (quarter * 32 < wn) {
          __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(pr.out) + static_cast<size_t>(tile.row0) * pr.ldo +
                               tile.n0 + quarter * 32;
          for (int j = 0; j < n_tok; j += 32) {
            uint32_t gt[32], up[32];
            tmem_ld_32x32b_x32(t0 + j, gt);
            tmem_ld_32x32b_x32(t0 + kWqDCols + j, up);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i)
              gt[i] = __float_as_uint(gelu_tanh(__uint_as_float(gt[i]) * sc0) * (__uint_as_float(up[i]) * sc1));
            store_cols_bf16x32(stg, gt, lane, out + static_cast<size_t>(j) * pr.ldo, pr.ldo, n_tok - j);
          }
        }
      } else {
        // D0: columns n0 + 32 quarter + lane, D1: the same plus 128
        for (int b = 0; b < 2; ++b) {
          const int c = b * kBM + quarter * 32;
          if (c >= wn) continue;
          for (int j = 0; j < n_tok; j += 32) {
            uint32_t a[32];
            tmem_ld_32x32b_x32(t0 + b * kWqDCols + j, a);
            tmem_ld_wait();
            if (FMT == kWfSfp8) {
#pragma unroll
              for (int i = 0; i < 32; ++i) a[i] = __float_as_uint(__uint_as_float(a[i]) * sc0);
            }
            const size_t off = static_cast<size_t>(tile.row0 + j) * pr.ldo + tile.n0 + c;
            if (pr.out_f32)
              store_cols_f32x32(stg, a, lane, reinterpret_cast<float*>(pr.out) + off, pr.ldo, n_tok - j);
            else
              store_cols_bf16x32(stg, a, lane, reinterpret_cast<__nv_bfloat16*>(pr.out) + off, pr.ldo, n_tok - j);
          }
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// --------------------------------------------------------------- quantiser

// SFP8 magnitude of code m (0..127) as a float.
__device__ __forceinline__ float sfp8_value(int m) {
  return __uint_as_float(static_cast<uint32_t>(sfp8_bf16_bits(static_cast<uint32_t>(m))) << 16);
}

// Nearest SFP8 code of v (ties to the even code; saturating at 1.875; sign
// kept). Table values have at most 4 significant bits, so |v| minus a
// neighbouring table value is exact in fp32 and the comparison is exact.
__device__ __forceinline__ uint8_t sfp8_encode_dev(float v) {
  const float a = fminf(fabsf(v), 1.875f);
  int lo = 0, hi = 127;  // largest m with value(m) <= a
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (sfp8_value(mid) <= a) lo = mid; else hi = mid - 1;
  }
  int m = lo;
  if (lo < 127) {
    const float dl = a - sfp8_value(lo), dh = sfp8_value(lo + 1) - a;
    if (dh < dl || (dh == dl && ((lo + 1) & 1) == 0)) m = lo + 1;
  }
  return static_cast<uint8_t>(m | (signbit(v) ? 0x80 : 0));
}

// S = amax / 1.875 (1 for an all-zero matrix), from the amax bit patterns.
__global__ void sfp8_scale_kernel(const uint32_t* __restrict__ amax_bits, float* __restrict__ s, int n) {
  pdl_wait_then_release();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float a = __uint_as_float(amax_bits[i]);
  s[i] = a > 0.f ? __fdiv_rn(a, 1.875f) : 1.0f;
}

// One thread per (group, output column n, 64-deep K block) of w [G][K][N]
// (N contiguous): that column's 64 weights into the block layout above (the
// destination must be zeroed beforehand, so padding rows stay zero). SFP8
// takes the matrix scales s; Q4_0 computes its block scales itself.
template <int FMT>
__global__ void wq_quant_kernel(const __nv_bfloat16* __restrict__ w, int K, int N, const float* __restrict__ s,
                                uint8_t* __restrict__ out) {
  pdl_wait_then_release();
  constexpr int kBlk = wq_block_bytes<FMT>();
  const int g = blockIdx.y;
  const int kbs = K / kBK, nb = (N + 127) / 128;
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<long long>(N) * kbs) return;
  const int n = static_cast<int>(idx % N), kb = static_cast<int>(idx / N);
  const __nv_bfloat16* col = w + (static_cast<size_t>(g) * K + static_cast<size_t>(kb) * kBK) * N + n;
  uint8_t* blk = out + ((static_cast<size_t>(g) * nb + (n >> 7)) * kbs + kb) * kBlk;
  const int r = n & 127;
  float x[kBK];
#pragma unroll
  for (int i = 0; i < kBK; ++i) x[i] = __bfloat162float(col[static_cast<size_t>(i) * N]);
  if (FMT == kWfSfp8) {
    const float sc = s[g];
    uint32_t words[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      uint32_t wd = 0;
#pragma unroll
      for (int b = 0; b < 4; ++b) wd |= static_cast<uint32_t>(sfp8_encode_dev(__fdiv_rn(x[4 * j + b], sc))) << (8 * b);
      words[j] = wd;
    }
    uint4* dst = reinterpret_cast<uint4*>(blk + r * 64);  // piece j at position j ^ ((r >> 1) & 3)
#pragma unroll
    for (int j = 0; j < 4; ++j)
      dst[j ^ ((r >> 1) & 3)] = make_uint4(words[4 * j], words[4 * j + 1], words[4 * j + 2], words[4 * j + 3]);
  } else {
    uint32_t words[8];
    __half scales[2];
#pragma unroll
    for (int hb = 0; hb < 2; ++hb) {
      // the first element of largest magnitude, sign kept (element 0 when all are zero)
      float m = x[32 * hb];
#pragma unroll
      for (int i = 1; i < 32; ++i)
        if (fabsf(x[32 * hb + i]) > fabsf(m)) m = x[32 * hb + i];
      const float d = __fdiv_rn(m, -8.0f);
      const float inv = d != 0.f ? __fdiv_rn(1.0f, d) : 0.f;
      scales[hb] = __float2half_rn(d);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t wd = 0;
#pragma unroll
        for (int b = 0; b < 8; ++b) {
          const float t = __fadd_rn(__fmul_rn(x[32 * hb + 8 * j + b], inv), 8.5f);
          const int q = min(15, static_cast<int>(truncf(t)));
          wd |= static_cast<uint32_t>(q) << (4 * b);
        }
        words[4 * hb + j] = wd;
      }
    }
    uint4* dst = reinterpret_cast<uint4*>(blk + r * 32);  // piece j at position j ^ ((r >> 2) & 1)
    dst[(r >> 2) & 1] = make_uint4(words[0], words[1], words[2], words[3]);
    dst[((r >> 2) & 1) ^ 1] = make_uint4(words[4], words[5], words[6], words[7]);
    __half2 hs;
    hs.x = scales[0];
    hs.y = scales[1];
    *reinterpret_cast<__half2*>(blk + 4096 + r * 4) = hs;
  }
}

}  // namespace moe
