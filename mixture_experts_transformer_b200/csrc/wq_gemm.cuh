// Grouped GEMM with the weights in a weight-only format, SFP8 or Q4_0 (the
// formats the pages name by their footprint; readings below), activations in
// bf16. The tensor cores take bf16 operands, so converter warps decode each
// stage's weight codes into bf16 in shared memory, in the 128-byte-swizzled
// K-major layout the MMA reads; everything else is the grouped GEMM of
// grouped_gemm.cuh (same tile lists, epilogues and barriers).
//
//   GATEUP: h[row, n] = gelu_tanh(A Wg^)[row, n] * (A Wu^)[row, n]   (bf16 out)
//   DOWN:   y[row, n] = (A Wd^)[row, n]                              (bf16 or fp32 out)
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
// (Q4_0: element 2j of a row's 64 in the low nibble of byte j; a row's two
// scales cover K 0-31 and 32-63 of the block.) Rows past N hold zeros.
//
// Roles (512 threads, one CTA per SM; 16 warps, so 4 per SM sub-partition):
//   warp 0        producer: tiles from the work counter into the tile ring,
//                 and the A rows of every stage into the A ring
//   warp 1        MMA issuer: waits for a stage's A rows and decoded weights,
//                 4 x tcgen05.mma (K = 16), frees both
//   warps 2..5    epilogue, one per TMEM lane quarter
//   warps 6..13   converters: a stage's codes -> bf16 weights (K-major, 128-byte
//                 swizzle) in a 2-deep ring, then a proxy fence and arrival
//   warps 14, 15  the weight blocks of every stage (block 0 and block 1) into
//                 the code ring (one thread issues ~2.2 M copies per second,
//                 so the A copy and the two block copies go to three threads)
// The rings are separate: A slots are freed by the MMAs, code slots by the
// converters as soon as they have read them. The weight stream, which carries
// nearly all of the bytes at small batches, so runs as far ahead as the code
// ring is deep (5 stages of SFP8, 8 of Q4_0), not only as far as the
// converters may run ahead of the MMAs.
// Shared memory: A ring 4 x 16 KB, code ring 80 KB, decoded weights 2 x 32 KB.
// TMEM: 2 accumulators x 256 columns.
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

constexpr int kWqAStages = 4;
constexpr int kWqBStages = 2;
constexpr int kWqEpiWarps = 4;
constexpr int kWqConvWarps = 8;
constexpr int kWqCopyWarps = 2;  // the two weight-block issuers
constexpr int kWqThreads = 32 * (2 + kWqEpiWarps + kWqConvWarps + kWqCopyWarps);
constexpr int kWqConvThreads = 32 * kWqConvWarps;
constexpr int kWqCodeRing = 80 * 1024;          // code ring bytes
constexpr int kWqMaxCStages = 8;
template <int FMT>
__host__ __device__ constexpr int wq_code_stage() {  // two 128-row weight blocks
  return 2 * wq_block_bytes<FMT>();
}
template <int FMT>
__host__ __device__ constexpr int wq_cstages() {
  return kWqCodeRing / wq_code_stage<FMT>() < kWqMaxCStages ? kWqCodeRing / wq_code_stage<FMT>() : kWqMaxCStages;
}
constexpr int kWqBStage = 256 * kBK * 2;        // 256 weight rows x 64 K bf16
constexpr int kWqSmemBytes = kWqAStages * kAStageBytes + kWqCodeRing + kWqBStages * kWqBStage +
                             kWqEpiWarps * kStgWarpBytes + 1024 /*align*/ + 512 /*barriers*/;
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

// Bytes 0 and 2 of x, each replaced by copies of its top bit, in both bytes
// of their 16-bit halves: prmt's sign-replicating selectors (CUDA's
// __byte_perm keeps only the byte-select bits of a selector).
__device__ __forceinline__ uint32_t replicate_top_bits_b02(uint32_t x) {
  uint32_t r;
  asm("prmt.b32 %0, %1, 0, 0xAA88;" : "=r"(r) : "r"(x));
  return r;
}

// Two SFP8 codes, in bytes 0 and 2 of v (bytes 1 and 3 are ignored), to two
// bf16 bit patterns: m >= 64 -> 0x3800 + 16 m, 1 <= m < 64 -> 0x3400 + 32 m,
// m = 0 -> 0, sign to bit 15. Both candidates are computed in packed 16-bit
// lanes and selected by per-lane masks spread from one bit of each code
// (bit 6: m >= 64; the carry of m + 127 into bit 7: m != 0). Equal to
// sfp8_bf16_bits for all 2^16 code pairs.
__device__ __forceinline__ uint32_t sfp8x2_to_bf16x2(uint32_t v) {
  const uint32_t m = v & 0x007F007Fu;
  const uint32_t lg = m * 16u + 0x38003800u;
  const uint32_t sm = m * 32u + 0x34003400u;
  const uint32_t big = replicate_top_bits_b02(v << 1);
  const uint32_t nz = replicate_top_bits_b02(m + 0x007F007Fu);
  return (((lg & big) | (sm & ~big)) & nz) | ((v << 8) & 0x80008000u);
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

template <int FMT, bool GATEUP>
__global__ void __launch_bounds__(kWqThreads, 1) wq_gemm_kernel(const __grid_constant__ WqParams P) {
  constexpr int kBlk = wq_block_bytes<FMT>();
  constexpr int kCS = wq_code_stage<FMT>();
  constexpr int kCStages = wq_cstages<FMT>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + kWqAStages * kAStageBytes;
  uint8_t* sC = sB + kWqBStages * kWqBStage;
  uint8_t* sStg = sC + kWqCodeRing;
  uint64_t* afull = reinterpret_cast<uint64_t*>(sStg + kWqEpiWarps * kStgWarpBytes);
  uint64_t* aempty = afull + kWqAStages;
  uint64_t* cfull = aempty + kWqAStages;
  uint64_t* cempty = cfull + kWqMaxCStages;
  uint64_t* bfull = cempty + kWqMaxCStages;
  uint64_t* bempty = bfull + kWqBStages;
  uint64_t* acc_full = bempty + kWqBStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
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
    for (int s = 0; s < kWqAStages; ++s) {
      mbar_init(&afull[s], 1);
      mbar_init(&aempty[s], 1);  // the MMAs have read the A rows
    }
    for (int s = 0; s < kCStages; ++s) {
      mbar_init(&cfull[s], kWqCopyWarps);   // one arrival (with its bytes) per block issuer
      mbar_init(&cempty[s], kWqConvWarps);  // every converter warp has read the codes
    }
    for (int b = 0; b < kWqBStages; ++b) {
      mbar_init(&bfull[b], kWqConvWarps);
      mbar_init(&bempty[b], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], kWqEpiWarps);
    }
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

  if (warp == 0) {
    // ------------------------------------------- producer (tiles, A rows)
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
          waited = mbar_wait(&aempty[s], ph ^ 1, abort_flag, P.err);
          if (waited) {
            mbar_arrive_expect_tx(&afull[s], a_small ? kASmallBytes : kAStageBytes);
            tma_load_2d(sA + s * kAStageBytes, a_small ? &P.tmAs[p] : &P.tmA[p], &afull[s], kb * kBK, tile.row0);
          }
        }
        if (!__shfl_sync(0xffffffffu, waited, 0)) {
          ok = false;
          break;
        }
        ++issued;
        if (++s == kWqAStages) {
          s = 0;
          ph ^= 1;
        }
      }
      if (!ok) break;
      ti = __shfl_sync(0xffffffffu, next, 0);
    }
    __syncwarp();
    if (lane == 0 && *abort_flag) drain_ring(afull, kWqAStages, s, ph, issued);
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------- MMA issuer
      int s = 0, b = 0, acc = 0;
      uint32_t ph = 0, bph = 0, acc_ph = 0;
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
        const int wn = wq_tile_cols<GATEUP>(pr, tile.n0);
        const uint32_t idesc = idesc_bf16_m128(GATEUP ? 2 * wn : wn, 0);  // B K-major
        const int kb_end = pr.K / kBK;
        if (!mbar_wait(&acc_empty[acc], acc_ph ^ 1, abort_flag, P.err)) break;
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + acc * kAccCols;
        bool ok = true;
        for (int kb = 0; kb < kb_end; ++kb) {
          if (!mbar_wait(&afull[s], ph, abort_flag, P.err) || !mbar_wait(&bfull[b], bph, abort_flag, P.err)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t a_addr = smem_u32(sA + s * kAStageBytes);
          const uint32_t b_addr = smem_u32(sB + b * kWqBStage);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            // both operands K-major, rows of 128 B, 8-row groups 1024 B apart; +32 B per 16 K
            const uint64_t ad = sdesc_sw128(a_addr + k * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(b_addr + k * 32, 16, 1024);
            umma_f16(d_tmem, ad, bd, idesc, (kb | k) != 0);
          }
          any = true;
          umma_commit(&aempty[s]);  // A of this stage read
          umma_commit(&bempty[b]);  // decoded weights read
          if (++s == kWqAStages) {
            s = 0;
            ph ^= 1;
          }
          if (++b == kWqBStages) {
            b = 0;
            bph ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&acc_full[acc]);
        if (++acc == 2) {
          acc = 0;
          acc_ph ^= 1;
        }
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
        const int wn = wq_tile_cols<GATEUP>(pr, tile.n0);
        const bool mine = GATEUP || q == 0 || wn > 128;
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
    // Item i of a stage: weight row r = i / 8 (B row: GATEUP gate rows
    // 0..wn-1 then up rows, DOWN output columns), 16-byte piece c = i % 8
    // (K 8c..8c+7 of the stage's 64).
    const int ct = threadIdx.x - 32 * kConv0;
    int s = 0, b = 0;
    uint32_t ph = 0, bph = 0;
    int rs = 0;
    uint32_t rph = 0;
    while (true) {
      const int ti = next_from_ring(rs, rph, true);
      if (ti < 0) break;
      const Tile tile = P.tiles[ti];
      if (!tile_ok(tile)) break;
      const WqProblem& pr = P.prob[tile.pg >> 16];
      const int wn = wq_tile_cols<GATEUP>(pr, tile.n0);
      const int rows_b = GATEUP ? 2 * wn : wn;
      const int kb_end = pr.K / kBK;
      bool ok = true;
      for (int kb = 0; kb < kb_end; ++kb) {
        const bool got =
            mbar_wait(&cfull[s], ph, abort_flag, P.err) && mbar_wait(&bempty[b], bph ^ 1, abort_flag, P.err);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        const uint8_t* cs = sC + s * kCS;
        uint8_t* bs = sB + b * kWqBStage;
        // A thread's (up to) kIt items of the stage: all code loads first, then
        // the decodes, then the stores, so that the shared-memory latencies of
        // the items overlap instead of adding up.
        constexpr int kIt = 256 * 8 / kWqConvThreads;
        const int n_items = rows_b * 8;
        uint32_t w0[kIt], w1[kIt];
        float dsc[kIt];
#pragma unroll
        for (int j = 0; j < kIt; ++j) {
          const int i = ct + j * kWqConvThreads;
          if (i >= n_items) continue;
          const int r = i >> 3, c = i & 7;
          // which copied block, and which of its rows, holds B row r
          const int blk = GATEUP ? (r >= wn) : (r >> 7);
          const int sr = GATEUP ? (r >= wn ? r - wn : r) : (r & 127);
          const uint8_t* src = cs + blk * kBlk;
          if (FMT == kWfSfp8) {
            const uint2 raw = *reinterpret_cast<const uint2*>(src + sr * 64 + 8 * c);
            w0[j] = raw.x;
            w1[j] = raw.y;
          } else {
            w0[j] = *reinterpret_cast<const uint32_t*>(src + sr * 32 + 4 * c);
            dsc[j] = __half2float(*reinterpret_cast<const __half*>(src + 4096 + sr * 4 + 2 * (c >> 2)));
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&cempty[s]);  // this warp is done with the stage's codes
        uint4 o[kIt];
#pragma unroll
        for (int j = 0; j < kIt; ++j) {
          const int i = ct + j * kWqConvThreads;
          if (i >= n_items) continue;
          uint32_t v[4];
          if (FMT == kWfSfp8) {
            // two codes per 32-bit word (one per 16-bit half), decoded together
            v[0] = sfp8x2_to_bf16x2(__byte_perm(w0[j], 0u, 0x4140));
            v[1] = sfp8x2_to_bf16x2(__byte_perm(w0[j], 0u, 0x4342));
            v[2] = sfp8x2_to_bf16x2(__byte_perm(w1[j], 0u, 0x4140));
            v[3] = sfp8x2_to_bf16x2(__byte_perm(w1[j], 0u, 0x4342));
          } else {
            // A nibble q at bit 8 (12) of a word, or'ed into the mantissa of
            // 1.0, is the float f = 1 + q 2^-15 (1 + q 2^-11); one fma
            // f A + B with A = d 2^15, B = -d (2^15 + 8) (2^11 for bit 12)
            // gives (q - 8) d: A and B are exact (at most 13 x 11 significant
            // bits), and so is (q - 8) d (4 x 11), so the fma's one rounding
            // leaves it exact; then one rounding to bf16.
            const float d = dsc[j];
            const float a8 = __fmul_rn(d, 32768.0f), b8 = __fmul_rn(d, -32776.0f);
            const float a12 = __fmul_rn(d, 2048.0f), b12 = __fmul_rn(d, -2056.0f);
            const uint32_t x[4] = {w0[j] << 8, w0[j], w0[j] >> 8, w0[j] >> 16};  // elements 2qq, 2qq + 1 at bits 8, 12
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
              const float lo = __uint_as_float((x[qq] & 0x00000F00u) | 0x3F800000u);
              const float hi = __uint_as_float((x[qq] & 0x0000F000u) | 0x3F800000u);
              v[qq] = pack_bf16x2(__fmaf_rn(lo, a8, b8), __fmaf_rn(hi, a12, b12));
            }
          }
          o[j] = make_uint4(v[0], v[1], v[2], v[3]);
        }
#pragma unroll
        for (int j = 0; j < kIt; ++j) {
          const int i = ct + j * kWqConvThreads;
          if (i >= n_items) continue;
          const int r = i >> 3, c = i & 7;
          *reinterpret_cast<uint4*>(bs + (r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4)) = o[j];
        }
        fence_proxy_async_smem();  // the MMA reads these bytes through the async proxy
        __syncwarp();
        if (lane == 0) mbar_arrive(&bfull[b]);
        if (++s == kCStages) {
          s = 0;
          ph ^= 1;
        }
        if (++b == kWqBStages) {
          b = 0;
          bph ^= 1;
        }
      }
      if (!ok) break;
    }
  } else {
    // ----------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    int acc = 0;
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
      const bool ready = mbar_wait(&acc_full[acc], acc_ph, abort_flag, P.err);
      __syncwarp();
      if (!ready) break;
      tc_fence_after_sync();
      const uint32_t tbase = tmem_base + acc * kAccCols + (static_cast<uint32_t>(quarter * 32) << 16);
      const int rows_valid = tile.rows - quarter * 32;
      const size_t wrow = static_cast<size_t>(tile.row0 + quarter * 32);
      const float sc0 = (FMT == kWfSfp8 && pr.s0) ? pr.s0[g] : 1.0f;
      const float sc1 = (FMT == kWfSfp8 && pr.s1) ? pr.s1[g] : 1.0f;
      if (rows_valid > 0) {
        if (GATEUP) {
          __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(pr.out) + wrow * pr.ldo + tile.n0;
          for (int j = 0; j < wn; j += 32) {
            uint32_t gt[32], up[32];
            tmem_ld_32x32b_x32(tbase + j, gt);
            tmem_ld_32x32b_x32(tbase + wn + j, up);
            tmem_ld_wait();
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float h0 = gelu_tanh(__uint_as_float(gt[2 * i]) * sc0) * (__uint_as_float(up[2 * i]) * sc1);
              const float h1 =
                  gelu_tanh(__uint_as_float(gt[2 * i + 1]) * sc0) * (__uint_as_float(up[2 * i + 1]) * sc1);
              pk[i] = pack_bf16x2(h0, h1);
            }
            store_rows_bf16x32(stg, pk, lane, out + j, pr.ldo, rows_valid);
          }
        } else {
          for (int j = 0; j < wn; j += 32) {
            uint32_t a[32];
            tmem_ld_32x32b_x32(tbase + j, a);
            tmem_ld_wait();
            if (FMT == kWfSfp8) {
#pragma unroll
              for (int i = 0; i < 32; ++i) a[i] = __float_as_uint(__uint_as_float(a[i]) * sc0);
            }
            if (pr.out_f32) {
              store_rows_f32x32(stg, a, lane, reinterpret_cast<float*>(pr.out) + wrow * pr.ldo + tile.n0 + j, pr.ldo,
                                rows_valid);
            } else {
              uint32_t pk[16];
#pragma unroll
              for (int i = 0; i < 16; ++i)
                pk[i] = pack_bf16x2(__uint_as_float(a[2 * i]), __uint_as_float(a[2 * i + 1]));
              store_rows_bf16x32(stg, pk, lane,
                                 reinterpret_cast<__nv_bfloat16*>(pr.out) + wrow * pr.ldo + tile.n0 + j, pr.ldo,
                                 rows_valid);
            }
          }
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_ph ^= 1;
      }
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
    uint4* dst = reinterpret_cast<uint4*>(blk + r * 64);
#pragma unroll
    for (int j = 0; j < 4; ++j) dst[j] = make_uint4(words[4 * j], words[4 * j + 1], words[4 * j + 2], words[4 * j + 3]);
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
    uint4* dst = reinterpret_cast<uint4*>(blk + r * 32);
    dst[0] = make_uint4(words[0], words[1], words[2], words[3]);
    dst[1] = make_uint4(words[4], words[5], words[6], words[7]);
    __half2 hs;
    hs.x = scales[0];
    hs.y = scales[1];
    *reinterpret_cast<__half2*>(blk + 4096 + r * 4) = hs;
  }
}

}  // namespace moe
