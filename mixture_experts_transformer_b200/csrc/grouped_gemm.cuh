// Persistent grouped GEMM on the 5th-generation tensor cores (tcgen05 + TMEM),
// fed by TMA. One launch runs up to two "problems" (the routed experts and the
// shared MLP) as a single list of 128-row work tiles built on the device.
//
//   GATEUP: h[row, n] = gelu_tanh(A Bg)[row, n] * (A Bu)[row, n]   (bf16 out)
//   DOWN:   y[row, n] = (A Bd)[row, n]                            (bf16 or fp32 out)
//
// A is [rows, K] bf16, K-major (the activations). B is [groups, K, N] bf16 with
// N contiguous (the weights exactly as given), which the tensor core reads as
// an MN-major operand, so no weight is repacked.
//
// Roles (384 threads, one CTA per SM):
//   warp 0      TMA producer: schedules the tiles (work counter, tile ring) and,
//               with warps 10 and 11, issues each stage's copies (copy i of a
//               stage from thread i % 3: the A rows, the gate chunks, the up
//               chunks): one thread issues ~2.2 M copies per second however many
//               are in flight, and more issuing warps scale that (measured).
//               Per stage: A tile 128x64 and B chunks 64(K)x64(N),
//               in as few copies as the tile allows (one 256-row box for the
//               two row blocks of a paired tile, a 32-row box for a tile of at
//               most 32 rows, one box for all of a projection's chunks through
//               a 4-D view of B): measured, the copy count per stage matters as
//               much as the bytes. Small batches stream B with an L2
//               evict-first policy (each weight tile is read by one row block).
//               A tile may cover a K range only (split-K partial sums).
//   warp 1      MMA issuer (one thread): 4 x tcgen05.mma (K = 16) per stage
//   warps 2..9  epilogue, two warps per TMEM lane quarter (each half of the
//               column chunks): tcgen05.ld the fp32 accumulator, apply GeGLU
//               or convert, store rows that belong to the tile
//   warps 10,11 copy warps: lane 0 reads each tile from the ring and issues
//               copy threads 1 and 2's share of its stages
// Shared memory: 4 stages x (16 KB A + 32 KB B), 128-byte swizzle.
// TMEM: 2 accumulator buffers x 256 fp32 columns, so the epilogue of one tile
// overlaps the main loop of the next.
//
// GATEUP tiles put 64-column chunks of the gate weights and the same columns
// of the up weights side by side in shared memory, so ONE MMA of N = 2*wn
// computes both projections of wn output columns (wn = 128, or 64 for the
// last columns): TMEM columns [0, wn) hold x Bg, [wn, 2 wn) hold x Bu.
//
// PAIRED (large batches): a tile carries two 128-row blocks of the same
// expert and column tile; each stage holds both A blocks and one B, the MMA
// thread issues two M=128 MMAs per K step into two 256-column accumulators,
// and epilogue warps 2..5 / 6..9 drain one each. Sharing B cuts the bytes per
// FLOP by a third and 3 stages of 64 KB keep ~1.6 us of loads in flight, which
// is what lets the tensor cores run at their rate instead of waiting on data.
// The accumulators then fill TMEM, so they are single-buffered.
#pragma once

#include "ptx.cuh"

namespace moe {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kStages = 4;
constexpr int kAStageBytes = kBM * kBK * 2;   // 16 KB
constexpr int kBChunkBytes = kBK * 64 * 2;    // 8 KB: 64 K-rows x 64 N-columns
constexpr int kMaxBChunks = 4;
constexpr int kASmallRows = 32;                  // rows of the small A box
constexpr int kASmallBytes = kASmallRows * kBK * 2;  // 4 KB
constexpr int kBStageBytes = kMaxBChunks * kBChunkBytes;
constexpr int kAccCols = 256;
constexpr int kTmemCols = 512;
constexpr int kGemmThreads = 320;
// The single-SM grouped GEMM issues a stage's copies from kNProd threads in
// different warps (warp 0 and warps 10, 11): one thread issues ~2.2 M TMA
// copies per second however many are in flight, and more issuing warps
// scale that linearly (measured).
constexpr int kNProd = 3;
constexpr int kGemmThreadsSm = kGemmThreads + 32 * (kNProd - 1);
constexpr int kEpiWarps = 8;
constexpr int kTileRing = 8;  // tile indices handed from the producer to the MMA and epilogue warps
constexpr int kStageBytesTotal = kStages * (kAStageBytes + kBStageBytes);
constexpr int kStgWarpBytes = 4096;  // epilogue staging: 32 rows x 128 B per warp
constexpr int kGemmSmemBytes = kStageBytesTotal + kEpiWarps * kStgWarpBytes + 1024 /*align*/ + 512 /*barriers, ring*/;

// One 128-row work tile. pg = (problem << 16) | group. 16-byte aligned so a
// tile moves as two vector accesses.
struct __align__(16) Tile {
  int32_t pg;
  int32_t row0;   // first A row
  int32_t rows;   // rows of A that belong to this tile (1..128)
  int32_t n0;     // first output column (per projection for GATEUP)
  int32_t row1;   // PAIRED: first row of the second 128-row block; split-K tiles: the split
  int32_t rows1;  // PAIRED: its rows (0: no second block)
  int32_t kb0;    // first 64-deep K block
  int32_t kbn;    // K blocks of the tile (0: the whole reduction)
};

struct GemmProblem {
  int K;        // reduction length, multiple of 64
  int N;        // output columns, multiple of 64
  int groups;   // number of B matrices (range check)
  int a_rows;   // rows of the tiles' row space (range check)
  void* out;    // [a_rows, ldo] bf16 or fp32
  int ldo;
  int out_f32;
  // split-K (down GEMM, fp32 out): a tile with kbn != 0 adds up K blocks
  // [kb0, kb0 + kbn) only and writes its partial sums at out + row1 * split_stride
  long long split_stride;
};

struct GemmParams {
  CUtensorMap tmA[2];   // [a_rows, K] bf16, box 64 x 128
  CUtensorMap tmB0[2];  // [groups, K, N] bf16, box 64 x 64 x 1 (gate, or the only B)
  CUtensorMap tmB1[2];  // [groups, K, N] bf16 (up; GATEUP only)
  // Wide boxes: fewer copy instructions per stage for the same bytes.
  // tmA2: box 64 x 256, the two consecutive 128-row blocks of a paired tile
  // (a_wide). tmBw0 / tmBw1: B viewed as [groups][N / 64][K][64] (64-column
  // chunks as a dimension), box 64 x 64 x bw_chunks x 1: bw_chunks adjacent
  // chunks in one copy, landing 8 KB apart as the per-chunk copies do.
  CUtensorMap tmA2[2];
  CUtensorMap tmBw0[2];
  CUtensorMap tmBw1[2];
  // tmAs: box 64 x 32 (a_small): a tile of at most 32 rows (small batches
  // spread over many experts) copies only those; the other 96 rows of its A
  // stage are left as they are, and the accumulator rows they feed are never
  // stored.
  CUtensorMap tmAs[2];
  int a_wide;
  int a_small;
  int bw_chunks;  // 0: per-chunk copies only
  GemmProblem prob[2];
  int nprob;
  // 1: every weight tile is read by one row block (small batches), so B loads
  // carry an L2 evict-first policy and the activations keep the cache
  int stream_weights;
  const Tile* tiles;
  const int32_t* num_tiles;
  int32_t* next_tile;  // work counter, zero at launch: CTAs take tiles in list order as they free up
  uint32_t* err;
};

template <bool GATEUP>
__device__ __forceinline__ int tile_cols(const GemmProblem& pr, int n0) {
  const int cap = GATEUP ? 128 : 256;
  const int rem = pr.N - n0;
  return rem < cap ? rem : cap;
}

template <bool GATEUP, bool PAIRED = false>
__global__ void __launch_bounds__(kGemmThreadsSm, 1) grouped_gemm_kernel(const __grid_constant__ GemmParams P) {
  constexpr int kSt = PAIRED ? 3 : kStages;
  constexpr int kAS = PAIRED ? 2 * kAStageBytes : kAStageBytes;
  static_assert(kSt * (kAS + kBStageBytes) <= kStages * (kAStageBytes + kBStageBytes), "shared memory budget");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kSt * kAS;
  uint8_t* sStg = smem + kStageBytesTotal;
  uint64_t* full = reinterpret_cast<uint64_t*>(sStg + kEpiWarps * kStgWarpBytes);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint64_t* tile_full = drain + 1;
  uint64_t* tile_empty = tile_full + kTileRing;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tile_empty + kTileRing);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* tile_ring = abort_flag + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], kNProd);  // one arrival (with its bytes) per issuing thread
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], PAIRED ? 4 : 8);  // one arrival per epilogue warp draining it
    }
    mbar_init(drain, 1);
    for (int r = 0; r < kTileRing; ++r) {
      mbar_init(&tile_full[r], 1);
      mbar_init(&tile_empty[r], 1 + kEpiWarps + (kNProd - 1));  // MMA thread, epilogue and copy warps read each index
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int p = 0; p < P.nprob; ++p) {
      tma_prefetch_desc(&P.tmA[p]);
      tma_prefetch_desc(&P.tmB0[p]);
      if (GATEUP) tma_prefetch_desc(&P.tmB1[p]);
      if (PAIRED && P.a_wide) tma_prefetch_desc(&P.tmA2[p]);
      if (P.a_small) tma_prefetch_desc(&P.tmAs[p]);
      if (P.bw_chunks) {
        tma_prefetch_desc(&P.tmBw0[p]);
        if (GATEUP) tma_prefetch_desc(&P.tmBw1[p]);
      }
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
  // everything above touched only this CTA's shared memory and TMEM; the tile
  // list, A and the outputs belong to the previous kernels
  pdl_wait_then_release();
  const int num_tiles = *P.num_tiles;

  const uint64_t wpol = l2_policy_evict_first();  // streamed weights go before activations
  // A tile's fields, checked before any copy is addressed from them.
  auto tile_ok = [&](const Tile& tile) -> bool {
    const int p = tile.pg >> 16, g = tile.pg & 0xFFFF;
    if (p >= P.nprob) return false;
    const GemmProblem& pr = P.prob[p];
    const bool has1 = PAIRED && tile.rows1 > 0;
    const int kb_all = pr.K / kBK;
    return !(g >= pr.groups || tile.row0 < 0 || tile.row0 >= pr.a_rows || tile.rows < 1 || tile.rows > kBM ||
             tile.n0 < 0 || tile.n0 >= pr.N || (tile.n0 & 63) ||
             (has1 && (tile.row1 < 0 || tile.row1 >= pr.a_rows || tile.rows1 > kBM)) || tile.kb0 < 0 ||
             tile.kbn < 0 || tile.kb0 + (tile.kbn ? tile.kbn : kb_all) > kb_all ||
             (tile.kbn && (GATEUP || !pr.out_f32 || tile.row1 < 0)));
  };
  // The copies of stage st (K block kb) of a tile, in a fixed order: the A
  // rows, then the B chunks. Copy i belongs to issuing thread i % kNProd;
  // returns the bytes of thread grp's copies and, with doit, issues them.
  auto stage_copies = [&](int grp, bool doit, int st, int kb, const Tile& tile) -> uint32_t {
    const int p = tile.pg >> 16, g = tile.pg & 0xFFFF;
    const GemmProblem& pr = P.prob[p];
    const bool has1 = PAIRED && tile.rows1 > 0;
    const int wn = tile_cols<GATEUP>(pr, tile.n0);
    const int cpp = wn >> 6;  // 64-column chunks per projection
    const int nch = GATEUP ? 2 * cpp : cpp;
    const bool a_small = P.a_small && !has1 && tile.rows <= kASmallRows;
    uint32_t bytes = 0;
    int i = 0;
    auto mine = [&]() { return (i++ % kNProd) == grp; };
    if (has1 && P.a_wide && tile.row1 == tile.row0 + kBM) {
      if (mine()) {  // both 128-row blocks
        bytes += 2 * kAStageBytes;
        if (doit) tma_load_2d(sA + st * kAS, &P.tmA2[p], &full[st], kb * kBK, tile.row0);
      }
    } else if (a_small) {
      if (mine()) {  // the tile's <= 32 rows
        bytes += kASmallBytes;
        if (doit) tma_load_2d(sA + st * kAS, &P.tmAs[p], &full[st], kb * kBK, tile.row0);
      }
    } else {
      if (mine()) {
        bytes += kAStageBytes;
        if (doit) tma_load_2d(sA + st * kAS, &P.tmA[p], &full[st], kb * kBK, tile.row0);
      }
      if (has1 && mine()) {
        bytes += kAStageBytes;
        if (doit) tma_load_2d(sA + st * kAS + kAStageBytes, &P.tmA[p], &full[st], kb * kBK, tile.row1);
      }
    }
    if (P.bw_chunks == cpp) {
      // each projection's cpp chunks in one copy (gate, then up at chunk cpp)
      for (int q = 0; q < (GATEUP ? 2 : 1); ++q) {
        if (!mine()) continue;
        bytes += cpp * kBChunkBytes;
        if (!doit) continue;
        void* dst = sB + st * kBStageBytes + q * cpp * kBChunkBytes;
        const CUtensorMap* mb = q ? &P.tmBw1[p] : &P.tmBw0[p];
        if (P.stream_weights)
          tma_load_4d_hint(dst, mb, &full[st], 0, kb * kBK, tile.n0 / 64, g, wpol);
        else
          tma_load_4d(dst, mb, &full[st], 0, kb * kBK, tile.n0 / 64, g);
      }
    } else {
      for (int c = 0; c < nch; ++c) {
        if (!mine()) continue;
        bytes += kBChunkBytes;
        if (!doit) continue;
        const bool up = GATEUP && c >= cpp;
        const int col = tile.n0 + (up ? c - cpp : c) * 64;
        void* dst = sB + st * kBStageBytes + c * kBChunkBytes;
        const CUtensorMap* mb = up ? &P.tmB1[p] : &P.tmB0[p];
        if (P.stream_weights)
          tma_load_3d_hint(dst, mb, &full[st], col, kb * kBK, g, wpol);
        else
          tma_load_3d(dst, mb, &full[st], col, kb * kBK, g);
      }
    }
    return bytes;
  };
  // one issuing thread's part of stage st: arm the barrier with its bytes, then copy
  auto arm_and_copy = [&](int grp, int st, int kb, const Tile& tile) {
    const uint32_t b = stage_copies(grp, false, st, kb, tile);
    if (b)
      mbar_arrive_expect_tx(&full[st], b);
    else
      mbar_arrive(&full[st]);
    stage_copies(grp, true, st, kb, tile);
  };
  // after an abort: let this thread's copies in flight land before the CTA's memory goes away
  auto drain_copies = [&](int s_now, uint32_t ph_now, int issued) {
    int st = s_now;
    uint32_t sp = ph_now;
    const int pending = issued < kSt ? issued : kSt;
    for (int i = 0; i < pending; ++i) {
      if (--st < 0) {
        st = kSt - 1;
        sp ^= 1;
      }
      uint32_t dummy = 0;
      mbar_wait(&full[st], sp, reinterpret_cast<volatile int*>(&dummy), P.err, 100000000ull);
    }
  };

  if (warp == 0) {
    // -------------------------------------------------------- TMA producer
    // The whole warp walks the tiles; lane 0 takes the next tile index from
    // the work counter, publishes it in the tile ring (-1 ends the work), and
    // issues its share of each stage's copies (copy thread 0).
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
      if (lane == 0) next = atomicAdd(P.next_tile, 1);  // its latency hides behind this tile's loads
      const Tile tile = P.tiles[ti];
      if (!tile_ok(tile)) {
        if (lane == 0) {
          atomicOr(P.err, kErrBadTile);
          *abort_flag = 1;
        }
        break;
      }
      const GemmProblem& pr = P.prob[tile.pg >> 16];
      const int kb_end = tile.kbn ? tile.kb0 + tile.kbn : pr.K / kBK;
      bool ok = true;
      for (int kb = tile.kb0; kb < kb_end; ++kb) {
        int waited = 1;
        if (lane == 0) {
          waited = mbar_wait(&empty[s], ph ^ 1, abort_flag, P.err);
          if (waited) arm_and_copy(0, s, kb, tile);
        }
        if (!__shfl_sync(0xffffffffu, waited, 0)) {
          ok = false;
          break;
        }
        ++issued;
        if (++s == kSt) {
          s = 0;
          ph ^= 1;
        }
      }
      if (!ok) break;
      ti = __shfl_sync(0xffffffffu, next, 0);
    }
    __syncwarp();
    if (lane == 0 && *abort_flag) drain_copies(s, ph, issued);
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------- MMA issuer
      int s = 0, acc = 0;
      uint32_t ph = 0, acc_ph = 0;
      bool any = false;
      int rs = 0;
      uint32_t rph = 0;
      while (true) {
        if (!mbar_wait(&tile_full[rs], rph, abort_flag, P.err)) break;
        const int ti = tile_ring[rs];
        mbar_arrive(&tile_empty[rs]);
        if (++rs == kTileRing) {
          rs = 0;
          rph ^= 1;
        }
        if (ti < 0) break;
        const Tile tile = P.tiles[ti];
        const int p = tile.pg >> 16;
        if (p >= P.nprob) break;
        const GemmProblem& pr = P.prob[p];
        const int wn = tile_cols<GATEUP>(pr, tile.n0);
        const int n_mma = GATEUP ? 2 * wn : wn;
        const uint32_t idesc = idesc_bf16_m128(n_mma, 1);
        const int kb_end = tile.kbn ? tile.kb0 + tile.kbn : pr.K / kBK;
        const bool has1 = PAIRED && tile.rows1 > 0;
        if (!mbar_wait(&acc_empty[acc], acc_ph ^ 1, abort_flag, P.err)) break;
        if (PAIRED && !mbar_wait(&acc_empty[1], acc_ph ^ 1, abort_flag, P.err)) break;
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + acc * kAccCols;
        bool ok = true;
        for (int kb = tile.kb0; kb < kb_end; ++kb) {
          const uint32_t acc_in = kb != tile.kb0;  // the tile's first K block overwrites the accumulator
          if (!mbar_wait(&full[s], ph, abort_flag, P.err)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t a_addr = smem_u32(sA + s * kAS);
          const uint32_t b_addr = smem_u32(sB + s * kBStageBytes);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            // A: K-major, rows of 128 B, 8-row groups 1024 B apart; +32 B per 16 K.
            const uint64_t ad = sdesc_sw128(a_addr + k * 32, 16, 1024);
            // B: N-major; 8 K-rows form a 1024 B swizzle atom (SBO), 64-column
            // chunks are 8 KB apart (LBO); +16 K-rows = +2048 B.
            const uint64_t bd = sdesc_sw128(b_addr + k * 2048, kBChunkBytes, 1024);
            umma_f16(d_tmem, ad, bd, idesc, acc_in | (k != 0));
            if (has1) umma_f16(tmem_base + kAccCols, sdesc_sw128(a_addr + kAStageBytes + k * 32, 16, 1024), bd, idesc,
                               acc_in | (k != 0));
          }
          any = true;
          umma_commit(&empty[s]);  // frees the stage once these MMAs have read it
          if (++s == kSt) {
            s = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&acc_full[acc]);  // accumulator(s) complete
        if (PAIRED) {
          acc_ph ^= 1;
        } else if (++acc == 2) {
          acc = 0;
          acc_ph ^= 1;
        }
      }
      if (any) {
        // all MMAs of this CTA have finished before TMEM is released
        umma_commit(drain);
        uint32_t dummy = 0;
        mbar_wait(drain, 0, reinterpret_cast<volatile int*>(&dummy), P.err);
      }
    }
  } else if (warp >= 2 + kEpiWarps) {
    // -------------------------------------------------- copy warps 10, 11
    // Lane 0 walks the tiles of the ring and issues copy thread grp's share of
    // every stage (the stage order and barriers of the producer warp).
    const int grp = warp - (1 + kEpiWarps);  // 1, 2
    if (lane == 0) {
      int s = 0, issued = 0;
      uint32_t ph = 0;
      int rs = 0;
      uint32_t rph = 0;
      while (true) {
        if (!mbar_wait(&tile_full[rs], rph, abort_flag, P.err)) break;
        const int ti = tile_ring[rs];
        mbar_arrive(&tile_empty[rs]);
        if (++rs == kTileRing) {
          rs = 0;
          rph ^= 1;
        }
        if (ti < 0) break;
        const Tile tile = P.tiles[ti];
        if (!tile_ok(tile)) break;  // the producer warp reports it
        const GemmProblem& pr = P.prob[tile.pg >> 16];
        const int kb_end = tile.kbn ? tile.kb0 + tile.kbn : pr.K / kBK;
        bool ok = true;
        for (int kb = tile.kb0; kb < kb_end; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, P.err)) {
            ok = false;
            break;
          }
          arm_and_copy(grp, s, kb, tile);
          ++issued;
          if (++s == kSt) {
            s = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
      }
      if (*abort_flag) drain_copies(s, ph, issued);
    }
  } else {
    // ----------------------------------------------------------- epilogue
    const int quarter = warp & 3;  // TMEM lanes this warp may access: 32*quarter..+31
    const int half = (warp - 2) >> 2;  // unpaired: column chunks j = 32 * half + 64 c; PAIRED: the accumulator
    const int j_first = PAIRED ? 0 : 32 * half;
    const int j_step = PAIRED ? 32 : 64;
    int acc = 0;
    uint32_t acc_ph = 0;
    int rs = 0;
    uint32_t rph = 0;
    while (true) {
      const bool got = mbar_wait(&tile_full[rs], rph, abort_flag, P.err);
      int ti = got ? tile_ring[rs] : -1;
      __syncwarp();
      if (lane == 0 && got) mbar_arrive(&tile_empty[rs]);
      if (++rs == kTileRing) {
        rs = 0;
        rph ^= 1;
      }
      ti = __shfl_sync(0xffffffffu, ti, 0);
      if (ti < 0) break;
      const Tile tile = P.tiles[ti];
      const int p = tile.pg >> 16;
      if (p >= P.nprob) break;
      const GemmProblem& pr = P.prob[p];
      const int wn = tile_cols<GATEUP>(pr, tile.n0);
      const bool ready = mbar_wait(&acc_full[acc], acc_ph, abort_flag, P.err);
      __syncwarp();
      if (!ready) break;
      tc_fence_after_sync();
      const int a_id = PAIRED ? half : acc;  // accumulator this warp drains
      const uint32_t tbase = tmem_base + a_id * kAccCols + (static_cast<uint32_t>(quarter * 32) << 16);
      const int t_rows = (PAIRED && half) ? tile.rows1 : tile.rows;
      const int t_row0 = (PAIRED && half) ? tile.row1 : tile.row0;
      const int rows_valid = t_rows - quarter * 32;  // of this warp's 32 rows
      const size_t wrow = static_cast<size_t>(t_row0 + quarter * 32);
      uint8_t* stg = sStg + (warp - 2) * kStgWarpBytes;
      if (!(PAIRED && half && t_rows <= 0)) {
      if (GATEUP) {
        __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(pr.out) + wrow * pr.ldo + tile.n0;
        for (int j = j_first; j < wn; j += j_step) {
          uint32_t g[32], u[32];
          tmem_ld_32x32b_x32(tbase + j, g);
          tmem_ld_32x32b_x32(tbase + wn + j, u);
          tmem_ld_wait();
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float h0 = gelu_tanh(__uint_as_float(g[2 * i])) * __uint_as_float(u[2 * i]);
            const float h1 = gelu_tanh(__uint_as_float(g[2 * i + 1])) * __uint_as_float(u[2 * i + 1]);
            pk[i] = pack_bf16x2(h0, h1);
          }
          store_rows_bf16x32(stg, pk, lane, out + j, pr.ldo, rows_valid);
        }
      } else {
        for (int j = j_first; j < wn; j += j_step) {
          uint32_t a[32];
          tmem_ld_32x32b_x32(tbase + j, a);
          tmem_ld_wait();
          if (pr.out_f32) {
            float* of = reinterpret_cast<float*>(pr.out) + (tile.kbn ? tile.row1 * pr.split_stride : 0);
            store_rows_f32x32(stg, a, lane, of + wrow * pr.ldo + tile.n0 + j, pr.ldo, rows_valid);
          } else {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(__uint_as_float(a[2 * i]), __uint_as_float(a[2 * i + 1]));
            store_rows_bf16x32(stg, pk, lane, reinterpret_cast<__nv_bfloat16*>(pr.out) + wrow * pr.ldo + tile.n0 + j,
                               pr.ldo, rows_valid);
          }
        }
      }
      }  // end of the drained accumulator's work
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[PAIRED ? half : acc]);
      if (PAIRED) {
        acc_ph ^= 1;
      } else if (++acc == 2) {
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

}  // namespace moe
