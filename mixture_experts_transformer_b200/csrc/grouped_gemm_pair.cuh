// The grouped GEMM of grouped_gemm.cuh on SM pairs (large batches).
//
// A cluster of two CTAs on an SM pair works on one pair tile of the paired
// tile lists: two 128-row blocks of one expert (the even CTA's block row0,
// the odd CTA's block row1) and one column tile. The even CTA issues
// tcgen05.mma.cta_group::2 with M = 256: each CTA holds its own 128 A rows and
// HALF of the B columns in its shared memory, and receives its 128 rows x N
// fp32 accumulator in its own TMEM. Against the single-SM kernel each SM moves
// 32 KB instead of 48 KB per 64-deep K step for the same MMA work, so six
// stages (192 KB) cover ~1.5 us of load latency at the tensor-core rate, and
// the accumulators stay double-buffered (2 x 256 TMEM columns).
//
//   GATEUP: the even CTA loads the gate columns, the odd CTA the same columns
//           of the up weights; TMEM columns [0, wn) = x Bg, [wn, 2 wn) = x Bu.
//   DOWN:   the even CTA loads output columns [n0, n0 + wn/2), the odd CTA the
//           rest; requires wn % 128 == 0.
//
// Roles per CTA (320 threads): warp 0 lane 0 TMA producer (both CTAs; copies
// complete on the even CTA's stage barrier), warp 1 lane 0 of the even CTA
// issues the MMAs, warps 2..9 drain their CTA's accumulator (GeGLU or convert,
// staged stores). Both CTAs walk the same tiles (static, cluster-strided).
// Every mbarrier wait is bounded; both CTAs always reach the two cluster
// barriers (start and end), so a timeout in one CTA cannot strand the other.
#pragma once

#include "grouped_gemm.cuh"

namespace moe {

// Arrive without release semantics, for the barrier that hands the peer's
// MMA thread back an accumulator: its tcgen05.ld results are in registers
// (tcgen05.wait::ld and tcgen05.fence::before_thread_sync come first), and a
// release at cluster scope would first wait for every global store of the
// epilogue to complete.
__device__ __forceinline__ void mbar_arrive_cluster_relaxed(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

constexpr int kP2Stages = 6;
constexpr int kP2AStage = kBM * kBK * 2;        // 16 KB: this CTA's 128 rows
constexpr int kP2BStage = 2 * kBChunkBytes;     // 16 KB: this CTA's half of B (<= 128 columns)
constexpr int kP2StageTotal = kP2Stages * (kP2AStage + kP2BStage);
constexpr int kP2SmemBytes = kP2StageTotal + kEpiWarps * kStgWarpBytes + 1024 + 512;

template <bool GATEUP>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ GemmParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kP2Stages * kP2AStage;
  uint8_t* sStg = smem + kP2StageTotal;
  uint64_t* full = reinterpret_cast<uint64_t*>(sStg + kEpiWarps * kStgWarpBytes);
  uint64_t* empty = full + kP2Stages;
  uint64_t* acc_full = empty + kP2Stages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kP2Stages; ++s) {
      mbar_init(&full[s], 1);   // the even CTA's producer arms it; both CTAs' copies complete on it
      mbar_init(&empty[s], 1);  // the MMA commit, multicast to both CTAs
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 2 * kEpiWarps);  // every epilogue warp of both CTAs
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init_cluster();
  }
  if (warp == 0 && lane == 0) {
    for (int p = 0; p < P.nprob; ++p) {
      tma_prefetch_desc(&P.tmA[p]);
      tma_prefetch_desc(&P.tmB0[p]);
      if (GATEUP) tma_prefetch_desc(&P.tmB1[p]);
      if (P.bw_chunks) {
        tma_prefetch_desc(&P.tmBw0[p]);
        if (GATEUP) tma_prefetch_desc(&P.tmBw1[p]);
      }
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before_sync();
  cluster_sync();  // both CTAs' barriers initialised and TMEM allocated
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait_then_release();
  const int num_tiles = *P.num_tiles;
  const uint32_t full_even = mapa_shared(&full[0], 0);
  const uint32_t acc_empty_even = mapa_shared(&acc_empty[0], 0);
  // Both CTAs walk the tiles in the same static cluster-strided order. (A work
  // counter shared through the pair's shared memory measured slower here.)
  const int cid = static_cast<int>(cluster_id_x());
  const int ncl = static_cast<int>(nclusters_x());

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ TMA producer
      int s = 0, issued = 0;
      uint32_t ph = 0;
      const uint64_t wpol = l2_policy_evict_first();  // streamed weights go before activations
      for (int ti = cid; ti < num_tiles; ti += ncl) {
        const Tile tile = P.tiles[ti];
        const int p = tile.pg >> 16, g = tile.pg & 0xFFFF;
        const bool bad_p = p >= P.nprob;
        const GemmProblem& pr = P.prob[bad_p ? 0 : p];
        const bool has1 = tile.rows1 > 0;
        const int wn = tile_cols<GATEUP>(pr, tile.n0);
        if (bad_p || g >= pr.groups || tile.row0 < 0 || tile.row0 >= pr.a_rows || tile.rows < 1 ||
            tile.rows > kBM || tile.n0 < 0 || tile.n0 >= pr.N || (!GATEUP && (wn & 127)) ||
            (has1 && (tile.row1 < 0 || tile.row1 >= pr.a_rows || tile.rows1 > kBM))) {
          atomicOr(P.err, kErrBadTile);
          *abort_flag = 1;
          break;
        }
        const int nch = GATEUP ? wn >> 6 : wn >> 7;  // this CTA's 64-column chunks of B
        const bool my_a = leader || has1;
        const uint32_t both = (has1 ? 2 : 1) * kP2AStage + 2 * nch * kBChunkBytes;
        const int row = leader ? tile.row0 : tile.row1;
        const int col0 = GATEUP ? tile.n0 : tile.n0 + static_cast<int>(rank) * (wn >> 1);
        const CUtensorMap* mb = (GATEUP && !leader) ? &P.tmB1[p] : &P.tmB0[p];
        const int nkb = pr.K / kBK;
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, P.err)) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&full[s], both);
          const uint32_t bar = full_even + 8u * s;
          if (my_a) tma_load_2d_pair(sA + s * kP2AStage, &P.tmA[p], bar, kb * kBK, row);
          if (P.bw_chunks == nch) {  // this CTA's chunks in one copy
            const CUtensorMap* mw = (GATEUP && !leader) ? &P.tmBw1[p] : &P.tmBw0[p];
            if (P.stream_weights)
              tma_load_4d_pair_hint(sB + s * kP2BStage, mw, bar, 0, kb * kBK, col0 / 64, g, wpol);
            else
              tma_load_4d_pair(sB + s * kP2BStage, mw, bar, 0, kb * kBK, col0 / 64, g);
          } else {
            for (int c = 0; c < nch; ++c)
              if (P.stream_weights)
                tma_load_3d_pair_hint(sB + s * kP2BStage + c * kBChunkBytes, mb, bar, col0 + c * 64, kb * kBK, g,
                                      wpol);
              else
                tma_load_3d_pair(sB + s * kP2BStage + c * kBChunkBytes, mb, bar, col0 + c * 64, kb * kBK, g);
          }
          ++issued;
          if (++s == kP2Stages) {
            s = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
      }
      if (leader && *abort_flag) {
        // copies of both CTAs still in flight complete on these barriers
        const int pending = issued < kP2Stages ? issued : kP2Stages;
        for (int i = 0; i < pending; ++i) {
          if (--s < 0) {
            s = kP2Stages - 1;
            ph ^= 1;
          }
          uint32_t dummy = 0;
          mbar_wait(&full[s], ph, reinterpret_cast<volatile int*>(&dummy), P.err, 100000000ull);
        }
      }
    }
  } else if (warp == 1) {
    if (leader && lane == 0) {
      // -------------------------------------------------------- MMA issuer
      int s = 0, acc = 0;
      uint32_t ph = 0, acc_ph = 0;
      for (int ti = cid; ti < num_tiles; ti += ncl) {
        const Tile tile = P.tiles[ti];
        const int p = tile.pg >> 16;
        if (p >= P.nprob) break;
        const GemmProblem& pr = P.prob[p];
        const int wn = tile_cols<GATEUP>(pr, tile.n0);
        const int n_mma = GATEUP ? 2 * wn : wn;  // over both CTAs' halves of B
        const uint32_t idesc = idesc_bf16_m256(n_mma, 1);
        const int nkb = pr.K / kBK;
        if (!mbar_wait_cluster(&acc_empty[acc], acc_ph ^ 1, abort_flag, P.err)) break;
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + acc * kAccCols;
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&full[s], ph, abort_flag, P.err)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t a_addr = smem_u32(sA + s * kP2AStage);
          const uint32_t b_addr = smem_u32(sB + s * kP2BStage);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            umma_f16_pair(d_tmem, sdesc_sw128(a_addr + k * 32, 16, 1024),
                          sdesc_sw128(b_addr + k * 2048, kBChunkBytes, 1024), idesc, (kb | k) != 0);
          umma_commit_pair(&empty[s], 0x3);  // frees the stage in both CTAs
          if (++s == kP2Stages) {
            s = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        umma_commit_pair(&acc_full[acc], 0x3);
        if (++acc == 2) {
          acc = 0;
          acc_ph ^= 1;
        }
      }
      umma_commit_pair(drain, 0x3);  // both CTAs learn when every MMA has completed
    }
  } else {
    // ------------------------------------------------------------- epilogue
    const int quarter = warp & 3;      // TMEM lanes this warp may access: 32*quarter..+31
    const int half = (warp - 2) >> 2;  // column chunks j = 32 * half + 64 c
    uint8_t* stg = sStg + (warp - 2) * kStgWarpBytes;
    int acc = 0;
    uint32_t acc_ph = 0;
    for (int ti = cid; ti < num_tiles; ti += ncl) {
      const Tile tile = P.tiles[ti];
      const int p = tile.pg >> 16;
      if (p >= P.nprob) break;
      const GemmProblem& pr = P.prob[p];
      const int wn = tile_cols<GATEUP>(pr, tile.n0);
      const bool ready = mbar_wait(&acc_full[acc], acc_ph, abort_flag, P.err);
      __syncwarp();
      if (!ready) break;
      tc_fence_after_sync();
      const uint32_t tbase = tmem_base + acc * kAccCols + (static_cast<uint32_t>(quarter * 32) << 16);
      const int t_rows = leader ? tile.rows : tile.rows1;
      const int t_row0 = leader ? tile.row0 : tile.row1;
      const int rows_valid = t_rows - quarter * 32;  // of this warp's 32 rows
      const size_t wrow = static_cast<size_t>(t_row0 + quarter * 32);
      if (rows_valid > 0) {
        if (GATEUP) {
          __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(pr.out) + wrow * pr.ldo + tile.n0;
          for (int j = 32 * half; j < wn; j += 64) {
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
          for (int j = 32 * half; j < wn; j += 64) {
            uint32_t a[32];
            tmem_ld_32x32b_x32(tbase + j, a);
            tmem_ld_wait();
            if (pr.out_f32) {
              store_rows_f32x32(stg, a, lane, reinterpret_cast<float*>(pr.out) + wrow * pr.ldo + tile.n0 + j, pr.ldo,
                                rows_valid);
            } else {
              uint32_t pk[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(__uint_as_float(a[2 * i]), __uint_as_float(a[2 * i + 1]));
              store_rows_bf16x32(stg, pk, lane, reinterpret_cast<__nv_bfloat16*>(pr.out) + wrow * pr.ldo + tile.n0 + j,
                                 pr.ldo, rows_valid);
            }
          }
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster_relaxed(acc_empty_even + 8u * acc);
      if (++acc == 2) {
        acc = 0;
        acc_ph ^= 1;
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  // No MMA may still write either CTA's TMEM, and no copy may still target
  // either CTA's shared memory, when the pair deallocates and exits.
  if (warp == 1 && lane == 0) {
    uint32_t dummy = 0;
    mbar_wait(drain, 0, reinterpret_cast<volatile int*>(&dummy), P.err);
  }
  __syncwarp();
  tc_fence_before_sync();
  cluster_sync();
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc_pair(tmem_base, kTmemCols);
}

}  // namespace moe
