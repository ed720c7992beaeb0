// NVFP4 variant of the block: e2m1 values in groups of 16 along K with e4m3
// group scales and an fp32 tensor scale (G4-MeroMero-26B-A4B-NVFP4
// config.json, quantization_config.config_groups.group_0: "num_bits": 4,
// "type": float, "group_size": 16, "scale_dtype": float8_e4m3fn, strategy
// "tensor_group"; weights static, input activations "dynamic": "local"; the
// routers stay bf16, they are on the "ignore" list).
//
// Quantisation, per group of 16 values under tensor scale G (all fp32, IEEE
// round-to-nearest operations, so the codes are reproducible bit for bit):
//   G     = 448 * 6 / amax(tensor)                  (weights; activations: calibrated)
//   s     = e4m3_satfinite(RN(RN(amax16 / 6) * G))  (s = 0: the whole group is 0)
//   q_i   = e2m1_satfinite(RN(x_i * RN(G / s)))
//   x^_i  = e2m1(q_i) * s / G
//
// Storage (also the tcgen05 block-scaled operand layout):
//   codes  [rows][K/2] bytes, K-major, element 2j in the low nibble of byte j;
//   scales [rows/128][K/64][512] bytes: the 16-bit-group scales of rows
//          128a .. 128a+127 and K range 64b .. 64b+63 form one 512-byte atom,
//          row r, group c (0..3) at byte 16*(r%32) + 4*(r/32) + c.
//
// The GEMM (fp4_gemm_kernel) is the bf16 grouped GEMM's structure with
// `tcgen05.mma.kind::mxf4nvf4.block_scale.block16`: TMA brings 256-K stages of
// A and B codes plus the matching scale atoms (a bulk copy); four scale warps
// write each stage's atoms into TMEM from their registers (tcgen05.st, each
// atom row replicated to the four lane quarters), so the MMA thread's tensor
// stream holds only the MMAs: one M=128, N=256 MMA per 64-K step covering
// both 128-column halves of the tile. Eight epilogue warps (two per TMEM lane
// quarter, each half of the columns) multiply by 1/(G_act * G_weight); the
// gate|up epilogue then quantises the GeGLU rows h to NVFP4 for the down
// projection.
#pragma once

#include "grouped_gemm.cuh"
#include "ptx.cuh"
#include "router.cuh"

namespace moe {

constexpr float kFp4Max = 6.0f;
constexpr float kE4m3Max = 448.0f;

// ----------------------------------------------------------- quantisation

__device__ __forceinline__ uint32_t e4m3_code(float v) {  // v >= 0, finite
  unsigned short s;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(s) : "f"(0.0f), "f"(v));
  return s & 0xFFu;
}

__device__ __forceinline__ float e4m3_value(uint32_t c) {  // c in [0, 0x7E]
  const uint32_t e = (c >> 3) & 0xFu, m = c & 7u;
  if (e == 0) return static_cast<float>(m) * 0.001953125f;  // m * 2^-9
  return __uint_as_float(((e + 120u) << 23) | (m << 20));    // (1 + m/8) * 2^(e-7)
}

// two e2m1 codes in one byte: lo in bits 0-3, hi in bits 4-7
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Quantise 16 values under tensor scale g: returns the scale code, writes the
// 8 code bytes (little-endian: value 0 in the low nibble of byte 0) to *codes.
__device__ __forceinline__ uint32_t nvfp4_group(const float (&v)[16], float g, uint2* codes) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const uint32_t sc = e4m3_code(__fmul_rn(__fdiv_rn(amax, kFp4Max), g));
  const float sv = e4m3_value(sc);
  uint32_t w[2] = {0u, 0u};
  if (sv > 0.f) {
    const float r = __fdiv_rn(g, sv);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t word = 0;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int i = h * 8 + b * 2;
        word |= e2m1x2(__fmul_rn(v[i], r), __fmul_rn(v[i + 1], r)) << (8 * b);
      }
      w[h] = word;
    }
  }
  *codes = make_uint2(w[0], w[1]);
  return sc;
}

// Byte offset of the scale of (row, group c16) in a [rows/128][K/64][512] atom array.
__device__ __forceinline__ size_t sf_offset(int row, int c16, int k64_blocks) {
  return (static_cast<size_t>(row >> 7) * k64_blocks + (c16 >> 2)) * 512 + 16 * (row & 31) + 4 * ((row & 127) >> 5) +
         (c16 & 3);
}

__device__ __forceinline__ void load16_bf16(const __nv_bfloat16* p, float (&v)[16]) {
  const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
  const uint4 b = __ldg(reinterpret_cast<const uint4*>(p) + 1);
  const __nv_bfloat16* pa = reinterpret_cast<const __nv_bfloat16*>(&a);
  const __nv_bfloat16* pb = reinterpret_cast<const __nv_bfloat16*>(&b);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[i] = __bfloat162float(pa[i]);
    v[8 + i] = __bfloat162float(pb[i]);
  }
}

// ------------------------------------------------------- weight quantiser

// amax over each group's [K][N] matrix into amax_bits[g] (float bits; amax >= 0
// so the integer maximum is the float maximum). amax_bits must be zero.
__global__ void weight_amax_kernel(const __nv_bfloat16* __restrict__ w, size_t per_group,
                                   uint32_t* __restrict__ amax_bits) {
  pdl_wait_then_release();
  const int g = blockIdx.y;
  const __nv_bfloat16* base = w + per_group * g;
  float m = 0.f;
  for (size_t i = (static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 8; i < per_group;
       i += static_cast<size_t>(gridDim.x) * blockDim.x * 8) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(base + i));
    const __nv_bfloat16* b = reinterpret_cast<const __nv_bfloat16*>(&v);
#pragma unroll
    for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(__bfloat162float(b[j])));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits + g, __float_as_uint(m));
}

// G = 448 * 6 / amax (1 for an all-zero tensor).
__global__ void tensor_scale_kernel(const uint32_t* __restrict__ amax_bits, float* __restrict__ g, int n) {
  pdl_wait_then_release();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float a = __uint_as_float(amax_bits[i]);
  g[i] = a > 0.f ? __fdiv_rn(kE4m3Max * kFp4Max, a) : 1.0f;
}

// One thread per (n, 16-group of K) of w [G][K][N] (N contiguous): codes into
// q [G][N][K/2], scale into the atoms of sf [G][ceil(N/128)][K/64][512]
// (cleared beforehand, so padding rows keep scale 0).
__global__ void weight_quant_kernel(const __nv_bfloat16* __restrict__ w, int K, int N, const float* __restrict__ gs,
                                    uint8_t* __restrict__ q, uint8_t* __restrict__ sf) {
  pdl_wait_then_release();
  const int g = blockIdx.y;
  const int kg_count = K / 16;
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<long long>(N) * kg_count) return;
  const int n = static_cast<int>(idx % N);
  const int kg = static_cast<int>(idx / N);
  const __nv_bfloat16* src = w + (static_cast<size_t>(g) * K + kg * 16) * N + n;
  float v[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __bfloat162float(src[static_cast<size_t>(i) * N]);
  uint2 codes;
  const uint32_t sc = nvfp4_group(v, gs[g], &codes);
  *reinterpret_cast<uint2*>(q + (static_cast<size_t>(g) * N + n) * (K / 2) + kg * 8) = codes;
  const int nb = (N + 127) / 128;
  sf[static_cast<size_t>(g) * nb * (K / 64) * 512 + sf_offset(n, kg, K / 64)] = static_cast<uint8_t>(sc);
}

// --------------------------------------------------- activation quantiser

// One warp per row of x [rows][K] bf16 -> q [rows][K/2] and the row's scales.
__global__ void act_quant_kernel(const __nv_bfloat16* __restrict__ x, int rows, int K, float g,
                                 uint8_t* __restrict__ q, uint8_t* __restrict__ sf) {
  pdl_wait_then_release();
  const int lane = threadIdx.x & 31;
  for (int r = blockIdx.x * 8 + (threadIdx.x >> 5); r < rows; r += gridDim.x * 8) {
    for (int c = lane; c < K / 16; c += 32) {
      float v[16];
      load16_bf16(x + static_cast<size_t>(r) * K + c * 16, v);
      uint2 codes;
      const uint32_t sc = nvfp4_group(v, g, &codes);
      *reinterpret_cast<uint2*>(q + static_cast<size_t>(r) * (K / 2) + c * 8) = codes;
      sf[sf_offset(r, c, K / 64)] = static_cast<uint8_t>(sc);
    }
  }
}

// The NVFP4 block's scatter: one warp per token. The warp finds the routed
// row of each of the token's k slots in the 128-padded expert-major row space
// (from the bitmasks), quantises x[t] ONCE - each lane whole 64-element blocks,
// i.e. 4 groups of 16: 32 bytes of codes and 4 scale bytes, which are one
// aligned word of the scale atom - and writes the result to the token-order
// buffer (the shared MLP's input) and to each routed row.
__global__ void __launch_bounds__(256) route_scatter_fp4_kernel(
    const int32_t* __restrict__ idx, const uint32_t* __restrict__ masks, const int32_t* __restrict__ base, int T,
    int k, int E, int D, const __nv_bfloat16* __restrict__ x, float g_x, int32_t* __restrict__ row_of,
    uint8_t* __restrict__ xq_perm, uint8_t* __restrict__ xsf_perm, uint8_t* __restrict__ xq_tok,
    uint8_t* __restrict__ xsf_tok, int rows, uint32_t* __restrict__ err) {
  __shared__ int s_rows[8][128];  // k <= num_experts <= 128
  pdl_wait_then_release();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int k64 = D / 64;
  for (int t = blockIdx.x * 8 + wid; t < T; t += gridDim.x * 8) {
    for (int j = lane; j < k; j += 32) {
      const long long a = static_cast<long long>(t) * k + j;
      const int e = __ldg(idx + a);
      int row = -1;
      if (e >= 0 && e < E) {
        const size_t cw = static_cast<size_t>(t / kMaskTokens) * E + e;
        const uint32_t below = __ldg(masks + cw) & ((1u << (t & (kMaskTokens - 1))) - 1u);
        row = __ldg(base + cw) + __popc(below);
        if (row < 0 || row >= rows) {  // never write outside the routed-row buffers
          atomicOr(err, kErrBadIndex);
          row = -1;
        } else {
          row_of[a] = row;
        }
      }
      s_rows[wid][j] = row;
    }
    __syncwarp();
    for (int b = lane; b < k64; b += 32) {
      uint2 codes[4];
      uint32_t scw = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float v[16];
        load16_bf16(x + static_cast<size_t>(t) * D + b * 64 + q * 16, v);
        scw |= (nvfp4_group(v, g_x, &codes[q]) & 0xFFu) << (8 * q);
      }
      const uint4 c0 = make_uint4(codes[0].x, codes[0].y, codes[1].x, codes[1].y);
      const uint4 c1 = make_uint4(codes[2].x, codes[2].y, codes[3].x, codes[3].y);
      uint4* qt = reinterpret_cast<uint4*>(xq_tok + static_cast<size_t>(t) * (D / 2) + b * 32);
      qt[0] = c0;
      qt[1] = c1;
      *reinterpret_cast<uint32_t*>(xsf_tok + sf_offset(t, 4 * b, k64)) = scw;
      for (int j = 0; j < k; ++j) {
        const int row = s_rows[wid][j];
        if (row < 0) continue;
        uint4* qp = reinterpret_cast<uint4*>(xq_perm + static_cast<size_t>(row) * (D / 2) + b * 32);
        qp[0] = c0;
        qp[1] = c1;
        *reinterpret_cast<uint32_t*>(xsf_perm + sf_offset(row, 4 * b, k64)) = scw;
      }
    }
    __syncwarp();
  }
}

// ------------------------------------------------------------- FP4 GEMM

constexpr int kF4KStage = 256;                   // K elements per stage (128 bytes of codes per row)
constexpr int kF4ABytes = 128 * 128;             // 128 rows x 128 B
constexpr int kF4BBytes = 2 * 128 * 128;         // two 128-row blocks
constexpr int kF4SfBytes = 4 * 512;              // 4 atoms (4 x 64 K) of one 128-row block
constexpr int kF4Stages = 4;
constexpr int kF4SfSlots = 16;                   // TMEM scale slots (ring over 64-K steps)
constexpr int kF4Threads = 320;                  // producer, MMA, 8 epilogue warps (2 per TMEM lane quarter)
// Both GEMMs add 4 scale warps (see the kernel): measured at T=2048, gate|up
// 122 -> 98 us with them.
template <bool GATEUP>
__host__ __device__ constexpr int f4_threads() {
  return kF4Threads + 128;
}
constexpr int kF4StgWarpBytes = 1024;            // epilogue staging per warp (32 rows x 32 B)
constexpr int kF4SmemBytes = kF4Stages * (kF4ABytes + kF4BBytes + 3 * kF4SfBytes) + 8 * kF4StgWarpBytes + 1024 + 512;

struct Fp4Problem {
  int K;          // multiple of 64
  int N;          // multiple of 64
  int groups;
  int a_rows;     // rows of A (a multiple of 128)
  const uint8_t* sfa;   // [a_rows/128][K/64][512]
  const uint8_t* sfb0;  // [groups][ceil(N/128)][K/64][512]
  const uint8_t* sfb1;  // (up; GATEUP only)
  const float* gb0;     // [groups] weight tensor scales
  const float* gb1;
  float ga;             // activation tensor scale
  void* out;            // GATEUP: codes [rows][N/2]; DOWN: bf16 / fp32 [rows][ldo]
  uint8_t* out_sf;      // GATEUP: scales [rows/128][N/64][512]
  float g_out;          // GATEUP: tensor scale of the quantised output
  int ldo;
  int out_f32;
};

struct Fp4Params {
  CUtensorMap tmA[2];   // codes [a_rows][K/2] u8, box 128 x 128, 128-byte swizzle
  CUtensorMap tmB0[2];  // codes [groups][N][K/2] u8, box 128 x 128 x 1
  CUtensorMap tmB1[2];
  CUtensorMap tmBw[2];  // down: the same codes, box 128 x 256 x 1 (both 128-row halves of a tile in one copy)
  Fp4Problem prob[2];
  int nprob;
  const Tile* tiles;
  const int32_t* num_tiles;
  int32_t* next_tile;   // work counter (zero at launch): tiles go to CTAs as they free up
  uint32_t* err;
};

// Instruction descriptor of kind::mxf4nvf4 (e2m1 A and B, ue4m3 scales),
// K-major A and B, M = 128.
__host__ __device__ constexpr uint32_t idesc_nvf4_m128(int n) {
  return (1u << 7)                                  // A format e2m1
         | (1u << 10)                               // B format e2m1
         | (static_cast<uint32_t>(n >> 3) << 17)    // N / 8
         | (static_cast<uint32_t>(128 >> 4) << 24);   // M / 16
}

// 4 consecutive 32-bit TMEM columns of this warp's 32 lanes from registers.
__device__ __forceinline__ void tmem_st_32x32b_x4(uint32_t taddr, uint4 v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }


__device__ __forceinline__ void umma_nvf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// Output columns of a tile: GATEUP 128 per projection (gate and up side by
// side in the 256-column accumulator), DOWN 256.
template <bool GATEUP>
__device__ __forceinline__ int f4_tile_cols(const Fp4Problem& pr, int n0) {
  const int cap = GATEUP ? 128 : 256;
  const int rem = pr.N - n0;
  return rem < cap ? rem : cap;
}

// TMEM columns [0, 256): one accumulator (GATEUP: gate 0..127, up 128..255;
// DOWN: output columns n0 .. n0+255) - a second one would not leave room for
// the scale slots, so the epilogue stages it in registers and releases it at
// once. From 256: scale slots, slot i holding the A scales at +0, B block 0 at
// +4, B block 1 at +8.
template <bool GATEUP>
__global__ void __launch_bounds__(f4_threads<GATEUP>(), 1) fp4_gemm_kernel(const __grid_constant__ Fp4Params P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + kF4Stages * kF4ABytes;
  uint8_t* sSfA = sB + kF4Stages * kF4BBytes;
  uint8_t* sSfB = sSfA + kF4Stages * kF4SfBytes;  // per stage: block 0 atoms, then block 1 atoms
  uint8_t* sStg = sSfB + kF4Stages * 2 * kF4SfBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sStg + 8 * kF4StgWarpBytes);
  uint64_t* empty = full + kF4Stages;
  constexpr int kAccStages = 1;
  constexpr uint32_t kAccStride = 256;
  uint64_t* acc_full = empty + kF4Stages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint64_t* sf_ready = drain + 1;  // a stage's scale atoms are in TMEM (one arrival per scale warp)
  uint64_t* tile_full = sf_ready + kF4Stages;
  uint64_t* tile_empty = tile_full + kTileRing;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tile_empty + kTileRing);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* tile_ring = abort_flag + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kF4Stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sf_ready[s], 4);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 8);  // one arrival per epilogue warp
    }
    mbar_init(drain, 1);
    for (int r = 0; r < kTileRing; ++r) {
      mbar_init(&tile_full[r], 1);
      mbar_init(&tile_empty[r], 1 + 8 + 4);  // MMA thread, epilogue and scale warps read each index
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int p = 0; p < P.nprob; ++p) {
      tma_prefetch_desc(&P.tmA[p]);
      tma_prefetch_desc(&P.tmB0[p]);
      tma_prefetch_desc(&P.tmB1[p]);
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
  // The producer takes tile indices from the work counter and publishes them
  // in the ring (-1 ends the work); the other roles read them in order. A
  // consumer's next index: lane 0 of its warp waits, the warp shares it
  // (-1 as well when the wait gave up).
  int rs = 0;
  uint32_t rph = 0;
  auto next_tile = [&](bool whole_warp) -> int {
    int ti = -1;
    if (lane == 0) {
      if (mbar_wait(&tile_full[rs], rph, abort_flag, P.err)) {
        ti = tile_ring[rs];
        mbar_arrive(&tile_empty[rs]);
      }
    }
    if (whole_warp) ti = __shfl_sync(0xffffffffu, ti, 0);
    if (++rs == kTileRing) {
      rs = 0;
      rph ^= 1;
    }
    return ti;
  };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ TMA producer
      int s = 0, issued = 0;
      uint32_t ph = 0;
      int ti = atomicAdd(P.next_tile, 1);
      while (true) {
        if (!mbar_wait(&tile_empty[rs], rph ^ 1, abort_flag, P.err)) break;
        tile_ring[rs] = ti < num_tiles ? ti : -1;
        mbar_arrive(&tile_full[rs]);
        if (++rs == kTileRing) {
          rs = 0;
          rph ^= 1;
        }
        if (ti >= num_tiles) break;
        const int next = atomicAdd(P.next_tile, 1);  // its latency hides behind this tile's loads
        const Tile tile = P.tiles[ti];
        const int p = tile.pg >> 16, g = tile.pg & 0xFFFF;
        if (p >= P.nprob) {
          atomicOr(P.err, kErrBadTile);
          *abort_flag = 1;
          break;
        }
        const Fp4Problem& pr = P.prob[p];
        if (g >= pr.groups || tile.row0 < 0 || tile.row0 >= pr.a_rows || (tile.row0 & 127) || tile.n0 < 0 ||
            tile.n0 >= pr.N) {
          atomicOr(P.err, kErrBadTile);
          *abort_flag = 1;
          break;
        }
        const int k64 = pr.K / 64;
        const int nstage = (pr.K + kF4KStage - 1) / kF4KStage;
        const int nbr = (pr.N + 127) / 128;
        const int nb0 = tile.n0 >> 7;
        const int nb1 = GATEUP ? nb0 : nb0 + 1;
        const uint8_t* sfa = pr.sfa + static_cast<size_t>(tile.row0 >> 7) * k64 * 512;
        const uint8_t* sfb0 = pr.sfb0 + (static_cast<size_t>(g) * nbr + nb0) * k64 * 512;
        const uint8_t* sfb1 = (GATEUP ? pr.sfb1 : pr.sfb0) + (static_cast<size_t>(g) * nbr + nb1) * k64 * 512;
        const bool two_b = GATEUP || (tile.n0 + 128 < pr.N);
        bool ok = true;
        for (int ks = 0; ks < nstage; ++ks) {
          if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, P.err)) {
            ok = false;
            break;
          }
          const int nks = min(4, k64 - 4 * ks);
          const uint32_t sf_bytes = nks * 512;
          const uint32_t bytes = kF4ABytes + (two_b ? 2 : 1) * (kF4BBytes / 2) + sf_bytes * (two_b ? 3 : 2);
          mbar_arrive_expect_tx(&full[s], bytes);
          tma_load_2d(sA + s * kF4ABytes, &P.tmA[p], &full[s], ks * 128, tile.row0);
          if (!GATEUP && two_b) {
            tma_load_3d(sB + s * kF4BBytes, &P.tmBw[p], &full[s], ks * 128, tile.n0, g);  // 256 rows
          } else {
            tma_load_3d(sB + s * kF4BBytes, &P.tmB0[p], &full[s], ks * 128, tile.n0, g);
            if (two_b) tma_load_3d(sB + s * kF4BBytes + kF4BBytes / 2, &P.tmB1[p], &full[s], ks * 128, tile.n0, g);
          }
          bulk_load(sSfA + s * kF4SfBytes, sfa + static_cast<size_t>(4 * ks) * 512, sf_bytes, &full[s]);
          bulk_load(sSfB + (2 * s) * kF4SfBytes, sfb0 + static_cast<size_t>(4 * ks) * 512, sf_bytes, &full[s]);
          if (two_b)
            bulk_load(sSfB + (2 * s + 1) * kF4SfBytes, sfb1 + static_cast<size_t>(4 * ks) * 512, sf_bytes, &full[s]);
          ++issued;
          if (++s == kF4Stages) {
            s = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        ti = next;
      }
      if (*abort_flag) {
        int st = s;
        uint32_t sp = ph;
        const int pending = issued < kF4Stages ? issued : kF4Stages;
        for (int i = 0; i < pending; ++i) {
          if (--st < 0) {
            st = kF4Stages - 1;
            sp ^= 1;
          }
          uint32_t dummy = 0;
          mbar_wait(&full[st], sp, reinterpret_cast<volatile int*>(&dummy), P.err, 100000000ull);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------- MMA issuer
      int s = 0, slot = 0, acc = 0;
      uint32_t ph = 0, acc_ph = 0;
      bool any = false;
      const uint32_t idesc = idesc_nvf4_m128(128);
      const uint32_t idesc256 = idesc_nvf4_m128(256);
      while (true) {
        const int ti = next_tile(false);
        if (ti < 0) break;
        const Tile tile = P.tiles[ti];
        const int p = tile.pg >> 16;
        if (p >= P.nprob) break;
        const Fp4Problem& pr = P.prob[p];
        const int k64 = pr.K / 64;
        const int nstage = (pr.K + kF4KStage - 1) / kF4KStage;
        const bool two_b = GATEUP || (tile.n0 + 128 < pr.N);
        if (!mbar_wait(&acc_empty[acc], acc_ph ^ 1, abort_flag, P.err)) break;
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + acc * kAccStride;
        bool ok = true;
        for (int ks = 0; ks < nstage; ++ks) {
          if (!mbar_wait(&full[s], ph, abort_flag, P.err)) {
            ok = false;
            break;
          }
          // the stage's scale atoms are written into TMEM by the scale warps
          // (tcgen05.st), off this thread's MMA stream
          if (!mbar_wait(&sf_ready[s], ph, abort_flag, P.err)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const int nks = min(4, k64 - 4 * ks);
          const uint32_t a_addr = smem_u32(sA + s * kF4ABytes);
          const uint32_t b_addr = smem_u32(sB + s * kF4BBytes);
          for (int i = 0; i < nks; ++i) {
            const uint32_t cols = tmem_base + kAccCols + ((slot + i) % kF4SfSlots) * 16;
            // 64 K of e2m1 = 32 B per row inside the 128-byte swizzled rows
            const uint64_t ad = sdesc_sw128(a_addr + i * 32, 16, 1024);
            const uint64_t bd0 = sdesc_sw128(b_addr + i * 32, 16, 1024);
            const uint32_t accum = (ks | i) != 0;
            // both B blocks (gate | up, or 256 output columns) are consecutive
            // 128-row halves of the stage and their scale atoms sit at cols + 4
            // and cols + 8, which is the N = 256 layout: one MMA covers both
            umma_nvf4(d_tmem, ad, bd0, two_b ? idesc256 : idesc, cols, cols + 4, accum);
          }
          slot = (slot + nks) % kF4SfSlots;
          any = true;
          umma_commit(&empty[s]);
          if (++s == kF4Stages) {
            s = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&acc_full[acc]);
        if (++acc == kAccStages) {
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
  } else if (warp >= 10) {
    // ------------------------------------------------------- scale warps
    // Warps 10..13 (TMEM lane quarters 2, 3, 0, 1): for every stage, in the
    // MMA thread's order, each writes its quarter of the stage's scale atoms
    // into the TMEM slots the MMAs read. An atom (512 B) holds 32 rows of
    // 16 B; row i goes to columns c..c+3 of lane 32 q + i in every quarter q,
    // the layout tcgen05.cp .32x128b.warpx4 would produce, but from the
    // warps' registers, so the tensor pipe runs only MMAs. A slot is rewritten
    // only after full[] of its stage completed, i.e. after the MMAs that read
    // its previous contents (four stages back) have finished.
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    int s = 0, slot = 0;
    uint32_t ph = 0;
    while (true) {
      const int ti = next_tile(true);
      if (ti < 0) break;
      const Tile tile = P.tiles[ti];
      const int p = tile.pg >> 16;
      if (p >= P.nprob) break;
      const Fp4Problem& pr = P.prob[p];
      const int k64 = pr.K / 64;
      const int nstage = (pr.K + kF4KStage - 1) / kF4KStage;
      const bool two_b = GATEUP || (tile.n0 + 128 < pr.N);
      bool ok = true;
      for (int ks = 0; ks < nstage; ++ks) {
        int got = 1;
        if (lane == 0) got = mbar_wait(&full[s], ph, abort_flag, P.err);
        if (!__shfl_sync(0xffffffffu, got, 0)) {
          ok = false;
          break;
        }
        const int nks = min(4, k64 - 4 * ks);
        const uint8_t* sfa = sSfA + s * kF4SfBytes + lane * 16;
        const uint8_t* sfb = sSfB + (2 * s) * kF4SfBytes + lane * 16;
        for (int i = 0; i < nks; ++i) {
          const uint32_t cols = tmem_base + lane_base + kAccCols + ((slot + i) % kF4SfSlots) * 16;
          tmem_st_32x32b_x4(cols, *reinterpret_cast<const uint4*>(sfa + i * 512));
          tmem_st_32x32b_x4(cols + 4, *reinterpret_cast<const uint4*>(sfb + i * 512));
          if (two_b) tmem_st_32x32b_x4(cols + 8, *reinterpret_cast<const uint4*>(sfb + kF4SfBytes + i * 512));
        }
        tmem_st_wait();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sf_ready[s]);
        slot = (slot + nks) % kF4SfSlots;
        if (++s == kF4Stages) {
          s = 0;
          ph ^= 1;
        }
      }
      if (!ok) break;
    }
  } else {
    // ----------------------------------------------------------- epilogue
    // warps 2..9: TMEM lane quarter warp % 4, column half (warp - 2) / 4
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;
    int acc_i = 0;
    uint32_t acc_ph = 0;
    while (true) {
      const int ti = next_tile(true);
      if (ti < 0) break;
      const Tile tile = P.tiles[ti];
      const int p = tile.pg >> 16, g = tile.pg & 0xFFFF;
      if (p >= P.nprob) break;
      const Fp4Problem& pr = P.prob[p];
      const int wn = f4_tile_cols<GATEUP>(pr, tile.n0);
      const bool ready = mbar_wait(&acc_full[acc_i], acc_ph, abort_flag, P.err);
      __syncwarp();
      if (!ready) break;
      tc_fence_after_sync();
      const uint32_t tbase = tmem_base + acc_i * kAccStride + (static_cast<uint32_t>(quarter * 32) << 16);
      const bool valid = r < tile.rows;
      const int grow = tile.row0 + r;
      // Column chunks of 32: j = half * 32 + 64 c (c = 0..3 while j < wn).
      // Gate|up brings this thread's accumulator columns (gate and up of
      // chunks 0, 1) into registers and hands TMEM back, so the next tile's
      // MMAs overlap the quantisation and stores below. Down holds 4
      // chunks: chunks 0, 1 are converted and stored first, then chunks 2, 3
      // are loaded and TMEM handed back (64 values in registers at a time).
      uint32_t acc[4][32];
      auto release_acc = [&]() {
        tmem_ld_wait();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[acc_i]);
        if (++acc_i == kAccStages) {
          acc_i = 0;
          acc_ph ^= 1;
        }
      };
      if (GATEUP) {
        // Chunk 0 (gate and up columns j0 = 32 half) is loaded, turned into h
        // and quantised before chunk 1 (j0 + 64) is loaded and TMEM handed
        // back: at most 64 accumulator values live at a time, no spills.
        const float ag = 1.0f / (pr.ga * pr.gb0[g]);
        const float au = 1.0f / (pr.ga * pr.gb1[g]);
        uint8_t* q = reinterpret_cast<uint8_t*>(pr.out) + static_cast<size_t>(grow) * (pr.N / 2);
        uint4 qc[2];
        uint32_t sc[2][2];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int j = half * 32 + 64 * c;
          if (j < wn) {
            tmem_ld_32x32b_x32(tbase + j, acc[0]);
            tmem_ld_32x32b_x32(tbase + 128 + j, acc[1]);
          }
          if (c == 1) {
            release_acc();
          } else {
            tmem_ld_wait();
          }
          if (j >= wn) continue;
          uint2 codes[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            float v[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              v[i] = gelu_tanh(__uint_as_float(acc[0][16 * h + i]) * ag) * (__uint_as_float(acc[1][16 * h + i]) * au);
            sc[c][h] = nvfp4_group(v, pr.g_out, &codes[h]);
          }
          qc[c] = make_uint4(codes[0].x, codes[0].y, codes[1].x, codes[1].y);
        }
        if (valid) {
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const int j = half * 32 + 64 * c;
            if (j >= wn) continue;
            *reinterpret_cast<uint4*>(q + (tile.n0 + j) / 2) = qc[c];
            const int c16 = (tile.n0 + j) / 16;
            pr.out_sf[sf_offset(grow, c16, pr.N / 64)] = static_cast<uint8_t>(sc[c][0]);
            pr.out_sf[sf_offset(grow, c16 + 1, pr.N / 64)] = static_cast<uint8_t>(sc[c][1]);
          }
        }
      } else {
        // staged through the warp's buffer: whole-sector stores in row order
        const float alpha = 1.0f / (pr.ga * pr.gb0[g]);
        uint8_t* stg = sStg + (warp - 2) * kF4StgWarpBytes;
        const int rows_valid = tile.rows - quarter * 32;
        const size_t wrow = static_cast<size_t>(tile.row0 + quarter * 32);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int j = half * 32 + 64 * c;
          if ((c & 1) == 0) {  // load chunks c, c + 1; after the second pair TMEM is no longer needed
#pragma unroll
            for (int u = 0; u < 2; ++u)
              if (j + 64 * u < wn) tmem_ld_32x32b_x32(tbase + j + 64 * u, acc[u]);
            if (c == 2) {
              release_acc();
            } else {
              tmem_ld_wait();
            }
          }
          if (j >= wn) continue;
          uint32_t* a = acc[c & 1];
          if (pr.out_f32) {
#pragma unroll
            for (int i = 0; i < 32; ++i) a[i] = __float_as_uint(__uint_as_float(a[i]) * alpha);
            uint8_t* base = reinterpret_cast<uint8_t*>(reinterpret_cast<float*>(pr.out) + wrow * pr.ldo + tile.n0 + j);
#pragma unroll
            for (int q = 0; q < 4; ++q) store_rows_32B(stg, a + 8 * q, lane, base + 32 * q, pr.ldo * 4, rows_valid);
          } else {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = pack_bf16x2(__uint_as_float(a[2 * i]) * alpha, __uint_as_float(a[2 * i + 1]) * alpha);
            uint8_t* base =
                reinterpret_cast<uint8_t*>(reinterpret_cast<__nv_bfloat16*>(pr.out) + wrow * pr.ldo + tile.n0 + j);
#pragma unroll
            for (int q = 0; q < 2; ++q) store_rows_32B(stg, pk + 8 * q, lane, base + 32 * q, pr.ldo * 2, rows_valid);
          }
        }
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

// --------------------------------------------------------------- combine

// f[t] = s[t] + sum_j w[t, j] y[row_of[t, j]] in fp32 (slot order), then
// optionally the RMSNorm f / sqrt(mean(f^2) + 1e-6) (model card: RMSNorm, eps
// 1e-06) - unlearned between the blocks of the NVFP4 stack, or times a learned
// scale gamma (the post-FFN norm of the sandwich) - and optionally plus the
// block's raw input xres (the residual). One CTA per token; each thread keeps
// up to kCombVec 8-column vectors in registers.
constexpr int kCombThreads = 128;
constexpr int kCombVec = 4;  // supports D <= 128 * 4 * 8 = 4096

__global__ void __launch_bounds__(kCombThreads) combine_norm_kernel(
    const float* __restrict__ s, const __nv_bfloat16* __restrict__ y, const int32_t* __restrict__ row_of,
    const float* __restrict__ w, int T, int k, int D, int rows, int rms_norm, const __nv_bfloat16* __restrict__ gamma,
    const __nv_bfloat16* __restrict__ xres, __nv_bfloat16* __restrict__ out, float* __restrict__ out_f32,
    uint32_t* __restrict__ err) {
  __shared__ int s_row[128];
  __shared__ float s_w[128];
  __shared__ float s_red[kCombThreads / 32];
  pdl_wait_then_release();
  const int t = blockIdx.x;
  for (int j = threadIdx.x; j < k; j += blockDim.x) {
    int r = row_of[static_cast<size_t>(t) * k + j];
    float wj = w[static_cast<size_t>(t) * k + j];
    if (r < 0 || r >= rows) {  // a routed row outside y: report, never address it
      atomicOr(err, kErrBadIndex);
      r = 0;
      wj = 0.f;
    }
    s_row[j] = r;
    s_w[j] = wj;
  }
  __syncthreads();
  const int nvec = D >> 3;
  float acc[kCombVec][8];
  float ss = 0.f;
#pragma unroll
  for (int u = 0; u < kCombVec; ++u) {
    const int v = threadIdx.x + u * kCombThreads;
    if (v >= nvec) continue;
    const float4* sp = reinterpret_cast<const float4*>(s + static_cast<size_t>(t) * D) + 2 * v;
    const float4 s0 = sp[0], s1 = sp[1];
    acc[u][0] = s0.x; acc[u][1] = s0.y; acc[u][2] = s0.z; acc[u][3] = s0.w;
    acc[u][4] = s1.x; acc[u][5] = s1.y; acc[u][6] = s1.z; acc[u][7] = s1.w;
    for (int j = 0; j < k; ++j) {
      const uint4 yv = __ldg(reinterpret_cast<const uint4*>(y + static_cast<size_t>(s_row[j]) * D) + v);
      const __nv_bfloat16* yb = reinterpret_cast<const __nv_bfloat16*>(&yv);
      const float wj = s_w[j];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[u][i] = fmaf(wj, __bfloat162float(yb[i]), acc[u][i]);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) ss = fmaf(acc[u][i], acc[u][i], ss);
  }
  float scale = 1.0f;
  if (rms_norm) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
    for (int i = 0; i < kCombThreads / 32; ++i) tot += s_red[i];
    scale = 1.0f / sqrtf(tot / static_cast<float>(D) + 1e-6f);
  }
#pragma unroll
  for (int u = 0; u < kCombVec; ++u) {
    const int v = threadIdx.x + u * kCombThreads;
    if (v >= nvec) continue;
    float o[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = acc[u][i] * scale;
    if (gamma) {  // learned scale of the normalisation
      const uint4 gv = __ldg(reinterpret_cast<const uint4*>(gamma) + v);
      const __nv_bfloat16* gb = reinterpret_cast<const __nv_bfloat16*>(&gv);
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] *= __bfloat162float(gb[i]);
    }
    if (xres) {  // residual: the block's raw input
      const uint4 xv = __ldg(reinterpret_cast<const uint4*>(xres + static_cast<size_t>(t) * D) + v);
      const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(&xv);
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = __bfloat162float(xb[i]) + o[i];
    }
    reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * D)[v] =
        make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]), pack_bf16x2(o[6], o[7]));
    if (out_f32) {
      float4* op = reinterpret_cast<float4*>(out_f32 + static_cast<size_t>(t) * D) + 2 * v;
      op[0] = make_float4(o[0], o[1], o[2], o[3]);
      op[1] = make_float4(o[4], o[5], o[6], o[7]);
    }
  }
}

// amax of |a| over n fp32 / bf16 values into *amax_bits (zero on entry).
__global__ void amax_bf16_kernel(const __nv_bfloat16* __restrict__ a, size_t n, uint32_t* __restrict__ amax_bits) {
  pdl_wait_then_release();
  float m = 0.f;
  for (size_t i = (static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 8; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x * 8) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(a + i));
    const __nv_bfloat16* b = reinterpret_cast<const __nv_bfloat16*>(&v);
#pragma unroll
    for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(__bfloat162float(b[j])));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, __float_as_uint(m));
}

}  // namespace moe
