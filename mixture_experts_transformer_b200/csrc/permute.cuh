// Token -> expert permutation (integer work, bit-exact) and the GEMM work lists.
//
// The T*k (token, slot) assignments are put in expert-major order: rows of
// expert e occupy [off[e], off[e] + cnt[e]) with tokens ascending. The pages
// state only the routing (top_k_experts = 8 of num_experts = 128 per token,
// gm.nn.Gemma4_26B_A4B TransformerConfig); no capacity factor or token
// dropping is mentioned, so every assignment gets a row.
//
// Everything derives from the 32-token expert bitmasks mask[c][e] (bit i set
// when token 32c + i chose expert e):
//   cnt[e]          = sum_c popc(mask[c][e])
//   base[c][e]      = off[e] + sum_{c' < c} popc(mask[c'][e])
//   row of (t, e)   = base[t/32][e] + popc(mask[t/32][e] & ((1 << t%32) - 1))
// so the scan is one small CTA and the scatter has no loops at all.
#pragma once

#include "grouped_gemm.cuh"
#include "router.cuh"

namespace moe {

constexpr int kScanThreads = 1024;
// row_of of a (token, slot) whose expert belongs to another expert shard
constexpr int32_t kRowNotLocal = -1;
constexpr int kScanSegs = kScanThreads / 128;
// CTAs of the scan (each recomputes the offsets from the masks and emits a
// share of the tiles and of base)
constexpr int kScanCtas = 8;

struct TileCounts {
  int32_t gateup;
  int32_t down;
  int32_t next_gateup;  // the GEMMs' work counters, cleared by the scan
  int32_t next_down;
};

// Bitmasks of a given idx [T, k] (moe_permute's entry; the forward pass gets
// them from router_topk_kernel). masks must be zero on entry.
__global__ void build_masks_kernel(const int32_t* __restrict__ idx, int T, int k, int E, uint32_t* __restrict__ masks,
                                   uint32_t* err) {
  pdl_wait_then_release();
  const int n = T * k;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const int t = i / k;
    const int e = idx[i];
    if (e < 0 || e >= E) {
      atomicOr(err, kErrBadIndex);
      continue;
    }
    atomicOr(masks + static_cast<size_t>(t / kMaskTokens) * E + e, 1u << (t & (kMaskTokens - 1)));
  }
}

// kScanCtas CTAs of 1024 threads, each computing the same per-expert counts
// and offsets (thread (e, seg) walks one eighth of the 32-token chunks of
// expert e); CTA b then writes base[c][e] for the chunks of segment b and
// every kScanCtas-th entry of the tile lists. Produces cnt, off, base and the tile lists
// (gate|up tiles gu_cols output columns per projection, down tiles dn_cols wide):
// shared-MLP tiles first (problem 1), then expert tiles (problem 0) expert by
// expert, column tile, then row tile, so CTAs that run at the same time read
// the same weight columns and share them through L2.
//
// An expert shard (expert parallelism) owns experts [e_begin, e_begin +
// e_count): only they get routed rows and tiles (their cnt is the real count,
// every other expert's is 0), and a tile's weight group is the expert's index
// within the shard. The whole block is e_begin = 0, e_count = E.
__global__ void __launch_bounds__(kScanThreads) route_scan_kernel(const uint32_t* __restrict__ masks, int nchunks,
                                                                  int T, int E, int F, int S, int D,
                                                                  int32_t* __restrict__ base,
                                                                  int32_t* __restrict__ cnt_out,
                                                                  int32_t* __restrict__ off_out,
                                                                  Tile* __restrict__ tiles_gu,
                                                                  Tile* __restrict__ tiles_dn,
                                                                  TileCounts* __restrict__ counts, int padded,
                                                                  int dn_cols, int gu_cols, int pair_gu, int pair_dn,
                                                                  int e_begin, int e_count) {
  __shared__ int s_seg[kScanSegs][128];
  __shared__ int s_off[129];
  __shared__ int s_mtoff[129];
  __shared__ int s_ptoff[129];  // prefix of 128-row block pairs per expert (paired GEMM tiles)
  __shared__ int s_cnt[128];
  pdl_wait_then_release();
  const int e = threadIdx.x & 127;
  const int seg = threadIdx.x >> 7;
  const int c0 = static_cast<int>((static_cast<long long>(seg) * nchunks) / kScanSegs);
  const int c1 = static_cast<int>((static_cast<long long>(seg + 1) * nchunks) / kScanSegs);
  const bool local = e >= e_begin && e < e_begin + e_count && e < E;
  int part = 0;
  if (local) {
#pragma unroll 8
    for (int c = c0; c < c1; ++c) part += __popc(__ldg(masks + static_cast<size_t>(c) * E + e));
  }
  s_seg[seg][e] = part;
  __syncthreads();
  if (seg == 0) {
    int run = 0;
    for (int s = 0; s < kScanSegs; ++s) {
      const int v = s_seg[s][e];
      s_seg[s][e] = run;
      run += v;
    }
    s_cnt[e] = e < E ? run : 0;
  }
  __syncthreads();
  if (threadIdx.x < 32) {  // exclusive scans over experts, one warp
    const int lane = threadIdx.x;
    int carry = 0, mcarry = 0, pcarry = 0;
    for (int b = 0; b < 128; b += 32) {
      const int v = s_cnt[b + lane];
      const int mv = (v + kBM - 1) / kBM;
      const int pv = (mv + 1) / 2;
      int inc = v, minc = mv, pinc = pv;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int a = __shfl_up_sync(0xffffffffu, inc, o);
        const int ma = __shfl_up_sync(0xffffffffu, minc, o);
        const int pa = __shfl_up_sync(0xffffffffu, pinc, o);
        if (lane >= o) {
          inc += a;
          minc += ma;
          pinc += pa;
        }
      }
      s_off[b + lane] = carry + inc - v;
      s_mtoff[b + lane] = mcarry + minc - mv;
      s_ptoff[b + lane] = pcarry + pinc - pv;
      carry += __shfl_sync(0xffffffffu, inc, 31);
      mcarry += __shfl_sync(0xffffffffu, minc, 31);
      pcarry += __shfl_sync(0xffffffffu, pinc, 31);
    }
    if (lane == 0) {
      s_off[E] = carry;
      s_mtoff[E] = mcarry;
      s_ptoff[E] = pcarry;
    }
  }
  __syncthreads();
  const int c_e = s_cnt[e];
  // first routed row of expert e: packed (bf16 path) or padded to whole
  // 128-row tiles (NVFP4 path: every tile starts on a scale-atom boundary)
  const int row_base = padded ? s_mtoff[e] * kBM : s_off[e];
  if (local && seg % gridDim.x == blockIdx.x) {
    int run = row_base + s_seg[seg][e];
#pragma unroll 8
    for (int c = c0; c < c1; ++c) {
      base[static_cast<size_t>(c) * E + e] = run;
      run += __popc(__ldg(masks + static_cast<size_t>(c) * E + e));
    }
  }
  if (blockIdx.x == 0) {
    if (e < E && seg == 0) {
      cnt_out[e] = c_e;
      off_out[e] = s_off[e];
    }
    if (threadIdx.x == 0) off_out[E] = s_off[E];
  }
  const int gt = blockIdx.x * kScanThreads + threadIdx.x;  // this thread's first list entry
  const int gstride = gridDim.x * kScanThreads;

  // A tile takes one 128-row block, or (paired GEMM) two consecutive blocks of
  // the same expert and column tile. Gate|up tiles are gu_cols output columns
  // per projection, down tiles dn_cols wide.
  const int mt_sh = (T + kBM - 1) / kBM;
  const int nt_gu = (F + gu_cols - 1) / gu_cols;
  const int nt_dn = (D + dn_cols - 1) / dn_cols;
  auto emit = [&](Tile* tiles, int pair, int ncol_sh, int ncol, int cw) -> int {
    const int mstep = pair ? 2 : 1;
    const int* offs = pair ? s_ptoff : s_mtoff;
    const int pt_sh = (mt_sh + mstep - 1) / mstep;
    const int n_sh = ncol_sh * pt_sh;
    for (int i = gt; i < n_sh; i += gstride) {
      const int nt = i / pt_sh, m = (i % pt_sh) * mstep;
      const int r1 = pair ? max(0, min(kBM, T - (m + 1) * kBM)) : 0;
      tiles[i] = Tile{1 << 16, m * kBM, min(kBM, T - m * kBM), nt * cw, (m + 1) * kBM, r1, 0, 0};
    }
    // expert tiles, spread over all threads (one expert may own most of them):
    // flat index f -> expert by binary search over the tile-offset prefix
    const int n_e = offs[E] * ncol;
    for (int f = gt; f < n_e; f += gstride) {
      int lo = 0, hi = E - 1;  // largest ex with offs[ex] * ncol <= f
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (offs[mid] * ncol <= f) lo = mid; else hi = mid - 1;
      }
      const int ex = lo;
      const int ce = s_cnt[ex];
      const int pt = offs[ex + 1] - offs[ex];
      const int i = f - offs[ex] * ncol;
      const int nt = i / pt, m = (i % pt) * mstep;
      const int rb = padded ? s_mtoff[ex] * kBM : s_off[ex];
      const int r1 = pair ? max(0, min(kBM, ce - (m + 1) * kBM)) : 0;
      tiles[n_sh + f] =
          Tile{ex - e_begin, rb + m * kBM, min(kBM, ce - m * kBM), nt * cw, rb + (m + 1) * kBM, r1, 0, 0};
    }
    return n_sh + n_e;
  };
  const int n_gu = emit(tiles_gu, pair_gu, (S + gu_cols - 1) / gu_cols, nt_gu, gu_cols);
  const int n_dn = emit(tiles_dn, pair_dn, (D + dn_cols - 1) / dn_cols, nt_dn, dn_cols);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    counts->gateup = n_gu;
    counts->down = n_dn;
    counts->next_gateup = 0;
    counts->next_down = 0;
  }
}

// Work tiles of a dense feed-forward (one problem, no routing): rows [0, T)
// in 128-row blocks (pairs of blocks when pair), column tiles 128 wide per
// projection for gate|up and dn_cols wide for down. With dn_ksplit > 1 (small
// batches, too few down tiles to occupy the GPU) every down tile is cut along
// the reduction into dn_ksplit K ranges of S / 64 / dn_ksplit blocks (+-1),
// each writing its own fp32 partial sums. Also clears the GEMMs' work
// counters. One CTA.
__global__ void __launch_bounds__(256) dense_tiles_kernel(int T, int S, int D, int pair_gu, int pair_dn,
                                                          int dn_cols, int dn_ksplit, Tile* __restrict__ tiles_gu,
                                                          Tile* __restrict__ tiles_dn,
                                                          TileCounts* __restrict__ counts) {
  pdl_wait_then_release();
  const int mt = (T + kBM - 1) / kBM;
  auto emit = [&](Tile* tiles, int pair, int ncol, int cw) -> int {
    const int mstep = pair ? 2 : 1;
    const int pt = (mt + mstep - 1) / mstep;
    for (int i = threadIdx.x; i < ncol * pt; i += blockDim.x) {
      const int nt = i / pt, m = (i % pt) * mstep;
      const int r1 = pair ? max(0, min(kBM, T - (m + 1) * kBM)) : 0;
      tiles[i] = Tile{0, m * kBM, min(kBM, T - m * kBM), nt * cw, (m + 1) * kBM, r1, 0, 0};
    }
    return ncol * pt;
  };
  const int n_gu = emit(tiles_gu, pair_gu, (S + 127) / 128, 128);
  int n_dn;
  if (dn_ksplit > 1) {
    // (column tile, split) pairs, row blocks innermost: the blocks of a split share its weights
    const int ncol = (D + dn_cols - 1) / dn_cols, nkb = S / 64;
    n_dn = ncol * dn_ksplit * mt;
    for (int i = threadIdx.x; i < n_dn; i += blockDim.x) {
      const int m = i % mt, q = i / mt, sp = q % dn_ksplit, nt = q / dn_ksplit;
      const int k0 = static_cast<int>(static_cast<long long>(sp) * nkb / dn_ksplit);
      const int k1 = static_cast<int>(static_cast<long long>(sp + 1) * nkb / dn_ksplit);
      tiles_dn[i] = Tile{0, m * kBM, min(kBM, T - m * kBM), nt * dn_cols, sp, 0, k0, k1 - k0};
    }
  } else {
    n_dn = emit(tiles_dn, pair_dn, (D + dn_cols - 1) / dn_cols, dn_cols);
  }
  if (threadIdx.x == 0) {
    counts->gateup = n_gu;
    counts->down = n_dn;
    counts->next_gateup = 0;
    counts->next_down = 0;
  }
}

// dst = RNE_bf16(part[0] + part[1] + ... + part[nsplit-1]), summed in split
// order in fp32 (deterministic); out_f32 (optional) gets the fp32 sums. Four
// values per thread.
__global__ void __launch_bounds__(256) reduce_splits_kernel(const float* __restrict__ part, int nsplit, size_t n4,
                                                            float* __restrict__ out_f32,
                                                            __nv_bfloat16* __restrict__ dst) {
  pdl_wait_then_release();
  const size_t stride4 = n4;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    float4 a = reinterpret_cast<const float4*>(part)[i];
    for (int sp = 1; sp < nsplit; ++sp) {
      const float4 b = __ldg(reinterpret_cast<const float4*>(part) + sp * stride4 + i);
      a.x += b.x;
      a.y += b.y;
      a.z += b.z;
      a.w += b.w;
    }
    if (out_f32) reinterpret_cast<float4*>(out_f32)[i] = a;
    reinterpret_cast<uint2*>(dst)[i] = make_uint2(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w));
  }
}

// fp32 -> bf16 (round to nearest even), 8 values per thread.
__global__ void __launch_bounds__(256) round_bf16_kernel(const float* __restrict__ src, size_t n8,
                                                         __nv_bfloat16* __restrict__ dst) {
  pdl_wait_then_release();
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const float4 a = reinterpret_cast<const float4*>(src)[2 * i];
    const float4 b = reinterpret_cast<const float4*>(src)[2 * i + 1];
    reinterpret_cast<uint4*>(dst)[i] = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w),
                                                  pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
  }
}

// One warp per (token, slot): its routed row from the bitmasks; lane 0 writes
// row_of / token_of, and (when x is given) the warp copies x[t] into
// x_perm[row] with 16-byte vectors, so the GEMM's A tiles are plain boxes.
// Slots whose expert lies outside the shard [e_begin, e_begin + e_count) get
// row_of = kRowNotLocal and no row.
__global__ void __launch_bounds__(256) route_scatter_kernel(const int32_t* __restrict__ idx,
                                                            const uint32_t* __restrict__ masks,
                                                            const int32_t* __restrict__ base, int T, int k, int E,
                                                            int D, const __nv_bfloat16* __restrict__ x,
                                                            int32_t* __restrict__ row_of,
                                                            int32_t* __restrict__ token_of,
                                                            __nv_bfloat16* __restrict__ x_perm, long long rows,
                                                            uint32_t* __restrict__ err, int e_begin, int e_count) {
  pdl_wait_then_release();
  const int lane = threadIdx.x & 31;
  const long long R = static_cast<long long>(T) * k;
  for (long long a = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5); a < R;
       a += static_cast<long long>(gridDim.x) * 8) {
    const int t = static_cast<int>(a / k);
    const int e = __ldg(idx + a);
    if (e < 0 || e >= E) continue;  // reported by build_masks_kernel
    if (e < e_begin || e >= e_begin + e_count) {
      if (lane == 0) row_of[a] = kRowNotLocal;
      continue;
    }
    const size_t cw = static_cast<size_t>(t / kMaskTokens) * E + e;
    const uint32_t below = __ldg(masks + cw) & ((1u << (t & (kMaskTokens - 1))) - 1u);
    const int row = __ldg(base + cw) + __popc(below);
    if (row < 0 || row >= rows) {  // never write outside the routed-row buffers
      if (lane == 0) atomicOr(err, kErrBadIndex);
      continue;
    }
    if (lane == 0) {
      row_of[a] = row;
      token_of[row] = t;
    }
    if (x) {
      const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * D);
      uint4* dst = reinterpret_cast<uint4*>(x_perm + static_cast<size_t>(row) * D);
      for (int i = lane; i < (D >> 3); i += 32) dst[i] = __ldg(src + i);
    }
  }
}

// out[t] = RNE_bf16(s[t] + w[t,0] y[row_of[t,0]] + ... + w[t,k-1] y[row_of[t,k-1]]),
// accumulated in fp32 in slot order (deterministic, no atomics). Grid (T,
// dsplit): CTA (t, q) handles the q-th slice of the row's 8-column vectors.
// Slots marked kRowNotLocal (an expert shard's foreign experts) are left out;
// out (bf16) may be null when only out_f32 is wanted.
__global__ void __launch_bounds__(128) combine_kernel(const float* __restrict__ s, const __nv_bfloat16* __restrict__ y,
                                                     const int32_t* __restrict__ row_of,
                                                     const float* __restrict__ w, int T, int k, int D, int rows,
                                                     __nv_bfloat16* __restrict__ out, float* __restrict__ out_f32,
                                                     uint32_t* __restrict__ err) {
  __shared__ int s_row[128];
  __shared__ float s_w[128];
  __shared__ int s_k;
  pdl_wait_then_release();
  const int t = blockIdx.x;
  for (int j = threadIdx.x; j < k; j += blockDim.x) {
    s_row[j] = row_of[static_cast<size_t>(t) * k + j];
    s_w[j] = w[static_cast<size_t>(t) * k + j];
  }
  __syncthreads();
  if (threadIdx.x == 0) {  // keep the token's slots with a routed row here, in slot order
    int kk = 0;
    for (int j = 0; j < k; ++j) {
      const int r = s_row[j];
      if (r == kRowNotLocal) continue;
      if (r < 0 || r >= rows) {  // a routed row outside y: report, never address it
        atomicOr(err, kErrBadIndex);
        continue;
      }
      s_row[kk] = r;
      s_w[kk] = s_w[j];
      ++kk;
    }
    s_k = kk;
  }
  __syncthreads();
  k = s_k;
  const int nvec = D >> 3;
  const int per = (nvec + gridDim.y - 1) / gridDim.y;
  const int v0 = blockIdx.y * per, v1 = min(nvec, v0 + per);
  for (int v = v0 + threadIdx.x; v < v1; v += blockDim.x) {
    const float4* sp = reinterpret_cast<const float4*>(s + static_cast<size_t>(t) * D) + 2 * v;
    const float4 s0 = sp[0], s1 = sp[1];
    float acc[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
    int j = 0;
    for (; j + 4 <= k; j += 4) {  // four rows' loads in flight, accumulated in slot order
      uint4 yv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        yv[u] = __ldg(reinterpret_cast<const uint4*>(y + static_cast<size_t>(s_row[j + u]) * D) + v);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const __nv_bfloat16* yb = reinterpret_cast<const __nv_bfloat16*>(&yv[u]);
        const float wj = s_w[j + u];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = fmaf(wj, __bfloat162float(yb[i]), acc[i]);
      }
    }
    for (; j < k; ++j) {
      const uint4 yv = __ldg(reinterpret_cast<const uint4*>(y + static_cast<size_t>(s_row[j]) * D) + v);
      const __nv_bfloat16* yb = reinterpret_cast<const __nv_bfloat16*>(&yv);
      const float wj = s_w[j];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = fmaf(wj, __bfloat162float(yb[i]), acc[i]);
    }
    if (out) {
      uint4 o;
      o.x = pack_bf16x2(acc[0], acc[1]);
      o.y = pack_bf16x2(acc[2], acc[3]);
      o.z = pack_bf16x2(acc[4], acc[5]);
      o.w = pack_bf16x2(acc[6], acc[7]);
      reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * D)[v] = o;
    }
    if (out_f32) {
      float4* op = reinterpret_cast<float4*>(out_f32 + static_cast<size_t>(t) * D) + 2 * v;
      op[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      op[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
  }
}

// Workspace guard words (a debug aid): the pattern a guarded call writes
// after its workspace data before its first kernel, and the check after its
// last kernel, which records kErrGuard when any word changed.
constexpr uint32_t kGuardPattern = 0x5AC3E13Bu;
constexpr int kGuardWords = 64;  // 256 bytes

__global__ void guard_fill_kernel(uint32_t* __restrict__ g) {
  pdl_wait_then_release();
  if (threadIdx.x < kGuardWords) g[threadIdx.x] = kGuardPattern ^ (threadIdx.x * 0x9E3779B9u);
}

__global__ void guard_check_kernel(const uint32_t* __restrict__ g, uint32_t* __restrict__ err) {
  pdl_wait_then_release();
  if (threadIdx.x < kGuardWords && g[threadIdx.x] != (kGuardPattern ^ (threadIdx.x * 0x9E3779B9u)))
    atomicOr(err, kErrGuard);
}

// A kernel that waits, bounded, on a barrier nothing completes: the failure
// path of every bounded wait in the library, exercised on purpose.
__global__ void timeout_probe_kernel(uint32_t* err, unsigned long long timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  pdl_wait_then_release();
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, reinterpret_cast<volatile int*>(&abort_flag), err, timeout_ns);
}

}  // namespace moe
