// Token -> expert permutation (integer work, bit-exact) and the GEMM work lists.
//
// The T*k (token, slot) assignments are put in expert-major order: rows of
// expert e occupy [off[e], off[e] + cnt[e]) with tokens ascending. The pages
// state only the routing (top_k_experts = 8 of num_experts = 128 per token,
// gm.nn.Gemma4_26B_A4B TransformerConfig); no capacity factor or token
// dropping is mentioned, so every assignment gets a row.
//
//   router_topk_kernel   counts tokens per expert for each chunk of 128 tokens
//   route_scan_kernel    cnt, off, per-chunk first rows, GEMM tile lists
//   route_scatter_kernel row_of[t, j] and token_of[row]
//   gather_rows_kernel   x_perm[row] = x[token_of[row]]
#pragma once

#include "grouped_gemm.cuh"
#include "router.cuh"

namespace moe {

struct TileCounts {
  int32_t gateup;
  int32_t down;
};

// Tokens per expert for each chunk of kTopkChunk tokens of a given idx
// [T, k] (the same counts router_topk_kernel produces as a side result).
__global__ void __launch_bounds__(128) chunk_histogram_kernel(const int32_t* __restrict__ idx, int T, int k, int E,
                                                              int32_t* __restrict__ chunk_cnt, uint32_t* err) {
  __shared__ int s_cnt[128];
  if (threadIdx.x < 128) s_cnt[threadIdx.x] = 0;
  __syncthreads();
  const int t0 = blockIdx.x * kTopkChunk;
  const int n = (min(T, t0 + kTopkChunk) - t0) * k;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int e = idx[static_cast<size_t>(t0) * k + i];
    if (e < 0 || e >= E) {
      atomicOr(err, kErrBadIndex);
      continue;
    }
    atomicAdd(&s_cnt[e], 1);
  }
  __syncthreads();
  if (threadIdx.x < E) chunk_cnt[static_cast<size_t>(blockIdx.x) * E + threadIdx.x] = s_cnt[threadIdx.x];
}

// One CTA, thread e = expert. chunk_cnt[c][e] (tokens of chunk c routed to e)
// becomes the first routed row of chunk c's assignments to e. Also writes the
// tile lists: shared-MLP tiles first (problem 1), then expert tiles (problem 0),
// expert-major, then column tile, then row tile, so CTAs that run at the same
// time read the same weight columns and share them through L2.
__global__ void __launch_bounds__(128) route_scan_kernel(int32_t* __restrict__ chunk_cnt, int nchunks, int T, int E,
                                                         int F, int S, int D, int32_t* __restrict__ cnt_out,
                                                         int32_t* __restrict__ off_out, Tile* __restrict__ tiles_gu,
                                                         Tile* __restrict__ tiles_dn,
                                                         TileCounts* __restrict__ counts) {
  __shared__ int s_off[129];
  __shared__ int s_mtoff[129];
  __shared__ int s_cnt[128];
  const int e = threadIdx.x;
  int c_e = 0;
  if (e < E) {
    for (int c = 0; c < nchunks; ++c) {
      const int v = chunk_cnt[static_cast<size_t>(c) * E + e];
      chunk_cnt[static_cast<size_t>(c) * E + e] = c_e;
      c_e += v;
    }
  }
  s_cnt[e] = e < E ? c_e : 0;
  __syncthreads();
  if (e == 0) {
    int o = 0, mo = 0;
    for (int i = 0; i < E; ++i) {
      s_off[i] = o;
      s_mtoff[i] = mo;
      o += s_cnt[i];
      mo += (s_cnt[i] + kBM - 1) / kBM;
    }
    s_off[E] = o;
    s_mtoff[E] = mo;
  }
  __syncthreads();
  if (e < E) {
    cnt_out[e] = c_e;
    off_out[e] = s_off[e];
    for (int c = 0; c < nchunks; ++c) chunk_cnt[static_cast<size_t>(c) * E + e] += s_off[e];
  }
  if (e == 0) off_out[E] = s_off[E];

  const int mt_sh = (T + kBM - 1) / kBM;
  const int nt_gu_sh = (S + 127) / 128;
  const int nt_gu = (F + 127) / 128;
  const int nt_dn = (D + 255) / 256;
  const int n_sh_gu = nt_gu_sh * mt_sh;
  const int n_sh_dn = nt_dn * mt_sh;
  for (int i = threadIdx.x; i < n_sh_gu; i += blockDim.x) {
    const int nt = i / mt_sh, m = i % mt_sh;
    tiles_gu[i] = Tile{1 << 16, m * kBM, min(kBM, T - m * kBM), nt * 128};
  }
  for (int i = threadIdx.x; i < n_sh_dn; i += blockDim.x) {
    const int nt = i / mt_sh, m = i % mt_sh;
    tiles_dn[i] = Tile{1 << 16, m * kBM, min(kBM, T - m * kBM), nt * 256};
  }
  if (e < E && c_e > 0) {
    const int mt = (c_e + kBM - 1) / kBM;
    const int base_gu = n_sh_gu + s_mtoff[e] * nt_gu;
    const int base_dn = n_sh_dn + s_mtoff[e] * nt_dn;
    for (int nt = 0; nt < nt_gu; ++nt)
      for (int m = 0; m < mt; ++m)
        tiles_gu[base_gu + nt * mt + m] = Tile{e, s_off[e] + m * kBM, min(kBM, c_e - m * kBM), nt * 128};
    for (int nt = 0; nt < nt_dn; ++nt)
      for (int m = 0; m < mt; ++m)
        tiles_dn[base_dn + nt * mt + m] = Tile{e, s_off[e] + m * kBM, min(kBM, c_e - m * kBM), nt * 256};
  }
  if (e == 0) {
    counts->gateup = n_sh_gu + s_mtoff[E] * nt_gu;
    counts->down = n_sh_dn + s_mtoff[E] * nt_dn;
  }
}

// CTA c, thread e: walk chunk c's tokens in order and hand out expert e's rows.
__global__ void __launch_bounds__(128) route_scatter_kernel(const int32_t* __restrict__ idx,
                                                            const int32_t* __restrict__ chunk_first_row, int T,
                                                            int k, int E, int32_t* __restrict__ row_of,
                                                            int32_t* __restrict__ token_of) {
  const int e = threadIdx.x;
  const int c = blockIdx.x;
  if (e >= E) return;
  int r = chunk_first_row[static_cast<size_t>(c) * E + e];
  const int t_end = min(T, (c + 1) * kTopkChunk);
  for (int t = c * kTopkChunk; t < t_end; ++t) {
    const int32_t* it = idx + static_cast<size_t>(t) * k;
    for (int j = 0; j < k; ++j) {
      if (__ldg(it + j) == e) {
        row_of[static_cast<size_t>(t) * k + j] = r;
        token_of[r] = t;
        ++r;
        break;
      }
    }
  }
}

// x_perm[row, :] = x[token_of[row], :]; one warp per row, 16-byte vectors.
__global__ void __launch_bounds__(256) gather_rows_kernel(const __nv_bfloat16* __restrict__ x,
                                                          const int32_t* __restrict__ token_of, int R, int D,
                                                          __nv_bfloat16* __restrict__ xp) {
  const int lane = threadIdx.x & 31;
  const int nvec = D >> 3;
  for (int row = blockIdx.x * 8 + (threadIdx.x >> 5); row < R; row += gridDim.x * 8) {
    const int t = __ldg(token_of + row);
    const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * D);
    uint4* dst = reinterpret_cast<uint4*>(xp + static_cast<size_t>(row) * D);
    for (int i = lane; i < nvec; i += 32) dst[i] = __ldg(src + i);
  }
}

// out[t] = RNE_bf16(s[t] + w[t,0] y[row_of[t,0]] + ... + w[t,k-1] y[row_of[t,k-1]]),
// accumulated in fp32 in slot order (deterministic, no atomics).
__global__ void __launch_bounds__(128) combine_kernel(const float* __restrict__ s, const __nv_bfloat16* __restrict__ y,
                                                     const int32_t* __restrict__ row_of,
                                                     const float* __restrict__ w, int T, int k, int D,
                                                     __nv_bfloat16* __restrict__ out, float* __restrict__ out_f32) {
  __shared__ int s_row[128];
  __shared__ float s_w[128];
  const int t = blockIdx.x;
  for (int j = threadIdx.x; j < k; j += blockDim.x) {
    s_row[j] = row_of[static_cast<size_t>(t) * k + j];
    s_w[j] = w[static_cast<size_t>(t) * k + j];
  }
  __syncthreads();
  const int nvec = D >> 3;
  for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
    const float4* sp = reinterpret_cast<const float4*>(s + static_cast<size_t>(t) * D) + 2 * v;
    const float4 s0 = sp[0], s1 = sp[1];
    float acc[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
    for (int j = 0; j < k; ++j) {
      const uint4 yv = __ldg(reinterpret_cast<const uint4*>(y + static_cast<size_t>(s_row[j]) * D) + v);
      const __nv_bfloat16* yb = reinterpret_cast<const __nv_bfloat16*>(&yv);
      const float wj = s_w[j];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = fmaf(wj, __bfloat162float(yb[i]), acc[i]);
    }
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * D)[v] = o;
    if (out_f32) {
      float4* op = reinterpret_cast<float4*>(out_f32 + static_cast<size_t>(t) * D) + 2 * v;
      op[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      op[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
  }
}

// Copy the routing of each token into caller buffers (debug outputs).
__global__ void copy_i32_kernel(const int32_t* __restrict__ a, int32_t* __restrict__ b, int n) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) b[i] = a[i];
}

// A kernel that waits, bounded, on a barrier nothing completes: the failure
// path of every bounded wait in the library, exercised on purpose.
__global__ void timeout_probe_kernel(uint32_t* err, unsigned long long timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, reinterpret_cast<volatile int*>(&abort_flag), err, timeout_ns);
}

}  // namespace moe
