// Router: logits = x W_router in fp32 on the CUDA cores, then top-k
// selection, softmax of the kept logits and a per-chunk expert histogram.
//
// Follows the layer statement: softmax gating over the expert logits, the
// top_k_experts largest kept, their weights renormalised to sum to one
// (Gemma-4-26B-A4B model card: "Gating function over expert logits",
// "Routed experts selected per token", "Selected expert weights are
// renormalized"). The softmax over all experts restricted to the kept ones
// and renormalised equals the softmax of the kept logits alone, which is what
// is evaluated here.
#pragma once

#include "ptx.cuh"

namespace moe {

constexpr int kRouterTokens = 32;   // tokens per CTA tile
constexpr int kRouterKChunk = 32;   // reduction elements staged per step
constexpr int kRouterThreads = 128;
constexpr int kTopkChunk = 128;     // tokens per top-k CTA (and per histogram chunk)
constexpr int kTopkThreads = 256;

// partial[split][t][e] = sum over this split's slice of d of x[t, d] W[d, e].
// CTA tile: 32 tokens x 128 experts; thread (tg, eg) owns tokens tg*4..+3 and
// experts eg*8..+7. Requires E % 8 == 0, E <= 128, D % 32 == 0.
__global__ void __launch_bounds__(kRouterThreads) router_logits_kernel(const __nv_bfloat16* __restrict__ x,
                                                                       const __nv_bfloat16* __restrict__ w,
                                                                       float* __restrict__ partial, int T, int D,
                                                                       int E, int nsplit) {
  __shared__ __align__(16) float xs[kRouterTokens][kRouterKChunk + 4];
  __shared__ __align__(16) float ws[kRouterKChunk][128];

  const int tid = threadIdx.x;
  const int t0 = blockIdx.x * kRouterTokens;
  const int split = blockIdx.y;
  const int nchunks = D / kRouterKChunk;
  const int c_begin = static_cast<int>((static_cast<long long>(split) * nchunks) / nsplit);
  const int c_end = static_cast<int>((static_cast<long long>(split + 1) * nchunks) / nsplit);

  const int tg = tid >> 4;  // 0..7  -> tokens tg*4 .. tg*4+3
  const int eg = tid & 15;  // 0..15 -> experts eg*8 .. eg*8+7
  float acc[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  for (int c = c_begin; c < c_end; ++c) {
    const int k0 = c * kRouterKChunk;
    {  // x tile: 32 tokens x 32 bf16 = 128 x 16 B, one vector per thread
      const int r = tid >> 2, q = tid & 3;
      const int t = t0 + r;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (t < T) v = *reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * D + k0 + q * 8);
      const __nv_bfloat16* b = reinterpret_cast<const __nv_bfloat16*>(&v);
#pragma unroll
      for (int i = 0; i < 8; ++i) xs[r][q * 8 + i] = __bfloat162float(b[i]);
    }
    // W tile: 32 rows x E bf16 (E/8 vectors per row)
    const int vec_per_row = E >> 3;
    for (int v_i = tid; v_i < kRouterKChunk * 16; v_i += kRouterThreads) {
      const int r = v_i >> 4, q = v_i & 15;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (q < vec_per_row) v = *reinterpret_cast<const uint4*>(w + static_cast<size_t>(k0 + r) * E + q * 8);
      const __nv_bfloat16* b = reinterpret_cast<const __nv_bfloat16*>(&v);
#pragma unroll
      for (int i = 0; i < 8; ++i) ws[r][q * 8 + i] = __bfloat162float(b[i]);
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kRouterKChunk; ++kk) {
      const float4 b0 = *reinterpret_cast<const float4*>(&ws[kk][eg * 8]);
      const float4 b1 = *reinterpret_cast<const float4*>(&ws[kk][eg * 8 + 4]);
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float a = xs[tg * 4 + i][kk];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a, bv[j], acc[i][j]);
      }
    }
    __syncthreads();
  }

  if (eg * 8 >= E) return;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + tg * 4 + i;
    if (t >= T) continue;
    float* dst = partial + (static_cast<size_t>(split) * T + t) * E + eg * 8;
    *reinterpret_cast<float4*>(dst) = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
    *reinterpret_cast<float4*>(dst + 4) = make_float4(acc[i][4], acc[i][5], acc[i][6], acc[i][7]);
  }
}

// One warp per token: sum the split partials in split order, add the bias,
// pick the k largest (ties: lower index), softmax over them. Lane l holds
// experts l, l+32, l+64, l+96. Also counts tokens per expert for this CTA's
// chunk of kTopkChunk tokens into chunk_cnt[blockIdx.x][e].
__global__ void __launch_bounds__(kTopkThreads) router_topk_kernel(const float* __restrict__ partial,
                                                                   const float* __restrict__ bias, int T, int E,
                                                                   int nsplit, int k, int32_t* __restrict__ idx,
                                                                   float* __restrict__ wts,
                                                                   int32_t* __restrict__ chunk_cnt) {
  __shared__ int s_cnt[128];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x < 128) s_cnt[threadIdx.x] = 0;
  __syncthreads();

  const int tokens_per_warp = kTopkChunk / (kTopkThreads / 32);
  const int t_first = blockIdx.x * kTopkChunk + warp * tokens_per_warp;
  for (int i = 0; i < tokens_per_warp; ++i) {
    const int t = t_first + i;
    if (t >= T) break;
    float l[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int e = lane + 32 * q;
      float v = -INFINITY;
      if (e < E) {
        float s = 0.f;
        for (int sp = 0; sp < nsplit; ++sp) s += partial[(static_cast<size_t>(sp) * T + t) * E + e];
        if (bias) s += bias[e];
        v = isnan(s) ? -INFINITY : s;  // a NaN never wins, so the k winners stay valid experts
      }
      l[q] = v;
    }
    bool taken[4] = {false, false, false, false};
    float top_max = 0.f, sum = 0.f;
    float my_p = 0.f;  // lane (j % 32) keeps slot j's exp(logit_j - logit_0)
    int my_e = 0;
    for (int j = 0; j < k; ++j) {
      // lane-local best among the not-yet-taken (ties: lower index = lower q)
      float bv = -INFINITY;
      int be = 0x7fffffff;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int e = lane + 32 * q;
        if (e < E && !taken[q] && (l[q] > bv || (l[q] == bv && e < be))) {
          bv = l[q];
          be = e;
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
        const int oe = __shfl_xor_sync(0xffffffffu, be, off);
        if (ov > bv || (ov == bv && oe < be)) {
          bv = ov;
          be = oe;
        }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (be == lane + 32 * q) taken[q] = true;
      if (j == 0) top_max = bv;
      const float p = expf(bv - top_max);
      sum += p;
      if (lane == (j & 31)) {
        my_p = p;
        my_e = be;
      }
      if ((j & 31) == 31 || j == k - 1) {  // park up to 32 slots (unnormalised)
        const int base = j & ~31;
        if (lane <= j - base) {
          idx[static_cast<size_t>(t) * k + base + lane] = my_e;
          wts[static_cast<size_t>(t) * k + base + lane] = my_p;
        }
      }
    }
    // every lane holds the same sum; each lane rescales the slots it parked
    for (int j = lane; j < k; j += 32) {
      const size_t o = static_cast<size_t>(t) * k + j;
      wts[o] = wts[o] / sum;
      atomicAdd(&s_cnt[idx[o]], 1);
    }
  }
  __syncthreads();
  if (threadIdx.x < E) chunk_cnt[static_cast<size_t>(blockIdx.x) * E + threadIdx.x] = s_cnt[threadIdx.x];
}

}  // namespace moe
