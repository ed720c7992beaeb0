// Router: logits = x W_router in fp32 on the CUDA cores, then top-k
// selection and the softmax of the kept logits.
//
// Follows the layer statement: softmax gating over the expert logits, the
// top_k_experts largest kept, their weights renormalised to sum to one
// (Gemma-4-26B-A4B model card: "Gating function over expert logits",
// "Routed experts selected per token", "Selected expert weights are
// renormalized"). The softmax over all experts restricted to the kept ones
// and renormalised equals the softmax of the kept logits alone, which is what
// is evaluated here.
//
// Besides idx / w, top-k sets bit (t % 32) of mask[t / 32][e] for every kept
// expert e: 32-token expert bitmasks from which the permutation derives every
// row index with popcounts.
#pragma once

#include "ptx.cuh"

namespace moe {

constexpr int kRouterTokens = 128;  // tokens per CTA tile
constexpr int kRouterKChunk = 32;   // reduction elements staged per step
constexpr int kRouterThreads = 128;
constexpr int kMaskTokens = 32;     // tokens per bitmask word
constexpr int kTopkWarps = 4;       // one warp per token

__device__ __forceinline__ void ffma2(unsigned long long& acc, unsigned long long a, unsigned long long b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}

__device__ __forceinline__ unsigned long long dup2(float a) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %1};" : "=l"(r) : "f"(a));
  return r;
}

__device__ __forceinline__ float2 unpack2(unsigned long long v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}

// partial[split][t][e] = sum over this split's slice of d of x[t, d] W[d, e].
//
// CTA tile 128 tokens x 128 experts, 128 threads; a warp owns 32 tokens, and
// lane (tg = lane / 8, eg = lane % 8) owns tokens tg*4 + {0..3, 16..19} of the
// warp and experts eg*4 + 32n + {0..3} (n = 0..3): 8 x 16 fp32 accumulators
// held as packed pairs, updated with fma.rn.f32x2 (two experts of one token
// per instruction). Shared memory holds the chunk as fp32, x transposed
// ([k][token]) and W as is ([k][expert]); per k a lane reads its 8 x values
// (a broadcast within each group of 8 lanes) and its 16 W values (8 lanes read
// 128 contiguous bytes), so the reads are conflict-free: 6 16-byte loads feed
// 128 FMAs. Every accumulator sums its slice in increasing d, so the result is
// deterministic. CTAs of split 0 also clear the token-expert bitmask words of
// their tokens. Requires E % 8 == 0, E <= 128, D % 32 == 0.
__global__ void __launch_bounds__(kRouterThreads) router_logits_kernel(const __nv_bfloat16* __restrict__ x,
                                                                       const __nv_bfloat16* __restrict__ w,
                                                                       float* __restrict__ partial,
                                                                       uint32_t* __restrict__ masks, int T, int D,
                                                                       int E, int nsplit) {
  __shared__ __align__(16) float xs[kRouterKChunk][kRouterTokens];
  __shared__ __align__(16) float ws[kRouterKChunk][128];

  pdl_wait_then_release();
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int tg = lane >> 3, eg = lane & 7;
  const int t0 = blockIdx.x * kRouterTokens;
  const int split = blockIdx.y;
  if (split == 0) {
    const int words = (min(T, t0 + kRouterTokens) - t0 + kMaskTokens - 1) / kMaskTokens;
    for (int i = tid; i < words * E; i += kRouterThreads) masks[static_cast<size_t>(t0 / kMaskTokens) * E + i] = 0u;
  }
  const int nchunks = D / kRouterKChunk;
  const int c_begin = static_cast<int>((static_cast<long long>(split) * nchunks) / nsplit);
  const int c_end = static_cast<int>((static_cast<long long>(split + 1) * nchunks) / nsplit);

  unsigned long long acc[8][8];  // [token][expert pair]
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int p = 0; p < 8; ++p) acc[i][p] = 0ull;

  // global -> registers for the next chunk while the current one is consumed
  uint4 xr[4], wr[4];
  const int my_t = t0 + tid;  // staging: thread tid brings token t0 + tid
  auto load_chunk = [&](int c) {
    const int k0 = c * kRouterKChunk;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      xr[q] = make_uint4(0, 0, 0, 0);
      if (my_t < T) xr[q] = __ldg(reinterpret_cast<const uint4*>(x + static_cast<size_t>(my_t) * D + k0) + q);
      const int v = tid + q * kRouterThreads;  // 32 rows x 16 vectors of 8 experts
      const int r = v >> 4, c8 = v & 15;
      wr[q] = make_uint4(0, 0, 0, 0);
      if (c8 * 8 < E) wr[q] = __ldg(reinterpret_cast<const uint4*>(w + static_cast<size_t>(k0 + r) * E + c8 * 8));
    }
  };
  auto store_chunk = [&]() {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(&xr[q]);
#pragma unroll
      for (int i = 0; i < 8; ++i) xs[q * 8 + i][tid] = __bfloat162float(xb[i]);
      const int v = tid + q * kRouterThreads;
      const int r = v >> 4, c8 = v & 15;
      const __nv_bfloat16* wb = reinterpret_cast<const __nv_bfloat16*>(&wr[q]);
      *reinterpret_cast<float4*>(&ws[r][c8 * 8]) = make_float4(
          __bfloat162float(wb[0]), __bfloat162float(wb[1]), __bfloat162float(wb[2]), __bfloat162float(wb[3]));
      *reinterpret_cast<float4*>(&ws[r][c8 * 8 + 4]) = make_float4(
          __bfloat162float(wb[4]), __bfloat162float(wb[5]), __bfloat162float(wb[6]), __bfloat162float(wb[7]));
    }
  };

  const int a_col = warp * 32 + tg * 4;
  if (c_begin < c_end) load_chunk(c_begin);
  for (int c = c_begin; c < c_end; ++c) {
    __syncthreads();  // the previous chunk's readers are done
    store_chunk();
    __syncthreads();
    if (c + 1 < c_end) load_chunk(c + 1);
#pragma unroll 4
    for (int kk = 0; kk < kRouterKChunk; ++kk) {
      const float4 a_lo = *reinterpret_cast<const float4*>(&xs[kk][a_col]);
      const float4 a_hi = *reinterpret_cast<const float4*>(&xs[kk][a_col + 16]);
      const float a[8] = {a_lo.x, a_lo.y, a_lo.z, a_lo.w, a_hi.x, a_hi.y, a_hi.z, a_hi.w};
      unsigned long long b[8];
#pragma unroll
      for (int n = 0; n < 4; ++n) {
        const ulonglong2 bb = *reinterpret_cast<const ulonglong2*>(&ws[kk][eg * 4 + 32 * n]);
        b[2 * n] = bb.x;
        b[2 * n + 1] = bb.y;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const unsigned long long ad = dup2(a[i]);
#pragma unroll
        for (int p = 0; p < 8; ++p) ffma2(acc[i][p], ad, b[p]);
      }
    }
  }

#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int t = t0 + a_col + (i & 3) + (i >> 2) * 16;
    if (t >= T) continue;
    float* dst = partial + (static_cast<size_t>(split) * T + t) * E;
#pragma unroll
    for (int n = 0; n < 4; ++n) {
      const int e = eg * 4 + 32 * n;
      if (e >= E) continue;
      const float2 lo = unpack2(acc[i][2 * n]), hi = unpack2(acc[i][2 * n + 1]);
      *reinterpret_cast<float4*>(dst + e) = make_float4(lo.x, lo.y, hi.x, hi.y);
    }
  }
}

// One warp per token: sum the split partials in split order, add the bias,
// pick the k largest (ties: lower index), softmax over them, set the token's
// bits in the expert bitmasks. Lane l holds experts l, l+32, l+64, l+96.
__global__ void __launch_bounds__(kTopkWarps * 32) router_topk_kernel(const float* __restrict__ partial,
                                                                     const float* __restrict__ bias, int T, int E,
                                                                     int nsplit, int k, int32_t* __restrict__ idx,
                                                                     float* __restrict__ wts,
                                                                     uint32_t* __restrict__ masks) {
  pdl_wait_then_release();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kTopkWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  float l[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) l[q] = 0.f;
  const size_t split_stride = static_cast<size_t>(T) * E;
  const float* base = partial + static_cast<size_t>(t) * E;
  int sp = 0;
  for (; sp + 4 <= nsplit; sp += 4) {  // four splits' loads in flight, summed in order
    float v[4][4];
#pragma unroll
    for (int s = 0; s < 4; ++s)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int e = lane + 32 * q;
        v[s][q] = e < E ? __ldg(base + (sp + s) * split_stride + e) : 0.f;
      }
#pragma unroll
    for (int s = 0; s < 4; ++s)
#pragma unroll
      for (int q = 0; q < 4; ++q) l[q] += v[s][q];
  }
  for (; sp < nsplit; ++sp)
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int e = lane + 32 * q;
      l[q] += e < E ? __ldg(base + sp * split_stride + e) : 0.f;
    }
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int e = lane + 32 * q;
    float v = -INFINITY;
    if (e < E) {
      v = l[q] + (bias ? bias[e] : 0.f);
      if (isnan(v)) v = -INFINITY;  // a NaN never wins, so the k winners stay valid experts
    }
    l[q] = v;
  }

  bool taken[4] = {false, false, false, false};
  float top_max = 0.f, sum = 0.f;
  float my_p = 0.f;  // lane (j % 32) keeps slot j's exp(logit_j - logit_0)
  int my_e = 0;
  const uint32_t bit = 1u << (t & (kMaskTokens - 1));
  uint32_t* mrow = masks + static_cast<size_t>(t / kMaskTokens) * E;
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
      const int slot0 = j & ~31;
      if (lane <= j - slot0) {
        idx[static_cast<size_t>(t) * k + slot0 + lane] = my_e;
        wts[static_cast<size_t>(t) * k + slot0 + lane] = my_p;
        atomicOr(mrow + my_e, bit);
      }
    }
  }
  // every lane holds the same sum; each lane rescales the slots it parked
  for (int j = lane; j < k; j += 32) {
    const size_t o = static_cast<size_t>(t) * k + j;
    wts[o] = wts[o] / sum;
  }
}

}  // namespace moe
