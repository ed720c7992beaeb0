// Router: logits = x W_router on the tensor cores (bf16 products, fp32
// accumulation), then top-k selection and the softmax of the kept logits.
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

constexpr int kRouterTokens = 128;  // tokens per CTA tile (the MMA's M)
constexpr int kRouterBK = 64;       // reduction elements per pipeline stage
constexpr int kRouterStages = 4;
constexpr int kRouterThreads = 128;
constexpr int kRouterAStage = kRouterTokens * kRouterBK * 2;  // 16 KB of x
constexpr int kRouterBChunk = kRouterBK * 64 * 2;             // 8 KB: 64 K-rows x 64 experts
constexpr int kRouterBStage = 2 * kRouterBChunk;              // up to 128 experts
constexpr int kRouterSmemBytes = kRouterStages * (kRouterAStage + kRouterBStage) + 1024 + 256;
constexpr int kMaskTokens = 32;     // tokens per bitmask word
constexpr int kTopkWarps = 4;       // one warp per token
constexpr int kMaxRouterSplits = 22; // splits of the router's reduction (at most)

struct RouterParams {
  CUtensorMap tmX;  // x [T, D] bf16, box 64 (K) x 128 (tokens), 128-byte swizzle
  CUtensorMap tmW;  // W_router [1, D, E] bf16 (experts contiguous), box 64 x 64 x 1
  float* partial;   // [nsplit][T][E] fp32
  uint32_t* masks;  // [ceil(T / 32)][E], cleared here for top-k's atomicOr
  uint32_t* err;
  int T, D, E, nsplit;
};

// partial[split][t][e] = sum over this split's slice of d of x[t, d] W[d, e].
//
// One CTA per (128-token tile, split of the reduction), 128 threads. Thread 0
// streams the split's 64-wide slices of x (K-major) and W (read as an N-major
// operand, so the weights are used exactly as stored) into a 4-stage ring by
// TMA; thread 32 issues tcgen05.mma (M = 128 tokens, N = 64 or 128 experts,
// K = 16 per instruction) into a 128-column fp32 TMEM accumulator; then the
// four warps each read their 32 TMEM lanes (tokens) and write the partial
// logits. The products of bf16 values are exact in fp32 and the accumulation
// order inside a split is fixed by the hardware, so the result is
// deterministic. Tokens past T and experts past E are zero-filled by the copy
// engine and never stored. CTAs of split 0 also clear the token-expert bitmask
// words of their tokens. Requires E % 8 == 0, E <= 128, D % 64 == 0.
__global__ void __launch_bounds__(kRouterThreads) router_logits_kernel(const __grid_constant__ RouterParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kRouterStages * kRouterAStage;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kRouterStages * (kRouterAStage + kRouterBStage));
  uint64_t* empty = full + kRouterStages;
  uint64_t* acc_full = empty + kRouterStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * kRouterTokens;
  const int split = blockIdx.y;
  const int nkb_all = P.D / kRouterBK;
  const int kb0 = static_cast<int>((static_cast<long long>(split) * nkb_all) / P.nsplit);
  const int kb1 = static_cast<int>((static_cast<long long>(split + 1) * nkb_all) / P.nsplit);
  const int nch = (P.E + 63) >> 6;  // 64-expert chunks of B
  const int n_mma = 64 * nch;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRouterStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&P.tmX);
    tma_prefetch_desc(&P.tmW);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait_then_release();

  if (split == 0 && warp >= 2) {  // warps 2 and 3, while the pipeline fills
    const int words = (min(P.T, t0 + kRouterTokens) - t0 + kMaskTokens - 1) / kMaskTokens;
    for (int i = threadIdx.x - 64; i < words * P.E; i += kRouterThreads - 64)
      P.masks[static_cast<size_t>(t0 / kMaskTokens) * P.E + i] = 0u;
  }

  if (threadIdx.x == 0) {
    // ------------------------------------------------------------ producer
    const uint32_t bytes = kRouterAStage + nch * kRouterBChunk;
    int s = 0, issued = 0;
    uint32_t ph = 0;
    for (int kb = kb0; kb < kb1; ++kb) {
      if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, P.err)) break;
      mbar_arrive_expect_tx(&full[s], bytes);
      tma_load_2d(sA + s * kRouterAStage, &P.tmX, &full[s], kb * kRouterBK, t0);
      for (int c = 0; c < nch; ++c)
        tma_load_3d(sB + s * kRouterBStage + c * kRouterBChunk, &P.tmW, &full[s], c * 64, kb * kRouterBK, 0);
      ++issued;
      if (++s == kRouterStages) {
        s = 0;
        ph ^= 1;
      }
    }
    if (*abort_flag) {
      // let the copies in flight land before the CTA's shared memory goes away
      const int pending = issued < kRouterStages ? issued : kRouterStages;
      for (int i = 0; i < pending; ++i) {
        if (--s < 0) {
          s = kRouterStages - 1;
          ph ^= 1;
        }
        uint32_t dummy = 0;
        mbar_wait(&full[s], ph, reinterpret_cast<volatile int*>(&dummy), P.err, 100000000ull);
      }
    }
  } else if (threadIdx.x == 32) {
    // ---------------------------------------------------------- MMA issuer
    const uint32_t idesc = idesc_bf16_m128(n_mma, 1);
    int s = 0;
    uint32_t ph = 0;
    bool any = false;
    for (int kb = kb0; kb < kb1; ++kb) {
      if (!mbar_wait(&full[s], ph, abort_flag, P.err)) break;
      tc_fence_after_sync();
      const uint32_t a_addr = smem_u32(sA + s * kRouterAStage);
      const uint32_t b_addr = smem_u32(sB + s * kRouterBStage);
#pragma unroll
      for (int k = 0; k < kRouterBK / 16; ++k) {
        // A: K-major rows of 128 B, 8-row groups 1024 B apart, +32 B per 16 K.
        // B: N-major, 8 K-rows per 1024 B swizzle atom, 64-expert chunks 8 KB
        // apart, +2048 B per 16 K.
        umma_f16(tmem_base, sdesc_sw128(a_addr + k * 32, 16, 1024), sdesc_sw128(b_addr + k * 2048, kRouterBChunk, 1024),
                 idesc, (kb != kb0 || k != 0) ? 1u : 0u);
      }
      any = true;
      umma_commit(&empty[s]);
      if (++s == kRouterStages) {
        s = 0;
        ph ^= 1;
      }
    }
    if (any) {
      umma_commit(acc_full);  // every MMA above has completed once this arrives
    } else {
      mbar_arrive(acc_full);  // empty split (never with D >= 64 * nsplit): the partials are zero
    }
    // even after an abort, no MMA may still be running when TMEM is released
    uint32_t dummy = 0;
    mbar_wait(acc_full, 0, reinterpret_cast<volatile int*>(&dummy), P.err);
  }
  __syncwarp();

  // -------------------------------------------------------------- epilogue
  const int arrived = mbar_wait(acc_full, 0, abort_flag, P.err) && !*abort_flag;
  const bool ready = __all_sync(0xffffffffu, arrived);
  if (ready && kb1 > kb0) {
    tc_fence_after_sync();
    const int t = t0 + warp * 32 + lane;
    float* dst = P.partial + (static_cast<size_t>(split) * P.T + t) * P.E;
    for (int j = 0; j < n_mma; j += 32) {
      uint32_t a[32];
      tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(warp * 32) << 16) + j, a);
      tmem_ld_wait();
      if (t < P.T) {
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          if (j + 4 * v < P.E)
            *reinterpret_cast<float4*>(dst + j + 4 * v) =
                make_float4(__uint_as_float(a[4 * v]), __uint_as_float(a[4 * v + 1]), __uint_as_float(a[4 * v + 2]),
                            __uint_as_float(a[4 * v + 3]));
        }
      }
    }
  } else if (ready) {
    const int t = t0 + warp * 32 + lane;
    if (t < P.T)
      for (int e = 0; e < P.E; e += 4)
        *reinterpret_cast<float4*>(P.partial + (static_cast<size_t>(split) * P.T + t) * P.E + e) =
            make_float4(0.f, 0.f, 0.f, 0.f);
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, 128);
  }
}

// One warp per token: sum the split partials in split order, add the bias,
// pick the k largest (ties: lower index), softmax over them, set the token's
// bits in the expert bitmasks; with logits_out, also write the summed logits
// (bias included) as a debug output. Lane l holds experts l, l+32, l+64, l+96.
// ALL_SPLITS (small batches, many splits of the router's reduction): every
// split's loads are in flight at once, one memory round trip instead of one
// per four splits; large batches keep the leaner loop, whose lower register
// count keeps more token warps resident. The sum order is the same.
template <bool ALL_SPLITS>
__global__ void __launch_bounds__(kTopkWarps * 32) router_topk_kernel(const float* __restrict__ partial,
                                                                     const float* __restrict__ bias, int T, int E,
                                                                     int nsplit, int k, int32_t* __restrict__ idx,
                                                                     float* __restrict__ wts,
                                                                     uint32_t* __restrict__ masks,
                                                                     float* __restrict__ logits_out) {
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
  if (ALL_SPLITS) {
    float v[kMaxRouterSplits][4];
#pragma unroll
    for (int s = 0; s < kMaxRouterSplits; ++s)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int e = lane + 32 * q;
        v[s][q] = (s < nsplit && e < E) ? __ldg(base + s * split_stride + e) : 0.f;
      }
#pragma unroll
    for (int s = 0; s < kMaxRouterSplits; ++s)
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (s < nsplit) l[q] += v[s][q];
    sp = nsplit;
  }
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
      if (logits_out) logits_out[static_cast<size_t>(t) * E + e] = v;
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

// The same selection with two tokens per warp (large batches, E <= 128,
// k <= 16): each half-warp holds one token's logits, 8 per lane (expert
// e = lane % 16 + 16 q), so a round's reduction is 4 shuffle steps over 8
// candidates a lane instead of 5 over 4 for one token. The outputs are the
// same: logits summed over the splits in split order, the same order of
// winners (ties: lower index) and the same softmax arithmetic.
__global__ void __launch_bounds__(kTopkWarps * 32) router_topk_pair_kernel(const float* __restrict__ partial,
                                                                          const float* __restrict__ bias, int T,
                                                                          int E, int nsplit, int k,
                                                                          int32_t* __restrict__ idx,
                                                                          float* __restrict__ wts,
                                                                          uint32_t* __restrict__ masks,
                                                                          float* __restrict__ logits_out) {
  pdl_wait_then_release();
  const int lane = threadIdx.x & 31;
  const int hl = lane & 15;
  const int t = (blockIdx.x * kTopkWarps + (threadIdx.x >> 5)) * 2 + (lane >> 4);
  const bool live = t < T;  // a dead half-warp still runs the rounds (its shuffles stay in its half)
  float l[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) l[q] = 0.f;
  const size_t split_stride = static_cast<size_t>(T) * E;
  const float* base = partial + static_cast<size_t>(live ? t : 0) * E;
  int sp = 0;
  for (; sp + 4 <= nsplit; sp += 4) {  // four splits' loads in flight, summed in order
    float v[4][8];
#pragma unroll
    for (int s2 = 0; s2 < 4; ++s2)
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int e = hl + 16 * q;
        v[s2][q] = (live && e < E) ? __ldg(base + (sp + s2) * split_stride + e) : 0.f;
      }
#pragma unroll
    for (int s2 = 0; s2 < 4; ++s2)
#pragma unroll
      for (int q = 0; q < 8; ++q) l[q] += v[s2][q];
  }
  for (; sp < nsplit; ++sp)
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int e = hl + 16 * q;
      l[q] += (live && e < E) ? __ldg(base + sp * split_stride + e) : 0.f;
    }
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int e = hl + 16 * q;
    float v = -INFINITY;
    if (e < E) {
      v = l[q] + (bias ? bias[e] : 0.f);
      if (live && logits_out) logits_out[static_cast<size_t>(t) * E + e] = v;
      if (isnan(v)) v = -INFINITY;  // a NaN never wins, so the k winners stay valid experts
    }
    l[q] = v;
  }

  uint32_t taken = 0u;  // bit q: candidate q of this lane is chosen
  float top_max = 0.f, sum = 0.f;
  float my_p = 0.f;  // lane (j % 16) of the half-warp keeps slot j's exp(logit_j - logit_0)
  int my_e = 0;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int e = hl + 16 * q;
      if (e < E && !((taken >> q) & 1u) && (l[q] > bv || (l[q] == bv && e < be))) {
        bv = l[q];
        be = e;
      }
    }
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oe = __shfl_xor_sync(0xffffffffu, be, off);
      if (ov > bv || (ov == bv && oe < be)) {
        bv = ov;
        be = oe;
      }
    }
    if ((be & 15) == hl) taken |= 1u << ((be >> 4) & 7);
    if (j == 0) top_max = bv;
    const float p = expf(bv - top_max);
    sum += p;
    if (hl == j) {
      my_p = p;
      my_e = be;
    }
  }
  if (live && hl < k) {
    const size_t o = static_cast<size_t>(t) * k + hl;
    idx[o] = my_e;
    wts[o] = my_p / sum;
    atomicOr(masks + static_cast<size_t>(t / kMaskTokens) * E + my_e, 1u << (t & (kMaskTokens - 1)));
  }
}

}  // namespace moe
