// RMSNorm of rows with a learned scale: the pre-FFN norm of the block's
// normalisation sandwich (Gemma-4-26B-A4B model card: "Normalization layer
// type in the blocks": RMSNorm, "Pre-norm, post-norm, or sandwich":
// sandwich, epsilon 1e-06).
//
//   out[t, :] = RNE_bf16(gamma * x[t, :] / sqrt(mean(x[t, :]^2) + 1e-6))
//
// in fp32: one 128-thread CTA per row, each thread holding up to 4 of the
// row's 8-column vectors in registers (D <= 4096), so the row is read once;
// each thread sums its squares in order, then a fixed warp-xor tree and the
// warps in order: deterministic.
#pragma once

#include "ptx.cuh"

namespace moe {

constexpr int kNormThreads = 128;
constexpr int kNormVec = 4;  // D <= 128 * 4 * 8 = 4096

__global__ void __launch_bounds__(kNormThreads) rms_norm_rows_kernel(const __nv_bfloat16* __restrict__ x,
                                                                    const __nv_bfloat16* __restrict__ gamma, int T,
                                                                    int D, __nv_bfloat16* __restrict__ out) {
  __shared__ float s_red[kNormThreads / 32];
  pdl_wait_then_release();
  const int t = blockIdx.x;
  const int nvec = D >> 3;
  const uint4* row = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * D);
  uint4 xv[kNormVec];
  float ss = 0.f;
#pragma unroll
  for (int u = 0; u < kNormVec; ++u) {
    const int v = threadIdx.x + u * kNormThreads;
    xv[u] = v < nvec ? __ldg(row + v) : make_uint4(0, 0, 0, 0);
    const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(&xv[u]);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float f = __bfloat162float(xb[i]);
      ss = fmaf(f, f, ss);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int i = 0; i < kNormThreads / 32; ++i) tot += s_red[i];
  const float r = 1.0f / sqrtf(tot / static_cast<float>(D) + 1e-6f);
  uint4* dst = reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * D);
#pragma unroll
  for (int u = 0; u < kNormVec; ++u) {
    const int v = threadIdx.x + u * kNormThreads;
    if (v >= nvec) continue;
    const uint4 gv = __ldg(reinterpret_cast<const uint4*>(gamma) + v);
    const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(&xv[u]);
    const __nv_bfloat16* gb = reinterpret_cast<const __nv_bfloat16*>(&gv);
    float o[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = __bfloat162float(xb[i]) * r * __bfloat162float(gb[i]);
    dst[v] = make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]),
                        pack_bf16x2(o[6], o[7]));
  }
}

}  // namespace moe
