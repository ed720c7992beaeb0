// RMSNorm of rows with a learned scale: the pre-FFN norm of the block's
// normalisation sandwich (Gemma-4-26B-A4B model card: "Normalization layer
// type in the blocks": RMSNorm, "Pre-norm, post-norm, or sandwich":
// sandwich, epsilon 1e-06).
//
//   out[t, :] = RNE_bf16(gamma * x[t, :] / sqrt(mean(x[t, :]^2) + 1e-6))
//
// in fp32: one warp per row; each lane sums the squares of its 8-column
// vectors in order and the lanes combine by a fixed xor tree, so the result
// is deterministic. The row is read twice (the second pass from L1/L2).
#pragma once

#include "ptx.cuh"

namespace moe {

constexpr int kNormWarps = 8;

__global__ void __launch_bounds__(kNormWarps * 32) rms_norm_rows_kernel(const __nv_bfloat16* __restrict__ x,
                                                                       const __nv_bfloat16* __restrict__ gamma,
                                                                       int T, int D, __nv_bfloat16* __restrict__ out) {
  pdl_wait_then_release();
  const int lane = threadIdx.x & 31;
  const int nvec = D >> 3;
  for (int t = blockIdx.x * kNormWarps + (threadIdx.x >> 5); t < T; t += gridDim.x * kNormWarps) {
    const uint4* row = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * D);
    float ss = 0.f;
    for (int v = lane; v < nvec; v += 32) {
      const uint4 xv = __ldg(row + v);
      const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(&xv);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float f = __bfloat162float(xb[i]);
        ss = fmaf(f, f, ss);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float r = 1.0f / sqrtf(ss / static_cast<float>(D) + 1e-6f);
    uint4* dst = reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * D);
    for (int v = lane; v < nvec; v += 32) {
      const uint4 xv = __ldg(row + v);
      const uint4 gv = __ldg(reinterpret_cast<const uint4*>(gamma) + v);
      const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(&xv);
      const __nv_bfloat16* gb = reinterpret_cast<const __nv_bfloat16*>(&gv);
      float o[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = __bfloat162float(xb[i]) * r * __bfloat162float(gb[i]);
      dst[v] = make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]),
                          pack_bf16x2(o[6], o[7]));
    }
  }
}

}  // namespace moe
