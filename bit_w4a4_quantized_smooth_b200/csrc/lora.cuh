// LoRA adapters joined to the SVDQuant low-rank branch on the device
// (chattools.cn article 584, "main functions", item LoRA integration; the
// ai-digest.ru abstract: adapters join without re-quantising the 4-bit
// residual).  With Xh = X diag(lambda)^-1, an adapter A [K][ra], B [ra][N]
// joins as
//     L1' = [L1 | bf16(RN_f32(lambda_k A_kj))],   L2' = [L2 ; B],
// so that Xh L1' L2' = Xh L1 L2 + X A B, and the packed residual is kept.
#pragma once

#include "common.cuh"

namespace svdq {

constexpr int kLoraThreads = 256;

// One thread per 8 consecutive output elements (16 bytes): the rows of L1'
// first, then L2' = [L2 ; B] as one contiguous copy.
__global__ void __launch_bounds__(kLoraThreads) attach_lora_kernel(
    const __nv_bfloat16* __restrict__ L1, const __nv_bfloat16* __restrict__ L2, const float* __restrict__ lambda,
    const __nv_bfloat16* __restrict__ A, const __nv_bfloat16* __restrict__ B, int K, int N, int r, int ra,
    __nv_bfloat16* __restrict__ L1o, __nv_bfloat16* __restrict__ L2o) {
  const int ro = r + ra;
  const int64_t c1 = static_cast<int64_t>(K) * (ro / 8);          // 8-element chunks of L1'
  const int64_t c2 = static_cast<int64_t>(ro) * N / 8;            // ... of L2'
  const int64_t c2a = static_cast<int64_t>(r) * N / 8;            // ... of L2' that come from L2
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < c1 + c2;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    uint4 out;
    if (i < c1) {
      const int64_t k = i / (ro / 8);
      const int c = static_cast<int>(i % (ro / 8));
      if (8 * c < r) {
        out = *reinterpret_cast<const uint4*>(L1 + k * r + 8 * c);
      } else {
        const uint4 a = *reinterpret_cast<const uint4*>(A + k * ra + (8 * c - r));
        const float lam = lambda[k];
        const uint32_t w[4] = {a.x, a.y, a.z, a.w};
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          o[e] = pack_bf16x2(__fmul_rn(lam, bf16_lo(w[e])), __fmul_rn(lam, bf16_hi(w[e])));
        out = make_uint4(o[0], o[1], o[2], o[3]);
      }
      *reinterpret_cast<uint4*>(L1o + k * ro + 8 * c) = out;
    } else {
      const int64_t j = i - c1;
      out = j < c2a ? reinterpret_cast<const uint4*>(L2)[j] : reinterpret_cast<const uint4*>(B)[j - c2a];
      reinterpret_cast<uint4*>(L2o)[j] = out;
    }
  }
}

}  // namespace svdq
