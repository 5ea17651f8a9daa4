// Residual packer of the SVDQuant W4A4 linear layer (sm_100a): the residual
// R = diag(lambda) W - L1 L2 (the part of the smoothed weight the low-rank
// branch leaves; chattools.cn article 584, "technical principles") is
// quantised to NVFP4 once per weight.
#pragma once

#include "common.cuh"

namespace svdq {

// ================================================== residual packer ======
// grid (ceil(N/128), K/64), 128 threads.  The CTA transposes a 64 (K) x 128
// (N) fp32 tile through shared memory; thread t owns output row n0 + t and
// writes its 32 code bytes and one 4-byte scale word (one full 512-byte
// scale tile per CTA, zero for padding rows n >= N).
constexpr int kPackThreads = 128;

__global__ void __launch_bounds__(kPackThreads) pack_residual_kernel(const float* __restrict__ R,
                                                                     int K, int N,
                                                                     uint8_t* __restrict__ codes,
                                                                     uint8_t* __restrict__ scales) {
  __shared__ __align__(16) float tile[64][128];
  const int t = threadIdx.x;
  const int n0 = blockIdx.x * 128;
  const int k0 = blockIdx.y * 64;
#pragma unroll
  for (int q = 0; q < 64 * 32 / kPackThreads; ++q) {
    const int i = t + q * kPackThreads;
    const int row = i >> 5, c4 = i & 31;
    const int n = n0 + 4 * c4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (n < N) v = __ldg(reinterpret_cast<const float4*>(R + static_cast<size_t>(k0 + row) * N + n));
    *reinterpret_cast<float4*>(&tile[row][4 * c4]) = v;
  }
  __syncthreads();
  const int n = n0 + t;
  uint32_t cw[8];
  uint32_t sw = 0;
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    float v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = tile[g * 16 + i][t];
    const uint32_t s = nvfp4_group(v, cw[2 * g], cw[2 * g + 1]);
    sw |= s << (8 * g);
  }
  if (n < N) {
    uint4* dst = reinterpret_cast<uint4*>(codes + static_cast<size_t>(n) * (K >> 1) + (k0 >> 1));
    dst[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
    dst[1] = make_uint4(cw[4], cw[5], cw[6], cw[7]);
  }
  *reinterpret_cast<uint32_t*>(scales + scale_word_offset(n, k0 >> 4, K)) = sw;
}

}  // namespace svdq
