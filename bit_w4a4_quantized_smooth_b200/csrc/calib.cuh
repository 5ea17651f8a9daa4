// Smoothing statistics of the SVDQuant W4A4 layer (chattools.cn article 584,
// "technical principles"): the smoothing factor of input channel k is set
// from the largest magnitude the channel takes on calibration activations,
// lambda_k = sqrt(max_i |X_ik|) / sqrt(max_n |W_kn|).  This kernel folds one
// batch of activations into a running per-channel maximum, so that the
// statistic of many calibration batches is gathered on the device.
#pragma once

#include "common.cuh"

namespace svdq {

constexpr int kAbsmaxThreads = 128;

// Thread = 8 consecutive channels (one 16-byte load per row), a block
// covers 1024 channels of a range of rows; the maximum of |bf16| is taken
// on the magnitude bits (order-preserving for non-negative values) and
// merged with atomicMax on the fp32 bit pattern: the result does not depend
// on the order of rows, blocks or batches.  NaN inputs (magnitude bits above
// those of infinity) propagate into the channel's statistic as a NaN.
__global__ void __launch_bounds__(kAbsmaxThreads) channel_absmax_kernel(const __nv_bfloat16* __restrict__ X, int M,
                                                                        int K, int rows_per_block,
                                                                        unsigned int* __restrict__ amax_bits) {
  const int c8 = blockIdx.x * kAbsmaxThreads + threadIdx.x;  // 8-channel chunk
  if (8 * c8 >= K) return;
  const int i0 = blockIdx.y * rows_per_block;
  const int i1 = min(M, i0 + rows_per_block);
  uint32_t m[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  const uint4* src = reinterpret_cast<const uint4*>(X) + static_cast<int64_t>(i0) * (K / 8) + c8;
#pragma unroll 4
  for (int i = i0; i < i1; ++i, src += K / 8) {
    const uint4 v = __ldcs(src);  // streamed once: evict first
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      m[2 * e] = max(m[2 * e], w[e] & 0x7FFFu);
      m[2 * e + 1] = max(m[2 * e + 1], (w[e] >> 16) & 0x7FFFu);
    }
  }
  if (i0 >= i1) return;
#pragma unroll
  for (int e = 0; e < 8; ++e) atomicMax(amax_bits + 8 * c8 + e, m[e] << 16);
}

}  // namespace svdq
