// Device helpers shared by the SVDQuant kernels: shared-memory alignment,
// the NVFP4 group quantiser, the block-scale tile layout and bf16 packing.
//
// NVFP4 (the 4-bit format of the SVDQuant pages' FLUX results, taicenter.com
// news article on the MIT Han Song team's FLUX work): E2M1 elements with one
// unsigned E4M3 scale per 16 consecutive elements, scale = amax / 6.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace svdq {

// First 1024-byte aligned byte of the dynamic shared memory (128-byte
// swizzled TMA / MMA tiles need it).  The offset is added to the shared array
// itself, so the compiler keeps every derived pointer in the shared window
// (LDS/STS) instead of falling back to generic addressing.
__device__ __forceinline__ uint8_t* align_smem_1024(uint8_t* smem_raw) {
  return smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
}

// ------------------------------------------------------ NVFP4 quantiser --
// One group of 16 fp32 values (NVFP4: E2M1 elements, one unsigned E4M3
// scale per 16, scale = amax / 6):
//   s_f = RN_f32(amax / 6); s = E4M3_RNE_satfinite(s_f);
//   rcp = RN_f32(1 / decode(s)) (0 when decode(s) == 0);
//   q_i = E2M1_RNE_satfinite(RN_f32(v_i * rcp)).
// Returns the scale byte; the 16 codes come back as two little-endian words.
__device__ __forceinline__ uint32_t nvfp4_group(const float* v, uint32_t& lo, uint32_t& hi) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const float sf = __fdiv_rn(amax, 6.0f);
  const uint32_t s = cvt_e4m3_satfinite(sf);
  const float sd = e4m3_to_f32(s);
  const float rcp = sd == 0.0f ? 0.0f : __frcp_rn(sd);
  float p[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) p[i] = __fmul_rn(v[i], rcp);
  lo = cvt_e2m1x8(p);
  hi = cvt_e2m1x8(p + 8);
  return s;
}

// Byte offset of the 4 scales (groups g..g+3, g % 4 == 0) of `row` in the
// block-scale tile layout (128-row bands, 512-byte tiles of 128 rows x 4).
__device__ __forceinline__ size_t scale_word_offset(int row, int g, int K) {
  return (static_cast<size_t>(row >> 7) * (K >> 6) + (g >> 2)) * 512 + (row & 31) * 16 +
         ((row & 127) >> 5) * 4;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);  // .x = a (low half)
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Byte offset of the scale of (row, group g) in the block-scale tile layout.
__device__ __forceinline__ size_t scale_byte_offset(int row, int g, int K) {
  return scale_word_offset(row, g & ~3, K) + (g & 3);
}

// (d0, d1) = (a0 * b0, a1 * b1), each rounded to nearest fp32 (packed fp32 pipe).
__device__ __forceinline__ void mul2_rn(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "mul.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

__device__ __forceinline__ void add2_rn(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "add.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

}  // namespace svdq
