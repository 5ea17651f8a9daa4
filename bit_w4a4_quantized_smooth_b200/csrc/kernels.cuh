// Device kernels of the SVDQuant W4A4 linear layer for sm_100a.
//
//   pack_residual_kernel   R fp32 [K][N] -> NVFP4 codes [N][K/2] + tiled scales
//   quantize_act_kernel    X bf16 [M][K] -> Xh = X * inv_lambda -> NVFP4 codes
//                          and scales, and T = bf16(bf16(Xh) L1) on tcgen05
//   linear_kernel          Y = deq(x) deq(R)^T + T L2 + bias on tcgen05:
//                          block-scaled FP4 MMAs and the rank-r bf16 MMAs
//                          accumulate into one fp32 tensor-memory tile.
//
// Method: SVDQuant (ai-digest.ru abstract; chattools.cn article 584,
// "technical principles"): smoothing moves activation outliers into the
// weights, a 16-bit low-rank branch from the SVD absorbs the weight outliers,
// the residual and the activation are quantised to 4 bits, and the engine
// fuses the low-rank kernels into the 4-bit ones so the activation is not
// read twice.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace svdq {

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

// ============================================ activation quantise + T =====
// One CTA per tile of `rows` consecutive rows of X (rows in {16, 32, .., 128},
// chosen so that the tiles fill the SMs once), over all of K: no split of the
// reduction, hence no partial sums to combine across CTAs.  704 threads:
// warps 0-15 quantise (two teams of 8 taking alternate stages), warp 16 is the
// TMA producer, warp 17 owns the tensor memory and issues the MMAs (both
// issue warp-wide through elect.sync), warps 18-21 keep the fp32 sum of T.
// A stage covers 128 columns of K (two 64-column atoms) in a ring of up to 8:
//   L1 rows [k, k + 128) as two MN-major 128-byte-swizzled atoms of 64 (r) x
//   64 (k) (a second r-atom when r > 64; columns >= r arrive as zeros);
//   the X tile, rows x 128 columns as two K-major 128-byte-swizzled atoms;
//   the 128 inv_lambda values (bulk copy).
// Warp w of a team quantises group w % 8 (16 columns) of every row, one row
// per lane: codes and scale go to global memory, bf16(Xh) back into the
// swizzled tile in place.
// The MMA warp then adds T^T += L1^T Xh^T with tcgen05 bf16 MMAs (M = 128
// lanes of TMEM = the columns of L1, N = rows, K = 16): the row tile is the N
// side, so any multiple of 16 rows is a valid tile.  When r <= 64 the upper
// 64 lanes of A come from a zeroed shared-memory atom.
// The tensor cores' accumulation over a long K loses precision (measured: an
// error growing about linearly with K, biased towards zero, several bf16 ulps
// of small T entries at K = 12288), so every kQaPromote stages the partial
// product (K = 256) goes to one of two tensor-memory blocks, and warps 18-21
// add it into an fp32 running sum on the CUDA cores (fixed order: block 0, 1,
// ...), overlapping the next block's MMAs.  With the last block they write T
// rows as bf16 (lane j of the accumulator = column j of T).
constexpr int kQaQuantWarps = 16;
constexpr int kQaThreads = kQaQuantWarps * 32 + 64 + 128;
constexpr int kQaPromote = 2;  // stages (of 128 columns) per tensor-core partial sum
constexpr int kQaMaxStages = 8;
constexpr int kQaMaxRows = 128;
constexpr uint32_t kQaZeroBytes = 8192;
constexpr uint32_t kQaBarBytes = 256;
constexpr uint32_t kQaSmemLimit = 232448;  // 227 KB opt-in dynamic shared memory

struct QaParams {
  const float* inv_lambda;
  uint8_t* x_codes;
  uint8_t* x_scales;
  __nv_bfloat16* T;
  int M, K, r, rows, stages, m_pad;
  uint32_t stage_bytes;
  uint64_t timeout_ns;
};

// L1 bytes of a stage: two k-atoms of one (r <= 64) or two (r > 64) 8 KB r-atoms
__host__ __device__ constexpr uint32_t qa_l1_bytes(int r) {
  return r == 0 ? 0u : (r > 64 ? 32768u : 16384u);
}
__host__ __device__ constexpr uint32_t qa_stage_bytes(int r, int rows) {
  return (qa_l1_bytes(r) + 2u * static_cast<uint32_t>(rows) * 128u + 512u + 1023u) & ~1023u;
}
__host__ __device__ constexpr uint32_t qa_zero_bytes(int r) {
  return (r > 0 && r <= 64) ? kQaZeroBytes : 0u;
}

// Byte offset of the scale of (row, group g) in the block-scale tile layout.
__device__ __forceinline__ size_t scale_byte_offset(int row, int g, int K) {
  return scale_word_offset(row, g & ~3, K) + (g & 3);
}

__global__ void __launch_bounds__(kQaThreads, 1)
    quantize_act_kernel(const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ CUtensorMap tm_l1, const QaParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int r = p.r;
  const bool has_lr = r > 0;
  const int S = p.stages;
  const int rows = p.rows;
  const int K = p.K;
  const uint32_t stage_bytes = p.stage_bytes;
  const uint32_t l1_bytes = qa_l1_bytes(r);
  const uint32_t katom_l1 = l1_bytes / 2;
  const uint32_t x_atom = static_cast<uint32_t>(rows) * 128u;
  const uint32_t x_bytes = 2u * x_atom;
  uint8_t* zero = smem + S * stage_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(zero + qa_zero_bytes(r));
  uint64_t* full = bars;               // TMA landed
  uint64_t* quant = bars + S;          // 8 quantising warps done with the stage
  uint64_t* freed = bars + 2 * S;      // MMAs done reading the stage
  uint64_t* fin = bars + 3 * S;        // every MMA of the CTA complete
  uint64_t* acc_full = fin + 1;        // [2] a block's partial product is in tensor memory
  uint64_t* acc_empty = fin + 3;       // [2] ... and has been added into the running sum
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int row0 = blockIdx.x * rows;
  const int nst = (K / 64 + 1) / 2;  // stages of 128 columns; the last may hold one atom
  // tensor memory: running sum at column 0, partial-product blocks at RW, 2 RW
  const uint32_t RW = rows <= 32 ? 32u : (rows <= 64 ? 64u : 128u);
  const uint32_t tmem_cols = 4 * RW;
  const int nblk = (nst + kQaPromote - 1) / kQaPromote;

  if (warp == 17 && has_lr) {
    tmem_alloc(smem_u32(tmem_slot), tmem_cols);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&quant[s]), kQaQuantWarps / 2);
      mbar_init(smem_u32(&freed[s]), 1);
    }
    mbar_init(smem_u32(fin), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&acc_full[b]), 1);
      mbar_init(smem_u32(&acc_empty[b]), 4);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (qa_zero_bytes(r) && tid < static_cast<int>(kQaZeroBytes / 16)) {
    reinterpret_cast<uint4*>(zero)[tid] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = has_lr ? *tmem_slot : 0u;
  const uint32_t smem_base = smem_u32(smem);

  if (warp == 16) {
    // --------------------------------------------------------- producer --
    if (lane == 0) {
      prefetch_tmap(&tm_x);
      if (has_lr) prefetch_tmap(&tm_l1);
    }
    __syncwarp();
    int issued = 0;
    for (int c = 0; c < nst; ++c) {
      const int s = c % S;
      if (c >= S) {
        // the stage's previous chunk: MMAs done reading it (or, without a
        // low-rank branch, its quantisers done)
        if (!warp_wait(smem_u32(&freed[s]), ((c / S) - 1) & 1, p.timeout_ns, 11)) {
          *abort_flag = 1;
          break;
        }
      }
      const int k = c * 128;
      const int na = K - k >= 128 ? 2 : 1;  // 64-column atoms in this stage
      const uint32_t fb = smem_u32(&full[s]);
      const uint32_t dst = smem_base + s * stage_bytes;
      e_arrive_expect_tx(fb, na * (katom_l1 + x_atom + 256u));
      for (int a = 0; a < na; ++a) {
        e_tma_load_2d(dst + l1_bytes + a * x_atom, &tm_x, fb, k + 64 * a, row0);
        if (has_lr) {
          e_tma_load_2d(dst + a * katom_l1, &tm_l1, fb, 0, k + 64 * a);
          if (r > 64) e_tma_load_2d(dst + a * katom_l1 + 8192u, &tm_l1, fb, 64, k + 64 * a);
        }
      }
      e_bulk_load(dst + l1_bytes + x_bytes, p.inv_lambda + k, na * 256u, fb);
      ++issued;
    }
    if (warp_flag(abort_flag))  // let this CTA's own copies land before it can exit
      for (int c = issued > S ? issued - S : 0; c < issued; ++c)
        warp_wait(smem_u32(&full[c % S]), (c / S) & 1, p.timeout_ns, 14);
  } else if (warp == 17) {
    // ------------------------------------------------------- MMA issuer --
    // bf16 x bf16 -> fp32, A = L1^T MN-major, B = Xh K-major, M = 128, N = rows
    const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) |
                           (static_cast<uint32_t>(rows >> 3) << 17) | (8u << 24);
    const uint32_t zero_addr = smem_u32(zero);
    for (int c = 0; c < nst; ++c) {
      const int s = c % S;
      const int b = c / kQaPromote;
      const uint32_t buf = b & 1;
      const bool first = c % kQaPromote == 0;
      if (warp_flag(abort_flag)) break;
      if (has_lr && first && b >= 2 &&
          !warp_wait(smem_u32(&acc_empty[buf]), ((b >> 1) - 1) & 1, p.timeout_ns, 15)) {
        *abort_flag = 1;
        break;
      }
      if (!warp_wait(smem_u32(&quant[s]), (c / S) & 1, p.timeout_ns, 10)) {
        *abort_flag = 1;
        break;
      }
      if (has_lr) {
        tc_fence_after();
        const uint32_t d = tmem + RW * (1 + buf);
        const int na = K - c * 128 >= 128 ? 2 : 1;
        const uint32_t st = smem_base + s * stage_bytes;
        for (int a = 0; a < na; ++a) {
          const uint32_t l1a = st + a * katom_l1;
          const uint32_t xa = st + l1_bytes + a * x_atom;
          // second r-atom (A rows 64..127): loaded for r > 64, else the zero atom
          const uint32_t lbo = r > 64 ? 8192u : zero_addr - l1a;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            e_mma_bf16(d, make_sdesc(l1a + kk * 2048, lbo, 1024, 2), make_sdesc(xa + kk * 32, 16, 1024, 2),
                       idesc, (first && (a | kk) == 0) ? 0u : 1u);
        }
        e_commit(smem_u32(&freed[s]));
        if (c % kQaPromote == kQaPromote - 1 || c == nst - 1) e_commit(smem_u32(&acc_full[buf]));
      } else {
        e_arrive(smem_u32(&freed[s]));
      }
    }
    if (has_lr) e_commit(smem_u32(fin));
  } else if (warp >= 18) {
    // ------------------------------------------- fp32 running sum of T --
    const int q = warp & 3;  // tensor-memory lane quadrant of this warp
    const bool active = 32 * q < r;
    const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
    const int j = 32 * q + lane;  // column of T held by this lane
    for (int b = 0; has_lr && b < nblk; ++b) {
      const uint32_t buf = b & 1;
      if (!warp_wait(smem_u32(&acc_full[buf]), (b >> 1) & 1, p.timeout_ns, 16)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      if (active) {
        const bool last = b == nblk - 1;
        for (int n0 = 0; n0 < rows; n0 += 16) {
          uint32_t v[16], t[16];
          tmem_ld_32x32b_x16(tmem + lane_base + RW * (1 + buf) + n0, v);
          if (b > 0) tmem_ld_32x32b_x16(tmem + lane_base + n0, t);
          tmem_ld_wait();
          if (b > 0) {
#pragma unroll
            for (int i = 0; i < 16; ++i)
              v[i] = __float_as_uint(__fadd_rn(__uint_as_float(t[i]), __uint_as_float(v[i])));
          }
          if (!last) {
            tmem_st_32x32b_x16(tmem + lane_base + n0, v);
          } else if (j < r) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int m = row0 + n0 + i;
              if (m < p.M) p.T[static_cast<size_t>(m) * r + j] = __float2bfloat16_rn(__uint_as_float(v[i]));
            }
          }
        }
        if (!last) tmem_st_wait();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&acc_empty[buf]));
    }
  } else {
    // ------------------------------------------------------- quantisers --
    const int team = warp >> 3;
    const int g = warp & 7;  // the 16-column group of each stage this warp quantises
    for (int c = team; c < nst; c += 2) {
      const int s = c % S;
      // warp-uniform outcome: the warp meets __syncwarp below together
      const bool ok = !warp_flag(abort_flag) && warp_wait(smem_u32(&full[s]), (c / S) & 1, p.timeout_ns, 12);
      if (!ok) {
        *abort_flag = 1;
        break;
      }
      const int k = c * 128;
      const int ng = K - k >= 128 ? 8 : 4;  // groups per row in this stage
      if (g < ng) {
        uint8_t* stage = smem + s * stage_bytes;
        const float4* lam = reinterpret_cast<const float4*>(stage + l1_bytes + x_bytes) + 4 * g;
        const float4 l0 = lam[0], l1 = lam[1], l2 = lam[2], l3 = lam[3];
        const int kg = k + 16 * g;
        const int j0 = (g & 3) * 2;  // logical 16-byte chunk of the row
        uint8_t* atom = stage + l1_bytes + (g >> 2) * x_atom;
        for (int rr = lane; rr < rows; rr += 32) {
          uint8_t* row = atom + rr * 128;
          const int sw = rr & 7;  // 128-byte swizzle phase of the row
          uint4 w0 = *reinterpret_cast<const uint4*>(row + ((j0 ^ sw) << 4));
          uint4 w1 = *reinterpret_cast<const uint4*>(row + (((j0 + 1) ^ sw) << 4));
          float v[16];
          v[0] = __fmul_rn(bf16_lo(w0.x), l0.x);  v[1] = __fmul_rn(bf16_hi(w0.x), l0.y);
          v[2] = __fmul_rn(bf16_lo(w0.y), l0.z);  v[3] = __fmul_rn(bf16_hi(w0.y), l0.w);
          v[4] = __fmul_rn(bf16_lo(w0.z), l1.x);  v[5] = __fmul_rn(bf16_hi(w0.z), l1.y);
          v[6] = __fmul_rn(bf16_lo(w0.w), l1.z);  v[7] = __fmul_rn(bf16_hi(w0.w), l1.w);
          v[8] = __fmul_rn(bf16_lo(w1.x), l2.x);  v[9] = __fmul_rn(bf16_hi(w1.x), l2.y);
          v[10] = __fmul_rn(bf16_lo(w1.y), l2.z); v[11] = __fmul_rn(bf16_hi(w1.y), l2.w);
          v[12] = __fmul_rn(bf16_lo(w1.z), l3.x); v[13] = __fmul_rn(bf16_hi(w1.z), l3.y);
          v[14] = __fmul_rn(bf16_lo(w1.w), l3.z); v[15] = __fmul_rn(bf16_hi(w1.w), l3.w);
          uint32_t lo, hi;
          const uint32_t sc = nvfp4_group(v, lo, hi);
          if (has_lr) {
            w0 = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                            pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
            w1 = make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]),
                            pack_bf16x2(v[12], v[13]), pack_bf16x2(v[14], v[15]));
            *reinterpret_cast<uint4*>(row + ((j0 ^ sw) << 4)) = w0;
            *reinterpret_cast<uint4*>(row + (((j0 + 1) ^ sw) << 4)) = w1;
          }
          const int m = row0 + rr;
          if (m < p.M)
            *reinterpret_cast<uint2*>(p.x_codes + static_cast<size_t>(m) * (K >> 1) + (kg >> 1)) =
                make_uint2(lo, hi);
          if (m < p.m_pad) p.x_scales[scale_byte_offset(m, kg >> 4, K)] = static_cast<uint8_t>(sc);
        }
      }
      if (has_lr) fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&quant[s]));
    }
    // scale-layout padding rows that no tile covers: zero scales
    const int covered = gridDim.x * rows;
    if (blockIdx.x == gridDim.x - 1 && covered < p.m_pad) {
      const int gk = K >> 4;
      for (int i = tid; i < (p.m_pad - covered) * gk; i += kQaQuantWarps * 32)
        p.x_scales[scale_byte_offset(covered + i / gk, i % gk, K)] = 0;
    }
  }

  if (has_lr) {
    // every MMA of this CTA (also after an abort) completes before the
    // tensor memory is released
    if (!mbar_wait(smem_u32(fin), 0, p.timeout_ns, 13)) *abort_flag = 1;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 17 && has_lr) tmem_dealloc(tmem, tmem_cols);
}

// ================================================== fused 4-bit linear ====
// Persistent CTA pairs (clusters of 2): grid = 2 x min(pair tiles, SMs / 2),
// 192 threads per CTA: warp 0 TMA producer, warp 1 TMEM owner and (even CTA)
// MMA issuer, warps 2-5 epilogue.  Issue loops run warp-wide and elect one
// lane per instruction.
// A pair computes 256 x 256 output tiles, visited M-fastest (tile t ->
// m = t % Mt, n = t / Mt); pair p takes tiles p, p + pairs, ...  CTA c of the
// pair holds rows [128 c, 128 c + 128) of the tile's x codes and columns
// [128 c, 128 c + 128) of its R codes; the even CTA issues 2-SM tcgen05 MMAs
// (M = 256, N = 256) that read both CTAs' operands and leave each CTA's 128
// output rows in its own tensor memory.
// A 5-stage shared-memory ring per CTA carries, for each tile in order:
//   ceil(r/64) low-rank stages: 128 rows of T [x 64 ranks] in the A slot and
//     this CTA's 128 columns of L2 [64 ranks x 128] (N-major) in the B slot,
//     consumed by r/16 bf16 MMAs (the first one initialises the accumulator);
//   ceil(K/256) FP4 stages: x codes [128 x 128 B] and R codes [128 x 128 B]
//     (K-major, 128-byte swizzle), the scale tiles of this CTA's 128 x rows
//     and of all 256 R rows of the tile; per 64-wide K block the MMA warp
//     copies the scales into tensor memory (tcgen05.cp, both CTAs at once)
//     and issues one block-scaled MMA.  The tensor pipe runs a thread's
//     copies and MMAs in order, so one scale region suffices and no
//     handshake sits between scale copies and MMAs.
// All TMA loads of a stage (both CTAs, codes and scales) complete on the
// even CTA's barrier.
// Two 128 x 256 fp32 accumulators overlap in each CTA's TMEM: tile i uses
// columns [0, 256) if i is even, [192, 448) if odd; scales sit in [448, 496).
// The epilogue drains the 64 shared columns first and releases them, so the
// next tile's MMAs start while the epilogue is still running; each warp
// writes its 32 x 64 output blocks through a 128-byte-swizzled staging
// buffer with TMA stores (which also clip the M and N tails).
constexpr int kLinThreads = 192;
constexpr int kLinStages = 5;
constexpr int kLinBM = 256, kLinBN = 256, kLinBK = 256;   // pair tile; K per stage
constexpr uint32_t kLinABytes = 16384, kLinBBytes = 16384, kLinSfaBytes = 2048, kLinSfbBytes = 4096;
constexpr uint32_t kLinStageBytes = kLinABytes + kLinBBytes + kLinSfaBytes + kLinSfbBytes;
constexpr uint32_t kLinTmemCols = 512;
constexpr uint32_t kLinAcc1Col = 192;       // second accumulator; [192, 256) shared
constexpr uint32_t kLinSfaCol = 448, kLinSfbCol = 464;
constexpr uint32_t kLinStageOut = kLinStages * kLinStageBytes + 1024;  // after the bias buffer
constexpr uint32_t kLinOutBytes = 4096;     // one warp's 32 x 64 bf16 output block
constexpr uint32_t kLinBarOffset = kLinStageOut + 4 * 2 * kLinOutBytes;  // 2 blocks per epilogue warp
constexpr int kLinNumBars = 2 * kLinStages + 2 + 2 + 1 + 1;

struct LinParams {
  const __nv_bfloat16* bias;
  __nv_bfloat16* Y;
  int M, K, N, r;
  int m_tiles, tiles;  // pair tiles: ceil(M / 256) x ceil(N / 256)
  uint64_t timeout_ns;
};

// FULL_K: K is a multiple of 256, every FP4 stage has four K blocks and
// runs a straight-line issue sequence (scale copies, then four MMAs).
template <bool FULL_K>
__global__ void __launch_bounds__(kLinThreads, 1)
    linear_kernel(const __grid_constant__ CUtensorMap tm_xc, const __grid_constant__ CUtensorMap tm_rc,
                  const __grid_constant__ CUtensorMap tm_xs, const __grid_constant__ CUtensorMap tm_rs,
                  const __grid_constant__ CUtensorMap tm_t, const __grid_constant__ CUtensorMap tm_l2,
                  const __grid_constant__ CUtensorMap tm_y, const LinParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  float* bias_s = reinterpret_cast<float*>(smem + kLinStages * kLinStageBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kLinBarOffset);
  uint64_t* full = bars;                           // [S] even CTA: both CTAs' stage landed
  uint64_t* empty = full + kLinStages;             // [S] the stage's MMAs and copies are done
  uint64_t* acc_full = empty + kLinStages;         // [2] tile accumulated (both CTAs)
  uint64_t* acc_empty = acc_full + 2;              // [2] even CTA: 8 epilogue warps drained it
  uint64_t* ovl_free = acc_empty + 2;              // even CTA: shared columns drained
  uint64_t* fin = ovl_free + 1;                    // even CTA: every MMA complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kLinNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const uint32_t rank = cluster_ctarank();  // 0 = even CTA (MMA issuer)
  const int pair = blockIdx.x >> 1;
  const int pairs = gridDim.x >> 1;
  const int K = p.K, N = p.N, r = p.r;
  const int n_lr = (r + 63) / 64;
  const int n_k = (K + kLinBK - 1) / kLinBK;
  const int total = n_lr + n_k;
  const int tiles_k = K >> 6;

  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), kLinTmemCols);
    tmem_relinquish_pair();
  }
  if (tid == 0) {
    for (int s = 0; s < kLinStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&acc_full[b]), 1);
      mbar_init(smem_u32(&acc_empty[b]), 8);
    }
    mbar_init(smem_u32(ovl_free), 8);
    mbar_init(smem_u32(fin), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the even CTA's barriers exist before anyone signals them
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sbase = smem_u32(smem);
  auto lead = [&](const uint64_t* bar) { return map_shared_rank(smem_u32(bar), 0); };

  if (warp == 0) {
    // ------------------------------------------------------- producer --
    if (lane == 0) {
      prefetch_tmap(&tm_xc);
      prefetch_tmap(&tm_rc);
      prefetch_tmap(&tm_xs);
      prefetch_tmap(&tm_rs);
      if (r > 0) {
        prefetch_tmap(&tm_t);
        prefetch_tmap(&tm_l2);
      }
    }
    __syncwarp();
    uint32_t g = 0;
    bool ok = true;
    for (int t = pair; t < p.tiles && ok && !warp_flag(abort_flag); t += pairs) {
      const int band = (t % p.m_tiles) * 2 + static_cast<int>(rank);  // this CTA's 128 rows
      const int m0 = band * 128;
      const int n0 = (t / p.m_tiles) * kLinBN;
      const int nb = n0 + 128 * static_cast<int>(rank);  // this CTA's R rows
      for (int it = 0; it < total; ++it, ++g) {
        const int s = g % kLinStages;
        const uint32_t ph = (g / kLinStages) & 1;
        ok = warp_wait(smem_u32(&empty[s]), ph ^ 1, p.timeout_ns, 20);
        if (!ok) {
          *abort_flag = 1;
          break;
        }
        const uint32_t fb = lead(&full[s]);
        const uint32_t a_s = sbase + s * kLinStageBytes;
        const uint32_t b_s = a_s + kLinABytes;
        if (it < n_lr) {
          if (rank == 0) e_arrive_expect_tx(smem_u32(&full[s]), 2 * (kLinABytes + kLinBBytes));
          const int j0 = it * 64;
          e_tma_load_2d_pair(a_s, &tm_t, fb, j0, m0);
          e_tma_load_2d_pair(b_s, &tm_l2, fb, nb, j0);
          e_tma_load_2d_pair(b_s + 8192, &tm_l2, fb, nb + 64, j0);
        } else {
          if (rank == 0) e_arrive_expect_tx(smem_u32(&full[s]), 2 * kLinStageBytes);
          const int kt = (it - n_lr) * (kLinBK / 64);
          const uint32_t sfa_s = b_s + kLinBBytes;
          const uint32_t sfb_s = sfa_s + kLinSfaBytes;
          e_tma_load_2d_pair(a_s, &tm_xc, fb, kt * 32, m0);
          e_tma_load_2d_pair(b_s, &tm_rc, fb, kt * 32, nb);
          // scale tiles: [512-byte tile][4 K blocks]; boxes past the end of
          // a band (or of the tensor) read zeros and are never used
          e_tma_load_3d_pair(sfa_s, &tm_xs, fb, 0, 0, band * tiles_k + kt);
          e_tma_load_3d_pair(sfb_s, &tm_rs, fb, 0, 0, (n0 >> 7) * tiles_k + kt);
          e_tma_load_3d_pair(sfb_s + 2048, &tm_rs, fb, 0, 0, ((n0 >> 7) + 1) * tiles_k + kt);
        }
      }
    }
    // after an abort: the even CTA's barriers see both CTAs' copies land
    // before the pair can pass its final cluster barrier
    if (rank == 0 && warp_flag(abort_flag))
      for (uint32_t j = g > kLinStages ? g - kLinStages : 0; j < g; ++j)
        warp_wait(smem_u32(&full[j % kLinStages]), (j / kLinStages) & 1, p.timeout_ns, 26);
  } else if (warp == 1) {
    if (rank == 0) {
      // -------------------------------------------------- MMA issuer --
      const uint32_t idesc_f4 = (1u << 7) | (1u << 10) | ((kLinBN >> 3) << 17) | ((kLinBM >> 4) << 24);
      const uint32_t idesc_bf = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                ((kLinBN >> 3) << 17) | ((kLinBM >> 4) << 24);
      const uint32_t sfa_t = tmem + kLinSfaCol;
      const uint32_t sfb_t = tmem + kLinSfbCol;
      uint32_t g = 0;
      int i = 0;
      bool ok = true;
      for (int t = pair; t < p.tiles && ok && !warp_flag(abort_flag); t += pairs, ++i) {
        const int b = i & 1;
        const uint32_t acc = tmem + (b ? kLinAcc1Col : 0u);
        if (i >= 2) ok = warp_wait_cluster(smem_u32(&acc_empty[b]), ((i >> 1) - 1) & 1, p.timeout_ns, 21);
        if (ok && i >= 1) ok = warp_wait_cluster(smem_u32(ovl_free), (i - 1) & 1, p.timeout_ns, 22);
        if (!ok) break;
        tc_fence_after();
        for (int it = 0; it < total && ok; ++it, ++g) {
          const int s = g % kLinStages;
          const uint32_t ph = (g / kLinStages) & 1;
          ok = warp_wait(smem_u32(&full[s]), ph, p.timeout_ns, 23);
          if (!ok) break;
          const uint32_t a_s = sbase + s * kLinStageBytes;
          const uint32_t b_s = a_s + kLinABytes;
          tc_fence_after();
          if (it < n_lr) {
            const int nk16 = min(4, (r - it * 64) / 16);
            for (int kk = 0; kk < nk16; ++kk)
              e_mma_bf16_pair(acc, make_sdesc(a_s + kk * 32, 16, 1024, 2),
                              make_sdesc(b_s + kk * 2048, 8192, 1024, 2), idesc_bf, (it > 0 || kk > 0) ? 1u : 0u);
          } else {
            const uint32_t sfa_s = b_s + kLinBBytes;
            const uint32_t sfb_s = sfa_s + kLinSfaBytes;
            if constexpr (FULL_K) {
              // copies first, then the MMAs: copies issued back to back cost
              // the tensor pipe far less than copies interleaved with MMAs
              const uint32_t first = (it > 0) ? 1u : 0u;
#pragma unroll
              for (int kb = 0; kb < 4; ++kb)
                e_tmem_cp_pair_32x128b_warpx4(sfa_t + 4 * kb, make_sdesc(sfa_s + kb * 512, 0, 128, 0));
#pragma unroll
              for (int kb = 0; kb < 4; ++kb) {
                e_tmem_cp_pair_32x128b_warpx4(sfb_t + 8 * kb, make_sdesc(sfb_s + kb * 512, 0, 128, 0));
                e_tmem_cp_pair_32x128b_warpx4(sfb_t + 8 * kb + 4, make_sdesc(sfb_s + 2048 + kb * 512, 0, 128, 0));
              }
#pragma unroll
              for (int kb = 0; kb < 4; ++kb)
                e_mma_nvf4_pair(acc, make_sdesc(a_s + kb * 32, 16, 1024, 2), make_sdesc(b_s + kb * 32, 16, 1024, 2),
                                idesc_f4, sfa_t + 4 * kb, sfb_t + 8 * kb, kb > 0 ? 1u : first);
            } else {
              const int k0 = (it - n_lr) * kLinBK;
              const int nkb = min(4, (K - k0) / 64);
              for (int kb = 0; kb < nkb; ++kb) {
                e_tmem_cp_pair_32x128b_warpx4(sfa_t + 4 * kb, make_sdesc(sfa_s + kb * 512, 0, 128, 0));
                e_tmem_cp_pair_32x128b_warpx4(sfb_t + 8 * kb, make_sdesc(sfb_s + kb * 512, 0, 128, 0));
                e_tmem_cp_pair_32x128b_warpx4(sfb_t + 8 * kb + 4, make_sdesc(sfb_s + 2048 + kb * 512, 0, 128, 0));
                e_mma_nvf4_pair(acc, make_sdesc(a_s + kb * 32, 16, 1024, 2), make_sdesc(b_s + kb * 32, 16, 1024, 2),
                                idesc_f4, sfa_t + 4 * kb, sfb_t + 8 * kb, (it > 0 || kb > 0) ? 1u : 0u);
              }
            }
          }
          e_commit_pair_both(smem_u32(&empty[s]));
        }
        e_commit_pair_both(smem_u32(&acc_full[b]));
      }
      if (!ok) *abort_flag = 1;
      // own MMAs (which write both CTAs' tensor memory) complete before the
      // pair may release it
      e_commit_pair_both(smem_u32(fin));
      if (!warp_wait(smem_u32(fin), 0, p.timeout_ns, 25)) *abort_flag = 1;
    }
  } else {
    // ------------------------------------------------------- epilogue --
    const int et = tid - 64;   // 0..127
    const int q = warp & 3;    // TMEM lane quadrant this warp may access
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    uint8_t* out_s = smem + kLinStageOut + (warp - 2) * 2 * kLinOutBytes;
    int i = 0;
    for (int t = pair; t < p.tiles; t += pairs, ++i) {
      const int b = i & 1;
      const int m0 = ((t % p.m_tiles) * 2 + static_cast<int>(rank)) * 128;
      const int n0 = (t / p.m_tiles) * kLinBN;
      named_bar_sync(1, 128);  // everyone is done with the previous tile's bias
      for (int j = et; j < kLinBN; j += 128) {
        const int n = n0 + j;
        bias_s[j] = (p.bias && n < N) ? __bfloat162float(p.bias[n]) : 0.0f;
      }
      named_bar_sync(1, 128);
      // no early exit: all four warps must keep meeting the named barriers
      const bool ok = !warp_flag(abort_flag) && warp_wait(smem_u32(&acc_full[b]), (i >> 1) & 1, p.timeout_ns, 30);
      if (!ok) {
        *abort_flag = 1;
        continue;
      }
      tc_fence_after();
      const uint32_t acc_col = b ? kLinAcc1Col : 0u;
#pragma unroll 1
      for (int gi = 0; gi < 4; ++gi) {
        // 64-column groups; the 64 shared columns ([192, 256)) come first
        const int c0 = b ? 2 * gi : ((6 + 2 * gi) & 7);  // first 32-column chunk
        uint32_t v[64];
        tmem_ld_32x32b_x32(tmem + lane_base + acc_col + 32 * c0, v);
        tmem_ld_32x32b_x32(tmem + lane_base + acc_col + 32 * c0 + 32, v + 32);
        tmem_ld_wait();
        if (gi == 0 || gi == 3) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(lead(gi == 0 ? ovl_free : &acc_empty[b]));
        }
        // staging block (alternating per group) must no longer be read by
        // this warp's previous TMA store
        uint8_t* blk = out_s + (gi & 1) * kLinOutBytes;
        if (lane == 0) bulk_wait_group_read<1>();
        __syncwarp();
        uint8_t* rowp = blk + lane * 128;
        const float* bs = bias_s + 32 * c0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {  // 16-byte chunk j = columns 8 j .. 8 j + 7
          const uint4 w = make_uint4(pack_bf16x2(__uint_as_float(v[8 * j + 0]) + bs[8 * j + 0],
                                                 __uint_as_float(v[8 * j + 1]) + bs[8 * j + 1]),
                                     pack_bf16x2(__uint_as_float(v[8 * j + 2]) + bs[8 * j + 2],
                                                 __uint_as_float(v[8 * j + 3]) + bs[8 * j + 3]),
                                     pack_bf16x2(__uint_as_float(v[8 * j + 4]) + bs[8 * j + 4],
                                                 __uint_as_float(v[8 * j + 5]) + bs[8 * j + 5]),
                                     pack_bf16x2(__uint_as_float(v[8 * j + 6]) + bs[8 * j + 6],
                                                 __uint_as_float(v[8 * j + 7]) + bs[8 * j + 7]));
          *reinterpret_cast<uint4*>(rowp + ((j ^ (lane & 7)) << 4)) = w;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tm_y, smem_u32(blk), n0 + 32 * c0, m0 + 32 * q);
          bulk_commit_group();
        }
      }
    }
    if (lane == 0) bulk_wait_group<0>();  // stores complete before the CTA exits
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the pair's MMAs are complete before either CTA frees TMEM
  if (warp == 1) tmem_dealloc_pair(tmem, kLinTmemCols);
}

// ============================================== bounded-wait self test ====
// One thread waits on a barrier that nothing completes; the wait expires
// after `timeout_ns` and records SVDQ_ERR_TIMEOUT (id 1).
__global__ void wait_timeout_selftest_kernel(uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
    mbar_wait(smem_u32(&bar), 0, timeout_ns, 1);
  }
}

}  // namespace svdq
