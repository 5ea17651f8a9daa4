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
// grid (ks, ceil(M/128)) with clusters of ks CTAs along x; 288 threads:
// warps 0-7 quantise, warp 8 is the producer and MMA issuer.
// CTA (q, b) handles rows [128 b, 128 b + 128) and K-chunks
// [q * cpc, (q + 1) * cpc) of 64 columns.  Per chunk, in a 4-stage ring:
//   warp 8 loads by TMA the X tile (128 rows x 128 B, 128-byte swizzle), the
//   matching 64 x r rows of L1 (8-column core-matrix interleave) and the 64
//   inv_lambda values (bulk copy);
//   quantising thread t handles row t % 128, columns 32 (t / 128) .. + 32 (two
//   NVFP4 groups): codes and scales go to global memory and bf16(Xh) back into
//   the swizzled tile in place, which makes it the K-major A operand;
//   warp 8 then issues four tcgen05 bf16 MMAs (M = 128, N = r, K = 16) adding
//   Xh L1 into an fp32 [128 x r] tensor-memory accumulator and, once they
//   have read the stage, refills it.
// The ks partial T tiles are summed in a fixed order across the cluster
// through distributed shared memory and rounded once to bf16.
constexpr int kQaCompute = 256;
constexpr int kQaThreads = kQaCompute + 32;
constexpr int kQaStages = 4;
constexpr uint32_t kQaXBytes = 16384;

struct QaParams {
  const float* inv_lambda;
  uint8_t* x_codes;
  uint8_t* x_scales;
  __nv_bfloat16* T;
  int M, K, r, cpc, ks;
  uint64_t timeout_ns;
};

__host__ __device__ constexpr uint32_t qa_stage_bytes(int r) {
  return kQaXBytes + static_cast<uint32_t>(r) * 128u + 1024u;  // X | L1 | inv_lambda (padded)
}

__global__ void __launch_bounds__(kQaThreads, 1)
    quantize_act_kernel(const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ CUtensorMap tm_l1, const QaParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int r = p.r;
  const bool has_lr = r > 0;
  const uint32_t l1_bytes = static_cast<uint32_t>(r) * 128u;
  const uint32_t stage_bytes = qa_stage_bytes(r);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kQaStages * stage_bytes);
  uint64_t* full = bars;                    // TMA landed
  uint64_t* quant = bars + kQaStages;       // 8 quantising warps done with the stage
  uint64_t* freed = bars + 2 * kQaStages;   // MMAs done reading the stage
  uint64_t* fin = bars + 3 * kQaStages;     // every MMA of the CTA complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int row0 = blockIdx.y * 128;
  const int rank = blockIdx.x;
  const int nch = p.cpc;
  const int kc0 = rank * nch;
  const int K = p.K;
  const uint32_t tmem_cols = r <= 32 ? 32u : (r <= 64 ? 64u : 128u);

  if (warp == 8 && has_lr) {
    tmem_alloc(smem_u32(tmem_slot), tmem_cols);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < kQaStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&quant[s]), kQaCompute / 32);
      mbar_init(smem_u32(&freed[s]), 1);
    }
    mbar_init(smem_u32(fin), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = has_lr ? *tmem_slot : 0u;
  const uint32_t smem_base = smem_u32(smem);

  if (warp == 8) {
    if (lane == 0) {
      // ------------------------------------------- producer + MMA issuer --
      prefetch_tmap(&tm_x);
      if (has_lr) prefetch_tmap(&tm_l1);
      auto issue = [&](int c) {
        const int s = c % kQaStages;
        const int k = (kc0 + c) * 64;
        const uint32_t fb = smem_u32(&full[s]);
        const uint32_t dst = smem_base + s * stage_bytes;
        mbar_arrive_expect_tx(fb, kQaXBytes + l1_bytes + 256u);
        tma_load_2d(dst, &tm_x, fb, k, row0);
        if (has_lr) tma_load_3d(dst + kQaXBytes, &tm_l1, fb, 0, k, 0);
        bulk_load(dst + kQaXBytes + l1_bytes, p.inv_lambda + k, 256u, fb);
      };
      int issued = 0;
      for (int c = 0; c < nch && c < kQaStages; ++c, ++issued) issue(c);
      // bf16 MMA, M = 128, N = r, A K-major (swizzled X tile), B N-major (L1)
      const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                             (static_cast<uint32_t>(r >> 3) << 17) | (8u << 24);
      for (int c = 0; c < nch; ++c) {
        const int s = c % kQaStages;
        const uint32_t ph = (c / kQaStages) & 1;
        if (*abort_flag) break;
        if (!mbar_wait(smem_u32(&quant[s]), ph, p.timeout_ns, 10)) {
          *abort_flag = 1;
          break;
        }
        if (has_lr) {
          tc_fence_after();
          const uint32_t a0 = smem_base + s * stage_bytes;
          const uint32_t b0 = a0 + kQaXBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tmem, make_sdesc(a0 + kk * 32, 16, 1024, 2), make_sdesc(b0 + kk * 256, 128, 1024, 0),
                     idesc, (c > 0 || kk > 0) ? 1u : 0u);
          tc_commit(smem_u32(&freed[s]));
        } else {
          mbar_arrive(smem_u32(&freed[s]));
        }
        if (c + kQaStages < nch) {
          if (!mbar_wait(smem_u32(&freed[s]), ph, p.timeout_ns, 11)) {
            *abort_flag = 1;
            break;
          }
          issue(c + kQaStages);
          ++issued;
        }
      }
      if (*abort_flag)  // let this CTA's own copies land before it can exit
        for (int c = issued > kQaStages ? issued - kQaStages : 0; c < issued; ++c)
          mbar_wait(smem_u32(&full[c % kQaStages]), (c / kQaStages) & 1, p.timeout_ns, 14);
      if (has_lr) tc_commit(smem_u32(fin));
    }
  } else {
    // ------------------------------------------------------- quantisers --
    const int rr = tid & 127;  // row inside the tile
    const int h = tid >> 7;    // which 32-column half of the chunk
    const int m = row0 + rr;
    const int sw = rr & 7;     // 128-byte swizzle phase of the row
    for (int c = 0; c < nch; ++c) {
      const int s = c % kQaStages;
      const uint32_t ph = (c / kQaStages) & 1;
      bool ok = !*abort_flag;
      if (ok) ok = mbar_wait(smem_u32(&full[s]), ph, p.timeout_ns, 12);
      if (!ok) {
        *abort_flag = 1;
        break;
      }
      const int k = (kc0 + c) * 64;
      uint8_t* stage = smem + s * stage_bytes;
      uint8_t* row = stage + rr * 128;
      const float4* il = reinterpret_cast<const float4*>(stage + kQaXBytes + l1_bytes) + 8 * h;
      uint32_t cw[4];
      uint32_t swd = 0;
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        const int j0 = 4 * h + 2 * g;  // logical 16-byte chunk of the row
        uint4 w0 = *reinterpret_cast<const uint4*>(row + ((j0 ^ sw) << 4));
        uint4 w1 = *reinterpret_cast<const uint4*>(row + (((j0 + 1) ^ sw) << 4));
        const float4 l0 = il[4 * g + 0], l1 = il[4 * g + 1], l2 = il[4 * g + 2], l3 = il[4 * g + 3];
        float v[16];
        v[0] = __fmul_rn(bf16_lo(w0.x), l0.x);  v[1] = __fmul_rn(bf16_hi(w0.x), l0.y);
        v[2] = __fmul_rn(bf16_lo(w0.y), l0.z);  v[3] = __fmul_rn(bf16_hi(w0.y), l0.w);
        v[4] = __fmul_rn(bf16_lo(w0.z), l1.x);  v[5] = __fmul_rn(bf16_hi(w0.z), l1.y);
        v[6] = __fmul_rn(bf16_lo(w0.w), l1.z);  v[7] = __fmul_rn(bf16_hi(w0.w), l1.w);
        v[8] = __fmul_rn(bf16_lo(w1.x), l2.x);  v[9] = __fmul_rn(bf16_hi(w1.x), l2.y);
        v[10] = __fmul_rn(bf16_lo(w1.y), l2.z); v[11] = __fmul_rn(bf16_hi(w1.y), l2.w);
        v[12] = __fmul_rn(bf16_lo(w1.z), l3.x); v[13] = __fmul_rn(bf16_hi(w1.z), l3.y);
        v[14] = __fmul_rn(bf16_lo(w1.w), l3.z); v[15] = __fmul_rn(bf16_hi(w1.w), l3.w);
        swd |= nvfp4_group(v, cw[2 * g], cw[2 * g + 1]) << (8 * g);
        if (has_lr) {
          w0 = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                          pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
          w1 = make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]),
                          pack_bf16x2(v[12], v[13]), pack_bf16x2(v[14], v[15]));
          *reinterpret_cast<uint4*>(row + ((j0 ^ sw) << 4)) = w0;
          *reinterpret_cast<uint4*>(row + (((j0 + 1) ^ sw) << 4)) = w1;
        }
      }
      if (m < p.M)
        *reinterpret_cast<uint4*>(p.x_codes + static_cast<size_t>(m) * (K >> 1) + (k >> 1) + 16 * h) =
            make_uint4(cw[0], cw[1], cw[2], cw[3]);
      *reinterpret_cast<uint16_t*>(p.x_scales + scale_word_offset(m, k >> 4, K) + 2 * h) =
          static_cast<uint16_t>(swd);
      if (has_lr) fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&quant[s]));
    }
  }

  if (has_lr) {
    // every MMA of this CTA (also after an abort) completes before the
    // accumulator is read or the tensor memory released
    const bool ok = mbar_wait(smem_u32(fin), 0, p.timeout_ns, 13);
    if (!ok) *abort_flag = 1;
    __syncthreads();
    tc_fence_after();
    const bool good = !*abort_flag;
    float* part = reinterpret_cast<float*>(smem);  // ring is idle: reuse it
    if (warp < 4 && good) {
      const int m = row0 + tid;
      const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
      for (int c0 = 0; c0 < r; c0 += 16) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(tmem + lane_base + c0, v);
        tmem_ld_wait();
        if (p.ks == 1) {
          if (m < p.M) {
            uint4* dst = reinterpret_cast<uint4*>(p.T + static_cast<size_t>(m) * r + c0);
#pragma unroll
            for (int j = 0; j < 2; ++j)
              dst[j] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * j]), __uint_as_float(v[8 * j + 1])),
                                  pack_bf16x2(__uint_as_float(v[8 * j + 2]), __uint_as_float(v[8 * j + 3])),
                                  pack_bf16x2(__uint_as_float(v[8 * j + 4]), __uint_as_float(v[8 * j + 5])),
                                  pack_bf16x2(__uint_as_float(v[8 * j + 6]), __uint_as_float(v[8 * j + 7])));
          }
        } else {
#pragma unroll
          for (int j = 0; j < 16; j += 4)
            *reinterpret_cast<uint4*>(part + tid * r + c0 + j) = make_uint4(v[j], v[j + 1], v[j + 2], v[j + 3]);
        }
      }
    }
    if (p.ks > 1) {
      cluster_sync();
      const int rows_per = 128 / p.ks;
      const int q4 = r >> 2;
      const uint32_t part_s = smem_u32(part);
      for (int it = tid; it < rows_per * q4; it += kQaThreads) {
        const int rr = rank * rows_per + it / q4;
        const int j = (it % q4) * 4;
        float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int src = 0; src < p.ks; ++src) {
          const float4 v = ld_shared_cluster_f4(map_shared_rank(part_s + (rr * r + j) * 4, src));
          sum.x += v.x; sum.y += v.y; sum.z += v.z; sum.w += v.w;
        }
        const int mm = row0 + rr;
        if (good && mm < p.M)
          *reinterpret_cast<uint2*>(p.T + static_cast<size_t>(mm) * r + j) =
              make_uint2(pack_bf16x2(sum.x, sum.y), pack_bf16x2(sum.z, sum.w));
      }
      cluster_sync();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8 && has_lr) tmem_dealloc(tmem, tmem_cols);
}

// ================================================== fused 4-bit linear ====
// Persistent: grid = min(tiles, SMs), 192 threads:
//   warp 0: TMA producer, warp 1: TMEM owner + MMA issuer, warps 2-5: epilogue.
// Output tiles are 128 x 256, visited M-fastest (tile t -> m = t % Mt,
// n = t / Mt), CTA b takes tiles b, b + grid, ...  A 4-stage shared-memory
// ring feeds, for each tile in order:
//   ceil(r/64) low-rank stages: T [128 x 64] (K-major, 128-byte swizzle) in
//     the A slot and L2 [64 x 256] (N-major, 128-byte swizzle) in the B slot,
//     consumed by r/16 bf16 MMAs (the first one initialises the accumulator);
//   ceil(K/256) FP4 stages: x codes [128 x 128 B], R codes [256 x 128 B]
//     (K-major, 128-byte swizzle) and their scale tiles, consumed by four
//     block-scaled MMAs (K = 64 each) after tcgen05.cp moves the scales
//     into tensor memory.
// Two 128 x 256 fp32 accumulators overlap in TMEM: tile i uses columns
// [0, 256) if i is even, [192, 448) if odd; scale factors sit in [448, 496).
// The epilogue drains the 64 shared columns first and releases them, so the
// MMAs of tile i + 1 start while the epilogue of tile i is still running.
constexpr int kLinThreads = 192;
constexpr int kLinStages = 4;
constexpr int kLinBM = 128, kLinBN = 256, kLinBK = 256;
constexpr uint32_t kLinABytes = 16384, kLinBBytes = 32768, kLinSfaBytes = 2048, kLinSfbBytes = 4096;
constexpr uint32_t kLinStageBytes = kLinABytes + kLinBBytes + kLinSfaBytes + kLinSfbBytes;
constexpr uint32_t kLinTmemCols = 512;
constexpr uint32_t kLinAcc1Col = 192, kLinSfaCol = 448, kLinSfbCol = 464;
constexpr uint32_t kLinBarOffset = kLinStages * kLinStageBytes + 1024;  // after the bias buffer

struct LinParams {
  const uint8_t* x_scales;
  const uint8_t* r_scales;
  const __nv_bfloat16* bias;
  __nv_bfloat16* Y;
  int M, K, N, r;
  int m_tiles, tiles;
  uint64_t timeout_ns;
};

__global__ void __launch_bounds__(kLinThreads, 1)
    linear_kernel(const __grid_constant__ CUtensorMap tm_xc, const __grid_constant__ CUtensorMap tm_rc,
                  const __grid_constant__ CUtensorMap tm_t, const __grid_constant__ CUtensorMap tm_l2,
                  const LinParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  float* bias_s = reinterpret_cast<float*>(smem + kLinStages * kLinStageBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kLinBarOffset);
  uint64_t* full = bars;                        // [4] TMA landed
  uint64_t* empty = bars + kLinStages;          // [4] MMAs done reading the stage
  uint64_t* acc_full = bars + 2 * kLinStages;   // [2] tile accumulated
  uint64_t* acc_empty = acc_full + 2;           // [2] epilogue drained the accumulator
  uint64_t* ovl_free = acc_full + 4;            // epilogue drained the shared columns
  uint64_t* fin = acc_full + 5;                 // every MMA of the CTA complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 6);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int K = p.K, N = p.N, r = p.r;
  const int n_lr = (r + 63) / 64;
  const int n_k = (K + kLinBK - 1) / kLinBK;
  const int total = n_lr + n_k;
  const int n_pad = (N + 127) & ~127;

  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kLinTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < kLinStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&acc_full[b]), 1);
      mbar_init(smem_u32(&acc_empty[b]), 4);
    }
    mbar_init(smem_u32(ovl_free), 4);
    mbar_init(smem_u32(fin), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sbase = smem_u32(smem);

  if (warp == 0) {
    if (lane == 0) {
      // ----------------------------------------------------- producer --
      prefetch_tmap(&tm_xc);
      prefetch_tmap(&tm_rc);
      if (r > 0) {
        prefetch_tmap(&tm_t);
        prefetch_tmap(&tm_l2);
      }
      const size_t tiles_k = static_cast<size_t>(K >> 6);
      uint32_t g = 0;
      for (int t = blockIdx.x; t < p.tiles && !*abort_flag; t += gridDim.x) {
        const int m0 = (t % p.m_tiles) * kLinBM;
        const int n0 = (t / p.m_tiles) * kLinBN;
        const int n_atoms = (n0 + 128 < n_pad) ? 2 : 1;
        for (int it = 0; it < total; ++it, ++g) {
          const int s = g % kLinStages;
          const uint32_t ph = (g / kLinStages) & 1;
          if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1, p.timeout_ns, 20)) {
            *abort_flag = 1;
            break;
          }
          const uint32_t fb = smem_u32(&full[s]);
          const uint32_t a_s = sbase + s * kLinStageBytes;
          const uint32_t b_s = a_s + kLinABytes;
          if (it < n_lr) {
            const int j0 = it * 64;
            mbar_arrive_expect_tx(fb, kLinABytes + kLinBBytes);
            tma_load_2d(a_s, &tm_t, fb, j0, m0);
#pragma unroll
            for (int q = 0; q < 4; ++q) tma_load_2d(b_s + q * 8192, &tm_l2, fb, n0 + 64 * q, j0);
          } else {
            const int k0 = (it - n_lr) * kLinBK;
            const int nkb = min(4, (K - k0) / 64);
            const uint32_t sfa_s = b_s + kLinBBytes;
            const uint32_t sfb_s = sfa_s + kLinSfaBytes;
            const uint32_t sf_bytes = static_cast<uint32_t>(nkb) * 512u;
            mbar_arrive_expect_tx(fb, kLinABytes + kLinBBytes + sf_bytes * (1 + n_atoms));
            tma_load_2d(a_s, &tm_xc, fb, k0 >> 1, m0);
            tma_load_2d(b_s, &tm_rc, fb, k0 >> 1, n0);
            const size_t kt = static_cast<size_t>(k0 >> 6);
            bulk_load(sfa_s, p.x_scales + ((m0 >> 7) * tiles_k + kt) * 512, sf_bytes, fb);
            for (int a = 0; a < n_atoms; ++a)
              bulk_load(sfb_s + a * 2048, p.r_scales + (((n0 >> 7) + a) * tiles_k + kt) * 512, sf_bytes, fb);
          }
        }
      }
      if (*abort_flag)  // let this CTA's own copies land before it can exit
        for (uint32_t j = g > kLinStages ? g - kLinStages : 0; j < g; ++j)
          mbar_wait(smem_u32(&full[j % kLinStages]), (j / kLinStages) & 1, p.timeout_ns, 26);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // -------------------------------------------------- MMA issuer --
      const uint32_t idesc_f4 = (1u << 7) | (1u << 10) | ((kLinBN >> 3) << 17) | ((kLinBM >> 4) << 24);
      const uint32_t idesc_bf = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                ((kLinBN >> 3) << 17) | ((kLinBM >> 4) << 24);
      const uint32_t sfa_t = tmem + kLinSfaCol;
      const uint32_t sfb_t = tmem + kLinSfbCol;
      uint32_t g = 0;
      int i = 0;
      for (int t = blockIdx.x; t < p.tiles && !*abort_flag; t += gridDim.x, ++i) {
        const int b = i & 1;
        const uint32_t acc = tmem + (b ? kLinAcc1Col : 0u);
        const int n0 = (t / p.m_tiles) * kLinBN;
        const int n_atoms = (n0 + 128 < n_pad) ? 2 : 1;
        if (i >= 2 && !mbar_wait(smem_u32(&acc_empty[b]), ((i >> 1) - 1) & 1, p.timeout_ns, 21)) {
          *abort_flag = 1;
          break;
        }
        if (i >= 1 && !mbar_wait(smem_u32(ovl_free), (i - 1) & 1, p.timeout_ns, 22)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        for (int it = 0; it < total; ++it, ++g) {
          const int s = g % kLinStages;
          const uint32_t ph = (g / kLinStages) & 1;
          if (!mbar_wait(smem_u32(&full[s]), ph, p.timeout_ns, 23)) {
            *abort_flag = 1;
            break;
          }
          tc_fence_after();
          const uint32_t a_s = sbase + s * kLinStageBytes;
          const uint32_t b_s = a_s + kLinABytes;
          if (it < n_lr) {
            const int nk16 = min(4, (r - it * 64) / 16);
            for (int kk = 0; kk < nk16; ++kk)
              mma_bf16(acc, make_sdesc(a_s + kk * 32, 16, 1024, 2), make_sdesc(b_s + kk * 2048, 8192, 1024, 2),
                       idesc_bf, (it > 0 || kk > 0) ? 1u : 0u);
          } else {
            const int k0 = (it - n_lr) * kLinBK;
            const int nkb = min(4, (K - k0) / 64);
            const uint32_t sfa_s = b_s + kLinBBytes;
            const uint32_t sfb_s = sfa_s + kLinSfaBytes;
            for (int kb = 0; kb < nkb; ++kb) {
              tmem_cp_32x128b_warpx4(sfa_t + 4 * kb, make_sdesc(sfa_s + kb * 512, 0, 128, 0));
              tmem_cp_32x128b_warpx4(sfb_t + 8 * kb, make_sdesc(sfb_s + kb * 512, 0, 128, 0));
              if (n_atoms == 2)
                tmem_cp_32x128b_warpx4(sfb_t + 8 * kb + 4, make_sdesc(sfb_s + 2048 + kb * 512, 0, 128, 0));
            }
            for (int kb = 0; kb < nkb; ++kb)
              mma_nvf4(acc, make_sdesc(a_s + kb * 32, 16, 1024, 2), make_sdesc(b_s + kb * 32, 16, 1024, 2),
                       idesc_f4, sfa_t + 4 * kb, sfb_t + 8 * kb, (it > 0 || kb > 0) ? 1u : 0u);
          }
          tc_commit(smem_u32(&empty[s]));
        }
        tc_commit(smem_u32(&acc_full[b]));
      }
      // own MMAs complete before the tensor memory can be released
      tc_commit(smem_u32(fin));
      if (!mbar_wait(smem_u32(fin), 0, p.timeout_ns, 24)) *abort_flag = 1;
    }
  } else {
    // ------------------------------------------------------- epilogue --
    const int et = tid - 64;   // 0..127
    const int q = warp & 3;    // TMEM lane quadrant this warp may access
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    int i = 0;
    for (int t = blockIdx.x; t < p.tiles; t += gridDim.x, ++i) {
      const int b = i & 1;
      const int m0 = (t % p.m_tiles) * kLinBM;
      const int n0 = (t / p.m_tiles) * kLinBN;
      const int row = m0 + q * 32 + lane;
      named_bar_sync(1, 128);  // everyone is done with the previous tile's bias
      for (int j = et; j < kLinBN; j += 128) {
        const int n = n0 + j;
        bias_s[j] = (p.bias && n < N) ? __bfloat162float(p.bias[n]) : 0.0f;
      }
      named_bar_sync(1, 128);
      // no early exit: all four warps must keep meeting the named barriers
      const bool ok = !*abort_flag && mbar_wait(smem_u32(&acc_full[b]), (i >> 1) & 1, p.timeout_ns, 25);
      if (!ok) {
        *abort_flag = 1;
        continue;
      }
      tc_fence_after();
      const uint32_t acc_col = b ? kLinAcc1Col : 0u;
      for (int ci = 0; ci < 4; ++ci) {
        const int c = b ? ci : ((ci + 3) & 3);  // shared columns first
        uint32_t v[64];
        tmem_ld_32x32b_x32(tmem + lane_base + acc_col + 64 * c, v);
        tmem_ld_32x32b_x32(tmem + lane_base + acc_col + 64 * c + 32, v + 32);
        tmem_ld_wait();
        if (ci == 0) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(ovl_free));
        }
        const int nb = n0 + 64 * c;
        if (row < p.M) {
          __nv_bfloat16* yrow = p.Y + static_cast<size_t>(row) * N;
#pragma unroll
          for (int j = 0; j < 64; j += 16) {
            if (nb + j < N) {
              const float* bs = bias_s + 64 * c + j;
              uint4* dst = reinterpret_cast<uint4*>(yrow + nb + j);
              dst[0] = make_uint4(pack_bf16x2(__uint_as_float(v[j + 0]) + bs[0], __uint_as_float(v[j + 1]) + bs[1]),
                                  pack_bf16x2(__uint_as_float(v[j + 2]) + bs[2], __uint_as_float(v[j + 3]) + bs[3]),
                                  pack_bf16x2(__uint_as_float(v[j + 4]) + bs[4], __uint_as_float(v[j + 5]) + bs[5]),
                                  pack_bf16x2(__uint_as_float(v[j + 6]) + bs[6], __uint_as_float(v[j + 7]) + bs[7]));
              dst[1] = make_uint4(pack_bf16x2(__uint_as_float(v[j + 8]) + bs[8], __uint_as_float(v[j + 9]) + bs[9]),
                                  pack_bf16x2(__uint_as_float(v[j + 10]) + bs[10], __uint_as_float(v[j + 11]) + bs[11]),
                                  pack_bf16x2(__uint_as_float(v[j + 12]) + bs[12], __uint_as_float(v[j + 13]) + bs[13]),
                                  pack_bf16x2(__uint_as_float(v[j + 14]) + bs[14], __uint_as_float(v[j + 15]) + bs[15]));
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&acc_empty[b]));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, kLinTmemCols);
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
