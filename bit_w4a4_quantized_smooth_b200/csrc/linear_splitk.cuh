// Fused 4-bit linear of the SVDQuant W4A4 layer for sm_100a, small-M path:
// Y = deq(x) deq(R)^T + T L2 + bias for inputs with few rows (a handful of
// tokens), where the large-M kernel's 256 x 256 tiles would leave most SMs
// idle and walk all of K in series on the few that work.
//
// A CTA computes one 128 x 128 output tile over a contiguous range of the
// 256-column K stages; the `splits` CTAs of a tile form a cluster along K.
// Single-CTA tcgen05 MMAs (M = 128, N = 128): block-scaled FP4 with K = 64
// per MMA, and in the cluster's first CTA the rank-r bf16 up-projection
// T L2 into the same fp32 accumulator (ai-digest.ru abstract: the low-rank
// branch is fused into the 4-bit kernel).  192 threads: warp 0 TMA producer,
// warp 1 tensor-memory owner and MMA issuer, warps 2-5 epilogue (warp w reads
// tensor-memory lanes [32 (w % 4), +32), one output row per thread).
// The partial accumulators meet in distributed shared memory: CTA j adds the
// rows [j 128 / splits, (j + 1) 128 / splits) (of those below M) of every
// CTA's partial in rank order, adds the bias, rounds once to bf16 and stores
// Y.  No global scratch memory, and the sum's order is fixed.
#pragma once

#include "common.cuh"

namespace svdq {

constexpr int kLsThreads = 192;
constexpr int kLsBM = 128, kLsBN = 128, kLsBK = 256;
constexpr uint32_t kLsABytes = 16384, kLsBBytes = 16384, kLsSfaBytes = 2048, kLsSfbBytes = 2048;
constexpr uint32_t kLsStageBytes = kLsABytes + kLsBBytes + kLsSfaBytes + kLsSfbBytes;  // 36 KB
constexpr int kLsMaxStages = 6;
constexpr int kLsMaxSplits = 8;
constexpr uint32_t kLsHeadBytes = 1024;
constexpr uint32_t kLsTmemCols = 256;       // accumulator [0, 128), scale factors [128, 160)
constexpr uint32_t kLsSfaCol = 128, kLsSfbCol = 144;
constexpr int kLsPitch = kLsBN + 4;         // floats per row of a partial (16-byte skew)
constexpr uint32_t kLsPartBytes = kLsBM * kLsPitch * 4;

struct LsParams {
  const __nv_bfloat16* bias;
  __nv_bfloat16* Y;
  float alpha;  // a power of two: the 4-bit product's global scales g_x g_w (1 without them)
  int M, K, N, r;
  int splits;   // CTAs per output tile (cluster size along K)
  int spc;      // FP4 stages (256 columns of K) per CTA
  int stages;   // ring depth
  uint64_t timeout_ns;
};

__global__ void __launch_bounds__(kLsThreads, 1)
    linear_splitk_kernel(const __grid_constant__ CUtensorMap tm_xc, const __grid_constant__ CUtensorMap tm_rc,
                         const __grid_constant__ CUtensorMap tm_xs, const __grid_constant__ CUtensorMap tm_rs,
                         const __grid_constant__ CUtensorMap tm_t, const __grid_constant__ CUtensorMap tm_l2,
                         const LsParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  const int S = p.stages;
  // [0, 1024): barriers and flags; the ring follows
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);  // [S] stage landed
  uint64_t* empty = full + S;                          // [S] the stage's MMAs and copies are done
  uint64_t* fin = empty + S;                           // every MMA of the CTA complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint8_t* ring = smem + kLsHeadBytes;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int split = blockIdx.x;
  const int n0 = blockIdx.y * kLsBN;
  const int m0 = blockIdx.z * kLsBM;
  const int K = p.K, r = p.r;
  const int n_k = (K + kLsBK - 1) / kLsBK;
  const int kt0 = split * p.spc;
  const int nk = min(p.spc, n_k - kt0);                // FP4 stages of this CTA (>= 1)
  const int n_lr = (split == 0 && r > 0) ? (r + 63) / 64 : 0;
  const int total = n_lr + nk;
  const int tiles_k = K >> 6;

  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kLsTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(fin), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // The next layer's activation step may now be scheduled (after the tensor
  // memory is held, so that no later CTA can hold it while waiting for us).
  griddep_launch_dependents();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sbase = smem_u32(ring);

  if (warp == 0) {
    // ---------------------------------------------------------- producer --
    if (lane == 0) {
      prefetch_tmap(&tm_xc);
      prefetch_tmap(&tm_rc);
      prefetch_tmap(&tm_xs);
      prefetch_tmap(&tm_rs);
      if (n_lr) {
        prefetch_tmap(&tm_t);
        prefetch_tmap(&tm_l2);
      }
    }
    __syncwarp();
    // While the activation step ahead finishes: the weight halves (L2, R
    // codes and scales) of the stages the ring loads first into L2.
    for (int it = 0; it < min(total, S); ++it) {
      if (it < n_lr) {
        e_tma_prefetch_2d(&tm_l2, n0, it * 64);
        e_tma_prefetch_2d(&tm_l2, n0 + 64, it * 64);
      } else {
        const int ks = kt0 + it - n_lr;
        e_tma_prefetch_2d(&tm_rc, ks * 128, n0);
        e_tma_prefetch_3d(&tm_rs, 0, 0, (n0 >> 7) * tiles_k + 4 * ks);
      }
    }
    griddep_wait();
    int issued = 0;
    for (int it = 0; it < total; ++it) {
      const int s = it % S;
      if (it >= S && !warp_wait(smem_u32(&empty[s]), ((it / S) - 1) & 1, p.timeout_ns, 50)) {
        *abort_flag = 1;
        break;
      }
      if (warp_flag(abort_flag)) break;
      const uint32_t fb = smem_u32(&full[s]);
      const uint32_t a_s = sbase + s * kLsStageBytes;
      const uint32_t b_s = a_s + kLsABytes;
      if (it < n_lr) {
        e_arrive_expect_tx(fb, kLsABytes + kLsBBytes);
        const int j0 = it * 64;
        e_tma_load_2d(a_s, &tm_t, fb, j0, m0);
        e_tma_load_2d(b_s, &tm_l2, fb, n0, j0);
        e_tma_load_2d(b_s + 8192, &tm_l2, fb, n0 + 64, j0);
      } else {
        e_arrive_expect_tx(fb, kLsStageBytes);
        const int ks = kt0 + it - n_lr;  // global K stage
        const uint32_t sfa_s = b_s + kLsBBytes;
        const uint32_t sfb_s = sfa_s + kLsSfaBytes;
        e_tma_load_2d(a_s, &tm_xc, fb, ks * 128, m0);
        e_tma_load_2d(b_s, &tm_rc, fb, ks * 128, n0);
        // scale tiles: [512-byte tile][4 K blocks]; boxes past the end of a
        // band (or of the tensor) read zeros and are never used
        e_tma_load_3d(sfa_s, &tm_xs, fb, 0, 0, (m0 >> 7) * tiles_k + 4 * ks);
        e_tma_load_3d(sfb_s, &tm_rs, fb, 0, 0, (n0 >> 7) * tiles_k + 4 * ks);
      }
      ++issued;
    }
    // after an abort: this CTA's own copies land before it may exit
    if (warp_flag(abort_flag))
      for (int c = issued > S ? issued - S : 0; c < issued; ++c)
        warp_wait(smem_u32(&full[c % S]), (c / S) & 1, p.timeout_ns, 51);
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer --
    griddep_wait();  // bounded waits start once the kernel ahead is done
    const uint32_t idesc_f4 = (1u << 7) | (1u << 10) | ((kLsBN >> 3) << 17) | ((kLsBM >> 4) << 24);
    const uint32_t idesc_bf =
        (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((kLsBN >> 3) << 17) | ((kLsBM >> 4) << 24);
    const uint32_t sfa_t = tmem + kLsSfaCol;
    const uint32_t sfb_t = tmem + kLsSfbCol;
    bool first = true;
    for (int it = 0; it < total; ++it) {
      const int s = it % S;
      const bool ok = !warp_flag(abort_flag) && warp_wait(smem_u32(&full[s]), (it / S) & 1, p.timeout_ns, 52);
      if (!ok) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t a_s = sbase + s * kLsStageBytes;
      const uint32_t b_s = a_s + kLsABytes;
      if (it < n_lr) {
        const int nk16 = min(4, (r - it * 64) / 16);
        for (int kk = 0; kk < nk16; ++kk) {
          e_mma_bf16(tmem, make_sdesc(a_s + kk * 32, 16, 1024, 2), make_sdesc(b_s + kk * 2048, 8192, 1024, 2),
                     idesc_bf, first ? 0u : 1u);
          first = false;
        }
      } else {
        const uint32_t sfa_s = b_s + kLsBBytes;
        const uint32_t sfb_s = sfa_s + kLsSfaBytes;
        const int k0 = (kt0 + it - n_lr) * kLsBK;
        const int nkb = min(4, (K - k0) / 64);
        for (int kb = 0; kb < nkb; ++kb) {
          e_tmem_cp_32x128b_warpx4(sfa_t + 4 * kb, make_sdesc(sfa_s + kb * 512, 0, 128, 0));
          e_tmem_cp_32x128b_warpx4(sfb_t + 4 * kb, make_sdesc(sfb_s + kb * 512, 0, 128, 0));
          e_mma_nvf4(tmem, make_sdesc(a_s + kb * 32, 16, 1024, 2), make_sdesc(b_s + kb * 32, 16, 1024, 2), idesc_f4,
                     sfa_t + 4 * kb, sfb_t + 4 * kb, first ? 0u : 1u);
          first = false;
        }
      }
      e_commit(smem_u32(&empty[s]));
    }
    // every MMA (also after an abort) completes before the accumulator is
    // read or the tensor memory released
    e_commit(smem_u32(fin));
    if (!warp_wait(smem_u32(fin), 0, p.timeout_ns, 53)) *abort_flag = 1;
  }

  // --------------------------------------------------------- epilogue --
  griddep_wait();   // the bias and Y may belong to the kernel ahead
  __syncthreads();  // every role is done: the ring is idle, the MMAs complete
  const bool aborted = *abort_flag != 0;
  float* part = reinterpret_cast<float*>(ring);  // [128][kLsPitch], over the idle ring
  const int vrows = min(kLsBM, p.M - m0);        // tile rows below M
  if (warp >= 2 && !aborted && warp_wait(smem_u32(fin), 0, p.timeout_ns, 54)) {
    tc_fence_after();
    const int q = warp & 3;
    const int rr = 32 * q + lane;
    const int m = m0 + rr;
    const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
    for (int cb = 0; cb < kLsBN; cb += 32) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(tmem + lane_base + cb, v);
      tmem_ld_wait();
      if (p.splits == 1) {
        if (rr < vrows) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {  // 8 columns per 16-byte store; N % 16 == 0
            const int n = n0 + cb + 8 * j;
            if (n < p.N) {
              float b[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) b[e] = p.bias ? __bfloat162float(p.bias[n + e]) : 0.0f;
              // alpha is a power of two: acc alpha is exact
              auto y = [&](int e) { return __fmul_rn(__uint_as_float(v[8 * j + e]), p.alpha) + b[e]; };
              *reinterpret_cast<uint4*>(p.Y + static_cast<size_t>(m) * p.N + n) =
                  make_uint4(pack_bf16x2(y(0), y(1)), pack_bf16x2(y(2), y(3)), pack_bf16x2(y(4), y(5)),
                             pack_bf16x2(y(6), y(7)));
            }
          }
        }
      } else if (rr < vrows) {
        float4* dst = reinterpret_cast<float4*>(part + rr * kLsPitch + cb);
#pragma unroll
        for (int e = 0; e < 8; ++e)
          dst[e] = make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]), __uint_as_float(v[4 * e + 2]),
                               __uint_as_float(v[4 * e + 3]));
      }
    }
  }
  if (p.splits > 1) {
    cluster_sync();  // every CTA's partial is in its shared memory
    const int per = (vrows + p.splits - 1) / p.splits;
    const int lo_row = split * per;
    const int hi_row = min(vrows, lo_row + per);
    const uint32_t part_u = smem_u32(part);
    constexpr int n4 = kLsBN / 4;
    for (int e = tid; e < (hi_row > lo_row ? (hi_row - lo_row) * n4 : 0); e += kLsThreads) {
      const int row = lo_row + e / n4;
      const int c4 = e % n4;
      const int n = n0 + 4 * c4;
      if (n >= p.N) continue;
      const uint32_t off = part_u + static_cast<uint32_t>((row * kLsPitch + 4 * c4) * 4);
      float4 acc = ld_dsmem_f32x4(map_shared_rank(off, 0));
      for (int src = 1; src < p.splits; ++src) {  // rank order
        const float4 b = ld_dsmem_f32x4(map_shared_rank(off, static_cast<uint32_t>(src)));
        acc.x = __fadd_rn(acc.x, b.x);
        acc.y = __fadd_rn(acc.y, b.y);
        acc.z = __fadd_rn(acc.z, b.z);
        acc.w = __fadd_rn(acc.w, b.w);
      }
      acc.x = __fmul_rn(acc.x, p.alpha);
      acc.y = __fmul_rn(acc.y, p.alpha);
      acc.z = __fmul_rn(acc.z, p.alpha);
      acc.w = __fmul_rn(acc.w, p.alpha);
      if (p.bias) {
        acc.x = __fadd_rn(acc.x, __bfloat162float(p.bias[n]));
        acc.y = __fadd_rn(acc.y, __bfloat162float(p.bias[n + 1]));
        acc.z = __fadd_rn(acc.z, __bfloat162float(p.bias[n + 2]));
        acc.w = __fadd_rn(acc.w, __bfloat162float(p.bias[n + 3]));
      }
      if (!aborted)
        *reinterpret_cast<uint2*>(p.Y + static_cast<size_t>(m0 + row) * p.N + n) =
            make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
    }
    cluster_sync();  // no CTA leaves while another still reads its partial
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, kLsTmemCols);
}

}  // namespace svdq
