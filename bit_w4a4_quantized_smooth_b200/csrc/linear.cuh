// Fused 4-bit linear of the SVDQuant W4A4 layer for sm_100a, large-M path:
// block-scaled FP4 MMAs and the rank-r bf16 up-projection accumulate into one
// fp32 tensor-memory tile on CTA pairs (ai-digest.ru abstract: the low-rank
// branch is fused into the 4-bit kernel so it adds no activation traffic).
#pragma once

#include "common.cuh"

namespace svdq {

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
constexpr int kLinNumBars = 2 * kLinStages + 2 + 2 + 1 + 1 + 1;

struct LinParams {
  const __nv_bfloat16* bias;
  __nv_bfloat16* Y;
  float alpha;  // a power of two: the 4-bit product's global scales g_x g_w (1 without them)
  int M, K, N, r;
  int m_tiles, tiles;  // pair tiles: ceil(M / 256) x ceil(N / 256)
  uint64_t timeout_ns;
};

// FULL_K: K is a multiple of 256, every FP4 stage has four K blocks and
// runs a straight-line issue sequence.
template <bool FULL_K>
__global__ void __launch_bounds__(kLinThreads, 1)
    linear_kernel(const __grid_constant__ CUtensorMap tm_xc, const __grid_constant__ CUtensorMap tm_rc,
                  const __grid_constant__ CUtensorMap tm_xs, const __grid_constant__ CUtensorMap tm_rs,
                  const __grid_constant__ CUtensorMap tm_t, const __grid_constant__ CUtensorMap tm_l2,
                  const __grid_constant__ CUtensorMap tm_y, const LinParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  float* bias_s = reinterpret_cast<float*>(smem + kLinStages * kLinStageBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kLinBarOffset);
  uint64_t* full = bars;                           // [S] even CTA: both CTAs' stage landed
  uint64_t* empty = full + kLinStages;             // [S] the stage's MMAs and copies are done
  uint64_t* acc_full = empty + kLinStages;         // [2] tile accumulated (both CTAs)
  uint64_t* acc_empty = acc_full + 2;              // [2] even CTA: 8 epilogue warps drained it
  uint64_t* ovl_free = acc_empty + 2;              // even CTA: shared columns drained
  uint64_t* fin = ovl_free + 1;                    // even CTA: every MMA complete
  uint64_t* odd_done = fin + 1;                    // even CTA: the odd producer published its count
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kLinNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile uint32_t* odd_issued = tmem_slot + 2;   // even CTA: stages the odd producer issued

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
    mbar_init(smem_u32(odd_done), 1);
    *odd_issued = 0;
    *abort_flag = 0;
    fence_barrier_init();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the even CTA's barriers exist before anyone signals them
  tc_fence_after();
  // The next layer's activation step may now be scheduled (after the tensor
  // memory is held, so that no later CTA can hold it while waiting for us).
  griddep_launch_dependents();
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
    // While the activation step ahead finishes: the weight halves (L2, R
    // codes and scales) of the stages the ring loads first into L2 (measured
    // on B200, same box: the linear alone 96.2-96.5 us with these five
    // stages, 96.5-97.2 us with sixteen, 98.3-98.4 us without).
    if (pair < p.tiles) {
      const int n0 = (pair / p.m_tiles) * kLinBN;
      const int nb = n0 + 128 * static_cast<int>(rank);
      for (int it = 0; it < min(total, kLinStages); ++it) {
        if (it < n_lr) {
          e_tma_prefetch_2d(&tm_l2, nb, it * 64);
          e_tma_prefetch_2d(&tm_l2, nb + 64, it * 64);
        } else {
          const int kt = (it - n_lr) * (kLinBK / 64);
          e_tma_prefetch_2d(&tm_rc, kt * 32, nb);
          e_tma_prefetch_3d(&tm_rs, 0, 0, (n0 >> 7) * tiles_k + kt);
          e_tma_prefetch_3d(&tm_rs, 0, 0, ((n0 >> 7) + 1) * tiles_k + kt);
        }
      }
    }
    griddep_wait();
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
    // Both producers' copies complete on the even CTA's full[] barriers, which
    // only the even producer arms.  The odd producer publishes how many
    // stages it issued; after an abort the even producer walks the last
    // stages either CTA issued and makes each phase completable before it
    // waits for it: a stage only the odd CTA issued is armed for the odd
    // CTA's bytes, a stage only the even CTA issued has the odd CTA's share
    // retired.  Every copy into either CTA has landed before the pair passes
    // its final cluster barrier.  (The two counts differ by at most the ring
    // depth: a producer issues stage j only after stage j - S was consumed,
    // which needed both CTAs' copies of it.)
    if (rank == 1) {
      if (lane == 0) {
        st_dsmem_u32(map_shared_rank(smem_u32(const_cast<uint32_t*>(odd_issued)), 0), g);
        mbar_arrive_cluster(lead(odd_done));
      }
      __syncwarp();
    } else if (warp_flag(abort_flag)) {
      const bool have = warp_wait_cluster(smem_u32(odd_done), 0, 2 * p.timeout_ns + 100000000ull, 27);
      const uint32_t g_odd = have ? __shfl_sync(0xffffffffu, *odd_issued, 0) : g;
      const uint32_t hi = g > g_odd ? g : g_odd;
      for (uint32_t j = hi > kLinStages ? hi - kLinStages : 0; j < hi; ++j) {
        const uint32_t s = j % kLinStages;
        const int it = static_cast<int>(j % static_cast<uint32_t>(total));
        const uint32_t per_cta = it < n_lr ? kLinABytes + kLinBBytes : kLinStageBytes;
        if (j >= g) e_arrive_expect_tx(smem_u32(&full[s]), per_cta);      // only the odd CTA issued it
        else if (j >= g_odd) e_mbar_complete_tx(smem_u32(&full[s]), per_cta);  // only this CTA issued it
        warp_wait(smem_u32(&full[s]), (j / kLinStages) & 1, p.timeout_ns, 26);
      }
    }
  } else if (warp == 1) {
    griddep_wait();  // bounded waits start once the kernel ahead is done
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
            // per K block: its three scale copies, then its MMA (measured on
            // B200: 4% less tensor-pipe time per stage than all twelve copies
            // ahead of the four MMAs)
            const int nkb = FULL_K ? 4 : min(4, (K - (it - n_lr) * kLinBK) / 64);
#pragma unroll
            for (int kb = 0; kb < nkb; ++kb) {
              e_tmem_cp_pair_32x128b_warpx4(sfa_t + 4 * kb, make_sdesc(sfa_s + kb * 512, 0, 128, 0));
              e_tmem_cp_pair_32x128b_warpx4(sfb_t + 8 * kb, make_sdesc(sfb_s + kb * 512, 0, 128, 0));
              e_tmem_cp_pair_32x128b_warpx4(sfb_t + 8 * kb + 4, make_sdesc(sfb_s + 2048 + kb * 512, 0, 128, 0));
              e_mma_nvf4_pair(acc, make_sdesc(a_s + kb * 32, 16, 1024, 2), make_sdesc(b_s + kb * 32, 16, 1024, 2),
                              idesc_f4, sfa_t + 4 * kb, sfb_t + 8 * kb, (it > 0 || kb > 0) ? 1u : 0u);
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
    griddep_wait();            // the bias and Y may belong to the kernel ahead
    const int et = tid - 64;   // 0..127
    const int q = warp & 3;    // TMEM lane quadrant this warp may access
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    uint8_t* out_s = smem + kLinStageOut + (warp - 2) * 2 * kLinOutBytes;
    const float alpha = p.alpha;
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
          if (lane == 0) mbar_arrive_remote(lead(gi == 0 ? ovl_free : &acc_empty[b]));
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
          // alpha is a power of two, so the product is exact: Y = bf16(acc alpha + bias)
          auto y = [&](int e) { return __fmul_rn(__uint_as_float(v[8 * j + e]), alpha) + bs[8 * j + e]; };
          const uint4 w = make_uint4(pack_bf16x2(y(0), y(1)), pack_bf16x2(y(2), y(3)), pack_bf16x2(y(4), y(5)),
                                     pack_bf16x2(y(6), y(7)));
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
