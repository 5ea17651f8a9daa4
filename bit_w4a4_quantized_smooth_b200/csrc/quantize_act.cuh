// Activation step of the SVDQuant W4A4 linear layer for sm_100a: smoothing,
// NVFP4 quantisation and the low-rank down-projection T = bf16(bf16(Xh) L1)
// from one read of X (ai-digest.ru abstract and chattools.cn article 584,
// "technical principles": Xh = X diag(lambda)^-1 carries the 4-bit branch
// and the 16-bit low-rank branch, and fusing the two keeps the low-rank
// branch from reading the activation a second time).
//
// Work split.  A CTA owns a tile of 128 rows and a contiguous range of the
// 64-column atoms of K; `splits` CTAs share a row tile when the row tiles
// alone are fewer than the SMs.  One CTA per SM, each streaming its atoms
// through a deep shared-memory ring (the ring's depth, not the bandwidth,
// sets the pace: every slot waits out a loaded TMA latency and a few warp
// hand-offs before it is refilled):
//   warp 16     TMA producer: per atom the X tile (128
//               rows x 64 columns, K-major, 128-byte swizzle), the atom's L1
//               rows (64 k x 64 or 128 ranks, rank-contiguous, 128-byte
//               swizzle; ranks past r arrive as zeros) and its 64 inv_lambda;
//   warps 0-15  quantisers: thread = row, one 16-element group per atom
//               (warp w takes the rows of tensor-memory lane quadrant w % 4
//               and the atom's group w / 4): codes and scale into the
//               stage's staging tiles, bf16(Xh) back into the X tile in place;
//   warp 17     owns the tensor memory and issues, once the sixteen
//               quantisers have written an atom, four tcgen05 kind::f16
//               MMAs (M = 128 rows, N = 64 or 128 ranks, K = 16) of
//               T_part += bf16(Xh) L1 into a tensor-memory accumulator;
//   warp 18     writes the atom's staged codes (one TMA store of 128 rows x
//               32 bytes) and scales (one 512-byte bulk store: the scales of
//               128 rows x 4 groups are one contiguous tile of the block-scale
//               layout), so that the stores leave the SM as whole sectors (a
//               thread per row storing its own 8 bytes would scatter every
//               warp store over 32 rows).
// A slot is refilled once the MMAs and the stores have read it.
// The tensor cores' fp32 accumulation over thousands of terms drifts by a
// few bf16 ulps of small outputs (measured on B200), so each accumulator
// takes at most `fold` atoms (512 columns at the least) and the accumulators
// are added on the CUDA cores in a fixed order.
// With splits > 1 the CTAs of a row tile combine their partial T through the
// caller's workspace: each writes its fp32 partial (rows below M), then
// counts itself in the tile's counter; the CTA that counts last adds the
// partials in split order, rounds once to bf16, stores T and resets the
// counter.  The order of the sum is fixed, whichever CTA finishes last.
#pragma once

#include "common.cuh"

namespace svdq {

constexpr int kQaRows = 128;                 // rows per CTA tile (MMA M)
constexpr int kQaQuantWarps = 16;
constexpr int kQaProducerWarp = 16;
constexpr int kQaMmaWarp = 17;
constexpr int kQaStoreWarp = 18;
constexpr int kQaThreads = 19 * 32;
constexpr int kQaMaxStages = 8;
constexpr int kQaMaxSplits = 16;
constexpr uint32_t kQaXBytes = kQaRows * 128;  // one X atom
constexpr uint32_t kQaL1AtomBytes = 64 * 128;  // 64 k-rows x 64 ranks of L1
constexpr uint32_t kQaCodeStage = kQaRows * 32;  // staged codes of one atom (128 rows x 32 bytes)
constexpr uint32_t kQaScaleStage = 512;          // staged scales of one atom (one scale tile)
constexpr uint32_t kQaHeadBytes = 1024;        // barriers, flags, reciprocal table
constexpr uint32_t kQaSmemLimit = 232448;      // 227 KB opt-in dynamic shared memory
constexpr size_t kQaCounterBytes = 256;        // workspace granule of the per-tile counters

struct QaParams {
  const float* inv_lambda;
  uint8_t* x_codes;
  uint8_t* x_scales;
  __nv_bfloat16* T;
  unsigned int* counters;  // [row tiles] (workspace; zero between calls)
  float* partials;         // [row tiles][splits][128][r] (workspace)
  int M, K, r;
  int splits;        // CTAs per row tile along K
  int apc;           // 64-column atoms per CTA (the last CTA of a tile may have fewer)
  int stages;        // ring depth
  int n_l1;          // 64-rank L1 atoms per stage (0, 1 or 2)
  int fold;          // atoms per tensor-memory accumulator
  uint32_t stage_bytes;
  uint32_t tmem_cols;
  uint64_t timeout_ns;
};

// A ring stage: [X atom][L1 atoms][staged codes][inv_lambda][staged scales].
__host__ __device__ constexpr uint32_t qa_stage_bytes(int n_l1) {
  return (kQaXBytes + static_cast<uint32_t>(n_l1) * kQaL1AtomBytes + kQaCodeStage + 256u + kQaScaleStage + 1023u) &
         ~1023u;
}

// Workspace bytes of a launch: the counters, then the partial sums.
__host__ __device__ constexpr size_t qa_workspace_bytes(int64_t row_tiles, int splits, int r) {
  return (splits > 1 && r > 0)
             ? kQaCounterBytes * ((static_cast<size_t>(row_tiles) * 4 + kQaCounterBytes - 1) / kQaCounterBytes) +
                   static_cast<size_t>(row_tiles) * static_cast<size_t>(splits) * kQaRows * static_cast<size_t>(r) * 4
             : 0;
}

// GELU(x) = 0.5 x (1 + erf(x / sqrt 2)), erf from the purely rational
// approximation of Abramowitz and Stegun, Handbook of Mathematical Functions,
// formula 7.1.28:  erf(z) ~ 1 - (1 + a1 z + ... + a6 z^6)^-16  (z >= 0, odd
// in z; |error| <= 3e-7 in exact arithmetic).  Evaluated with one rounded fp32
// operation per step, no fused multiply-add, in a fixed order, so that the
// result is reproducible bit for bit: z = |x| RN(1/sqrt 2); Horner from a6
// (a multiply, then an add); four squarings; e = 1 - RN(1/p16); sign of x;
// (0.5 x) (1 + erf).
// Two elements at a time with packed fp32x2 multiplies and adds (each lane
// rounded as the scalar operation would be); 1/p16 is the correctly rounded
// reciprocal, the same value as the IEEE quotient 1/p16.
__device__ __forceinline__ void gelu_as2(float& x0, float& x1) {
  float z0, z1, p0 = 0.0000430638f, p1 = 0.0000430638f;
  mul2_rn(z0, z1, fabsf(x0), fabsf(x1), 0.70710678118654752f, 0.70710678118654752f);
  const float c[6] = {0.0002765672f, 0.0001520143f, 0.0092705272f, 0.0422820123f, 0.0705230784f, 1.0f};
#pragma unroll
  for (int i = 0; i < 6; ++i) {
    mul2_rn(p0, p1, p0, p1, z0, z1);
    add2_rn(p0, p1, p0, p1, c[i], c[i]);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) mul2_rn(p0, p1, p0, p1, p0, p1);
  float e0, e1;
  add2_rn(e0, e1, 1.0f, 1.0f, -__frcp_rn(p0), -__frcp_rn(p1));
  float h0, h1, s0, s1;
  mul2_rn(h0, h1, 0.5f, 0.5f, x0, x1);
  add2_rn(s0, s1, 1.0f, 1.0f, signbit(x0) ? -e0 : e0, signbit(x1) ? -e1 : e1);
  mul2_rn(x0, x1, h0, h1, s0, s1);
}

// GELU: the input goes through gelu_as (in fp32, no bf16 rounding between)
// before the smoothing multiply, Xh = RN_f32(GELU(x) inv_lambda): the MLP's
// activation fused with the next layer's quantisation.
template <bool GELU>
__global__ void __launch_bounds__(kQaThreads, 1)
    quantize_act_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_l1,
                        const __grid_constant__ CUtensorMap tm_xc, const QaParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  const int S = p.stages;
  const int r = p.r;
  const bool has_lr = r > 0;
  const int K = p.K;
  const uint32_t l1_bytes = static_cast<uint32_t>(p.n_l1) * kQaL1AtomBytes;
  const uint32_t code_off = kQaXBytes + l1_bytes;
  const uint32_t lam_off = code_off + kQaCodeStage;
  const uint32_t scale_off = lam_off + 256u;
  // [0, 1024): barriers, flags and the reciprocal table; the ring follows
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);  // [S] stage landed
  uint64_t* xready = full + S;  // [S] the 16 quantisers wrote the stage's staging and bf16(Xh)
  uint64_t* empty = xready + S; // [S] the stage may be refilled (stores read it, MMAs done)
  uint64_t* fin = empty + S;    // every MMA of the CTA complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* is_last = abort_flag + 1;
  float* rcp_tab = reinterpret_cast<float*>(smem + 256);  // [128]
  uint8_t* ring = smem + 1024;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int split = blockIdx.x;
  const int tile = blockIdx.y;
  const int row0 = tile * kQaRows;
  const int atoms = K >> 6;
  const int a0 = split * p.apc;
  const int na = min(p.apc, atoms - a0);  // atoms of this CTA (>= 1)

  if (warp == kQaMmaWarp && has_lr) {
    tmem_alloc(smem_u32(tmem_slot), p.tmem_cols);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&xready[s]), kQaQuantWarps);
      mbar_init(smem_u32(&empty[s]), has_lr ? 2 : 1);
    }
    mbar_init(smem_u32(fin), 1);
    *abort_flag = 0;
    *is_last = 0;
    fence_barrier_init();
  }
  if (tid < 128) {
    // reciprocals of the 127 finite E4M3 scale values (0 for the zero scale)
    const float sd = e4m3_to_f32(static_cast<uint32_t>(tid));
    rcp_tab[tid] = sd == 0.0f ? 0.0f : __frcp_rn(sd);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // The kernel behind this one may now be scheduled; only now, with this
  // CTA's tensor memory held: a later kernel's CTA that took it first would
  // wait in its griddep_wait for this grid while this CTA waited for its
  // tensor memory.
  griddep_launch_dependents();
  griddep_wait();  // X, the outputs and the workspace may belong to the kernel ahead
  const uint32_t tmem = has_lr ? *tmem_slot : 0u;
  const uint32_t sbase = smem_u32(ring);

  if (warp == kQaProducerWarp) {
    // ---------------------------------------------------------- producer --
    if (lane == 0) {
      prefetch_tmap(&tm_x);
      prefetch_tmap(&tm_xc);
      if (has_lr) prefetch_tmap(&tm_l1);
    }
    __syncwarp();
    // No L2 prefetch ahead of the ring: measured on B200, prefetching the
    // CTA's atoms first delayed the ring's own first loads by about 2 us and
    // lengthened the stream (4 us at K = 3072, 8 us at K = 12288); the ring's
    // loads alone keep enough bytes in flight.
    const uint32_t tx = kQaXBytes + l1_bytes + 256u;
    int issued = 0;
    int s = 0;
    uint32_t ph = 0;  // this use's phase of the slot; the previous use had ph ^ 1
    for (int c = 0; c < na; ++c) {
      if (c >= S && !warp_wait(smem_u32(&empty[s]), ph ^ 1u, p.timeout_ns, 40)) {
        *abort_flag = 1;
        break;
      }
      if (warp_flag(abort_flag)) break;
      const int k = (a0 + c) * 64;
      const uint32_t fb = smem_u32(&full[s]);
      const uint32_t dst = sbase + s * p.stage_bytes;
      e_arrive_expect_tx(fb, tx);
      e_tma_load_2d(dst, &tm_x, fb, k, row0);
      for (int t = 0; t < p.n_l1; ++t) e_tma_load_2d(dst + kQaXBytes + t * kQaL1AtomBytes, &tm_l1, fb, 64 * t, k);
      e_bulk_load(dst + lam_off, p.inv_lambda + k, 256u, fb);
      ++issued;
      if (++s == S) {
        s = 0;
        ph ^= 1u;
      }
    }
    // after an abort: this CTA's own copies land before it may exit
    if (warp_flag(abort_flag))
      for (int c = issued > S ? issued - S : 0; c < issued; ++c)
        warp_wait(smem_u32(&full[c % S]), (c / S) & 1, p.timeout_ns, 41);
  } else if (warp == kQaMmaWarp) {
    // ------------------------------------------------------- MMA issuer --
    if (has_lr) {
      // bf16 x bf16 -> fp32; A = bf16(Xh) K-major, B = L1 rank-contiguous (MN-major)
      const uint32_t n_acc_cols = 64u * static_cast<uint32_t>(p.n_l1);
      const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((n_acc_cols >> 3) << 17) |
                             (static_cast<uint32_t>(kQaRows >> 4) << 24);
      int s = 0;
      uint32_t ph = 0;
      for (int c = 0; c < na; ++c) {
        const bool ok = !warp_flag(abort_flag) && warp_wait(smem_u32(&xready[s]), ph, p.timeout_ns, 42);
        if (!ok) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t st = sbase + s * p.stage_bytes;
        const uint32_t acc = tmem + static_cast<uint32_t>(c / p.fold) * n_acc_cols;
        const uint32_t first = (c % p.fold) == 0 ? 1u : 0u;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          e_mma_bf16(acc, make_sdesc(st + kk * 32, 16, 1024, 2),
                     make_sdesc(st + kQaXBytes + kk * 2048, kQaL1AtomBytes, 1024, 2), idesc,
                     (first && kk == 0) ? 0u : 1u);
        e_commit(smem_u32(&empty[s]));  // the MMAs' share of releasing the slot
        if (++s == S) {
          s = 0;
          ph ^= 1u;
        }
      }
      // every MMA of the CTA (also after an abort) completes before the
      // tensor memory is read or released
      e_commit(smem_u32(fin));
      if (!warp_wait(smem_u32(fin), 0, p.timeout_ns, 43)) *abort_flag = 1;
    }
  } else if (warp == kQaStoreWarp) {
    // ------------------------------------------------------------ stores --
    int s = 0;
    uint32_t ph = 0;
    for (int c = 0; c < na; ++c) {
      const bool ok = !warp_flag(abort_flag) && warp_wait(smem_u32(&xready[s]), ph, p.timeout_ns, 47);
      if (!ok) {
        *abort_flag = 1;
        break;
      }
      if (lane == 0) {
        const uint32_t st = sbase + s * p.stage_bytes;
        const int a = a0 + c;
        tma_store_2d(&tm_xc, st + code_off, 32 * a, row0);
        bulk_store(p.x_scales + (static_cast<size_t>(tile) * static_cast<size_t>(atoms) + a) * 512, st + scale_off,
                   kQaScaleStage);
        bulk_commit_group();
        bulk_wait_group_read<0>();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&empty[s]));  // the stores' share of releasing the slot
      if (++s == S) {
        s = 0;
        ph ^= 1u;
      }
    }
    if (lane == 0) bulk_wait_group<0>();  // the stores are complete before the CTA exits
    __syncwarp();
  } else {
    // -------------------------------------------------------- quantisers --
    const int q = warp & 3;      // rows [32 q, 32 q + 32) of the tile
    const int g = warp >> 2;     // group g (columns [16 g, 16 g + 16)) of each atom
    const int rr = 32 * q + lane;
    const uint32_t sw = static_cast<uint32_t>(rr & 7);
    const uint32_t off0 = static_cast<uint32_t>(rr * 128) + (((2u * g) ^ sw) << 4);
    const uint32_t off1 = static_cast<uint32_t>(rr * 128) + (((2u * g + 1u) ^ sw) << 4);
    const uint32_t code_sm = static_cast<uint32_t>(rr * 32 + 8 * g);
    const uint32_t scale_sm = static_cast<uint32_t>((rr & 31) * 16 + (rr >> 5) * 4 + g);
    int s = 0;
    uint32_t ph = 0;
    for (int c = 0; c < na; ++c) {
      const bool ok = !warp_flag(abort_flag) && warp_wait(smem_u32(&full[s]), ph, p.timeout_ns, 44);
      if (!ok) {
        *abort_flag = 1;
        break;
      }
      uint8_t* stage = ring + s * p.stage_bytes;
      const uint4 x0 = *reinterpret_cast<const uint4*>(stage + off0);
      const uint4 x1 = *reinterpret_cast<const uint4*>(stage + off1);
      const float4* lam = reinterpret_cast<const float4*>(stage + lam_off) + 4 * g;
      const float4 l0 = lam[0], l1 = lam[1], l2 = lam[2], l3 = lam[3];
      float v[16];
      {
        float xi[16] = {bf16_lo(x0.x), bf16_hi(x0.x), bf16_lo(x0.y), bf16_hi(x0.y),
                        bf16_lo(x0.z), bf16_hi(x0.z), bf16_lo(x0.w), bf16_hi(x0.w),
                        bf16_lo(x1.x), bf16_hi(x1.x), bf16_lo(x1.y), bf16_hi(x1.y),
                        bf16_lo(x1.z), bf16_hi(x1.z), bf16_lo(x1.w), bf16_hi(x1.w)};
        if constexpr (GELU) {
#pragma unroll
          for (int e = 0; e < 16; e += 2) gelu_as2(xi[e], xi[e + 1]);
        }
        mul2_rn(v[0], v[1], xi[0], xi[1], l0.x, l0.y);
        mul2_rn(v[2], v[3], xi[2], xi[3], l0.z, l0.w);
        mul2_rn(v[4], v[5], xi[4], xi[5], l1.x, l1.y);
        mul2_rn(v[6], v[7], xi[6], xi[7], l1.z, l1.w);
        mul2_rn(v[8], v[9], xi[8], xi[9], l2.x, l2.y);
        mul2_rn(v[10], v[11], xi[10], xi[11], l2.z, l2.w);
        mul2_rn(v[12], v[13], xi[12], xi[13], l3.x, l3.y);
        mul2_rn(v[14], v[15], xi[14], xi[15], l3.z, l3.w);
      }
      float a0m = fmaxf(fabsf(v[0]), fabsf(v[1])), a1m = fmaxf(fabsf(v[2]), fabsf(v[3]));
      float a2m = fmaxf(fabsf(v[4]), fabsf(v[5])), a3m = fmaxf(fabsf(v[6]), fabsf(v[7]));
      a0m = fmaxf(a0m, fmaxf(fabsf(v[8]), fabsf(v[9])));
      a1m = fmaxf(a1m, fmaxf(fabsf(v[10]), fabsf(v[11])));
      a2m = fmaxf(a2m, fmaxf(fabsf(v[12]), fabsf(v[13])));
      a3m = fmaxf(a3m, fmaxf(fabsf(v[14]), fabsf(v[15])));
      const float amax = fmaxf(fmaxf(a0m, a1m), fmaxf(a2m, a3m));
      const uint32_t sc = cvt_e4m3_satfinite(__fdiv_rn(amax, 6.0f));
      const float rcp = rcp_tab[sc];
      float pq[16];
#pragma unroll
      for (int e = 0; e < 16; e += 2) mul2_rn(pq[e], pq[e + 1], v[e], v[e + 1], rcp, rcp);
      const uint32_t lo = cvt_e2m1x8(pq);
      const uint32_t hi = cvt_e2m1x8(pq + 8);
      if (has_lr) {
        *reinterpret_cast<uint4*>(stage + off0) = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                                             pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
        *reinterpret_cast<uint4*>(stage + off1) = make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]),
                                                             pack_bf16x2(v[12], v[13]), pack_bf16x2(v[14], v[15]));
      }
      // staged codes: row rr's 32 bytes, group g at byte 8 g; staged scales:
      // (rr, g) at (rr % 32) 16 + (rr / 32) 4 + g, the block-scale tile's
      // order.  Rows past M read zeros (TMA fill) and give the zero scale;
      // the TMA store clips their codes.
      *reinterpret_cast<uint2*>(stage + code_off + code_sm) = make_uint2(lo, hi);
      stage[scale_off + scale_sm] = static_cast<uint8_t>(sc);
      fence_proxy_async_smem();  // staged bytes and bf16(Xh) before the async proxy reads them
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&xready[s]));
      if (++s == S) {
        s = 0;
        ph ^= 1u;
      }
    }
  }

  // ---------------------------------------------- T: fold and combine --
  __syncthreads();  // every role is done: the ring is idle, the MMAs complete
  const bool aborted = *abort_flag != 0;
  const int vrows = min(kQaRows, p.M - row0);  // rows of the tile below M
  if (has_lr && warp < 4 && 32 * warp < vrows && warp_wait(smem_u32(fin), 0, p.timeout_ns, 45)) {
    tc_fence_after();
    const int rr = 32 * warp + lane;
    const int m = row0 + rr;
    const uint32_t lane_base = static_cast<uint32_t>(32 * warp) << 16;
    const uint32_t n_acc_cols = 64u * static_cast<uint32_t>(p.n_l1);
    const int n_acc = (na + p.fold - 1) / p.fold;
    for (int cb = 0; cb < r; cb += 16) {
      float t16[16];
      {
        uint32_t v[16];
        tmem_ld_32x32b_x16(tmem + lane_base + cb, v);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) t16[e] = __uint_as_float(v[e]);
      }
      for (int ac = 1; ac < n_acc; ++ac) {  // accumulators in a fixed order
        uint32_t v[16];
        tmem_ld_32x32b_x16(tmem + lane_base + ac * n_acc_cols + cb, v);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) t16[e] = __fadd_rn(t16[e], __uint_as_float(v[e]));
      }
      if (m < p.M && !aborted) {
        if (p.splits == 1) {
          uint4* dst = reinterpret_cast<uint4*>(p.T + static_cast<size_t>(m) * r + cb);
          dst[0] = make_uint4(pack_bf16x2(t16[0], t16[1]), pack_bf16x2(t16[2], t16[3]), pack_bf16x2(t16[4], t16[5]),
                              pack_bf16x2(t16[6], t16[7]));
          dst[1] = make_uint4(pack_bf16x2(t16[8], t16[9]), pack_bf16x2(t16[10], t16[11]),
                              pack_bf16x2(t16[12], t16[13]), pack_bf16x2(t16[14], t16[15]));
        } else {
          float4* dst = reinterpret_cast<float4*>(
              p.partials + ((static_cast<size_t>(tile) * p.splits + split) * kQaRows + rr) * r + cb);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_float4(t16[4 * e], t16[4 * e + 1], t16[4 * e + 2], t16[4 * e + 3]);
        }
      }
    }
  }
  if (has_lr && p.splits > 1) {
    // Count this CTA in the tile's counter once its partial is visible; the
    // CTA that counts last combines the partials.  Every CTA counts exactly
    // once (also after an abort), so the counter ends each call at zero.
    __threadfence();
    __syncthreads();
    if (tid == 0) {
      const unsigned int before = atomicAdd(&p.counters[tile], 1u);
      if (before == static_cast<unsigned int>(p.splits) - 1u) {
        *is_last = 1;
        p.counters[tile] = 0u;  // no CTA of this launch touches it again
      }
    }
    __syncthreads();
    if (*is_last) {
      __threadfence();  // the other CTAs' partials, published before their count
      const int n4 = r >> 2;
      const float* base = p.partials + static_cast<size_t>(tile) * p.splits * kQaRows * r;
      for (int e = tid; e < vrows * n4; e += kQaThreads) {
        const int row = e / n4;
        const int c4 = e % n4;
        const float* src = base + static_cast<size_t>(row) * r + 4 * c4;
        float4 acc = __ldcg(reinterpret_cast<const float4*>(src));
        for (int j = 1; j < p.splits; ++j) {  // split order
          const float4 b = __ldcg(reinterpret_cast<const float4*>(src + static_cast<size_t>(j) * kQaRows * r));
          acc.x = __fadd_rn(acc.x, b.x);
          acc.y = __fadd_rn(acc.y, b.y);
          acc.z = __fadd_rn(acc.z, b.z);
          acc.w = __fadd_rn(acc.w, b.w);
        }
        if (!aborted)
          *reinterpret_cast<uint2*>(p.T + static_cast<size_t>(row0 + row) * r + 4 * c4) =
              make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kQaMmaWarp && has_lr) tmem_dealloc(tmem, p.tmem_cols);
}

}  // namespace svdq
