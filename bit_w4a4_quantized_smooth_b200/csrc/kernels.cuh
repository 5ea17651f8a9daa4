// Device kernels of the SVDQuant W4A4 linear layer for sm_100a.
//
//   pack_residual_kernel   R fp32 [K][N] -> NVFP4 codes [N][K/2] + tiled scales
//   quantize_act_kernel    X bf16 [M][K] -> Xh = X * inv_lambda -> NVFP4 codes
//                          and scales, and T = bf16(bf16(Xh) L1) on warp-level
//                          tensor-core MMAs from the same read of X
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
// chosen so that the tiles fill the SMs once, and with rows x r <= 8192 so
// that a warp holds at most two 16 x 16 tiles of T), over all of K: no split of the
// reduction, hence no partial sums to combine across CTAs.  512 threads, all
// computing; warp 0 also issues the TMA loads (warp-wide, elect.sync), one
// stage behind the consumers, so that four warps per sub-core keep up to 128
// registers each.
//
// A ring stage holds xw = 512, 256 or 128 columns of the tile (the widest
// that still leaves a few stages of shared memory): the X atoms (64 columns,
// K-major, 128-byte swizzle), the matching xw rows of L1 as atoms of aw = r
// (16 or 32) or 64 columns (32/64/128-byte swizzle, columns past r arrive as
// zeros) and the inv_lambda values.
// Per stage every compute warp
//   1. quantises its two items, (16-column group, 32-row block) number w and
//      w + 16 of the stage (one row per lane; the same items every stage, so
//      their offsets are computed once), interleaved so that each thread has
//      two independent dependency chains in flight: codes and scale to global
//      memory, bf16(Xh) back into the X atom in place;
//   2. after all 16 warps have written bf16(Xh) (an mbarrier), adds its share
//      of Xh L1 with warp-level tensor-core MMAs (m16n8k16, bf16 in, fp32 out;
//      fragments by ldmatrix from the swizzled atoms) into a stage partial,
//      then folds that partial into fp32 running sums on the CUDA cores.
// The low-rank contraction (2 rows K r flops) is small and its N = r is at
// most 128: a tcgen05 kind::f16 MMA costs about 85 cycles whatever its N up
// to 128 (measured), and one issuing thread per CTA would need K / 16 of them
// in series, 8 us at K = 3072.  Spread over 16 warps and the four sub-core
// tensor units it hides under the HBM stream.  Folding each stage's partial
// (K <= 512) into fp32 keeps long K as accurate as an fp32 sum (tensor-core
// accumulation over thousands of terms drifts by several bf16 ulps).
// T tiles (16 x 16) are split over the warps; when there are fewer than 16,
// several warps share a tile over disjoint k-steps and the partials are summed
// in a fixed order at the end.
constexpr int kQaWarps = 16;
constexpr int kQaThreads = kQaWarps * 32;
constexpr int kQaMaxStages = 8;
constexpr int kQaMaxRows = 128;
constexpr int kQaMaxUnits = 2;  // 16 x 16 T tiles per warp: rows x r <= 8192
constexpr uint32_t kQaBarBytes = 256 + 512;  // barriers, abort flag, reciprocal table
constexpr uint32_t kQaSmemLimit = 232448;  // 227 KB opt-in dynamic shared memory

struct QaParams {
  const float* inv_lambda;
  uint8_t* x_codes;
  uint8_t* x_scales;
  __nv_bfloat16* T;
  int M, K, r, rows, m_pad;
  int xw;      // columns per stage (512, 256 or 128)
  int aw;      // columns per L1 atom (16, 32 or 64)
  int stages;
  uint32_t stage_bytes;
  uint64_t timeout_ns;
};

__host__ __device__ constexpr int qa_xw(int rows, int r) {
  return (rows <= 32 && r <= 32) ? 512 : ((rows <= 64 && r <= 64) ? 256 : 128);
}
__host__ __device__ constexpr int qa_aw(int r) { return r <= 16 ? 16 : (r <= 32 ? 32 : 64); }
__host__ __device__ constexpr int qa_natoms(int r) { return r == 0 ? 0 : (r + qa_aw(r) - 1) / qa_aw(r); }
__host__ __device__ constexpr uint32_t qa_stage_bytes(int rows, int r) {
  return (static_cast<uint32_t>(qa_xw(rows, r)) *
              (2u * static_cast<uint32_t>(rows) + 2u * static_cast<uint32_t>(qa_natoms(r) * qa_aw(r)) + 4u) +
          1023u) & ~1023u;
}

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

__global__ void __launch_bounds__(kQaThreads, 1)
    quantize_act_kernel(const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ CUtensorMap tm_l1, const QaParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  const int r = p.r;
  const bool has_lr = r > 0;
  const int rows = p.rows;
  const int K = p.K;
  const int xw = p.xw;
  const int aw = p.aw;
  const int S = p.stages;
  const int xa = xw / 64;   // X atoms per stage
  const int gs = xw / 16;   // 16-column groups per row per stage
  const uint32_t x_atom = static_cast<uint32_t>(rows) * 128u;
  const uint32_t x_bytes = xa * x_atom;
  const uint32_t l1_atom = static_cast<uint32_t>(xw * aw * 2);
  const int natoms = has_lr ? (r + aw - 1) / aw : 0;
  const uint32_t l1_bytes = natoms * l1_atom;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * p.stage_bytes);  // [S] stage landed
  uint64_t* xready = full + S;   // [S] all 16 warps wrote bf16(Xh) of the stage
  uint64_t* empty = xready + S;  // [S] all 16 warps done with the stage
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + S);
  float* rcp_tab = reinterpret_cast<float*>(empty + S + 1);  // [128]

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int row0 = blockIdx.x * rows;
  const int nst = (K + xw - 1) / xw;

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&xready[s]), kQaWarps);
      mbar_init(smem_u32(&empty[s]), kQaWarps);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  // T tiles of 16 rows x 16 columns ("units"); see the header comment
  const int nbr = r / 16;               // 16-column blocks of T
  const int U = (rows / 16) * nbr;
  int wpu = 1, kp = 0, nu = 0;
  if (U >= kQaWarps) {
    nu = (U - warp + kQaWarps - 1) / kQaWarps;  // units warp, warp + 16, ...
  } else if (U > 0) {
    wpu = kQaWarps / U;                  // warps sharing a unit
    if (warp < U * wpu) {
      nu = 1;
      kp = warp / U;
    }
  }
  float tot[kQaMaxUnits][8];
#pragma unroll
  for (int i = 0; i < kQaMaxUnits; ++i)
#pragma unroll
    for (int e = 0; e < 8; ++e) tot[i][e] = 0.0f;

  // TMA loads of stage c into its ring slot (warp 0, warp-wide)
  auto load_stage = [&](int c, int slot) {
    const int k = c * xw;
    const int na = min(xa, (K - k) / 64);  // X atoms inside K
    const uint32_t fb = smem_u32(&full[slot]);
    const uint32_t dst = smem_u32(smem + slot * p.stage_bytes);
    // L1 boxes hold at most 256 rows (a TMA limit); an atom is xw rows, and
    // boxes that would start past K are not loaded (no MMA reads them)
    const int lb = xw < 256 ? xw : 256;
    const int nlb = (min(xw, K - k) + lb - 1) / lb;
    e_arrive_expect_tx(fb, na * (x_atom + 256u) + natoms * nlb * lb * aw * 2);
    for (int a = 0; a < na; ++a) e_tma_load_2d(dst + a * x_atom, &tm_x, fb, k + 64 * a, row0);
    for (int t = 0; t < natoms; ++t)
      for (int h = 0; h < nlb; ++h)
        e_tma_load_2d(dst + x_bytes + t * l1_atom + h * lb * aw * 2, &tm_l1, fb, t * aw, k + h * lb);
    e_bulk_load(dst + x_bytes + l1_bytes, p.inv_lambda + k, na * 256u, fb);
  };
  int issued = 0;
  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tm_x);
      if (has_lr) prefetch_tmap(&tm_l1);
    }
    __syncwarp();
    for (; issued < S && issued < nst; ++issued) load_stage(issued, issued);
  }
  {
    const int gs_log2 = 31 - __clz(gs);
    const int items = gs * ((rows + 31) >> 5);  // (group, 32-row block) pairs per stage, <= 32
    // This warp's items are warp and warp + 16 in every stage (items <= 32),
    // so their offsets are fixed: per stage only the column base moves.
    int q_g[2];
    bool q_row[2], q_code[2], q_scale[2];
    uint32_t q_s0[2], q_s1[2];      // shared offsets of the item's two 16-byte chunks
    size_t q_code_base[2], q_scale_base[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int item = warp + kQaWarps * t;
      const int ii = item < items ? item : warp;  // a duplicate is computed, not stored
      q_g[t] = ii & (gs - 1);
      const int rr = ((ii >> gs_log2) << 5) + lane;
      q_row[t] = item < items && rr < rows;
      const int rrc = rr < rows ? rr : 0;
      const uint32_t sw = static_cast<uint32_t>(rrc & 7) << 4;
      const uint32_t c0 = static_cast<uint32_t>((q_g[t] & 3) * 2) << 4;
      q_s0[t] = (q_g[t] >> 2) * x_atom + rrc * 128 + (c0 ^ sw);
      q_s1[t] = (q_g[t] >> 2) * x_atom + rrc * 128 + ((c0 + 16u) ^ sw);
      const int m = row0 + rrc;
      q_code[t] = q_row[t] && m < p.M;
      q_scale[t] = q_row[t] && m < p.m_pad;
      q_code_base[t] = static_cast<size_t>(m) * static_cast<size_t>(K >> 1) + 8 * q_g[t];
      q_scale_base[t] = static_cast<size_t>(m >> 7) * static_cast<size_t>(K >> 6) * 512 + (m & 31) * 16 +
                        ((m & 127) >> 5) * 4 + (q_g[t] >> 2) * 512 + (q_g[t] & 3);
    }
    const int mi = lane >> 3;            // ldmatrix: matrix this lane addresses
    // reciprocals of the 127 finite E4M3 scale values (0 for the zero scale)
    if (warp < 4) {
      const float sd = e4m3_to_f32(static_cast<uint32_t>(tid));
      rcp_tab[tid] = sd == 0.0f ? 0.0f : __frcp_rn(sd);
    }
    __syncthreads();
    // per-unit constants of the low-rank MMAs (unit u of this warp: slot i)
    uint32_t a_off[kQaMaxUnits], b_off[kQaMaxUnits];
    int a_sw[kQaMaxUnits];
#pragma unroll
    for (int i = 0; i < kQaMaxUnits; ++i) {
      const int u = i < nu ? (U >= kQaWarps ? warp + kQaWarps * i : warp % U) : 0;
      const int rb = nbr ? u / nbr : 0, nb = nbr ? u % nbr : 0;
      const int arow = rb * 16 + (lane & 7) + ((mi & 1) << 3);
      a_off[i] = static_cast<uint32_t>(arow * 128);
      a_sw[i] = arow & 7;
      const int bn = nb * 16 + ((mi >> 1) << 3);
      const int bk = (lane & 7) + ((mi & 1) << 3);  // k offset inside a 16-step (swizzle is periodic in 16)
      const int bsw = aw == 64 ? (bk & 7) : (aw == 32 ? ((bk >> 1) & 3) : ((bk >> 2) & 1));
      b_off[i] = static_cast<uint32_t>((bn / aw) * l1_atom + bk * (aw * 2) + ((((bn % aw) >> 3) ^ bsw) << 4));
    }
    const uint32_t b_kstep = static_cast<uint32_t>(16 * aw * 2);  // bytes of 16 L1 rows
    int s = 0;
    uint32_t ph = 0;
    for (int c = 0; c < nst; ++c) {
      const bool ok = !warp_flag(abort_flag) && warp_wait(smem_u32(&full[s]), ph, p.timeout_ns, 12);
      if (!ok) {
        *abort_flag = 1;
        break;
      }
      const int k = c * xw;
      const int kv = min(xw, K - k);      // columns of this stage inside K
      uint8_t* stage = smem + s * p.stage_bytes;
      // 1. quantise this warp's two items (independent chains, interleaved)
      {
        uint4 w0[2], w1[2];
        float4 lm[2][4];
        const float4* lam = reinterpret_cast<const float4*>(stage + x_bytes + l1_bytes);
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          w0[t] = *reinterpret_cast<const uint4*>(stage + q_s0[t]);
          w1[t] = *reinterpret_cast<const uint4*>(stage + q_s1[t]);
#pragma unroll
          for (int e = 0; e < 4; ++e) lm[t][e] = lam[4 * q_g[t] + e];
        }
        float v[2][16];
        uint32_t sc[2], lo[2], hi[2];
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          mul2_rn(v[t][0], v[t][1], bf16_lo(w0[t].x), bf16_hi(w0[t].x), lm[t][0].x, lm[t][0].y);
          mul2_rn(v[t][2], v[t][3], bf16_lo(w0[t].y), bf16_hi(w0[t].y), lm[t][0].z, lm[t][0].w);
          mul2_rn(v[t][4], v[t][5], bf16_lo(w0[t].z), bf16_hi(w0[t].z), lm[t][1].x, lm[t][1].y);
          mul2_rn(v[t][6], v[t][7], bf16_lo(w0[t].w), bf16_hi(w0[t].w), lm[t][1].z, lm[t][1].w);
          mul2_rn(v[t][8], v[t][9], bf16_lo(w1[t].x), bf16_hi(w1[t].x), lm[t][2].x, lm[t][2].y);
          mul2_rn(v[t][10], v[t][11], bf16_lo(w1[t].y), bf16_hi(w1[t].y), lm[t][2].z, lm[t][2].w);
          mul2_rn(v[t][12], v[t][13], bf16_lo(w1[t].z), bf16_hi(w1[t].z), lm[t][3].x, lm[t][3].y);
          mul2_rn(v[t][14], v[t][15], bf16_lo(w1[t].w), bf16_hi(w1[t].w), lm[t][3].z, lm[t][3].w);
        }
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          float a0 = fmaxf(fabsf(v[t][0]), fabsf(v[t][1])), a1 = fmaxf(fabsf(v[t][2]), fabsf(v[t][3]));
          float a2 = fmaxf(fabsf(v[t][4]), fabsf(v[t][5])), a3 = fmaxf(fabsf(v[t][6]), fabsf(v[t][7]));
          a0 = fmaxf(a0, fmaxf(fabsf(v[t][8]), fabsf(v[t][9])));
          a1 = fmaxf(a1, fmaxf(fabsf(v[t][10]), fabsf(v[t][11])));
          a2 = fmaxf(a2, fmaxf(fabsf(v[t][12]), fabsf(v[t][13])));
          a3 = fmaxf(a3, fmaxf(fabsf(v[t][14]), fabsf(v[t][15])));
          const float amax = fmaxf(fmaxf(a0, a1), fmaxf(a2, a3));
          sc[t] = cvt_e4m3_satfinite(__fdiv_rn(amax, 6.0f));
        }
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const float rcp = rcp_tab[sc[t]];
          float pq[16];
#pragma unroll
          for (int e = 0; e < 16; e += 2) mul2_rn(pq[e], pq[e + 1], v[t][e], v[t][e + 1], rcp, rcp);
          lo[t] = cvt_e2m1x8(pq);
          hi[t] = cvt_e2m1x8(pq + 8);
        }
        const size_t code_k = static_cast<size_t>(k >> 1);
        const size_t scale_k = static_cast<size_t>(k >> 6) * 512;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (!q_row[t] || 16 * q_g[t] >= kv) continue;
          if (has_lr) {
            *reinterpret_cast<uint4*>(stage + q_s0[t]) =
                make_uint4(pack_bf16x2(v[t][0], v[t][1]), pack_bf16x2(v[t][2], v[t][3]),
                           pack_bf16x2(v[t][4], v[t][5]), pack_bf16x2(v[t][6], v[t][7]));
            *reinterpret_cast<uint4*>(stage + q_s1[t]) =
                make_uint4(pack_bf16x2(v[t][8], v[t][9]), pack_bf16x2(v[t][10], v[t][11]),
                           pack_bf16x2(v[t][12], v[t][13]), pack_bf16x2(v[t][14], v[t][15]));
          }
          if (q_code[t]) *reinterpret_cast<uint2*>(p.x_codes + q_code_base[t] + code_k) = make_uint2(lo[t], hi[t]);
          if (q_scale[t]) p.x_scales[q_scale_base[t] + scale_k] = static_cast<uint8_t>(sc[t]);
        }
      }
      // 2. low-rank partial product of the stage
      if (has_lr) {
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&xready[s]));
        if (!warp_wait(smem_u32(&xready[s]), ph, p.timeout_ns, 15)) {
          *abort_flag = 1;
          break;
        }
        const uint32_t xs_u = smem_u32(stage);
        const uint32_t l1_u = xs_u + x_bytes;
        const int ksv = kv / 16;
#pragma unroll
        for (int i = 0; i < kQaMaxUnits; ++i) {
          if (i >= nu) break;
          float acc[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
          for (int ks = kp; ks < ksv; ks += wpu) {
            const uint32_t ac = static_cast<uint32_t>((((ks & 3) << 1) | (mi >> 1)) ^ a_sw[i]) << 4;
            uint32_t a[4], b[4];
            ldsm_x4(xs_u + (ks >> 2) * x_atom + a_off[i] + ac, a[0], a[1], a[2], a[3]);
            ldsm_x4_trans(l1_u + b_off[i] + ks * b_kstep, b[0], b[1], b[2], b[3]);
            mma_bf16_16816(acc, a, b[0], b[1], acc);
            mma_bf16_16816(acc + 4, a, b[2], b[3], acc + 4);
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) tot[i][e] = __fadd_rn(tot[i][e], acc[e]);
        }
        fence_proxy_async_smem();  // bf16(Xh) writes before the next TMA into the stage
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
      // warp 0 refills the slot of the previous stage once every warp is done with it
      if (warp == 0 && c >= 1 && c - 1 + S < nst) {
        const int sp = s == 0 ? S - 1 : s - 1;
        const uint32_t pp = s == 0 ? ph ^ 1u : ph;
        if (!warp_wait(smem_u32(&empty[sp]), pp, p.timeout_ns, 11)) {
          *abort_flag = 1;
          break;
        }
        load_stage(c - 1 + S, sp);
        ++issued;
      }
      if (++s == S) {
        s = 0;
        ph ^= 1u;
      }
    }
    if (warp == 0 && warp_flag(abort_flag))  // let this CTA's own copies land before it can exit
      for (int c = issued > S ? issued - S : 0; c < issued; ++c)
        warp_wait(smem_u32(&full[c % S]), (c / S) & 1, p.timeout_ns, 14);
    // scale-layout padding rows that no tile covers: zero scales
    const int covered = gridDim.x * rows;
    if (blockIdx.x == gridDim.x - 1 && covered < p.m_pad) {
      const int gk = K >> 4;
      for (int i = tid; i < (p.m_pad - covered) * gk; i += kQaWarps * 32)
        p.x_scales[scale_byte_offset(covered + i / gk, i % gk, K)] = 0;
    }
  }

  if (has_lr) {
    // T = bf16(sum of the warps' partials), summed in the order kp = 0, 1, ..
    float* part = reinterpret_cast<float*>(smem);  // the ring is idle now
    __syncthreads();
    if (nu > 0 && kp > 0)
#pragma unroll
      for (int e = 0; e < 8; e += 4)
        *reinterpret_cast<float4*>(part + (((kp - 1) * U + warp % U) * 32 + lane) * 8 + e) =
            make_float4(tot[0][e], tot[0][e + 1], tot[0][e + 2], tot[0][e + 3]);
    __syncthreads();
    if (nu > 0 && kp == 0 && !*abort_flag) {
      const int gq = lane >> 2, tq = lane & 3;
#pragma unroll
      for (int i = 0; i < kQaMaxUnits; ++i) {
        if (i >= nu) break;
        const int u = U >= kQaWarps ? warp + kQaWarps * i : warp % U;
        float t8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) t8[e] = tot[i][e];
        for (int q = 1; q < wpu; ++q) {
          const float* src = part + (((q - 1) * U + u) * 32 + lane) * 8;
#pragma unroll
          for (int e = 0; e < 8; ++e) t8[e] = __fadd_rn(t8[e], src[e]);
        }
        const int rb = u / nbr, nb = u % nbr;
#pragma unroll
        for (int jn = 0; jn < 2; ++jn) {
          const int col = nb * 16 + jn * 8 + 2 * tq;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int m = row0 + rb * 16 + gq + 8 * h;
            if (m < p.M)
              *reinterpret_cast<uint32_t*>(p.T + static_cast<size_t>(m) * r + col) =
                  pack_bf16x2(t8[4 * jn + 2 * h], t8[4 * jn + 2 * h + 1]);
          }
        }
      }
    }
  }
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
  uint8_t* smem = align_smem_1024(smem_raw);
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
