// C ABI of the SVDQuant W4A4 linear layer (see include/svdq.h): argument
// validation, TMA tensor maps and kernel launches.  Host code only launches
// the kernels in kernels.cuh; no step of the layer runs on the host.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/svdq.h"
#include "kernels.cuh"

namespace {


uint64_t g_timeout_ns = 0;
std::once_flag g_timeout_once;

uint64_t wait_timeout_ns() {
  std::call_once(g_timeout_once, [] {
    uint64_t ms = 2000;
    if (const char* e = std::getenv("SVDQ_WAIT_TIMEOUT_MS")) {
      long long v = std::atoll(e);
      if (v > 0) ms = static_cast<uint64_t>(v);
    }
    g_timeout_ns = ms * 1000000ull;
  });
  return g_timeout_ns;
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_rank(int64_t r) { return r >= 0 && r <= 128 && r % 16 == 0; }

// 2D/3D tiled tensor map; dims/strides innermost first, strides in bytes.
int make_tmap(CUtensorMap* map, CUtensorMapDataType dtype, uint32_t rank, const void* base,
              const uint64_t* dims, const uint64_t* strides, const uint32_t* box,
              CUtensorMapSwizzle swizzle) {
  auto enc = encode_fn();
  if (!enc) return SVDQ_ERR_CUDA;
  uint32_t estr[3] = {1, 1, 1};
  CUresult rc = enc(map, dtype, rank, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return rc == CUDA_SUCCESS ? SVDQ_OK : SVDQ_ERR_CUDA;
}

int launch_status() { return cudaGetLastError() == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA; }

// Streaming multiprocessors of the current device (cached per device id).
int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev < 0 || dev >= 64) return 0;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cached[dev] = n;
  }
  return cached[dev];
}

// Rows per activation tile: a multiple of 16 in [16, 128] such that the
// tiles cover M in about one wave over the SMs (one CTA per SM), and such that
// the 16 x 16 tiles of T number at most two per warp (rows x r <= 8192).
int choose_rows(int64_t M, int sms, int64_t r) {
  int64_t rows = (M + sms - 1) / sms;
  rows = (rows + 15) / 16 * 16;
  int64_t cap = svdq::kQaMaxRows;
  if (r > 0) {
    const int64_t by_units = (2 * 16 / (r / 16)) * 16;
    if (by_units < cap) cap = by_units;
  }
  if (rows > cap) rows = cap;
  if (rows < 16) rows = 16;
  return static_cast<int>(rows);
}

}  // namespace

extern "C" {

const char* svdq_status_string(int status) {
  switch (status) {
    case SVDQ_OK: return "SVDQ_OK";
    case SVDQ_ERR_INVALID_ARG: return "SVDQ_ERR_INVALID_ARG";
    case SVDQ_ERR_UNSUPPORTED_SHAPE: return "SVDQ_ERR_UNSUPPORTED_SHAPE";
    case SVDQ_ERR_MISALIGNED: return "SVDQ_ERR_MISALIGNED";
    case SVDQ_ERR_CUDA: return "SVDQ_ERR_CUDA";
    case SVDQ_ERR_TIMEOUT: return "SVDQ_ERR_TIMEOUT";
    default: return "SVDQ_UNKNOWN_STATUS";
  }
}

int svdq_packed_sizes(int64_t rows, int64_t K, size_t* codes_bytes, size_t* scales_bytes) {
  if (rows < 0 || K <= 0 || !codes_bytes || !scales_bytes) return SVDQ_ERR_INVALID_ARG;
  if (K % 64 != 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  *codes_bytes = static_cast<size_t>(rows) * static_cast<size_t>(K / 2);
  *scales_bytes = static_cast<size_t>((rows + 127) / 128) * 128 * static_cast<size_t>(K / 16);
  return SVDQ_OK;
}

int svdq_pack_residual(const float* R, int64_t K, int64_t N, uint8_t* r_codes, uint8_t* r_scales,
                       void* stream) {
  if (!R || !r_codes || !r_scales || K <= 0 || N <= 0) return SVDQ_ERR_INVALID_ARG;
  if (K % 64 != 0 || N % 16 != 0 || K > (1 << 30) || N > (1 << 30)) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(R) || !aligned16(r_codes) || !aligned16(r_scales)) return SVDQ_ERR_MISALIGNED;
  dim3 grid(static_cast<unsigned>((N + 127) / 128), static_cast<unsigned>(K / 64));
  svdq::pack_residual_kernel<<<grid, svdq::kPackThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      R, static_cast<int>(K), static_cast<int>(N), r_codes, r_scales);
  return launch_status();
}

int svdq_quantize_act(const void* X, const float* inv_lambda, const void* L1, int64_t M, int64_t K,
                      int64_t r, uint8_t* x_codes, uint8_t* x_scales, void* T, void* stream) {
  if (!X || !inv_lambda || !x_codes || !x_scales || M <= 0 || K <= 0) return SVDQ_ERR_INVALID_ARG;
  if (r > 0 && (!L1 || !T)) return SVDQ_ERR_INVALID_ARG;
  if (K % 64 != 0 || !valid_rank(r) || M > (1 << 30) || K > (1 << 30)) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(X) || !aligned16(inv_lambda) || !aligned16(x_codes) || !aligned16(x_scales) ||
      (r > 0 && (!aligned16(L1) || !aligned16(T))))
    return SVDQ_ERR_MISALIGNED;

  const int sms = sm_count();
  if (sms <= 0) return SVDQ_ERR_CUDA;
  const int rows = choose_rows(M, sms, r);
  CUtensorMap tm_x, tm_l1;
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(M)};
    const uint64_t strides[1] = {static_cast<uint64_t>(K) * 2};
    const uint32_t box[2] = {64, static_cast<uint32_t>(rows)};
    int rc = make_tmap(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, X, dims, strides, box,
                       CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
  }
  const int ri = static_cast<int>(r);
  const int xw = svdq::qa_xw(rows, ri);
  const int aw = svdq::qa_aw(ri);
  if (r > 0) {
    // L1 [K][r] in atoms of aw columns x xw rows (boxes of up to 256 rows); the swizzle width is the
    // atom's row (32, 64 or 128 bytes); columns past r arrive as zeros
    const uint64_t dims[2] = {static_cast<uint64_t>(r), static_cast<uint64_t>(K)};
    const uint64_t strides[1] = {static_cast<uint64_t>(r) * 2};
    const uint32_t box[2] = {static_cast<uint32_t>(aw), static_cast<uint32_t>(xw < 256 ? xw : 256)};
    const CUtensorMapSwizzle sw = aw == 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                                           : (aw == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
    int rc = make_tmap(&tm_l1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, L1, dims, strides, box, sw);
    if (rc) return rc;
  } else {
    std::memset(&tm_l1, 0, sizeof(tm_l1));
  }

  const uint32_t stage_bytes = svdq::qa_stage_bytes(rows, ri);
  const uint32_t fixed = 1024 + svdq::kQaBarBytes;
  int stages = static_cast<int>((svdq::kQaSmemLimit - fixed) / stage_bytes);
  if (stages > svdq::kQaMaxStages) stages = svdq::kQaMaxStages;
  if (stages < 2) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  svdq::QaParams p;
  p.inv_lambda = inv_lambda;
  p.x_codes = x_codes;
  p.x_scales = x_scales;
  p.T = static_cast<__nv_bfloat16*>(T);
  p.M = static_cast<int>(M);
  p.K = static_cast<int>(K);
  p.r = ri;
  p.rows = rows;
  p.m_pad = static_cast<int>((M + 127) / 128 * 128);
  p.xw = xw;
  p.aw = aw;
  p.stages = stages;
  p.stage_bytes = stage_bytes;
  p.timeout_ns = wait_timeout_ns();

  const size_t smem = fixed + static_cast<size_t>(stages) * stage_bytes;
  if (cudaFuncSetAttribute(svdq::quantize_act_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return SVDQ_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((M + rows - 1) / rows));
  cfg.blockDim = dim3(svdq::kQaThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cfg.attrs = nullptr;
  cfg.numAttrs = 0;
  if (cudaLaunchKernelEx(&cfg, svdq::quantize_act_kernel, tm_x, tm_l1, p) != cudaSuccess)
    return SVDQ_ERR_CUDA;
  return launch_status();
}

int svdq_linear(const uint8_t* x_codes, const uint8_t* x_scales, const void* T, const uint8_t* r_codes,
                const uint8_t* r_scales, const void* L2, const void* bias, int64_t M, int64_t K,
                int64_t N, int64_t r, void* Y, void* stream) {
  if (!x_codes || !x_scales || !r_codes || !r_scales || !Y || M <= 0 || K <= 0 || N <= 0)
    return SVDQ_ERR_INVALID_ARG;
  if (r > 0 && (!T || !L2)) return SVDQ_ERR_INVALID_ARG;
  if (K % 64 != 0 || N % 16 != 0 || !valid_rank(r) || M > (1 << 30) || N > (1 << 30) ||
      K > (1 << 30))
    return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(x_codes) || !aligned16(x_scales) || !aligned16(r_codes) || !aligned16(r_scales) ||
      !aligned16(Y) || (bias && !aligned16(bias)) || (r > 0 && (!aligned16(T) || !aligned16(L2))))
    return SVDQ_ERR_MISALIGNED;

  CUtensorMap tm_xc, tm_rc, tm_t, tm_l2;
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(K / 2), static_cast<uint64_t>(M)};
    const uint64_t strides[1] = {static_cast<uint64_t>(K / 2)};
    const uint32_t box[2] = {128, 128};
    int rc = make_tmap(&tm_xc, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, x_codes, dims, strides, box,
                       CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(K / 2), static_cast<uint64_t>(N)};
    const uint64_t strides[1] = {static_cast<uint64_t>(K / 2)};
    const uint32_t box[2] = {128, 128};  // each CTA of a pair loads 128 R rows
    int rc = make_tmap(&tm_rc, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, r_codes, dims, strides, box,
                       CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
  }
  // scale tiles viewed as [tiles][2][256] bytes: a box of 4 tiles is the
  // 2 KB of scales of one 256-wide K stage of a 128-row band
  CUtensorMap tm_xs, tm_rs;
  {
    const uint64_t dims[3] = {256, 2, static_cast<uint64_t>((M + 127) / 128) * static_cast<uint64_t>(K / 64)};
    const uint64_t strides[2] = {256, 512};
    const uint32_t box[3] = {256, 2, 4};
    int rc = make_tmap(&tm_xs, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, x_scales, dims, strides, box,
                       CU_TENSOR_MAP_SWIZZLE_NONE);
    if (rc) return rc;
  }
  {
    const uint64_t dims[3] = {256, 2, static_cast<uint64_t>((N + 127) / 128) * static_cast<uint64_t>(K / 64)};
    const uint64_t strides[2] = {256, 512};
    const uint32_t box[3] = {256, 2, 4};
    int rc = make_tmap(&tm_rs, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, r_scales, dims, strides, box,
                       CU_TENSOR_MAP_SWIZZLE_NONE);
    if (rc) return rc;
  }
  if (r > 0) {
    const uint64_t dt[2] = {static_cast<uint64_t>(r), static_cast<uint64_t>(M)};
    const uint64_t st[1] = {static_cast<uint64_t>(r) * 2};
    const uint32_t bt[2] = {64, 128};
    int rc = make_tmap(&tm_t, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, T, dt, st, bt,
                       CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
    const uint64_t dl[2] = {static_cast<uint64_t>(N), static_cast<uint64_t>(r)};
    const uint64_t sl[1] = {static_cast<uint64_t>(N) * 2};
    const uint32_t bl[2] = {64, 64};
    rc = make_tmap(&tm_l2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, L2, dl, sl, bl,
                   CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
  } else {
    std::memset(&tm_t, 0, sizeof(tm_t));
    std::memset(&tm_l2, 0, sizeof(tm_l2));
  }

  CUtensorMap tm_y;
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(N), static_cast<uint64_t>(M)};
    const uint64_t strides[1] = {static_cast<uint64_t>(N) * 2};
    const uint32_t box[2] = {64, 32};  // one epilogue warp's 32 x 64 block
    int rc = make_tmap(&tm_y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Y, dims, strides, box,
                       CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
  }

  svdq::LinParams p;
  p.bias = static_cast<const __nv_bfloat16*>(bias);
  p.Y = static_cast<__nv_bfloat16*>(Y);
  p.M = static_cast<int>(M);
  p.K = static_cast<int>(K);
  p.N = static_cast<int>(N);
  p.r = static_cast<int>(r);
  p.timeout_ns = wait_timeout_ns();
  p.m_tiles = static_cast<int>((M + svdq::kLinBM - 1) / svdq::kLinBM);
  p.tiles = p.m_tiles * static_cast<int>((N + svdq::kLinBN - 1) / svdq::kLinBN);

  const size_t smem = 1024 + svdq::kLinBarOffset + (svdq::kLinNumBars + 2) * 8;
  const bool full_k = (K % svdq::kLinBK) == 0;
  auto kern = full_k ? svdq::linear_kernel<true> : svdq::linear_kernel<false>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
      cudaSuccess)
    return SVDQ_ERR_CUDA;
  const int sms = sm_count();
  if (sms < 2) return SVDQ_ERR_CUDA;
  const int pairs = p.tiles < sms / 2 ? p.tiles : sms / 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
  cfg.blockDim = dim3(svdq::kLinThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, tm_xc, tm_rc, tm_xs, tm_rs, tm_t, tm_l2, tm_y, p) != cudaSuccess)
    return SVDQ_ERR_CUDA;
  return launch_status();
}

int svdq_sync_status(void* stream, int* where) {
  if (where) *where = 0;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SVDQ_ERR_CUDA;
  unsigned int code = 0, w = 0;
  if (cudaMemcpyFromSymbol(&code, svdq::g_status_code, sizeof(code)) != cudaSuccess ||
      cudaMemcpyFromSymbol(&w, svdq::g_status_where, sizeof(w)) != cudaSuccess)
    return SVDQ_ERR_CUDA;
  if (code != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(svdq::g_status_code, &zero, sizeof(zero)) != cudaSuccess ||
        cudaMemcpyToSymbol(svdq::g_status_where, &zero, sizeof(zero)) != cudaSuccess)
      return SVDQ_ERR_CUDA;
    if (where) *where = static_cast<int>(w);
    return static_cast<int>(code);
  }
  return SVDQ_OK;
}

int svdq_selftest_wait_timeout(uint64_t timeout_ns, void* stream) {
  if (timeout_ns == 0 || timeout_ns > 10000000000ull) return SVDQ_ERR_INVALID_ARG;
  svdq::wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(timeout_ns);
  return launch_status();
}

}  // extern "C"
