// C ABI of the SVDQuant W4A4 linear layer (include/svdq.h): argument
// validation, TMA tensor maps and kernel launches.  Host code only launches
// the kernels of the headers below; no step of the layer runs on the host.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <unordered_map>

#include "../../include/svdq.h"
#include "calib.cuh"
#include "linear.cuh"
#include "linear_splitk.cuh"
#include "lora.cuh"
#include "pack_residual.cuh"
#include "quantize_act.cuh"

namespace {

// ------------------------------------------------------------- limits --
// Rows (M, N) up to 2^22 and K up to 2^20 keep every grid dimension, tile
// count and 32-bit index product of the kernels in range.
constexpr int64_t kMaxRows = int64_t(1) << 22;
constexpr int64_t kMaxK = int64_t(1) << 20;

// Which linear kernel svdq_linear launches: 0 picks by shape, 1 forces the
// large-M kernel, 2 the small-M kernel (svdq_set_linear_path).
std::atomic<int> g_linear_path{0};

// Whether the layer's launches carry the programmatic stream-serialisation
// attribute (svdq_set_launch_overlap; default on).  With it a layer kernel
// may be scheduled while the kernel ahead of it in the stream finishes; it
// sets up (barriers, tensor memory, L2 prefetch of weights) and then waits
// in-kernel for that kernel before it touches anything it could share with it.
std::atomic<int> g_overlap{1};

// Appends the overlap attribute to attrs[n] when the setting is on.
unsigned add_overlap_attr(cudaLaunchAttribute* attrs, unsigned n) {
  if (!g_overlap.load(std::memory_order_relaxed)) return n;
  attrs[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[n].val.programmaticStreamSerializationAllowed = 1;
  return n + 1;
}

// -------------------------------------------------------- wait timeout --
std::atomic<uint64_t> g_timeout_ns{0};

uint64_t wait_timeout_ns() {
  uint64_t t = g_timeout_ns.load(std::memory_order_relaxed);
  if (t == 0) {
    uint64_t ms = 2000;
    if (const char* e = std::getenv("SVDQ_WAIT_TIMEOUT_MS")) {
      long long v = std::atoll(e);
      if (v > 0) ms = static_cast<uint64_t>(v);
    }
    t = ms * 1000000ull;
    uint64_t expected = 0;
    if (!g_timeout_ns.compare_exchange_strong(expected, t)) t = expected;
  }
  return t;
}

// --------------------------------------------------------- tensor maps --
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}

// A tensor map is a pure function of its encoding parameters (the global
// address among them), so encoded maps are kept in a small cache keyed by
// all of them: a call whose buffers and shapes repeat an earlier call's
// reuses the earlier encoding instead of encoding again.
struct MapKey {
  uint64_t words[12];
  bool operator==(const MapKey& o) const { return std::memcmp(words, o.words, sizeof(words)) == 0; }
};
struct MapKeyHash {
  size_t operator()(const MapKey& k) const {
    uint64_t h = 1469598103934665603ull;
    for (uint64_t w : k.words) {
      h ^= w;
      h *= 1099511628211ull;
    }
    return static_cast<size_t>(h);
  }
};
constexpr size_t kMapCacheCap = 4096;
std::mutex g_map_mu;
std::unordered_map<MapKey, CUtensorMap, MapKeyHash> g_maps;

// 2D/3D tiled tensor map; dims/strides innermost first, strides in bytes.
svdq_status make_tmap(CUtensorMap* map, CUtensorMapDataType dtype, uint32_t rank, const void* base,
                      const uint64_t* dims, const uint64_t* strides, const uint32_t* box,
                      CUtensorMapSwizzle swizzle) {
  MapKey key;
  std::memset(&key, 0, sizeof(key));
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SVDQ_ERR_CUDA;
  key.words[0] = static_cast<uint64_t>(dtype) | (static_cast<uint64_t>(rank) << 8) |
                 (static_cast<uint64_t>(swizzle) << 16) | (static_cast<uint64_t>(dev) << 32);
  key.words[1] = reinterpret_cast<uintptr_t>(base);
  for (uint32_t i = 0; i < rank; ++i) {
    key.words[2 + i] = dims[i];
    key.words[5 + i] = box[i];
    if (i + 1 < rank) key.words[8 + i] = strides[i];
  }
  {
    std::lock_guard<std::mutex> lock(g_map_mu);
    auto it = g_maps.find(key);
    if (it != g_maps.end()) {
      *map = it->second;
      return SVDQ_OK;
    }
  }
  auto enc = encode_fn();
  if (!enc) return SVDQ_ERR_CUDA;
  uint32_t estr[3] = {1, 1, 1};
  CUresult rc = enc(map, dtype, rank, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (rc != CUDA_SUCCESS) return SVDQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_map_mu);
  if (g_maps.size() >= kMapCacheCap) g_maps.clear();
  g_maps.emplace(key, *map);
  return SVDQ_OK;
}

// ---------------------------------------------------- device properties --
constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];

int current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  return dev;
}

int sm_count(int dev) {
  int n = g_sm_count[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    g_sm_count[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

// The largest dynamic shared memory size set so far, per (kernel, device):
// cudaFuncSetAttribute runs once per kernel and device unless a launch needs
// more than any earlier one.
std::mutex g_attr_mu;
std::unordered_map<uint64_t, int> g_smem_set;

svdq_status ensure_smem(const void* kern, int dev, size_t bytes) {
  const uint64_t key = (reinterpret_cast<uintptr_t>(kern) << 8) ^ static_cast<uint64_t>(dev);
  std::lock_guard<std::mutex> lock(g_attr_mu);
  auto it = g_smem_set.find(key);
  if (it != g_smem_set.end() && static_cast<size_t>(it->second) >= bytes) return SVDQ_OK;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes)) !=
      cudaSuccess)
    return SVDQ_ERR_CUDA;
  g_smem_set[key] = static_cast<int>(bytes);
  return SVDQ_OK;
}

// Dynamic shared memory per CTA such that CTAs that each allocate
// `tmem_cols` tensor-memory columns never oversubscribe the SM's 512: the
// request is raised until shared memory alone admits no more CTAs per SM
// than the tensor memory does.  (A CTA blocked in tcgen05.alloc behind a CTA
// of its own cluster would wait for it forever.)
size_t smem_for_tmem(int dev, size_t smem, uint32_t tmem_cols) {
  if (tmem_cols == 0) return smem;
  int per_sm = 0, reserved = 0;
  if (cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess)
    return 0;
  const size_t allowed = 512 / tmem_cols;
  const size_t floor_bytes = static_cast<size_t>(per_sm) / (allowed + 1) + 1;  // > per_sm / (allowed + 1)
  if (smem + static_cast<size_t>(reserved) < floor_bytes) smem = floor_bytes - static_cast<size_t>(reserved);
  return smem;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_rank(int64_t r) { return r >= 0 && r <= 128 && r % 16 == 0; }

svdq_status launch_status() { return cudaGetLastError() == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA; }

uint32_t pow2_at_least(uint32_t x) {
  uint32_t p = 32;
  while (p < x) p <<= 1;
  return p;
}

// Work split of the activation step: 128-row tiles; when they are fewer
// than the SMs, the 64-column atoms of K are split over up to 16 CTAs per
// tile (no CTA without atoms).
struct QaPlan {
  int64_t row_tiles;
  int splits, apc;
};

QaPlan qa_plan(int64_t M, int64_t K, int sms) {
  QaPlan pl;
  pl.row_tiles = (M + svdq::kQaRows - 1) / svdq::kQaRows;
  const int atoms = static_cast<int>(K / 64);
  int splits = 1;
  if (pl.row_tiles < sms) {
    splits = static_cast<int>(sms / pl.row_tiles);
    if (splits > svdq::kQaMaxSplits) splits = svdq::kQaMaxSplits;
    if (splits > atoms) splits = atoms;
    if (splits < 1) splits = 1;
  }
  pl.apc = (atoms + splits - 1) / splits;
  pl.splits = (atoms + pl.apc - 1) / pl.apc;
  return pl;
}

// Small-M linear: 128 x 128 tiles, K stages split over a cluster.  The
// split minimises the stages the busiest SM runs (tiles x splits CTAs over
// the SMs, each CTA ceil(stages / splits) stages, plus one for the cluster's
// reduction), the smaller split on ties.
svdq_status launch_linear_splitk(const CUtensorMap& tm_xc, const CUtensorMap& tm_rc, const CUtensorMap& tm_xs,
                                 const CUtensorMap& tm_rs, const CUtensorMap& tm_t, const CUtensorMap& tm_l2,
                                 const void* bias, void* Y, int64_t M, int64_t K, int64_t N, int64_t r, float alpha,
                                 int dev, int sms, void* stream) {
  const int64_t tiles_m = (M + svdq::kLsBM - 1) / svdq::kLsBM;
  const int64_t tiles_n = (N + svdq::kLsBN - 1) / svdq::kLsBN;
  const int64_t tiles = tiles_m * tiles_n;
  const int n_k = static_cast<int>((K + svdq::kLsBK - 1) / svdq::kLsBK);
  const int n_lr = static_cast<int>((r + 63) / 64);
  int best_s = 1;
  int64_t best_cost = -1;
  for (int s = 1; s <= svdq::kLsMaxSplits && s <= n_k; ++s) {
    const int spc = (n_k + s - 1) / s;
    const int se = (n_k + spc - 1) / spc;
    if (se != s) continue;
    const int64_t cost = ((tiles * se + sms - 1) / sms) * (spc + n_lr) + (se > 1 ? 1 : 0);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best_s = s;
    }
  }
  const int splits = best_s;
  const int spc = (n_k + splits - 1) / splits;
  int stages = spc + n_lr;
  if (stages > svdq::kLsMaxStages) stages = svdq::kLsMaxStages;
  uint32_t ring = static_cast<uint32_t>(stages) * svdq::kLsStageBytes;
  if (splits > 1 && ring < svdq::kLsPartBytes) ring = svdq::kLsPartBytes;
  const size_t smem = smem_for_tmem(dev, 1024 + svdq::kLsHeadBytes + ring, svdq::kLsTmemCols);
  if (smem == 0 || smem > 232448) return SVDQ_ERR_CUDA;
  const void* kern = reinterpret_cast<const void*>(svdq::linear_splitk_kernel);
  if (svdq_status rc = ensure_smem(kern, dev, smem)) return rc;

  svdq::LsParams p;
  p.bias = static_cast<const __nv_bfloat16*>(bias);
  p.Y = static_cast<__nv_bfloat16*>(Y);
  p.alpha = alpha;
  p.M = static_cast<int>(M);
  p.K = static_cast<int>(K);
  p.N = static_cast<int>(N);
  p.r = static_cast<int>(r);
  p.splits = splits;
  p.spc = spc;
  p.stages = stages;
  p.timeout_ns = wait_timeout_ns();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(splits), static_cast<unsigned>(tiles_n), static_cast<unsigned>(tiles_m));
  cfg.blockDim = dim3(svdq::kLsThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[2];
  unsigned na = 0;
  if (splits > 1) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(splits);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    na = 1;
  }
  cfg.attrs = attr;
  cfg.numAttrs = add_overlap_attr(attr, na);
  if (cudaLaunchKernelEx(&cfg, svdq::linear_splitk_kernel, tm_xc, tm_rc, tm_xs, tm_rs, tm_t, tm_l2, p) !=
      cudaSuccess)
    return SVDQ_ERR_CUDA;
  return launch_status();
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

svdq_status svdq_packed_sizes(int64_t rows, int64_t K, size_t* codes_bytes, size_t* scales_bytes) {
  if (rows < 0 || K <= 0 || !codes_bytes || !scales_bytes) return SVDQ_ERR_INVALID_ARG;
  if (K % 64 != 0 || K > kMaxK || rows > kMaxRows) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  *codes_bytes = static_cast<size_t>(rows) * static_cast<size_t>(K / 2);
  *scales_bytes = static_cast<size_t>((rows + 127) / 128) * 128 * static_cast<size_t>(K / 16);
  return SVDQ_OK;
}

svdq_status svdq_pack_residual(const float* R, int64_t K, int64_t N, uint8_t* r_codes, uint8_t* r_scales,
                               void* stream) {
  if (!R || !r_codes || !r_scales || K <= 0 || N <= 0) return SVDQ_ERR_INVALID_ARG;
  if (K % 64 != 0 || N % 16 != 0 || K > kMaxK || N > kMaxRows) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(R) || !aligned16(r_codes) || !aligned16(r_scales)) return SVDQ_ERR_MISALIGNED;
  dim3 grid(static_cast<unsigned>((N + 127) / 128), static_cast<unsigned>(K / 64));
  svdq::pack_residual_kernel<<<grid, svdq::kPackThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      R, static_cast<int>(K), static_cast<int>(N), r_codes, r_scales);
  return launch_status();
}

svdq_status svdq_quantize_act_workspace(int64_t M, int64_t K, int64_t r, size_t* bytes) {
  if (!bytes || M <= 0 || K <= 0) return SVDQ_ERR_INVALID_ARG;
  if (K % 64 != 0 || !valid_rank(r) || M > kMaxRows || K > kMaxK) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  const int dev = current_device();
  if (dev < 0) return SVDQ_ERR_CUDA;
  const int sms = sm_count(dev);
  if (sms <= 0) return SVDQ_ERR_CUDA;
  const QaPlan pl = qa_plan(M, K, sms);
  *bytes = svdq::qa_workspace_bytes(pl.row_tiles, pl.splits, static_cast<int>(r));
  return SVDQ_OK;
}

namespace {
svdq_status quantize_act_impl(const void* X, const float* inv_lambda, const void* L1, int64_t M, int64_t K,
                              int64_t r, uint8_t* x_codes, uint8_t* x_scales, void* T, void* workspace,
                              size_t workspace_bytes, void* stream, bool gelu);
}  // namespace

svdq_status svdq_quantize_act(const void* X, const float* inv_lambda, const void* L1, int64_t M, int64_t K,
                              int64_t r, uint8_t* x_codes, uint8_t* x_scales, void* T, void* workspace,
                              size_t workspace_bytes, void* stream) {
  return quantize_act_impl(X, inv_lambda, L1, M, K, r, x_codes, x_scales, T, workspace, workspace_bytes, stream,
                           false);
}

svdq_status svdq_quantize_act_gelu(const void* X, const float* inv_lambda, const void* L1, int64_t M, int64_t K,
                                   int64_t r, uint8_t* x_codes, uint8_t* x_scales, void* T, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  return quantize_act_impl(X, inv_lambda, L1, M, K, r, x_codes, x_scales, T, workspace, workspace_bytes, stream,
                           true);
}

namespace {
svdq_status quantize_act_impl(const void* X, const float* inv_lambda, const void* L1, int64_t M, int64_t K,
                              int64_t r, uint8_t* x_codes, uint8_t* x_scales, void* T, void* workspace,
                              size_t workspace_bytes, void* stream, bool gelu) {
  if (!X || !inv_lambda || !x_codes || !x_scales || M <= 0 || K <= 0) return SVDQ_ERR_INVALID_ARG;
  if (r > 0 && (!L1 || !T)) return SVDQ_ERR_INVALID_ARG;
  if (K % 64 != 0 || !valid_rank(r) || M > kMaxRows || K > kMaxK) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(X) || !aligned16(inv_lambda) || !aligned16(x_codes) || !aligned16(x_scales) ||
      (r > 0 && (!aligned16(L1) || !aligned16(T))) || (workspace && !aligned16(workspace)))
    return SVDQ_ERR_MISALIGNED;
  const int dev = current_device();
  if (dev < 0) return SVDQ_ERR_CUDA;
  const int sms = sm_count(dev);
  if (sms <= 0) return SVDQ_ERR_CUDA;

  const QaPlan pl = qa_plan(M, K, sms);
  const int ri = static_cast<int>(r);
  const size_t ws_need = svdq::qa_workspace_bytes(pl.row_tiles, pl.splits, ri);
  if (ws_need > 0 && (!workspace || workspace_bytes < ws_need)) return SVDQ_ERR_INVALID_ARG;
  const int n_l1 = r == 0 ? 0 : (r <= 64 ? 1 : 2);
  const uint32_t stage_bytes = svdq::qa_stage_bytes(n_l1);
  const uint32_t fixed = 1024 + svdq::kQaHeadBytes;
  int stages = static_cast<int>((svdq::kQaSmemLimit - fixed) / stage_bytes);
  if (stages > svdq::kQaMaxStages) stages = svdq::kQaMaxStages;
  if (stages > pl.apc) stages = pl.apc;
  if (stages < 1) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  // tensor-memory accumulators of at least 8 atoms (512 columns of K) each,
  // within the SM's 512 columns
  const int n_acc_cols = 64 * n_l1;
  int fold = pl.apc;
  uint32_t tmem_cols = 0;
  if (r > 0) {
    const int max_acc = 512 / n_acc_cols;
    fold = 8;
    if ((pl.apc + fold - 1) / fold > max_acc) fold = (pl.apc + max_acc - 1) / max_acc;
    tmem_cols = pow2_at_least(static_cast<uint32_t>(((pl.apc + fold - 1) / fold) * n_acc_cols));
  }
  const size_t smem = smem_for_tmem(dev, fixed + static_cast<size_t>(stages) * stage_bytes, tmem_cols);
  if (smem == 0 || smem > svdq::kQaSmemLimit) return SVDQ_ERR_CUDA;
  auto kfn = gelu ? svdq::quantize_act_kernel<true> : svdq::quantize_act_kernel<false>;
  const void* kern = reinterpret_cast<const void*>(kfn);
  if (svdq_status rc = ensure_smem(kern, dev, smem)) return rc;

  CUtensorMap tm_x, tm_l1, tm_xc;
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(M)};
    const uint64_t strides[1] = {static_cast<uint64_t>(K) * 2};
    const uint32_t box[2] = {64, static_cast<uint32_t>(svdq::kQaRows)};
    svdq_status rc = make_tmap(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, X, dims, strides, box,
                               CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
  }
  {
    // codes [M][K/2]: one store box per atom, 32 bytes x 128 rows (rows past M clipped)
    const uint64_t dims[2] = {static_cast<uint64_t>(K / 2), static_cast<uint64_t>(M)};
    const uint64_t strides[1] = {static_cast<uint64_t>(K / 2)};
    const uint32_t box[2] = {32, static_cast<uint32_t>(svdq::kQaRows)};
    svdq_status rc = make_tmap(&tm_xc, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, x_codes, dims, strides, box,
                               CU_TENSOR_MAP_SWIZZLE_NONE);
    if (rc) return rc;
  }
  if (r > 0) {
    // L1 [K][r]: boxes of 64 k-rows x 64 ranks, 128-byte swizzle; ranks past
    // r arrive as zeros
    const uint64_t dims[2] = {static_cast<uint64_t>(r), static_cast<uint64_t>(K)};
    const uint64_t strides[1] = {static_cast<uint64_t>(r) * 2};
    const uint32_t box[2] = {64, 64};
    svdq_status rc = make_tmap(&tm_l1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, L1, dims, strides, box,
                               CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
  } else {
    std::memset(&tm_l1, 0, sizeof(tm_l1));
  }

  svdq::QaParams p;
  p.inv_lambda = inv_lambda;
  p.x_codes = x_codes;
  p.x_scales = x_scales;
  p.T = static_cast<__nv_bfloat16*>(T);
  p.counters = ws_need ? static_cast<unsigned int*>(workspace) : nullptr;
  p.partials = ws_need ? reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                                  svdq::kQaCounterBytes *
                                                      ((static_cast<size_t>(pl.row_tiles) * 4 +
                                                        svdq::kQaCounterBytes - 1) /
                                                       svdq::kQaCounterBytes))
                       : nullptr;
  p.M = static_cast<int>(M);
  p.K = static_cast<int>(K);
  p.r = ri;
  p.splits = pl.splits;
  p.apc = pl.apc;
  p.stages = stages;
  p.n_l1 = n_l1;
  p.fold = fold;
  p.stage_bytes = stage_bytes;
  p.tmem_cols = tmem_cols;
  p.timeout_ns = wait_timeout_ns();

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(pl.splits), static_cast<unsigned>(pl.row_tiles));
  cfg.blockDim = dim3(svdq::kQaThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  cfg.attrs = attr;
  cfg.numAttrs = add_overlap_attr(attr, 0);
  if (cudaLaunchKernelEx(&cfg, kfn, tm_x, tm_l1, tm_xc, p) != cudaSuccess)
    return SVDQ_ERR_CUDA;
  return launch_status();
}
}  // namespace

svdq_status svdq_linear(const uint8_t* x_codes, const uint8_t* x_scales, const void* T, const uint8_t* r_codes,
                        const uint8_t* r_scales, const void* L2, const void* bias, int64_t M, int64_t K, int64_t N,
                        int64_t r, void* Y, void* stream) {
  return svdq_linear_scaled(x_codes, x_scales, T, r_codes, r_scales, L2, bias, M, K, N, r, 1.0f, Y, stream);
}

svdq_status svdq_linear_scaled(const uint8_t* x_codes, const uint8_t* x_scales, const void* T,
                               const uint8_t* r_codes, const uint8_t* r_scales, const void* L2, const void* bias,
                               int64_t M, int64_t K, int64_t N, int64_t r, float alpha, void* Y, void* stream) {
  // alpha: a power of two in [2^-100, 2^100] (the product acc * alpha is then exact)
  int alpha_exp = 0;
  if (!(alpha > 0.0f) || !std::isfinite(alpha) || std::frexp(alpha, &alpha_exp) != 0.5f || alpha_exp < -99 ||
      alpha_exp > 101)
    return SVDQ_ERR_INVALID_ARG;
  if (!x_codes || !x_scales || !r_codes || !r_scales || !Y || M <= 0 || K <= 0 || N <= 0)
    return SVDQ_ERR_INVALID_ARG;
  if (r > 0 && (!T || !L2)) return SVDQ_ERR_INVALID_ARG;
  if (K % 64 != 0 || N % 16 != 0 || !valid_rank(r) || M > kMaxRows || N > kMaxRows || K > kMaxK)
    return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(x_codes) || !aligned16(x_scales) || !aligned16(r_codes) || !aligned16(r_scales) ||
      !aligned16(Y) || (bias && !aligned16(bias)) || (r > 0 && (!aligned16(T) || !aligned16(L2))))
    return SVDQ_ERR_MISALIGNED;
  const int dev = current_device();
  if (dev < 0) return SVDQ_ERR_CUDA;
  const int sms = sm_count(dev);
  if (sms < 2) return SVDQ_ERR_CUDA;

  CUtensorMap tm_xc, tm_rc, tm_t, tm_l2;
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(K / 2), static_cast<uint64_t>(M)};
    const uint64_t strides[1] = {static_cast<uint64_t>(K / 2)};
    const uint32_t box[2] = {128, 128};
    svdq_status rc = make_tmap(&tm_xc, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, x_codes, dims, strides, box,
                               CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(K / 2), static_cast<uint64_t>(N)};
    const uint64_t strides[1] = {static_cast<uint64_t>(K / 2)};
    const uint32_t box[2] = {128, 128};  // each CTA of a pair loads 128 R rows
    svdq_status rc = make_tmap(&tm_rc, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, r_codes, dims, strides, box,
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
    svdq_status rc = make_tmap(&tm_xs, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, x_scales, dims, strides, box,
                               CU_TENSOR_MAP_SWIZZLE_NONE);
    if (rc) return rc;
  }
  {
    const uint64_t dims[3] = {256, 2, static_cast<uint64_t>((N + 127) / 128) * static_cast<uint64_t>(K / 64)};
    const uint64_t strides[2] = {256, 512};
    const uint32_t box[3] = {256, 2, 4};
    svdq_status rc = make_tmap(&tm_rs, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, r_scales, dims, strides, box,
                               CU_TENSOR_MAP_SWIZZLE_NONE);
    if (rc) return rc;
  }
  if (r > 0) {
    const uint64_t dt[2] = {static_cast<uint64_t>(r), static_cast<uint64_t>(M)};
    const uint64_t st[1] = {static_cast<uint64_t>(r) * 2};
    const uint32_t bt[2] = {64, 128};
    svdq_status rc = make_tmap(&tm_t, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, T, dt, st, bt, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
    const uint64_t dl[2] = {static_cast<uint64_t>(N), static_cast<uint64_t>(r)};
    const uint64_t sl[1] = {static_cast<uint64_t>(N) * 2};
    const uint32_t bl[2] = {64, 64};
    rc = make_tmap(&tm_l2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, L2, dl, sl, bl, CU_TENSOR_MAP_SWIZZLE_128B);
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
    svdq_status rc = make_tmap(&tm_y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Y, dims, strides, box,
                               CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
  }

  // At most 128 rows with tiles for under a quarter of the SMs: the large-M
  // kernel would leave most SMs idle, each busy pair walking all of K; the
  // small-M kernel splits K over a cluster instead.  Measured on B200
  // (K, N in {3072, 12288}): the small-M kernel is faster only there; from
  // 256 rows, or with N = 12288 at any M, the large-M kernel is.
  const int64_t pair_tiles = ((M + svdq::kLinBM - 1) / svdq::kLinBM) * ((N + svdq::kLinBN - 1) / svdq::kLinBN);
  const int path = g_linear_path.load(std::memory_order_relaxed);
  if (path == 2 || (path == 0 && M <= 128 && 4 * pair_tiles < sms))
    return launch_linear_splitk(tm_xc, tm_rc, tm_xs, tm_rs, tm_t, tm_l2, bias, Y, M, K, N, r, alpha, dev, sms,
                                stream);

  svdq::LinParams p;
  p.alpha = alpha;
  p.bias = static_cast<const __nv_bfloat16*>(bias);
  p.Y = static_cast<__nv_bfloat16*>(Y);
  p.M = static_cast<int>(M);
  p.K = static_cast<int>(K);
  p.N = static_cast<int>(N);
  p.r = static_cast<int>(r);
  p.timeout_ns = wait_timeout_ns();
  p.m_tiles = static_cast<int>((M + svdq::kLinBM - 1) / svdq::kLinBM);
  p.tiles = p.m_tiles * static_cast<int>((N + svdq::kLinBN - 1) / svdq::kLinBN);

  const size_t smem = 1024 + svdq::kLinBarOffset + (svdq::kLinNumBars + 4) * 8;
  const bool full_k = (K % svdq::kLinBK) == 0;
  auto kern = full_k ? svdq::linear_kernel<true> : svdq::linear_kernel<false>;
  if (svdq_status rc = ensure_smem(reinterpret_cast<const void*>(kern), dev, smem)) return rc;
  const int pairs = p.tiles < sms / 2 ? p.tiles : sms / 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
  cfg.blockDim = dim3(svdq::kLinThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = add_overlap_attr(attr, 1);
  if (cudaLaunchKernelEx(&cfg, kern, tm_xc, tm_rc, tm_xs, tm_rs, tm_t, tm_l2, tm_y, p) != cudaSuccess)
    return SVDQ_ERR_CUDA;
  return launch_status();
}

svdq_status svdq_attach_lora(const void* L1, const void* L2, const float* lambda, const void* A, const void* B,
                             int64_t K, int64_t N, int64_t r, int64_t ra, void* L1_out, void* L2_out, void* stream) {
  if (!lambda || !A || !B || !L1_out || !L2_out || K <= 0 || N <= 0 || r < 0 || ra <= 0)
    return SVDQ_ERR_INVALID_ARG;
  if (r > 0 && (!L1 || !L2)) return SVDQ_ERR_INVALID_ARG;
  if (r % 16 != 0 || ra % 16 != 0 || r + ra > 128 || N % 16 != 0 || K > kMaxK || N > kMaxRows)
    return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if ((r > 0 && (!aligned16(L1) || !aligned16(L2))) || !aligned16(lambda) || !aligned16(A) || !aligned16(B) ||
      !aligned16(L1_out) || !aligned16(L2_out))
    return SVDQ_ERR_MISALIGNED;
  const int dev = current_device();
  if (dev < 0) return SVDQ_ERR_CUDA;
  const int sms = sm_count(dev);
  if (sms <= 0) return SVDQ_ERR_CUDA;
  const int64_t chunks = K * ((r + ra) / 8) + (r + ra) * N / 8;
  int64_t blocks = (chunks + svdq::kLoraThreads - 1) / svdq::kLoraThreads;
  if (blocks > 8 * sms) blocks = 8 * sms;
  svdq::attach_lora_kernel<<<static_cast<unsigned>(blocks), svdq::kLoraThreads, 0,
                             static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(L1), static_cast<const __nv_bfloat16*>(L2), lambda,
      static_cast<const __nv_bfloat16*>(A), static_cast<const __nv_bfloat16*>(B), static_cast<int>(K),
      static_cast<int>(N), static_cast<int>(r), static_cast<int>(ra), static_cast<__nv_bfloat16*>(L1_out),
      static_cast<__nv_bfloat16*>(L2_out));
  return launch_status();
}

svdq_status svdq_channel_absmax(const void* X, int64_t M, int64_t K, float* amax, void* stream) {
  if (!X || !amax || M <= 0 || K <= 0) return SVDQ_ERR_INVALID_ARG;
  if (K % 8 != 0 || K > kMaxK || M > kMaxRows) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(X) || !aligned16(amax)) return SVDQ_ERR_MISALIGNED;
  const int dev = current_device();
  if (dev < 0) return SVDQ_ERR_CUDA;
  const int sms = sm_count(dev);
  if (sms <= 0) return SVDQ_ERR_CUDA;
  // enough row ranges for about four blocks per SM, at least 32 rows each
  const int64_t col_blocks = (K / 8 + svdq::kAbsmaxThreads - 1) / svdq::kAbsmaxThreads;
  int64_t row_blocks = (4 * static_cast<int64_t>(sms) + col_blocks - 1) / col_blocks;
  if (row_blocks > (M + 31) / 32) row_blocks = (M + 31) / 32;
  if (row_blocks > 65535) row_blocks = 65535;
  const int64_t rows_per_block = (M + row_blocks - 1) / row_blocks;
  row_blocks = (M + rows_per_block - 1) / rows_per_block;
  const dim3 grid(static_cast<unsigned>(col_blocks), static_cast<unsigned>(row_blocks));
  svdq::channel_absmax_kernel<<<grid, svdq::kAbsmaxThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(X), static_cast<int>(M), static_cast<int>(K),
      static_cast<int>(rows_per_block), reinterpret_cast<unsigned int*>(amax));
  return launch_status();
}

svdq_status svdq_sync_status(void* stream, int* where) {
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
    return static_cast<svdq_status>(code);
  }
  return SVDQ_OK;
}

svdq_status svdq_set_wait_timeout(uint64_t timeout_ns) {
  if (timeout_ns == 0 || timeout_ns > 60000000000ull) return SVDQ_ERR_INVALID_ARG;
  g_timeout_ns.store(timeout_ns, std::memory_order_relaxed);
  return SVDQ_OK;
}

svdq_status svdq_set_linear_path(int path) {
  if (path < 0 || path > 2) return SVDQ_ERR_INVALID_ARG;
  g_linear_path.store(path, std::memory_order_relaxed);
  return SVDQ_OK;
}

svdq_status svdq_set_launch_overlap(int enable) {
  if (enable != 0 && enable != 1) return SVDQ_ERR_INVALID_ARG;
  g_overlap.store(enable, std::memory_order_relaxed);
  return SVDQ_OK;
}

svdq_status svdq_selftest_wait_timeout(uint64_t timeout_ns, void* stream) {
  if (timeout_ns == 0 || timeout_ns > 10000000000ull) return SVDQ_ERR_INVALID_ARG;
  svdq::wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(timeout_ns);
  return launch_status();
}

// ------------------------------------------------ allocation-free variant --
// svdq_quantize_act with its scratch in a fixed array of this library instead
// of a caller's buffer, for callers that can neither allocate device memory
// nor pass scratch (see include/svdq.h).  Every device that loads the library
// holds the array until the process exits.
}  // extern "C"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on `dev` (the current device), set up
// on the first call there: the array's host-side name is only a stand-in, so
// the address comes from cudaGetSymbolAddress with the device current, and the
// array is zero-filled once (the counters of the partial-sum exchange must
// start at zero; every call leaves them at zero again).
svdq_status noalloc_scratch(int dev, void** ptr) {
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return SVDQ_ERR_CUDA;
    if (cudaMemset(p, 0, kNoAllocScratchBytes) != cudaSuccess) return SVDQ_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *ptr = g_noalloc_ptr[dev];
  return SVDQ_OK;
}

}  // namespace

extern "C" {

svdq_status svdq_quantize_act_noalloc(const void* X, const float* inv_lambda, const void* L1, int64_t M, int64_t K,
                                      int64_t r, uint8_t* x_codes, uint8_t* x_scales, void* T, void* stream) {
  size_t need = 0;
  if (svdq_status rc = svdq_quantize_act_workspace(M, K, r, &need)) return rc;
  if (need > kNoAllocScratchBytes) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  void* scratch = nullptr;
  if (need > 0) {
    const int dev = current_device();
    if (dev < 0) return SVDQ_ERR_CUDA;
    if (svdq_status rc = noalloc_scratch(dev, &scratch)) return rc;
  }
  return svdq_quantize_act(X, inv_lambda, L1, M, K, r, x_codes, x_scales, T, scratch, need ? kNoAllocScratchBytes : 0,
                           stream);
}

}  // extern "C"
