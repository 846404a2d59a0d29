// C-ABI entry points (include/coda.h): argument validation, workspace carving,
// TMA tensor-map encoding and the launch sequence of each fused pass.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <initializer_list>

#include "coda.h"
#include "coda_aux.cuh"
#include "coda_gemm.cuh"
#include "coda_unfused.cuh"

namespace coda {
namespace {

constexpr size_t kStatusBytes = 256;
std::atomic<unsigned long long> g_wait_limit_ns{4000000000ull};

// One-shot event pairs armed by coda_profile_arm, per host thread, in arming order.
struct ProfileSlot {
  int kernel;
  cudaEvent_t start, stop;
};
constexpr int kProfileSlots = 16;
thread_local ProfileSlot g_prof[kProfileSlots];
thread_local int g_prof_n = 0;
thread_local int g_launch_tag = -1;  // the GEMM launcher's epilogue id around its launch

// Remove and return the first pair armed for kernel id `tag`.
bool profile_take(int tag, cudaEvent_t& start, cudaEvent_t& stop) {
  for (int i = 0; i < g_prof_n; ++i) {
    if (g_prof[i].kernel != tag) continue;
    start = g_prof[i].start;
    stop = g_prof[i].stop;
    for (int j = i + 1; j < g_prof_n; ++j) g_prof[j - 1] = g_prof[j];
    --g_prof_n;
    return true;
  }
  return false;
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int cdiv(long long a, long long b) { return (int)((a + b - 1) / b); }

// ------------------------------------------------------------------ device checks

constexpr int kKernelSlots = 64;  // (EPI, A major, B major, pair) instantiations: (7 * 4) * 2
struct DevInfo {
  int num_sms = 0;
  int major = 0;
  bool configured[kKernelSlots] = {};
  int max_clusters[kKernelSlots] = {};
};
constexpr int kMaxDevices = 64;  // device ordinals the per-device tables cover
DevInfo g_dev[kMaxDevices];

int g_last_sms = 148;
int num_sms() { return g_last_sms; }
// Grid for grid-stride elementwise kernels over n_vec8 8-element vectors.
inline int ew_grid(long long n_vec8) { return (int)std::min<long long>(cdiv(n_vec8, 256), (long long)num_sms() * 16); }

coda_status current_device(int& dev) {
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CODA_ERR_CUDA;
  DevInfo& di = g_dev[dev];
  if (di.num_sms == 0) {
    int sms = 0, major = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return CODA_ERR_CUDA;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return CODA_ERR_CUDA;
    di.major = major;
    di.num_sms = sms;
  }
  if (di.major != 10) return CODA_ERR_NO_SM100;
  g_last_sms = di.num_sms;
  return CODA_OK;
}

// ------------------------------------------------------------------ tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// Encoded tensor maps, cached per host thread.  A map is a pure function of
// the arguments below, so a hit returns exactly what encoding would, and a
// repeated launch over the same tensors skips the driver call.
struct TmapKey {
  const void* base;
  long long rows, cols;
  int box_cols, box_rows, swizzle;
  bool operator==(const TmapKey& o) const {
    return base == o.base && rows == o.rows && cols == o.cols && box_cols == o.box_cols &&
           box_rows == o.box_rows && swizzle == o.swizzle;
  }
};
struct TmapSlot {
  TmapKey key;
  CUtensorMap map;
  bool valid;
};
constexpr int kTmapCacheSlots = 64;
thread_local TmapSlot t_tmap_cache[kTmapCacheSlots];

int tmap_slot(const TmapKey& k) {
  uint64_t h = reinterpret_cast<uintptr_t>(k.base) >> 4;
  for (uint64_t v : {(uint64_t)k.rows, (uint64_t)k.cols, (uint64_t)k.box_cols, (uint64_t)k.box_rows,
                     (uint64_t)k.swizzle})
    h = (h ^ v) * 0x9E3779B97F4A7C15ull;
  return (int)((h >> 32) % kTmapCacheSlots);
}

// Row-major bf16 matrix [rows][cols] (cols contiguous), swizzled boxes of
// box_cols x box_rows (128-byte swizzle unless given); out-of-range elements
// load as zero and are not written by stores.
bool make_tmap(CUtensorMap* m, const void* base, long long rows, long long cols, int box_cols, int box_rows,
               CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  const TmapKey key{base, rows, cols, box_cols, box_rows, (int)swizzle};
  TmapSlot& slot = t_tmap_cache[tmap_slot(key)];
  if (slot.valid && slot.key == key) {
    *m = slot.map;
    return true;
  }
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  slot.key = key;
  slot.map = *m;
  slot.valid = true;
  return true;
}

// Operand with logical shape [mn, k].  K-major storage is [mn][k]; MN-major
// storage is [k][mn].  box_mn is the tile extent along mn for K-major maps.
bool make_operand_map(CUtensorMap* m, const void* base, long long mn, long long k, bool mn_major, int box_mn) {
  if (!mn_major) return make_tmap(m, base, mn, k, BK, box_mn);
  return make_tmap(m, base, k, mn, 64, BK);
}

// ------------------------------------------------------------------ GEMM launch

// CTA-pair (cta_group::2, 256-row tiles) is the default GEMM mode; setting
// the environment variable CODA_CTA_PAIR=0 selects one 128-row tile per CTA.
bool use_pair() {
  static const bool v = [] {
    const char* e = std::getenv("CODA_CTA_PAIR");
    return !(e != nullptr && e[0] == '0');
  }();
  return v;
}
inline int tile_m(bool pair) { return pair ? 256 : 128; }

// Programmatic dependent launch between the kernels of a pass (each kernel
// waits for its predecessor with griddepcontrol.wait before touching global
// memory); CODA_PDL=0 turns it off.
bool use_pdl() {
  static const bool v = [] {
    const char* e = std::getenv("CODA_PDL");
    return !(e != nullptr && e[0] == '0');
  }();
  return v;
}

// Timing-hook id of a light-pass kernel (-1 for kernels the hook does not name).
template <typename Fn>
int aux_tag(Fn kern) {
  const void* f = reinterpret_cast<const void*>(kern);
  if (f == reinterpret_cast<const void*>(fold_gain_kernel)) return CODA_KERNEL_FOLD_GAIN;
  if (f == reinterpret_cast<const void*>(swiglu_bwd_rowstat_kernel)) return CODA_KERNEL_SWIGLU_BWD_ROWSTAT;
  if (f == reinterpret_cast<const void*>(col_reduce_kernel)) return CODA_KERNEL_COL_REDUCE;
  if (f == reinterpret_cast<const void*>(rowcoef_reduce_kernel)) return CODA_KERNEL_ROWCOEF_REDUCE;
  if (f == reinterpret_cast<const void*>(xent_reduce_kernel)) return CODA_KERNEL_XENT_REDUCE;
  if (f == reinterpret_cast<const void*>(rope_unrotate_kernel)) return CODA_KERNEL_ROPE_UNROTATE;
  return -1;
}

// Launch with the optional cluster size and the PDL attribute, inside the
// timing hook's event pair when one is armed for this kernel.
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, int cluster,
                      Args&&... args) {
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (cluster > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  if (use_pdl()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = n;
  cudaEvent_t ev0 = nullptr, ev1 = nullptr;
  const bool timed = g_prof_n > 0 && profile_take(g_launch_tag >= 0 ? g_launch_tag : aux_tag(kern), ev0, ev1);
  if (timed) {
    const cudaError_t e = cudaEventRecord(ev0, s);
    if (e != cudaSuccess) return e;
  }
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
  if (timed && e == cudaSuccess) e = cudaEventRecord(ev1, s);
  return e;
}

// Rasterisation.  Concurrent tiles read the same k-slices at about the same
// time, so a wave of gm x gn tiles reads gm A tiles and gn B tiles from HBM.
// The operand with the smaller total is kept resident across waves: its group
// (row tiles for A, column tiles for B) holds ~32 MiB (CODA_RASTER_MB
// overrides), and is at least sqrt(concurrent tiles) wide so each wave is
// close to square; the other operand streams through once per group.
int raster_budget_mb() {
  static const int v = [] {
    const char* e = std::getenv("CODA_RASTER_MB");
    const int x = e ? std::atoi(e) : 0;
    return x > 0 ? x : 32;
  }();
  return v;
}
int pick_group(long long a_rows, long long b_rows, long long K, int num_m, int num_n, bool pair, int num_sms) {
  const int units = pair ? num_sms / 2 : num_sms;
  int side = 1;
  while (side * side < units) ++side;
  const long long budget = (long long)raster_budget_mb() << 20;
  if (a_rows <= b_rows) {
    const long long tile_bytes = (long long)tile_m(pair) * K * 2;
    const long long g = std::max<long long>(side, budget / std::max(tile_bytes, 1LL));
    return (int)std::min<long long>(num_m, g);
  }
  const long long tile_bytes = (long long)BN * K * 2;
  const long long g = std::max<long long>(side, budget / std::max(tile_bytes, 1LL));
  return -(int)std::min<long long>(num_n, g);
}

template <int EPI, bool A_MN, bool B_MN, bool PAIR>
coda_status launch_gemm_mode(const CUtensorMap& ta, const CUtensorMap& tb, GemmParams p, cudaStream_t s) {
  using C = TileCfg<PAIR>;
  int dev = 0;
  coda_status st = current_device(dev);
  if (st != CODA_OK) return st;
  auto kern = gemm_tc_kernel<EPI, A_MN, B_MN, PAIR>;
  const int slot = ((EPI * 4 + (A_MN ? 2 : 0) + (B_MN ? 1 : 0)) * 2) + (PAIR ? 1 : 0);
  static_assert(((EPI * 4 + 3) * 2 + 1) < kKernelSlots, "kernel slot table too small");
  DevInfo& di = g_dev[dev];
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C::CTAS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = PAIR ? 1 : 0;
  if (!di.configured[slot]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
      return CODA_ERR_CUDA;
    int clusters = di.num_sms / C::CTAS;
    if (PAIR) {
      cfg.gridDim = dim3(2 * clusters, 1, 1);
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n > 0) clusters = std::min(clusters, n);
    }
    di.max_clusters[slot] = clusters;
    di.configured[slot] = true;
  }
  // Output maps for the epilogue's tile stores: 32 x 32 boxes, 64-byte swizzle
  // (the staging layout).  The second output (a/b or Hg) shares the rows.
  CUtensorMap to1, to2;
  std::memset(&to1, 0, sizeof(to1));
  std::memset(&to2, 0, sizeof(to2));
  if (p.out != nullptr && !make_tmap(&to1, p.out, p.M, p.ldo, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
    return CODA_ERR_CUDA;
  const int ld2 = (EPI == EPI_SWIGLU) ? p.ldo2 : p.ldo;
  if (p.out2 != nullptr && !make_tmap(&to2, p.out2, p.M, ld2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
    return CODA_ERR_CUDA;
  p.kernel_id = (uint32_t)(slot + 1);
  p.wait_limit_ns = g_wait_limit_ns.load();
  if (p.group_m == 0) p.group_m = 1;
  const int tiles = p.num_m_tiles * p.num_n_tiles;
  const int units = std::min(tiles, di.max_clusters[slot]);  // persistent: one tile stream per CTA (pair)
  if (units <= 0) return CODA_OK;
  g_launch_tag = EPI;
  const cudaError_t e =
      launch_ex(kern, dim3(units * C::CTAS), dim3(NUM_THREADS), C::SMEM_BYTES, s, C::CTAS, ta, tb, to1, to2, p);
  g_launch_tag = -1;
  if (e != cudaSuccess) return CODA_ERR_CUDA;
  return cudaPeekAtLastError() == cudaSuccess ? CODA_OK : CODA_ERR_CUDA;
}

template <int EPI, bool A_MN, bool B_MN>
coda_status launch_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const GemmParams& p, cudaStream_t s,
                        bool pair) {
  return pair ? launch_gemm_mode<EPI, A_MN, B_MN, true>(ta, tb, p, s)
              : launch_gemm_mode<EPI, A_MN, B_MN, false>(ta, tb, p, s);
}

GemmParams base_params(int M, int N, int K, int tile_n, void* ws, bool pair) {
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  p.M = M;
  p.N = N;
  p.K = K;
  p.num_m_tiles = cdiv(M, tile_m(pair));
  p.num_n_tiles = cdiv(N, tile_n);
  p.k_blocks = cdiv(K, BK);
  p.status = static_cast<uint32_t*>(ws);
  return p;
}

inline __nv_bfloat16* bf(void* p) { return static_cast<__nv_bfloat16*>(p); }
inline const __nv_bfloat16* cbf(const void* p) { return static_cast<const __nv_bfloat16*>(p); }

// Plain C = op(A) op(B)^T with the EPI_STORE epilogue (optional column scale).
coda_status gemm_store(const void* A, const void* B, void* C, int M, int N, int K, bool a_mn, bool b_mn,
                       const void* colscale, void* ws, cudaStream_t s) {
  const bool pair = use_pair();
  CUtensorMap ta, tb;
  if (!make_operand_map(&ta, A, M, K, a_mn, BM) || !make_operand_map(&tb, B, N, K, b_mn, pair ? BN / 2 : BN))
    return CODA_ERR_CUDA;
  GemmParams p = base_params(M, N, K, BN, ws, pair);
  p.group_m = pick_group(M, N, K, p.num_m_tiles, p.num_n_tiles, pair, num_sms());
  p.out = bf(C);
  p.ldo = N;
  p.colvec = cbf(colscale);
  if (!a_mn && !b_mn) return launch_gemm<EPI_STORE, false, false>(ta, tb, p, s, pair);
  if (!a_mn && b_mn) return launch_gemm<EPI_STORE, false, true>(ta, tb, p, s, pair);
  if (a_mn && b_mn) return launch_gemm<EPI_STORE, true, true>(ta, tb, p, s, pair);
  return launch_gemm<EPI_STORE, true, false>(ta, tb, p, s, pair);
}

coda_status launch_status(cudaError_t e) { return e == cudaSuccess ? CODA_OK : CODA_ERR_CUDA; }

// The RMSNorm row scale's source for the gate/up GEMM: the partial sums of
// squares P [M, T] of GEMM1's epilogue, from which the epilogue forms r and
// stores it to r_out (the block's forward, no separate row reduce).
struct RowScaleFromPartials {
  const float* P;
  int T;
  float inv_d, eps;
  float* r_out;
};

// Gate/up GEMM with the row-scale + SwiGLU epilogue: r from `rs` when given,
// else read from r (which may be null: no row scale).
coda_status gemm_swiglu(const void* A, const void* Wgu, const float* r, void* Y, void* AB, int M, int K, int F,
                        void* ws, cudaStream_t s, const RowScaleFromPartials* rs = nullptr) {
  CUtensorMap ta, tb;
  if (!make_operand_map(&ta, A, M, K, false, BM) || !make_operand_map(&tb, Wgu, 2LL * F, K, false, BN / 2))
    return CODA_ERR_CUDA;
  const bool pair = use_pair();
  GemmParams p = base_params(M, F, K, BN / 2, ws, pair);
  p.group_m = pick_group(M, 2LL * F, K, p.num_m_tiles, p.num_n_tiles, pair, num_sms());
  p.split = F;
  p.out = bf(Y);
  p.ldo = F;
  p.out2 = bf(AB);
  p.ldo2 = 2 * F;
  p.rowvec = r;
  if (rs != nullptr) {
    p.part = const_cast<float*>(rs->P);
    p.ld_part = rs->T;
    p.inv_d = rs->inv_d;
    p.eps = rs->eps;
    p.outf = rs->r_out;
  }
  return launch_gemm<EPI_SWIGLU, false, false>(ta, tb, p, s, pair);
}

}  // namespace
}  // namespace coda

using namespace coda;

#define CODA_TRY(expr)                 \
  do {                                 \
    coda_status _s = (expr);           \
    if (_s != CODA_OK) return _s;      \
  } while (0)

extern "C" {

const char* coda_status_string(int s) {
  switch (s) {
    case CODA_OK: return "ok";
    case CODA_ERR_INVALID_ARG: return "invalid argument";
    case CODA_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case CODA_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case CODA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case CODA_ERR_NO_SM100: return "device is not sm_100 (B200)";
    case CODA_ERR_CUDA: return "CUDA error";
    case CODA_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    default: return "unknown status";
  }
}

int coda_version(void) { return 100; }

void coda_set_wait_limit_ns(uint64_t ns) {
  ns = std::max<uint64_t>(ns, 1000ull);
  ns = std::min<uint64_t>(ns, 60000000000ull);
  g_wait_limit_ns.store(ns);
}

coda_status coda_profile_arm(int kernel, void* ev_start, void* ev_stop) {
  static_assert(CODA_EPI_STORE == EPI_STORE && CODA_EPI_RESID_RMS == EPI_RESID_RMS && CODA_EPI_SWIGLU == EPI_SWIGLU &&
                    CODA_EPI_DN == EPI_DN && CODA_EPI_SWIGLU_BWD == EPI_SWIGLU_BWD && CODA_EPI_XENT == EPI_XENT &&
                    CODA_EPI_XENT_BWD == EPI_XENT_BWD && CODA_EPI_ROPE == EPI_ROPE,
                "public epilogue ids");
  if (ev_start == nullptr && ev_stop == nullptr) {
    g_prof_n = 0;
    return CODA_OK;
  }
  const bool known = (kernel >= CODA_EPI_STORE && kernel <= CODA_EPI_ROPE) ||
                     (kernel >= CODA_KERNEL_FOLD_GAIN && kernel <= CODA_KERNEL_ROPE_UNROTATE);
  if (ev_start == nullptr || ev_stop == nullptr || !known || g_prof_n >= kProfileSlots) return CODA_ERR_INVALID_ARG;
  g_prof[g_prof_n++] = ProfileSlot{kernel, static_cast<cudaEvent_t>(ev_start), static_cast<cudaEvent_t>(ev_stop)};
  return CODA_OK;
}

coda_status coda_selftest_wait_timeout(void* ws, uint64_t limit_ns, void* stream) {
  if (ws == nullptr) return CODA_ERR_INVALID_ARG;
  if (!aligned16(ws)) return CODA_ERR_MISALIGNED;
  int dev;
  CODA_TRY(current_device(dev));
  limit_ns = std::min<uint64_t>(std::max<uint64_t>(limit_ns, 1000ull), 60000000000ull);
  selftest_wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<uint32_t*>(ws),
                                                                              (unsigned long long)limit_ns);
  return launch_status(cudaPeekAtLastError());
}

coda_status coda_status_clear(void* ws, void* stream) {
  if (ws == nullptr) return CODA_ERR_INVALID_ARG;
  return launch_status(cudaMemsetAsync(ws, 0, kStatusBytes, static_cast<cudaStream_t>(stream)));
}

coda_status coda_status_query(const void* ws, void* stream, uint32_t* detail) {
  if (ws == nullptr) return CODA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return CODA_ERR_CUDA;
  uint32_t w[2] = {0, 0};
  if (cudaMemcpy(w, ws, sizeof(w), cudaMemcpyDeviceToHost) != cudaSuccess) return CODA_ERR_CUDA;
  if (detail != nullptr) *detail = w[1];
  return static_cast<coda_status>(w[0]);
}

// ------------------------------------------------------------------ plain GEMM

namespace coda {
namespace {
// An empty batch (M == 0) has no row to read or write; each weight gradient
// is then a sum over no rows and is written as zeros.  Row-sized pointers may
// be NULL; the weight-gradient pointers must be valid.
struct ZeroSpan {
  void* p;
  size_t bytes;
};
coda_status zero_fill(std::initializer_list<ZeroSpan> spans, void* stream) {
  for (const ZeroSpan& z : spans) {
    if (z.p == nullptr) return CODA_ERR_INVALID_ARG;
    if (!aligned16(z.p)) return CODA_ERR_MISALIGNED;
  }
  int dev;
  CODA_TRY(current_device(dev));
  for (const ZeroSpan& z : spans)
    if (cudaMemsetAsync(z.p, 0, z.bytes, static_cast<cudaStream_t>(stream)) != cudaSuccess) return CODA_ERR_CUDA;
  return CODA_OK;
}
}  // namespace
}  // namespace coda

size_t coda_gemm_workspace_bytes(void) { return kStatusBytes; }

coda_status coda_gemm(const void* A, const void* B, void* C, int M, int N, int K, int a_mn_major, int b_mn_major,
                      void* ws, size_t ws_bytes, void* stream) {
  if (M < 0 || N < 0 || K < 0) return CODA_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return CODA_OK;                               // empty output
  if (K == 0) return zero_fill({{C, (size_t)M * N * 2}}, stream);     // empty sums
  if (!A || !B || !C || !ws) return CODA_ERR_INVALID_ARG;
  if (M < 1 || N < 1 || K < 1) return CODA_ERR_INVALID_ARG;
  if (N % 32 != 0) return CODA_ERR_UNSUPPORTED_SHAPE;
  if ((a_mn_major ? M : K) % 8 != 0 || (b_mn_major ? N : K) % 8 != 0) return CODA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(A) || !aligned16(B) || !aligned16(C) || !aligned16(ws)) return CODA_ERR_MISALIGNED;
  if (ws_bytes < coda_gemm_workspace_bytes()) return CODA_ERR_WORKSPACE_TOO_SMALL;
  int dev;
  CODA_TRY(current_device(dev));
  return gemm_store(A, B, C, M, N, K, a_mn_major != 0, b_mn_major != 0, nullptr, ws,
                    static_cast<cudaStream_t>(stream));
}

coda_status coda_gemm_swiglu(const void* A, const void* Wgu, const float* r_or_null, void* Y, void* AB_or_null,
                             int M, int K, int F, void* ws, size_t ws_bytes, void* stream) {
  if (M == 0) return (K < 1 || F < 1) ? CODA_ERR_INVALID_ARG
                    : (K % 64 != 0 || F % 64 != 0) ? CODA_ERR_UNSUPPORTED_SHAPE : CODA_OK;
  if (!A || !Wgu || !Y || !ws) return CODA_ERR_INVALID_ARG;
  if (M < 1 || K < 1 || F < 1) return CODA_ERR_INVALID_ARG;
  if (K % 64 != 0 || F % 64 != 0) return CODA_ERR_UNSUPPORTED_SHAPE;
  const void* ptrs[] = {A, Wgu, r_or_null, Y, AB_or_null, ws};
  for (const void* q : ptrs)
    if (q && !aligned16(q)) return CODA_ERR_MISALIGNED;
  if (ws_bytes < coda_gemm_workspace_bytes()) return CODA_ERR_WORKSPACE_TOO_SMALL;
  int dev;
  CODA_TRY(current_device(dev));
  return gemm_swiglu(A, Wgu, r_or_null, Y, AB_or_null, M, K, F, ws, static_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------------ gain fold

coda_status coda_fold_gain(const void* W2, const void* g, void* W2g, int d, int N, void* stream) {
  if (!W2 || !g || !W2g) return CODA_ERR_INVALID_ARG;
  if (d < 1 || N < 1) return CODA_ERR_INVALID_ARG;
  if (d % 8 != 0) return CODA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(W2) || !aligned16(g) || !aligned16(W2g)) return CODA_ERR_MISALIGNED;
  int dev;
  CODA_TRY(current_device(dev));
  const long long nv = (long long)N * d / 8;
  const int grid = (int)std::min<long long>(cdiv(nv, 256), (long long)g_dev[dev].num_sms * 8);
  return launch_status(launch_ex(fold_gain_kernel, dim3(grid), dim3(256), 0, static_cast<cudaStream_t>(stream), 1,
                                 cbf(W2), cbf(g), bf(W2g), d, nv));
}

// ------------------------------------------------------------------ GRG forward

namespace {
constexpr int kRmsTile = BN;  // columns per partial sum of squares
struct FwdWs {
  size_t p_off, w2g_off, total;
};
FwdWs fwd_ws(int M, int d, int N, bool prefolded) {
  FwdWs w;
  const int T = cdiv(d, kRmsTile);
  w.p_off = kStatusBytes;
  w.w2g_off = align_up(w.p_off + (size_t)M * T * 4, 256);
  w.total = w.w2g_off + (prefolded ? 0 : align_up((size_t)N * d * 2, 256));
  return w;
}

coda_status check_grg_shapes(int M, int K, int d, int N) {
  if (M < 1 || K < 1 || d < 1 || N < 2) return CODA_ERR_INVALID_ARG;
  if (K % 64 != 0 || d % 64 != 0 || N % 128 != 0) return CODA_ERR_UNSUPPORTED_SHAPE;
  return CODA_OK;
}
}  // namespace

size_t coda_grg_fwd_workspace_bytes(int M, int K, int d, int N, int prefolded) {
  (void)K;
  if (M < 1 || d < 1 || N < 1) return kStatusBytes;
  return fwd_ws(M, d, N, prefolded != 0).total;
}

coda_status coda_grg_fwd(const void* X, const void* W1, const void* R, const void* g, const void* W2,
                         const void* W2g_or_null, void* H, float* r, void* Y, void* AB_or_null, int M, int K, int d,
                         int N, float eps, void* ws, size_t ws_bytes, void* stream) {
  if (M == 0) return !(eps > 0.f) ? CODA_ERR_INVALID_ARG : check_grg_shapes(1, K, d, N);  // empty batch
  if (!X || !W1 || !R || !H || !r || !Y || !ws) return CODA_ERR_INVALID_ARG;
  if (W2g_or_null == nullptr && (!g || !W2)) return CODA_ERR_INVALID_ARG;
  if (!(eps > 0.f)) return CODA_ERR_INVALID_ARG;
  CODA_TRY(check_grg_shapes(M, K, d, N));
  const void* ptrs[] = {X, W1, R, g, W2, W2g_or_null, H, r, Y, AB_or_null, ws};
  for (const void* q : ptrs)
    if (q && !aligned16(q)) return CODA_ERR_MISALIGNED;
  const bool prefolded = W2g_or_null != nullptr;
  const FwdWs w = fwd_ws(M, d, N, prefolded);
  if (ws_bytes < w.total) return CODA_ERR_WORKSPACE_TOO_SMALL;
  int dev;
  CODA_TRY(current_device(dev));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  float* P = reinterpret_cast<float*>(wsb + w.p_off);
  const int T = cdiv(d, kRmsTile);
  const int F = N / 2;

  // Gain fold (skipped when the caller supplies diag(g)-scaled W2).
  const void* W2g = W2g_or_null;
  if (!prefolded) {
    W2g = wsb + w.w2g_off;
    CODA_TRY(coda_fold_gain(W2, g, const_cast<void*>(W2g), d, N, stream));
  }

  // GEMM1 + residual + partial sums of squares.
  {
    const bool pair = use_pair();
    CUtensorMap ta, tb;
    if (!make_operand_map(&ta, X, M, K, false, BM) || !make_operand_map(&tb, W1, d, K, false, pair ? BN / 2 : BN))
      return CODA_ERR_CUDA;
    GemmParams p = base_params(M, d, K, BN, ws, pair);
    p.group_m = pick_group(M, d, K, p.num_m_tiles, p.num_n_tiles, pair, num_sms());
    p.out = bf(H);
    p.ldo = d;
    p.in0 = cbf(R);
    p.ld_in0 = d;
    p.part = P;
    p.ld_part = T;
    CODA_TRY((launch_gemm<EPI_RESID_RMS, false, false>(ta, tb, p, s, pair)));
  }
  // GEMM2 (gate|up): its epilogue forms r from the partial sums (the light
  // row reduction), stores it, scales the rows by it and applies SwiGLU.
  const RowScaleFromPartials rs{P, T, 1.0f / (float)d, eps, r};
  return gemm_swiglu(H, W2g, nullptr, Y, AB_or_null, M, d, F, ws, s, &rs);
}

size_t coda_grg_fwd_hg_workspace_bytes(int M, int K, int d, int N, int hg_given) {
  (void)K, (void)N;
  if (M < 1 || d < 1) return kStatusBytes;
  const int T = cdiv(d, kRmsTile);
  size_t tot = align_up(kStatusBytes + (size_t)M * T * 4, 256);
  if (!hg_given) tot += align_up((size_t)M * d * 2, 256);
  return tot;
}

coda_status coda_grg_fwd_hg(const void* X, const void* W1, const void* R, const void* g, const void* W2, void* H,
                            void* Hg_or_null, float* r, void* Y, void* AB_or_null, int M, int K, int d, int N,
                            float eps, void* ws, size_t ws_bytes, void* stream) {
  if (M == 0) return !(eps > 0.f) ? CODA_ERR_INVALID_ARG : check_grg_shapes(1, K, d, N);  // empty batch
  if (!X || !W1 || !R || !g || !W2 || !H || !r || !Y || !ws) return CODA_ERR_INVALID_ARG;
  if (!(eps > 0.f)) return CODA_ERR_INVALID_ARG;
  CODA_TRY(check_grg_shapes(M, K, d, N));
  const void* ptrs[] = {X, W1, R, g, W2, H, Hg_or_null, r, Y, AB_or_null, ws};
  for (const void* q : ptrs)
    if (q && !aligned16(q)) return CODA_ERR_MISALIGNED;
  if (ws_bytes < coda_grg_fwd_hg_workspace_bytes(M, K, d, N, Hg_or_null != nullptr)) return CODA_ERR_WORKSPACE_TOO_SMALL;
  int dev;
  CODA_TRY(current_device(dev));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  float* P = reinterpret_cast<float*>(wsb + kStatusBytes);
  const int T = cdiv(d, kRmsTile);
  void* Hg = Hg_or_null ? Hg_or_null : wsb + align_up(kStatusBytes + (size_t)M * T * 4, 256);
  const int F = N / 2;
  {
    const bool pair = use_pair();
    CUtensorMap ta, tb;
    if (!make_operand_map(&ta, X, M, K, false, BM) || !make_operand_map(&tb, W1, d, K, false, pair ? BN / 2 : BN))
      return CODA_ERR_CUDA;
    GemmParams p = base_params(M, d, K, BN, ws, pair);
    p.group_m = pick_group(M, d, K, p.num_m_tiles, p.num_n_tiles, pair, num_sms());
    p.out = bf(H);
    p.ldo = d;
    p.in0 = cbf(R);
    p.ld_in0 = d;
    p.part = P;
    p.ld_part = T;
    p.out2 = bf(Hg);
    p.colvec = cbf(g);
    CODA_TRY((launch_gemm<EPI_RESID_RMS, false, false>(ta, tb, p, s, pair)));
  }
  const RowScaleFromPartials rs{P, T, 1.0f / (float)d, eps, r};
  return gemm_swiglu(Hg, W2, nullptr, Y, AB_or_null, M, d, F, ws, s, &rs);
}

// ------------------------------------------------------------------ GRG backward

namespace {
struct BwdWs {
  size_t dap_off, c_off, pg_off, total;
  int pg_rows;
};
BwdWs bwd_ws(int M, int d, int N) {
  BwdWs w;
  w.dap_off = kStatusBytes;
  w.c_off = align_up(w.dap_off + (size_t)M * N * 2, 256);
  w.pg_off = align_up(w.c_off + (size_t)M * 4, 256);
  w.pg_rows = cdiv(M, 256) * 8;  // enough for either tile height
  w.total = align_up(w.pg_off + (size_t)w.pg_rows * d * 4, 256);
  return w;
}
}  // namespace

namespace {
// The backward after dA' = r [da | db] and c are known:
//   dn GEMM: dR = dH = g * (dA' W2) - c * H (+ dH_in), with dg column partials;
//   dg column reduce;  dW2 = g * (dA'^T H);  dX = dH W1;  dW1 = dH^T X.
coda_status grg_bwd_tail(const __nv_bfloat16* dAp, const float* cvec, float* Pg, const void* dH_in_or_null,
                         const void* X, const void* W1, const void* H, const void* g, const void* W2, void* dX,
                         void* dR, void* dW1, void* dW2, float* dg, int M, int K, int d, int N, void* ws,
                         cudaStream_t s, bool pair) {
  {
    CUtensorMap ta, tb;
    if (!make_operand_map(&ta, dAp, M, N, false, BM) || !make_operand_map(&tb, W2, d, N, true, BN))
      return CODA_ERR_CUDA;
    GemmParams p = base_params(M, d, N, BN, ws, pair);
    p.group_m = pick_group(M, d, N, p.num_m_tiles, p.num_n_tiles, pair, num_sms());
    p.out = bf(dR);
    p.ldo = d;
    p.in0 = cbf(H);
    p.ld_in0 = d;
    p.in1 = cbf(dH_in_or_null);
    p.colvec = cbf(g);
    p.rowvec = cvec;
    p.part = Pg;
    p.ld_part = d;
    CODA_TRY((launch_gemm<EPI_DN, false, true>(ta, tb, p, s, pair)));
  }
  // One partial row per 32 output rows of every (possibly partial) row tile.
  CODA_TRY(launch_status(launch_ex(col_reduce_kernel, dim3(cdiv(d, 32)), dim3(COLRED_THREADS), 0, s, 1,
                                   (const float*)Pg, cdiv(M, tile_m(pair)) * tile_m(pair) / 32, d, dg)));
  CODA_TRY(gemm_store(dAp, H, dW2, N, d, M, true, true, g, ws, s));
  CODA_TRY(gemm_store(dR, W1, dX, M, K, d, false, true, nullptr, ws, s));
  return gemm_store(dR, X, dW1, d, K, M, true, true, nullptr, ws, s);
}
}  // namespace

size_t coda_grg_bwd_workspace_bytes(int M, int K, int d, int N) {
  (void)K;
  if (M < 1 || d < 1 || N < 1) return kStatusBytes;
  return bwd_ws(M, d, N).total;
}

coda_status coda_grg_bwd(const void* dY, const void* dH_in_or_null, const void* X, const void* W1, const void* H,
                         const float* r, const void* AB, const void* g, const void* W2, void* dX, void* dR,
                         void* dW1, void* dW2, float* dg, int M, int K, int d, int N, void* ws, size_t ws_bytes,
                         void* stream) {
  if (M == 0) {  // empty batch: zero weight gradients
    CODA_TRY(check_grg_shapes(1, K, d, N));
    return zero_fill({{dW1, (size_t)d * K * 2}, {dW2, (size_t)N * d * 2}, {dg, (size_t)d * 4}}, stream);
  }
  if (!dY || !X || !W1 || !H || !r || !AB || !g || !W2 || !dX || !dR || !dW1 || !dW2 || !dg || !ws)
    return CODA_ERR_INVALID_ARG;
  CODA_TRY(check_grg_shapes(M, K, d, N));
  const void* ptrs[] = {dY, dH_in_or_null, X, W1, H, r, AB, g, W2, dX, dR, dW1, dW2, dg, ws};
  for (const void* q : ptrs)
    if (q && !aligned16(q)) return CODA_ERR_MISALIGNED;
  const BwdWs w = bwd_ws(M, d, N);
  if (ws_bytes < w.total) return CODA_ERR_WORKSPACE_TOO_SMALL;
  int dev;
  CODA_TRY(current_device(dev));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  __nv_bfloat16* dAp = reinterpret_cast<__nv_bfloat16*>(wsb + w.dap_off);
  float* cvec = reinterpret_cast<float*>(wsb + w.c_off);
  float* Pg = reinterpret_cast<float*>(wsb + w.pg_off);
  const int F = N / 2;

  const bool pair = use_pair();
  // SwiGLU backward + RMSNorm row statistic.
  CODA_TRY(launch_status(launch_ex(swiglu_bwd_rowstat_kernel, dim3(M), dim3(ROWSTAT_THREADS), 0, s, 1, cbf(dY),
                                   cbf(AB), r, dAp, cvec, F, 1.0f / (float)d)));
  return grg_bwd_tail(dAp, cvec, Pg, dH_in_or_null, X, W1, H, g, W2, dX, dR, dW1, dW2, dg, M, K, d, N, ws, s, pair);
}

// ------------------------------------------------------------------ SwiGLU MLP

namespace {
coda_status check_swiglu_shapes(int M, int d, int F) {
  if (M < 1 || d < 1 || F < 1) return CODA_ERR_INVALID_ARG;
  if (d % 64 != 0 || F % 64 != 0) return CODA_ERR_UNSUPPORTED_SHAPE;
  return CODA_OK;
}
}  // namespace

size_t coda_swiglu_fwd_workspace_bytes(int M, int d, int F) {
  (void)M, (void)d, (void)F;
  return kStatusBytes;
}

coda_status coda_swiglu_fwd(const void* X, const void* Wgu, const void* Wdown, void* Y, void* AB_or_null,
                            void* Out, int M, int d, int F, void* ws, size_t ws_bytes, void* stream) {
  if (M == 0) return check_swiglu_shapes(1, d, F);  // empty batch
  if (!X || !Wgu || !Wdown || !Y || !Out || !ws) return CODA_ERR_INVALID_ARG;
  CODA_TRY(check_swiglu_shapes(M, d, F));
  const void* ptrs[] = {X, Wgu, Wdown, Y, AB_or_null, Out, ws};
  for (const void* q : ptrs)
    if (q && !aligned16(q)) return CODA_ERR_MISALIGNED;
  if (ws_bytes < coda_swiglu_fwd_workspace_bytes(M, d, F)) return CODA_ERR_WORKSPACE_TOO_SMALL;
  int dev;
  CODA_TRY(current_device(dev));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  CODA_TRY(gemm_swiglu(X, Wgu, nullptr, Y, AB_or_null, M, d, F, ws, s));
  return gemm_store(Y, Wdown, Out, M, d, F, false, false, nullptr, ws, s);
}

size_t coda_swiglu_bwd_workspace_bytes(int M, int d, int F) {
  (void)d;
  if (M < 1 || F < 1) return kStatusBytes;
  return align_up(kStatusBytes + (size_t)M * 2 * F * 2, 256);
}

coda_status coda_swiglu_bwd(const void* dOut, const void* X, const void* Wgu, const void* Wdown, const void* Y,
                            const void* AB, void* dX, void* dWgu, void* dWdown, int M, int d, int F, void* ws,
                            size_t ws_bytes, void* stream) {
  if (M == 0) {  // empty batch: zero weight gradients
    CODA_TRY(check_swiglu_shapes(1, d, F));
    return zero_fill({{dWgu, (size_t)2 * F * d * 2}, {dWdown, (size_t)d * F * 2}}, stream);
  }
  if (!dOut || !X || !Wgu || !Wdown || !Y || !AB || !dX || !dWgu || !dWdown || !ws) return CODA_ERR_INVALID_ARG;
  CODA_TRY(check_swiglu_shapes(M, d, F));
  const void* ptrs[] = {dOut, X, Wgu, Wdown, Y, AB, dX, dWgu, dWdown, ws};
  for (const void* q : ptrs)
    if (!aligned16(q)) return CODA_ERR_MISALIGNED;
  if (ws_bytes < coda_swiglu_bwd_workspace_bytes(M, d, F)) return CODA_ERR_WORKSPACE_TOO_SMALL;
  int dev;
  CODA_TRY(current_device(dev));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  __nv_bfloat16* dA = reinterpret_cast<__nv_bfloat16*>(static_cast<uint8_t*>(ws) + kStatusBytes);
  // Down-projection dgrad with the SwiGLU backward in its epilogue.
  {
    CUtensorMap ta, tb;
    if (!make_operand_map(&ta, dOut, M, d, false, BM) || !make_operand_map(&tb, Wdown, F, d, true, BN))
      return CODA_ERR_CUDA;
    const bool pair = use_pair();
    GemmParams p = base_params(M, F, d, BN, ws, pair);
    p.group_m = pick_group(M, F, d, p.num_m_tiles, p.num_n_tiles, pair, num_sms());
    p.split = F;
    p.out = dA;
    p.ldo = 2 * F;
    p.in0 = cbf(AB);
    p.ld_in0 = 2 * F;
    CODA_TRY((launch_gemm<EPI_SWIGLU_BWD, false, true>(ta, tb, p, s, pair)));
  }
  CODA_TRY(gemm_store(dOut, Y, dWdown, d, F, M, true, true, nullptr, ws, s));
  CODA_TRY(gemm_store(dA, X, dWgu, 2 * F, d, M, true, true, nullptr, ws, s));
  CODA_TRY(gemm_store(dA, Wgu, dX, M, d, 2 * F, false, true, nullptr, ws, s));
  return CODA_OK;
}

}  // extern "C"

// ------------------------------------------------------------------ cross-entropy on the LM head

extern "C" {

size_t coda_xent_fwd_workspace_bytes(int M, int d, int V) {
  (void)d;
  if (M < 1 || V < 1) return kStatusBytes;
  return kStatusBytes + align_up((size_t)M * cdiv(V, BN) * 8, 256) + align_up((size_t)M * 4, 256);
}

namespace {
coda_status check_xent(const void* X, const void* W, const void* t, int M, int d, int V) {
  if (!W || (M > 0 && (!X || !t))) return CODA_ERR_INVALID_ARG;
  if (M < 0 || d < 1 || V < 1) return CODA_ERR_INVALID_ARG;
  if (d % 64 != 0 || V % 64 != 0) return CODA_ERR_UNSUPPORTED_SHAPE;
  return CODA_OK;
}
}  // namespace

coda_status coda_xent_fwd(const void* X, const void* W, const int32_t* targets, float* loss, float* lse, int M,
                          int d, int V, void* ws, size_t ws_bytes, void* stream) {
  CODA_TRY(check_xent(X, W, targets, M, d, V));
  if (M == 0) return CODA_OK;  // empty batch
  if (!loss || !lse || !ws) return CODA_ERR_INVALID_ARG;
  const void* ptrs[] = {X, W, targets, loss, lse, ws};
  for (const void* q : ptrs)
    if (!aligned16(q)) return CODA_ERR_MISALIGNED;
  if (ws_bytes < coda_xent_fwd_workspace_bytes(M, d, V)) return CODA_ERR_WORKSPACE_TOO_SMALL;
  int dev;
  CODA_TRY(current_device(dev));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int T = cdiv(V, BN);
  uint8_t* wsb = static_cast<uint8_t*>(ws) + kStatusBytes;
  float* part = reinterpret_cast<float*>(wsb);
  float* tlogit = reinterpret_cast<float*>(wsb + align_up((size_t)M * T * 8, 256));
  // A target that no tile owns leaves NaN here, so its loss is NaN.
  CODA_TRY(launch_status(cudaMemsetAsync(tlogit, 0xFF, (size_t)M * 4, s)));
  {
    const bool pair = use_pair();
    CUtensorMap ta, tb;
    if (!make_operand_map(&ta, X, M, d, false, BM) || !make_operand_map(&tb, W, V, d, false, pair ? BN / 2 : BN))
      return CODA_ERR_CUDA;
    GemmParams p = base_params(M, V, d, BN, ws, pair);
    p.group_m = pick_group(M, V, d, p.num_m_tiles, p.num_n_tiles, pair, num_sms());
    p.tgt = targets;
    p.part = part;
    p.ld_part = T;
    p.outf = tlogit;
    CODA_TRY((launch_gemm<EPI_XENT, false, false>(ta, tb, p, s, pair)));
  }
  return launch_status(launch_ex(xent_reduce_kernel, dim3(cdiv(M, 8)), dim3(256), 0, s, 1,
                                 (const float2*)part, T, (const float*)tlogit, lse, loss, M));
}

size_t coda_xent_bwd_workspace_bytes(int M, int d, int V) {
  (void)d;
  if (M < 1 || V < 1) return kStatusBytes;
  return kStatusBytes + align_up((size_t)M * V * 2, 256);
}

coda_status coda_xent_bwd(const void* X, const void* W, const int32_t* targets, const float* lse,
                          const float* dloss, void* dX, void* dW, int M, int d, int V, void* ws, size_t ws_bytes,
                          void* stream) {
  CODA_TRY(check_xent(X, W, targets, M, d, V));
  if (M == 0) return zero_fill({{dW, (size_t)V * d * 2}}, stream);  // empty batch: zero weight gradient
  if (!lse || !dloss || !dX || !dW || !ws) return CODA_ERR_INVALID_ARG;
  const void* ptrs[] = {X, W, targets, lse, dloss, dX, dW, ws};
  for (const void* q : ptrs)
    if (!aligned16(q)) return CODA_ERR_MISALIGNED;
  if (ws_bytes < coda_xent_bwd_workspace_bytes(M, d, V)) return CODA_ERR_WORKSPACE_TOO_SMALL;
  int dev;
  CODA_TRY(current_device(dev));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  __nv_bfloat16* dlogits = reinterpret_cast<__nv_bfloat16*>(static_cast<uint8_t*>(ws) + kStatusBytes);
  {
    const bool pair = use_pair();
    CUtensorMap ta, tb;
    if (!make_operand_map(&ta, X, M, d, false, BM) || !make_operand_map(&tb, W, V, d, false, pair ? BN / 2 : BN))
      return CODA_ERR_CUDA;
    GemmParams p = base_params(M, V, d, BN, ws, pair);
    p.group_m = pick_group(M, V, d, p.num_m_tiles, p.num_n_tiles, pair, num_sms());
    p.tgt = targets;
    p.rowvec = lse;
    p.rowvec2 = dloss;
    p.out = dlogits;
    p.ldo = V;
    CODA_TRY((launch_gemm<EPI_XENT_BWD, false, false>(ta, tb, p, s, pair)));
  }
  CODA_TRY(gemm_store(dlogits, W, dX, M, d, V, false, true, nullptr, ws, s));
  return gemm_store(dlogits, X, dW, V, d, M, true, true, nullptr, ws, s);
}

}  // extern "C"

// ------------------------------------------------------------------ full MLP block

extern "C" {

size_t coda_mlp_block_fwd_workspace_bytes(int M, int K, int d, int F) {
  return coda_grg_fwd_workspace_bytes(M, K, d, 2 * F, 0);
}

coda_status coda_mlp_block_fwd(const void* X, const void* W1, const void* R, const void* g, const void* W2,
                               const void* Wdown, void* H, float* r, void* Y, void* AB, void* Out, int M, int K,
                               int d, int F, float eps, void* ws, size_t ws_bytes, void* stream) {
  if (M == 0) return !(eps > 0.f) ? CODA_ERR_INVALID_ARG : check_grg_shapes(1, K, d, 2 * F);  // empty batch
  if (!Wdown || !Out || !AB) return CODA_ERR_INVALID_ARG;
  if (!aligned16(Wdown) || !aligned16(Out)) return CODA_ERR_MISALIGNED;
  // Validates every other argument and runs the block's forward.
  CODA_TRY(coda_grg_fwd(X, W1, R, g, W2, nullptr, H, r, Y, AB, M, K, d, 2 * F, eps, ws, ws_bytes, stream));
  // Down projection with the residual in its epilogue: Out = Y Wdown^T + H.
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool pair = use_pair();
  CUtensorMap ta, tb;
  if (!make_operand_map(&ta, Y, M, F, false, BM) || !make_operand_map(&tb, Wdown, d, F, false, pair ? BN / 2 : BN))
    return CODA_ERR_CUDA;
  GemmParams p = base_params(M, d, F, BN, ws, pair);
  p.group_m = pick_group(M, d, F, p.num_m_tiles, p.num_n_tiles, pair, num_sms());
  p.out = bf(Out);
  p.ldo = d;
  p.in0 = cbf(H);
  p.ld_in0 = d;
  return launch_gemm<EPI_RESID_RMS, false, false>(ta, tb, p, s, pair);
}

namespace {
struct BlockBwdWs {
  BwdWs b;
  size_t pc_off, total;
  int T;
};
BlockBwdWs block_bwd_ws(int M, int d, int F) {
  BlockBwdWs w;
  w.b = bwd_ws(M, d, 2 * F);
  w.T = cdiv(F, BN);
  w.pc_off = w.b.total;
  w.total = align_up(w.pc_off + (size_t)M * w.T * 4, 256);
  return w;
}
}  // namespace

size_t coda_mlp_block_bwd_workspace_bytes(int M, int K, int d, int F) {
  (void)K;
  if (M < 1 || d < 1 || F < 1) return kStatusBytes;
  return block_bwd_ws(M, d, F).total;
}

coda_status coda_mlp_block_bwd(const void* dOut, const void* X, const void* W1, const void* H, const float* r,
                               const void* AB, const void* Y, const void* g, const void* W2, const void* Wdown,
                               void* dX, void* dR, void* dW1, void* dW2, float* dg, void* dWdown, int M, int K, int d,
                               int F, void* ws, size_t ws_bytes, void* stream) {
  if (M == 0) {  // empty batch: zero weight gradients
    CODA_TRY(check_grg_shapes(1, K, d, 2 * F));
    return zero_fill({{dW1, (size_t)d * K * 2}, {dW2, (size_t)2 * F * d * 2}, {dg, (size_t)d * 4},
                      {dWdown, (size_t)d * F * 2}},
                     stream);
  }
  if (!dOut || !X || !W1 || !H || !r || !AB || !Y || !g || !W2 || !Wdown || !dX || !dR || !dW1 || !dW2 || !dg ||
      !dWdown || !ws)
    return CODA_ERR_INVALID_ARG;
  CODA_TRY(check_grg_shapes(M, K, d, 2 * F));
  const void* ptrs[] = {dOut, X, W1, H, r, AB, Y, g, W2, Wdown, dX, dR, dW1, dW2, dg, dWdown, ws};
  for (const void* q : ptrs)
    if (!aligned16(q)) return CODA_ERR_MISALIGNED;
  const BlockBwdWs w = block_bwd_ws(M, d, F);
  if (ws_bytes < w.total) return CODA_ERR_WORKSPACE_TOO_SMALL;
  int dev;
  CODA_TRY(current_device(dev));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  __nv_bfloat16* dAp = reinterpret_cast<__nv_bfloat16*>(wsb + w.b.dap_off);
  float* cvec = reinterpret_cast<float*>(wsb + w.b.c_off);
  float* Pg = reinterpret_cast<float*>(wsb + w.b.pg_off);
  float* Pc = reinterpret_cast<float*>(wsb + w.pc_off);
  const int N = 2 * F;
  const bool pair = use_pair();
  // Down-projection dgrad with the SwiGLU backward, the r scale and the row
  // partials of c in its epilogue: dY never reaches HBM.
  {
    CUtensorMap ta, tb;
    if (!make_operand_map(&ta, dOut, M, d, false, BM) || !make_operand_map(&tb, Wdown, F, d, true, BN))
      return CODA_ERR_CUDA;
    GemmParams p = base_params(M, F, d, BN, ws, pair);
    p.group_m = pick_group(M, F, d, p.num_m_tiles, p.num_n_tiles, pair, num_sms());
    p.split = F;
    p.out = dAp;
    p.ldo = N;
    p.in0 = cbf(AB);
    p.ld_in0 = N;
    p.rowvec = r;
    p.part = Pc;
    p.ld_part = w.T;
    CODA_TRY((launch_gemm<EPI_SWIGLU_BWD, false, true>(ta, tb, p, s, pair)));
  }
  CODA_TRY(launch_status(launch_ex(rowcoef_reduce_kernel, dim3(cdiv(M, 256)), dim3(256), 0, s, 1, (const float*)Pc,
                                   w.T, r, cvec, M, 1.0f / (float)d)));
  CODA_TRY(gemm_store(dOut, Y, dWdown, d, F, M, true, true, nullptr, ws, s));
  // The residual Out = ... + H sends dOut straight into dH.
  return grg_bwd_tail(dAp, cvec, Pg, dOut, X, W1, H, g, W2, dX, dR, dW1, dW2, dg, M, K, d, N, ws, s, pair);
}

}  // extern "C"

// ------------------------------------------------------------------ QKV projection with RoPE

namespace coda {
namespace {
coda_status check_rope(const void* X, const void* W, int M, int d, int n_q, int n_kv, int head_dim, int seq_len,
                       float base) {
  if (!W || (M > 0 && !X)) return CODA_ERR_INVALID_ARG;
  if (M < 0 || d < 1 || n_q < 1 || n_kv < 1 || seq_len < 1 || !(base > 1.f)) return CODA_ERR_INVALID_ARG;
  if (d % 64 != 0 || !(head_dim == 64 || head_dim == 128 || head_dim == 256)) return CODA_ERR_UNSUPPORTED_SHAPE;
  return CODA_OK;
}
float rope_k(int head_dim, float base) { return -2.0f * log2f(base) / (float)head_dim; }
}  // namespace
}  // namespace coda

extern "C" {

coda_status coda_qkv_rope_fwd(const void* X, const void* Wqkv, void* QKV, int M, int d, int n_q, int n_kv,
                              int head_dim, int seq_len, float base, void* ws, size_t ws_bytes, void* stream) {
  CODA_TRY(check_rope(X, Wqkv, M, d, n_q, n_kv, head_dim, seq_len, base));
  if (M == 0) return CODA_OK;  // empty batch
  if (!QKV || !ws) return CODA_ERR_INVALID_ARG;
  const void* ptrs[] = {X, Wqkv, QKV, ws};
  for (const void* q : ptrs)
    if (!aligned16(q)) return CODA_ERR_MISALIGNED;
  if (ws_bytes < coda_gemm_workspace_bytes()) return CODA_ERR_WORKSPACE_TOO_SMALL;
  int dev;
  CODA_TRY(current_device(dev));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int ncols = (n_q + 2 * n_kv) * head_dim;
  const bool pair = use_pair();
  CUtensorMap ta, tb;
  if (!make_operand_map(&ta, X, M, d, false, BM) || !make_operand_map(&tb, Wqkv, ncols, d, false, pair ? BN / 2 : BN))
    return CODA_ERR_CUDA;
  GemmParams p = base_params(M, ncols, d, BN, ws, pair);
  p.group_m = pick_group(M, ncols, d, p.num_m_tiles, p.num_n_tiles, pair, num_sms());
  p.out = bf(QKV);
  p.ldo = ncols;
  p.head_dim = head_dim;
  p.rot_cols = (n_q + n_kv) * head_dim;
  p.seq_len = seq_len;
  p.rope_k = rope_k(head_dim, base);
  return launch_gemm<EPI_ROPE, false, false>(ta, tb, p, s, pair);
}

size_t coda_qkv_rope_bwd_workspace_bytes(int M, int d, int n_q, int n_kv, int head_dim) {
  (void)d;
  if (M < 1 || n_q < 1 || n_kv < 1 || head_dim < 1) return kStatusBytes;
  return kStatusBytes + align_up((size_t)M * (n_q + 2 * n_kv) * head_dim * 2, 256);
}

coda_status coda_qkv_rope_bwd(const void* dQKV, const void* X, const void* Wqkv, void* dX, void* dW, int M, int d,
                              int n_q, int n_kv, int head_dim, int seq_len, float base, void* ws, size_t ws_bytes,
                              void* stream) {
  CODA_TRY(check_rope(X, Wqkv, M, d, n_q, n_kv, head_dim, seq_len, base));
  if (M == 0) return zero_fill({{dW, (size_t)(n_q + 2 * n_kv) * head_dim * d * 2}}, stream);  // empty batch
  if (!dQKV || !dX || !dW || !ws) return CODA_ERR_INVALID_ARG;
  const void* ptrs[] = {dQKV, X, Wqkv, dX, dW, ws};
  for (const void* q : ptrs)
    if (!aligned16(q)) return CODA_ERR_MISALIGNED;
  if (ws_bytes < coda_qkv_rope_bwd_workspace_bytes(M, d, n_q, n_kv, head_dim)) return CODA_ERR_WORKSPACE_TOO_SMALL;
  int dev;
  CODA_TRY(current_device(dev));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int ncols = (n_q + 2 * n_kv) * head_dim;
  __nv_bfloat16* dpre = reinterpret_cast<__nv_bfloat16*>(static_cast<uint8_t*>(ws) + kStatusBytes);
  const int rot_cols = (n_q + n_kv) * head_dim;
  const long long rot_groups = cdiv(rot_cols / head_dim, ROPE_HEADS);
  const long long items = (long long)M * (rot_groups * (head_dim / 16) + (ncols - rot_cols) / ROPE_COPY_COLS);
  CODA_TRY(launch_status(launch_ex(rope_unrotate_kernel, dim3(ew_grid(items)), dim3(256), 0, s, 1, cbf(dQKV),
                                   dpre, M, ncols, head_dim, rot_cols, seq_len, rope_k(head_dim, base))));
  CODA_TRY(gemm_store(dpre, Wqkv, dX, M, d, ncols, false, true, nullptr, ws, s));
  return gemm_store(dpre, X, dW, ncols, d, M, true, true, nullptr, ws, s);
}

}  // extern "C"

// ------------------------------------------------------------------ unfused comparison sequence


extern "C" {

size_t coda_grg_fwd_unfused_workspace_bytes(int M, int K, int d, int N) {
  (void)K, (void)N;
  if (M < 1 || d < 1) return kStatusBytes;
  return kStatusBytes + align_up((size_t)M * d * 2, 256);
}

coda_status coda_grg_fwd_unfused(const void* X, const void* W1, const void* R, const void* g, const void* W2,
                                 void* H, float* r, void* Y, void* AB, void* U, int M, int K, int d, int N,
                                 float eps, void* ws, size_t ws_bytes, void* stream) {
  if (M == 0) return !(eps > 0.f) ? CODA_ERR_INVALID_ARG : check_grg_shapes(1, K, d, N);  // empty batch
  if (!X || !W1 || !R || !g || !W2 || !H || !r || !Y || !AB || !U || !ws) return CODA_ERR_INVALID_ARG;
  if (!(eps > 0.f)) return CODA_ERR_INVALID_ARG;
  CODA_TRY(check_grg_shapes(M, K, d, N));
  const void* ptrs[] = {X, W1, R, g, W2, H, r, Y, AB, U, ws};
  for (const void* q : ptrs)
    if (!aligned16(q)) return CODA_ERR_MISALIGNED;
  if (ws_bytes < coda_grg_fwd_unfused_workspace_bytes(M, K, d, N)) return CODA_ERR_WORKSPACE_TOO_SMALL;
  int dev;
  CODA_TRY(current_device(dev));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  __nv_bfloat16* T = reinterpret_cast<__nv_bfloat16*>(static_cast<uint8_t*>(ws) + kStatusBytes);
  const int F = N / 2;
  CODA_TRY(gemm_store(X, W1, T, M, d, K, false, false, nullptr, ws, s));
  const long long nh = (long long)M * d / 8;
  CODA_TRY(launch_status(launch_ex(unf_residual_add_kernel, dim3(ew_grid(nh)), dim3(256), 0, s, 1,
                                   (const __nv_bfloat16*)T, cbf(R), bf(H), nh)));
  CODA_TRY(launch_status(launch_ex(unf_rmsnorm_fwd_kernel, dim3(M), dim3(UNF_THREADS), 0, s, 1, cbf(H), cbf(g),
                                   bf(U), r, d, eps)));
  CODA_TRY(gemm_store(U, W2, AB, M, N, d, false, false, nullptr, ws, s));
  const long long ny = (long long)M * F / 8;
  CODA_TRY(launch_status(launch_ex(unf_swiglu_fwd_kernel, dim3(ew_grid(ny)), dim3(256), 0, s, 1, cbf(AB), bf(Y), F,
                                   ny)));
  return CODA_OK;
}

size_t coda_grg_bwd_unfused_workspace_bytes(int M, int K, int d, int N) {
  (void)K;
  if (M < 1 || d < 1 || N < 1) return kStatusBytes;
  return kStatusBytes + align_up((size_t)M * N * 2, 256) + align_up((size_t)M * d * 2, 256) +
         align_up((size_t)cdiv(M, UNF_DG_ROWS) * d * 4, 256);
}

coda_status coda_grg_bwd_unfused(const void* dY, const void* dH_in_or_null, const void* X, const void* W1,
                                 const void* H, const float* r, const void* AB, const void* U, const void* g,
                                 const void* W2, void* dX, void* dR, void* dW1, void* dW2, float* dg, int M, int K,
                                 int d, int N, void* ws, size_t ws_bytes, void* stream) {
  if (M == 0) {  // empty batch: zero weight gradients
    CODA_TRY(check_grg_shapes(1, K, d, N));
    return zero_fill({{dW1, (size_t)d * K * 2}, {dW2, (size_t)N * d * 2}, {dg, (size_t)d * 4}}, stream);
  }
  if (!dY || !X || !W1 || !H || !r || !AB || !U || !g || !W2 || !dX || !dR || !dW1 || !dW2 || !dg || !ws)
    return CODA_ERR_INVALID_ARG;
  CODA_TRY(check_grg_shapes(M, K, d, N));
  const void* ptrs[] = {dY, dH_in_or_null, X, W1, H, r, AB, U, g, W2, dX, dR, dW1, dW2, dg, ws};
  for (const void* q : ptrs)
    if (q && !aligned16(q)) return CODA_ERR_MISALIGNED;
  if (ws_bytes < coda_grg_bwd_unfused_workspace_bytes(M, K, d, N)) return CODA_ERR_WORKSPACE_TOO_SMALL;
  int dev;
  CODA_TRY(current_device(dev));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws) + kStatusBytes;
  __nv_bfloat16* dA = reinterpret_cast<__nv_bfloat16*>(wsb);
  wsb += align_up((size_t)M * N * 2, 256);
  __nv_bfloat16* du = reinterpret_cast<__nv_bfloat16*>(wsb);
  wsb += align_up((size_t)M * d * 2, 256);
  float* part = reinterpret_cast<float*>(wsb);
  const int F = N / 2;
  const long long ny = (long long)M * F / 8;
  CODA_TRY(launch_status(launch_ex(unf_swiglu_bwd_kernel, dim3(ew_grid(ny)), dim3(256), 0, s, 1, cbf(dY), cbf(AB),
                                   dA, F, ny)));
  CODA_TRY(gemm_store(dA, W2, du, M, d, N, false, true, nullptr, ws, s));
  CODA_TRY(gemm_store(dA, U, dW2, N, d, M, true, true, nullptr, ws, s));
  const int parts = cdiv(M, UNF_DG_ROWS);
  CODA_TRY(launch_status(launch_ex(unf_dg_partial_kernel, dim3(cdiv(d, 256), parts), dim3(256), 0, s, 1,
                                   (const __nv_bfloat16*)du, cbf(H), r, part, M, d)));
  CODA_TRY(launch_status(launch_ex(col_reduce_kernel, dim3(cdiv(d, 32)), dim3(COLRED_THREADS), 0, s, 1, (const float*)part,
                                   parts, d, dg)));
  CODA_TRY(launch_status(launch_ex(unf_rmsnorm_bwd_kernel, dim3(M), dim3(UNF_THREADS), 0, s, 1,
                                   (const __nv_bfloat16*)du, cbf(H), cbf(g), r, cbf(dH_in_or_null), bf(dR), d)));
  CODA_TRY(gemm_store(dR, W1, dX, M, K, d, false, true, nullptr, ws, s));
  CODA_TRY(gemm_store(dR, X, dW1, d, K, M, true, true, nullptr, ws, s));
  return CODA_OK;
}

}  // extern "C"

// ------------------------------------------------------------------ unfused SwiGLU MLP

extern "C" {

coda_status coda_swiglu_fwd_unfused(const void* X, const void* Wgu, const void* Wdown, void* Y, void* AB, void* Out,
                                    int M, int d, int F, void* ws, size_t ws_bytes, void* stream) {
  if (M == 0) return check_swiglu_shapes(1, d, F);  // empty batch
  if (!X || !Wgu || !Wdown || !Y || !AB || !Out || !ws) return CODA_ERR_INVALID_ARG;
  CODA_TRY(check_swiglu_shapes(M, d, F));
  const void* ptrs[] = {X, Wgu, Wdown, Y, AB, Out, ws};
  for (const void* q : ptrs)
    if (!aligned16(q)) return CODA_ERR_MISALIGNED;
  if (ws_bytes < coda_gemm_workspace_bytes()) return CODA_ERR_WORKSPACE_TOO_SMALL;
  int dev;
  CODA_TRY(current_device(dev));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  CODA_TRY(gemm_store(X, Wgu, AB, M, 2 * F, d, false, false, nullptr, ws, s));
  const long long ny = (long long)M * F / 8;
  CODA_TRY(launch_status(launch_ex(unf_swiglu_fwd_kernel, dim3(ew_grid(ny)), dim3(256), 0, s, 1, cbf(AB), bf(Y), F,
                                   ny)));
  return gemm_store(Y, Wdown, Out, M, d, F, false, false, nullptr, ws, s);
}

size_t coda_swiglu_bwd_unfused_workspace_bytes(int M, int d, int F) {
  (void)d;
  if (M < 1 || F < 1) return kStatusBytes;
  return kStatusBytes + align_up((size_t)M * F * 2, 256) + align_up((size_t)M * 2 * F * 2, 256);
}

coda_status coda_swiglu_bwd_unfused(const void* dOut, const void* X, const void* Wgu, const void* Wdown,
                                    const void* Y, const void* AB, void* dX, void* dWgu, void* dWdown, int M, int d,
                                    int F, void* ws, size_t ws_bytes, void* stream) {
  if (M == 0) {  // empty batch: zero weight gradients
    CODA_TRY(check_swiglu_shapes(1, d, F));
    return zero_fill({{dWgu, (size_t)2 * F * d * 2}, {dWdown, (size_t)d * F * 2}}, stream);
  }
  if (!dOut || !X || !Wgu || !Wdown || !Y || !AB || !dX || !dWgu || !dWdown || !ws) return CODA_ERR_INVALID_ARG;
  CODA_TRY(check_swiglu_shapes(M, d, F));
  const void* ptrs[] = {dOut, X, Wgu, Wdown, Y, AB, dX, dWgu, dWdown, ws};
  for (const void* q : ptrs)
    if (!aligned16(q)) return CODA_ERR_MISALIGNED;
  if (ws_bytes < coda_swiglu_bwd_unfused_workspace_bytes(M, d, F)) return CODA_ERR_WORKSPACE_TOO_SMALL;
  int dev;
  CODA_TRY(current_device(dev));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws) + kStatusBytes;
  __nv_bfloat16* dY = reinterpret_cast<__nv_bfloat16*>(wsb);
  __nv_bfloat16* dA = reinterpret_cast<__nv_bfloat16*>(wsb + align_up((size_t)M * F * 2, 256));
  CODA_TRY(gemm_store(dOut, Wdown, dY, M, F, d, false, true, nullptr, ws, s));
  const long long ny = (long long)M * F / 8;
  CODA_TRY(launch_status(launch_ex(unf_swiglu_bwd_kernel, dim3(ew_grid(ny)), dim3(256), 0, s, 1,
                                   (const __nv_bfloat16*)dY, cbf(AB), dA, F, ny)));
  CODA_TRY(gemm_store(dOut, Y, dWdown, d, F, M, true, true, nullptr, ws, s));
  CODA_TRY(gemm_store(dA, X, dWgu, 2 * F, d, M, true, true, nullptr, ws, s));
  return gemm_store(dA, Wgu, dX, M, d, 2 * F, false, true, nullptr, ws, s);
}

}  // extern "C"

// ------------------------------------------------------------------ forward without allocation
//
// For callers that cannot allocate device memory.  The scratch of the GRG
// forward (status word + partial sums of squares) lives in this file-scope
// device array instead of a caller workspace.  In host code the name
// g_static_scratch is only a host-side stand-in: the device address comes
// from cudaGetSymbolAddress, looked up once per device with that device
// current and cached.  All calls on a device share the array.

namespace coda {
namespace {
constexpr size_t kStaticScratchBytes = kStatusBytes + (size_t)CODA_STATIC_PARTIALS_MAX * sizeof(float);
__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];
std::atomic<void*> g_static_scratch_addr[kMaxDevices];

coda_status static_scratch(int dev, void** out) {
  if (dev < 0 || dev >= kMaxDevices) return CODA_ERR_CUDA;
  void* p = g_static_scratch_addr[dev].load();
  if (p == nullptr) {
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return CODA_ERR_CUDA;
    g_static_scratch_addr[dev].store(p);
  }
  *out = p;
  return CODA_OK;
}
}  // namespace
}  // namespace coda

extern "C" coda_status coda_grg_fwd_prefolded_static(const void* X, const void* W1, const void* R, const void* W2g,
                                                     void* H, float* r, void* Y, void* AB_or_null, int M, int K,
                                                     int d, int N, float eps, void* stream) {
  if (M == 0) return !(eps > 0.f) ? CODA_ERR_INVALID_ARG : check_grg_shapes(1, K, d, N);  // empty batch
  if (!X || !W1 || !R || !W2g || !H || !r || !Y) return CODA_ERR_INVALID_ARG;
  if (!(eps > 0.f)) return CODA_ERR_INVALID_ARG;
  CODA_TRY(check_grg_shapes(M, K, d, N));
  const void* ptrs[] = {X, W1, R, W2g, H, r, Y, AB_or_null};
  for (const void* q : ptrs)
    if (q && !aligned16(q)) return CODA_ERR_MISALIGNED;
  const int T = cdiv(d, kRmsTile);
  if ((unsigned long long)M * (unsigned long long)T > (unsigned long long)CODA_STATIC_PARTIALS_MAX)
    return CODA_ERR_WORKSPACE_TOO_SMALL;  // the static scratch is too small for this shape
  int dev;
  CODA_TRY(current_device(dev));
  void* scratch = nullptr;
  CODA_TRY(static_scratch(dev, &scratch));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The status word must start at zero; P is fully overwritten by GEMM1's epilogue.
  CODA_TRY(launch_status(cudaMemsetAsync(scratch, 0, kStatusBytes, s)));
  float* P = reinterpret_cast<float*>(static_cast<uint8_t*>(scratch) + kStatusBytes);
  const int F = N / 2;
  {
    const bool pair = use_pair();
    CUtensorMap ta, tb;
    if (!make_operand_map(&ta, X, M, K, false, BM) || !make_operand_map(&tb, W1, d, K, false, pair ? BN / 2 : BN))
      return CODA_ERR_CUDA;
    GemmParams p = base_params(M, d, K, BN, scratch, pair);
    p.group_m = pick_group(M, d, K, p.num_m_tiles, p.num_n_tiles, pair, num_sms());
    p.out = bf(H);
    p.ldo = d;
    p.in0 = cbf(R);
    p.ld_in0 = d;
    p.part = P;
    p.ld_part = T;
    CODA_TRY((launch_gemm<EPI_RESID_RMS, false, false>(ta, tb, p, s, pair)));
  }
  const RowScaleFromPartials rs{P, T, 1.0f / (float)d, eps, r};
  return gemm_swiglu(H, W2g, nullptr, Y, AB_or_null, M, d, F, scratch, s, &rs);
}

extern "C" coda_status coda_static_status_query(void* stream, uint32_t* detail) {
  int dev;
  CODA_TRY(current_device(dev));
  void* scratch = nullptr;
  CODA_TRY(static_scratch(dev, &scratch));
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return CODA_ERR_CUDA;
  uint32_t w[2] = {0, 0};
  if (cudaMemcpy(w, scratch, sizeof(w), cudaMemcpyDeviceToHost) != cudaSuccess) return CODA_ERR_CUDA;
  if (detail != nullptr) *detail = w[1];
  return static_cast<coda_status>(w[0]);
}
