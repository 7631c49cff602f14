// rfb_attn.cu -- host side of the C ABI declared in include/rfb_attn.h:
// argument checks, TMA tensor-map encoding, kernel selection and launch.
//
// The library allocates no device memory and never synchronises on the
// caller's stream; everything after the argument checks is an asynchronous
// launch on `stream`.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "rfb_attn.h"
#include "bias_project.cuh"
#include "bwd_kernels.cuh"
#include "bwd_window.cuh"
#include "fwd_kernels.cuh"

namespace rfb {

// Device error word, one per device context.
__device__ int g_err_word = 0;

__global__ void selftest_wait_kernel(int* err, uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const WaitGuard g{&abort_flag, err, timeout_ns, -1};
    wait_bounded(smem_u32(&bar), 0, g, 99);  // nothing ever arrives on this barrier
  }
  __syncthreads();
}

// Scratch of rfb_attn_bwd_noalloc: a fixed module array, so that entry point
// needs no allocation.  In host code this name is only a stand-in; its device
// address comes from cudaGetSymbolAddress (noalloc_scratch below).
static __device__ __align__(256) unsigned char g_noalloc_scratch[RFB_NOALLOC_SCRATCH_BYTES];

__global__ void selftest_exp2_kernel(const float* x, float* y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    soft_exp2_x2(x[i], x[i + 1], y[i], y[i + 1]);
  } else if (i < n) {
    float dummy;
    soft_exp2_x2(x[i], 0.f, y[i], dummy);
  }
}

namespace {

constexpr uint64_t kWaitTimeoutNs = 2000000000ull;  // 2 s per wait
constexpr int kMaxDevices = 64;

// Test hook (rfb_debug_set_wait_limit): the main-loop wait limit and the wait
// site that gives up at once, passed to every kernel launched afterwards.
std::atomic<uint64_t> g_wait_limit_ns{kWaitTimeoutNs};
std::atomic<int> g_fail_site{-1};

// Last failing CUDA call (error code and the site that saw it), for diagnostics.
std::atomic<int> g_last_cuda_err{0};
std::atomic<int> g_last_cuda_site{0};

enum CudaSite {
  kSiteGetDevice = 1, kSiteAttribute = 2, kSiteSymbol = 3, kSiteEncoder = 4, kSiteEncode = 5,
  kSiteFuncAttr = 6, kSiteLaunch = 7, kSiteSync = 8
};

int cuda_fail(int err, int site) {
  g_last_cuda_err.store(err);
  g_last_cuda_site.store(site);
  return RFB_ERR_CUDA;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encoder() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

struct DeviceInfo {
  int sms = 0;
  int* err_word = nullptr;
};

int device_info(DeviceInfo* out) {
  static DeviceInfo cache[kMaxDevices];
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) return cuda_fail(e, kSiteGetDevice);
  // Binds this host thread to the device's primary context in this library's
  // runtime (a no-op when already bound); callers may come from any thread.
  if ((e = cudaSetDevice(dev)) != cudaSuccess) return cuda_fail(e, kSiteGetDevice);
  std::lock_guard<std::mutex> lock(mu);
  DeviceInfo& d = cache[dev];
  if (d.sms == 0) {
    int sms = 0;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_fail(e, kSiteAttribute);
    void* p = nullptr;
    if ((e = cudaGetSymbolAddress(&p, g_err_word)) != cudaSuccess) return cuda_fail(e, kSiteSymbol);
    d.err_word = static_cast<int*>(p);
    d.sms = sms;
  }
  *out = d;
  return RFB_OK;
}

// Raise the dynamic shared-memory limit of a kernel once per device.
template <typename K>
int ensure_smem(K kernel, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev >= kMaxDevices) return cuda_fail(e, kSiteGetDevice);
  const uint64_t bit = 1ull << dev;
  if (done.load(std::memory_order_acquire) & bit) return RFB_OK;
  if ((e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes)) !=
      cudaSuccess)
    return cuda_fail(e, kSiteFuncAttr);
  done.fetch_or(bit, std::memory_order_acq_rel);
  return RFB_OK;
}

CUtensorMapSwizzle swizzle_for(int row_bytes) {
  switch (row_bytes) {
    case 128: return CU_TENSOR_MAP_SWIZZLE_128B;
    case 64: return CU_TENSOR_MAP_SWIZZLE_64B;
    default: return CU_TENSOR_MAP_SWIZZLE_32B;
  }
}

// 3-D bf16 map over a contiguous [BH, N, cols] tensor.  The box is
// (box_cols, box_rows, box_heads); box_cols may exceed cols (zero fill).
// Host cache of encoded tensor maps.  A map depends only on the address, the
// tensor extents and the box, so a hit returns exactly what encoding would;
// entries are replaced round-robin.
struct MapCache {
  struct Entry {
    const void* ptr;
    int kind, cols, N, BH, bc, br, bh;
    CUtensorMap map;
  };
  static constexpr int kSize = 64;
  std::mutex mu;
  Entry e[kSize];
  int used = 0, next = 0;

  bool find(const Entry& k, CUtensorMap* out) {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i) {
      const Entry& x = e[i];
      if (x.ptr == k.ptr && x.kind == k.kind && x.cols == k.cols && x.N == k.N && x.BH == k.BH &&
          x.bc == k.bc && x.br == k.br && x.bh == k.bh) {
        *out = x.map;
        return true;
      }
    }
    return false;
  }
  void put(const Entry& k) {
    std::lock_guard<std::mutex> lock(mu);
    if (used < kSize) {
      e[used++] = k;
    } else {
      e[next] = k;
      next = (next + 1) % kSize;
    }
  }
};
MapCache g_maps;

int encode_3d_uncached(CUtensorMap* m, const void* ptr, int cols, int N, int BH, int box_cols,
                       int box_rows, int box_heads);

int encode_3d(CUtensorMap* m, const void* ptr, int cols, int N, int BH, int box_cols, int box_rows,
              int box_heads) {
  MapCache::Entry k{ptr, 0, cols, N, BH, box_cols, box_rows, box_heads, {}};
  if (g_maps.find(k, m)) return RFB_OK;
  const int rc = encode_3d_uncached(m, ptr, cols, N, BH, box_cols, box_rows, box_heads);
  if (rc == RFB_OK) {
    k.map = *m;
    g_maps.put(k);
  }
  return rc;
}

int encode_3d_uncached(CUtensorMap* m, const void* ptr, int cols, int N, int BH, int box_cols,
                       int box_rows, int box_heads) {
  EncodeTiledFn enc = get_encoder();
  if (!enc) return cuda_fail(0, kSiteEncoder);
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols) * 2,
                                 static_cast<cuuint64_t>(cols) * 2 * static_cast<cuuint64_t>(N)};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows),
                             static_cast<cuuint32_t>(box_heads)};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult rc = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          swizzle_for(box_cols * 2), CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return rc == CUDA_SUCCESS ? RFB_OK : cuda_fail(static_cast<int>(rc), kSiteEncode);
}

// 3-D fp32 map over the [BH, N, cols] dQ|dU accumulator, box (32, 32, 1),
// 128-byte swizzle (32 fp32 per row); used for the bulk reductions, one per
// warp and chunk (32 query rows each).
int encode_acc_3d_uncached(CUtensorMap* m, void* ptr, int cols, int N, int BH);

int encode_acc_3d(CUtensorMap* m, void* ptr, int cols, int N, int BH) {
  MapCache::Entry k{ptr, 1, cols, N, BH, 0, 0, 0, {}};
  if (g_maps.find(k, m)) return RFB_OK;
  const int rc = encode_acc_3d_uncached(m, ptr, cols, N, BH);
  if (rc == RFB_OK) {
    k.map = *m;
    g_maps.put(k);
  }
  return rc;
}

int encode_acc_3d_uncached(CUtensorMap* m, void* ptr, int cols, int N, int BH) {
  EncodeTiledFn enc = get_encoder();
  if (!enc) return cuda_fail(0, kSiteEncoder);
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols) * 4,
                                 static_cast<cuuint64_t>(cols) * 4 * static_cast<cuuint64_t>(N)};
  const cuuint32_t box[3] = {32, 32, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult rc = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, ptr, dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return rc == CUDA_SUCCESS ? RFB_OK : cuda_fail(static_cast<int>(rc), kSiteEncode);
}

// bf16 map of any rank (dims innermost first, strides in bytes for dims 1..),
// not cached (the image-window maps).
int encode_nd(CUtensorMap* m, const void* ptr, int rank, const cuuint64_t* dims,
              const cuuint64_t* strides, const cuuint32_t* box) {
  EncodeTiledFn enc = get_encoder();
  if (!enc) return cuda_fail(0, kSiteEncoder);
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const CUresult rc = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(ptr), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          swizzle_for(static_cast<int>(box[0]) * 2),
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return rc == CUDA_SUCCESS ? RFB_OK : cuda_fail(static_cast<int>(rc), kSiteEncode);
}

int pad_rank(int r) { return r == 0 ? 0 : r <= 16 ? 16 : r <= 32 ? 32 : 64; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shared shape / scalar checks.  Returns RFB_OK, or an error; *empty is set
// when there is nothing to compute.
int check_shape(int B, int H, int N, int d, int r, float scale, bool* empty) {
  *empty = false;
  if (B < 0 || H < 0 || N < 0 || d < 0 || r < 0) return RFB_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.0f)) return RFB_ERR_INVALID_ARG;
  if (d != 32 && d != 64) return RFB_ERR_UNSUPPORTED;
  if (r > 64 || (r % 8) != 0) return RFB_ERR_UNSUPPORTED;
  if (B == 0 || H == 0 || N == 0) {
    *empty = true;
    return RFB_OK;
  }
  const long long bh = static_cast<long long>(B) * H;
  if (bh > 0x7fffffffLL) return RFB_ERR_UNSUPPORTED;
  if (bh * N * (d + r) > (1LL << 40)) return RFB_ERR_UNSUPPORTED;
  return RFB_OK;
}

// Launches a kernel with programmatic stream serialisation: it may start while
// the grid before it in the stream finishes (every kernel launched this way
// waits for that grid itself before touching global memory, grid_dep_wait()).
// The long kernels (the persistent forward over N > 128, the backward main
// pass) go without it: for them it hides nothing, and their forwards measured
// about 1 % slower with it.  A launch error is left for launch_status().
template <typename... KArgs, typename... Args>
void launch_k(bool pdl, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
              cudaStream_t st, const Args&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  (void)cudaLaunchKernelEx(&cfg, kernel, args...);
}
template <typename... KArgs, typename... Args>
void launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                const Args&... args) {
  launch_k(true, kernel, grid, block, smem, st, args...);
}
template <typename... KArgs, typename... Args>
void launch_plain(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                  const Args&... args) {
  launch_k(false, kernel, grid, block, smem, st, args...);
}

int launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? RFB_OK : cuda_fail(e, kSiteLaunch);
}

// ------------------------------------------------------- per-kernel timing
enum KernelId { kIdFwd = 0, kIdBwdPre = 1, kIdBwdMain = 2, kIdBwdPost = 3 };

struct Profiler {
  std::atomic<bool> on{false};
  std::mutex mu;
  struct Rec {
    int id;
    cudaEvent_t a, b;
  };
  Rec recs[8192];
  int n = 0;
  cudaEvent_t pool[16384];
  int pool_n = 0;

  cudaEvent_t get() {
    if (pool_n > 0) return pool[--pool_n];
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
  }
  void put(cudaEvent_t e) {
    if (pool_n < 16384) pool[pool_n++] = e;
    else cudaEventDestroy(e);
  }
};
Profiler g_prof;

// RAII bracket around one launch; records nothing when profiling is off.
struct LaunchTimer {
  int id;
  cudaStream_t st;
  cudaEvent_t a = nullptr;
  LaunchTimer(int kid, cudaStream_t s) : id(kid), st(s) {
    if (!g_prof.on.load(std::memory_order_relaxed)) return;
    std::lock_guard<std::mutex> lock(g_prof.mu);
    a = g_prof.get();
    if (a) cudaEventRecord(a, st);
  }
  ~LaunchTimer() {
    if (!a) return;
    std::lock_guard<std::mutex> lock(g_prof.mu);
    cudaEvent_t b = g_prof.get();
    if (!b) return;
    cudaEventRecord(b, st);
    if (g_prof.n < 8192) g_prof.recs[g_prof.n++] = {id, a, b};
  }
};

struct Maps {
  CUtensorMap q, k, v, u, w, g, acc, o, aug;
};

// ---------------------------------------------------------------- forward
template <int D, int RP, int NP>
int launch_window(const Maps& m, const FwdArgs& a, int sms, cudaStream_t st) {
  using C = WinCfg<D, RP, NP>;
  static std::atomic<uint64_t> done{0};
  constexpr int kMaxSmem = 232448;
  if (int rc = ensure_smem(fwd_window_kernel<D, RP, NP>, kMaxSmem, done)) return rc;
  const int tiles = (a.BH + C::NW - 1) / C::NW;
  const int grid = tiles < sms ? tiles : sms;
  FwdArgs args = a;
  int smem = C::SMEM;
  if (RP > 0 && args.bias_mode == kBiasWindow) {
    // Shared factors: keep every head resident in shared memory when they fit
    // beside the input ring (every CTA would otherwise re-read the same few
    // lines of U and W for each tile).
    const long long need = C::OFF_RES + static_cast<long long>(C::res_bytes(args.bias_heads)) + 1024;
    if (need <= kMaxSmem) {
      args.bias_mode = kBiasResident;
      smem = static_cast<int>(need);
    }
  }
  LaunchTimer timer(kIdFwd, st);
  launch_pdl(fwd_window_kernel<D, RP, NP>, grid, kWinThreads, smem, st,
      m.q, m.k, m.v, m.u, m.w, m.o, args);
  return launch_status();
}

template <int D, int RP>
int launch_long(const Maps& m, const FwdArgs& a, int sms, cudaStream_t st) {
  using C = LongCfg<D, RP>;
  static std::atomic<uint64_t> done{0};
  if (int rc = ensure_smem(fwd_long_kernel<D, RP>, C::SMEM, done)) return rc;
  // Persistent: one CTA per SM (at most one per unit).
  const long long units = static_cast<long long>((a.N + 2 * kTile - 1) / (2 * kTile)) * a.BH;
  const dim3 grid(static_cast<unsigned>(units < sms ? units : sms));
  LaunchTimer timer(kIdFwd, st);
  launch_plain(fwd_long_kernel<D, RP>, grid, kLongThreads, C::SMEM, st,
      m.q, m.k, m.v, m.u, m.w, a);
  return launch_status();
}

// Shifted windows gathered from feature maps (window kernel, IMG).
template <int D, int RP>
int launch_window_img(const Maps& m, const FwdArgs& a, int sms, cudaStream_t st) {
  using C = WinCfg<D, RP, 64, true>;
  static std::atomic<uint64_t> done{0};
  constexpr int kMaxSmem = 232448;
  if (int rc = ensure_smem(fwd_window_kernel<D, RP, 64, true>, kMaxSmem, done)) return rc;
  const long long need =
      RP > 0 ? C::OFF_RES + static_cast<long long>(C::res_bytes(a.bias_heads)) + 1024 : C::SMEM;
  if (need > kMaxSmem) return RFB_ERR_UNSUPPORTED;  // factors of all heads must stay resident
  const int tiles = (a.BH + C::NW - 1) / C::NW;
  const int grid = tiles < sms ? tiles : sms;
  LaunchTimer timer(kIdFwd, st);
  launch_pdl(fwd_window_kernel<D, RP, 64, true>, grid, kWinThreads, static_cast<int>(need), st,
      m.q, m.k, m.v, m.u, m.w, m.o, a);
  return launch_status();
}

int dispatch_window_img(int d, int rp, const Maps& m, const FwdArgs& a, int sms, cudaStream_t st) {
#define RFB_IMG_CASE(DD, RR) \
  if (d == DD && rp == RR) return launch_window_img<DD, RR>(m, a, sms, st);
  RFB_IMG_CASE(32, 0) RFB_IMG_CASE(32, 16) RFB_IMG_CASE(32, 32) RFB_IMG_CASE(32, 64)
  RFB_IMG_CASE(64, 0) RFB_IMG_CASE(64, 16) RFB_IMG_CASE(64, 32) RFB_IMG_CASE(64, 64)
#undef RFB_IMG_CASE
  return RFB_ERR_UNSUPPORTED;
}

// The materialised-bias comparator (long kernel, DENSE).
template <int D>
int launch_long_dense(const Maps& m, const FwdArgs& a, int sms, cudaStream_t st) {
  using C = LongCfg<D, 0, true>;
  static std::atomic<uint64_t> done{0};
  if (int rc = ensure_smem(fwd_long_kernel<D, 0, true>, C::SMEM, done)) return rc;
  const long long units = static_cast<long long>((a.N + 2 * kTile - 1) / (2 * kTile)) * a.BH;
  const dim3 grid(static_cast<unsigned>(units < sms ? units : sms));
  LaunchTimer timer(kIdFwd, st);
  launch_plain(fwd_long_kernel<D, 0, true>, grid, kLongThreads, C::SMEM, st,
      m.q, m.k, m.v, m.u, m.w, a);
  return launch_status();
}

template <int D, int RP>
int dispatch_fwd(const Maps& m, const FwdArgs& a, int sms, cudaStream_t st) {
  if (a.N <= 64) return launch_window<D, RP, 64>(m, a, sms, st);
  if (a.N <= 128) return launch_window<D, RP, 128>(m, a, sms, st);
  return launch_long<D, RP>(m, a, sms, st);
}

int dispatch_fwd_rp(int d, int rp, const Maps& m, const FwdArgs& a, int sms, cudaStream_t st) {
#define RFB_FWD_CASE(DD, RR) \
  if (d == DD && rp == RR) return dispatch_fwd<DD, RR>(m, a, sms, st);
  RFB_FWD_CASE(32, 0) RFB_FWD_CASE(32, 16) RFB_FWD_CASE(32, 32) RFB_FWD_CASE(32, 64)
  RFB_FWD_CASE(64, 0) RFB_FWD_CASE(64, 16) RFB_FWD_CASE(64, 32) RFB_FWD_CASE(64, 64)
#undef RFB_FWD_CASE
  return RFB_ERR_UNSUPPORTED;
}

// --------------------------------------------------------------- backward
struct WsLayout {
  size_t aug, acc, uprime, dw_part, total;
  int npad;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Backward workspace: the query rows' -LSE / s and -D as bf16 parts
// [BH, Npad, 16], the fp32 dQ | dU accumulator [BH, N, d + r], U' [bias heads,
// N, r] bf16 and, for shared factors, the fp32 per-window dW [BH, N, r].
WsLayout ws_layout(int B, int H, int N, int d, int r, bool shared = false) {
  WsLayout L{};
  const size_t bh = static_cast<size_t>(B) * H;
  const size_t bias_heads = shared ? static_cast<size_t>(H) : bh;
  L.npad = (N + kTile - 1) / kTile * kTile;
  L.aug = 0;
  L.acc = align256(bh * L.npad * 16 * 2);
  L.uprime = L.acc + align256(bh * N * static_cast<size_t>(d + r) * sizeof(float));
  L.dw_part = L.uprime + align256(bias_heads * N * static_cast<size_t>(r) * 2);
  L.total = L.dw_part + (shared ? align256(bh * N * static_cast<size_t>(r) * sizeof(float)) : 0);
  return L;
}

template <int D, int RP>
int launch_bwd_main(const Maps& m, const BwdArgs& a, cudaStream_t st) {
  using C = BwdCfg<D, RP>;
  static std::atomic<uint64_t> done{0};
  if (int rc = ensure_smem(bwd_main_kernel<D, RP>, C::SMEM, done)) return rc;
  const dim3 grid((a.N + kTile - 1) / kTile, a.BH);
  LaunchTimer timer(kIdBwdMain, st);
  launch_plain(bwd_main_kernel<D, RP>, grid, kBwdThreads, C::SMEM, st,
      m.q, m.k, m.v, m.u, m.w, m.g, m.acc, m.aug, a);
  return launch_status();
}

int dispatch_bwd_main(int d, int rp, const Maps& m, const BwdArgs& a, cudaStream_t st) {
#define RFB_BWD_CASE(DD, RR) \
  if (d == DD && rp == RR) return launch_bwd_main<DD, RR>(m, a, st);
  RFB_BWD_CASE(32, 0) RFB_BWD_CASE(32, 16) RFB_BWD_CASE(32, 32) RFB_BWD_CASE(32, 64)
  RFB_BWD_CASE(64, 0) RFB_BWD_CASE(64, 16) RFB_BWD_CASE(64, 32) RFB_BWD_CASE(64, 64)
#undef RFB_BWD_CASE
  return RFB_ERR_UNSUPPORTED;
}

// Window backward (d = 32, r_pad <= 16, N <= 128): one persistent kernel.
struct WinBwdMaps {
  CUtensorMap q, k, v, g, o, u, w, dq, dk, dv;
};

template <int RP, int NP, bool IMG>
int launch_bwd_window(const WinBwdMaps& m, const BwdWinArgs& a, int sms, cudaStream_t st) {
  using C = BwdWinCfg<RP, NP, IMG>;
  static std::atomic<uint64_t> done{0};
  if (int rc = ensure_smem(bwd_window_kernel<RP, NP, IMG>, C::SMEM, done)) return rc;
  const int tiles = (a.BH + C::NW - 1) / C::NW;
  const int grid = tiles < sms ? tiles : sms;
  LaunchTimer timer(kIdBwdMain, st);
  launch_pdl(bwd_window_kernel<RP, NP, IMG>, grid, kBwdWinThreads, C::SMEM, st,
      m.q, m.k, m.v, m.g, m.o, m.u, m.w, m.dq, m.dk, m.dv, a);
  return launch_status();
}

int dispatch_bwd_window(int rp, int N, bool img, const WinBwdMaps& m, const BwdWinArgs& a, int sms,
                        cudaStream_t st) {
  if (img) return rp == 0 ? launch_bwd_window<0, 64, true>(m, a, sms, st)
                          : launch_bwd_window<16, 64, true>(m, a, sms, st);
  if (N <= 64)
    return rp == 0 ? launch_bwd_window<0, 64, false>(m, a, sms, st)
                   : launch_bwd_window<16, 64, false>(m, a, sms, st);
  return rp == 0 ? launch_bwd_window<0, 128, false>(m, a, sms, st)
                 : launch_bwd_window<16, 128, false>(m, a, sms, st);
}

// Whether the window backward takes these sizes.
bool window_bwd_ok(int N, int d, int rp) { return d == 32 && rp <= 16 && N <= kTile; }

int grid_for(long long work, int per_block, int sms) {
  long long g = (work + per_block - 1) / per_block;
  const long long cap = static_cast<long long>(sms) * 8;
  if (g > cap) g = cap;
  return g < 1 ? 1 : static_cast<int>(g);
}

// Device address of g_noalloc_scratch on the current device, looked up once
// per device with that device current.  Returns RFB_OK or RFB_ERR_CUDA.
int noalloc_scratch(void** out) {
  static void* addr[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) return cuda_fail(e, kSiteGetDevice);
  if ((e = cudaSetDevice(dev)) != cudaSuccess) return cuda_fail(e, kSiteGetDevice);
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if ((e = cudaGetSymbolAddress(&p, g_noalloc_scratch)) != cudaSuccess)
      return cuda_fail(e, kSiteSymbol);
    addr[dev] = p;
  }
  *out = addr[dev];
  return RFB_OK;
}

}  // namespace
}  // namespace rfb

namespace rfb {
namespace {
// Forward of both entry points; `shared`: U, W are [H, N, r], one pair per head.
int attn_fwd_impl(const void* q, const void* k, const void* v, const void* u, const void* w,
                  void* o, float* lse, int B, int H, int N, int d, int r, float scale,
                  void* stream, bool shared) {
  bool empty = false;
  if (int rc = check_shape(B, H, N, d, r, scale, &empty)) return rc;
  if (empty) return RFB_OK;
  if (!q || !k || !v || !o || !lse || (r > 0 && (!u || !w))) return RFB_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      (r > 0 && (!aligned16(u) || !aligned16(w))))
    return RFB_ERR_ALIGNMENT;
  DeviceInfo dev;
  if (int rc = device_info(&dev)) return rc;
  const int BH = B * H;
  const int rp = pad_rank(r);
  Maps m;
  std::memset(&m, 0, sizeof(m));
  int rows = kTile, heads = 1;
  if (N <= 64) {
    rows = 64;
    heads = 2;
  }
  int rc = encode_3d(&m.q, q, d, N, BH, d, rows, heads);
  if (!rc) rc = encode_3d(&m.k, k, d, N, BH, d, rows, heads);
  if (!rc) rc = encode_3d(&m.v, v, d, N, BH, d, rows, heads);
  // The window kernel writes O by TMA stores of 32 rows.
  if (!rc && N <= kTile) rc = encode_3d(&m.o, o, d, N, BH, d, 32, 1);
  // Shared factors: [H, N, r], one window's rows per copy.
  const int bias_heads = shared ? H : BH;
  const int bias_box = shared ? 1 : heads;
  if (!rc && r > 0) rc = encode_3d(&m.u, u, r, N, bias_heads, rp, rows, bias_box);
  if (!rc && r > 0) rc = encode_3d(&m.w, w, r, N, bias_heads, rp, rows, bias_box);
  if (rc) return rc;
  FwdArgs a;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.err = dev.err_word;
  a.BH = BH;
  a.N = N;
  a.bias_heads = bias_heads;
  a.bias_mode = shared ? kBiasWindow : kBiasTile;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.inv_scale = 1.0f / scale;
  a.timeout_ns = g_wait_limit_ns.load();
  a.fail_site = g_fail_site.load();
  return dispatch_fwd_rp(d, rp, m, a, dev.sms, static_cast<cudaStream_t>(stream));
}
}  // namespace
}  // namespace rfb

namespace rfb {
namespace {
// Backward of both entry points; `shared`: U, W, dU, dW are [H, N, r] and dU,
// dW are summed over the B windows.
int attn_bwd_impl(const void* q, const void* k, const void* v, const void* u, const void* w,
                  const void* o, const float* lse, const void* dout, void* dq, void* dk,
                  void* dv, void* du, void* dw, void* workspace, size_t workspace_bytes, int B,
                  int H, int N, int d, int r, float scale, void* stream, bool shared,
                  const int* img_mask = nullptr) {
  bool empty = false;
  if (int rc = check_shape(B, H, N, d, r, scale, &empty)) return rc;
  if (empty) return RFB_OK;
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv ||
      (r > 0 && (!u || !w || !du || !dw)))
    return RFB_ERR_INVALID_ARG;
  const void* all[] = {q, k, v, o, lse, dout, dq, dk, dv};
  for (const void* p : all)
    if (!aligned16(p)) return RFB_ERR_ALIGNMENT;
  if (r > 0 && (!aligned16(u) || !aligned16(w) || !aligned16(du) || !aligned16(dw)))
    return RFB_ERR_ALIGNMENT;
  const WsLayout L = ws_layout(B, H, N, d, r, shared);
  if (!workspace || workspace_bytes < L.total) return RFB_ERR_WORKSPACE;
  if (!aligned16(workspace)) return RFB_ERR_ALIGNMENT;
  DeviceInfo dev;
  if (int rc = device_info(&dev)) return rc;
  const int BH = B * H;
  const int bias_heads = shared ? H : BH;
  const int rp = pad_rank(r);
  if (!img_mask && window_bwd_ok(N, d, rp)) {
    // Whole windows per tile: one kernel, plus the sum over the windows of the
    // shared factors' gradients.
    const int np = N <= 64 ? 64 : kTile, nw = kTile / np;
    WinBwdMaps wm;
    std::memset(&wm, 0, sizeof(wm));
    int rc = encode_3d(&wm.q, q, d, N, BH, d, np, nw);
    if (!rc) rc = encode_3d(&wm.k, k, d, N, BH, d, np, nw);
    if (!rc) rc = encode_3d(&wm.v, v, d, N, BH, d, np, nw);
    if (!rc) rc = encode_3d(&wm.g, dout, d, N, BH, d, np, nw);
    if (!rc) rc = encode_3d(&wm.o, o, d, N, BH, d, np, nw);
    if (!rc && r > 0) rc = encode_3d(&wm.u, u, r, N, bias_heads, d, np, shared ? 1 : nw);
    if (!rc && r > 0) rc = encode_3d(&wm.w, w, r, N, bias_heads, d, np, shared ? 1 : nw);
    if (!rc) rc = encode_3d(&wm.dq, dq, d, N, BH, d, 32, 1);
    if (!rc) rc = encode_3d(&wm.dk, dk, d, N, BH, d, 32, 1);
    if (!rc) rc = encode_3d(&wm.dv, dv, d, N, BH, d, 32, 1);
    if (rc) return rc;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    BwdWinArgs a;
    std::memset(&a, 0, sizeof(a));
    a.lse = lse;
    a.du = static_cast<__nv_bfloat16*>(du);
    a.dw = static_cast<__nv_bfloat16*>(dw);
    if (shared && r > 0) {  // fp32 rows per window-head in the workspace
      a.du_part = reinterpret_cast<float*>(ws + L.acc);
      a.dw_part = reinterpret_cast<float*>(ws + L.dw_part);
    }
    a.err = dev.err_word;
    a.BH = BH;
    a.N = N;
    a.r = r;
    a.bias_heads = bias_heads;
    a.shared = shared ? 1 : 0;
    a.img_heads = 1;
    a.scale = scale;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.inv_scale = 1.0f / scale;
    a.timeout_ns = g_wait_limit_ns.load();
    a.fail_site = g_fail_site.load();
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((rc = dispatch_bwd_window(rp, N, false, wm, a, dev.sms, st))) return rc;
    if (shared && r > 0) {
      LaunchTimer timer(kIdBwdPost, st);
      launch_pdl(sum_bias_grads_kernel, H * N, 256, 0, st,
          a.du_part, r, a.dw_part, r, a.du, a.dw, B, H, N, r);
    }
    return launch_status();
  }
  Maps m;
  std::memset(&m, 0, sizeof(m));
  int rc = encode_3d(&m.q, q, d, N, BH, d, kTile, 1);
  if (!rc) rc = encode_3d(&m.k, k, d, N, BH, d, kTile, 1);
  if (!rc) rc = encode_3d(&m.v, v, d, N, BH, d, kTile, 1);
  if (!rc) rc = encode_3d(&m.g, dout, d, N, BH, d, kTile, 1);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  // The backward stages U' = U / s once (bwd_pre) and tiles that copy.
  // With d = 64 the U' and W tiles are staged 64 columns wide (zero padded), so
  // they sit beside Q and K as one MMA operand each.
  if (!rc && r > 0)
    rc = encode_3d(&m.u, ws + L.uprime, r, N, bias_heads, d == 64 ? 64 : rp, kTile, 1);
  if (!rc && r > 0) rc = encode_3d(&m.w, w, r, N, bias_heads, d == 64 ? 64 : rp, kTile, 1);
  if (!rc) rc = encode_acc_3d(&m.acc, ws + L.acc, d + r, N, BH);
  if (!rc) rc = encode_3d(&m.aug, ws + L.aug, 16, L.npad, BH, 16, kTile, 1);
  if (rc) return rc;
  BwdArgs a;
  a.o = static_cast<const __nv_bfloat16*>(o);
  a.lse = lse;
  a.dout = static_cast<const __nv_bfloat16*>(dout);
  a.u = static_cast<const __nv_bfloat16*>(u);
  a.uprime = reinterpret_cast<__nv_bfloat16*>(ws + L.uprime);
  a.aug = reinterpret_cast<__nv_bfloat16*>(ws + L.aug);
  a.acc = reinterpret_cast<float*>(ws + L.acc);
  a.dq = static_cast<__nv_bfloat16*>(dq);
  a.dk = static_cast<__nv_bfloat16*>(dk);
  a.dv = static_cast<__nv_bfloat16*>(dv);
  a.du = static_cast<__nv_bfloat16*>(du);
  a.dw = static_cast<__nv_bfloat16*>(dw);
  a.dw_part = shared ? reinterpret_cast<float*>(ws + L.dw_part) : nullptr;
  a.bias_heads = bias_heads;
  a.err = dev.err_word;
  a.BH = BH;
  a.N = N;
  a.Npad = L.npad;
  a.D = d;
  a.r = r;
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.inv_scale = 1.0f / scale;
  a.timeout_ns = g_wait_limit_ns.load();
  a.fail_site = g_fail_site.load();
  // img_mask = {shift, windows per map row, windows per map column, heads}
  a.mask_shift = img_mask ? img_mask[0] : 0;
  a.mask_nwx = img_mask ? img_mask[1] : 1;
  a.mask_nwy = img_mask ? img_mask[2] : 1;
  a.mask_heads = img_mask ? img_mask[3] : 1;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long rows = static_cast<long long>(BH) * L.npad;
  {
    LaunchTimer timer(kIdBwdPre, st);
    launch_pdl(bwd_pre_kernel, grid_for(rows, 256 / (d / 8), dev.sms), 256, 0, st, a);
  }
  if ((rc = launch_status())) return rc;
  if ((rc = dispatch_bwd_main(d, rp, m, a, st))) return rc;
  const long long groups = static_cast<long long>(BH) * N * ((d + r) / 8);
  {
    LaunchTimer timer(kIdBwdPost, st);
    launch_pdl(bwd_post_kernel, grid_for(groups, 256, dev.sms), 256, 0, st, a);
    if (shared && r > 0) {
      if ((rc = launch_status())) return rc;
      // dU from the accumulator's dU columns, dW from the per-window fp32 rows
      launch_pdl(sum_bias_grads_kernel, H * N, 256, 0, st,
          a.acc + d, d + r, a.dw_part, r, a.du, a.dw, B, H, N, r);
    }
  }
  return launch_status();
}

// Image-window backward workspace: the eight window tensors (Q, K, V, O, dO
// gathered; dQ, dK, dV before their scatter), the gathered LSE, then the
// shared-factor backward's own workspace.
struct ImgWsLayout {
  size_t win[8], lse, inner, total;
};

ImgWsLayout img_ws_layout(long long BH, int heads, int d, int r) {
  ImgWsLayout L;
  const size_t t = align256(static_cast<size_t>(BH) * 64 * d * 2);
  size_t off = 0;
  for (int i = 0; i < 8; ++i) {
    L.win[i] = off;
    off += t;
  }
  L.lse = off;
  off += align256(static_cast<size_t>(BH) * 64 * sizeof(float));
  L.inner = off;
  off += ws_layout(static_cast<int>(BH / heads), heads, 64, d, r, true).total;
  L.total = off;
  return L;
}

// Shape checks shared by the image-window entry points; *bh receives the
// number of window-heads (0: nothing to do).
int check_image_windows(int B, int img_h, int img_w, int heads, int d, int r, int win, int shift,
                        float scale, long long* bh) {
  bool empty = false;
  *bh = 0;
  if (int rc = check_shape(B, heads, 64, d, r, scale, &empty)) return rc;
  if (B < 0 || img_h < 0 || img_w < 0) return RFB_ERR_INVALID_ARG;
  if (win != 8 || (shift != 0 && shift != 4)) return RFB_ERR_UNSUPPORTED;
  if (img_h % 8 != 0 || img_w % 8 != 0) return RFB_ERR_UNSUPPORTED;
  if (empty || img_h == 0 || img_w == 0) return RFB_OK;
  const long long n = static_cast<long long>(B) * (img_h / 8) * (img_w / 8) * heads;
  if (n > 0x7fffffffLL / 64) return RFB_ERR_UNSUPPORTED;
  *bh = n;
  return RFB_OK;
}
}  // namespace
}  // namespace rfb

using namespace rfb;

extern "C" {


int rfb_attn_fwd(const void* q, const void* k, const void* v, const void* u, const void* w,
                 void* o, float* lse, int B, int H, int N, int d, int r, float scale,
                 void* stream) {
  return attn_fwd_impl(q, k, v, u, w, o, lse, B, H, N, d, r, scale, stream, false);
}

int rfb_attn_fwd_shared_bias(const void* q, const void* k, const void* v, const void* u,
                             const void* w, void* o, float* lse, int B, int H, int N, int d,
                             int r, float scale, void* stream) {
  return attn_fwd_impl(q, k, v, u, w, o, lse, B, H, N, d, r, scale, stream, true);
}

int rfb_attn_fwd_dense_bias(const void* q, const void* k, const void* v, const void* bias,
                            void* o, float* lse, int B, int H, int N, int d, int bias_heads,
                            float scale, void* stream) {
  bool empty = false;
  if (int rc = check_shape(B, H, N, d, 0, scale, &empty)) return rc;
  if (empty) return RFB_OK;
  if (!q || !k || !v || !bias || !o || !lse) return RFB_ERR_INVALID_ARG;
  const int BH = B * H;
  if (bias_heads != H && bias_heads != BH) return RFB_ERR_INVALID_ARG;
  if (N % 8 != 0) return RFB_ERR_UNSUPPORTED;  // bias rows must be 16-byte multiples
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(bias) || !aligned16(o) ||
      !aligned16(lse))
    return RFB_ERR_ALIGNMENT;
  DeviceInfo dev;
  if (int rc = device_info(&dev)) return rc;
  Maps m;
  std::memset(&m, 0, sizeof(m));
  int rc = encode_3d(&m.q, q, d, N, BH, d, kTile, 1);
  if (!rc) rc = encode_3d(&m.k, k, d, N, BH, d, kTile, 1);
  if (!rc) rc = encode_3d(&m.v, v, d, N, BH, d, kTile, 1);
  if (!rc) rc = encode_3d(&m.u, bias, N, N, bias_heads, 64, kTile, 1);
  if (rc) return rc;
  FwdArgs a;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.err = dev.err_word;
  a.BH = BH;
  a.N = N;
  a.bias_heads = bias_heads;
  a.bias_mode = kBiasTile;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.inv_scale = 1.0f / scale;
  a.timeout_ns = g_wait_limit_ns.load();
  a.fail_site = g_fail_site.load();
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return d == 32 ? launch_long_dense<32>(m, a, dev.sms, st) : launch_long_dense<64>(m, a, dev.sms, st);
}

int rfb_attn_fwd_image_windows(const void* q, const void* k, const void* v, const void* u,
                               const void* w, void* o, float* lse, int B, int img_h, int img_w,
                               int heads, int d, int r, int win, int shift, float scale,
                               void* stream) {
  bool empty = false;
  if (int rc = check_shape(B, heads, 64, d, r, scale, &empty)) return rc;
  if (B < 0 || img_h < 0 || img_w < 0) return RFB_ERR_INVALID_ARG;
  if (win != 8 || (shift != 0 && shift != 4)) return RFB_ERR_UNSUPPORTED;
  if (img_h % 8 != 0 || img_w % 8 != 0) return RFB_ERR_UNSUPPORTED;
  if (empty || img_h == 0 || img_w == 0) return RFB_OK;
  if (!q || !k || !v || !o || !lse || (r > 0 && (!u || !w))) return RFB_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      (r > 0 && (!aligned16(u) || !aligned16(w))))
    return RFB_ERR_ALIGNMENT;
  const long long bh = static_cast<long long>(B) * (img_h / 8) * (img_w / 8) * heads;
  if (bh > 0x7fffffffLL) return RFB_ERR_UNSUPPORTED;
  DeviceInfo dev;
  if (int rc = device_info(&dev)) return rc;
  const int rp = pad_rank(r);
  Maps m;
  std::memset(&m, 0, sizeof(m));
  // Q, K, V: (d, heads, W, H, B), a 4 x 4-token box of one head.
  const cuuint64_t dims[5] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(heads),
                              static_cast<cuuint64_t>(img_w), static_cast<cuuint64_t>(img_h),
                              static_cast<cuuint64_t>(B)};
  const cuuint64_t row = static_cast<cuuint64_t>(d) * 2;
  const cuuint64_t strides[4] = {row, row * heads, row * heads * img_w,
                                 row * heads * img_w * img_h};
  const cuuint32_t box[5] = {static_cast<cuuint32_t>(d), 1, 4, 4, 1};
  int rc = encode_nd(&m.q, q, 5, dims, strides, box);
  if (!rc) rc = encode_nd(&m.k, k, 5, dims, strides, box);
  if (!rc) rc = encode_nd(&m.v, v, 5, dims, strides, box);
  if (!rc) rc = encode_nd(&m.o, o, 5, dims, strides, box);
  if (!rc && r > 0) {
    // U, W [heads, 64, r] as (r, 8, 8, heads), a 4 x 4 box.
    const cuuint64_t udims[4] = {static_cast<cuuint64_t>(r), 8, 8, static_cast<cuuint64_t>(heads)};
    const cuuint64_t urow = static_cast<cuuint64_t>(r) * 2;
    const cuuint64_t ustr[3] = {urow, urow * 8, urow * 64};
    const cuuint32_t ubox[4] = {static_cast<cuuint32_t>(rp), 4, 4, 1};
    rc = encode_nd(&m.u, u, 4, udims, ustr, ubox);
    if (!rc) rc = encode_nd(&m.w, w, 4, udims, ustr, ubox);
  }
  if (rc) return rc;
  FwdArgs a;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.err = dev.err_word;
  a.BH = static_cast<int>(bh);
  a.N = 64;
  a.bias_heads = heads;
  a.bias_mode = kBiasResident;
  a.img_h = img_h;
  a.img_w = img_w;
  a.img_heads = heads;
  a.shift = shift;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.inv_scale = 1.0f / scale;
  a.timeout_ns = g_wait_limit_ns.load();
  a.fail_site = g_fail_site.load();
  return dispatch_window_img(d, rp, m, a, dev.sms, static_cast<cudaStream_t>(stream));
}

size_t rfb_attn_bwd_workspace_size(int B, int H, int N, int d, int r) {
  bool empty = false;
  if (check_shape(B, H, N, d, r, 1.0f, &empty) != RFB_OK || empty) return 0;
  return ws_layout(B, H, N, d, r).total;
}


int rfb_attn_bwd(const void* q, const void* k, const void* v, const void* u, const void* w,
                 const void* o, const float* lse, const void* dout, void* dq, void* dk, void* dv,
                 void* du, void* dw, void* workspace, size_t workspace_bytes, int B, int H,
                 int N, int d, int r, float scale, void* stream) {
  return attn_bwd_impl(q, k, v, u, w, o, lse, dout, dq, dk, dv, du, dw, workspace,
                       workspace_bytes, B, H, N, d, r, scale, stream, false);
}

size_t rfb_attn_bwd_shared_bias_workspace_size(int B, int H, int N, int d, int r) {
  bool empty = false;
  if (check_shape(B, H, N, d, r, 1.0f, &empty) != RFB_OK || empty) return 0;
  return ws_layout(B, H, N, d, r, true).total;
}

int rfb_attn_bwd_shared_bias(const void* q, const void* k, const void* v, const void* u,
                             const void* w, const void* o, const float* lse, const void* dout,
                             void* dq, void* dk, void* dv, void* du, void* dw, void* workspace,
                             size_t workspace_bytes, int B, int H, int N, int d, int r,
                             float scale, void* stream) {
  return attn_bwd_impl(q, k, v, u, w, o, lse, dout, dq, dk, dv, du, dw, workspace,
                       workspace_bytes, B, H, N, d, r, scale, stream, true);
}

size_t rfb_attn_bwd_image_windows_workspace_size(int B, int img_h, int img_w, int heads, int d,
                                                  int r) {
  long long bh = 0;
  if (check_image_windows(B, img_h, img_w, heads, d, r, 8, 0, 1.0f, &bh) != RFB_OK || bh == 0)
    return 0;
  return img_ws_layout(bh, heads, d, r).total;
}

int rfb_attn_bwd_image_windows(const void* q, const void* k, const void* v, const void* u,
                               const void* w, const void* o, const float* lse, const void* dout,
                               void* dq, void* dk, void* dv, void* du, void* dw, void* workspace,
                               size_t workspace_bytes, int B, int img_h, int img_w, int heads,
                               int d, int r, int win, int shift, float scale, void* stream) {
  long long bh = 0;
  if (int rc = check_image_windows(B, img_h, img_w, heads, d, r, win, shift, scale, &bh))
    return rc;
  if (bh == 0) return RFB_OK;
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv ||
      (r > 0 && (!u || !w || !du || !dw)))
    return RFB_ERR_INVALID_ARG;
  const void* all[] = {q, k, v, o, lse, dout, dq, dk, dv, workspace};
  for (const void* p : all)
    if (!aligned16(p)) return RFB_ERR_ALIGNMENT;
  const ImgWsLayout L = img_ws_layout(bh, heads, d, r);
  if (!workspace || workspace_bytes < L.total) return RFB_ERR_WORKSPACE;
  DeviceInfo dev;
  if (int rc = device_info(&dev)) return rc;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int rp = pad_rank(r);
  if (window_bwd_ok(64, d, rp)) {
    // One kernel gathers the rolled windows from the maps and scatters dQ, dK,
    // dV back in its TMA addressing; the factors' fp32 rows per window-head go
    // to the workspace and are summed over the windows afterwards.
    WinBwdMaps wm;
    std::memset(&wm, 0, sizeof(wm));
    const cuuint64_t dims[5] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(heads),
                                static_cast<cuuint64_t>(img_w), static_cast<cuuint64_t>(img_h),
                                static_cast<cuuint64_t>(B)};
    const cuuint64_t rowb = static_cast<cuuint64_t>(d) * 2;
    const cuuint64_t strides[4] = {rowb, rowb * heads, rowb * heads * img_w,
                                   rowb * heads * img_w * img_h};
    const cuuint32_t box[5] = {static_cast<cuuint32_t>(d), 1, 4, 4, 1};
    int rc = encode_nd(&wm.q, q, 5, dims, strides, box);
    if (!rc) rc = encode_nd(&wm.k, k, 5, dims, strides, box);
    if (!rc) rc = encode_nd(&wm.v, v, 5, dims, strides, box);
    if (!rc) rc = encode_nd(&wm.g, dout, 5, dims, strides, box);
    if (!rc) rc = encode_nd(&wm.o, o, 5, dims, strides, box);
    if (!rc) rc = encode_nd(&wm.dq, dq, 5, dims, strides, box);
    if (!rc) rc = encode_nd(&wm.dk, dk, 5, dims, strides, box);
    if (!rc) rc = encode_nd(&wm.dv, dv, 5, dims, strides, box);
    if (!rc && r > 0) {
      // U, W [heads, 64, r] as (r, 8, 8, heads), a 4 x 4 box 32 columns wide
      // (zero filled beyond r)
      const cuuint64_t udims[4] = {static_cast<cuuint64_t>(r), 8, 8,
                                   static_cast<cuuint64_t>(heads)};
      const cuuint64_t urow = static_cast<cuuint64_t>(r) * 2;
      const cuuint64_t ustr[3] = {urow, urow * 8, urow * 64};
      const cuuint32_t ubox[4] = {static_cast<cuuint32_t>(d), 4, 4, 1};
      rc = encode_nd(&wm.u, u, 4, udims, ustr, ubox);
      if (!rc) rc = encode_nd(&wm.w, w, 4, udims, ustr, ubox);
    }
    if (rc) return rc;
    const int nwin = static_cast<int>(bh / heads);
    const WsLayout inner = ws_layout(nwin, heads, 64, d, r, true);
    BwdWinArgs a;
    std::memset(&a, 0, sizeof(a));
    a.lse = lse;
    a.du = static_cast<__nv_bfloat16*>(du);
    a.dw = static_cast<__nv_bfloat16*>(dw);
    if (r > 0) {
      a.du_part = reinterpret_cast<float*>(ws + L.inner + inner.acc);
      a.dw_part = reinterpret_cast<float*>(ws + L.inner + inner.dw_part);
    }
    a.err = dev.err_word;
    a.BH = static_cast<int>(bh);
    a.N = 64;
    a.r = r;
    a.bias_heads = heads;
    a.shared = 1;
    a.img_h = img_h;
    a.img_w = img_w;
    a.img_heads = heads;
    a.shift = shift;
    a.scale = scale;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.inv_scale = 1.0f / scale;
    a.timeout_ns = g_wait_limit_ns.load();
    a.fail_site = g_fail_site.load();
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((rc = dispatch_bwd_window(rp, 64, true, wm, a, dev.sms, st))) return rc;
    if (r > 0) {
      LaunchTimer timer(kIdBwdPost, st);
      launch_pdl(sum_bias_grads_kernel, heads * 64, 256, 0, st,
          a.du_part, r, a.dw_part, r, a.du, a.dw, nwin, heads, 64, r);
    }
    return launch_status();
  }
  auto wt = [&](int i) { return reinterpret_cast<__nv_bfloat16*>(ws + L.win[i]); };
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long pieces = bh * 64 * (d / 8);
  // 1. maps -> windows: Q, K, V, O, dO and the LSE.
  ImgMoveArgs g;
  std::memset(&g, 0, sizeof(g));
  const void* srcs[5] = {q, k, v, o, dout};
  for (int i = 0; i < 5; ++i) {
    g.src[i] = static_cast<const __nv_bfloat16*>(srcs[i]);
    g.dst[i] = wt(i);
  }
  g.lse_src = lse;
  g.lse_dst = reinterpret_cast<float*>(ws + L.lse);
  g.ntensor = 5;
  g.BH = static_cast<int>(bh);
  g.img_h = img_h;
  g.img_w = img_w;
  g.heads = heads;
  g.d = d;
  g.shift = shift;
  g.to_windows = 1;
  launch_pdl(img_move_kernel, grid_for(pieces, 256, dev.sms), 256, 0, st, g);
  if (int rc = launch_status()) return rc;
  // 2. the shared-factor backward on the windows, with the shifted-window mask.
  const int mask[4] = {shift, img_w / 8, img_h / 8, heads};
  const int nwin = static_cast<int>(bh / heads);
  if (int rc = attn_bwd_impl(wt(0), wt(1), wt(2), u, w, wt(3), reinterpret_cast<float*>(ws + L.lse),
                             wt(4), wt(5), wt(6), wt(7), du, dw, ws + L.inner, L.total - L.inner,
                             nwin, heads, 64, d, r, scale, stream, true, mask))
    return rc;
  // 3. windows -> maps: dQ, dK, dV.
  ImgMoveArgs sc;
  std::memset(&sc, 0, sizeof(sc));
  void* dsts[3] = {dq, dk, dv};
  for (int i = 0; i < 3; ++i) {
    sc.src[i] = wt(5 + i);
    sc.dst[i] = static_cast<__nv_bfloat16*>(dsts[i]);
  }
  sc.ntensor = 3;
  sc.BH = static_cast<int>(bh);
  sc.img_h = img_h;
  sc.img_w = img_w;
  sc.heads = heads;
  sc.d = d;
  sc.shift = shift;
  sc.to_windows = 0;
  launch_pdl(img_move_kernel, grid_for(pieces, 256, dev.sms), 256, 0, st, sc);
  return launch_status();
}

int rfb_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* u,
                         const void* w, const void* o, const float* lse, const void* dout,
                         void* dq, void* dk, void* dv, void* du, void* dw, int B, int H, int N,
                         int d, int r, float scale, void* stream) {
  bool empty = false;
  if (int rc = check_shape(B, H, N, d, r, scale, &empty)) return rc;
  void* scratch = nullptr;
  // An empty call does only the set-up: looking up the array's address loads
  // the library's kernels on this device, which reserves the array, and caches
  // the address -- so a caller can do both before it reserves the rest of the
  // device's memory or captures a stream.
  if (empty) return noalloc_scratch(&scratch);
  if (ws_layout(B, H, N, d, r).total > RFB_NOALLOC_SCRATCH_BYTES) return RFB_ERR_WORKSPACE;
  if (int rc = noalloc_scratch(&scratch)) return rc;
  // The backward's first kernel zeroes the accumulator and rewrites the row
  // statistics, so what an earlier call left in the array does not matter.
  return rfb_attn_bwd(q, k, v, u, w, o, lse, dout, dq, dk, dv, du, dw, scratch,
                      RFB_NOALLOC_SCRATCH_BYTES, B, H, N, d, r, scale, stream);
}

int rfb_bias_project(const float* bias, const float* x, float* out, int H, int N, int k,
                     int transpose, void* stream) {
  if (H < 0 || N < 0 || k < 1 || k > kProjMaxK) return k > kProjMaxK ? RFB_ERR_UNSUPPORTED
                                                                    : RFB_ERR_INVALID_ARG;
  if (H == 0 || N == 0) return RFB_OK;
  if (!bias || !x || !out) return RFB_ERR_INVALID_ARG;
  if (!aligned16(bias) || !aligned16(x) || !aligned16(out)) return RFB_ERR_ALIGNMENT;
  if (static_cast<long long>(N) > 65535LL * kProjRows || H > 65535) return RFB_ERR_UNSUPPORTED;
  DeviceInfo dev;
  if (int rc = device_info(&dev)) return rc;
  const dim3 grid((N + kProjRows - 1) / kProjRows, H);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (transpose)
    launch_pdl(bias_project_kernel<true>, grid, kProjThreads, 0, st, bias, x, out, N, k);
  else
    launch_pdl(bias_project_kernel<false>, grid, kProjThreads, 0, st, bias, x, out, N, k);
  return launch_status();
}

int rfb_debug_set_wait_limit(unsigned int limit_us, int fail_site) {
  if (fail_site < -1 || fail_site > 255) return RFB_ERR_INVALID_ARG;
  g_wait_limit_ns.store(limit_us == 0 ? kWaitTimeoutNs : static_cast<uint64_t>(limit_us) * 1000ull);
  g_fail_site.store(fail_site);
  return RFB_OK;
}

const char* rfb_strerror(int status) {
  switch (status) {
    case RFB_OK: return "success";
    case RFB_ERR_INVALID_ARG:
      return "invalid argument (null pointer, negative size, or scale not finite and > 0)";
    case RFB_ERR_UNSUPPORTED: return "unsupported shape (d must be 32 or 64; r a multiple of 8 in [0, 64])";
    case RFB_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case RFB_ERR_WORKSPACE: return "workspace missing or too small";
    case RFB_ERR_CUDA: return "CUDA runtime or driver call failed";
    case RFB_ERR_DEVICE_TIMEOUT: return "a kernel's bounded wait expired";
    default: return "unknown status";
  }
}

int rfb_last_device_error(void) {
  if (cudaDeviceSynchronize() != cudaSuccess) return -RFB_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_err_word, sizeof(int)) != cudaSuccess) return -RFB_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_err_word, &zero, sizeof(int)) != cudaSuccess) return -RFB_ERR_CUDA;
  return v;
}

int rfb_selftest_soft_exp2(const float* x, float* y, int n, void* stream) {
  if (n < 0 || (n > 0 && (!x || !y))) return RFB_ERR_INVALID_ARG;
  if (n == 0) return RFB_OK;
  DeviceInfo dev;
  if (int rc = device_info(&dev)) return rc;
  const int pairs = (n + 1) / 2;
  selftest_exp2_kernel<<<(pairs + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n);
  return launch_status();
}

int rfb_selftest_wait_timeout(unsigned int timeout_us, void* stream) {
  DeviceInfo dev;
  if (int rc = device_info(&dev)) return rc;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      dev.err_word, static_cast<uint64_t>(timeout_us) * 1000ull);
  return launch_status();
}

int rfb_profile_enable(int on) {
  g_prof.on.store(on != 0, std::memory_order_relaxed);
  return RFB_OK;
}

int rfb_profile_read(float* ms, int* launches) {
  if (!ms || !launches) return RFB_ERR_INVALID_ARG;
  for (int i = 0; i < RFB_PROFILE_KERNELS; ++i) {
    ms[i] = 0.f;
    launches[i] = 0;
  }
  std::lock_guard<std::mutex> lock(g_prof.mu);
  int rc = RFB_OK;
  for (int i = 0; i < g_prof.n; ++i) {
    Profiler::Rec& r = g_prof.recs[i];
    float t = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess)
      rc = RFB_ERR_CUDA;
    if (r.id >= 0 && r.id < RFB_PROFILE_KERNELS) {
      ms[r.id] += t;
      launches[r.id] += 1;
    }
    g_prof.put(r.a);
    g_prof.put(r.b);
  }
  g_prof.n = 0;
  return rc;
}

const char* rfb_profile_kernel_name(int id) {
  switch (id) {
    case kIdFwd: return "fwd";
    case kIdBwdPre: return "bwd_pre";
    case kIdBwdMain: return "bwd_main";
    case kIdBwdPost: return "bwd_post";
    default: return "unknown";
  }
}

int rfb_last_cuda_error(int* site) {
  if (site) *site = g_last_cuda_site.load();
  return g_last_cuda_err.load();
}

const char* rfb_version(void) { return "rfb_attn 0.1 (sm_100a)"; }

}  // extern "C"
