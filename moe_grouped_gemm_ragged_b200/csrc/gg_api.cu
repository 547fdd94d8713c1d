// C-ABI entry points of the ragged grouped GEMM: argument checks, TMA tensor-map encoding
// and the persistent launch. No entry point reads the offsets on the host, allocates,
// synchronises or clears memory; everything is ordered on the caller's stream.
#include <atomic>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "gg.h"
#include "gg_kernel.cuh"
#include "gg_masked.cuh"

namespace {

using gg::Mode;

constexpr int kMaxDevices = 64;
constexpr uint64_t kDefaultWatchdogNs = 4000000000ull;

std::atomic<uint64_t> g_watchdog_ns{kDefaultWatchdogNs};

// Text of the last failure in this thread (gg_last_error).
thread_local char g_err[256] = "";

gg_status cuda_fail(const char* where, cudaError_t e) {
  snprintf(g_err, sizeof(g_err), "%s: %s", where, cudaGetErrorString(e));
  return GG_ERR_CUDA;
}
std::atomic<int> g_skip_first_load{0};
// test hook: 0 automatic, 1 single CTA, 2 CTA pair, 3 wide CTA pair (256 x 512 tiles)
std::atomic<int> g_force_variant{0};

static_assert(gg::DEV_BAD_OFFSETS == GG_DEV_BAD_OFFSETS, "status bit mismatch");
static_assert(gg::DEV_BAD_MASKED_M == GG_DEV_BAD_MASKED_M, "status bit mismatch");
static_assert(gg::DEV_TIMEOUT == GG_DEV_TIMEOUT, "status bit mismatch");
static_assert(gg::DEV_LAUNCHED == GG_DEV_LAUNCHED, "status bit mismatch");

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

struct DeviceInfo {
  int dev = 0;
  int sms = 0;
  bool sm100 = false;
};

// Per device: filled once (under the mutex), then read without locking.
struct DeviceSlot {
  std::atomic<bool> ready{false};
  int sms = 0;
  bool sm100 = false;
};
DeviceSlot g_dev[kMaxDevices];
std::mutex g_dev_mu;

// Driver entry point that tells whether the calling thread has a current context.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(ptr);
  });
  return fn;
}

gg_status device_info(DeviceInfo* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
  if (dev < 0 || dev >= kMaxDevices) return GG_ERR_UNSUPPORTED;
  // Tensor maps are encoded with a driver call, which needs a current context; a thread
  // that has not touched CUDA yet (e.g. an autograd worker) may have none, and then the
  // device is made current (which creates its primary context).
  CUcontext ctx = nullptr;
  auto get_current = ctx_get_current_fn();
  if (get_current == nullptr || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr)
    if ((e = cudaSetDevice(dev)) != cudaSuccess) return cuda_fail("cudaSetDevice", e);
  DeviceSlot& d = g_dev[dev];
  if (!d.ready.load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (!d.ready.load(std::memory_order_relaxed)) {
      int major = 0, minor = 0, sms = 0;
      if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
          (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
          (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return cuda_fail("cudaDeviceGetAttribute", e);
      d.sms = sms;
      d.sm100 = (major == 10 && minor == 0);
      d.ready.store(true, std::memory_order_release);
    }
  }
  out->dev = dev;
  out->sms = d.sms;
  out->sm100 = d.sm100;
  return GG_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Recently encoded tensor maps of this thread. A map is a pure function of its description
// (address, sizes, strides, box), so a cached one stays valid whatever the memory holds;
// repeated calls on the same buffers skip the encoding.
struct MapKey {
  const void* base;
  int rank;
  uint64_t dims[4];
  uint64_t strides[3];
  uint32_t box[4];
};
struct MapCache {
  static constexpr int kSlots = 16;
  MapKey key[kSlots];
  CUtensorMap map[kSlots];
  int used = 0;
  int next = 0;  // slot replaced next (round robin)
};
thread_local MapCache t_maps;

bool make_map_uncached(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
                       const uint64_t* strides_bytes, const uint32_t* box);

// Tiled bf16 tensor map with 128-byte swizzle; out-of-range elements read as zero.
bool make_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
              const uint64_t* strides_bytes, const uint32_t* box) {
  MapKey k;
  std::memset(&k, 0, sizeof(k));
  k.base = base;
  k.rank = rank;
  for (int i = 0; i < rank; ++i) {
    k.dims[i] = dims[i];
    k.box[i] = box[i];
  }
  for (int i = 0; i + 1 < rank; ++i) k.strides[i] = strides_bytes[i];
  MapCache& c = t_maps;
  for (int i = 0; i < c.used; ++i)
    if (std::memcmp(&c.key[i], &k, sizeof(k)) == 0) {
      *m = c.map[i];
      return true;
    }
  if (!make_map_uncached(m, base, rank, dims, strides_bytes, box)) return false;
  const int slot = c.used < MapCache::kSlots ? c.used++ : c.next;
  if (c.used == MapCache::kSlots) c.next = (slot + 1) % MapCache::kSlots;
  c.key[slot] = k;
  c.map[slot] = *m;
  return true;
}

bool make_map_uncached(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
                       const uint64_t* strides_bytes, const uint32_t* box) {
  auto fn = encode_fn();
  if (fn == nullptr) {
    snprintf(g_err, sizeof(g_err), "cuTensorMapEncodeTiled: driver entry point not found");
    return false;
  }
  cuuint64_t gdim[4];
  cuuint64_t gstr[3];
  cuuint32_t bdim[4];
  cuuint32_t estr[4] = {1, 1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    gdim[i] = dims[i];
    bdim[i] = box[i];
  }
  for (int i = 0; i + 1 < rank; ++i) gstr[i] = strides_bytes[i];
  std::memset(m, 0, sizeof(*m));
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base),
                  gdim, gstr, bdim, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    snprintf(g_err, sizeof(g_err), "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
  return r == CUDA_SUCCESS;
}

// 2-D map over a row-major [rows, cols] bf16 matrix.
bool map_2d(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, uint32_t box_cols,
            uint32_t box_rows) {
  const uint64_t dims[2] = {(uint64_t)cols, (uint64_t)(rows > 0 ? rows : 1)};
  const uint64_t str[1] = {(uint64_t)cols * 2u};
  const uint32_t box[2] = {box_cols, box_rows};
  return make_map(m, base, 2, dims, str, box);
}

// 3-D map over a row-major [rows, cols] bf16 matrix whose columns are split into 64-wide
// chunks (dims innermost first: 64, rows, cols/64): one box of `nchunks` chunks x box_rows
// rows lands in shared memory as [chunk][row][64]. Needs cols % 64 == 0.
bool map_2d_chunked(CUtensorMap* m, const void* base, int64_t rows, int64_t cols,
                    uint32_t box_rows, uint32_t nchunks) {
  const uint64_t dims[3] = {64u, (uint64_t)(rows > 0 ? rows : 1), (uint64_t)cols / 64u};
  const uint64_t str[2] = {(uint64_t)cols * 2u, 128u};
  const uint32_t box[3] = {64u, box_rows, nchunks};
  return make_map(m, base, 3, dims, str, box);
}

// 4-D map over W[E, K, N] with N split into 64-wide chunks (dims innermost first: 64, K,
// N/64, E): one box of `nchunks` chunks x box_k rows of K lands as [chunk][k][64].
// Needs N % 64 == 0.
bool map_w_chunked(CUtensorMap* m, const void* W, int64_t E, int64_t K, int64_t N,
                   uint32_t box_k, uint32_t nchunks) {
  const uint64_t dims[4] = {64u, (uint64_t)K, (uint64_t)N / 64u, (uint64_t)E};
  const uint64_t str[3] = {(uint64_t)N * 2u, 128u, (uint64_t)K * (uint64_t)N * 2u};
  const uint32_t box[4] = {64u, box_k, nchunks, 1u};
  return make_map(m, W, 4, dims, str, box);
}

// 3-D map over the packed weights W[E, K, N] (dims innermost first: N, K, E).
bool map_w(CUtensorMap* m, const void* W, int64_t E, int64_t K, int64_t N, uint32_t box_n,
           uint32_t box_k) {
  const uint64_t dims[3] = {(uint64_t)N, (uint64_t)K, (uint64_t)E};
  const uint64_t str[2] = {(uint64_t)N * 2u, (uint64_t)K * (uint64_t)N * 2u};
  const uint32_t box[3] = {box_n, box_k, 1};
  return make_map(m, W, 3, dims, str, box);
}

template <Mode MODE, int BN, int STAGES, bool PAIR, bool F32 = false, int ACT = 0>
gg_status launch(const CUtensorMap& a, const CUtensorMap& b, const gg::Params& p,
                 int64_t tiles_upper, const DeviceInfo& di, cudaStream_t stream,
                 const CUtensorMap* c = nullptr) {
  auto kern = gg::grouped_gemm_kernel<MODE, BN, STAGES, PAIR, F32, ACT>;
  using L = gg::Layout<BN, STAGES, PAIR, gg::bk_of<MODE>(),
                       gg::staging_bytes<MODE, BN, PAIR, F32, ACT>()>;
  static_assert(L::bytes(GG_MAX_EXPERTS) <= 227u * 1024u, "shared memory of a CTA exceeded");
  const CUtensorMap& mc = c != nullptr ? *c : a;  // the output map, where the kernel stores by TMA
  const size_t smem = L::bytes(p.E);
  const int dev = di.dev;
  cudaError_t ce = cudaSuccess;
  // per device, once: the shared-memory attribute and the resident units (read without a
  // lock afterwards)
  static std::atomic<bool> attr_done[kMaxDevices];
  static int max_units[kMaxDevices] = {};
  static std::mutex mu;
  if (!attr_done[dev].load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lk(mu);
    if (!attr_done[dev].load(std::memory_order_relaxed)) {
      const int max_smem = (int)L::bytes(GG_MAX_EXPERTS);
      if ((ce = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     max_smem)) != cudaSuccess)
        return cuda_fail("cudaFuncSetAttribute", ce);
      int units = di.sms;
      if (PAIR) {
        // persistent grid: as many CTA pairs as can be resident at once
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3(2 * (di.sms / 2), 1, 1);
        cfg.blockDim = dim3(gg::NUM_THREADS, 1, 1);
        cfg.dynamicSmemBytes = (size_t)max_smem;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int clusters = 0;
        if ((ce = cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg)) != cudaSuccess)
          return cuda_fail("cudaOccupancyMaxActiveClusters", ce);
        if (clusters < 1) return cuda_fail("cudaOccupancyMaxActiveClusters", cudaErrorUnknown);
        units = clusters;
      }
      max_units[dev] = units;
      attr_done[dev].store(true, std::memory_order_release);
    }
  }
  int64_t units = tiles_upper < max_units[dev] ? tiles_upper : max_units[dev];
  if (units < 1) units = 1;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  unsigned na = 0;
  if (PAIR) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 2;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  const bool pdl = GG_PDL != 0;
  if (pdl) {
    // may start while the previous kernel of the stream finishes (the kernel waits for it
    // before its first global access)
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.gridDim = dim3((unsigned)(PAIR ? 2 * units : units), 1, 1);
  cfg.blockDim = dim3(gg::NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = na;
  ce = cudaLaunchKernelEx(&cfg, kern, a, b, mc, p);
  if (ce != cudaSuccess && pdl) {
    // a stream or capture that does not take programmatic launches: launch plainly
    (void)cudaGetLastError();
    cfg.numAttrs = na - 1;
    ce = cudaLaunchKernelEx(&cfg, kern, a, b, mc, p);
  }
  if (ce != cudaSuccess) return cuda_fail("cudaLaunchKernelEx", ce);
  ce = cudaGetLastError();
  return ce == cudaSuccess ? GG_OK : cuda_fail("kernel launch", ce);
}

gg::Params base_params(const int32_t* groups, void* out, int32_t* status, int64_t rows_alloc,
                       int32_t E) {
  gg::Params p;
  std::memset(&p, 0, sizeof(p));
  p.groups = groups;
  p.out = reinterpret_cast<__nv_bfloat16*>(out);
  p.status = status;
  p.rows_alloc = rows_alloc;
  p.E = E;
  p.watchdog_ns = g_watchdog_ns.load();
  p.debug_flags = g_skip_first_load.load() ? 1 : 0;
  return p;
}

// 256-bit epilogue stores need every output row to start on a 32-byte boundary.
void set_store_width(gg::Params* p, const void* out, int64_t cols) {
  p->out_v8 = ((reinterpret_cast<uintptr_t>(out) & 31u) == 0 && cols % 16 == 0) ? 1 : 0;
}

gg_status check_common(int64_t rows_alloc, int64_t K, int64_t N, int32_t E,
                       const int32_t* groups, const int32_t* dev_status, DeviceInfo* di) {
  if (E < 1 || K < 1 || N < 1 || rows_alloc < 0 || groups == nullptr) return GG_ERR_INVALID_ARG;
  if (E > GG_MAX_EXPERTS) return GG_ERR_UNSUPPORTED;
  if ((K % 8) != 0 || (N % 8) != 0) return GG_ERR_UNSUPPORTED;
  if (rows_alloc >= (int64_t(1) << 31) || K >= (int64_t(1) << 31) || N >= (int64_t(1) << 31))
    return GG_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(groups) & 3u) != 0) return GG_ERR_UNSUPPORTED;
  if (dev_status != nullptr && (reinterpret_cast<uintptr_t>(dev_status) & 3u) != 0)
    return GG_ERR_UNSUPPORTED;
  gg_status s = device_info(di);
  if (s != GG_OK) return s;
  if (!di->sm100) return GG_ERR_UNSUPPORTED;
  return GG_OK;
}

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

constexpr int kBN = 256;
constexpr int kStages = 4;      // single CTA: 48 KB per stage
constexpr int kPairStages = 6;  // CTA pair: 32 KB per stage and CTA
constexpr int kWgBK = gg::bk_of<Mode::Wgrad>();  // token rows per wgrad stage
constexpr int kWgStages = kStages;
constexpr int kWgPairStages = kPairStages;
// bf16 wgrad of CTA pairs with 256-column tiles stores dW through 32 KB of shared memory and
// TMA, which leaves room for five operand stages
constexpr int kWgPairStagesTma = gg::tma_store_epilogue<Mode::Wgrad, 256, true, false, 0>()
                                     ? 5 : kWgPairStages;
// Wide CTA-pair tiles: 256 x 512 with one accumulator (all 512 TMEM columns), 48 KB per
// stage and CTA. Per flop they move a quarter less operand data into shared memory than
// 256 x 256 pair tiles and, in wgrad, cover twice as much of dW per wave.
constexpr int kWideBN = 512;
constexpr int kWideStages = 4;

// CTA pairs halve the operand traffic per SM but quantise groups to 256-row tiles; they pay
// off once the average group is long.
bool use_pair(int64_t rows, int32_t E) {
  const int v = g_force_variant.load();
  if (v == 1) return false;
  if (v == 2 || v == 3) return true;
  return rows >= 512 * (int64_t)E;
}

// Forward and dgrad on 256 x 512 CTA-pair tiles wherever CTA pairs are used: per flop they
// bring a quarter less operand data from L2 into shared memory, and the operand supply is
// what bounds the 256 x 256 tiles (alternating runs at 1965 MHz, wide vs 256 x 256: gate-up
// forward 994 vs 976 TFLOP/s and dgrad 978 vs 944, down-proj forward 1323 vs 1274 and dgrad
// 1405 vs 1313; large shape forward 1279 vs 1205, dgrad 1219 vs 1188). The SiLU-and-mul
// epilogue of a wide tile releases its accumulator only after its stores, which a short
// reduction does not hide: with it, wide tiles only from a reduction of 4096 on (SiLU
// forward, wide vs 256 x 256: large slice 1503 vs 1440; gate-up 917 vs 1003, down-proj 1199
// vs 1302).
bool use_wide(int64_t rows, int32_t E, int64_t red_len, bool silu = false) {
  const int v = g_force_variant.load();
  if (v == 1 || v == 2) return false;
  if (v == 3) return true;
  return use_pair(rows, E) && (!silu || red_len >= 4096);
}

// Wgrad launch shape: 0 single CTAs, 1 CTA pairs, 2 wide CTA pairs. A wgrad tile is as long
// as its expert, so the shapes trade per-stage efficiency against balance: wide pairs on
// long groups (large shape 1363 TFLOP/s vs 1181 single, 1134 pair; down-proj 1333 vs 1144,
// 1205), plain pairs on the Zipf gate-up shape (average 512 rows: 776 vs 737 single, 731
// wide), single CTAs below.
int wgrad_shape(int64_t rows, int32_t E) {
  const int v = g_force_variant.load();
  if (v == 1) return 0;
  if (v == 2) return 1;
  if (v == 3) return 2;
  if (rows >= 1024 * (int64_t)E) return 2;
  if (rows >= 256 * (int64_t)E) return 1;
  return 0;
}

gg_status wgrad_impl(const void* A, const void* dY, const int32_t* offs, void* dW, bool f32,
                     float alpha, float beta, int64_t rows_alloc, int64_t K, int64_t N,
                     int32_t E, int32_t* dev_status, cudaStream_t stream) {
  DeviceInfo di;
  gg_status s = check_common(rows_alloc, K, N, E, offs, dev_status, &di);
  if (s != GG_OK) return s;
  if (dW == nullptr) return GG_ERR_INVALID_ARG;
  if (!aligned16(dW)) return GG_ERR_UNSUPPORTED;
  if (rows_alloc > 0) {
    if (A == nullptr || dY == nullptr) return GG_ERR_INVALID_ARG;
    if (!aligned16(A) || !aligned16(dY)) return GG_ERR_UNSUPPORTED;
  } else {
    // every group is empty: the maps are never used; dW only gets zeros (or beta * dW)
    A = dW;
    dY = dW;
  }
  const bool a_chunked = (K % 64) == 0, b_chunked = (N % 64) == 0;
  // Single CTAs with 128 x 256 tiles, CTA pairs with 256 x 256 tiles, or CTA pairs with
  // 256 x 512 tiles and one accumulator: the tiles in flight then cover twice as much of an
  // expert's dW, so each operand row streams from HBM half as often.
  const int shape = wgrad_shape(rows_alloc, E);
  const bool wide = shape == 2;
  const bool pair = shape >= 1;
  const uint32_t bcols = wide ? kWideBN / 2 : pair ? kBN / 2 : kBN;  // dY columns per CTA
  CUtensorMap ma, mb;
  if (a_chunked ? !map_2d_chunked(&ma, A, rows_alloc, K, kWgBK, gg::BM / 64)
                : !map_2d(&ma, A, rows_alloc, K, 64, kWgBK))
    return GG_ERR_CUDA;
  if (b_chunked ? !map_2d_chunked(&mb, dY, rows_alloc, N, kWgBK, bcols / 64)
                : !map_2d(&mb, dY, rows_alloc, N, 64, kWgBK))
    return GG_ERR_CUDA;
  gg::Params p = base_params(offs, f32 ? nullptr : dW, dev_status, rows_alloc, E);
  p.out_cols = (int32_t)N;
  p.prod_cols = (int32_t)N;
  p.wg_K = (int32_t)K;
  p.a_chunked = a_chunked ? 1 : 0;
  p.b_chunked = b_chunked ? 1 : 0;
  p.out_f32 = f32 ? reinterpret_cast<float*>(dW) : nullptr;
  p.alpha = alpha;
  p.beta = beta;
  set_store_width(&p, dW, N);
  if (wide) {
    const int64_t tiles = (int64_t)E * cdiv(K, 2 * gg::BM) * cdiv(N, kWideBN);
    if (f32)
      return launch<Mode::Wgrad, kWideBN, kWideStages, true, true>(ma, mb, p, tiles, di, stream);
    return launch<Mode::Wgrad, kWideBN, kWideStages, true>(ma, mb, p, tiles, di, stream);
  }
  if (pair) {
    const int64_t tiles = (int64_t)E * cdiv(K, 2 * gg::BM) * cdiv(N, kBN);
    if (f32) return launch<Mode::Wgrad, kBN, kWgPairStages, true, true>(ma, mb, p, tiles, di, stream);
    // dW as [E][K][N] for the tensor stores: boxes of 64 columns x 32 rows of one expert
    CUtensorMap mc;
    const uint64_t dims[3] = {(uint64_t)N, (uint64_t)K, (uint64_t)E};
    const uint64_t str[2] = {(uint64_t)N * 2u, (uint64_t)K * (uint64_t)N * 2u};
    const uint32_t box[3] = {64u, 32u, 1u};
    if (!make_map(&mc, dW, 3, dims, str, box)) return GG_ERR_CUDA;
    return launch<Mode::Wgrad, kBN, kWgPairStagesTma, true>(ma, mb, p, tiles, di, stream, &mc);
  }
  const int64_t tiles = (int64_t)E * cdiv(K, gg::BM) * cdiv(N, kBN);
  if (f32) return launch<Mode::Wgrad, kBN, kWgStages, false, true>(ma, mb, p, tiles, di, stream);
  return launch<Mode::Wgrad, kBN, kWgStages, false>(ma, mb, p, tiles, di, stream);
}

// Checks the epilogue description and stores it in p. act SiLU-and-mul needs N % 256 == 0
// (gate/up blocks of 128 columns inside every 256-column tile) and halves the output width.
gg_status set_epilogue(gg::Params* p, const gg_epilogue* epi, int64_t N) {
  p->bias_ld = (int32_t)N;
  if (epi == nullptr) return GG_OK;
  if (epi->act != GG_ACT_NONE && epi->act != GG_ACT_SILU_MUL) return GG_ERR_INVALID_ARG;
  if (epi->bias != nullptr && !aligned16(epi->bias)) return GG_ERR_UNSUPPORTED;
  if (epi->bias_scale != nullptr && (reinterpret_cast<uintptr_t>(epi->bias_scale) & 3u) != 0)
    return GG_ERR_UNSUPPORTED;
  if (epi->act == GG_ACT_SILU_MUL && (N % kBN) != 0) return GG_ERR_UNSUPPORTED;
  if ((epi->flags & GG_FLAG_GATE_UP_CONCAT) && epi->act != GG_ACT_SILU_MUL)
    return GG_ERR_INVALID_ARG;
  p->bias = reinterpret_cast<const __nv_bfloat16*>(epi->bias);
  p->bias_scale = epi->bias != nullptr ? epi->bias_scale : nullptr;
  p->gate_up_concat = (epi->flags & GG_FLAG_GATE_UP_CONCAT) ? 1 : 0;
  return GG_OK;
}

// Forward, out = A . W[e] (+ epilogue). W is [E, K, N] (MN-major B: the forward pipeline)
// or, with GG_FLAG_W_NK, [E, N, K] (K-major B: the pipeline of dgrad).
gg_status forward_impl(const void* A, const void* W, const int32_t* offs, void* out,
                       int64_t rows_alloc, int64_t K, int64_t N, int32_t E,
                       const gg_epilogue* epi, int32_t* dev_status, cudaStream_t stream) {
  DeviceInfo di;
  gg_status s = check_common(rows_alloc, K, N, E, offs, dev_status, &di);
  if (s != GG_OK) return s;
  if (W == nullptr) return GG_ERR_INVALID_ARG;
  if (rows_alloc == 0) return GG_OK;  // no row can belong to a group
  if (A == nullptr || out == nullptr) return GG_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(W) || !aligned16(out)) return GG_ERR_UNSUPPORTED;
  const int32_t flags = epi != nullptr ? epi->flags : 0;
  if (flags & ~(GG_FLAG_ZERO_TAIL | GG_FLAG_W_NK | GG_FLAG_GATE_UP_CONCAT))
    return GG_ERR_INVALID_ARG;
  const bool silu = epi != nullptr && epi->act == GG_ACT_SILU_MUL;
  const bool wnk = (flags & GG_FLAG_W_NK) != 0;
  // [gate | up] weights are loaded as 128-column gate and up blocks
  const bool concat = (flags & GG_FLAG_GATE_UP_CONCAT) != 0;
  const bool pair = use_pair(rows_alloc, E);
  const bool wide = pair && use_wide(rows_alloc, E, K, silu);
  const bool chunked = (N % 64) == 0;
  const uint32_t bcols = wide ? kWideBN / 2 : pair ? kBN / 2 : kBN;
  const uint32_t bbox = concat ? 128u : bcols;  // columns of W per box
  CUtensorMap ma, mb;
  if (!map_2d(&ma, A, rows_alloc, K, 64, gg::BM)) return GG_ERR_CUDA;
  if (wnk) {
    // W[e] is [N, K]: K-major B, one box of bcols rows of N per stage
    if (!map_w(&mb, W, E, N, K, 64, bbox)) return GG_ERR_CUDA;
  } else if (chunked ? !map_w_chunked(&mb, W, E, K, N, 64, bbox / 64)
                     : !map_w(&mb, W, E, K, N, 64, 64)) {
    return GG_ERR_CUDA;
  }
  gg::Params p = base_params(offs, out, dev_status, rows_alloc, E);
  p.red_len = (int32_t)K;
  p.b_chunked = (!wnk && chunked) ? 1 : 0;
  p.zero_tail = (flags & GG_FLAG_ZERO_TAIL) ? 1 : 0;
  if ((s = set_epilogue(&p, epi, N)) != GG_OK) return s;
  const int64_t out_cols = silu ? N / 2 : N;
  p.out_cols = (int32_t)out_cols;
  p.prod_cols = (int32_t)N;
  set_store_width(&p, out, out_cols);
  const int64_t tiles =
      (cdiv(rows_alloc, (pair ? 2 : 1) * gg::BM) + E + 1) * cdiv(N, wide ? kWideBN : kBN);
  if (wide) {
    if (wnk) {
      if (silu) return launch<Mode::Dgrad, kWideBN, kWideStages, true, false, 1>(ma, mb, p, tiles, di, stream);
      return launch<Mode::Dgrad, kWideBN, kWideStages, true>(ma, mb, p, tiles, di, stream);
    }
    if (silu) return launch<Mode::Forward, kWideBN, kWideStages, true, false, 1>(ma, mb, p, tiles, di, stream);
    return launch<Mode::Forward, kWideBN, kWideStages, true>(ma, mb, p, tiles, di, stream);
  }
  if (wnk) {
    if (pair) {
      if (silu) return launch<Mode::Dgrad, kBN, kPairStages, true, false, 1>(ma, mb, p, tiles, di, stream);
      return launch<Mode::Dgrad, kBN, kPairStages, true>(ma, mb, p, tiles, di, stream);
    }
    if (silu) return launch<Mode::Dgrad, kBN, kStages, false, false, 1>(ma, mb, p, tiles, di, stream);
    return launch<Mode::Dgrad, kBN, kStages, false>(ma, mb, p, tiles, di, stream);
  }
  if (pair) {
    if (silu) return launch<Mode::Forward, kBN, kPairStages, true, false, 1>(ma, mb, p, tiles, di, stream);
    return launch<Mode::Forward, kBN, kPairStages, true>(ma, mb, p, tiles, di, stream);
  }
  if (silu) return launch<Mode::Forward, kBN, kStages, false, false, 1>(ma, mb, p, tiles, di, stream);
  return launch<Mode::Forward, kBN, kStages, false>(ma, mb, p, tiles, di, stream);
}

// dgrad, dX = dY . W[e]^T. W is [E, K, N] (K-major B: the dgrad pipeline) or, with
// GG_FLAG_W_NK, [E, N, K] (MN-major B: the pipeline of the forward).
gg_status dgrad_impl(const void* dY, const void* W, const int32_t* offs, void* dX,
                     int64_t rows_alloc, int64_t K, int64_t N, int32_t E, int32_t flags,
                     int32_t* dev_status, cudaStream_t stream) {
  DeviceInfo di;
  gg_status s = check_common(rows_alloc, K, N, E, offs, dev_status, &di);
  if (s != GG_OK) return s;
  if (flags & ~(GG_FLAG_ZERO_TAIL | GG_FLAG_W_NK)) return GG_ERR_INVALID_ARG;
  if (W == nullptr) return GG_ERR_INVALID_ARG;
  if (rows_alloc == 0) return GG_OK;
  if (dY == nullptr || dX == nullptr) return GG_ERR_INVALID_ARG;
  if (!aligned16(dY) || !aligned16(W) || !aligned16(dX)) return GG_ERR_UNSUPPORTED;
  const bool wnk = (flags & GG_FLAG_W_NK) != 0;
  const bool pair = use_pair(rows_alloc, E);
  const bool wide = pair && use_wide(rows_alloc, E, N);
  const uint32_t bcols = wide ? kWideBN / 2 : pair ? kBN / 2 : kBN;
  const bool chunked = (K % 64) == 0;
  CUtensorMap ma, mb;
  if (!map_2d(&ma, dY, rows_alloc, N, 64, gg::BM)) return GG_ERR_CUDA;
  if (wnk) {
    // W[e] is [N, K] with the output dimension K contiguous: MN-major B over (K, N)
    if (chunked ? !map_w_chunked(&mb, W, E, N, K, 64, bcols / 64)
                : !map_w(&mb, W, E, N, K, 64, 64))
      return GG_ERR_CUDA;
  } else if (!map_w(&mb, W, E, K, N, 64, bcols)) {
    return GG_ERR_CUDA;
  }
  gg::Params p = base_params(offs, dX, dev_status, rows_alloc, E);
  p.red_len = (int32_t)N;
  p.out_cols = (int32_t)K;
  p.prod_cols = (int32_t)K;
  p.b_chunked = (wnk && chunked) ? 1 : 0;
  p.zero_tail = (flags & GG_FLAG_ZERO_TAIL) ? 1 : 0;
  set_store_width(&p, dX, K);
  const int64_t tiles =
      (cdiv(rows_alloc, (pair ? 2 : 1) * gg::BM) + E + 1) * cdiv(K, wide ? kWideBN : kBN);
  if (wide) {
    if (wnk) return launch<Mode::Forward, kWideBN, kWideStages, true>(ma, mb, p, tiles, di, stream);
    return launch<Mode::Dgrad, kWideBN, kWideStages, true>(ma, mb, p, tiles, di, stream);
  }
  if (wnk) {
    if (pair) return launch<Mode::Forward, kBN, kPairStages, true>(ma, mb, p, tiles, di, stream);
    return launch<Mode::Forward, kBN, kStages, false>(ma, mb, p, tiles, di, stream);
  }
  if (pair) return launch<Mode::Dgrad, kBN, kPairStages, true>(ma, mb, p, tiles, di, stream);
  return launch<Mode::Dgrad, kBN, kStages, false>(ma, mb, p, tiles, di, stream);
}

// Launch of the masked forward kernel (weight columns as the MMA's M): one CTA per SM at
// most, no cluster, programmatic dependent launch as in launch().
template <int SW, int ST>
gg_status launch_masked(const CUtensorMap& mw, const CUtensorMap (&mt)[3],
                        const gg::masked::Params& p, int64_t units, int dev,
                        cudaStream_t stream) {
  auto kern = gg::masked::masked_forward_kernel<SW, ST>;
  using L = gg::masked::Layout<SW, ST>;
  static_assert(L::bytes(GG_MAX_EXPERTS) <= 227 * 1024, "shared memory of a CTA exceeded");
  cudaError_t ce = cudaSuccess;
  static std::atomic<bool> attr_done[kMaxDevices];
  static std::mutex mu;
  if (!attr_done[dev].load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lk(mu);
    if (!attr_done[dev].load(std::memory_order_relaxed)) {
      if ((ce = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)L::bytes(GG_MAX_EXPERTS))) != cudaSuccess)
        return cuda_fail("cudaFuncSetAttribute", ce);
      attr_done[dev].store(true, std::memory_order_release);
    }
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3((unsigned)units, 1, 1);
  cfg.blockDim = dim3(gg::masked::THREADS, 1, 1);
  cfg.dynamicSmemBytes = L::bytes(p.E);
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = GG_PDL != 0 ? 1 : 0;
  ce = cudaLaunchKernelEx(&cfg, kern, mw, mt[0], mt[1], mt[2], p);
  if (ce != cudaSuccess && cfg.numAttrs == 1) {
    (void)cudaGetLastError();
    cfg.numAttrs = 0;
    ce = cudaLaunchKernelEx(&cfg, kern, mw, mt[0], mt[1], mt[2], p);
  }
  if (ce != cudaSuccess) return cuda_fail("cudaLaunchKernelEx", ce);
  ce = cudaGetLastError();
  return ce == cudaSuccess ? GG_OK : cuda_fail("kernel launch", ce);
}

// Weight and token stages of the masked forward kernel, 16 KB each: a reduction step needs
// one of each (6 + 6, 7 + 5, 5 + 7 and 8 + 4 measured within 2% of one another on the
// sglang shape).
constexpr int kMaskedWStages = 6;
constexpr int kMaskedTStages = 6;

// Masked forward without an activation: the small-batch kernel of gg_masked.cuh (bias and
// per-row bias scale fused; checked as in set_epilogue).
gg_status masked_small_impl(const void* A, const void* W, const int32_t* masked_m, void* out,
                            int64_t mmax, int64_t K, int64_t N, int32_t E,
                            const gg_epilogue* epi, int32_t* dev_status, const DeviceInfo& di,
                            cudaStream_t stream) {
  gg::Params chk;
  std::memset(&chk, 0, sizeof(chk));
  gg_status s = set_epilogue(&chk, epi, N);
  if (s != GG_OK) return s;
  CUtensorMap mw, mt[3];
  const bool chunked = (N % 64) == 0;
  if (chunked ? !map_w_chunked(&mw, W, E, K, N, gg::masked::KBLK, 2)
              : !map_w(&mw, W, E, K, N, 64, gg::masked::KBLK))
    return GG_ERR_CUDA;
  // token rows in boxes of 32, 64 and 128 rows: one or two boxes cover a block's active rows
  for (int i = 0; i < 3; ++i)
    if (!map_2d(&mt[i], A, (int64_t)E * mmax, K, gg::masked::KBLK, 32u << i)) return GG_ERR_CUDA;
  gg::masked::Params p;
  std::memset(&p, 0, sizeof(p));
  p.masked_m = masked_m;
  p.out = reinterpret_cast<__nv_bfloat16*>(out);
  p.status = dev_status;
  p.bias = chk.bias;
  p.bias_scale = chk.bias_scale;
  p.E = E;
  p.mmax = (int32_t)mmax;
  p.K = (int32_t)K;
  p.N = (int32_t)N;
  p.watchdog_ns = g_watchdog_ns.load();
  p.debug_flags = g_skip_first_load.load() ? 1 : 0;
  p.w_chunked = chunked ? 1 : 0;
  // every (expert, row block, column tile), active or not; when each can have a CTA of its
  // own, the CTAs need no tile table (one-tile schedule)
  const int64_t tiles = (int64_t)E * cdiv(mmax, gg::masked::TILE_T) * cdiv(N, gg::masked::TILE_N);
  p.one_tile = tiles <= di.sms ? 1 : 0;
  const int64_t units = tiles < di.sms ? tiles : di.sms;
  return launch_masked<kMaskedWStages, kMaskedTStages>(mw, mt, p, units < 1 ? 1 : units, di.dev,
                                                       stream);
}

gg_status masked_impl(const void* A, const void* W, const int32_t* masked_m, void* out,
                      int64_t mmax, int64_t K, int64_t N, int32_t E, const gg_epilogue* epi,
                      int32_t* dev_status, cudaStream_t stream) {
  DeviceInfo di;
  if (mmax < 0) return GG_ERR_INVALID_ARG;
  if ((int64_t)E * mmax >= (int64_t(1) << 31)) return GG_ERR_UNSUPPORTED;
  gg_status s = check_common((int64_t)E * mmax, K, N, E, masked_m, dev_status, &di);
  if (s != GG_OK) return s;
  if (W == nullptr) return GG_ERR_INVALID_ARG;
  if (epi != nullptr && (epi->flags & ~GG_FLAG_GATE_UP_CONCAT)) return GG_ERR_INVALID_ARG;
  if (mmax == 0) return GG_OK;
  if (A == nullptr || out == nullptr) return GG_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(W) || !aligned16(out)) return GG_ERR_UNSUPPORTED;
  const bool silu = epi != nullptr && epi->act == GG_ACT_SILU_MUL;
  if (!silu)
    return masked_small_impl(A, W, masked_m, out, mmax, K, N, E, epi, dev_status, di, stream);
  // SiLU-and-mul needs the gate and up columns of a row in one tile: token rows as the MMA's
  // M, 256-wide column tiles (gate and up blocks of 128), A fetched in 32-row boxes covering
  // only the active rows.
  const int bn = kBN;
  const bool chunked = (N % 64) == 0;
  CUtensorMap ma, mb;
  if (!map_2d(&ma, A, (int64_t)E * mmax, K, 64, 32)) return GG_ERR_CUDA;
  const bool concat = (epi->flags & GG_FLAG_GATE_UP_CONCAT) != 0;  // 128-column blocks
  if (chunked ? !map_w_chunked(&mb, W, E, K, N, 64, (concat ? 128 : bn) / 64)
              : !map_w(&mb, W, E, K, N, 64, 64))
    return GG_ERR_CUDA;
  gg::Params p = base_params(masked_m, out, dev_status, (int64_t)E * mmax, E);
  p.b_chunked = chunked ? 1 : 0;
  p.mmax = (int32_t)mmax;
  p.red_len = (int32_t)K;
  if ((s = set_epilogue(&p, epi, N)) != GG_OK) return s;
  const int64_t out_cols = silu ? N / 2 : N;
  p.out_cols = (int32_t)out_cols;
  p.prod_cols = (int32_t)N;
  set_store_width(&p, out, out_cols);
  const int64_t tiles = (int64_t)E * cdiv(mmax, gg::BM) * cdiv(N, bn);
  return launch<Mode::Masked, kBN, kStages, false, false, 1>(ma, mb, p, tiles, di, stream);
}

}  // namespace

extern "C" {

gg_status gg_forward(const void* A, const void* W, const int32_t* offs, void* out,
                     int64_t rows_alloc, int64_t K, int64_t N, int32_t E, int32_t* dev_status,
                     cudaStream_t stream) {
  return forward_impl(A, W, offs, out, rows_alloc, K, N, E, nullptr, dev_status, stream);
}

gg_status gg_forward_ex(const void* A, const void* W, const int32_t* offs, void* out,
                        int64_t rows_alloc, int64_t K, int64_t N, int32_t E,
                        const gg_epilogue* epi, int32_t* dev_status, cudaStream_t stream) {
  return forward_impl(A, W, offs, out, rows_alloc, K, N, E, epi, dev_status, stream);
}

gg_status gg_masked_forward(const void* A, const void* W, const int32_t* masked_m, void* out,
                            int64_t mmax, int64_t K, int64_t N, int32_t E, int32_t* dev_status,
                            cudaStream_t stream) {
  return masked_impl(A, W, masked_m, out, mmax, K, N, E, nullptr, dev_status, stream);
}

gg_status gg_masked_forward_ex(const void* A, const void* W, const int32_t* masked_m, void* out,
                               int64_t mmax, int64_t K, int64_t N, int32_t E,
                               const gg_epilogue* epi, int32_t* dev_status,
                               cudaStream_t stream) {
  return masked_impl(A, W, masked_m, out, mmax, K, N, E, epi, dev_status, stream);
}

gg_status gg_dgrad(const void* dY, const void* W, const int32_t* offs, void* dX,
                   int64_t rows_alloc, int64_t K, int64_t N, int32_t E, int32_t* dev_status,
                   cudaStream_t stream) {
  return dgrad_impl(dY, W, offs, dX, rows_alloc, K, N, E, 0, dev_status, stream);
}

gg_status gg_dgrad_ex(const void* dY, const void* W, const int32_t* offs, void* dX,
                      int64_t rows_alloc, int64_t K, int64_t N, int32_t E, int32_t flags,
                      int32_t* dev_status, cudaStream_t stream) {
  return dgrad_impl(dY, W, offs, dX, rows_alloc, K, N, E, flags, dev_status, stream);
}

gg_status gg_wgrad(const void* A, const void* dY, const int32_t* offs, void* dW,
                   int64_t rows_alloc, int64_t K, int64_t N, int32_t E, int32_t* dev_status,
                   cudaStream_t stream) {
  return wgrad_impl(A, dY, offs, dW, false, 1.f, 0.f, rows_alloc, K, N, E, dev_status, stream);
}

gg_status gg_wgrad_ex(const void* A, const void* dY, const int32_t* offs, void* dW,
                      int64_t rows_alloc, int64_t K, int64_t N, int32_t E, int32_t flags,
                      int32_t* dev_status, cudaStream_t stream) {
  if (flags & ~GG_FLAG_W_NK) return GG_ERR_INVALID_ARG;
  if (flags & GG_FLAG_W_NK)  // dW[e] = dY_e^T A_e, stored [E, N, K]
    return wgrad_impl(dY, A, offs, dW, false, 1.f, 0.f, rows_alloc, N, K, E, dev_status, stream);
  return wgrad_impl(A, dY, offs, dW, false, 1.f, 0.f, rows_alloc, K, N, E, dev_status, stream);
}

gg_status gg_wgrad_f32(const void* A, const void* dY, const int32_t* offs, float* dW,
                       float alpha, float beta, int64_t rows_alloc, int64_t K, int64_t N,
                       int32_t E, int32_t* dev_status, cudaStream_t stream) {
  return wgrad_impl(A, dY, offs, dW, true, alpha, beta, rows_alloc, K, N, E, dev_status,
                    stream);
}

const char* gg_status_string(gg_status s) {
  switch (s) {
    case GG_OK: return "GG_OK";
    case GG_ERR_INVALID_ARG: return "GG_ERR_INVALID_ARG: a pointer, size or count is invalid";
    case GG_ERR_UNSUPPORTED:
      return "GG_ERR_UNSUPPORTED: unsupported device, alignment, size or expert count";
    case GG_ERR_CUDA: return "GG_ERR_CUDA: a CUDA runtime or driver call failed";
    case GG_ERR_TOO_LARGE:
      return "GG_ERR_TOO_LARGE: the problem needs more than the fixed scratch array of "
             "gg_route_noalloc (GG_ROUTE_NOALLOC_MAX_COUNTS entries)";
  }
  return "unknown gg_status";
}

uint64_t gg_set_watchdog_ns(uint64_t ns) {
  return g_watchdog_ns.exchange(ns == 0 ? kDefaultWatchdogNs : ns);
}

int gg_testing_skip_first_load(int enable) { return g_skip_first_load.exchange(enable ? 1 : 0); }

int gg_testing_force_variant(int variant) {
  return g_force_variant.exchange(variant >= 1 && variant <= 3 ? variant : 0);
}

int gg_version(void) { return 100; }

const char* gg_last_error(void) { return g_err; }

}  // extern "C"
