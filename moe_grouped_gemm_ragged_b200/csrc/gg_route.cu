// Token routing into the packed layout of the ragged grouped GEMM: per-expert cumulative end
// offsets, the packed row of every (token, slot) assignment and the packed activations,
// all on the device. A stable counting sort over the flattened assignments in three
// launches: per-block histograms, one scan, and a scatter that also copies the rows.
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "gg.h"

namespace ggr {

// The library is built for sm_100a only: the device must be compute capability 10.0 exactly.
gg_status check_device() {
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return GG_ERR_CUDA;
  return (major == 10 && minor == 0) ? GG_OK : GG_ERR_UNSUPPORTED;
}

constexpr int THREADS = 256;          // one assignment per thread and block
constexpr int WARPS = THREADS / 32;
constexpr int CHUNK = THREADS;        // assignments per block
constexpr int32_t DEV_BAD_ROUTE = 0x8;
static_assert(DEV_BAD_ROUTE == GG_DEV_BAD_ROUTE, "status bit mismatch");

// Histogram of the block's chunk: counts[e * nblk + b] for block b of nblk (ids < 0 are dropped
// silently, ids >= E are dropped and flagged). Expert-major, so that the scan reads the
// counts of one expert with consecutive lanes.
__global__ void __launch_bounds__(THREADS) count_kernel(const int32_t* __restrict__ ids,
                                                        int64_t n, int32_t E,
                                                        int32_t* __restrict__ counts,
                                                        int32_t* status) {
  __shared__ int32_t hist[GG_MAX_EXPERTS];
  for (int e = threadIdx.x; e < E; e += THREADS) hist[e] = 0;
  __syncthreads();
  const int64_t i = (int64_t)blockIdx.x * CHUNK + threadIdx.x;
  bool bad = false;
  if (i < n) {
    const int32_t e = ids[i];
    if (e >= 0 && e < E) atomicAdd(&hist[e], 1);
    bad = e >= E;
  }
  bad = __syncthreads_or(bad);
  for (int e = threadIdx.x; e < E; e += THREADS)
    counts[(int64_t)e * gridDim.x + blockIdx.x] = hist[e];
  if (bad && threadIdx.x == 0 && status != nullptr) atomicOr(status, DEV_BAD_ROUTE);
}

// One block: offs[e] = cumulative end of expert e; counts[e][b] becomes the first packed row
// of block b's assignments to expert e. Each expert's blocks are cut into P segments (P a
// power of two, 32 / E rounded down for fewer than 32 experts, else 1), one warp per segment
// at a time: the warp sums its segment with consecutive lanes on consecutive blocks, one
// exclusive scan runs over the E * P segment sums in (expert, segment) order, and each warp
// then turns its segment's counts into starts with a running warp-wide scan.
__device__ __forceinline__ int32_t warp_incl_scan(int32_t v, int lane) {
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int32_t o = __shfl_up_sync(0xffffffffu, v, d);
    if (lane >= d) v += o;
  }
  return v;
}

__global__ void __launch_bounds__(1024) scan_kernel(int32_t* __restrict__ counts, int32_t nblk,
                                                    int32_t E, int32_t* __restrict__ offs) {
  constexpr int U = 8;                        // loads in flight per lane
  __shared__ int32_t seg[GG_MAX_EXPERTS];     // per segment: sum, then exclusive start
  __shared__ int32_t warp_sum[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int P = 1;
  while (P * 2 * E <= 32) P *= 2;
  const int32_t S = E * P;                    // at most GG_MAX_EXPERTS segments
  const int32_t span = (nblk + P - 1) / P;
  // segment sg = e * P + p covers blocks [p * span, min((p + 1) * span, nblk)) of expert e
  for (int32_t sg = warp; sg < S; sg += 32) {
    const int32_t e = sg / P, p = sg % P;
    const int32_t b0 = min(p * span, nblk), b1 = min(b0 + span, nblk);
    const int32_t* row = counts + (int64_t)e * nblk;
    int32_t sum = 0;
    for (int32_t b = b0 + lane; b < b1; b += 32 * U) {
      int32_t c[U];
#pragma unroll
      for (int u = 0; u < U; ++u) c[u] = b + 32 * u < b1 ? row[b + 32 * u] : 0;
#pragma unroll
      for (int u = 0; u < U; ++u) sum += c[u];
    }
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, d);
    if (lane == 0) seg[sg] = sum;
  }
  __syncthreads();
  // block-wide exclusive scan of the segment sums (thread x takes segment x); the end of an
  // expert's last segment is its cumulative end offset
  const int32_t tx = (int)threadIdx.x < S ? seg[threadIdx.x] : 0;
  const int32_t v = warp_incl_scan(tx, lane);
  if (lane == 31) warp_sum[warp] = v;
  __syncthreads();
  if (warp == 0) warp_sum[lane] = warp_incl_scan(warp_sum[lane], lane);
  __syncthreads();
  if ((int)threadIdx.x < S) {
    const int32_t incl = v + (warp > 0 ? warp_sum[warp - 1] : 0);
    seg[threadIdx.x] = incl - tx;
    if ((int)threadIdx.x % P == P - 1) offs[threadIdx.x / P] = incl;
  }
  __syncthreads();
  for (int32_t sg = warp; sg < S; sg += 32) {
    const int32_t e = sg / P, p = sg % P;
    const int32_t b0 = min(p * span, nblk), b1 = min(b0 + span, nblk);
    int32_t* row = counts + (int64_t)e * nblk;
    int32_t carry = seg[sg];
    for (int32_t b = b0 + lane; b - lane < b1; b += 32 * U) {
      int32_t c[U];
#pragma unroll
      for (int u = 0; u < U; ++u) c[u] = b + 32 * u < b1 ? row[b + 32 * u] : 0;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int32_t incl = warp_incl_scan(c[u], lane);
        if (b + 32 * u < b1) row[b + 32 * u] = carry + incl - c[u];
        carry += __shfl_sync(0xffffffffu, incl, 31);
      }
    }
  }
}

// Stable ranks inside the block (warp by warp, lane by lane), row_of, and the row copies.
__global__ void __launch_bounds__(THREADS) scatter_kernel(
    const int32_t* __restrict__ ids, int64_t n, int32_t k, int32_t E,
    const int32_t* __restrict__ bases, const uint4* __restrict__ X, int64_t row_vecs,
    uint4* __restrict__ A_packed, int32_t* __restrict__ row_of) {
  extern __shared__ int32_t whist[];  // [WARPS][E]: per-warp counts, then per-warp bases
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < WARPS * E; i += THREADS) whist[i] = 0;
  __syncthreads();
  const int64_t i = (int64_t)blockIdx.x * CHUNK + threadIdx.x;
  const int32_t e = i < n ? ids[i] : -1;
  const bool valid = e >= 0 && e < E;
  // lanes with the same expert form one peer set; an invalid lane is alone
  const uint32_t peers = __match_any_sync(0xffffffffu, valid ? e : -1 - lane);
  const uint32_t rank = __popc(peers & ((1u << lane) - 1u));
  if (valid && rank == 0) whist[warp * E + e] = __popc(peers);
  __syncthreads();
  // exclusive scan over warps per expert, starting at the block's base
  for (int x = threadIdx.x; x < E; x += THREADS) {
    int32_t run = bases[(int64_t)x * gridDim.x + blockIdx.x];
    for (int w = 0; w < WARPS; ++w) {
      const int32_t c = whist[w * E + x];
      whist[w * E + x] = run;
      run += c;
    }
  }
  __syncthreads();
  const int32_t dest = valid ? whist[warp * E + e] + (int32_t)rank : -1;
  if (i < n) row_of[i] = dest;
  // Row copies. The lanes of one token are consecutive (i = t * k + slot), so the warp
  // reads each token's row once, 512 bytes per lane step, and stores that piece to every
  // destination of the token (reading the row once per slot re-read it from DRAM k times).
  // Every loop below is warp-uniform: its bounds come from ballots and shuffles.
  const int64_t tok = i / k;
  const int64_t tok_prev = __shfl_up_sync(0xffffffffu, tok, 1);
  uint32_t leaders = __ballot_sync(0xffffffffu, i < n && (lane == 0 || tok != tok_prev));
  const uint32_t has_dest = __ballot_sync(0xffffffffu, dest >= 0);
  while (leaders != 0u) {
    const int j = __ffs(leaders) - 1;
    leaders &= leaders - 1u;
    const int jend = leaders != 0u ? __ffs(leaders) - 1 : 32;
    const uint32_t upto = jend == 32 ? 0xffffffffu : ((1u << jend) - 1u);
    const uint32_t grp = upto & ~((1u << j) - 1u) & has_dest;  // lanes of this token
    if (grp == 0u) continue;  // every slot of the token dropped
    const int64_t t = __shfl_sync(0xffffffffu, tok, j);
    const uint4* src = X + t * row_vecs;
    for (int64_t base = 0; base < row_vecs; base += 128) {
      uint4 x[4] = {};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t v = base + lane + 32 * u;
        if (v < row_vecs) x[u] = src[v];
      }
      uint32_t g = grp;
      while (g != 0u) {
        const int jj = __ffs(g) - 1;
        g &= g - 1u;
        const int32_t d = __shfl_sync(0xffffffffu, dest, jj);
        uint4* dst = A_packed + (int64_t)d * row_vecs;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int64_t v = base + lane + 32 * u;
          if (v < row_vecs) __stcs(dst + v, x[u]);  // written once, read by the next kernel
        }
      }
    }
  }
}

int64_t blocks_for(int64_t n) { return (n + CHUNK - 1) / CHUNK; }

}  // namespace ggr

extern "C" {

size_t gg_route_workspace_bytes(int64_t n_assign, int32_t E) {
  if (n_assign < 0 || E < 1) return 0;
  return (size_t)ggr::blocks_for(n_assign) * (size_t)E * sizeof(int32_t);
}

gg_status gg_route(const int32_t* topk_ids, int64_t T_tok, int32_t k, int32_t E, const void* X,
                   int64_t K, void* A_packed, int32_t* row_of, int32_t* offs, void* workspace,
                   size_t workspace_bytes, int32_t* dev_status, cudaStream_t stream) {
  using namespace ggr;
  if (T_tok < 0 || k < 1 || E < 1 || K < 1) return GG_ERR_INVALID_ARG;
  if (E > GG_MAX_EXPERTS) return GG_ERR_UNSUPPORTED;
  if (K % 8 != 0) return GG_ERR_UNSUPPORTED;
  const int64_t n = T_tok * (int64_t)k;
  if (n >= (int64_t(1) << 31)) return GG_ERR_UNSUPPORTED;
  if (offs == nullptr) return GG_ERR_INVALID_ARG;
  if (n > 0 && (topk_ids == nullptr || X == nullptr || A_packed == nullptr ||
                row_of == nullptr || workspace == nullptr))
    return GG_ERR_INVALID_ARG;
  auto mis = [](const void* p, uintptr_t a) {
    return (reinterpret_cast<uintptr_t>(p) & (a - 1)) != 0;
  };
  if (mis(topk_ids, 4) || mis(row_of, 4) || mis(offs, 4) || mis(workspace, 4) ||
      mis(X, 16) || mis(A_packed, 16) || (dev_status != nullptr && mis(dev_status, 4)))
    return GG_ERR_UNSUPPORTED;
  if (workspace_bytes < gg_route_workspace_bytes(n, E)) return GG_ERR_INVALID_ARG;
  const gg_status ds = check_device();
  if (ds != GG_OK) return ds;
  const int64_t nblk = blocks_for(n);
  int32_t* counts = reinterpret_cast<int32_t*>(workspace);
  if (nblk > 0)
    count_kernel<<<(unsigned)nblk, THREADS, 0, stream>>>(topk_ids, n, E, counts, dev_status);
  scan_kernel<<<1, 1024, 0, stream>>>(counts, (int32_t)nblk, E, offs);  // nblk 0: offs = 0
  if (nblk == 0) return cudaGetLastError() == cudaSuccess ? GG_OK : GG_ERR_CUDA;
  const size_t smem = sizeof(int32_t) * WARPS * (size_t)E;
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return GG_ERR_CUDA;
  scatter_kernel<<<(unsigned)nblk, THREADS, smem, stream>>>(
      topk_ids, n, k, E, counts, reinterpret_cast<const uint4*>(X), K / 8,
      reinterpret_cast<uint4*>(A_packed), row_of);
  return cudaGetLastError() == cudaSuccess ? GG_OK : GG_ERR_CUDA;
}

}  // extern "C"

// ---------------------------------------------------------------- allocation-free routing
// gg_route_noalloc serves callers that cannot allocate device memory where they call the
// router (for example a runtime whose device memory is reserved up front by its own
// allocator, or code that must not enter the CUDA allocator at that point). Its per-block
// histograms live in this fixed array instead of a caller-provided workspace. Every GPU that
// loads the library holds the array (1 MiB) until the process exits. Host code only sees a
// stand-in for it, so its device address is looked up with cudaGetSymbolAddress while the
// device is current: once per device and context (a context that is destroyed and created
// again, e.g. after cudaDeviceReset, reloads the module, and the array may move).
static __device__ __align__(256) int32_t g_route_counts[GG_ROUTE_NOALLOC_MAX_COUNTS];

namespace ggr {

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
struct NoallocSlot {
  int32_t* counts = nullptr;
  unsigned long long ctx_id = 0;  // context the address belongs to
};
NoallocSlot g_noalloc[kMaxDevices];

// Unique id of the calling thread's current context (driver entry points, no link to the
// driver library); 0 when there is none or it cannot be read.
unsigned long long current_ctx_id() {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(f);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(f);
  });
  CUcontext c = nullptr;
  unsigned long long id = 0;
  if (get_current == nullptr || get_id == nullptr || get_current(&c) != CUDA_SUCCESS ||
      c == nullptr || get_id(c, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of g_route_counts on the current device, looked up on the first call in
// each context.
gg_status noalloc_counts(int32_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GG_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return GG_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  NoallocSlot& slot = g_noalloc[dev];
  const unsigned long long ctx = current_ctx_id();
  if (slot.counts == nullptr || ctx == 0 || ctx != slot.ctx_id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_counts) != cudaSuccess || p == nullptr)
      return GG_ERR_CUDA;
    slot.counts = static_cast<int32_t*>(p);
    slot.ctx_id = current_ctx_id();  // the lookup made the device's context current
  }
  *out = slot.counts;
  return GG_OK;
}

}  // namespace ggr

extern "C" {

gg_status gg_route_noalloc(const int32_t* topk_ids, int64_t T_tok, int32_t k, int32_t E,
                           const void* X, int64_t K, void* A_packed, int32_t* row_of,
                           int32_t* offs, int32_t* dev_status, cudaStream_t stream) {
  using namespace ggr;
  if (T_tok < 0 || k < 1 || E < 1 || K < 1) return GG_ERR_INVALID_ARG;
  if (E > GG_MAX_EXPERTS) return GG_ERR_UNSUPPORTED;
  if (K % 8 != 0) return GG_ERR_UNSUPPORTED;
  const int64_t n = T_tok * (int64_t)k;
  if (n >= (int64_t(1) << 31)) return GG_ERR_UNSUPPORTED;
  const int64_t nblk = blocks_for(n);
  if (nblk * (int64_t)E > GG_ROUTE_NOALLOC_MAX_COUNTS) return GG_ERR_TOO_LARGE;
  if (offs == nullptr) return GG_ERR_INVALID_ARG;
  if (n > 0 && (topk_ids == nullptr || X == nullptr || A_packed == nullptr ||
                row_of == nullptr))
    return GG_ERR_INVALID_ARG;
  auto mis = [](const void* p, uintptr_t a) {
    return (reinterpret_cast<uintptr_t>(p) & (a - 1)) != 0;
  };
  if (mis(topk_ids, 4) || mis(row_of, 4) || mis(offs, 4) || mis(X, 16) || mis(A_packed, 16) ||
      (dev_status != nullptr && mis(dev_status, 4)))
    return GG_ERR_UNSUPPORTED;
  const gg_status ds = check_device();  // before the symbol is touched or anything launches
  if (ds != GG_OK) return ds;
  int32_t* counts = nullptr;
  const gg_status s = noalloc_counts(&counts);
  if (s != GG_OK) return s;
  // The histogram kernel writes every entry the later kernels read, so the array needs no
  // clearing; calls that overlap on the GPU share it and race.
  if (nblk > 0)
    count_kernel<<<(unsigned)nblk, THREADS, 0, stream>>>(topk_ids, n, E, counts, dev_status);
  scan_kernel<<<1, 1024, 0, stream>>>(counts, (int32_t)nblk, E, offs);
  if (nblk == 0) return cudaGetLastError() == cudaSuccess ? GG_OK : GG_ERR_CUDA;
  const size_t smem = sizeof(int32_t) * WARPS * (size_t)E;
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return GG_ERR_CUDA;
  scatter_kernel<<<(unsigned)nblk, THREADS, smem, stream>>>(
      topk_ids, n, k, E, counts, reinterpret_cast<const uint4*>(X), K / 8,
      reinterpret_cast<uint4*>(A_packed), row_of);
  return cudaGetLastError() == cudaSuccess ? GG_OK : GG_ERR_CUDA;
}

}  // extern "C"
