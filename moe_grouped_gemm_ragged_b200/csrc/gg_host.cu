// Forward + backward of the grouped GEMM layer on operands that live in host memory,
// streamed through the GPU by expert chunks: while chunk c computes on the caller's stream,
// the operands of chunk c+1 travel host -> device on one copy stream and the results of
// chunk c-1 travel device -> host on another (the host link is full duplex), so a pass costs
// about the larger of the two transfers instead of their sum plus the GEMMs. Each pass waits
// only for its own operands and each result leaves as soon as its pass is done: W and A
// travel first and the forward starts while dY is still on its way, and the forward's
// output goes back while dgrad and wgrad run, which shortens the start and the end of the
// pipeline.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "gg.h"

namespace ggh {

constexpr int kMaxChunks = 32;
constexpr int kMaxDevices = 64;
constexpr int kDefaultChunks = 16;

// Per device: the two copy streams and the events that order the three streams. They are
// created on first use and kept; one process-wide lock serialises the enqueueing, and an
// event may be recorded again once the waits on its previous recording are enqueued.
struct DeviceCtx {
  bool ready = false;
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t start = nullptr, done = nullptr;
  // per chunk: W and A loaded, dY loaded; forward, dgrad and wgrad done
  cudaEvent_t loaded_aw[kMaxChunks] = {}, loaded[kMaxChunks] = {};
  cudaEvent_t fwd_done[kMaxChunks] = {}, dgrad_done[kMaxChunks] = {}, computed[kMaxChunks] = {};
};
std::mutex g_mu;
DeviceCtx g_ctx[kMaxDevices];

gg_status device_ctx(DeviceCtx** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GG_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return GG_ERR_UNSUPPORTED;
  DeviceCtx& c = g_ctx[dev];
  if (!c.ready) {
    const unsigned ef = cudaEventDisableTiming;
    if (cudaStreamCreateWithFlags(&c.h2d, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&c.d2h, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&c.start, ef) != cudaSuccess ||
        cudaEventCreateWithFlags(&c.done, ef) != cudaSuccess)
      return GG_ERR_CUDA;
    for (int i = 0; i < kMaxChunks; ++i)
      if (cudaEventCreateWithFlags(&c.loaded_aw[i], ef) != cudaSuccess ||
          cudaEventCreateWithFlags(&c.loaded[i], ef) != cudaSuccess ||
          cudaEventCreateWithFlags(&c.fwd_done[i], ef) != cudaSuccess ||
          cudaEventCreateWithFlags(&c.dgrad_done[i], ef) != cudaSuccess ||
          cudaEventCreateWithFlags(&c.computed[i], ef) != cudaSuccess)
        return GG_ERR_CUDA;
    c.ready = true;
  }
  *out = &c;
  return GG_OK;
}

// Chunk c holds experts [e0[c], e0[c+1]) and rows [r0[c], r0[c+1]).
struct Chunks {
  int32_t n;
  int32_t e0[kMaxChunks + 1];
  int64_t r0[kMaxChunks + 1];
};

// offs[e] -= first row of e's chunk: the offsets each chunk's calls see are relative to the
// chunk's first row, which is row 0 of the operand pointers they get.
__global__ void relative_offsets(int32_t* offs, int32_t E, Chunks ch) {
  const int32_t e = (int32_t)(blockIdx.x * blockDim.x + threadIdx.x);
  if (e >= E) return;
  int c = 0;
  while (c + 1 < ch.n && ch.e0[c + 1] <= e) ++c;
  offs[e] -= (int32_t)ch.r0[c];
}

// Contiguous expert ranges with about T / n rows each; every chunk holds at least one expert.
Chunks split(const int32_t* offs, int32_t E, int32_t want) {
  Chunks ch{};
  const int64_t T = offs[E - 1];
  int32_t n = want <= 0 ? kDefaultChunks : want;
  if (n > kMaxChunks) n = kMaxChunks;
  if (n > E) n = E;
  int32_t c = 0;
  ch.e0[0] = 0;
  ch.r0[0] = 0;
  for (int32_t e = 1; e < E && c + 1 < n; ++e) {
    const int64_t start = offs[e - 1];
    if (start * n >= (int64_t)(c + 1) * T) {
      ++c;
      ch.e0[c] = e;
      ch.r0[c] = start;
    }
  }
  ch.n = c + 1;
  ch.e0[ch.n] = E;
  ch.r0[ch.n] = T;
  return ch;
}

}  // namespace ggh

extern "C" {

gg_status gg_layer_step_host(const void* A_h, const void* W_h, const void* dY_h,
                             const int32_t* offs_h, void* out_h, void* dX_h, void* dW_h,
                             void* A_d, void* W_d, void* dY_d, int32_t* offs_d, void* out_d,
                             void* dX_d, void* dW_d, int64_t rows, int64_t K, int64_t N,
                             int32_t E, int32_t chunks, int32_t* dev_status,
                             cudaStream_t stream) {
  using namespace ggh;
  if (E < 1 || K < 1 || N < 1 || rows < 0 || chunks < 0) return GG_ERR_INVALID_ARG;
  if (E > GG_MAX_EXPERTS) return GG_ERR_UNSUPPORTED;
  const void* ptrs[] = {A_h, W_h, dY_h, offs_h, out_h, dX_h, dW_h,
                        A_d, W_d, dY_d, offs_d, out_d, dX_d, dW_d};
  for (const void* p : ptrs)
    if (p == nullptr) return GG_ERR_INVALID_ARG;
  // the per-chunk calls' own layout rules, checked up front so that nothing is half enqueued
  if (K % 8 != 0 || N % 8 != 0) return GG_ERR_UNSUPPORTED;
  const void* dev_ptrs[] = {A_d, W_d, dY_d, out_d, dX_d, dW_d};
  for (const void* p : dev_ptrs)
    if ((reinterpret_cast<uintptr_t>(p) & 15u) != 0) return GG_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(offs_d) & 3u) != 0) return GG_ERR_UNSUPPORTED;
  // the offsets are host data here: checked before anything is enqueued
  int32_t prev = 0;
  for (int32_t e = 0; e < E; ++e) {
    if (offs_h[e] < prev || offs_h[e] > rows) return GG_ERR_INVALID_ARG;
    prev = offs_h[e];
  }
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceCtx* cx = nullptr;
  gg_status s = device_ctx(&cx);
  if (s != GG_OK) return s;
  const Chunks ch = split(offs_h, E, chunks);
  const size_t eb = 2;  // bytes per bf16 element
  const size_t w_bytes = (size_t)K * (size_t)N * eb;  // one expert's weight (or dW) slice
  auto at = [](const void* base, size_t off) {
    return static_cast<char*>(const_cast<void*>(base)) + off;
  };
  auto ok = [](cudaError_t e) { return e == cudaSuccess; };

  // the copies start after the work the caller enqueued before this call
  if (!ok(cudaEventRecord(cx->start, stream)) || !ok(cudaStreamWaitEvent(cx->h2d, cx->start, 0)) ||
      !ok(cudaStreamWaitEvent(cx->d2h, cx->start, 0)))
    return GG_ERR_CUDA;
  if (!ok(cudaMemcpyAsync(offs_d, offs_h, sizeof(int32_t) * (size_t)E, cudaMemcpyHostToDevice,
                          cx->h2d)))
    return GG_ERR_CUDA;
  relative_offsets<<<(E + 255) / 256, 256, 0, cx->h2d>>>(offs_d, E, ch);
  if (!ok(cudaGetLastError())) return GG_ERR_CUDA;

  for (int32_t c = 0; c < ch.n && s == GG_OK; ++c) {
    const int64_t r0 = ch.r0[c], nr = ch.r0[c + 1] - ch.r0[c];
    const int32_t e0 = ch.e0[c], ne = ch.e0[c + 1] - ch.e0[c];
    const size_t a_off = (size_t)r0 * (size_t)K * eb, y_off = (size_t)r0 * (size_t)N * eb;
    const size_t w_off = (size_t)e0 * w_bytes;
    // W and A (the forward's operands), then dY
    if (!ok(cudaMemcpyAsync(at(W_d, w_off), at(W_h, w_off), (size_t)ne * w_bytes,
                            cudaMemcpyHostToDevice, cx->h2d)) ||
        !ok(cudaMemcpyAsync(at(A_d, a_off), at(A_h, a_off), (size_t)nr * K * eb,
                            cudaMemcpyHostToDevice, cx->h2d)) ||
        !ok(cudaEventRecord(cx->loaded_aw[c], cx->h2d)) ||
        !ok(cudaMemcpyAsync(at(dY_d, y_off), at(dY_h, y_off), (size_t)nr * N * eb,
                            cudaMemcpyHostToDevice, cx->h2d)) ||
        !ok(cudaEventRecord(cx->loaded[c], cx->h2d)) ||
        !ok(cudaStreamWaitEvent(stream, cx->loaded_aw[c], 0))) {
      s = GG_ERR_CUDA;
      break;
    }
    const int32_t* offs_c = offs_d + e0;
    s = gg_forward(at(A_d, a_off), at(W_d, w_off), offs_c, at(out_d, y_off), nr, K, N, ne,
                   dev_status, stream);
    if (s != GG_OK) break;
    // the forward's output leaves while dY arrives and the backward passes run
    if (!ok(cudaEventRecord(cx->fwd_done[c], stream)) ||
        !ok(cudaStreamWaitEvent(cx->d2h, cx->fwd_done[c], 0)) ||
        !ok(cudaMemcpyAsync(at(out_h, y_off), at(out_d, y_off), (size_t)nr * N * eb,
                            cudaMemcpyDeviceToHost, cx->d2h)) ||
        !ok(cudaStreamWaitEvent(stream, cx->loaded[c], 0))) {
      s = GG_ERR_CUDA;
      break;
    }
    s = gg_dgrad(at(dY_d, y_off), at(W_d, w_off), offs_c, at(dX_d, a_off), nr, K, N, ne,
                 dev_status, stream);
    if (s != GG_OK) break;
    if (!ok(cudaEventRecord(cx->dgrad_done[c], stream)) ||
        !ok(cudaStreamWaitEvent(cx->d2h, cx->dgrad_done[c], 0)) ||
        !ok(cudaMemcpyAsync(at(dX_h, a_off), at(dX_d, a_off), (size_t)nr * K * eb,
                            cudaMemcpyDeviceToHost, cx->d2h))) {
      s = GG_ERR_CUDA;
      break;
    }
    s = gg_wgrad(at(A_d, a_off), at(dY_d, y_off), offs_c, at(dW_d, w_off), nr, K, N, ne,
                 dev_status, stream);
    if (s != GG_OK) break;
    if (!ok(cudaEventRecord(cx->computed[c], stream)) ||
        !ok(cudaStreamWaitEvent(cx->d2h, cx->computed[c], 0)) ||
        !ok(cudaMemcpyAsync(at(dW_h, w_off), at(dW_d, w_off), (size_t)ne * w_bytes,
                            cudaMemcpyDeviceToHost, cx->d2h)))
      s = GG_ERR_CUDA;
  }
  // whatever was enqueued on either copy stream, the caller's stream is ordered after it
  if (!ok(cudaEventRecord(cx->done, cx->d2h)) || !ok(cudaStreamWaitEvent(stream, cx->done, 0)) ||
      !ok(cudaEventRecord(cx->start, cx->h2d)) || !ok(cudaStreamWaitEvent(stream, cx->start, 0)))
    return GG_ERR_CUDA;
  return s;
}

}  // extern "C"
