/*
 * gg.h -- ragged MoE grouped GEMM on NVIDIA B200 (sm_100a), C ABI.
 *
 * Operations (bf16 inputs, fp32 accumulation in tensor memory, bf16 outputs rounded to
 * nearest even):
 *
 *   gg_forward         out[r,:] = A[r,:] . W[e]            for every row r of group e
 *   gg_dgrad           dX[r,:]  = dY[r,:] . W[e]^T         for every row r of group e
 *   gg_wgrad           dW[e]    = A[rows of e]^T . dY[rows of e]   (overwrite)
 *   gg_masked_forward  out[e,r,:] = A[e,r,:] . W[e]        for r < masked_m[e]
 *
 * Groups. offs[E] holds cumulative END offsets with no leading zero: group e covers rows
 * [offs[e-1], offs[e]) with offs[-1] = 0. This is the contract of torch._grouped_mm(x, w,
 * offs) in PyTorch issue 152668 ("Easy repro scenario": 4 experts, offsets (8,16,32,40)
 * over 48 rows, and the empty-expert variant (8,8,32,40)). A group may be empty and may have
 * any size; no alignment is asked of the sizes (TransformerEngine PR 3224 names an
 * alignment contract on m_splits that this library does not have).
 *
 * Offsets and masked_m are read only on the device (TransformerEngine PR 3542, "Changes":
 * the per-expert row counts stay in GPU memory). No call synchronises with the host, allocates
 * memory, pads A or clears an output (TileOPs issue 1566, "Summary": the per-call zero
 * fill and pad cost ~2.8 ms on a ~20 ms GEMM). Every call is ordered on the caller's
 * stream and may be captured in a CUDA graph; the offsets may change between replays.
 * (gg_layer_step_host, whose operands are host data, is the exception: it reads the
 * offsets on the host and is not for stream capture; see its description.)
 * The grouped GEMM kernels are launched with programmatic dependent launch: one may be
 * scheduled while the kernel before it on the stream is still finishing, and it waits for
 * that kernel's completion (and its memory) before its first global read or write, so the
 * stream order above holds for any producer of the inputs. A stream that refuses such a
 * launch gets a plain one.
 *
 * Memory. All pointers are device pointers owned by the caller, on the device that is
 * current when the call is made (the kernels run there); bf16 arrays are row major
 * (last index contiguous) and 16-byte aligned. W is one packed [E,K,N] buffer (the single
 * grouped weight of TransformerEngine PR 3224). K and N must be multiples of 8.
 *
 * Untouched regions (TransformerEngine PR 3542, "Changes": outputs live in buffers the caller
 * owns, and their rows beyond the used capacity keep their contents):
 *   - out/dX rows at or past the last (effective) offset are never written, and A/dY rows
 *     there are never read into any result;
 *   - masked rows r >= masked_m[e] of out are never written; A rows there never reach a
 *     result (sglang PR 32385, "Fix": masked_m excludes them from the GEMM);
 *   - dW is always written in full; the dW of an empty expert is +0.0 everywhere.
 *
 * Errors. Problems visible on the host return a gg_status at once and launch nothing.
 * Problems in device-resident data are never fatal: the kernel ORs a GG_DEV_* bit into
 * *dev_status (when dev_status is not NULL), treats the offending group as described
 * below, and still computes every valid group. No call traps, asserts or hangs: every wait
 * inside a kernel is bounded by a watchdog, after which the kernel sets GG_DEV_TIMEOUT,
 * drains its own copies in flight, frees its tensor memory and returns.
 */
#ifndef GG_H_
#define GG_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime.h>

#if defined(__GNUC__)
#define GG_API __attribute__((visibility("default")))
#else
#define GG_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GG_OK = 0,
  GG_ERR_INVALID_ARG = 1,  /* null pointer, negative or zero size, E < 1, ...          */
  GG_ERR_UNSUPPORTED = 2,  /* K or N not a multiple of 8, misaligned pointer, E too large,
                              rows >= 2^31, or a device that is not sm_100                */
  GG_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed (launch, attribute, ...) */
  GG_ERR_TOO_LARGE = 4     /* gg_route_noalloc: the problem needs more than its fixed
                              scratch array (GG_ROUTE_NOALLOC_MAX_COUNTS entries)          */
} gg_status;

/* Bits OR-ed into *dev_status by the kernels. */
#define GG_DEV_BAD_OFFSETS  0x1u  /* an offset was negative, decreasing or > rows_alloc; the
                                     effective ends t'_e = clamp(offs[e], t'_{e-1},
                                     rows_alloc) (t'_{-1}=0) were used instead            */
#define GG_DEV_BAD_MASKED_M 0x2u  /* a masked_m was < 0 or > mmax; it was clamped         */
#define GG_DEV_TIMEOUT      0x4u  /* a pipeline wait exceeded the watchdog; results of this
                                     call are incomplete                                  */
#define GG_DEV_BAD_ROUTE    0x8u  /* gg_route: an expert id was >= E; that assignment was
                                     dropped                                              */
#define GG_DEV_ERROR_MASK   0xFFu
#define GG_DEV_LAUNCHED     0x100u /* informational: the sm_100a kernel ran to its end     */

/* Largest expert count a call accepts. */
#define GG_MAX_EXPERTS 1024

/*
 * Forward: out[r, n] = sum_k A[r, k] * W[e, k, n] for every row r of group e.
 *   A    bf16 [rows_alloc, K]      read only for rows inside a group
 *   W    bf16 [E, K, N]
 *   offs int32 [E], device         cumulative end offsets
 *   out  bf16 [rows_alloc, N]      rows inside a group overwritten; other rows untouched
 *   dev_status int32, device, may be NULL
 * Passage: PyTorch issue 152668, "Easy repro scenario" (o = torch._grouped_mm(x, w, offs)).
 */
GG_API gg_status gg_forward(const void* A, const void* W, const int32_t* offs, void* out,
                     int64_t rows_alloc, int64_t K, int64_t N, int32_t E,
                     int32_t* dev_status, cudaStream_t stream);

/*
 * Dgrad: dX[r, k] = sum_n dY[r, n] * W[e, k, n] for every row r of group e.
 *   dY bf16 [rows_alloc, N]; W bf16 [E, K, N]; dX bf16 [rows_alloc, K] (rows outside every
 *   group untouched).
 * Passage: PyTorch issue 152668 (o.backward: the grad of x over the same offsets);
 * TransformerEngine PR 3542, "Changes" (forward, dgrad and wgrad through one grouped GEMM).
 */
GG_API gg_status gg_dgrad(const void* dY, const void* W, const int32_t* offs, void* dX,
                   int64_t rows_alloc, int64_t K, int64_t N, int32_t E,
                   int32_t* dev_status, cudaStream_t stream);

/*
 * Wgrad: dW[e, k, n] = sum over rows r of group e of A[r, k] * dY[r, n].
 *   A bf16 [rows_alloc, K]; dY bf16 [rows_alloc, N]; dW bf16 [E, K, N], written in full
 *   (overwrite, not accumulate); an empty group yields +0.0.
 * Passage: TransformerEngine PR 3542, "Changes" ("overwrite wgrad"); PyTorch issue 152668
 * (the backward that must not hang on an empty expert).
 */
GG_API gg_status gg_wgrad(const void* A, const void* dY, const int32_t* offs, void* dW,
                   int64_t rows_alloc, int64_t K, int64_t N, int32_t E,
                   int32_t* dev_status, cudaStream_t stream);

/* gg_dgrad with flags: GG_FLAG_ZERO_TAIL (dX rows past the last offset become 0) and
   GG_FLAG_W_NK (W is [E, N, K]). */
GG_API gg_status gg_dgrad_ex(const void* dY, const void* W, const int32_t* offs, void* dX,
                             int64_t rows_alloc, int64_t K, int64_t N, int32_t E,
                             int32_t flags, int32_t* dev_status, cudaStream_t stream);

/* gg_wgrad with flags: GG_FLAG_W_NK writes dW as [E, N, K] (dW[e] = dY_e^T . A_e). */
GG_API gg_status gg_wgrad_ex(const void* A, const void* dY, const int32_t* offs, void* dW,
                             int64_t rows_alloc, int64_t K, int64_t N, int32_t E,
                             int32_t flags, int32_t* dev_status, cudaStream_t stream);

/*
 * Wgrad into an fp32 buffer with scaling and accumulation (the main-grad update):
 *   dW[e, k, n] = alpha * sum over rows r of group e of A[r, k] * dY[r, n]
 *                 + beta * dW[e, k, n]
 *   A bf16 [rows_alloc, K]; dY bf16 [rows_alloc, N]; dW fp32 [E, K, N], read (only when
 *   beta != 0) and written in full, in place; an empty group gives beta * dW (0 when
 *   beta == 0). The product is accumulated in fp32 and added without a bf16 rounding.
 * Passage: TransformerEngine PR 3542, "Changes" (FP32 outputs, fused accumulation and
 * explicit alpha/beta; a rounded BF16 product added separately would not keep the fused
 * accumulation's precision).
 */
GG_API gg_status gg_wgrad_f32(const void* A, const void* dY, const int32_t* offs, float* dW,
                              float alpha, float beta, int64_t rows_alloc, int64_t K,
                              int64_t N, int32_t E, int32_t* dev_status, cudaStream_t stream);

/*
 * Masked forward: out[e, r, n] = sum_k A[e, r, k] * W[e, k, n] for r < masked_m[e].
 *   A bf16 [E, mmax, K]; W bf16 [E, K, N]; masked_m int32 [E], device;
 *   out bf16 [E, mmax, N]: rows r >= masked_m[e] untouched.
 * Passage: sglang PR 32385, "Evidence" and "Fix" (the masked grouped GEMM
 * m_grouped_gemm_nt_masked(a, b, d, masked_m, expected_m); its expected-m hint has no
 * counterpart here).
 */
GG_API gg_status gg_masked_forward(const void* A, const void* W, const int32_t* masked_m,
                            void* out, int64_t mmax, int64_t K, int64_t N, int32_t E,
                            int32_t* dev_status, cudaStream_t stream);

/* Forward epilogue fused into gg_forward_ex / gg_masked_forward_ex.
 *   h[r, n] = sum_k A[r, k] * W[e, k, n] + s[r] * bias[e, n]
 *     bias        bf16 [E, N], 16-byte aligned, or NULL (no bias)
 *     bias_scale  fp32, indexed by output row (the flat row e*mmax + r in the masked layout);
 *                 read only for rows inside a group, i.e. the logical tokens, never for the
 *                 unused capacity; NULL means s = 1. Ignored when bias is NULL.
 *   act GG_ACT_NONE:     out[r, n] = h[r, n]                      (out has N columns)
 *   act GG_ACT_SILU_MUL: gate and up columns interleaved in blocks of 128 inside every block
 *                        of 256 columns (N % 256 == 0, else GG_ERR_UNSUPPORTED):
 *                        out[r, 128 b + i] = silu(h[r, 256 b + i]) * h[r, 256 b + 128 + i],
 *                        silu(x) = x / (1 + e^-x)                 (out has N / 2 columns)
 * Passages: TransformerEngine PR 3542 review (a bias per group, a bias scale per token, the
 * scaling limited to the logical rows and not the capacity); sglang PR 32385, "Cause"
 * (SiLU-and-mul between the gate-up and the down GEMM, written only for active rows). */
#define GG_ACT_NONE 0
#define GG_ACT_SILU_MUL 1
/* Flags of the _ex entry points.
 *   GG_FLAG_ZERO_TAIL  forward, dgrad: rows of out / dX at and past the last effective offset
 *                      are written with zeros (a complete tensor, e.g. for autograd) instead
 *                      of being left untouched
 *   GG_FLAG_W_NK       W (and dW) stored [E, N, K]: each expert's weight out-major, the way
 *                      TransformerEngine's GroupedLinear keeps it (TransformerEngine PR 3542,
 *                      "Changes": dispatch of the transposed operand layouts); forward
 *                      computes A . W[e]^T
 *   GG_FLAG_GATE_UP_CONCAT  with GG_ACT_SILU_MUL only (else GG_ERR_INVALID_ARG): gate and up
 *                      are the two halves of W's N columns, [gate | up], the usual layout of
 *                      a fused gate-up weight: out[r, j] = silu(h[r, j]) * h[r, N/2 + j]
 *                      (N % 256 == 0); accepted by gg_forward_ex and gg_masked_forward_ex */
#define GG_FLAG_ZERO_TAIL 0x1
#define GG_FLAG_W_NK 0x2
#define GG_FLAG_GATE_UP_CONCAT 0x4
typedef struct gg_epilogue {
  const void* bias;
  const float* bias_scale;
  int32_t act;
  int32_t flags; /* GG_FLAG_ZERO_TAIL | GG_FLAG_W_NK | GG_FLAG_GATE_UP_CONCAT */
} gg_epilogue;

/* gg_forward with a fused epilogue and flags (epi may be NULL: same as gg_forward). out is
   bf16 [rows_alloc, N] (GG_ACT_NONE) or [rows_alloc, N/2] (GG_ACT_SILU_MUL). With
   GG_FLAG_W_NK, W is [E, N, K]. */
GG_API gg_status gg_forward_ex(const void* A, const void* W, const int32_t* offs, void* out,
                               int64_t rows_alloc, int64_t K, int64_t N, int32_t E,
                               const gg_epilogue* epi, int32_t* dev_status, cudaStream_t stream);

/* gg_masked_forward with a fused epilogue; out is [E, mmax, N] or [E, mmax, N/2]. */
GG_API gg_status gg_masked_forward_ex(const void* A, const void* W, const int32_t* masked_m,
                                      void* out, int64_t mmax, int64_t K, int64_t N, int32_t E,
                                      const gg_epilogue* epi, int32_t* dev_status,
                                      cudaStream_t stream);

/*
 * Token routing into the packed layout of the grouped GEMM (the step before the path: it
 * plays the part of torchtitan's generate_permute_indices in PyTorch issue 152668, without
 * the alignment padding that issue relies on, and without a host round trip).
 *   topk_ids int32 [T_tok, k], device: expert of assignment i = t*k + s; ids < 0 mean
 *            "dropped", ids >= E are dropped and flag GG_DEV_BAD_ROUTE
 *   X        bf16 [T_tok, K]; A_packed bf16 [T_tok*k, K] (only its first offs[E-1] rows are
 *            written: row_of[i] of assignment i gets a copy of X[t])
 *   row_of   int32 [T_tok*k]: packed row of each assignment, -1 when dropped
 *   offs     int32 [E]: cumulative end offsets, ready for gg_forward & co.
 * Rows are ordered by expert and, inside an expert, by assignment index (a stable sort), so
 * the result is deterministic. `workspace` is caller-owned device memory of at least
 * gg_route_workspace_bytes(T_tok*k, E) bytes (4-byte aligned); it need not be cleared.
 */
GG_API size_t gg_route_workspace_bytes(int64_t n_assign, int32_t E);
GG_API gg_status gg_route(const int32_t* topk_ids, int64_t T_tok, int32_t k, int32_t E,
                          const void* X, int64_t K, void* A_packed, int32_t* row_of,
                          int32_t* offs, void* workspace, size_t workspace_bytes,
                          int32_t* dev_status, cudaStream_t stream);

/*
 * gg_route without a workspace argument, for callers that cannot allocate device memory
 * where they route tokens (for example a runtime whose device memory is reserved up front
 * by its own allocator, or code that must not enter the CUDA allocator at that point). The
 * pages have no counterpart of this entry point.
 * Same arguments, results and status bits as gg_route, minus the workspace. Instead of a
 * workspace the per-block histograms use one fixed device array inside the library:
 * GG_ROUTE_NOALLOC_MAX_COUNTS int32 entries (1 MiB), held by every GPU that loads the library
 * until the process exits. A call needs ceil(T_tok*k / 256) * E entries; larger problems
 * return GG_ERR_TOO_LARGE (e.g. at most 65536 assignments with 1024 experts, 1048576 with
 * 64). Nothing is allocated, freed or cleared: every entry a call reads it wrote itself.
 * All calls share the array, so calls that overlap on the GPU (other streams, other threads)
 * race; order them on one stream. Calls captured in a CUDA graph count the same way: two
 * replays of such a graph that may run at the same time, or two captured calls on parallel
 * branches of one graph, overlap and race, so serialise them like calls on two streams.
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress) with
 * that device current, and so does the first call after its context was destroyed and
 * created again (cudaDeviceReset); make such a call before any stream capture.
 */
#define GG_ROUTE_NOALLOC_MAX_COUNTS (1 << 18)
GG_API gg_status gg_route_noalloc(const int32_t* topk_ids, int64_t T_tok, int32_t k, int32_t E,
                                  const void* X, int64_t K, void* A_packed, int32_t* row_of,
                                  int32_t* offs, int32_t* dev_status, cudaStream_t stream);

/* A static, human-readable name for a status. */
/*
 * One forward + backward pass of the grouped GEMM layer on operands in HOST memory:
 *   out = forward(A, W, offs), dX = dgrad(dY, W, offs), dW = wgrad(A, dY, offs),
 * the same three definitions as gg_forward / gg_dgrad / gg_wgrad, streamed through the GPU in
 * chunks of consecutive experts: while one chunk computes on `stream`, the next chunk's
 * operands are copied host -> device and the previous chunk's results device -> host, on two
 * copy streams that the library creates once per device and keeps.
 *   host (pinned, or the copies do not overlap): A_h bf16 [rows, K], W_h bf16 [E, K, N],
 *     dY_h bf16 [rows, N], offs_h int32 [E] cumulative end offsets; results out_h
 *     [rows, N], dX_h [rows, K], dW_h [E, K, N]; rows >= offs_h[E-1] of out_h / dX_h are
 *     not written.
 *   device staging, caller-owned, the same shapes: A_d, W_d, dY_d, out_d, dX_d, dW_d, and
 *     offs_d int32 [E], which ends up holding chunk-relative offsets.
 *   chunks: number of expert chunks (0: 16; at most E and 32).
 * The offsets are host data here and are checked on the host: non-decreasing within
 * [0, rows], else GG_ERR_INVALID_ARG and nothing is enqueued. The call returns once all work
 * is enqueued; `stream` is ordered after the last copy back, so the host results are valid
 * once `stream` is synchronised, and the work starts after what `stream` held before the
 * call. Calls from several threads are serialised while they enqueue. Not for stream capture.
 * The pages have no counterpart: this is the host-buffer form of the three passes, with the
 * host link overlapped with the GEMMs.
 */
GG_API gg_status gg_layer_step_host(const void* A_h, const void* W_h, const void* dY_h,
                                    const int32_t* offs_h, void* out_h, void* dX_h,
                                    void* dW_h, void* A_d, void* W_d, void* dY_d,
                                    int32_t* offs_d, void* out_d, void* dX_d, void* dW_d,
                                    int64_t rows, int64_t K, int64_t N, int32_t E,
                                    int32_t chunks, int32_t* dev_status, cudaStream_t stream);

GG_API const char* gg_status_string(gg_status s);

/* Watchdog bound of every in-kernel wait, in nanoseconds, for later calls from any
   thread (default 4e9). Returns the previous value. 0 restores the default. The longest
   wait on a healthy call is the epilogue's wait for one tile's whole reduction (K for
   forward, N for dgrad, a group's rows for wgrad), about 0.5-1 us per 64 reduction
   elements on a B200: raise the bound for reductions beyond a few million elements. */
GG_API uint64_t gg_set_watchdog_ns(uint64_t ns);

/* Test hook: when enable != 0, later calls make CTA 0's load warp skip its first stage,
   so that the pipeline's first wait runs into the watchdog and the call reports
   GG_DEV_TIMEOUT. No GPU fault is involved. Returns the previous setting. */
GG_API int gg_testing_skip_first_load(int enable);

/* Test hook: choose the launch shape of gg_forward, gg_dgrad and gg_wgrad for later calls:
   0 = automatic (forward/dgrad: CTA pairs with 256 x 512 tiles when rows_alloc >= 512*E,
   with the SiLU-and-mul epilogue only when K >= 4096 (else 256 x 256), else single CTAs;
   wgrad: by the average group length), 1 = single CTAs (128 x 256 tiles),
   2 = CTA pairs (256 x 256 tiles on two SMs), 3 = CTA pairs with 256 x 512 tiles.
   Results are the same up to rounding order.
   Returns the previous setting. */
GG_API int gg_testing_force_variant(int variant);

/* Text of the CUDA failure behind the last GG_ERR_CUDA returned in this thread ("" if none).
   The pointer stays valid until the thread's next call into the library. */
GG_API const char* gg_last_error(void);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
GG_API int gg_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GG_H_ */
