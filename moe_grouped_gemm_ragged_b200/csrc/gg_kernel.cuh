// Persistent, warp-specialised ragged grouped GEMM for sm_100a.
//
// One kernel template serves the four operations of the library:
//   Forward  out[r,:]   = A[r,:] . W[e]                 (tile rows = token rows)
//   Dgrad    dX[r,:]    = dY[r,:] . W[e]^T              (tile rows = token rows)
//   Masked   out[e,r,:] = A[e,r,:] . W[e], r < masked_m[e]
//   Wgrad    dW[e]      = A[rows of e]^T . dY[rows of e] (tile rows = K index; the reduction
//                                                        runs over the ragged token rows)
//
// Launch shapes sharing this code:
//   single CTA (PAIR = false): a tile is 128 rows x BN columns, one CTA per SM;
//   CTA pair   (PAIR = true):  a cluster of 2 CTAs on neighbouring SMs computes one
//               256 x BN tile with tcgen05.mma.cta_group::2: each CTA loads its own 128 rows
//               of A and its own BN/2 columns of B into its own shared memory, the pair
//               leader issues the MMAs, and each CTA's tensor memory holds its 128 rows of
//               the accumulator;
//               with BN = 512 (wide pair) each reduction step issues two N = 256 MMAs into
//               one accumulator of all 512 TMEM columns.
//
// Roles of the 11 warps of a CTA (one CTA per SM, persistent over a strided tile list):
//   warp 0      TMA producer: one lane arms a stage barrier and issues the tensor loads
//   warp 1      tensor-memory owner and MMA issuer: one lane issues tcgen05.mma into a
//               double-buffered fp32 accumulator in TMEM (2 x BN columns), or into the single
//               accumulator of a wide pair, which the epilogue hands back half by half
//   warps 2..9  epilogue: two warps per 32-lane TMEM quadrant, each owning half of the
//               columns; tcgen05.ld (double-buffered registers), fp32 -> bf16 (nearest
//               even), predicated 32- or 16-byte stores of rows inside the group, columns < N
//   warp 10     wgrad only: zeroes the rows of a group's last stage that lie past the group
//
// Shared-memory stages use the 128-byte swizzle that both TMA and tcgen05 understand:
//   K-major operand  (reduction contiguous):  [rows][64 elements = 128 B]
//   MN-major operand (M/N contiguous):        [chunks of 64 M/N][64 reduction rows][128 B]
//
// The tile list comes from the offsets on the device: every CTA rebuilds the same table
// (group bounds under the clamp rule, tile prefix sums) in shared memory, so no host
// synchronisation and no global scratch is needed. Every wait is bounded by a watchdog.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace gg {

enum class Mode : int { Forward = 0, Dgrad = 1, Wgrad = 2, Masked = 3 };

constexpr int BM = 128;         // tile rows (TMEM lanes)
constexpr int BK = 64;          // reduction elements per stage (128 bytes of bf16)
constexpr int UMMA_K = 16;      // reduction per tcgen05.mma for 16-bit inputs
// Reduction elements per stage of each pass. All passes use BK: 32-row wgrad stages (twice
// as many in the same shared memory) measured half the throughput on the large shape, each
// stage taking about as long as a 64-row one.
template <Mode MODE>
__host__ __device__ constexpr int bk_of() { return BK; }
constexpr int EPI_WARPS = 8;      // two per TMEM lane quadrant, each owning half the columns
constexpr int FIX_WARP = 2 + EPI_WARPS;  // wgrad: zeroes the rows of a group's last stage
constexpr int NUM_THREADS = 32 * (FIX_WARP + 1);

// L2 eviction priority of the TMA loads: 0 normal, 1 evict-first, 2 evict-last.
//   GG_L2_TOKENS   token-major operand of forward/dgrad/masked (A or dY), reused by the
//                  N-tiles of one row band that run at the same time (evict-first here
//                  doubled the DRAM traffic of the large shape: 36 GB vs 18 GB per pass)
//   GG_L2_WEIGHTS  W[e], reused by every row band of group e
//   GG_L2_WGRAD    both operands of wgrad
#ifndef GG_L2_TOKENS
#define GG_L2_TOKENS 0
#endif
#ifndef GG_L2_WEIGHTS
#define GG_L2_WEIGHTS 2
#endif
#ifndef GG_L2_WGRAD
#define GG_L2_WGRAD 2
#endif
// tcgen05 fence after every stage's full-barrier wait (the operands were written by TMA and
// are ordered by the barrier itself; 0 leaves the fence out).
#ifndef GG_FENCE_PER_STAGE
#define GG_FENCE_PER_STAGE 1
#endif
// Longest suspension of one mbarrier probe (ns); the thread wakes early when the phase
// completes. It also bounds how late an aborting role notices the abort flag.
#ifndef GG_WAIT_SLICE_NS
#define GG_WAIT_SLICE_NS 200000
#endif
// Every other tile a CTA processes walks its reduction backwards, so that the operand
// slabs a wave reads last are the first the next wave needs (they are still in L2).
#ifndef GG_SERPENTINE
#define GG_SERPENTINE 1
#endif
// Back-off (ns) of the epilogue warps while they wait for an accumulator (0 = spin).
#ifndef GG_EPI_BACKOFF_NS
#define GG_EPI_BACKOFF_NS 0
#endif
// Programmatic dependent launch: a kernel may be scheduled while the previous kernel of its
// stream is still finishing; it initialises its barriers and tensor memory, then waits for
// that kernel's completion before its first global read or write (0 launches plainly).
#ifndef GG_PDL
#define GG_PDL 1
#endif

// Device status bits (same values as the public header).
constexpr int DEV_BAD_OFFSETS = 0x1;
constexpr int DEV_BAD_MASKED_M = 0x2;
constexpr int DEV_TIMEOUT = 0x4;
constexpr int DEV_LAUNCHED = 0x100;

struct Params {
  const int32_t* groups;   // offsets (ragged modes) or masked_m (masked mode), device
  __nv_bfloat16* out;      // output base, row major with out_cols columns
  int32_t* status;         // may be null
  int64_t rows_alloc;      // rows of the token-major buffers (E*mmax in masked mode)
  int32_t E;
  int32_t mmax;            // masked mode only
  int32_t red_len;         // reduction length (Forward/Masked: K, Dgrad: N; Wgrad: unused)
  int32_t out_cols;        // output columns (Forward/Masked/Wgrad: N, Dgrad: K; N/2 with
                           // the SiLU-and-mul epilogue)
  int32_t prod_cols;       // columns of the product the tiles cover (out_cols, or N)
  int32_t wg_K;            // Wgrad: K (rows of each dW[e])
  uint64_t watchdog_ns;
  int32_t debug_flags;     // bit 0: CTA 0 skips its first load (watchdog test)
  // 1 when the map of that operand covers all 64-wide chunks of a stage in one box (a
  // dimension split as [.., dim/64, 64]); 0 when each chunk is its own box.
  int32_t a_chunked;
  int32_t b_chunked;
  int32_t out_v8;          // 1 when every output row starts 32-byte aligned (256-bit stores)
  // fp32 output with scaling and accumulation (out_f32 = alpha * product + beta * out_f32)
  float* out_f32;
  float alpha;
  float beta;
  // forward epilogue: h = product + s[row] * bias[e, col] (bf16 [E, N], may be null; s from
  // bias_scale, fp32 indexed by output row, 1 when null); with SiLU-and-mul the output has
  // N/2 columns (out_cols) and the product N (bias_ld)
  const __nv_bfloat16* bias;
  const float* bias_scale;
  int32_t bias_ld;
  // forward/dgrad: rows at and past the last effective offset are written with zeros (a
  // pseudo-group after the last expert whose tiles have no reduction stages)
  int32_t zero_tail;
  // SiLU-and-mul with W's columns as [gate | up] halves (0: gate and up interleaved in
  // blocks of 128); the loads put the tile's gate block and up block side by side, so the
  // accumulator holds the same columns in both layouts
  int32_t gate_up_concat;
};

// Wgrad of CTA pairs with 256-column tiles and bf16 output stores dW through shared memory
// and TMA: each epilogue warp stages 32 rows x 64 columns (4 KB, 128-byte swizzle) at a time
// and issues one tensor store per block (0: predicated stores from registers).
#ifndef GG_WG_TMA_STORE
#define GG_WG_TMA_STORE 1
#endif
template <Mode MODE, int BN, bool PAIR, bool F32, int ACT>
__host__ __device__ constexpr bool tma_store_epilogue() {
  return GG_WG_TMA_STORE && MODE == Mode::Wgrad && PAIR && BN == 256 && !F32 && ACT == 0;
}
template <Mode MODE, int BN, bool PAIR, bool F32, int ACT>
__host__ __device__ constexpr uint32_t staging_bytes() {
  return tma_store_epilogue<MODE, BN, PAIR, F32, ACT>() ? EPI_WARPS * 4096u : 0u;
}

template <int BN, int STAGES, bool PAIR, int BKL = BK, uint32_t STG = 0>
struct Layout {
  static constexpr int B_COLS = PAIR ? BN / 2 : BN;  // columns of B this CTA loads
  static constexpr uint32_t A_BYTES = BM * BKL * 2;
  static constexpr uint32_t B_BYTES = B_COLS * BKL * 2;
  // an MN-major operand holds one BKL-row x 128-byte block per 64-wide chunk
  static constexpr uint32_t CHUNK_BYTES = BKL * 128;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr uint32_t OFF_A = 0;
  static constexpr uint32_t OFF_B = STAGES * A_BYTES;
  static constexpr uint32_t OFF_STG = STAGES * STAGE_BYTES;  // epilogue staging (STG bytes)
  static constexpr uint32_t OFF_BAR = OFF_STG + STG;
  // full, empty, landed, fixed (wgrad tail blocks) per stage; tfull x2, tempty x2, fin
  static constexpr uint32_t NUM_BARS = 4 * STAGES + 5;
  static constexpr uint32_t OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr uint32_t OFF_TAB = OFF_MISC + 16;
  // fp32 accumulators in tensor memory: two of BN columns (the epilogue drains one while the
  // next tile fills the other), or one when a tile is wider than 256 columns (512 columns,
  // all of an SM's tensor memory)
  static constexpr uint32_t ACC_BUFS = BN > 256 ? 1 : 2;
  static constexpr uint32_t TMEM_COLS = ACC_BUFS * BN;
  // gstart[E+1], gend[E+1], prefix[E+2], order[E] (int32); group E is the zero tail
  static __host__ __device__ constexpr uint32_t bytes(int E) {
    return OFF_TAB + 4u * (4u * ((uint32_t)E + 1u) + 1u) + 1024u /* alignment slack */;
  }
};

struct Tile {
  int32_t e;        // group / expert
  int64_t row0;     // first output row of the tile (flat row of out)
  int64_t row_end;  // rows >= row_end are not stored
  int32_t n0;       // first output column
  int32_t a_row0;   // token row of the first tile row (Forward/Dgrad/Masked)
  int32_t k0;       // Wgrad: first K index of the tile
  int32_t tok0;     // Wgrad: first token row of the group
  int32_t tok_len;  // Wgrad: rows in the group
  int32_t kblocks;  // reduction stages
};

struct Shared {
  uint64_t* full;
  uint64_t* empty;
  uint64_t* landed;
  uint64_t* fixed;
  uint64_t* tfull;
  uint64_t* tempty;
  uint64_t* fin;
  uint32_t* tmem_base;
  volatile int32_t* abort_flag;
  int32_t* total;
  int32_t* gstart;
  int32_t* gend;
  int32_t* prefix;
  int32_t* order;
};

__device__ __forceinline__ void set_status(const Params& p, int bits) {
  if (p.status != nullptr) atomicOr(p.status, bits);
}

// Bounded wait on one phase of an mbarrier, slow path: probes until the phase completes,
// the CTA aborts, or the watchdog expires (then the abort flag and GG_DEV_TIMEOUT are set).
// Each probe suspends the thread until the phase completes or about GG_WAIT_SLICE_NS pass.
// `cluster` selects acquire at cluster scope, for barriers that receive arrivals from the
// peer CTA.
__device__ __noinline__ bool wait_slow(uint64_t* bar, uint32_t parity, const Shared& sh,
                                       const Params& p, bool honour_abort, bool cluster,
                                       uint32_t backoff_ns) {
  const uint64_t t0 = ptx::globaltimer();
  for (;;) {
    if (backoff_ns) __nanosleep(backoff_ns);
    const bool done = cluster ? ptx::mbar_try_wait_cluster(bar, parity, GG_WAIT_SLICE_NS)
                              : ptx::mbar_try_wait(bar, parity, GG_WAIT_SLICE_NS);
    if (done) return true;
    if (honour_abort && *sh.abort_flag) return false;
    if (ptx::globaltimer() - t0 > p.watchdog_ns) {
      *sh.abort_flag = 1;
      set_status(p, DEV_TIMEOUT);
      return false;
    }
  }
}

// Bounded wait: one inline probe (the common case on a busy pipeline), then the slow path.
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, const Shared& sh,
                                             const Params& p, bool honour_abort,
                                             bool cluster = false, uint32_t backoff_ns = 0) {
  const bool done = cluster ? ptx::mbar_try_wait_cluster(bar, parity, GG_WAIT_SLICE_NS)
                            : ptx::mbar_try_wait(bar, parity, GG_WAIT_SLICE_NS);
  if (done) return true;
  return wait_slow(bar, parity, sh, p, honour_abort, cluster, backoff_ns);
}

// Single-lane wait whose outcome every lane of the warp shares.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const Shared& sh,
                                          const Params& p, bool cluster,
                                          uint32_t backoff_ns = 0) {
  bool ok = true;
  if (ptx::lane_id() == 0) ok = wait_bounded(bar, parity, sh, p, true, cluster, backoff_ns);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// ---------------------------------------------------------------- schedule
// Warp 0 builds the group table. Ragged modes: effective ends t'_e = clamp(offs[e],
// t'_{e-1}, rows_alloc) with t'_{-1} = 0, i.e. min(running max of offs (from 0), rows).
// Masked: group e starts at e*mmax and has clamp(masked_m[e], 0, mmax) rows.
template <Mode MODE, int BN, int TM>
__device__ void build_table(const Params& p, const Shared& sh) {
  const uint32_t lane = ptx::lane_id();
  const int32_t E = p.E;
  const int32_t NT = (p.prod_cols + BN - 1) / BN;
  int64_t run_max = 0;   // running max of offsets seen so far (starts at t'_{-1} = 0)
  int32_t prev_end = 0;  // t'_{base-1}
  int32_t tiles_carry = 0;
  bool bad = false;
  if (lane == 0) sh.prefix[0] = 0;
  for (int32_t base = 0; base < E; base += 32) {
    const int32_t e = base + (int32_t)lane;
    const bool valid = e < E;
    const int32_t g = valid ? p.groups[e] : 0;
    int32_t start, end;
    if constexpr (MODE == Mode::Masked) {
      int32_t m = g < 0 ? 0 : (g > p.mmax ? p.mmax : g);
      bad |= valid && (m != g);
      start = e * p.mmax;
      end = start + (valid ? m : 0);
    } else {
      int64_t v = valid ? (int64_t)g : INT64_MIN;
      // inclusive max-scan across the warp
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int64_t o = __shfl_up_sync(0xffffffffu, v, d);
        if ((int)lane >= d) v = v > o ? v : o;
      }
      v = v > run_max ? v : run_max;
      const int64_t t = v < p.rows_alloc ? v : p.rows_alloc;
      end = (int32_t)t;
      const int32_t up = __shfl_up_sync(0xffffffffu, end, 1);
      start = lane == 0 ? prev_end : up;
      bad |= valid && ((int64_t)end != (int64_t)g);
      run_max = __shfl_sync(0xffffffffu, v, 31);
      prev_end = __shfl_sync(0xffffffffu, end, 31);
    }
    int32_t tiles = 0;
    if (valid) {
      if constexpr (MODE == Mode::Wgrad) {
        tiles = 0;  // fixed grid, counted below
      } else {
        tiles = ((end - start + TM - 1) / TM) * NT;
      }
    }
    int32_t s = tiles;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int32_t o = __shfl_up_sync(0xffffffffu, s, d);
      if ((int)lane >= d) s += o;
    }
    if (valid) {
      sh.gstart[e] = start;
      sh.gend[e] = end;
      sh.prefix[e + 1] = tiles_carry + s;
    }
    tiles_carry += __shfl_sync(0xffffffffu, s, 31);
  }
  bad = __any_sync(0xffffffffu, bad);
  if (lane == 0) {
    if (bad) set_status(p, MODE == Mode::Masked ? DEV_BAD_MASKED_M : DEV_BAD_OFFSETS);
    if constexpr (MODE == Mode::Wgrad) {
      const int32_t KT = (p.wg_K + TM - 1) / TM;
      *sh.total = E * KT * NT;
    } else if (MODE != Mode::Masked && p.zero_tail) {
      // rows [t'_{E-1}, rows_alloc): one more group, of zero tiles
      const int32_t tail = (int32_t)(p.rows_alloc - prev_end);
      sh.gstart[E] = prev_end;
      sh.gend[E] = (int32_t)p.rows_alloc;
      sh.prefix[E + 1] = tiles_carry + ((tail + TM - 1) / TM) * NT;
      *sh.total = sh.prefix[E + 1];
    } else {
      *sh.total = tiles_carry;
    }
  }
}

// Wgrad visits experts in order of decreasing row count (ties by index) so that the
// longest reductions start first; order[rank] = expert. All threads take part.
__device__ void build_wgrad_order(const Params& p, const Shared& sh) {
  const int32_t E = p.E;
  for (int32_t e = threadIdx.x; e < E; e += blockDim.x) {
    const int32_t me = sh.gend[e] - sh.gstart[e];
    int32_t rank = 0;
    for (int32_t j = 0; j < E; ++j) {
      const int32_t mj = sh.gend[j] - sh.gstart[j];
      rank += (mj > me) || (mj == me && j < e);
    }
    sh.order[rank] = e;
  }
}

// Tile of unit `unit` (a CTA, or a CTA pair) in its it-th round. Wgrad tiles come sorted by
// decreasing length (experts by size); odd rounds hand them out in reverse unit order (snake
// order), so that the units that got the longest tiles of one round get the shortest of the
// next (on the Zipf-skewed gate-up shape the longest unit's work drops from 1.17x to 1.08x
// the mean). In every order a unit's tiles increase, so its walk stops at the first tile
// past the end.
template <Mode MODE>
__device__ __forceinline__ int32_t tile_at(int32_t unit, int32_t it, int32_t units) {
  if constexpr (MODE == Mode::Wgrad) return it * units + ((it & 1) ? units - 1 - unit : unit);
  else return it * units + unit;
}

template <Mode MODE, int BN, int TM>
__device__ __forceinline__ Tile decode_tile(int32_t t, const Params& p, const Shared& sh) {
  Tile tl;
  const int32_t NT = (p.prod_cols + BN - 1) / BN;
  if constexpr (MODE == Mode::Wgrad) {
    const int32_t KT = (p.wg_K + TM - 1) / TM;
    const int32_t per = KT * NT;
    const int32_t slot = t / per;
    const int32_t local = t - slot * per;
    const int32_t kt = local / NT;
    const int32_t nt = local - kt * NT;
    const int32_t e = sh.order[slot];
    tl.e = e;
    tl.k0 = kt * TM;
    tl.n0 = nt * BN;
    tl.tok0 = sh.gstart[e];
    tl.tok_len = sh.gend[e] - sh.gstart[e];
    tl.kblocks = (tl.tok_len + bk_of<MODE>() - 1) / bk_of<MODE>();
    tl.row0 = (int64_t)e * p.wg_K + tl.k0;
    tl.row_end = (int64_t)e * p.wg_K + p.wg_K;
    tl.a_row0 = 0;
  } else {
    // largest e with prefix[e] <= t (group E is the zero tail, when present)
    int32_t lo = 0, hi = (MODE != Mode::Masked && p.zero_tail) ? p.E : p.E - 1;
    while (lo < hi) {
      const int32_t mid = (lo + hi + 1) >> 1;
      if (sh.prefix[mid] <= t) lo = mid; else hi = mid - 1;
    }
    const int32_t e = lo;
    const int32_t local = t - sh.prefix[e];
    const int32_t mt = local / NT;
    const int32_t nt = local - mt * NT;
    tl.e = e;
    tl.a_row0 = sh.gstart[e] + mt * TM;
    tl.row0 = tl.a_row0;
    tl.row_end = sh.gend[e];
    tl.n0 = nt * BN;
    tl.kblocks = e < p.E ? (p.red_len + bk_of<MODE>() - 1) / bk_of<MODE>() : 0;
    tl.k0 = 0;
    tl.tok0 = 0;
    tl.tok_len = 0;
  }
  return tl;
}

// ---------------------------------------------------------------- kernel
// ACT 1: SiLU-and-mul epilogue (gate and up columns interleaved in blocks of BN/2).
template <Mode MODE, int BN, int STAGES, bool PAIR, bool F32 = false, int ACT = 0>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap mapA,
                        const __grid_constant__ CUtensorMap mapB,
                        const __grid_constant__ CUtensorMap mapC, const Params p) {
  constexpr int BKM = bk_of<MODE>();  // reduction elements per stage
  constexpr bool TMA_EPI = tma_store_epilogue<MODE, BN, PAIR, F32, ACT>();
  using L = Layout<BN, STAGES, PAIR, BKM, staging_bytes<MODE, BN, PAIR, F32, ACT>()>;
  static_assert(BN % 64 == 0 && BN >= 64 && (BN <= 256 || (BN == 512 && PAIR)),
                "BN must be 64, 128, 192 or 256, or 512 for a CTA pair");
  static_assert(!PAIR || BN % 128 == 0, "a CTA pair splits BN into two multiples of 64");
  static_assert(L::TMEM_COLS == 128 || L::TMEM_COLS == 256 || L::TMEM_COLS == 512,
                "TMEM allocation must be a power of two");
  constexpr int TM = PAIR ? 2 * BM : BM;  // rows of a tile
  // A operand MN-major only in Wgrad; B operand K-major only in Dgrad.
  constexpr uint32_t A_MN = (MODE == Mode::Wgrad) ? 1u : 0u;
  constexpr uint32_t B_MN = (MODE == Mode::Dgrad) ? 0u : 1u;
  // One MMA covers at most 256 columns; a 512-column pair tile issues two per reduction step,
  // each taking 128 of the 256 B columns that each CTA holds (TMEM columns [256h, 256h+256)
  // of MMA h: the first 128 from the leader's B, the next 128 from the follower's).
  constexpr int MMA_N = BN > 256 ? 256 : BN;
  constexpr int NSPLIT = BN / MMA_N;
  constexpr uint32_t IDESC = ptx::idesc_bf16_f32(TM, MMA_N, A_MN, B_MN);
  constexpr uint32_t EPI_ARRIVALS = (PAIR ? 2u : 1u) * EPI_WARPS;  // one per epilogue warp
  // In a pair's wgrad, the follower signals its fixed-up half of a group's last stage on the
  // leader's fixed[] barrier (a stage with whole rows only completes by its byte count).
  constexpr bool PAIR_WGRAD = PAIR && MODE == Mode::Wgrad;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = ptx::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);

  Shared sh;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  sh.full = bars;
  sh.empty = bars + STAGES;
  sh.landed = bars + 2 * STAGES;
  sh.fixed = bars + 3 * STAGES;
  sh.tfull = bars + 4 * STAGES;
  sh.tempty = bars + 4 * STAGES + 2;
  sh.fin = bars + 4 * STAGES + 4;
  sh.tmem_base = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  sh.abort_flag = reinterpret_cast<volatile int32_t*>(smem + L::OFF_MISC + 4);
  sh.total = reinterpret_cast<int32_t*>(smem + L::OFF_MISC + 8);
  int32_t* tab = reinterpret_cast<int32_t*>(smem + L::OFF_TAB);
  sh.gstart = tab;
  sh.gend = tab + (p.E + 1);
  sh.prefix = tab + 2 * (p.E + 1);
  sh.order = tab + 3 * (p.E + 1) + 1;

  const uint32_t warp = threadIdx.x / 32;
  const uint32_t lane = ptx::lane_id();
  const uint32_t rank = PAIR ? ptx::cluster_ctarank() : 0u;  // 0 = pair leader
  const bool leader = rank == 0;
  const int32_t unit0 = PAIR ? (int32_t)ptx::cluster_id_x() : (int32_t)blockIdx.x;
  const int32_t units = PAIR ? (int32_t)ptx::ncluster_x() : (int32_t)gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(&sh.full[s], 1);
      ptx::mbar_init(&sh.empty[s], 1);
      ptx::mbar_init(&sh.landed[s], 1);
      ptx::mbar_init(&sh.fixed[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(&sh.tfull[a], 1);
      ptx::mbar_init(&sh.tempty[a], EPI_ARRIVALS);
    }
    ptx::mbar_init(sh.fin, 1);
    *sh.abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&mapA);
    ptx::prefetch_tmap(&mapB);
    if constexpr (TMA_EPI) ptx::prefetch_tmap(&mapC);
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      ptx::tmem_alloc_pair(sh.tmem_base, L::TMEM_COLS);
      ptx::tmem_relinquish_pair();
    } else {
      ptx::tmem_alloc(sh.tmem_base, L::TMEM_COLS);
      ptx::tmem_relinquish();
    }
  }
  // Up to here only this CTA's own shared and tensor memory was touched. The inputs may be
  // the outputs of the previous kernel in the stream, which may still be running.
  ptx::griddep_wait();
  if (warp == 0) build_table<MODE, BN, TM>(p, sh);
  ptx::tc_fence_before();
  if constexpr (PAIR) ptx::cluster_sync();  // peer barriers initialised before any remote use
  else __syncthreads();
  ptx::tc_fence_after();
  if constexpr (MODE == Mode::Wgrad) {
    build_wgrad_order(p, sh);
    __syncthreads();
  }
  const uint32_t tmem_base = *sh.tmem_base;
  const int32_t total = *sh.total;
  // the next kernel may be scheduled on SMs as they free up; it waits for this grid as above
  ptx::griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // The whole warp walks the tile list; lane 0 waits and issues the loads. A wgrad stage
    // that ends its group lands on landed[] for the fix-up warp instead of on full[].
    const uint64_t pol_tok = ptx::l2_policy<GG_L2_TOKENS>();
    const uint64_t pol_w = ptx::l2_policy<GG_L2_WEIGHTS>();
    const uint64_t pol_wg = ptx::l2_policy<GG_L2_WGRAD>();
    uint32_t stage = 0, phase = 0;
    uint32_t armed = 0, armed_par = 0;  // per stage: loads in flight on full[], their phase
    uint32_t armed_l = 0, armed_lpar = 0;  // the same for loads on landed[] (wgrad tails)
    uint32_t landed_par = 0;  // per stage: phase of the next load on landed[]
    auto lp_of = [&](uint32_t st) { return (landed_par >> st) & 1u; };
    bool skip_first = (p.debug_flags & 1) && blockIdx.x == 0;
    bool ok = true;
    const int32_t row_off = (int32_t)rank * BM;         // this CTA's rows of a pair tile
    const int32_t col_off = (int32_t)rank * L::B_COLS;  // this CTA's columns of B
    for (int32_t it = 0, t = tile_at<MODE>(unit0, 0, units); t < total && ok;
         t = tile_at<MODE>(unit0, ++it, units)) {
      const Tile tl = decode_tile<MODE, BN, TM>(t, p, sh);
      const bool rev = GG_SERPENTINE && (it & 1);
      for (int32_t kq = 0; kq < tl.kblocks; ++kq) {
        const int32_t kb = rev ? tl.kblocks - 1 - kq : kq;  // reduction block of this stage
        if (!warp_wait(&sh.empty[stage], phase ^ 1u, sh, p, false)) { ok = false; break; }
        uint8_t* sA = smem + L::OFF_A + stage * L::A_BYTES;
        uint8_t* sB = smem + L::OFF_B + stage * L::B_BYTES;
        uint64_t* fb = &sh.full[stage];
        int32_t rem = BKM;  // wgrad: rows of the group in this stage
        if constexpr (MODE == Mode::Wgrad) rem = tl.tok_len - kb * BKM;
        const bool tail = MODE == Mode::Wgrad && rem < BKM;
        if (lane == 0) {
          armed &= ~(1u << stage);
          armed_l &= ~(1u << stage);
          if (skip_first) {
            skip_first = false;  // watchdog test: this stage is never armed
          } else if constexpr (PAIR && MODE == Mode::Wgrad) {
            const int32_t r = tl.tok0 + kb * BKM;
            const int32_t ka = tl.k0 + row_off;  // this CTA's 128 columns of A (K)
            const int32_t nb = tl.n0 + col_off;  // this CTA's columns of dY (N)
            if (tail) {
              // lands locally; the warp fixes it up and then arrives on the leader's barrier
              uint64_t* lb = &sh.landed[stage];
              ptx::mbar_arrive_expect_tx(lb, L::STAGE_BYTES);
              armed_l |= 1u << stage;
              armed_lpar = (armed_lpar & ~(1u << stage)) | (lp_of(stage) << stage);
              if (p.a_chunked) {
                ptx::tma_load_3d(sA, &mapA, lb, 0, r, ka / 64, pol_wg);
              } else {
                for (int j = 0; j < 2; ++j)
                  ptx::tma_load_2d(sA + j * L::CHUNK_BYTES, &mapA, lb, ka + j * 64, r, pol_wg);
              }
              if (p.b_chunked) {
                ptx::tma_load_3d(sB, &mapB, lb, 0, r, nb / 64, pol_wg);
              } else {
                for (int j = 0; j < L::B_COLS / 64; ++j)
                  ptx::tma_load_2d(sB + j * L::CHUNK_BYTES, &mapB, lb, nb + j * 64, r, pol_wg);
              }
            } else {
              const uint32_t fb_leader = ptx::mapa(ptx::smem_u32(fb), 0);
              if (leader) ptx::mbar_arrive_expect_tx(fb, 2 * L::STAGE_BYTES);
              if (p.a_chunked) {
                ptx::tma_load_3d_pair(sA, &mapA, fb_leader, 0, r, ka / 64, pol_wg);
              } else {
                for (int j = 0; j < 2; ++j)
                  ptx::tma_load_2d_pair(sA + j * L::CHUNK_BYTES, &mapA, fb_leader, ka + j * 64, r, pol_wg);
              }
              if (p.b_chunked) {
                ptx::tma_load_3d_pair(sB, &mapB, fb_leader, 0, r, nb / 64, pol_wg);
              } else {
                for (int j = 0; j < L::B_COLS / 64; ++j)
                  ptx::tma_load_2d_pair(sB + j * L::CHUNK_BYTES, &mapB, fb_leader, nb + j * 64, r, pol_wg);
              }
              if (leader) {
                armed |= 1u << stage;
                armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
              }
            }
          } else if constexpr (PAIR) {
            // the leader's full barrier counts the bytes of both CTAs
            const uint32_t fb_leader = ptx::mapa(ptx::smem_u32(fb), 0);
            if (leader) ptx::mbar_arrive_expect_tx(fb, 2 * L::STAGE_BYTES);
            ptx::tma_load_2d_pair(sA, &mapA, fb_leader, kb * BKM, tl.a_row0 + row_off, pol_tok);
            if (ACT == 1 && p.gate_up_concat) {
              // [gate | up] weights: this CTA's B columns are 128-wide gate and up blocks
              // (a 256-wide pair tile: the leader's gate block, the follower's up block)
              constexpr int PIECES = L::B_COLS / 128;
              for (int i = 0; i < PIECES; ++i) {
                const int32_t gu = PIECES == 1 ? (int32_t)rank : i;
                const int32_t blk = PIECES == 1 ? 0 : (int32_t)rank;
                const int32_t col = gu * (p.prod_cols / 2) + tl.n0 / 2 + 128 * blk;
                uint8_t* dst = sB + i * (128 * BKM * 2);
                if constexpr (MODE == Mode::Dgrad)
                  ptx::tma_load_3d_pair(dst, &mapB, fb_leader, kb * BKM, col, tl.e, pol_w);
                else
                  ptx::tma_load_4d_pair(dst, &mapB, fb_leader, 0, kb * BKM, col / 64, tl.e, pol_w);
              }
            } else if constexpr (MODE == Mode::Dgrad) {
              ptx::tma_load_3d_pair(sB, &mapB, fb_leader, kb * BKM, tl.n0 + col_off, tl.e, pol_w);
            } else if (p.b_chunked) {
              ptx::tma_load_4d_pair(sB, &mapB, fb_leader, 0, kb * BKM, (tl.n0 + col_off) / 64,
                                    tl.e, pol_w);
            } else {
#pragma unroll
              for (int j = 0; j < L::B_COLS / 64; ++j)
                ptx::tma_load_3d_pair(sB + j * L::CHUNK_BYTES, &mapB, fb_leader, tl.n0 + col_off + j * 64,
                                      kb * BKM, tl.e, pol_w);
            }
            if (leader) {
              armed |= 1u << stage;
              armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
            }
          } else {
            // a wgrad tail stage lands on landed[] first; full[] completes after the fix-up
            uint64_t* lb = tail ? &sh.landed[stage] : fb;
            if constexpr (MODE == Mode::Masked) {
              // only the group's rows of A, in 32-row boxes; the MMA also reads the stale
              // rows after them, which only reach accumulator rows that are never stored
              int64_t valid = tl.row_end - (int64_t)tl.a_row0;
              if (valid > BM) valid = BM;
              const int32_t nbox = (int32_t)((valid + 31) / 32);
              ptx::mbar_arrive_expect_tx(lb, (uint32_t)nbox * 32u * 128u + L::B_BYTES);
              for (int32_t b = 0; b < nbox; ++b)
                ptx::tma_load_2d(sA + b * 4096, &mapA, lb, kb * BKM, tl.a_row0 + b * 32, pol_tok);
            } else {
              ptx::mbar_arrive_expect_tx(lb, L::STAGE_BYTES);
            }
            if constexpr (MODE == Mode::Forward || MODE == Mode::Masked) {
              if constexpr (MODE == Mode::Forward)
                ptx::tma_load_2d(sA, &mapA, lb, kb * BKM, tl.a_row0, pol_tok);
              if (ACT == 1 && p.gate_up_concat) {
                // [gate | up] weights: the tile's gate block, then its up block
                for (int i = 0; i < 2; ++i)
                  ptx::tma_load_4d(sB + i * (128 * BKM * 2), &mapB, lb, 0, kb * BKM,
                                   (i * (p.prod_cols / 2) + tl.n0 / 2) / 64, tl.e, pol_w);
              } else if (p.b_chunked) {
                ptx::tma_load_4d(sB, &mapB, lb, 0, kb * BKM, tl.n0 / 64, tl.e, pol_w);
              } else {
#pragma unroll
                for (int j = 0; j < BN / 64; ++j)
                  ptx::tma_load_3d(sB + j * L::CHUNK_BYTES, &mapB, lb, tl.n0 + j * 64, kb * BKM, tl.e, pol_w);
              }
            } else if constexpr (MODE == Mode::Dgrad) {
              ptx::tma_load_2d(sA, &mapA, lb, kb * BKM, tl.a_row0, pol_tok);
              if (ACT == 1 && p.gate_up_concat) {
                for (int i = 0; i < 2; ++i)
                  ptx::tma_load_3d(sB + i * (128 * BKM * 2), &mapB, lb, kb * BKM,
                                   i * (p.prod_cols / 2) + tl.n0 / 2, tl.e, pol_w);
              } else {
                ptx::tma_load_3d(sB, &mapB, lb, kb * BKM, tl.n0, tl.e, pol_w);
              }
            } else {  // Wgrad
              const int32_t r = tl.tok0 + kb * BKM;
              if (p.a_chunked) {
                ptx::tma_load_3d(sA, &mapA, lb, 0, r, tl.k0 / 64, pol_wg);
              } else {
#pragma unroll
                for (int j = 0; j < 2; ++j)
                  ptx::tma_load_2d(sA + j * L::CHUNK_BYTES, &mapA, lb, tl.k0 + j * 64, r, pol_wg);
              }
              if (p.b_chunked) {
                ptx::tma_load_3d(sB, &mapB, lb, 0, r, tl.n0 / 64, pol_wg);
              } else {
#pragma unroll
                for (int j = 0; j < BN / 64; ++j)
                  ptx::tma_load_2d(sB + j * L::CHUNK_BYTES, &mapB, lb, tl.n0 + j * 64, r, pol_wg);
              }
            }
            if (!tail) {
              armed |= 1u << stage;
              armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
            } else {
              armed_l |= 1u << stage;
              armed_lpar = (armed_lpar & ~(1u << stage)) | (lp_of(stage) << stage);
            }
          }
        }
        if (tail) landed_par ^= 1u << stage;
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
    // Let every load this warp armed land before the CTA can exit (on the normal path these
    // phases have completed already; after an abort some may still be in flight). A pair
    // follower's loads complete on the leader's barriers; they were issued at least one
    // watchdog period before any abort could end this CTA.
    if (lane == 0)
      for (int s = 0; s < STAGES; ++s) {
        if (armed & (1u << s)) wait_bounded(&sh.full[s], (armed_par >> s) & 1u, sh, p, false);
        if (armed_l & (1u << s))
          wait_bounded(&sh.landed[s], (armed_lpar >> s) & 1u, sh, p, false);
      }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // One lane of the pair leader issues every MMA; the loop carries no warp-wide
    // synchronisation so that issue keeps ahead of the tensor pipe.
    if (leader && lane == 0) {
      // descriptor deltas per 16-element reduction step (address field is in 16-byte units)
      constexpr uint64_t A_STEP = A_MN ? (2048u >> 4) : (32u >> 4);
      constexpr uint64_t B_STEP = B_MN ? (2048u >> 4) : (32u >> 4);
      const uint32_t a_lbo = A_MN ? L::CHUNK_BYTES : 16u, b_lbo = B_MN ? L::CHUNK_BYTES : 16u;
      uint32_t stage = 0, phase = 0, acc_iter = 0;
      uint32_t fixed_par = 0;  // per stage: next phase of fixed[] (pair wgrad)
      bool ok = true;
      for (int32_t it = 0, t = tile_at<MODE>(unit0, 0, units); t < total && ok;
         t = tile_at<MODE>(unit0, ++it, units)) {
        const Tile tl = decode_tile<MODE, BN, TM>(t, p, sh);
        if (tl.kblocks == 0) continue;  // Wgrad of an empty expert: the epilogue writes zeros
        const bool rev = GG_SERPENTINE && (it & 1);
        const uint32_t a = acc_iter % L::ACC_BUFS;
        if (!wait_bounded(&sh.tempty[a], ((acc_iter / L::ACC_BUFS) & 1u) ^ 1u, sh, p, true,
                          PAIR)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem_base + a * BN;
        // rows of stage kq inside the group: BKM except in a wgrad group's last stage
        auto rows_of = [&](int32_t kq) {
          if constexpr (MODE == Mode::Wgrad) {
            const int32_t kb = rev ? tl.kblocks - 1 - kq : kq;
            const int32_t rem = tl.tok_len - kb * BKM;
            return rem < BKM ? rem : BKM;
          }
          return BKM;
        };
        // waits until stage `st` holds the operands of step kq (false: abort)
        auto stage_ready = [&](uint32_t st, uint32_t ph, int32_t kq) {
          if (!wait_bounded(&sh.full[st], ph, sh, p, true)) return false;
#if GG_FENCE_PER_STAGE
          ptx::tc_fence_after();
#endif
          if constexpr (PAIR_WGRAD) {
            if (rows_of(kq) < BKM) {
              // a group's last stage: the follower's half is fixed up on its own schedule
              const uint32_t fp = (fixed_par >> st) & 1u;
              fixed_par ^= 1u << st;
              if (!wait_bounded(&sh.fixed[st], fp, sh, p, true, true)) return false;
            }
          }
          return true;
        };
        // the MMAs of accumulator part h (of NSPLIT) for the operands in stage st
        auto issue = [&](uint32_t st, int32_t kq, int h) {
          const int nsub = (rows_of(kq) + UMMA_K - 1) / UMMA_K;
          const uint64_t adesc = ptx::smem_desc_sw128(
              ptx::smem_u32(smem + L::OFF_A + st * L::A_BYTES), a_lbo, 1024);
          // MMA h reads B columns [128h, 128h+128) of each CTA: 128 x BKM bf16 further on in
          // either operand layout (two 64-wide chunks, or 128 K-major rows)
          const uint64_t bdesc =
              ptx::smem_desc_sw128(ptx::smem_u32(smem + L::OFF_B + st * L::B_BYTES), b_lbo,
                                   1024) +
              (uint64_t)h * ((128u * BKM * 2u) >> 4);
#pragma unroll
          for (int k = 0; k < BKM / UMMA_K; ++k) {
            if (k < nsub) {
              const uint32_t acc = (kq > 0 || k > 0) ? 1u : 0u;  // the first stage overwrites
              if constexpr (PAIR)
                ptx::mma_bf16_pair(d_tmem + h * MMA_N, adesc + k * A_STEP, bdesc + k * B_STEP,
                                   IDESC, acc);
              else
                ptx::mma_bf16(d_tmem, adesc + k * A_STEP, bdesc + k * B_STEP, IDESC, acc);
            }
          }
        };
        // free stage st (in both CTAs of a pair) once the MMAs issued so far are done
        auto release = [&](uint32_t st) {
          if constexpr (PAIR) {
            const uint32_t eb = ptx::smem_u32(&sh.empty[st]);
            ptx::mma_commit_pair(ptx::mapa(eb, 0));
            ptx::mma_commit_pair(ptx::mapa(eb, 1));
          } else {
            ptx::mma_commit(&sh.empty[st]);
          }
        };
        int32_t kq = 0;
        if constexpr (NSPLIT == 2) {
          // One accumulator in two halves. The epilogue hands the first half back (tempty[0],
          // waited above) as soon as it holds it in registers, and the second half after
          // that: the first stages of the tile take their first-half MMAs while the previous
          // tile's outputs are still being stored, and their second-half MMAs once the second
          // half is free (tempty[1]); only then are those stages released.
          const int32_t D = tl.kblocks < STAGES ? tl.kblocks : STAGES;
          uint32_t st = stage, ph = phase;
          for (int32_t i = 0; i < D; ++i) {
            if (!stage_ready(st, ph, i)) { ok = false; break; }
            issue(st, i, 0);
            if (++st == STAGES) { st = 0; ph ^= 1u; }
          }
          if (!ok) break;
          if (!wait_bounded(&sh.tempty[1], ((acc_iter / L::ACC_BUFS) & 1u) ^ 1u, sh, p, true,
                            PAIR)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          for (; kq < D; ++kq) {
            issue(stage, kq, 1);
            release(stage);
            if (++stage == STAGES) { stage = 0; phase ^= 1u; }
          }
        }
        for (; kq < tl.kblocks; ++kq) {
          if (!stage_ready(stage, phase, kq)) { ok = false; break; }
#pragma unroll
          for (int h = 0; h < NSPLIT; ++h) issue(stage, kq, h);
          release(stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if constexpr (PAIR) {
          const uint32_t fb = ptx::smem_u32(&sh.tfull[a]);
          ptx::mma_commit_pair(ptx::mapa(fb, 0));
          ptx::mma_commit_pair(ptx::mapa(fb, 1));
        } else {
          ptx::mma_commit(&sh.tfull[a]);
        }
        ++acc_iter;
      }
      // every MMA issued by this CTA completes before tensor memory is released
      if constexpr (PAIR) ptx::mma_commit_pair(ptx::mapa(ptx::smem_u32(sh.fin), 0));
      else                ptx::mma_commit(sh.fin);
      wait_bounded(sh.fin, 0, sh, p, false);
    }
    __syncwarp();
  } else if (warp < FIX_WARP) {
    // ------------------------------------------------------------ epilogue
    const uint32_t q = warp & 3u;                 // TMEM lane quadrant this warp may access
    constexpr int CW = BN / 2;                    // columns per epilogue warp
    const int32_t c_off = ((int32_t)warp - 2) / 4 * CW;
    const int32_t row_in_tile = (int32_t)(rank * BM + q * 32 + lane);
    // tensor memory of this CTA's accumulator is released on the pair leader's barrier
    uint32_t tempty0 = ptx::smem_u32(&sh.tempty[0]), tempty1 = ptx::smem_u32(&sh.tempty[1]);
    if constexpr (PAIR) {
      tempty0 = ptx::mapa(tempty0, 0);
      tempty1 = ptx::mapa(tempty1, 0);
    }
    const bool v8 = p.out_v8 != 0;
    uint32_t acc_iter = 0;
    for (int32_t it = 0, t = tile_at<MODE>(unit0, 0, units); t < total;
         t = tile_at<MODE>(unit0, ++it, units)) {
      const Tile tl = decode_tile<MODE, BN, TM>(t, p, sh);
      const int64_t orow = tl.row0 + row_in_tile;
      const bool row_ok = orow < tl.row_end;
      __nv_bfloat16* orow_ptr = p.out + orow * (int64_t)p.out_cols;
      const int32_t col0 = tl.n0 + c_off;
      if (tl.kblocks == 0) {
        if (row_ok) {
          if constexpr (F32) {
            // the product is zero: out = beta * out (nothing is read when beta == 0)
            float* orow_f = p.out_f32 + orow * (int64_t)p.out_cols;
            for (int c = 0; c < CW; c += 4) {
              const int32_t col = col0 + c;
              if (col < p.out_cols) {
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (p.beta != 0.f) {
                  const float4 o = *reinterpret_cast<const float4*>(orow_f + col);
                  v = make_float4(p.beta * o.x, p.beta * o.y, p.beta * o.z, p.beta * o.w);
                }
                *reinterpret_cast<float4*>(orow_f + col) = v;
              }
            }
          } else {
            // SiLU-and-mul halves the columns: this warp's outputs start at half its offset
            const int32_t zc0 = ACT == 1 ? tl.n0 / 2 + c_off / 2 : col0;
            const int32_t zcw = ACT == 1 ? CW / 2 : CW;
            for (int c = 0; c < zcw; c += 8) {
              const int32_t col = zc0 + c;
              if (col < p.out_cols)
                *reinterpret_cast<uint4*>(orow_ptr + col) = make_uint4(0u, 0u, 0u, 0u);
            }
          }
        }
        continue;
      }
      const uint32_t a = acc_iter % L::ACC_BUFS;
      if (!warp_wait(&sh.tfull[a], (acc_iter / L::ACC_BUFS) & 1u, sh, p, false,
                     GG_EPI_BACKOFF_NS))
        break;
      ptx::tc_fence_after();
      float s_row = 1.f;  // per-row bias scale (read only for rows inside the group)
      if (p.bias != nullptr && p.bias_scale != nullptr && row_ok) s_row = p.bias_scale[orow];
      const __nv_bfloat16* bias_e =
          p.bias != nullptr ? p.bias + (int64_t)tl.e * p.bias_ld : nullptr;
      if constexpr (ACT == 1) {
        // SiLU-and-mul: this warp owns output columns [oc, oc + CW/2) of the tile; their gate
        // values are accumulator columns c_off/2 + j and their up values BN/2 further on. The
        // gate of accumulator column t < BN/2 is product column 256 (t / 128) + t % 128 and
        // its up value the column 128 after it (in a 512-wide pair tile the TMEM column
        // order of the two MMAs puts them there; in a 256-wide tile t < 128)
        const int32_t half = c_off / 2;
        const uint32_t tg = tmem_base + ((q * 32u) << 16) + a * BN + (uint32_t)half;
        const int32_t oc = tl.n0 / 2 + half;
#pragma unroll 1
        for (int c = 0; c < CW / 2; c += 32) {
          uint32_t rg[32], ru[32];
          ptx::tmem_ld_32x32b_x32(tg + c, rg);
          ptx::tmem_ld_32x32b_x32(tg + BN / 2 + c, ru);
          ptx::tmem_ld_wait();
          const int32_t col = oc + c;  // output column of rg[0]
          if (row_ok && col < p.out_cols) {
            if (bias_e != nullptr) {
              // gate and up biases of these 32 columns, 8 at a time (16-byte loads)
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const int32_t t = half + c + 8 * j;
                // gate and up columns of output column n0/2 + t
                const int32_t gcol = p.gate_up_concat ? tl.n0 / 2 + t
                                                      : tl.n0 + 256 * (t / 128) + t % 128;
                const int32_t ucol = p.gate_up_concat ? gcol + p.prod_cols / 2 : gcol + 128;
                const uint4 bg = __ldg(reinterpret_cast<const uint4*>(bias_e + gcol));
                const uint4 bu = __ldg(reinterpret_cast<const uint4*>(bias_e + ucol));
                const __nv_bfloat16* g8 = reinterpret_cast<const __nv_bfloat16*>(&bg);
                const __nv_bfloat16* u8 = reinterpret_cast<const __nv_bfloat16*>(&bu);
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                  rg[8 * j + u] = __float_as_uint(
                      fmaf(s_row, __bfloat162float(g8[u]), __uint_as_float(rg[8 * j + u])));
                  ru[8 * j + u] = __float_as_uint(
                      fmaf(s_row, __bfloat162float(u8[u]), __uint_as_float(ru[8 * j + u])));
                }
              }
            }
            uint32_t packed[16];
#pragma unroll
            for (int h = 0; h < 16; ++h) {
              float v2[2];
#pragma unroll
              for (int u = 0; u < 2; ++u) {
                const int i = 2 * h + u;
                const float g = __uint_as_float(rg[i]), up = __uint_as_float(ru[i]);
                v2[u] = g / (1.f + __expf(-g)) * up;
              }
              __nv_bfloat162 b2 = __floats2bfloat162_rn(v2[0], v2[1]);
              packed[h] = *reinterpret_cast<uint32_t*>(&b2);
            }
            __nv_bfloat16* dst = orow_ptr + col;
            if (v8) {
              ptx::st_global_v8(dst, packed);
              ptx::st_global_v8(dst + 16, packed + 8);
            } else {
#pragma unroll
              for (int j = 0; j < 4; ++j)
                *reinterpret_cast<uint4*>(dst + 8 * j) = make_uint4(
                    packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
            }
          }
        }
      } else if constexpr (L::ACC_BUFS == 1 && !F32) {
        // A 512-wide tile in two passes of 128 of this warp's TMEM columns: [0, 256) and then
        // [256, 512) of the accumulator. A pass takes its columns into registers as bf16,
        // hands that half of the accumulator back (tempty[pass]) and only then stores them,
        // so the next tile's MMAs overlap the stores.
        const int32_t sub = c_off / CW;
#pragma unroll 1
        for (int pass = 0; pass < 2; ++pass) {
          const int32_t tbase = pass * 256 + sub * 128;
          const uint32_t taddr = tmem_base + ((q * 32u) << 16) + (uint32_t)tbase;
          // output column of TMEM column t: column 128 (t / 256) + t % 128 of the leader's
          // (t % 256 < 128) or the follower's B half
          auto out_col = [&](int32_t t) {
            return tl.n0 + ((t % 256) / 128) * L::B_COLS + 128 * (t / 256) + t % 128;
          };
          uint32_t packed[64];
          uint32_t r0[32], r1[32];
          ptx::tmem_ld_32x32b_x32(taddr, r0);
#pragma unroll
          for (int c = 0; c < 128; c += 32) {
            uint32_t(&cur)[32] = ((c / 32) & 1) ? r1 : r0;
            uint32_t(&nxt)[32] = ((c / 32) & 1) ? r0 : r1;
            ptx::tmem_ld_wait();
            if (c + 32 < 128) ptx::tmem_ld_32x32b_x32(taddr + c + 32, nxt);
            const int32_t cc = out_col(tbase + c);
            if (bias_e != nullptr && row_ok && cc < p.out_cols) {
              // h = product + s_row * bias[e, col] (8-column groups up to out_cols)
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                if (cc + 8 * j < p.out_cols) {
                  const uint4 bv = *reinterpret_cast<const uint4*>(bias_e + cc + 8 * j);
                  const __nv_bfloat16* bb = reinterpret_cast<const __nv_bfloat16*>(&bv);
#pragma unroll
                  for (int u = 0; u < 8; ++u)
                    cur[8 * j + u] = __float_as_uint(
                        fmaf(s_row, __bfloat162float(bb[u]), __uint_as_float(cur[8 * j + u])));
                }
              }
            }
#pragma unroll
            for (int h = 0; h < 16; ++h) {
              __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(cur[2 * h]),
                                                        __uint_as_float(cur[2 * h + 1]));
              packed[c / 2 + h] = *reinterpret_cast<uint32_t*>(&b2);
            }
          }
          ptx::tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if constexpr (PAIR) ptx::mbar_arrive_cluster(pass ? tempty1 : tempty0);
            else                ptx::mbar_arrive(&sh.tempty[pass]);
          }
          if (row_ok) {
#pragma unroll
            for (int c = 0; c < 128; c += 32) {
              const int32_t cc = out_col(tbase + c);
              if (v8) {
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                  const int32_t col = cc + j * 16;
                  if (col < p.out_cols) ptx::st_global_v8(orow_ptr + col, packed + c / 2 + 8 * j);
                }
              } else {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  const int32_t col = cc + j * 8;
                  if (col < p.out_cols)
                    *reinterpret_cast<uint4*>(orow_ptr + col) =
                        make_uint4(packed[c / 2 + 4 * j], packed[c / 2 + 4 * j + 1],
                                   packed[c / 2 + 4 * j + 2], packed[c / 2 + 4 * j + 3]);
                }
              }
            }
          }
        }
      } else if constexpr (TMA_EPI) {
        // dW through shared memory and TMA: the warp's 128 columns in two blocks of 64, each
        // staged as 32 rows x 128 bytes (16-byte chunk j of row i at chunk j ^ (i % 8), the
        // 128-byte swizzle of the store's tensor map) and written by one tensor store; the map
        // covers dW as [E][K][N], so rows past K and columns past N are not written
        uint8_t* stg = smem + L::OFF_STG + (warp - 2) * 4096u;
        const uint32_t taddr = tmem_base + ((q * 32u) << 16) + a * BN + (uint32_t)c_off;
        const int32_t krow = tl.k0 + (int32_t)(rank * BM + q * 32);  // dW row of lane 0
#pragma unroll 1
        for (int blk = 0; blk < 2; ++blk) {
          uint32_t r0[32], r1[32];
          ptx::tmem_ld_32x32b_x32(taddr + blk * 64, r0);
          ptx::tmem_ld_32x32b_x32(taddr + blk * 64 + 32, r1);
          ptx::tmem_ld_wait();
          uint32_t packed[32];
#pragma unroll
          for (int h = 0; h < 16; ++h) {
            __nv_bfloat162 b0 = __floats2bfloat162_rn(__uint_as_float(r0[2 * h]),
                                                      __uint_as_float(r0[2 * h + 1]));
            __nv_bfloat162 b1 = __floats2bfloat162_rn(__uint_as_float(r1[2 * h]),
                                                      __uint_as_float(r1[2 * h + 1]));
            packed[h] = *reinterpret_cast<uint32_t*>(&b0);
            packed[16 + h] = *reinterpret_cast<uint32_t*>(&b1);
          }
          if (lane == 0) ptx::bulk_wait_read_all();  // the last store has read the buffer
          __syncwarp();
          uint8_t* row = stg + lane * 128u;
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<uint4*>(row + ((j ^ (int)(lane & 7u)) * 16)) =
                make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
          ptx::fence_proxy_async_smem();
          __syncwarp();
          // a box wholly past K or N (the last tiles of a K or N that is not a multiple of
          // the tile) is not stored at all; a box that only reaches past them is clipped
          const int32_t xcol = tl.n0 + c_off + blk * 64;
          if (lane == 0 && xcol < p.out_cols && krow < p.wg_K) {
            ptx::tma_store_3d(&mapC, stg, xcol, krow, tl.e);
            ptx::bulk_commit_group();
          }
        }
      } else {
      const uint32_t taddr = tmem_base + ((q * 32u) << 16) + a * BN + (uint32_t)c_off;
      // 32 columns per load; the next load is in flight while this chunk is stored
      uint32_t r0[32], r1[32];
      ptx::tmem_ld_32x32b_x32(taddr, r0);
#pragma unroll
      for (int c = 0; c < CW; c += 32) {
        uint32_t(&cur)[32] = ((c / 32) & 1) ? r1 : r0;
        uint32_t(&nxt)[32] = ((c / 32) & 1) ? r0 : r1;
        ptx::tmem_ld_wait();
        if (c + 32 < CW) ptx::tmem_ld_32x32b_x32(taddr + c + 32, nxt);
        // output column of the chunk's first accumulator column: TMEM column t of a 512-wide
        // pair tile is column 128 (t / 256) + t % 128 of the leader's (t % 256 < 128) or the
        // follower's B half; narrower tiles map TMEM columns to output columns one to one
        const int32_t tcol = c_off + c;
        const int32_t cc = BN > 256 ? tl.n0 + ((tcol % 256) / 128) * L::B_COLS +
                                          128 * (tcol / 256) + tcol % 128
                                    : col0 + c;
        if (F32 && row_ok) {
          // fp32 out = alpha * acc + beta * out; the old value is read only when beta != 0.
          // All of the chunk's old values are loaded before the first store, so that the
          // loads overlap instead of waiting behind stores the compiler cannot disambiguate.
          float* orow_f = p.out_f32 + orow * (int64_t)p.out_cols;
          float4 old[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) old[j] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (p.beta != 0.f) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
              if (cc + j * 4 < p.out_cols)
                old[j] = __ldg(reinterpret_cast<const float4*>(orow_f + cc + j * 4));
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int32_t col = cc + j * 4;
            if (col < p.out_cols) {
              float4 v = make_float4(p.alpha * __uint_as_float(cur[4 * j]),
                                     p.alpha * __uint_as_float(cur[4 * j + 1]),
                                     p.alpha * __uint_as_float(cur[4 * j + 2]),
                                     p.alpha * __uint_as_float(cur[4 * j + 3]));
              if (p.beta != 0.f) {
                v.x = fmaf(p.beta, old[j].x, v.x);
                v.y = fmaf(p.beta, old[j].y, v.y);
                v.z = fmaf(p.beta, old[j].z, v.z);
                v.w = fmaf(p.beta, old[j].w, v.w);
              }
              *reinterpret_cast<float4*>(orow_f + col) = v;
            }
          }
        } else if (row_ok) {
          if (bias_e != nullptr && cc < p.out_cols) {
            // h = product + s_row * bias[e, col]; out_cols is a multiple of 8, so a 32-wide
            // chunk is read only up to its last valid 8-column group
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              if (cc + 8 * j < p.out_cols) {
                const uint4 bv = *reinterpret_cast<const uint4*>(bias_e + cc + 8 * j);
                const __nv_bfloat16* bb = reinterpret_cast<const __nv_bfloat16*>(&bv);
#pragma unroll
                for (int u = 0; u < 8; ++u)
                  cur[8 * j + u] = __float_as_uint(
                      fmaf(s_row, __bfloat162float(bb[u]), __uint_as_float(cur[8 * j + u])));
              }
            }
          }
          uint32_t packed[16];
#pragma unroll
          for (int h = 0; h < 16; ++h) {
            __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(cur[2 * h]),
                                                      __uint_as_float(cur[2 * h + 1]));
            packed[h] = *reinterpret_cast<uint32_t*>(&b2);
          }
          if (v8) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const int32_t col = cc + j * 16;
              if (col < p.out_cols) ptx::st_global_v8(orow_ptr + col, packed + 8 * j);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int32_t col = cc + j * 8;
              if (col < p.out_cols)
                *reinterpret_cast<uint4*>(orow_ptr + col) =
                    make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
            }
          }
        }
      }
      }  // ACT
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (L::ACC_BUFS == 1) {
          // one accumulator, handed back in two halves: the register-staged bf16 epilogue
          // above has released both; the SiLU and fp32 epilogues release both here
          if constexpr (ACT == 1 || F32) {
            if constexpr (PAIR) {
              ptx::mbar_arrive_cluster(tempty0);
              ptx::mbar_arrive_cluster(tempty1);
            } else {
              ptx::mbar_arrive(&sh.tempty[0]);
              ptx::mbar_arrive(&sh.tempty[1]);
            }
          }
        } else {
          if constexpr (PAIR) ptx::mbar_arrive_cluster(a ? tempty1 : tempty0);
          else                ptx::mbar_arrive(&sh.tempty[a]);
        }
      }
      ++acc_iter;
    }
    if constexpr (TMA_EPI) {
      // every tensor store of this warp has written dW before the CTA can exit
      if (lane == 0) ptx::bulk_wait_all();
      __syncwarp();
    }
  } else if constexpr (MODE == Mode::Wgrad) {
    // ------------------------------------------------------------ wgrad tail fix-up
    // Walks the same stage sequence as the load warp. For a stage that ends its group, rows
    // [rem, ceil16(rem)) belong to the next group (or to no group): they are zeroed in both
    // operands so that they add nothing (the MMA reads no row past ceil16(rem)); a token row
    // is one 128-byte line of every 64-wide chunk.
    uint32_t stage = 0, landed_par = 0;
    for (int32_t it = 0, t = tile_at<MODE>(unit0, 0, units); t < total;
         t = tile_at<MODE>(unit0, ++it, units)) {
      const Tile tl = decode_tile<MODE, BN, TM>(t, p, sh);
      const bool rev = GG_SERPENTINE && (it & 1);
      bool ok = true;
      for (int32_t kq = 0; kq < tl.kblocks; ++kq) {
        const int32_t kb = rev ? tl.kblocks - 1 - kq : kq;
        const int32_t rem = tl.tok_len - kb * BKM;
        if (rem < BKM) {
          const uint32_t lp = (landed_par >> stage) & 1u;
          landed_par ^= 1u << stage;
          if (!warp_wait(&sh.landed[stage], lp, sh, p, false)) { ok = false; break; }
          uint8_t* sA = smem + L::OFF_A + stage * L::A_BYTES;
          uint8_t* sB = smem + L::OFF_B + stage * L::B_BYTES;
          const int nsub = (rem + UMMA_K - 1) / UMMA_K;
          const int zrows = nsub * UMMA_K - rem;
          const int lines_a = zrows * 2, lines_b = zrows * (L::B_COLS / 64);
          for (int i = (int)lane; i < (lines_a + lines_b) * 8; i += 32) {
            const int line = i >> 3, part = i & 7;
            uint8_t* dst;
            if (line < lines_a) {
              dst = sA + (line / zrows) * L::CHUNK_BYTES + (rem + line % zrows) * 128 + part * 16;
            } else {
              const int l2 = line - lines_a;
              dst = sB + (l2 / zrows) * L::CHUNK_BYTES + (rem + l2 % zrows) * 128 + part * 16;
            }
            *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
          }
          ptx::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (leader) ptx::mbar_arrive(&sh.full[stage]);  // the leader's half completes full[]
            else ptx::mbar_arrive_cluster(ptx::mapa(ptx::smem_u32(&sh.fixed[stage]), 0));
          }
        }
        if (++stage == STAGES) stage = 0;
      }
      if (!ok) break;
    }
  }

  ptx::tc_fence_before();
  if constexpr (PAIR) ptx::cluster_sync();  // no CTA of the pair leaves while the other may
  else __syncthreads();                      // still signal its barriers or tensor memory
  if (warp == 1) {
    ptx::tc_fence_after();
    if constexpr (PAIR) ptx::tmem_dealloc_pair(tmem_base, L::TMEM_COLS);
    else                ptx::tmem_dealloc(tmem_base, L::TMEM_COLS);
  }
  if (blockIdx.x == 0 && threadIdx.x == 0 && !*sh.abort_flag) set_status(p, DEV_LAUNCHED);
}

}  // namespace gg
