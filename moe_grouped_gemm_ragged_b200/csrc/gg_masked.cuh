// Masked forward for the small-batch layout of sglang PR 32385 ("Evidence": g, mmax, k, n =
// 8, 128, 768, 2048): out[e, r, :] = A[e, r, :] . W[e] for r < masked_m[e].
//
// With at most a few dozen active rows per expert this operation is bound by reading W from
// HBM once, not by the tensor cores. The kernel therefore makes the weight columns the MMA's
// M dimension (128 TMEM lanes) and the active token rows its N dimension (16 to 128 columns,
// rounded up from the expert's row count), so that:
//   - a stage of W is 128 columns x 64 reduction elements (16 KB) and a stage of tokens holds
//     only the rows that exist (one or two TMA boxes of 32, 64 or 128 rows); the two have
//     rings of their own, fed by two producer warps;
//   - the tensor work per stage shrinks with the number of active rows.
// On the shape above a call measures 8.6 us with its inputs coming from HBM, against 11.5 us
// for the grouped GEMM kernel's masked mode (token rows as the MMA's M, one ring of 32 KB
// stages).
// A tile is (expert, block of up to 128 active rows, 128 weight columns). The accumulator
// D[n, j] = sum_k W[e, k, n] * A[e, r0 + j, k] sits in TMEM with lane n and column j; the
// epilogue transposes 32 x 32 blocks through shared memory and writes 16-byte pieces of the
// output rows r < masked_m[e] only.
//
// Two schedules:
//   one tile per CTA (when every (expert, row block, column tile) has a CTA of its own, as in
//     the shape above: 8 x 1 x 16 = 128 tiles): a CTA's tile is its block index, so before the
//     grid dependency resolves it already prefetches its weight slice into L2, and right after
//     it issues the first weight stages, before the expert's row count has arrived; each role
//     reads masked_m[e] itself, and a tile with no active row just lets its loads land;
//   a tile list (otherwise): every CTA builds the table of active tiles from masked_m (clamp,
//     prefix sums) and takes tiles blockIdx.x, blockIdx.x + gridDim.x, ...
//
// Roles of the 11 warps: warp 0 loads W, warp 10 loads token rows, warp 1 owns tensor
// memory and issues the MMAs, warps 2..9 are the epilogue (two per TMEM lane quadrant, each
// taking every other 32-column block of the accumulator, i.e. 32 token rows). Every wait is
// bounded by the watchdog, as in the grouped GEMM kernel.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace gg {
namespace masked {

constexpr int TILE_N = 128;  // weight columns per tile: the MMA's M
constexpr int TILE_T = 128;  // token rows per tile at most: the MMA's N
constexpr int KBLK = 64;     // reduction elements per stage (128 bytes of bf16)
constexpr uint32_t W_STAGE = TILE_N * KBLK * 2;
constexpr uint32_t T_STAGE = TILE_T * KBLK * 2;
constexpr uint32_t W_CHUNK = KBLK * 128;  // one 64-column chunk of a weight stage
constexpr int EPI_WARP0 = 2;
// Epilogue warps: two per TMEM lane quadrant, taking 32-column blocks (32 token rows each)
// c and c + 2 (four per quadrant, one block each, measured slower on the sglang shape).
constexpr int EPI_WARPS = 8;
constexpr int TOK_WARP = EPI_WARP0 + EPI_WARPS;
constexpr int THREADS = 32 * (TOK_WARP + 1);
constexpr uint32_t EPI_BUF = 32 * 32 * 2;  // per epilogue warp: 32 rows x 32 columns of bf16
constexpr uint32_t TMEM_COLS = 2 * TILE_T;  // double-buffered accumulator

constexpr int DEV_BAD_MASKED_M = 0x2;
constexpr int DEV_TIMEOUT = 0x4;
constexpr int DEV_LAUNCHED = 0x100;

struct Params {
  const int32_t* masked_m;          // [E], device
  __nv_bfloat16* out;               // [E, mmax, N]
  int32_t* status;                  // may be null
  const __nv_bfloat16* bias;        // [E, N] or null
  const float* bias_scale;          // [E * mmax] (flat output row) or null; needs bias
  int32_t E;
  int32_t mmax;
  int32_t K;
  int32_t N;
  uint64_t watchdog_ns;
  int32_t debug_flags;              // bit 0: CTA 0 skips its first weight load
  int32_t w_chunked;                // N % 64 == 0: one 4-D box brings both column chunks
  int32_t one_tile;                 // the grid has one CTA per (expert, row block, column tile)
};

template <int SW, int ST>
struct Layout {
  static constexpr uint32_t OFF_W = 0;
  static constexpr uint32_t OFF_T = SW * W_STAGE;
  static constexpr uint32_t OFF_EPI = OFF_T + ST * T_STAGE;
  static constexpr uint32_t OFF_BAR = OFF_EPI + EPI_WARPS * EPI_BUF;
  // wfull, wempty per weight stage; tfull, tempty per token stage; afull x2, aempty x2, fin
  static constexpr uint32_t NUM_BARS = 2 * SW + 2 * ST + 5;
  static constexpr uint32_t OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr uint32_t OFF_TAB = OFF_MISC + 16;
  // tile-list schedule: rows[E] (clamped masked_m), prefix[E + 1] (tile prefix sums)
  static __host__ __device__ constexpr uint32_t bytes(int E) {
    return OFF_TAB + 4u * (2u * (uint32_t)E + 1u) + 1024u /* alignment slack */;
  }
};

struct Ctx {
  volatile int32_t* abort_flag;
  const Params* p;
};

__device__ __forceinline__ void set_status(const Params& p, int bits) {
  if (p.status != nullptr) atomicOr(p.status, bits);
}

// Bounded wait on one phase of an mbarrier (see the grouped GEMM kernel): true once the phase
// completed; false when the CTA aborts (honour_abort) or the watchdog expires, which sets the
// abort flag and GG_DEV_TIMEOUT.
__device__ __noinline__ bool wait_slow(uint64_t* bar, uint32_t parity, const Ctx& c,
                                       bool honour_abort) {
  const uint64_t t0 = ptx::globaltimer();
  for (;;) {
    if (ptx::mbar_try_wait(bar, parity, 200000)) return true;
    if (honour_abort && *c.abort_flag) return false;
    if (ptx::globaltimer() - t0 > c.p->watchdog_ns) {
      *c.abort_flag = 1;
      set_status(*c.p, DEV_TIMEOUT);
      return false;
    }
  }
}

__device__ __forceinline__ bool wait(uint64_t* bar, uint32_t parity, const Ctx& c,
                                     bool honour_abort = true) {
  if (ptx::mbar_try_wait(bar, parity, 200000)) return true;
  return wait_slow(bar, parity, c, honour_abort);
}

struct Tile {
  int32_t e;
  int32_t tok0;  // first row of the block inside the expert
  int32_t rows;  // active rows of the block (at most TILE_T; <= 0: no work)
  int32_t n0;    // first weight column
};

// Tile t of the list over active tiles: largest e with prefix[e] <= t (experts without tiles
// share their successor's prefix), then row block and column tile, column tile fastest.
__device__ __forceinline__ Tile decode_list(int32_t t, int32_t E, int32_t NT, const int32_t* rows,
                                            const int32_t* prefix) {
  int32_t lo = 0, hi = E - 1;
  while (lo < hi) {
    const int32_t mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= t) lo = mid; else hi = mid - 1;
  }
  Tile tl;
  tl.e = lo;
  const int32_t local = t - prefix[lo];
  const int32_t tb = local / NT;
  tl.n0 = (local - tb * NT) * TILE_N;
  tl.tok0 = tb * TILE_T;
  const int32_t left = rows[lo] - tl.tok0;
  tl.rows = left < TILE_T ? left : TILE_T;
  return tl;
}

// The one-tile schedule's tile of this CTA, row count not yet known.
__device__ __forceinline__ Tile decode_block(int32_t b, int32_t NT, int32_t TB) {
  Tile tl;
  tl.e = b / (TB * NT);
  const int32_t r = b - tl.e * (TB * NT);
  const int32_t tb = r / NT;
  tl.n0 = (r - tb * NT) * TILE_N;
  tl.tok0 = tb * TILE_T;
  tl.rows = 0;
  return tl;
}

// Active rows of the block from masked_m[e] (clamped to [0, mmax]); the status bit is set by
// the caller that passes report = true.
__device__ __forceinline__ int32_t block_rows(const Params& p, const Tile& tl, bool report) {
  const int32_t g = p.masked_m[tl.e];
  const int32_t m = g < 0 ? 0 : (g > p.mmax ? p.mmax : g);
  if (report && m != g) set_status(p, DEV_BAD_MASKED_M);
  const int32_t left = m - tl.tok0;
  return left < TILE_T ? left : TILE_T;
}

template <int SW, int ST>
__global__ void __launch_bounds__(THREADS, 1)
    masked_forward_kernel(const __grid_constant__ CUtensorMap mapW,
                          const __grid_constant__ CUtensorMap mapT32,
                          const __grid_constant__ CUtensorMap mapT64,
                          const __grid_constant__ CUtensorMap mapT128, const Params p) {
  using L = Layout<SW, ST>;
  static_assert(SW <= 32 && ST <= 32, "stage bitmasks are 32 bits wide");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = ptx::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* wfull = bars;
  uint64_t* wempty = bars + SW;
  uint64_t* tfull = bars + 2 * SW;
  uint64_t* tempty = bars + 2 * SW + ST;
  uint64_t* afull = bars + 2 * SW + 2 * ST;
  uint64_t* aempty = afull + 2;
  uint64_t* fin = afull + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(smem + L::OFF_MISC + 4);
  int32_t* total_p = reinterpret_cast<int32_t*>(smem + L::OFF_MISC + 8);
  int32_t* rows_tab = reinterpret_cast<int32_t*>(smem + L::OFF_TAB);
  int32_t* prefix = rows_tab + p.E;

  const uint32_t warp = threadIdx.x / 32;
  const uint32_t lane = ptx::lane_id();
  const Ctx ctx{abort_flag, &p};
  const int32_t E = p.E;
  const int32_t NT = (p.N + TILE_N - 1) / TILE_N;
  const int32_t TB = (p.mmax + TILE_T - 1) / TILE_T;
  const int32_t nkb = (p.K + KBLK - 1) / KBLK;
  const bool one_tile = p.one_tile != 0;
  const Tile mine = decode_block((int32_t)blockIdx.x, NT, TB);  // one-tile schedule only

  if (threadIdx.x == 0) {
    for (int s = 0; s < SW; ++s) {
      ptx::mbar_init(&wfull[s], 1);
      ptx::mbar_init(&wempty[s], 1);
    }
    for (int s = 0; s < ST; ++s) {
      ptx::mbar_init(&tfull[s], 1);
      ptx::mbar_init(&tempty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(&afull[a], 1);
      ptx::mbar_init(&aempty[a], EPI_WARPS);
    }
    ptx::mbar_init(fin, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&mapW);
    ptx::prefetch_tmap(&mapT32);
    ptx::prefetch_tmap(&mapT64);
    ptx::prefetch_tmap(&mapT128);
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  if (one_tile && threadIdx.x == 0) {
    // warm L2 with this CTA's weight slice while the previous kernel may still be running
    for (int32_t kb = 0; kb < nkb; ++kb) {
      if (p.w_chunked) {
        ptx::tma_prefetch_l2_4d(&mapW, 0, kb * KBLK, mine.n0 / 64, mine.e);
      } else {
        ptx::tma_prefetch_l2_3d(&mapW, mine.n0, kb * KBLK, mine.e);
        ptx::tma_prefetch_l2_3d(&mapW, mine.n0 + 64, kb * KBLK, mine.e);
      }
    }
  }
  // Up to here nothing was read that the previous kernel of the stream may write; from here
  // on its writes (and its completion) are visible.
  ptx::griddep_wait();
  int32_t total = 0;
  if (!one_tile) {
    // tile list: every thread fetches a share of masked_m, warp 0 clamps and prefix-sums
    for (int32_t i = threadIdx.x; i < E; i += THREADS) rows_tab[i] = p.masked_m[i];
    __syncthreads();
    if (warp == 0) {
      int32_t carry = 0;
      bool bad = false;
      if (lane == 0) prefix[0] = 0;
      for (int32_t base = 0; base < E; base += 32) {
        const int32_t e = base + (int32_t)lane;
        int32_t tiles = 0;
        if (e < E) {
          const int32_t g = rows_tab[e];
          const int32_t m = g < 0 ? 0 : (g > p.mmax ? p.mmax : g);
          bad |= m != g;
          rows_tab[e] = m;
          tiles = ((m + TILE_T - 1) / TILE_T) * NT;
        }
        int32_t s = tiles;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
          const int32_t o = __shfl_up_sync(0xffffffffu, s, d);
          if ((int)lane >= d) s += o;
        }
        if (e < E) prefix[e + 1] = carry + s;
        carry += __shfl_sync(0xffffffffu, s, 31);
      }
      if (__any_sync(0xffffffffu, bad) && lane == 0) set_status(p, DEV_BAD_MASKED_M);
      if (lane == 0) *total_p = carry;
    }
    __syncthreads();
    total = *total_p;
  }
  ptx::griddep_launch_dependents();

  // Tile i of this CTA (false past its last). In the one-tile schedule the row count comes
  // from masked_m, read by the caller (`rows` = -1: not read yet).
  auto tile_at = [&](int32_t i, Tile& tl) -> bool {
    if (one_tile) {
      if (i > 0) return false;
      tl = mine;
      return true;
    }
    const int32_t t = (int32_t)blockIdx.x + i * (int32_t)gridDim.x;
    if (t >= total) return false;
    tl = decode_list(t, E, NT, rows_tab, prefix);
    return true;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ weight producer
    // In the one-tile schedule the first stages go out before the row count is known; when
    // the block turns out to have no row, the MMA never consumes them and they only land.
    if (lane == 0) {
      const uint64_t pol = ptx::l2_policy<1>();  // each weight slice is read once
      bool skip = (p.debug_flags & 1) && blockIdx.x == 0;
      uint32_t s = 0, ph = 0, armed = 0, armed_ph = 0;
      bool ok = true;
      Tile tl;
      for (int32_t i = 0; ok && tile_at(i, tl); ++i) {
        for (int32_t kb = 0; kb < nkb; ++kb) {
          // one tile: stages 0..SW-1 start on a fresh ring; at stage SW the row count decides
          if (one_tile && kb == SW && block_rows(p, tl, false) <= 0) break;
          if (!one_tile || kb >= SW) {
            if (!wait(&wempty[s], ph ^ 1u, ctx)) { ok = false; break; }
          }
          uint8_t* dst = smem + L::OFF_W + s * W_STAGE;
          if (skip) {
            skip = false;  // watchdog test: this stage is never armed
          } else {
            armed |= 1u << s;
            armed_ph = (armed_ph & ~(1u << s)) | (ph << s);
            ptx::mbar_arrive_expect_tx(&wfull[s], W_STAGE);
            if (p.w_chunked) {
              ptx::tma_load_4d(dst, &mapW, &wfull[s], 0, kb * KBLK, tl.n0 / 64, tl.e, pol);
            } else {
              ptx::tma_load_3d(dst, &mapW, &wfull[s], tl.n0, kb * KBLK, tl.e, pol);
              ptx::tma_load_3d(dst + W_CHUNK, &mapW, &wfull[s], tl.n0 + 64, kb * KBLK, tl.e,
                               pol);
            }
          }
          if (++s == (uint32_t)SW) { s = 0; ph ^= 1u; }
        }
      }
      // every armed load lands before the CTA may exit (after an abort some may be in flight)
      for (int i = 0; i < SW; ++i)
        if (armed & (1u << i)) wait(&wfull[i], (armed_ph >> i) & 1u, ctx, false);
    }
    __syncwarp();
  } else if (warp == TOK_WARP) {
    // ------------------------------------------------------------ token producer
    if (lane == 0) {
      const uint64_t pol = ptx::l2_policy<2>();  // token rows are read by every column tile
      uint32_t s = 0, ph = 0, armed = 0, armed_ph = 0;
      bool ok = true;
      Tile tl;
      for (int32_t i = 0; ok && tile_at(i, tl); ++i) {
        if (one_tile) tl.rows = block_rows(p, tl, false);
        if (tl.rows <= 0) continue;
        const int32_t row0 = tl.e * p.mmax + tl.tok0;
        // one or two boxes covering the active rows: 32, 64, 64 + 32 or 128 rows (rows past
        // the active ones only reach accumulator columns that are never stored)
        const int32_t box_rows = tl.rows <= 32 ? 32 : tl.rows <= 64 ? 64 : tl.rows <= 96 ? 96 : 128;
        for (int32_t kb = 0; kb < nkb; ++kb) {
          if (!wait(&tempty[s], ph ^ 1u, ctx)) { ok = false; break; }
          uint8_t* dst = smem + L::OFF_T + s * T_STAGE;
          armed |= 1u << s;
          armed_ph = (armed_ph & ~(1u << s)) | (ph << s);
          ptx::mbar_arrive_expect_tx(&tfull[s], (uint32_t)box_rows * 128u);
          const int32_t x = kb * KBLK;
          if (box_rows == 32) {
            ptx::tma_load_2d(dst, &mapT32, &tfull[s], x, row0, pol);
          } else if (box_rows == 64) {
            ptx::tma_load_2d(dst, &mapT64, &tfull[s], x, row0, pol);
          } else if (box_rows == 96) {
            ptx::tma_load_2d(dst, &mapT64, &tfull[s], x, row0, pol);
            ptx::tma_load_2d(dst + 64 * 128, &mapT32, &tfull[s], x, row0 + 64, pol);
          } else {
            ptx::tma_load_2d(dst, &mapT128, &tfull[s], x, row0, pol);
          }
          if (++s == (uint32_t)ST) { s = 0; ph ^= 1u; }
        }
      }
      for (int i = 0; i < ST; ++i)
        if (armed & (1u << i)) wait(&tfull[i], (armed_ph >> i) & 1u, ctx, false);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t sw = 0, pw = 0, st = 0, pt = 0, acc_iter = 0;
      bool ok = true;
      Tile tl;
      for (int32_t i = 0; ok && tile_at(i, tl); ++i) {
        // the MMA issuer reports an out-of-range masked_m (once per expert)
        if (one_tile) tl.rows = block_rows(p, tl, tl.n0 == 0 && tl.tok0 == 0);
        if (tl.rows <= 0) continue;
        const uint32_t a = acc_iter & 1u;
        if (!wait(&aempty[a], ((acc_iter >> 1) & 1u) ^ 1u, ctx)) break;
        ptx::tc_fence_after();
        // M = 128 weight columns (MN-major in shared memory), N = the block's rows rounded up
        // to 16 (K-major); columns past the active rows are never stored
        const uint32_t n_mma = (uint32_t)((tl.rows + 15) / 16) * 16u;
        const uint32_t idesc = ptx::idesc_bf16_f32(TILE_N, n_mma, 1u, 0u);
        const uint32_t d_tmem = tmem_base + a * TILE_T;
        for (int32_t kb = 0; kb < nkb; ++kb) {
          if (!wait(&wfull[sw], pw, ctx) || !wait(&tfull[st], pt, ctx)) { ok = false; break; }
          ptx::tc_fence_after();
          const uint64_t adesc =
              ptx::smem_desc_sw128(ptx::smem_u32(smem + L::OFF_W + sw * W_STAGE), W_CHUNK, 1024);
          const uint64_t bdesc =
              ptx::smem_desc_sw128(ptx::smem_u32(smem + L::OFF_T + st * T_STAGE), 16, 1024);
#pragma unroll
          for (int k = 0; k < KBLK / 16; ++k)
            // 16 reduction rows of the MN-major weight stage are 2 KB on, 16 elements of a
            // K-major token row 32 bytes on (descriptor addresses count 16-byte units)
            ptx::mma_bf16(d_tmem, adesc + (uint64_t)k * (2048u >> 4),
                          bdesc + (uint64_t)k * (32u >> 4), idesc, (kb > 0 || k > 0) ? 1u : 0u);
          ptx::mma_commit(&wempty[sw]);
          ptx::mma_commit(&tempty[st]);
          if (++sw == (uint32_t)SW) { sw = 0; pw ^= 1u; }
          if (++st == (uint32_t)ST) { st = 0; pt ^= 1u; }
        }
        if (!ok) break;
        ptx::mma_commit(&afull[a]);
        ++acc_iter;
      }
      // every MMA issued completes before tensor memory is released
      ptx::mma_commit(fin);
      wait(fin, 0, ctx, false);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..17)
    const uint32_t q = warp & 3u;                       // TMEM lane quadrant = weight columns
    const int32_t c0 = ((int32_t)warp - EPI_WARP0) / 4;  // first 32-column block (32 rows)
    uint16_t* buf = reinterpret_cast<uint16_t*>(smem + L::OFF_EPI + (warp - EPI_WARP0) * EPI_BUF);
    uint32_t acc_iter = 0;
    Tile tl;
    for (int32_t i = 0; tile_at(i, tl); ++i) {
      if (one_tile) {
        int32_t r = 0;
        if (lane == 0) r = block_rows(p, tl, false);
        tl.rows = __shfl_sync(0xffffffffu, r, 0);
      }
      if (tl.rows <= 0) continue;
      const uint32_t a = acc_iter & 1u;
      bool ok = true;
      if (lane == 0) ok = wait(&afull[a], (acc_iter >> 1) & 1u, ctx);
      if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) break;
      ptx::tc_fence_after();
      for (int32_t c = c0; c * 32 < tl.rows; c += EPI_WARPS / 4) {
        uint32_t v[32];
        ptx::tmem_ld_32x32b_x32(tmem_base + ((q * 32u) << 16) + a * TILE_T + (uint32_t)c * 32u, v);
        ptx::tmem_ld_wait();
        const int32_t ncol = tl.n0 + (int32_t)(q * 32u + lane);  // this lane's weight column
        const int64_t row_base = (int64_t)tl.e * p.mmax + tl.tok0;  // flat output row of j = 0
        if (p.bias != nullptr) {
          // h = product + s[row] * bias[e, n]; s is read only for active rows
          const int32_t jr = c * 32 + (int32_t)lane;
          float s_l = 1.f;
          if (p.bias_scale != nullptr && jr < tl.rows) s_l = p.bias_scale[row_base + jr];
          const float b_n =
              ncol < p.N ? __bfloat162float(p.bias[(int64_t)tl.e * p.N + ncol]) : 0.f;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float s_j = __shfl_sync(0xffffffffu, s_l, j);
            v[j] = __float_as_uint(fmaf(s_j, b_n, __uint_as_float(v[j])));
          }
        }
        // transpose: buf[j][lane] holds row j, weight column lane of this warp's 32
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const __nv_bfloat16 x = __float2bfloat16_rn(__uint_as_float(v[j]));
          buf[j * 32 + (int)lane] = *reinterpret_cast<const uint16_t*>(&x);
        }
        __syncwarp();
        // 32 rows x 64 bytes: lane takes 16-byte piece (i * 32 + lane) -> row /4, part %4
#pragma unroll
        for (int i2 = 0; i2 < 4; ++i2) {
          const int idx = i2 * 32 + (int)lane;
          const int j = idx >> 2, part = idx & 3;
          const int32_t jr = c * 32 + j;
          const int32_t col = tl.n0 + (int32_t)q * 32 + part * 8;
          if (jr < tl.rows && col < p.N) {
            const uint4 val = *reinterpret_cast<const uint4*>(buf + j * 32 + part * 8);
            *reinterpret_cast<uint4*>(p.out + (row_base + jr) * (int64_t)p.N + col) = val;
          }
        }
        __syncwarp();
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&aempty[a]);
      ++acc_iter;
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, TMEM_COLS);
  }
  if (blockIdx.x == 0 && threadIdx.x == 0 && !*abort_flag) set_status(p, DEV_LAUNCHED);
}

}  // namespace masked
}  // namespace gg
