// fp8_gemm_kernels.cuh -- sm_100a kernels of the FP8 block-scaled NT GEMM.
//
// What they compute (see include/fp8gemm.h for the sources on the pages):
//   C[m,n] = bf16( sum_kb P_kb[m,n] * sfa[kb][m] * sfb[n/128][kb] ),
// P_kb = the 128-deep FP8 product of K block kb, formed by tcgen05.mma in TMEM
// and promoted by CUDA-core warps into FP32 register accumulators (the
// two-level accumulation of the news article's optimisation paragraph and of
// the turtlesai.it summary).
//
// Warp roles (kernel 2: 320 threads; kernel 1: 384 threads, the last four warps being
// warpgroup 2 of which warps 10-11 idle):
//   warps 0-7 : promotion + epilogue.  Warp w reads TMEM lanes 32*(w%4)..+31
//               (the lane quadrant its SM sub-partition can reach) and column
//               half w/4 of every partial tile.
//   warp 8    : TMA producer (one elected lane): A/B K-block tiles into an
//               S-stage shared-memory ring, 128-byte swizzled.
//   warp 9    : TMEM owner and MMA issuer (one lane): per K block, four
//               tcgen05.mma (K = 32 each) into a free TMEM partial buffer, then
//               tcgen05.commit to release the smem stage and to hand the
//               buffer to the promotion warps.
// TMEM holds several partial buffers so the MMA of block kb+1.. runs while
// block kb is being promoted; the FP32 accumulators live in registers.
//
// Kernel 1, fp8_gemm_tiled_kernel: persistent CTAs walk 128 x BN output tiles
//   (dense, M-grouped contiguous, M-grouped masked) in groups of m-blocks,
//   m-block fastest.  The masked walk enumerates only live tiles from masked_m
//   read on the device.  The epilogue stores bf16 through shared memory with TMA.
// Kernel 2, fp8_gemm_swap_streamk_kernel (dense, M <= 128, the decode shapes):
//   swap-AB -- 128 weight rows of B form the MMA's M side and the MP tokens
//   its N side -- and stream-K: the (n-block, K-block) units are split evenly
//   over the persistent CTAs; tiles split between CTAs are summed by the last
//   CTA to finish (fp32 partials in a workspace, fixed summation order, no
//   CTA waits on another).
#pragma once

#include <cuda_bf16.h>
#ifndef __CUDACC_RTC__
#include <cstdint>
#endif

#include "sm100_ptx.cuh"

namespace fg {

constexpr int kBlockK = 128;       // K block = scale granularity = one 128-byte swizzle row
constexpr int kBlockM = 128;       // MMA M (rows of the TMEM accumulator)
constexpr int kThreads = 320;
constexpr int kPromoWarps = 8;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s, far above any legal wait
constexpr int kErrTimeout = 6;       // FG_ERR_TIMEOUT
constexpr int kErrDeviceCheck = 7;   // FG_ERR_DEVICE_CHECK (debug builds only)
constexpr int kMaskedMaxGroups = 1024;
constexpr int kSwapScaleBytes = 12 * 1024;  // shared memory for staged combined scales (swap kernel)
constexpr int kSwapBarrierBytes = 512;      // shared memory for the swap kernel's mbarriers and flags
constexpr int kSaChunk = 8;                 // K blocks per staged scale chunk (tiled kernel)
constexpr int kTiledThreads = 384;          // tiled kernel: three warpgroups
constexpr int kTiledLaunchRegs = 168;       // registers per thread the tiled kernel is launched with
// Registers per thread after setmaxnreg, by tile width: the two promotion warpgroups hold the
// fp32 accumulators and a TMEM slice; the producer / MMA warpgroup needs more with the deeper ring
// and four TMEM buffers of the 128-wide tile.  Both must add up to at most the launch budget.
template <int BN>
struct RegSplit {
  static constexpr int promo = BN == 128 ? 216 : 232;
  static constexpr int ctrl = BN == 128 ? 72 : 40;
  static_assert(2 * 128 * promo + 128 * ctrl <= kTiledThreads * kTiledLaunchRegs, "register split");
};

enum Mode : int { kDense = 0, kContiguous = 1, kMasked = 2 };

// Promotion read pattern of the 256-wide tiles (promote_kblock's PIPE; a build-time knob).
#ifndef FG_PIPE_256
#define FG_PIPE_256 2
#endif

struct TiledParams {
  const float* sfa;
  const float* sfb;
  __nv_bfloat16* C;
  const int* m_indices;  // contiguous
  const int* masked_m;   // masked
  int* status;
  int M;        // dense: M, contiguous: M_total, masked: Mmax
  int N;
  int K;
  int G;
  int ld;       // sfa leading dimension
  int num_kb;   // ceil(K / 128)
  int num_nb;   // ceil(N / 128): sfb blocks per group
  int m_blocks; // ceil(M / 128)
  int n_blocks; // ceil(N / BN)
  int group_m;  // tile order: groups of group_m m-blocks, m-block fastest inside a group
  int b_resident;  // 1: the walk keeps B in L2 (n-block fastest): A loads evict first, B loads last
  uint32_t fmt_bits;  // operand formats in instruction-descriptor position (0: both e4m3)
  float* ws;        // stream-K tail: 2 * gridDim.x partial tiles of 128 x BN fp32
  int* counters;    // stream-K tail: one per tile of the last partial wave, zero between launches
  int counter_cap;  // entries of `counters`
  int sk_overhead;  // < 0: no stream-K tail; else the K blocks a split must save to be taken
};

struct SwapParams {
  const float* sfa;
  const float* sfb;
  __nv_bfloat16* C;
  float* ws;       // 2 * gridDim.x partial tiles of MP x 128 fp32
  int* counters;   // one per n-tile, zero between launches
  int counter_cap; // entries of `counters`
  int* status;
  int M, N, K, ld;
  int num_kb;
  int n_tiles;     // ceil(N / 128)
  int debug_stall; // test hook: 1 = the MMA thread first waits on a barrier no one arrives at
  uint32_t fmt_bits;  // operand formats in instruction-descriptor position (MMA A = weights)
  int tile_aligned;   // 1: CTA c takes whole tiles [c*T/P, (c+1)*T/P) (no split tiles, no fix-up)
  int cluster;        // S > 1: the S CTAs of cluster t split tile t in K and sum it through
                      // distributed shared memory (launched with cluster dims S, grid = tiles * S)
  int static_b;       // 1: B and sfb are not written by the preceding kernel of the stream, so the
                      // weight tiles of the first ring stages are loaded before waiting for it
};

__device__ __forceinline__ uint8_t* align_1024(uint8_t* p) {
  const uint32_t a = smem_addr(p);
  return p + ((1024u - (a & 1023u)) & 1023u);
}

__device__ __forceinline__ void report_timeout(int* status) { atomicCAS(status, 0, kErrTimeout); }

// Debug builds (-DFG_DEBUG): device-side checks of indices the kernels derive from their inputs
// or their schedule -- TMA tile coordinates, expert indices read from m_indices, split-K
// workspace slots and counters.  A failed check records FG_ERR_DEVICE_CHECK in the status word
// (first error wins) and the kernel carries on exactly as a release build would; nothing traps.
#ifdef FG_DEBUG
#define FG_DCHECK(cond, status)                                           \
  do {                                                                    \
    if (!(cond)) atomicCAS((status), 0, ::fg::kErrDeviceCheck);           \
  } while (0)
#else
#define FG_DCHECK(cond, status) \
  do {                          \
  } while (0)
#endif

// Wait for the phase of `bar` with parity `parity` regardless of the abort flag
// (used only to drain this CTA's own copies after an abort); bounded.
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > kWaitLimitNs) return;
  }
}

// Bounded barrier of the promotion threads: each arrives on `bar` (count =
// number of promotion threads) and waits for the phase to complete.  Unlike
// bar.sync it gives up after the wait limit, so an aborting warp cannot leave
// the others stuck.
__device__ __forceinline__ bool group_sync(uint64_t* bar, uint32_t& phase, volatile int* abort_flag) {
  mbar_arrive(bar);
  const bool ok = mbar_wait(bar, phase, abort_flag, kWaitLimitNs);
  phase ^= 1u;
  return ok;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Stream-K split of U units (one K block of one tile each, u = t * KB + kb) over P CTAs: CTA c
// owns units [sk_begin(c), sk_begin(c + 1)); with U >= P every CTA has at least one.  N * K < 2^40
// keeps the unit count below 2^26, so unit indices fit in 32 bits.
__device__ __forceinline__ int sk_begin(int c, int P, int U) {
  return static_cast<int>((static_cast<long long>(c) * U) / P);
}
__device__ __forceinline__ int sk_owner(int u, int P, int U) {
  return static_cast<int>(((static_cast<long long>(u) + 1) * P - 1) / U);
}
// Workspace slot of CTA c's piece of the tile whose first unit is tu0.
// Slot 2c holds the first segment of the CTA's range, slot 2c+1 its last (middle segments are
// whole tiles and never need a slot).
__device__ __forceinline__ int sk_slot(int c, int P, int U, int tu0) {
  return 2 * c + (sk_begin(c, P, U) >= tu0 ? 0 : 1);
}

// Work of one CTA of the tiled kernel.  Tiles [0, dp_end) are walked whole, CTA c taking tiles
// c, c + P, ...  When the last partial wave is split (the stream-K tail), its tiles dp_end ..
// form U = (tiles - dp_end) * KB units, spread over sk_ctas = min(U, P) CTAs so that every one of
// them has at least one unit; a tile split between CTAs is summed by the last of them to finish.
// The tail is taken only when its cost on the busiest CTA is at most the whole tile it replaces:
// its share of the units, plus `overhead` K blocks for publishing partial tiles, plus 2.4 K blocks
// for each piece the last CTA of a tile sums (the most pieces a tile can have).  overhead = 0
// takes the tail whenever the last wave is partial.
__device__ __host__ __forceinline__ bool tiled_tail_pays(int U, int ctas, int KB, int overhead) {
  const int per = (U + ctas - 1) / ctas;
  const int pieces = (KB + per - 1) / per + 1;
  return per + (overhead > 0 ? overhead + (12 * pieces + 4) / 5 : 0) <= KB;
}
struct TiledPlan {
  int dp_end;   // first tile of the stream-K tail (all tiles when there is none)
  int U;        // units of the tail
  int sk_ctas;  // CTAs sharing the tail
  int u_end;    // end of this CTA's unit range
};
struct TiledItem {
  int t;    // tile
  int kb0;  // K blocks [kb0, kb1) of it
  int kb1;
};
struct TiledCursor {
  int t;  // next whole tile
  int u;  // next unit of the tail
};

__device__ __forceinline__ TiledPlan tiled_plan(int num_tiles, int KB, int overhead, TiledCursor& cur) {
  const int P = gridDim.x;
  TiledPlan w;
  w.dp_end = num_tiles;
  w.U = 0;
  w.sk_ctas = 0;
  w.u_end = 0;
  cur.t = blockIdx.x;
  cur.u = 0;
  const int full = num_tiles / P;
  const int rem = num_tiles - full * P;
  if (overhead >= 0 && rem > 0) {
    const int U = rem * KB;
    const int ctas = U < P ? U : P;
    if (tiled_tail_pays(U, ctas, KB, overhead)) {
      w.dp_end = full * P;
      w.U = U;
      w.sk_ctas = ctas;
      if (static_cast<int>(blockIdx.x) < ctas) {
        cur.u = sk_begin(blockIdx.x, ctas, U);
        w.u_end = sk_begin(blockIdx.x + 1, ctas, U);
      }
    }
  }
  return w;
}

// Next work item of this CTA (whole tiles first, then its pieces of the tail); false when done.
__device__ __forceinline__ bool tiled_next(const TiledPlan& w, int KB, TiledCursor& cur, TiledItem& it) {
  if (cur.t < w.dp_end) {
    it.t = cur.t;
    it.kb0 = 0;
    it.kb1 = KB;
    cur.t += gridDim.x;
    return true;
  }
  if (cur.u < w.u_end) {
    const int tl = cur.u / KB;
    const int e = (w.u_end < (tl + 1) * KB) ? w.u_end : (tl + 1) * KB;
    it.t = w.dp_end + tl;
    it.kb0 = cur.u - tl * KB;
    it.kb1 = e - tl * KB;
    cur.u = e;
    return true;
  }
  return false;
}

// ============================================================================
// Kernel 1: tiled (dense / contiguous / masked)
// ============================================================================
struct TileInfo {
  int live;
  int g;       // group (0 for dense)
  int m0;      // first row of the tile within its row space (masked: within group g)
  int n0;
};

// Tile t of the walk -> (m-block, n-block).  The m-blocks (masked: the live ones) form groups of
// group_m; a group's tiles are consecutive, m-block fastest, so while a group is being worked on
// its A rows are re-read from L2 by every n-block rather than from DRAM.
__device__ __forceinline__ void tile_coords(int t, int mblocks, int n_blocks, int group_m, int& mb, int& nb) {
  const int per_group = group_m * n_blocks;
  const int mg = t / per_group;
  const int rem = t - mg * per_group;
  const int gm0 = mg * group_m;
  const int gm = (mblocks - gm0) < group_m ? (mblocks - gm0) : group_m;
  nb = rem / gm;
  mb = gm0 + (rem - nb * gm);
}

// ROWS: rows of an m-block (128, or 256 for the CTA-pair kernel); s_prefix counts such blocks.
template <int MODE, int ROWS = kBlockM>
__device__ __forceinline__ TileInfo tiled_tile(const TiledParams& p, const int* s_prefix, int live_mblocks, int t,
                                               int BN) {
  TileInfo ti;
  if (MODE == kMasked) {
    int lm, nb;
    tile_coords(t, live_mblocks, p.n_blocks, p.group_m, lm, nb);
    int lo = 0, hi = p.G;  // largest g with s_prefix[g] <= lm
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (s_prefix[mid] <= lm) lo = mid; else hi = mid;
    }
    ti.live = 1;
    ti.g = lo;
    ti.m0 = (lm - s_prefix[lo]) * ROWS;
    ti.n0 = nb * BN;
  } else {
    int mb, nb;
    tile_coords(t, p.m_blocks, p.n_blocks, p.group_m, mb, nb);
    ti.m0 = mb * ROWS;
    ti.n0 = nb * BN;
    if (MODE == kContiguous) {
      const int g = __ldg(p.m_indices + ti.m0);
      FG_DCHECK(g >= -1 && g < p.G, p.status);
      ti.live = (g >= 0 && g < p.G);
      ti.g = ti.live ? g : 0;
    } else {
      ti.live = 1;
      ti.g = 0;
    }
  }
  return ti;
}

// Scales of one chunk of kSaChunk K blocks of a 128-row tile as held in registers by one
// promotion thread: sfa for K block tid/32 and rows (tid%32)*4 .. +4, and (threads 0..15) one sfb
// value: 128-column block nb0 + tid/kSaChunk of the tile (a tile spans at most two), K block
// tid%kSaChunk.
struct ScaleChunkRegs {
  float4 a;
  float b;
};

template <int MODE>
__device__ __forceinline__ void load_scale_chunk(const TiledParams& p, const TileInfo& ti, int chunk, int tid,
                                                 ScaleChunkRegs& r) {
  r.a = make_float4(0.f, 0.f, 0.f, 0.f);
  r.b = 0.0f;
  if (tid >= kPromoWarps * 32) return;  // the first 256 promotion threads stage the scales
  const int kb = chunk * kSaChunk + (tid >> 5);
  const int r4 = (tid & 31) * 4;
  if (kb < p.num_kb) {
    const size_t g_sfa = (MODE == kMasked) ? static_cast<size_t>(ti.g) : 0;
    const float* sa = p.sfa + (g_sfa * p.num_kb + kb) * static_cast<size_t>(p.ld) + ti.m0 + r4;
    const int rows_left = p.M - (ti.m0 + r4);  // rows of the row space from this thread's first row on
    if (rows_left >= 4) {
      r.a = __ldg(reinterpret_cast<const float4*>(sa));
    } else {
      if (rows_left > 0) r.a.x = __ldg(sa);
      if (rows_left > 1) r.a.y = __ldg(sa + 1);
      if (rows_left > 2) r.a.z = __ldg(sa + 2);
    }
  }
  if (tid < 2 * kSaChunk) {
    const int kb2 = chunk * kSaChunk + tid % kSaChunk;
    const int nb = ti.n0 / kBlockK + tid / kSaChunk;
    if (kb2 < p.num_kb && nb < p.num_nb) {
      const size_t g_sfb = (MODE == kDense) ? 0 : static_cast<size_t>(ti.g);
      r.b = __ldg(p.sfb + (g_sfb * p.num_nb + nb) * p.num_kb + kb2);
    }
  }
}

// chunk layout in shared memory: sa[kSaChunk][128] floats, then sb[2][kSaChunk] floats
__device__ __forceinline__ void store_scale_chunk(float* buf, int tid, const ScaleChunkRegs& r) {
  if (tid >= kPromoWarps * 32) return;
  reinterpret_cast<float4*>(buf + (tid >> 5) * kBlockM + (tid & 31) * 4)[0] = r.a;
  if (tid < 2 * kSaChunk) buf[kSaChunk * kBlockM + tid] = r.b;
}

// One K block of promotion for one thread: the thread's 32 * NCH columns of the TMEM partial at
// taddr (its lane, consecutive columns) are read and added, times the block's scale -- s0, or s1
// for the 32-column chunks whose bit is set in hi_mask (the second 128-column sfb block) -- into
// the accumulator pairs acc[0 .. 16 NCH) with the packed FMA.  `release` (executed by the whole
// warp) hands the TMEM buffer back as soon as every chunk has landed in registers.
// PIPE = false: every chunk is loaded, one wait, then all are added (one load round trip per K
//   block; 32 NCH registers of slice).
// PIPE = 1: two 32-column chunks in flight at a time, chunk i+1 loading while chunk i is added
//   (64 registers of slice, so 128 x 256 tiles fit the register budget);
// PIPE = 2: the same with 16-column chunks (32 registers of slice);
// PIPE = 3: two rounds of half the slice each (load, wait, add), no overlap inside the warp but
//   only two load round trips per K block (NCH * 16 registers of slice).
template <int NCH, int PIPE, typename Release>
__device__ __forceinline__ void promote_kblock(uint32_t taddr, float2* acc, float s0, float s1, uint32_t hi_mask,
                                               Release&& release) {
  // add W columns (W/2 pairs) of chunk c (c in units of W columns) to the accumulators
  auto add = [&](const uint32_t* v, int c, int W) {
    const int i = c * W / 32;  // 32-column chunk: which sfb block
    const float sc = ((hi_mask >> i) & 1u) ? s1 : s0;
    const float2 s2 = make_float2(sc, sc);
#pragma unroll
    for (int j = 0; j < W / 2; ++j)
      acc[c * W / 2 + j] = __ffma2_rn(make_float2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1])), s2,
                                      acc[c * W / 2 + j]);
  };
  if constexpr (PIPE == 0) {
    uint32_t v[NCH][32];
#pragma unroll
    for (int i = 0; i < NCH; ++i) tmem_ld_32x32b_x32(taddr + 32 * i, v[i]);
    tmem_wait_ld();
    release();
#pragma unroll
    for (int i = 0; i < NCH; ++i) add(v[i], i, 32);
  } else if constexpr (PIPE == 3) {
    // two rounds of NCH/2 chunks: load, wait, add; the buffer is released after the second wait
    static_assert(NCH % 2 == 0, "PIPE 3 needs an even chunk count");
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      uint32_t v[NCH / 2][32];
#pragma unroll
      for (int i = 0; i < NCH / 2; ++i) tmem_ld_32x32b_x32(taddr + 32 * (r * NCH / 2 + i), v[i]);
      tmem_wait_ld();
      if (r == 1) release();
#pragma unroll
      for (int i = 0; i < NCH / 2; ++i) add(v[i], r * NCH / 2 + i, 32);
    }
  } else if constexpr (PIPE == 1) {
    uint32_t va[32], vb[32];
    tmem_ld_32x32b_x32(taddr, va);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      if (i + 1 < NCH) {
        tmem_ld_32x32b_x32(taddr + 32 * (i + 1), (i & 1) ? va : vb);
      } else {
        release();
      }
      add((i & 1) ? vb : va, i, 32);
      if (i + 1 < NCH) tmem_wait_ld();
    }
  } else {
    constexpr int N16 = 2 * NCH;
    uint32_t va[16], vb[16];
    tmem_ld_32x32b_x16(taddr, va);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < N16; ++i) {
      if (i + 1 < N16) {
        tmem_ld_32x32b_x16(taddr + 16 * (i + 1), (i & 1) ? va : vb);
      } else {
        release();
      }
      add((i & 1) ? vb : va, i, 16);
      if (i + 1 < N16) tmem_wait_ld();
    }
  }
}

// Output staging of one promotion warp: its 32 rows x COLS columns as COLS/32 boxes of 32 x 32
// bf16 (64-byte rows, 64-byte swizzle: the 16-byte chunk c of row r sits at chunk c ^ ((r/2)%4)),
// the layout the C tensor map stores from.
constexpr int kStoreBoxBytes = 32 * 64;

// Kernel 1 warp roles (384 threads, three warpgroups):
//   warpgroup 0 (warps 0-3) and 1 (warps 4-7): promotion + epilogue, column halves 0 and 1; each
//     raises its register budget (RegSplit) so a thread can hold the BN/2 fp32 accumulators of
//     its row and one whole BN/2-column slice loaded from TMEM;
//   warpgroup 2: warp 8 TMA producer, warp 9 TMEM owner + MMA issuer, warps 10-11 idle; it lowers
//     its budget.  The split assumes the kernel is launched with kTiledLaunchRegs
//     registers per thread, which the host checks before every launch.
// BN = 192 keeps one slice read (three 32-column TMEM loads) per K block within the register
// budget, so each TMEM buffer is handed back after a single load round trip; two buffers of 192
// columns fit the 512 TMEM columns.
template <int BN, int STAGES, int MODE, int PIPE = (BN > 192 ? FG_PIPE_256 : 0)>
__global__ void __launch_bounds__(kTiledThreads, 1)
    fp8_gemm_tiled_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                          const __grid_constant__ CUtensorMap tmC, const TiledParams p_in) {
#ifdef FG_JIT_NUM_KB
  // runtime-specialised build: the shape's K blocks, N, tile counts and tile-walk grouping are
  // compile-time constants (the compiler unrolls and folds the walk arithmetic for this shape)
  TiledParams p = p_in;
  p.num_kb = FG_JIT_NUM_KB;
  p.K = FG_JIT_K;
  p.N = FG_JIT_N;
  p.num_nb = FG_JIT_NUM_NB;
  p.n_blocks = FG_JIT_N_BLOCKS;
  p.group_m = FG_JIT_GROUP_M;
#else
  const TiledParams& p = p_in;
#endif
  constexpr int COLS = BN / 2;  // columns per promotion thread
  constexpr int NCH = COLS / 32;  // 32-column TMEM loads (and store boxes) per thread
  // tiles start at multiples of 64 columns, so no 32-column chunk straddles a 128-column sfb block
  static_assert(COLS % 32 == 0 && BN <= 256, "BN");
  constexpr int A_BYTES = kBlockM * kBlockK;
  constexpr int B_BYTES = BN * kBlockK;
  constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  constexpr int NUM_TBUF = 512 / BN;
  constexpr uint32_t TMEM_COLS = 512;
  constexpr int CHUNK_FLOATS = kSaChunk * kBlockM + 2 * kSaChunk;
  constexpr uint32_t IDESC = idesc_e4m3_f32(kBlockM, BN);
  constexpr int WARP_STORE_BYTES = NCH * kStoreBoxBytes;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_1024(smem_raw);
  uint8_t* s_out = smem + STAGES * STAGE_BYTES;                                    // [8 warps][NCH boxes]
  float* s_scale = reinterpret_cast<float*>(s_out + kPromoWarps * WARP_STORE_BYTES);  // [2][CHUNK_FLOATS]
  uint64_t* full = reinterpret_cast<uint64_t*>(s_scale + 2 * CHUNK_FLOATS);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + NUM_TBUF;
  uint64_t* mma_done = tempty + NUM_TBUF;
  uint64_t* pbar = mma_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pbar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* s_last = reinterpret_cast<volatile int*>(tmem_slot + 2);
  int* s_prefix = reinterpret_cast<int*>(tmem_slot + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (warp == kProducerWarp && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmC);
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int b = 0; b < NUM_TBUF; ++b) { mbar_init(&tfull[b], 1); mbar_init(&tempty[b], kPromoWarps); }
    mbar_init(mma_done, 1);
    mbar_init(pbar, kPromoWarps * 32);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) { tmem_alloc(tmem_slot, TMEM_COLS); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Everything above overlaps the previous kernel's tail; from here on global memory is touched.
  pdl_wait_prior_grid();
  pdl_launch_dependents();

  if (MODE == kMasked) {
    if (warp == 0) {
      // live 128-row blocks per group, exclusive prefix in s_prefix[0..G]
      int carry = 0;
      if (lane == 0) s_prefix[0] = 0;
      for (int base = 0; base < p.G; base += 32) {
        const int g = base + lane;
        int v = 0;
        if (g < p.G) {
          int cnt = __ldg(p.masked_m + g);
          cnt = cnt < 0 ? 0 : (cnt > p.M ? p.M : cnt);
          v = (cnt + kBlockM - 1) / kBlockM;
        }
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int u = __shfl_up_sync(0xffffffffu, v, o);
          if (lane >= o) v += u;
        }
        if (g < p.G) s_prefix[g + 1] = carry + v;
        carry += __shfl_sync(0xffffffffu, v, 31);
      }
    }
    __syncthreads();
  }

  int num_tiles, live_mblocks = 1;
  if (MODE == kMasked) {
    live_mblocks = s_prefix[p.G];
    num_tiles = live_mblocks * p.n_blocks;
  } else {
    num_tiles = p.m_blocks * p.n_blocks;
  }
  TiledCursor cur;
  const TiledPlan plan = tiled_plan(num_tiles, p.num_kb, p.sk_overhead, cur);
  TiledItem it;

  if (warp >= kPromoWarps) {
    // ================================================ warpgroup 2: producer, MMA, idle warps
    reg_dealloc<RegSplit<BN>::ctrl>();
    if (warp == kProducerWarp && lane == 0) {
      uint32_t stage = 0, phase = 0;
      uint32_t issued = 0;
      bool ok = true;
      // m-fastest groups: A rows are re-read by every n-block of a group, B tiles only by the
      // concurrent m-blocks; n fastest: the other way round
      const uint64_t pol_a = p.b_resident ? l2_policy_evict_first() : l2_policy_evict_last();
      const uint64_t pol_b = p.b_resident ? l2_policy_evict_last() : l2_policy_evict_first();
      while (ok && tiled_next(plan, p.num_kb, cur, it)) {
        const TileInfo ti = tiled_tile<MODE>(p, s_prefix, live_mblocks, it.t, BN);
        if (!ti.live) continue;
        const int ga = (MODE == kMasked) ? ti.g : 0;
        const int gb = (MODE == kDense) ? 0 : ti.g;
        FG_DCHECK(ti.m0 >= 0 && ti.m0 < p.M && ti.n0 >= 0 && ti.n0 < p.N && ti.g >= 0 && ti.g < p.G, p.status);
        FG_DCHECK(it.kb0 >= 0 && it.kb0 < it.kb1 && it.kb1 <= p.num_kb, p.status);
        for (int kb = it.kb0; kb < it.kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, kWaitLimitNs)) { ok = false; break; }
          uint8_t* st = smem + stage * STAGE_BYTES;
          mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
          tma_load_3d(st, &tmA, &full[stage], kb * kBlockK, ti.m0, ga, pol_a);
          tma_load_3d(st + A_BYTES, &tmB, &full[stage], kb * kBlockK, ti.n0, gb, pol_b);
          ++issued;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {  // drain this CTA's copies still in flight before the CTA exits
        const uint32_t first = issued > STAGES ? issued - STAGES : 0;
        for (uint32_t i = first; i < issued; ++i) mbar_drain(&full[i % STAGES], (i / STAGES) & 1u);
      }
    } else if (warp == kMmaWarp && lane == 0) {
      uint32_t stage = 0, phase = 0, tb = 0, tphase = 0;
      bool ok = true;
      while (ok && tiled_next(plan, p.num_kb, cur, it)) {
        const TileInfo ti = tiled_tile<MODE>(p, s_prefix, live_mblocks, it.t, BN);
        if (!ti.live) continue;
        for (int kb = it.kb0; kb < it.kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, kWaitLimitNs)) { ok = false; break; }
          if (!mbar_wait(&tempty[tb], tphase ^ 1u, abort_flag, kWaitLimitNs)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d = tmem_base + tb * BN;
          const uint32_t st = smem_addr(smem + stage * STAGE_BYTES);
          const uint64_t adesc = smem_desc_k128_sw128(st);
          const uint64_t bdesc = smem_desc_k128_sw128(st + A_BYTES);
#pragma unroll
          for (int j = 0; j < kBlockK / 32; ++j)  // 32 e4m3 = 32 bytes = 2 descriptor units per step
            mma_f8(d, adesc + 2 * j, bdesc + 2 * j, IDESC | p.fmt_bits, j > 0 ? 1u : 0u);
          mma_commit(&empty[stage]);
          mma_commit(&tfull[tb]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
          if (++tb == NUM_TBUF) { tb = 0; tphase ^= 1u; }
        }
      }
      // every MMA this thread issued has finished once mma_done flips
      mma_commit(mma_done);
      mbar_drain(mma_done, 0);
    }
  } else {
    // ================================================ warpgroups 0-1: promotion + epilogue
    reg_alloc<RegSplit<BN>::promo>();
    const int q = warp & 3;
    const int h = warp >> 2;
    const int row = q * 32 + lane;
    const int tid = threadIdx.x;  // 0..255 among promotion threads
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    uint8_t* s_w = s_out + warp * WARP_STORE_BYTES;  // this warp's output staging
    bool stores_pending = false;
    uint32_t tb = 0, tphase = 0, pphase = 0;
    bool ok = true;

    // next live work item of this CTA
    auto next_live = [&](TiledItem& item, TileInfo& info) -> bool {
      while (tiled_next(plan, p.num_kb, cur, item)) {
        info = tiled_tile<MODE>(p, s_prefix, live_mblocks, item.t, BN);
        if (info.live) return true;
      }
      return false;
    };
    TileInfo ti;
    bool have = next_live(it, ti);
    // Scale chunks (kSaChunk K blocks each) form one sequence over this CTA's work items; chunk X
    // of the sequence lives in s_scale[X % 2].  The registers hold the chunk after the one being
    // processed; it is stored into the other slot once this chunk is done, which is safe because
    // the barrier that ended the previous chunk guarantees that no thread still reads that slot.
    ScaleChunkRegs nxt;
    int buf = 0;
    if (have) {
      load_scale_chunk<MODE>(p, ti, it.kb0 / kSaChunk, tid, nxt);
      store_scale_chunk(s_scale, tid, nxt);
      ok = group_sync(pbar, pphase, abort_flag);
    }
    while (have && ok) {
      // the item after this one (for the chunk prefetch that crosses items)
      TiledItem it_next;
      TileInfo ti_next;
      const bool have_next = next_live(it_next, ti_next);
      const int m = ti.m0 + row;
      // sfb block (0: the tile's first, 1: the next) of each 32-column chunk of this thread
      uint32_t hi_mask = 0;
#pragma unroll
      for (int i = 0; i < NCH; ++i)
        hi_mask |= static_cast<uint32_t>((ti.n0 + h * COLS + 32 * i) / kBlockK - ti.n0 / kBlockK) << i;

      float2 acc[COLS / 2];  // column pairs: promoted with the packed fp32 FMA
#pragma unroll
      for (int j = 0; j < COLS / 2; ++j) acc[j] = make_float2(0.0f, 0.0f);

      const int c_lo = it.kb0 / kSaChunk;
      const int c_hi = (it.kb1 - 1) / kSaChunk;
      for (int c = c_lo; c <= c_hi && ok; ++c) {
        // prefetch the next chunk of the sequence into registers
        if (c < c_hi) load_scale_chunk<MODE>(p, ti, c + 1, tid, nxt);
        else if (have_next) load_scale_chunk<MODE>(p, ti_next, it_next.kb0 / kSaChunk, tid, nxt);
        const float* sa = s_scale + buf * CHUNK_FLOATS + row;
        const float* sb = s_scale + buf * CHUNK_FLOATS + kSaChunk * kBlockM;
        const int kb_begin = c * kSaChunk > it.kb0 ? c * kSaChunk : it.kb0;
        const int kb_end = (c + 1) * kSaChunk < it.kb1 ? (c + 1) * kSaChunk : it.kb1;
        for (int kb = kb_begin; kb < kb_end; ++kb) {
          const int kl = kb - c * kSaChunk;
          const float sav = sa[kl * kBlockM];
          const float s0 = sav * sb[kl];
          const float s1 = sav * sb[kSaChunk + kl];
          if (!mbar_wait(&tfull[tb], tphase, abort_flag, kWaitLimitNs)) { ok = false; break; }
          tc_fence_after();
          const uint32_t taddr = tmem_base + lane_off + tb * BN + h * COLS;
          // whole slice read: hand the TMEM buffer back to the MMA
          promote_kblock<NCH, PIPE>(taddr, acc, s0, s1, hi_mask, [&]() {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[tb]);
          });
          if (++tb == NUM_TBUF) { tb = 0; tphase ^= 1u; }
        }
        if (!ok) break;
        // publish the prefetched chunk into the other slot, then one barrier
        const int nbuf = buf ^ 1;
        if (c < c_hi || have_next) store_scale_chunk(s_scale + nbuf * CHUNK_FLOATS, tid, nxt);
        if (!group_sync(pbar, pphase, abort_flag)) { ok = false; break; }
        buf = nbuf;
      }
      if (!ok) break;

      if (it.kb0 != 0 || it.kb1 != p.num_kb) {
        // A piece of a split tile of the stream-K tail: publish the fp32 partial; the last CTA of
        // the tile to arrive sums every piece in CTA order (so results are bit-reproducible) and
        // writes the tile.  No CTA ever waits for another.  Thread tid's values sit at float4
        // positions i * 256 + tid of a partial, the same in every CTA.
        constexpr int TILE_F4 = kBlockM * BN / 4;
        const int tl = it.t - plan.dp_end;
        const int tu0 = tl * p.num_kb;
        const int c_first = sk_owner(tu0, plan.sk_ctas, plan.U);
        const int c_last = sk_owner(tu0 + p.num_kb - 1, plan.sk_ctas, plan.U);
        float4* ws4 = reinterpret_cast<float4*>(p.ws);
        FG_DCHECK(sk_slot(blockIdx.x, plan.sk_ctas, plan.U, tu0) < 2 * static_cast<int>(gridDim.x) &&
                      tl >= 0 && tl < p.counter_cap && c_first <= static_cast<int>(blockIdx.x) &&
                      static_cast<int>(blockIdx.x) <= c_last,
                  p.status);
        float4* wp = ws4 + static_cast<size_t>(sk_slot(blockIdx.x, plan.sk_ctas, plan.U, tu0)) * TILE_F4 + tid;
#pragma unroll
        for (int i = 0; i < COLS / 4; ++i)
          wp[i * kPromoWarps * 32] = make_float4(acc[2 * i].x, acc[2 * i].y, acc[2 * i + 1].x, acc[2 * i + 1].y);
        if (!group_sync(pbar, pphase, abort_flag)) { ok = false; break; }
        if (tid == 0) {
          fence_acq_rel_gpu();  // release this CTA's partial (ordered before by the barrier)
          const int prev = atomicAdd(p.counters + tl, 1);
          const int last = (prev == c_last - c_first);
          if (last) {
            fence_acq_rel_gpu();  // acquire the other CTAs' partials
            p.counters[tl] = 0;   // ready for the next launch
          }
          *s_last = last;
        }
        if (!group_sync(pbar, pphase, abort_flag)) { ok = false; break; }
        if (!*s_last) {
          it = it_next;
          ti = ti_next;
          have = have_next;
          continue;
        }
#pragma unroll
        for (int j = 0; j < COLS / 2; ++j) acc[j] = make_float2(0.0f, 0.0f);
        for (int c = c_first; c <= c_last; ++c) {
          const float4* src = ws4 + static_cast<size_t>(sk_slot(c, plan.sk_ctas, plan.U, tu0)) * TILE_F4 + tid;
#pragma unroll
          for (int i = 0; i < COLS / 4; ++i) {
            const float4 a = __ldcg(src + i * kPromoWarps * 32);
            acc[2 * i].x += a.x;
            acc[2 * i].y += a.y;
            acc[2 * i + 1].x += a.z;
            acc[2 * i + 1].y += a.w;
          }
        }
      }

      // epilogue: bf16 round-to-nearest-even.  A warp whose 32 rows are all to be written stages
      // them in shared memory and stores them with TMA; a warp with rows that must stay untouched
      // (past M, past masked_m, padding rows of another group) stores its valid rows directly.
      bool store_row = m < p.M;
      int cnt = p.M;
      if (MODE == kMasked) {
        cnt = __ldg(p.masked_m + ti.g);
        cnt = cnt > p.M ? p.M : cnt;
        store_row = m < cnt;
      } else if (MODE == kContiguous) {
        if (store_row) {
          const int gi = __ldg(p.m_indices + m);
          FG_DCHECK(gi >= -1 && gi < p.G, p.status);
          store_row = gi == ti.g;
        }
      }
      const int nbase = ti.n0 + h * COLS;
      if (__all_sync(0xffffffffu, store_row)) {
        if (stores_pending) {  // the previous tile's stores must have read the staging area
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
        }
        const uint32_t sw = static_cast<uint32_t>((lane >> 1) & 3);
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
          uint8_t* box_row = s_w + i * kStoreBoxBytes + lane * 64;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const float2* a = acc + 16 * i + 4 * c;
            uint4 val;
            val.x = pack_bf16x2(a[0].x, a[0].y);
            val.y = pack_bf16x2(a[1].x, a[1].y);
            val.z = pack_bf16x2(a[2].x, a[2].y);
            val.w = pack_bf16x2(a[3].x, a[3].y);
            *reinterpret_cast<uint4*>(box_row + ((c ^ sw) << 4)) = val;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const int y = ti.m0 + q * 32;
#pragma unroll
          for (int i = 0; i < NCH; ++i) {
            if (nbase + 32 * i < p.N) {
              if (MODE == kMasked) tma_store_3d(&tmC, s_w + i * kStoreBoxBytes, nbase + 32 * i, y, ti.g);
              else tma_store_2d(&tmC, s_w + i * kStoreBoxBytes, nbase + 32 * i, y);
            }
          }
          bulk_commit_group();
        }
        stores_pending = true;
      } else if (store_row) {
        __nv_bfloat16* crow = (MODE == kMasked) ? p.C + (static_cast<size_t>(ti.g) * p.M + m) * p.N
                                                : p.C + static_cast<size_t>(m) * p.N;
#pragma unroll
        for (int j = 0; j < COLS; j += 8) {
          if (nbase + j < p.N) {
            const float2* a = acc + j / 2;
            uint4 val;
            val.x = pack_bf16x2(a[0].x, a[0].y);
            val.y = pack_bf16x2(a[1].x, a[1].y);
            val.z = pack_bf16x2(a[2].x, a[2].y);
            val.w = pack_bf16x2(a[3].x, a[3].y);
            *reinterpret_cast<uint4*>(crow + nbase + j) = val;
          }
        }
      }
      it = it_next;
      ti = ti_next;
      have = have_next;
    }
    // the staging areas must outlive the stores' reads of them; the global writes complete
    // on their own before the grid completes
    if (stores_pending && lane == 0) bulk_wait_read_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
  if (threadIdx.x == 0 && *abort_flag) report_timeout(p.status);
}

// Thread shape of the CTA-pair kernel by promotion warpgroups PW: launch size, registers per
// thread at launch (the compiler's cap for that size), and the setmaxnreg split between the PW
// promotion warpgroups and the producer / MMA warpgroup.
template <int PW>
struct PairShape {
  static constexpr int threads = (PW + 1) * 128;
  static constexpr int launch_regs = PW == 2 ? kTiledLaunchRegs : 96;
  static constexpr int promo_regs = PW == 2 ? 232 : 112;
  static constexpr int ctrl_regs = PW == 2 ? 40 : 32;
  static_assert(PW * 128 * promo_regs + 128 * ctrl_regs <= threads * launch_regs, "register split");
};

// ============================================================================
// Kernel 3: CTA-pair tiled (dense M > 128, masked)
// ============================================================================
// The two CTAs of a cluster compute one 256 x BN output tile with tcgen05.mma.cta_group::2: CTA
// r loads A rows m0 + 128 r .. +127 and B rows n0 + r BN/2 .. +BN/2-1 of every K block into its
// own ring, the leader (rank 0) issues the pair MMAs (M = 256, N = BN), and the TMEM of CTA r
// holds rows m0 + 128 r .. +127 x BN columns, promoted and stored by CTA r as in kernel 1.  Each
// SM thus reads half of the B tile per K block instead of all of it.
// Barriers: full[s] of the leader counts the bytes of both CTAs (armed by the leader's producer);
// empty[s], tfull[b] and mma_done of both CTAs are arrived by the leader's multicast commits;
// tempty[b] of the leader counts the promotion warps of both CTAs.  Cluster barriers only right
// after set-up and right before teardown, which every thread of both CTAs reaches; every other
// wait is bounded.
// KPS: K blocks per ring stage.  KPS > 1 (K a multiple of 128) loads KPS consecutive K blocks of
// each operand with one 4-D copy over {128 bytes, rows, K blocks, groups}, laid out as KPS tiles
// one after the other (as KPS 3-D copies would), halving the copies per byte.
// PW: promotion warpgroups (2 or 4).  With 4, warpgroup h of the promotion warps owns columns
// [h BN/4, (h+1) BN/4) of the tile, so every SM sub-partition runs four promotion warps instead of
// two: twice the TMEM reads and FMAs in flight per K block, half the work per warp.
template <int BN, int STAGES, int MODE, int PIPE = (BN > 192 ? FG_PIPE_256 : 0), int KPS = 1, int PW = 2>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairShape<PW>::threads, 1)
    fp8_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                         const __grid_constant__ CUtensorMap tmC, const TiledParams p) {
  static_assert(MODE != kContiguous, "a pair tile needs both 128-row halves in one group");
  static_assert(PW == 2 || PW == 4, "PW");
  constexpr int NPW = 4 * PW;                  // promotion warps
  constexpr int PROD_WARP = NPW;               // TMA producer
  constexpr int MMA_WARP = NPW + 1;            // TMEM owner + MMA issuer
  constexpr int COLS = BN / PW;   // columns per promotion thread
  constexpr int NCH = COLS / 32;  // 32-column TMEM loads (and store boxes) per thread
  static_assert(COLS % 32 == 0 && BN <= 256, "BN");
  constexpr int PAIR_ROWS = 2 * kBlockM;
  constexpr int A_BYTES = kBlockM * kBlockK;   // one K block of this CTA's 128 rows of A
  constexpr int B_BYTES = (BN / 2) * kBlockK;  // one K block of this CTA's half of the B tile
  constexpr int STAGE_BYTES = KPS * (A_BYTES + B_BYTES);  // [KPS A tiles][KPS B tiles]
  constexpr int NUM_TBUF = 512 / BN;
  constexpr uint32_t TMEM_COLS = 512;
  constexpr int CHUNK_FLOATS = kSaChunk * kBlockM + 2 * kSaChunk;
  constexpr uint32_t IDESC = idesc_e4m3_f32(PAIR_ROWS, BN);
  constexpr int WARP_STORE_BYTES = NCH * kStoreBoxBytes;
  constexpr uint16_t kBoth = 0x3;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_1024(smem_raw);  // same offsets in both CTAs: the pair MMA relies on it
  uint8_t* s_out = smem + STAGES * STAGE_BYTES;
  float* s_scale = reinterpret_cast<float*>(s_out + NPW * WARP_STORE_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(s_scale + 2 * CHUNK_FLOATS);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + NUM_TBUF;
  uint64_t* mma_done = tempty + NUM_TBUF;
  uint64_t* pbar = mma_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pbar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_prefix = reinterpret_cast<int*>(tmem_slot + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = (rank == 0);
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int num_pairs = static_cast<int>(gridDim.x >> 1);

  if (warp == PROD_WARP && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmC);
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int b = 0; b < NUM_TBUF; ++b) { mbar_init(&tfull[b], 1); mbar_init(&tempty[b], 2 * NPW); }
    mbar_init(mma_done, 1);
    mbar_init(pbar, NPW * 32);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == MMA_WARP) { tmem_alloc_pair(tmem_slot, TMEM_COLS); tmem_relinquish_pair(); }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers are initialised before either CTA signals the other
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait_prior_grid();
  pdl_launch_dependents();

  if (MODE == kMasked) {
    if (warp == 0) {
      // live 256-row blocks per group, exclusive prefix in s_prefix[0..G]
      int carry = 0;
      if (lane == 0) s_prefix[0] = 0;
      for (int base = 0; base < p.G; base += 32) {
        const int g = base + lane;
        int v = 0;
        if (g < p.G) {
          int cnt = __ldg(p.masked_m + g);
          cnt = cnt < 0 ? 0 : (cnt > p.M ? p.M : cnt);
          v = (cnt + PAIR_ROWS - 1) / PAIR_ROWS;
        }
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int u = __shfl_up_sync(0xffffffffu, v, o);
          if (lane >= o) v += u;
        }
        if (g < p.G) s_prefix[g + 1] = carry + v;
        carry += __shfl_sync(0xffffffffu, v, 31);
      }
    }
    __syncthreads();
  }

  int num_tiles, live_blocks = 1;
  if (MODE == kMasked) {
    live_blocks = s_prefix[p.G];
    num_tiles = live_blocks * p.n_blocks;
  } else {
    num_tiles = p.m_blocks * p.n_blocks;  // m_blocks counts 256-row blocks here
  }

  if (warp >= NPW) {
    // ================================================ last warpgroup: producer, MMA, idle warps
    reg_dealloc<PairShape<PW>::ctrl_regs>();
    if (warp == PROD_WARP && lane == 0) {
      uint32_t stage = 0, phase = 0;
      uint32_t issued = 0;
      bool ok = true;
      const uint32_t full_leader = mapa_shared(smem_addr(full), 0);
      const uint64_t pol_a = p.b_resident ? l2_policy_evict_first() : l2_policy_evict_last();
      const uint64_t pol_b = p.b_resident ? l2_policy_evict_last() : l2_policy_evict_first();
      for (int t = pair; t < num_tiles && ok; t += num_pairs) {
        const TileInfo ti = tiled_tile<MODE, PAIR_ROWS>(p, s_prefix, live_blocks, t, BN);
        const int ga = (MODE == kMasked) ? ti.g : 0;
        const int gb = (MODE == kDense) ? 0 : ti.g;
        const int a_row = ti.m0 + static_cast<int>(rank) * kBlockM;
        const int b_row = ti.n0 + static_cast<int>(rank) * (BN / 2);
        FG_DCHECK(ti.m0 >= 0 && ti.m0 < p.M && ti.n0 >= 0 && ti.n0 < p.N && ti.g >= 0 && ti.g < p.G, p.status);
        for (int kb = 0; kb < p.num_kb; kb += KPS) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, kWaitLimitNs)) { ok = false; break; }
          uint8_t* st = smem + stage * STAGE_BYTES;
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * STAGE_BYTES);
          if constexpr (KPS == 1) {
            tma_load_3d_pair(st, &tmA, full_leader + stage * 8, kb * kBlockK, a_row, ga, pol_a);
            tma_load_3d_pair(st + A_BYTES, &tmB, full_leader + stage * 8, kb * kBlockK, b_row, gb, pol_b);
          } else {
            tma_load_4d_pair(st, &tmA, full_leader + stage * 8, 0, a_row, kb, ga, pol_a);
            tma_load_4d_pair(st + KPS * A_BYTES, &tmB, full_leader + stage * 8, 0, b_row, kb, gb, pol_b);
          }
          ++issued;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        // copies still in flight: the leader sees them complete on its own barriers; the peer's
        // land on the leader's barriers, so it gives them a fixed grace period instead
        if (leader) {
          const uint32_t first = issued > STAGES ? issued - STAGES : 0;
          for (uint32_t i = first; i < issued; ++i) mbar_drain(&full[i % STAGES], (i / STAGES) & 1u);
        } else {
          const uint64_t t0 = global_timer_ns();
          while (global_timer_ns() - t0 < 50000ull) {
          }
        }
      }
    } else if (warp == MMA_WARP && lane == 0) {
      if (leader) {
        uint32_t stage = 0, phase = 0, tb = 0, tphase = 0;
        bool ok = true;
        for (int t = pair; t < num_tiles && ok; t += num_pairs) {
          for (int kb = 0; kb < p.num_kb && ok; kb += KPS) {
            if (!mbar_wait(&full[stage], phase, abort_flag, kWaitLimitNs)) { ok = false; break; }
            const int nk = (p.num_kb - kb) < KPS ? (p.num_kb - kb) : KPS;
            for (int i = 0; i < nk; ++i) {
              if (!mbar_wait(&tempty[tb], tphase ^ 1u, abort_flag, kWaitLimitNs)) { ok = false; break; }
              tc_fence_after();
              const uint32_t d = tmem_base + tb * BN;
              const uint32_t st = smem_addr(smem + stage * STAGE_BYTES);
              const uint64_t adesc = smem_desc_k128_sw128(st + i * A_BYTES);
              const uint64_t bdesc = smem_desc_k128_sw128(st + KPS * A_BYTES + i * B_BYTES);
#pragma unroll
              for (int j = 0; j < kBlockK / 32; ++j)
                mma_f8_pair(d, adesc + 2 * j, bdesc + 2 * j, IDESC | p.fmt_bits, j > 0 ? 1u : 0u);
              if (i == nk - 1) mma_commit_pair(&empty[stage], kBoth);
              mma_commit_pair(&tfull[tb], kBoth);
              if (++tb == NUM_TBUF) { tb = 0; tphase ^= 1u; }
            }
            if (++stage == STAGES) { stage = 0; phase ^= 1u; }
          }
        }
        mma_commit_pair(mma_done, kBoth);  // arrives on both CTAs once every pair MMA has finished
      }
    }
  } else {
    // ================================================ warpgroups 0-1: promotion + epilogue
    reg_alloc<PairShape<PW>::promo_regs>();
    const int q = warp & 3;
    const int h = warp >> 2;
    const int row = q * 32 + lane;
    const int tid = threadIdx.x;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const int n_chunks = (p.num_kb + kSaChunk - 1) / kSaChunk;
    const uint32_t tempty_leader = mapa_shared(smem_addr(tempty), 0);
    uint8_t* s_w = s_out + warp * WARP_STORE_BYTES;
    bool stores_pending = false;
    uint32_t tb = 0, tphase = 0, pphase = 0;
    bool ok = true;

    // this CTA's half of the pair tile t
    auto my_tile = [&](int tt) {
      TileInfo ti = tiled_tile<MODE, PAIR_ROWS>(p, s_prefix, live_blocks, tt, BN);
      ti.m0 += static_cast<int>(rank) * kBlockM;
      return ti;
    };
    int t = pair;
    TileInfo ti;
    ti.live = 0;
    if (t < num_tiles) ti = my_tile(t);
    ScaleChunkRegs nxt;
    int buf = 0;
    if (t < num_tiles) {
      load_scale_chunk<MODE>(p, ti, 0, tid, nxt);
      store_scale_chunk(s_scale, tid, nxt);
      ok = group_sync(pbar, pphase, abort_flag);
    }
    while (t < num_tiles && ok) {
      const int t_next = t + num_pairs;
      TileInfo ti_next;
      ti_next.live = 0;
      if (t_next < num_tiles) ti_next = my_tile(t_next);
      const int m = ti.m0 + row;
      uint32_t hi_mask = 0;
#pragma unroll
      for (int i = 0; i < NCH; ++i)
        hi_mask |= static_cast<uint32_t>((ti.n0 + h * COLS + 32 * i) / kBlockK - ti.n0 / kBlockK) << i;

      float2 acc[COLS / 2];
#pragma unroll
      for (int j = 0; j < COLS / 2; ++j) acc[j] = make_float2(0.0f, 0.0f);

      for (int c = 0; c < n_chunks && ok; ++c) {
        if (c + 1 < n_chunks) load_scale_chunk<MODE>(p, ti, c + 1, tid, nxt);
        else if (t_next < num_tiles) load_scale_chunk<MODE>(p, ti_next, 0, tid, nxt);
        const float* sa = s_scale + buf * CHUNK_FLOATS + row;
        const float* sb = s_scale + buf * CHUNK_FLOATS + kSaChunk * kBlockM;
        const int kb_end = (c + 1) * kSaChunk < p.num_kb ? (c + 1) * kSaChunk : p.num_kb;
        for (int kb = c * kSaChunk; kb < kb_end; ++kb) {
          const int kl = kb - c * kSaChunk;
          const float sav = sa[kl * kBlockM];
          const float s0 = sav * sb[kl];
          const float s1 = sav * sb[kSaChunk + kl];
          if (!mbar_wait(&tfull[tb], tphase, abort_flag, kWaitLimitNs)) { ok = false; break; }
          tc_fence_after();
          const uint32_t taddr = tmem_base + lane_off + tb * BN + h * COLS;
          promote_kblock<NCH, PIPE>(taddr, acc, s0, s1, hi_mask, [&]() {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(tempty_leader + tb * 8);
          });
          if (++tb == NUM_TBUF) { tb = 0; tphase ^= 1u; }
        }
        if (!ok) break;
        const int nbuf = buf ^ 1;
        if (c + 1 < n_chunks || t_next < num_tiles) store_scale_chunk(s_scale + nbuf * CHUNK_FLOATS, tid, nxt);
        if (!group_sync(pbar, pphase, abort_flag)) { ok = false; break; }
        buf = nbuf;
      }
      if (!ok) break;

      // epilogue, as in kernel 1
      bool store_row = m < p.M;
      if (MODE == kMasked) {
        int cnt = __ldg(p.masked_m + ti.g);
        cnt = cnt > p.M ? p.M : cnt;
        store_row = m < cnt;
      }
      const int nbase = ti.n0 + h * COLS;
      if (__all_sync(0xffffffffu, store_row)) {
        if (stores_pending) {
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
        }
        const uint32_t sw = static_cast<uint32_t>((lane >> 1) & 3);
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
          uint8_t* box_row = s_w + i * kStoreBoxBytes + lane * 64;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const float2* a = acc + 16 * i + 4 * c;
            uint4 val;
            val.x = pack_bf16x2(a[0].x, a[0].y);
            val.y = pack_bf16x2(a[1].x, a[1].y);
            val.z = pack_bf16x2(a[2].x, a[2].y);
            val.w = pack_bf16x2(a[3].x, a[3].y);
            *reinterpret_cast<uint4*>(box_row + ((c ^ sw) << 4)) = val;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const int y = ti.m0 + q * 32;
#pragma unroll
          for (int i = 0; i < NCH; ++i) {
            if (nbase + 32 * i < p.N) {
              if (MODE == kMasked) tma_store_3d(&tmC, s_w + i * kStoreBoxBytes, nbase + 32 * i, y, ti.g);
              else tma_store_2d(&tmC, s_w + i * kStoreBoxBytes, nbase + 32 * i, y);
            }
          }
          bulk_commit_group();
        }
        stores_pending = true;
      } else if (store_row) {
        __nv_bfloat16* crow = (MODE == kMasked) ? p.C + (static_cast<size_t>(ti.g) * p.M + m) * p.N
                                                : p.C + static_cast<size_t>(m) * p.N;
#pragma unroll
        for (int j = 0; j < COLS; j += 8) {
          if (nbase + j < p.N) {
            const float2* a = acc + j / 2;
            uint4 val;
            val.x = pack_bf16x2(a[0].x, a[0].y);
            val.y = pack_bf16x2(a[1].x, a[1].y);
            val.z = pack_bf16x2(a[2].x, a[2].y);
            val.w = pack_bf16x2(a[3].x, a[3].y);
            *reinterpret_cast<uint4*>(crow + nbase + j) = val;
          }
        }
      }
      t = t_next;
      ti = ti_next;
    }
    // the staging areas must outlive the stores' reads of them; the global writes complete
    // on their own before the grid completes
    if (stores_pending && lane == 0) bulk_wait_read_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    // both CTAs: every pair MMA (which read this CTA's ring and wrote its TMEM) has finished; the
    // promotion above consumed every result, so this wait is short unless the CTA aborted
    if (lane == 0) {
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait_cluster(mma_done, 0)) {
        if (global_timer_ns() - t0 > kWaitLimitNs) { *abort_flag = 1; break; }
      }
    }
    __syncwarp();
  }
  cluster_sync_all();  // neither CTA touches the other's barriers, ring or TMEM any more
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
  if (threadIdx.x == 0 && *abort_flag) report_timeout(p.status);
}

// ============================================================================
// Kernel 2: swap-AB stream-K (dense, M <= MP <= 128)
// ============================================================================
// Units are (n-tile, K block) pairs split over the CTAs with sk_begin, or whole tiles per CTA
// (tile_aligned), or -- with cluster = S > 1 -- one tile per cluster of S CTAs, CTA r of the
// cluster taking K blocks [r KB / S, (r+1) KB / S): each CTA leaves its fp32 partial tile in its
// own shared memory, and after a cluster barrier CTA r sums rows [r 128/S, (r+1) 128/S) of the
// tile over the S partials (in rank order, so results are bit-reproducible) through distributed
// shared memory and writes them; a second cluster barrier keeps every CTA's shared memory alive
// until its peers have read it.  Every thread reaches both barriers, also after an abort.
// Cluster split-K reduction of the swap kernel: this CTA (rank `rank` of S) sums weight rows
// [rank 128/S, (rank+1) 128/S) of the tile over the S partials ([token][weight row] fp32 at shared
// address `part` in every CTA of the cluster), in rank order.  cluster_reduce_sum issues every
// distributed-shared-memory load of the thread (ITEMS float4 from each of the S CTAs) before the
// first sum, so that they take one round trip; cluster_reduce_write stores the sums as bf16.
template <int S, int MP>
struct ClusterReduce {
  static constexpr int R4 = kBlockM / S / 4;  // float4 per token row of this CTA's slice
  static constexpr int NPROMO = kPromoWarps * 32;
  static constexpr int ITEMS = (MP * R4 + NPROMO - 1) / NPROMO;
};

template <int S, int MP>
__device__ __forceinline__ void cluster_reduce_sum(const SwapParams& p, uint32_t part, int rank, int tid,
                                                   float4 (&r)[ClusterReduce<S, MP>::ITEMS]) {
  using CR = ClusterReduce<S, MP>;
  const int rows = p.M < MP ? p.M : MP;
  float4 v[CR::ITEMS][S];
#pragma unroll
  for (int it = 0; it < CR::ITEMS; ++it) {
    const int f = tid + it * CR::NPROMO;
    const int mm = f / CR::R4;
    const int col = rank * (kBlockM / S) + (f - mm * CR::R4) * 4;
    const uint32_t off = part + static_cast<uint32_t>((mm * kBlockM + col) * 4);
#pragma unroll
    for (int q = 0; q < S; ++q)
      v[it][q] = f < rows * CR::R4 ? ld_dsmem_f4(mapa_shared(off, static_cast<uint32_t>(q)))
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int it = 0; it < CR::ITEMS; ++it) {
    r[it] = v[it][0];
#pragma unroll
    for (int q = 1; q < S; ++q) {
      r[it].x += v[it][q].x; r[it].y += v[it][q].y; r[it].z += v[it][q].z; r[it].w += v[it][q].w;
    }
  }
}

template <int S, int MP>
__device__ __forceinline__ void cluster_reduce_write(const SwapParams& p, const float4 (&r)[ClusterReduce<S, MP>::ITEMS],
                                                     int rank, int n_base, int tid) {
  using CR = ClusterReduce<S, MP>;
  const int rows = p.M < MP ? p.M : MP;
#pragma unroll
  for (int it = 0; it < CR::ITEMS; ++it) {
    const int f = tid + it * CR::NPROMO;
    const int mm = f / CR::R4;
    const int col = rank * (kBlockM / S) + (f - mm * CR::R4) * 4;
    if (f < rows * CR::R4 && n_base + col < p.N) {  // N % 8 == 0, so the 4 columns are all inside
      uint2 val;
      val.x = pack_bf16x2(r[it].x, r[it].y);
      val.y = pack_bf16x2(r[it].z, r[it].w);
      *reinterpret_cast<uint2*>(p.C + static_cast<size_t>(mm) * p.N + n_base + col) = val;
    }
  }
}

// All threads of the CTA: sum this CTA's slice over the cluster (promotion warps, unless the
// kernel aborted), tell the cluster that this CTA has read its peers' shared memory, write the
// slice, and wait until every peer has read this CTA's shared memory before it may exit.
template <int S, int MP>
__device__ __forceinline__ void cluster_reduce_tail(const SwapParams& p, uint32_t part, int rank, int n_base,
                                                    bool reduce) {
  const int tid = threadIdx.x;
  float4 r[ClusterReduce<S, MP>::ITEMS];
  if (reduce) cluster_reduce_sum<S, MP>(p, part, rank, tid, r);
  __syncwarp();
  cluster_arrive_relaxed();
  if (reduce) cluster_reduce_write<S, MP>(p, r, rank, n_base, tid);
  __syncwarp();
  cluster_wait();
}

// KPS: K blocks per ring stage (and per unit of work).  KPS = 1 loads each K block's weight and
// token tiles with 2-D TMA copies; KPS > 1 (K a multiple of 128) loads KPS consecutive K blocks
// of each with one 3-D copy over the view {128 bytes, rows, K blocks} (strides K and 128 bytes),
// which lands as KPS tiles one after the other -- the layout KPS 2-D copies would give -- so a
// CTA streams its weights with half (a third, ...) of the copy operations: a CTA's copy rate is
// bounded by the number of copies in flight, not by their size, up to ~32 KB per copy.
template <int MP, int STAGES, int KPS = 1>
__global__ void __launch_bounds__(kThreads, 1)
    fp8_gemm_swap_streamk_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmT,
                                 const __grid_constant__ CUtensorMap tmC, const SwapParams p) {
  static_assert(MP == 32 || MP == 64 || MP == 128, "MP");
  static_assert(KPS == 1 || KPS == 2 || KPS == 4, "KPS");
  constexpr int W_BYTES = kBlockM * kBlockK;  // one K block of 128 weight rows
  constexpr int T_BYTES = MP * kBlockK;       // one K block of MP token rows
  constexpr int STAGE_BYTES = KPS * (W_BYTES + T_BYTES);  // [KPS weight tiles][KPS token tiles]
  constexpr int NUM_TBUF = MP <= 64 ? 8 : 4;  // TMEM buffers of MP columns (512 columns at most)
  constexpr uint32_t TMEM_COLS = (NUM_TBUF * MP) < 32 ? 32 : NUM_TBUF * MP;
  static_assert((2 * STAGES + 2 * NUM_TBUF + 2) * 8 + 3 * 4 <= kSwapBarrierBytes, "swap kernel barrier region");
  constexpr int COLS = MP / 2;                // token columns per promotion thread
  constexpr int NPROMO = kPromoWarps * 32;
  constexpr int SCALE_SLOTS = kSwapScaleBytes / (4 * MP);  // K blocks whose scales fit in shared memory
  constexpr int SCALE_CAP = SCALE_SLOTS / KPS;              // units whose scales fit
  constexpr int F4 = MP * kBlockM / 4 / NPROMO;          // float4 of a partial tile per thread
  constexpr int PPR = (16 / F4) < 1 ? 1 : 16 / F4;       // partials read per round in the fix-up
  constexpr int RING_SLOTS = (STAGES * STAGE_BYTES) / (MP * kBlockM * 4);  // partials the idle ring holds
  static_assert(RING_SLOTS >= 2, "ring slots");
  constexpr uint32_t IDESC = idesc_e4m3_f32(kBlockM, MP);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_1024(smem_raw);
  __nv_bfloat16* s_c = reinterpret_cast<__nv_bfloat16*>(smem + STAGES * STAGE_BYTES);  // [MP][128]
  float* s_scale = reinterpret_cast<float*>(s_c + MP * kBlockM);                        // [SCALE_SLOTS][MP]
  uint64_t* full = reinterpret_cast<uint64_t*>(s_scale + SCALE_SLOTS * MP);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + NUM_TBUF;
  uint64_t* mma_done = tempty + NUM_TBUF;
  uint64_t* pbar = mma_done + 1;  // promotion-group barrier
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pbar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* s_last = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int P = gridDim.x;
  const int NKB = p.num_kb;                 // K blocks
  const int KB = (NKB + KPS - 1) / KPS;     // units (groups of KPS K blocks) per tile
  const int U = p.n_tiles * KB;
  // unit range: stream-K (even split of the units, tiles split between CTAs) or, when the host
  // finds whole tiles cheaper, tile-aligned (an even split of the tiles; no tile is split)
  const int S = p.cluster;
  const int cl_tile = static_cast<int>(blockIdx.x) / S;
  const int cl_rank = static_cast<int>(blockIdx.x) - cl_tile * S;  // = %cluster_ctarank for cluster dims (S,1,1)
  const int u_begin = S > 1 ? cl_tile * KB + cl_rank * KB / S
                      : p.tile_aligned
                          ? static_cast<int>(static_cast<long long>(blockIdx.x) * p.n_tiles / P) * KB
                          : sk_begin(blockIdx.x, P, U);
  const int u_end = S > 1 ? cl_tile * KB + (cl_rank + 1) * KB / S
                    : p.tile_aligned
                        ? static_cast<int>(static_cast<long long>(blockIdx.x + 1) * p.n_tiles / P) * KB
                        : sk_begin(blockIdx.x + 1, P, U);
  // K blocks of unit u (the last unit of a tile may hold fewer than KPS)
  auto unit_kblocks = [&](int u) {
    const int kb0 = (u - (u / KB) * KB) * KPS;
    return (NKB - kb0) < KPS ? (NKB - kb0) : KPS;
  };

  const uint64_t pol_w = l2_policy_evict_first();  // each weight byte is read once
  const uint64_t pol_t = l2_policy_evict_last();   // tokens are re-read by every CTA
  // Producer state: next unit to load, smem ring position, loads issued.
  int p_u = u_begin;
  uint32_t p_stage = 0, p_phase = 0;
  uint32_t p_issued = 0;
  // weight / token copies of unit u into stage `st` (a K-block group: first K block kb)
  auto load_w = [&](int u, int st) {
    const int t = u / KB;
    const int kb = (u - t * KB) * KPS;
    FG_DCHECK(t >= 0 && t < p.n_tiles && t * kBlockM < p.N && kb * kBlockK < p.K, p.status);
    if constexpr (KPS == 1) tma_load_2d(smem + st * STAGE_BYTES, &tmW, &full[st], kb * kBlockK, t * kBlockM, pol_w);
    else tma_load_3d(smem + st * STAGE_BYTES, &tmW, &full[st], 0, t * kBlockM, kb, pol_w);
  };
  auto load_t = [&](int u, int st) {
    const int kb = (u - (u / KB) * KB) * KPS;
    if constexpr (KPS == 1) tma_load_2d(smem + st * STAGE_BYTES + W_BYTES, &tmT, &full[st], kb * kBlockK, 0, pol_t);
    else tma_load_3d(smem + st * STAGE_BYTES + KPS * W_BYTES, &tmT, &full[st], 0, 0, kb, pol_t);
  };
  auto issue = [&](int u) {
    mbar_arrive_expect_tx(&full[p_stage], STAGE_BYTES);  // whole boxes, also where they pass K
    load_w(u, p_stage);
    load_t(u, p_stage);
    ++p_issued;
    if (++p_stage == STAGES) { p_stage = 0; p_phase ^= 1u; }
  };

  if (warp == kProducerWarp && lane == 0) {
    prefetch_tmap(&tmW);
    prefetch_tmap(&tmT);
    prefetch_tmap(&tmC);
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int b = 0; b < NUM_TBUF; ++b) { mbar_init(&tfull[b], 1); mbar_init(&tempty[b], kPromoWarps); }
    mbar_init(mma_done, 1);
    mbar_init(pbar, NPROMO);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) { tmem_alloc(tmem_slot, TMEM_COLS); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Weights that the preceding kernel does not write (static_b) start streaming before the wait
  // for it: the weight half of each of the first ring stages (the token half, which that kernel
  // may produce, follows the wait).  Each stage's barrier is armed for the whole stage at once.
  int pre = 0;
  if (p.static_b && warp == kProducerWarp && lane == 0) {
    pre = (u_end - u_begin) < STAGES ? (u_end - u_begin) : STAGES;
    for (int s = 0; s < pre; ++s) {
      mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
      load_w(u_begin + s, s);
    }
  }
  // Everything above overlaps the previous kernel's tail; from here on global memory is touched
  // (apart from the weight loads above).
  pdl_wait_prior_grid();
  pdl_launch_dependents();

  if (warp == kProducerWarp) {
    if (lane == 0) {
      bool ok = true;
      for (int s = 0; s < pre; ++s) load_t(u_begin + s, s);  // token halves of the early stages
      p_issued = static_cast<uint32_t>(pre);
      p_u = u_begin + pre;
      p_stage = static_cast<uint32_t>(pre % STAGES);
      p_phase = pre == STAGES ? 1u : 0u;
      for (; p_u < u_end; ++p_u) {
        if (!mbar_wait(&empty[p_stage], p_phase ^ 1u, abort_flag, kWaitLimitNs)) { ok = false; break; }
        issue(p_u);
      }
      if (!ok) {
        const uint32_t first = p_issued > STAGES ? p_issued - STAGES : 0;
        for (uint32_t i = first; i < p_issued; ++i) mbar_drain(&full[i % STAGES], (i / STAGES) & 1u);
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      uint32_t stage = 0, phase = 0, tb = 0, tphase = 0;
      // Failure-injection hook for tests: mma_done completes its first phase only with the commit
      // below, so this bounded wait runs out, raises the abort flag and exercises the abort path.
      if (p.debug_stall) mbar_wait(mma_done, 0, abort_flag, kWaitLimitNs);
      bool ok = true;
      for (int u = u_begin; u < u_end && ok; ++u) {
        const int nk = unit_kblocks(u);
        const uint32_t sw = smem_addr(smem + stage * STAGE_BYTES);
        if (KPS == 2 && nk == 2) {
          // one TMEM partial per K block; the two K blocks' MMAs are issued interleaved (K step j
          // of both, then step j + 1), so that their chains of dependent MMAs -- each accumulating
          // into its own buffer -- overlap in the tensor pipe instead of running one after the
          // other (a decode step 5% faster at M = 64 than with the chains issued in turn).  The
          // TMEM buffers are claimed and the descriptors formed before the wait for the data, so
          // that only the MMAs follow its arrival.
          const uint32_t tb1 = tb + 1 == NUM_TBUF ? 0u : tb + 1;
          const uint32_t tph1 = tb + 1 == NUM_TBUF ? (tphase ^ 1u) : tphase;
          if (!mbar_wait(&tempty[tb], tphase ^ 1u, abort_flag, kWaitLimitNs)) break;
          if (!mbar_wait(&tempty[tb1], tph1 ^ 1u, abort_flag, kWaitLimitNs)) break;
          const uint32_t d0 = tmem_base + tb * MP, d1 = tmem_base + tb1 * MP;
          const uint64_t a0 = smem_desc_k128_sw128(sw), a1 = smem_desc_k128_sw128(sw + W_BYTES);
          const uint64_t b0 = smem_desc_k128_sw128(sw + KPS * W_BYTES);
          const uint64_t b1 = smem_desc_k128_sw128(sw + KPS * W_BYTES + T_BYTES);
          if (!mbar_wait(&full[stage], phase, abort_flag, kWaitLimitNs)) break;
          tc_fence_after();
#pragma unroll
          for (int j = 0; j < kBlockK / 32; ++j) {
            mma_f8(d0, a0 + 2 * j, b0 + 2 * j, IDESC | p.fmt_bits, j > 0 ? 1u : 0u);
            mma_f8(d1, a1 + 2 * j, b1 + 2 * j, IDESC | p.fmt_bits, j > 0 ? 1u : 0u);
          }
          mma_commit(&empty[stage]);
          mma_commit(&tfull[tb]);
          mma_commit(&tfull[tb1]);
          if (tb1 + 1 == NUM_TBUF || tb1 == 0) tphase ^= 1u;
          tb = tb1 + 1 == NUM_TBUF ? 0u : tb1 + 1;
        } else {
          if (!mbar_wait(&full[stage], phase, abort_flag, kWaitLimitNs)) break;
          for (int i = 0; i < nk; ++i) {  // one TMEM partial per K block
            if (!mbar_wait(&tempty[tb], tphase ^ 1u, abort_flag, kWaitLimitNs)) { ok = false; break; }
            tc_fence_after();
            const uint32_t d = tmem_base + tb * MP;
            const uint64_t adesc = smem_desc_k128_sw128(sw + i * W_BYTES);
            const uint64_t bdesc = smem_desc_k128_sw128(sw + KPS * W_BYTES + i * T_BYTES);
#pragma unroll
            for (int j = 0; j < kBlockK / 32; ++j)
              mma_f8(d, adesc + 2 * j, bdesc + 2 * j, IDESC | p.fmt_bits, j > 0 ? 1u : 0u);
            if (i == nk - 1) mma_commit(&empty[stage]);
            mma_commit(&tfull[tb]);
            if (++tb == NUM_TBUF) { tb = 0; tphase ^= 1u; }
          }
        }
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      mma_commit(mma_done);
      mbar_drain(mma_done, 0);
    }
  } else {
    // ------------------------------------------------ promotion + fix-up + epilogue
    const int q = warp & 3;
    const int h = warp >> 2;
    const int nl = q * 32 + lane;   // weight row within the n-tile (TMEM lane)
    const int tid = threadIdx.x;    // 0..255 among promotion threads
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    uint32_t tb = 0, tphase = 0, pphase = 0;
    bool ok = true;
    bool first_segment = true;
    int chunk_base = u_begin, chunk_end = u_begin;  // units whose scales are staged

    // bf16 tile from registers (thread = weight row nl, columns = tokens) -> C[m, t*128 + nl]:
    // transposed into the [token][weight row] staging tile, which one TMA store writes to C (rows
    // past M and columns past N clipped by the tensor map).  The store runs on while the warps go on
    // to the next tile; the staging tile is rewritten only after the store has read it.
    bool store_pending = false;
    auto store_tile = [&](const float* vals, int n_base) -> bool {
      if (store_pending) {
        if (tid == 0) bulk_wait_read_all();
        if (!group_sync(pbar, pphase, abort_flag)) return false;
      }
#pragma unroll
      for (int j = 0; j < COLS; ++j) s_c[(h * COLS + j) * kBlockM + nl] = __float2bfloat16_rn(vals[j]);
      fence_proxy_async_smem();
      if (!group_sync(pbar, pphase, abort_flag)) return false;
      if (tid == 0) {
        tma_store_2d(&tmC, s_c, n_base, 0);
        bulk_commit_group();
      }
      store_pending = true;
      return true;
    };

    for (int u = u_begin; u < u_end && ok;) {
      const int t = u / KB;
      const int tu0 = t * KB;
      const int kb0 = u - tu0;
      const int kb1 = (u_end < tu0 + KB ? u_end : tu0 + KB) - tu0;

      float acc[COLS];
#pragma unroll
      for (int j = 0; j < COLS; ++j) acc[j] = 0.0f;

      for (int kb = kb0; kb < kb1 && ok; ++kb) {
        const int uu = tu0 + kb;  // unit (group of KPS K blocks)
        if (uu >= chunk_end) {
          // combined scales sfa[k][m] * sfb[t][k] of the K blocks of the next SCALE_CAP units (zero
          // past M and past the last K block); slot sl = KPS * (unit - chunk_base) + i holds K
          // block i of the unit.  Thread tid owns column tid % MP of slots tid / MP + r * (256 /
          // MP), and every load of the chunk is issued before the first product is formed
          if (!group_sync(pbar, pphase, abort_flag)) { ok = false; break; }
          chunk_base = uu;
          chunk_end = (u_end < uu + SCALE_CAP) ? u_end : uu + SCALE_CAP;
          constexpr int STEP = NPROMO / MP;  // slots per pass of all threads
          constexpr int ITER = SCALE_SLOTS / STEP;
          const int mm = tid % MP;
          float a[ITER], b[ITER];
          // each slot's (tile, K block) is computed on its own, so that no load waits for an index
          // chain: all of a thread's scale loads are in flight together
#pragma unroll
          for (int r = 0; r < ITER; ++r) {
            a[r] = 0.0f;
            b[r] = 0.0f;
            const int sl = tid / MP + r * STEP;
            const int v = chunk_base + sl / KPS;
            if (v < chunk_end) {
              const int vt = v / KB;
              const int vkb = (v - vt * KB) * KPS + sl % KPS;
              if (vkb < NKB) {
                if (mm < p.M) a[r] = __ldg(p.sfa + static_cast<size_t>(vkb) * p.ld + mm);
                b[r] = __ldg(p.sfb + static_cast<size_t>(vt) * NKB + vkb);
              }
            }
          }
#pragma unroll
          for (int r = 0; r < ITER; ++r) s_scale[(tid / MP + r * STEP) * MP + mm] = a[r] * b[r];
          if (!group_sync(pbar, pphase, abort_flag)) { ok = false; break; }
        }
        const int nk = unit_kblocks(uu);
        for (int i = 0; i < nk; ++i) {
          if (!mbar_wait(&tfull[tb], tphase, abort_flag, kWaitLimitNs)) { ok = false; break; }
          tc_fence_after();
          const uint32_t taddr = tmem_base + lane_off + tb * MP + h * COLS;
          uint32_t v[COLS];
          if constexpr (COLS == 16) {
            uint32_t (&r16)[16] = *reinterpret_cast<uint32_t(*)[16]>(v);
            tmem_ld_32x32b_x16(taddr, r16);
          } else {
#pragma unroll
            for (int c0 = 0; c0 < COLS; c0 += 32) {
              uint32_t (&r32)[32] = *reinterpret_cast<uint32_t(*)[32]>(v + c0);
              tmem_ld_32x32b_x32(taddr + c0, r32);
            }
          }
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[tb]);
          const float4* sc4 =
              reinterpret_cast<const float4*>(s_scale + ((uu - chunk_base) * KPS + i) * MP + h * COLS);
#pragma unroll
          for (int j = 0; j < COLS; j += 4) {
            const float4 s4 = sc4[j / 4];
            acc[j + 0] = fmaf(__uint_as_float(v[j + 0]), s4.x, acc[j + 0]);
            acc[j + 1] = fmaf(__uint_as_float(v[j + 1]), s4.y, acc[j + 1]);
            acc[j + 2] = fmaf(__uint_as_float(v[j + 2]), s4.z, acc[j + 2]);
            acc[j + 3] = fmaf(__uint_as_float(v[j + 3]), s4.w, acc[j + 3]);
          }
          if (++tb == NUM_TBUF) { tb = 0; tphase ^= 1u; }
        }
      }
      if (!ok) break;

      const int n_base = t * kBlockM;
      if (kb0 == 0 && kb1 == KB) {  // whole tile
        if (!store_tile(acc, n_base)) { ok = false; break; }
      } else if (S > 1) {
        // the cluster's piece of its tile: the fp32 partial goes into this CTA's idle ring
        // ([token][weight row]; every load has landed and every MMA that read the ring is done)
        fence_proxy_async_smem();
        float* part = reinterpret_cast<float*>(smem);
#pragma unroll
        for (int j = 0; j < COLS; ++j) part[(h * COLS + j) * kBlockM + nl] = acc[j];
      } else {
        // split tile: the CTAs of the tile publish their fp32 partials; the last to arrive
        // (counter per tile) sums them in CTA order -- so results are bit-reproducible -- and
        // writes the bf16 tile.  No CTA ever waits for another.
        const int c_first = sk_owner(tu0, P, U);
        const int c_last = sk_owner(tu0 + KB - 1, P, U);
        const int slot = 2 * blockIdx.x + (first_segment ? 0 : 1);
        FG_DCHECK(t < p.counter_cap && c_first <= static_cast<int>(blockIdx.x) &&
                      static_cast<int>(blockIdx.x) <= c_last && c_first >= 0 && c_last < P,
                  p.status);
        // workspace slot of piece c: the tile's first CTA may hold it as the last segment of its
        // range (slot 2c+1); every later CTA holds it as its first segment (slot 2c)
        const int first_slot = sk_slot(c_first, P, U, tu0);
        auto piece_slot = [&](int c) { return c == c_first ? first_slot : 2 * c; };
        if (tu0 + kb1 >= u_end) {
          // The CTA's last segment usually ends after the tile's other pieces, which their CTAs
          // published early in their ranges: when the counter already holds all of them, this CTA
          // is the last to arrive and sums the pieces without publishing its own (its ring is idle
          // and holds its piece for the sum).  The sum runs in CTA order from zero, as on the
          // other path, so the result is the same bits.
          if (tid == 0) {
            const int last = ld_relaxed_gpu(p.counters + t) == c_last - c_first;
            if (last) {
              fence_acq_rel_gpu();  // acquire the other CTAs' partials
              p.counters[t] = 0;    // ready for the next launch
            }
            *s_last = last;
          }
          if (!group_sync(pbar, pphase, abort_flag)) { ok = false; break; }
          if (*s_last) {
            fence_proxy_async_smem();
            float* own = reinterpret_cast<float*>(smem) + nl;
#pragma unroll
            for (int j = 0; j < COLS; ++j) own[(h * COLS + j) * kBlockM] = acc[j];
            constexpr int PR = 1;  // pieces loaded per round (more spill registers)
            float r[COLS];
#pragma unroll
            for (int j = 0; j < COLS; ++j) r[j] = 0.0f;
#pragma unroll 1
            for (int c0 = c_first; c0 <= c_last; c0 += PR) {
              float v[PR][COLS];
#pragma unroll
              for (int k = 0; k < PR; ++k) {
                const int c = c0 + k;
                if (c == static_cast<int>(blockIdx.x)) {  // this CTA's piece, from shared memory
#pragma unroll
                  for (int j = 0; j < COLS; ++j) v[k][j] = own[(h * COLS + j) * kBlockM];
                } else if (c <= c_last) {
                  const float* src = p.ws + static_cast<size_t>(piece_slot(c)) * MP * kBlockM + nl;
#pragma unroll
                  for (int j = 0; j < COLS; ++j) v[k][j] = __ldcg(src + (h * COLS + j) * kBlockM);
                }
              }
#pragma unroll
              for (int k = 0; k < PR; ++k) {
                if (c0 + k <= c_last) {
#pragma unroll
                  for (int j = 0; j < COLS; ++j) r[j] += v[k][j];
                }
              }
            }
            if (!store_tile(r, n_base)) { ok = false; break; }
            first_segment = false;
            u = tu0 + kb1;
            continue;
          }
        }
        float* wp = p.ws + static_cast<size_t>(slot) * MP * kBlockM + nl;
#pragma unroll
        for (int j = 0; j < COLS; ++j) wp[static_cast<size_t>(h * COLS + j) * kBlockM] = acc[j];
        if (!group_sync(pbar, pphase, abort_flag)) { ok = false; break; }
        if (tid == 0) {
          fence_acq_rel_gpu();  // release the CTA's partial (ordered before by the barrier)
          const int prev = atomicAdd(p.counters + t, 1);
          const int last = (prev == c_last - c_first);
          if (last) {
            fence_acq_rel_gpu();  // acquire the other CTAs' partials
            p.counters[t] = 0;    // ready for the next launch
          }
          *s_last = last;
        }
        if (!group_sync(pbar, pphase, abort_flag)) { ok = false; break; }
        if (*s_last) {
          const float4* ws4 = reinterpret_cast<const float4*>(p.ws);
          float4 r[F4];
#pragma unroll
          for (int i = 0; i < F4; ++i) r[i] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (tu0 + kb1 >= u_end) {
            // The CTA's last segment: its ring is idle (every load consumed, every MMA done), so
            // the partials are pulled into it with cp.async, RING_SLOTS partials in flight, each
            // thread copying and reading back only its own float4 positions.  Summation order
            // is still c_first .. c_last.
            float4* ring4 = reinterpret_cast<float4*>(smem);
            const int npieces = c_last - c_first + 1;
#pragma unroll 1
            for (int k = 0; k < RING_SLOTS; ++k) {
              if (k < npieces) {
                const float4* src = ws4 + static_cast<size_t>(piece_slot(c_first + k)) * (MP * kBlockM / 4) + tid;
                float4* dst = ring4 + k * F4 * NPROMO + tid;
#pragma unroll
                for (int i = 0; i < F4; ++i) cp_async_16(dst + i * NPROMO, src + i * NPROMO);
              }
              cp_async_commit();
            }
#pragma unroll 1
            for (int k = 0; k < npieces; ++k) {
              cp_async_wait<RING_SLOTS - 1>();  // piece k has landed
              float4* slot = ring4 + (k % RING_SLOTS) * F4 * NPROMO + tid;
#pragma unroll
              for (int i = 0; i < F4; ++i) {
                const float4 a = slot[i * NPROMO];
                r[i].x += a.x; r[i].y += a.y; r[i].z += a.z; r[i].w += a.w;
              }
              if (k + RING_SLOTS < npieces) {
                const float4* src =
                    ws4 + static_cast<size_t>(piece_slot(c_first + k + RING_SLOTS)) * (MP * kBlockM / 4) + tid;
#pragma unroll
                for (int i = 0; i < F4; ++i) cp_async_16(slot + i * NPROMO, src + i * NPROMO);
              }
              cp_async_commit();
            }
          } else
          for (int c0 = c_first; c0 <= c_last; c0 += PPR) {
            float4 a[PPR][F4];
#pragma unroll
            for (int k = 0; k < PPR; ++k) {
              if (c0 + k <= c_last) {
                const float4* src = ws4 + static_cast<size_t>(piece_slot(c0 + k)) * (MP * kBlockM / 4) + tid;
#pragma unroll
                for (int i = 0; i < F4; ++i) a[k][i] = __ldcg(src + i * NPROMO);
              }
            }
#pragma unroll
            for (int k = 0; k < PPR; ++k) {
              if (c0 + k <= c_last) {
#pragma unroll
                for (int i = 0; i < F4; ++i) {
                  r[i].x += a[k][i].x; r[i].y += a[k][i].y; r[i].z += a[k][i].z; r[i].w += a[k][i].w;
                }
              }
            }
          }
#pragma unroll
          for (int i = 0; i < F4; ++i) {
            const int f = tid + i * NPROMO;  // float4 index in the [MP][128] tile
            const int mm = f >> 5;
            const int n = n_base + (f & 31) * 4;
            if (mm < p.M && n < p.N) {
              uint2 val;
              val.x = pack_bf16x2(r[i].x, r[i].y);
              val.y = pack_bf16x2(r[i].z, r[i].w);
              *reinterpret_cast<uint2*>(p.C + static_cast<size_t>(mm) * p.N + n) = val;
            }
          }
        }
      }
      first_segment = false;
      u = tu0 + kb1;
    }
    // the staging tile must outlive the last store's read of it; the global writes complete on
    // their own before the grid completes
    if (store_pending && tid == 0) bulk_wait_read_all();
  }

  if (S > 1) {
    // cluster split-K: sum rows [cl_rank R, (cl_rank + 1) R) of the tile over the S partials
    __syncwarp();
    cluster_sync_all();  // every CTA's partial is in its shared memory
    const bool reduce = warp < kPromoWarps && !*abort_flag;
    const uint32_t part = smem_addr(smem);
    const int n_base = cl_tile * kBlockM;
    if (S == 2) cluster_reduce_tail<2, MP>(p, part, cl_rank, n_base, reduce);
    else if (S == 4) cluster_reduce_tail<4, MP>(p, part, cl_rank, n_base, reduce);
    else cluster_reduce_tail<8, MP>(p, part, cl_rank, n_base, reduce);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
  if (threadIdx.x == 0 && *abort_flag) report_timeout(p.status);
}

}  // namespace fg
