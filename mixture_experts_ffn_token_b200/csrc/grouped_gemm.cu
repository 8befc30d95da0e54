// grouped_gemm.cu -- stages 3 and 4: the two grouped contractions over
// stacked expert weights on the 5th-generation tensor cores.
//
//   gate_up:  h[p, :] = act(split(Xp[p, :] . W_gu[e] + b_gu[e]))   for p in
//             expert e's segment [off[e], off[e+1]) of the permuted rows
//             (StackedMoE gate_up_proj [E, H, 2D]; GatedActivation fused
//             activations; concatenated or interleaved gate/up columns).
//   down:     Y[perm[p], :] = w[perm[p]] * (h[p, :] . W_d[e] + b_d[e])
//             (StackedMoE down_proj [E, D, H]; router weight after the expert,
//             down bias weighted with it as in NeMo _apply_bias), stored at
//             the slot row so the k-way combine reads tokens in order.
//
// Kernel design (one persistent CTA per SM, 320 threads):
//   warp 0      TMA producer: for every tile and 64-wide K block, one 128x64
//               box of A (K-major, 128-byte swizzle) and the 64x256 B tile
//               (N-major, 128-byte swizzle) into a 4-stage ring of 48 KB
//               stages, completion on a full[stage] mbarrier.  B arrives in
//               one copy through a {64 columns, K, column block, (gate/up,)
//               E} view of the weights where the column count is a multiple
//               of 64, else as four 64-column boxes (same shared image);
//   warp 1      TMEM allocator and MMA issuer: one thread issues four
//               tcgen05.mma 128x256x16 per stage (bf16 in, fp32 accumulate in
//               TMEM; M = 64 for a piece of at most 64 rows) and
//               tcgen05.commit's the stage back to the producer; two
//               256-column accumulators alternate between tiles;
//   warps 2..9  epilogue: tcgen05.ld of their 32 TMEM lanes (two warps per
//               lane quadrant split the columns), bias + activation (gate_up)
//               or bias x weight (down) in fp32, bf16 stores transposed
//               through a small shared staging block per warp.
// Tiles are the ragged expert segments cut in 128-row pieces times the
// output column blocks; the per-expert piece counts are rebuilt from the CSR
// offsets in shared memory at kernel start.  Within an expert the order is
// column block, then row piece, so CTAs running together share a weight
// column block through L2.  Rows of a piece beyond its expert's segment are
// computed and discarded.
//
// By default both contractions run in ONE cooperative launch (FUSED): the
// tile list is every gate_up tile, then every down tile; a down tile of a
// piece starts once all gate_up tiles of that piece have published their h
// (per-piece arrival counters, release/acquire); while it waits, its
// producer already copies the B stages the ring can hold (W_d does not
// depend on h).  CTAs take tiles with a static stride or, below 256 rows
// per expert, from an atomic counter.  A
// variant on CTA pairs (tcgen05 cta_group::2, 256x256 tiles, M = 128 over
// the pair for pieces of at most 128 rows; in the single launch with the
// static tile order, or as two launches) is kept selectable, and so is the
// gate_up GEMM gathering its rows of x itself (GATHER: tile::gather4 from
// every lane of the producer warp) instead of reading the gathered copy.
//
// Weights are read in their stored [K, N] (N-contiguous) layout: the B
// operand is MN-major, which tcgen05 supports for 16-bit types, so no
// transposed copy of the weights is needed.  Every mbarrier wait and
// cross-CTA wait is bounded; a timeout raises a CTA-wide abort, drains the
// copies and MMAs in flight, frees TMEM and records MOE_DEVICE_ERR_TIMEOUT_*
// in the status word.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdlib>
#include <mutex>
#include <vector>

#include "kernels.cuh"

namespace moe {
namespace {

constexpr int BM = 128;                 // rows per CTA (TMEM lanes)
constexpr int BN = 256;                 // accumulator columns per tile
constexpr int BK = 64;                  // K per stage: one 128-byte swizzle row of bf16
constexpr int UMMA_K = 16;              // K per tcgen05.mma (kind::f16)
constexpr int A_BYTES = BM * BK * 2;            // 16 KB
constexpr int B_BOX_BYTES = BK * 64 * 2;        // 8 KB: 64 K rows x 64 N columns
constexpr int NUM_EPI_WARPS = 8;              // two per TMEM lane quadrant, each half the columns
constexpr int NUM_THREADS = 64 + 32 * NUM_EPI_WARPS;  // producer warp, MMA warp, epilogue warps
constexpr uint32_t TMEM_COLS = 512;             // two BN-column fp32 accumulators
constexpr int CTRL_BYTES = 512;  // mbarriers (bytes 0..255) and flags (256..)
constexpr uint64_t kTimeoutNs = 2000000000ull;  // 2 s: far beyond any legitimate wait

// Per-CTA pipeline geometry.  PAIR = 1: one CTA computes a 128 x 256 tile and
// loads all four 64-column B boxes (48 KB a stage, 4 stages).  PAIR = 2: a
// cluster of two CTAs computes a 256 x 256 tile with tcgen05 cta_group::2;
// each CTA loads its 128 rows of A and its 128 columns of B (32 KB a stage,
// 6 stages), so each SM streams a third less operand data per FLOP.
template <int PAIR>
struct Geo {
  static constexpr int B_BOXES = 4 / PAIR;
  static constexpr int STAGE_BYTES = A_BYTES + B_BOXES * B_BOX_BYTES;
  static constexpr int STAGES = PAIR == 1 ? 4 : 6;
  static constexpr int PIECE = BM * PAIR;  // rows of one tile
  static constexpr uint32_t IDESC = idesc_bf16_f32(BM * PAIR, BN, /*a_mn_major=*/false, /*b_mn_major=*/true);
};

// Half tiles (single-CTA tiles only): an expert's last row piece with at most
// 64 valid rows is multiplied with M = 64 MMAs, half the tensor work of the
// full 128-row tile.  The M = 64 accumulator of tcgen05 (cta_group::1) puts
// row r in TMEM lane 32*(r/16) + r%16: the first 16 lanes of each 32-lane
// quadrant, so epilogue warp q reads rows 16q .. 16q+15 from its own lanes.
constexpr int HALF_ROWS = 64;
constexpr int HALF_A_BYTES = HALF_ROWS * BK * 2;  // 8 KB: the A rows a half tile copies
constexpr uint32_t IDESC_HALF = idesc_bf16_f32(HALF_ROWS, BN, /*a_mn_major=*/false, /*b_mn_major=*/true);
// CTA-pair tails: M = 128 over the pair (64 rows in each CTA); the
// accumulator layout is given with kPairTail below.
constexpr uint32_t IDESC_PAIR_TAIL = idesc_bf16_f32(BM, BN, /*a_mn_major=*/false, /*b_mn_major=*/true);

constexpr int MODE_GATE_UP_CONCAT = 0;
constexpr int MODE_GATE_UP_INTERLEAVED = 1;
constexpr int MODE_DOWN = 2;

struct GemmParams {
  const int32_t* offsets;
  const int32_t* perm;
  const float* weights;
  const __nv_bfloat16* bias;
  __nv_bfloat16* out;
  int* status;
  int E, R, H, D;
  int n_tiles, num_kb;
  int activation;
  float alpha, limit;
  int err_bit;
  int b_one_box;  // 1: the B tensor map delivers a stage's whole B tile in one copy
  // single launch: arrivals a down tile waits for beyond the real ones (0; 1
  // only under the test hook, which then never completes) and the time limit
  // of that wait
  int extra_arrivals;
  unsigned long long dep_timeout_ns;
  int a_direct;  // gate_up: A rows are rows within the expert's segment (A = x)
  int k;         // routed slots per token (a slot's token is slot / k)
};

struct TileCoord {
  int e, row0, rows, n, piece;  // piece: global index of the 128-row piece
};

// Tile t -> (expert, first permuted row of the tile, valid rows, output
// column block).  s_mt is the exclusive prefix of per-expert pieces of
// `piece` rows (s_mt[E] = total).
__device__ __forceinline__ TileCoord decode_tile(int t, int n_tiles, int E, const int* s_mt, const int* s_off,
                                                 int piece) {
  int lo = 0, hi = E;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_mt[mid] * n_tiles <= t) lo = mid;
    else hi = mid;
  }
  TileCoord c;
  c.e = lo;
  const int local = t - s_mt[lo] * n_tiles;
  const int mt = s_mt[lo + 1] - s_mt[lo];
  c.n = local / mt;
  const int m = local - c.n * mt;
  c.row0 = s_off[lo] + m * piece;
  c.rows = min(piece, s_off[lo + 1] - c.row0);
  c.piece = s_mt[lo] + m;
  return c;
}

__device__ __forceinline__ bool wait_time_only(uint32_t bar, uint32_t parity) {
  int never = 0;
  return mbar_wait(bar, parity, &never, kTimeoutNs);
}

// ------------------------------------------ single-launch cross-CTA hand-off
// A gate_up tile's epilogue warps each publish their h stores with one
// release add on the piece's arrival counter; the producer of a down tile
// waits (acquire) until all of the piece's gate_up tiles have arrived, then
// orders those generic-proxy stores before its TMA (async-proxy) reads.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ void red_release_add(int* addr, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ int ld_acquire(const int* addr) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(addr) : "memory");
  return v;
}

// Dynamic tile order of the single launch (when `sched` is given): the producer thread draws tile
// numbers from a global counter (one tile ahead, so the atomic's latency
// overlaps the current tile's copies) and hands each to the MMA thread and
// the epilogue warps through a ring of kTileRing slots in shared memory.
// Numbers are drawn in increasing order, so a down tile still only waits on
// tiles that were handed to running CTAs before it; CTAs that finish early
// simply draw more tiles, which evens out the end of the launch.  Without
// `sched` CTA c takes tiles c, c + grid, c + 2 grid, ... (static order).
constexpr int kTileRing = 8;

// Consumer side of the ring: the n-th tile number (n counts from 0), or
// false if the wait gave up.  Every lane of the calling warp reads the slot
// before `releaser` frees it.
__device__ __forceinline__ bool ring_take(uint32_t ring_full0, uint32_t ring_empty0, const volatile int* ring,
                                          int n, volatile int* abort, bool releaser, int* t) {
  const int slot = n % kTileRing;
  const uint32_t ph = static_cast<uint32_t>(n / kTileRing) & 1u;
  if (!mbar_wait(ring_full0 + 8 * slot, ph, abort, kTimeoutNs)) return false;
  *t = ring[slot];
  __syncwarp(__activemask());
  if (releaser) mbar_arrive(ring_empty0 + 8 * slot);
  return true;
}

// Bounded wait for *counter >= target.  Gives up (false, CTA abort raised,
// err bits recorded at once so other CTAs stop waiting too) after the
// timeout, when this CTA aborts, or when another CTA has recorded a timeout.
__device__ __forceinline__ bool wait_arrivals(const int* counter, int target, volatile int* abort,
                                              volatile int* status, int err_bits, uint64_t timeout_ns) {
  if (ld_acquire(counter) >= target) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1; it < (1u << 26); ++it) {
    __nanosleep(64);
    if (ld_acquire(counter) >= target) return true;
    if ((it & 15u) == 0) {
      if (*abort || (*status & err_bits) != 0) break;
      if (global_timer_ns() - t0 > timeout_ns) break;
    }
  }
  *abort = 1;
  atomicOr(const_cast<int*>(status), err_bits);
  return false;
}

// ----------------------------------------------------------- epilogues
// Each epilogue warp owns 32 tile rows (its TMEM lane quadrant) and half of
// the tile's output columns, which it walks in chunks of 32 output columns:
// every thread computes its row's 32 values from the fp32 accumulator, the
// warp transposes them through a 32 x 32 bf16 staging block in shared
// memory (row stride 80 B: conflict-free), then stores 8 rows x 64 B per
// instruction, so each store fills whole 32-byte sectors of contiguous
// columns instead of scattering 16-byte pieces over 32 rows.
constexpr int kStageRowBytes = 80;
constexpr int kStageWarpBytes = 32 * kStageRowBytes;  // 2560 B per epilogue warp
constexpr int kOutChunk = 32;                          // output columns per chunk

// gate_up: 32 h columns starting at tile h column hc (relative to the tile),
// whose accumulator columns start at TMEM column tcol: concatenated, gate
// of h column hc + i at tcol + i and up at tcol + up_off + i; interleaved,
// the (gate, up) pair at tcol + 2i, tcol + 2i + 1.
template <int MODE>
__device__ __forceinline__ void gate_up_chunk(const GemmParams& p, const TileCoord& tc, uint32_t tacc, int hc,
                                              int tcol, int up_off, uint32_t (&packed)[16]) {
  const int hcol0 = tc.n * 128 + hc;  // absolute h column of value 0
  const __nv_bfloat16* bg = p.bias != nullptr ? p.bias + static_cast<int64_t>(tc.e) * 2 * p.D : nullptr;
  uint32_t a0[32], a1[32];
  if constexpr (MODE == MODE_GATE_UP_CONCAT) {
    tmem_ld32(tacc + tcol, a0);           // gate columns
    tmem_ld32(tacc + tcol + up_off, a1);  // matching up columns
  } else {
    tmem_ld32(tacc + tcol, a0);       // (gate, up) pairs of h columns hc .. hc+15
    tmem_ld32(tacc + tcol + 32, a1);  // ... and hc+16 .. hc+31
  }
  tmem_ld_wait();
#pragma unroll
  for (int j = 0; j < 32; j += 2) {
    float h2[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int jj = j + q;
      float g, u;
      if constexpr (MODE == MODE_GATE_UP_CONCAT) {
        g = __uint_as_float(a0[jj]);
        u = __uint_as_float(a1[jj]);
      } else {
        const uint32_t* src = jj < 16 ? a0 : a1;
        const int m = jj & 15;
        g = __uint_as_float(src[2 * m]);
        u = __uint_as_float(src[2 * m + 1]);
      }
      const int col = hcol0 + jj;
      if (bg != nullptr && col < p.D) {
        if constexpr (MODE == MODE_GATE_UP_CONCAT) {
          g += __bfloat162float(bg[col]);
          u += __bfloat162float(bg[p.D + col]);
        } else {
          g += __bfloat162float(bg[2 * col]);
          u += __bfloat162float(bg[2 * col + 1]);
        }
      }
      h2[q] = gated_act(p.activation, g, u, p.alpha, p.limit);
    }
    packed[j / 2] = pack_bf16x2(h2[0], h2[1]);
  }
}

// down: 32 output columns starting at tile column oc, accumulator columns
// from TMEM column tcol: (acc + b_d[e]) * w.
__device__ __forceinline__ void down_chunk(const GemmParams& p, const TileCoord& tc, uint32_t tacc, int oc, int tcol,
                                           float wgt, uint32_t (&packed)[16]) {
  const int col0 = tc.n * BN + oc;
  const __nv_bfloat16* bd = p.bias != nullptr ? p.bias + static_cast<int64_t>(tc.e) * p.H : nullptr;
  uint32_t a[32];
  tmem_ld32(tacc + tcol, a);
  tmem_ld_wait();
#pragma unroll
  for (int j = 0; j < 32; j += 2) {
    float y[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      float v = __uint_as_float(a[j + q]);
      if (bd != nullptr && col0 + j + q < p.H) v += __bfloat162float(bd[col0 + j + q]);
      y[q] = v * wgt;
    }
    packed[j / 2] = pack_bf16x2(y[0], y[1]);
  }
}

// Accumulator shapes of a tile in this CTA's TMEM.
//   kFull      128 rows in lanes 0..127, the tile's 256 columns in TMEM
//              columns 0..255 (in the order of the stage's B tile);
//   kHalf      M = 64 (one CTA): row r in lane 32*(r/16) + r%16;
//   kPairTail  M = 128 over a CTA pair, 64 rows in each CTA: lanes 0..63
//              hold its rows for tile columns 0..127 and lanes 64..127 the
//              same rows for columns 128..255, both in TMEM columns 0..127.
constexpr int kFull = 0;
constexpr int kHalf = 1;
constexpr int kPairTail = 2;

// One tile's epilogue for one warp (TMEM lane quadrant `quad`, column part
// `part` of two).  A CTA pair's concatenated gate_up tile holds, per CTA B
// half, the gate and then the up columns of 64 h columns, so a gate and its
// up share a TMEM lane in every shape.
template <int MODE, int PAIR>
__device__ __forceinline__ void epilogue_tile(const GemmParams& p, const TileCoord& tc, uint32_t tacc, int quad,
                                              int part, int lane, uint8_t* stage, int shape) {
  constexpr bool kDown = MODE == MODE_DOWN;
  // tile row held by this thread's TMEM lane
  int row = quad * 32 + lane;
  bool has_row = true;
  if (shape == kHalf) {
    row = quad * 16 + lane;
    has_row = lane < 16;
  } else if (shape == kPairTail) {
    row = (quad & 1) * 32 + lane;
  }
  // destination row of this thread's tile row, or -1 if it is not stored
  int64_t dst = -1;
  float wgt = 0.f;
  if (has_row && row < tc.rows) {
    if constexpr (kDown) {
      const int slot = p.perm[tc.row0 + row];
      if (slot < 0 || slot >= p.R) {
        atomicOr(p.status, MOE_DEVICE_ERR_CSR);
      } else {
        dst = static_cast<int64_t>(slot) * p.H;
        wgt = p.weights != nullptr ? p.weights[slot] : 1.f;
      }
    } else {
      dst = (static_cast<int64_t>(tc.row0) + row) * p.D;
    }
  }
  // the 4 rows this lane stores in the transposed phase: 8*i + lane/4
  int64_t my_dst[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int src_lane = 8 * i + (lane >> 2);
    const int lo = __shfl_sync(0xffffffffu, static_cast<int>(dst & 0xffffffff), src_lane);
    const int hi = __shfl_sync(0xffffffffu, static_cast<int>(dst >> 32), src_lane);
    my_dst[i] = (static_cast<int64_t>(hi) << 32) | static_cast<uint32_t>(lo);
  }
  // this warp's output columns: n_chunks chunks of 32 from tile column rel0,
  // their accumulator columns from TMEM column tcol0, tstep apart
  const bool tail = shape == kPairTail;
  int rel0, tcol0, n_chunks, tstep, up_off = 128;
  if constexpr (kDown) {
    rel0 = tail ? (quad >> 1) * 128 + part * 64 : part * 128;
    tcol0 = tail ? part * 64 : rel0;
    n_chunks = tail ? 2 : 4;
    tstep = 32;
  } else if constexpr (MODE == MODE_GATE_UP_CONCAT) {
    rel0 = tail ? (quad >> 1) * 64 + part * 32 : part * 64;
    n_chunks = tail ? 1 : 2;
    tstep = 32;
    if constexpr (PAIR == 2) {
      up_off = 64;
      tcol0 = tail ? part * 32 : part * 128;
    } else {
      tcol0 = rel0;
    }
  } else {
    rel0 = tail ? (quad >> 1) * 64 + part * 32 : part * 64;
    tcol0 = tail ? part * 64 : 2 * rel0;
    n_chunks = tail ? 1 : 2;
    tstep = 64;
  }
  const int limit = kDown ? p.H : p.D;
  const int base_col = kDown ? tc.n * BN : tc.n * 128;
  const int q = lane & 3;  // 16-byte chunk of a 64-byte row segment
  uint8_t* my_row = stage + lane * kStageRowBytes;
#pragma unroll 1
  for (int ch = 0; ch < n_chunks; ++ch) {
    const int rel = rel0 + kOutChunk * ch;
    const int tcol = tcol0 + tstep * ch;
    uint32_t packed[16];
    __syncwarp();
    if constexpr (kDown) down_chunk(p, tc, tacc, rel, tcol, wgt, packed);
    else gate_up_chunk<MODE>(p, tc, tacc, rel, tcol, up_off, packed);
#pragma unroll
    for (int c = 0; c < 4; ++c)
      *reinterpret_cast<uint4*>(my_row + 16 * c) =
          make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
    __syncwarp();
    const int col = base_col + rel + 8 * q;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int rr = 8 * i + (lane >> 2);
      if (my_dst[i] >= 0 && col < limit) {
        const uint4 v = *reinterpret_cast<const uint4*>(stage + rr * kStageRowBytes + 16 * q);
        *reinterpret_cast<uint4*>(p.out + my_dst[i] + col) = v;
      }
    }
  }
}

// The B tile of one down-GEMM stage: 64 K rows (from kc) x the tile's 256
// output columns of W_d[e], in one copy or as four 64-column boxes.
__device__ __forceinline__ void load_down_b(uint32_t sb, const CUtensorMap* map, int one_box, uint32_t bar, int kc,
                                            const TileCoord& tc) {
  if (one_box) {
    tma_load_4d(sb, map, bar, 0, kc, 4 * tc.n, tc.e);
  } else {
    const int c0 = tc.n * BN;
#pragma unroll
    for (int j = 0; j < 4; ++j) tma_load_3d(sb + j * B_BOX_BYTES, map, bar, c0 + 64 * j, kc, tc.e);
  }
}

// ------------------------------------------------------------- the kernel
// FUSED = false: one contraction (MODE) over its tile list.  FUSED = true
// (single-CTA tiles only): the gate_up contraction (MODE, maps A/B, params p)
// followed in the same tile list by the down contraction (maps A2/B2, params
// p2); tile t < total1 is a gate_up tile, the rest are down tiles, and every
// CTA walks the list in increasing order, so a down tile only ever waits on
// gate_up tiles that precede it and that some resident CTA has already
// started (the launch is cooperative: all CTAs are resident).
template <int MODE, int PAIR, bool FUSED, bool GATHER>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                        const __grid_constant__ CUtensorMap mapA2, const __grid_constant__ CUtensorMap mapB2,
                        const __grid_constant__ CUtensorMap mapAh, const __grid_constant__ CUtensorMap mapA2h,
                        const GemmParams p, const GemmParams p2, int* arrivals, int* sched) {
  static_assert(!FUSED || MODE != MODE_DOWN, "the fused form is gate_up then down");
  static_assert(!GATHER || (PAIR == 1 && MODE != MODE_DOWN), "rows are gathered for gate_up tiles of one CTA");
  using G = Geo<PAIR>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint8_t* ctrl = smem + G::STAGES * G::STAGE_BYTES;
  const uint32_t full0 = smem_u32(ctrl);              // STAGES mbarriers
  const uint32_t empty0 = full0 + 8 * G::STAGES;      // STAGES mbarriers
  const uint32_t tfull0 = empty0 + 8 * G::STAGES;     // 2 mbarriers
  const uint32_t tempty0 = tfull0 + 16;               // 2 mbarriers
  const uint32_t drain_bar = tempty0 + 16;            // 1 mbarrier
  const uint32_t ring_full0 = drain_bar + 8;          // kTileRing mbarriers (FUSED)
  const uint32_t ring_empty0 = ring_full0 + 8 * kTileRing;  // kTileRing mbarriers (FUSED)
  // the dynamic tile order (and its ring of tile numbers) is for one CTA a tile
  constexpr bool kRing = FUSED && PAIR == 1;
  static_assert((2 * G::STAGES + 5 + (kRing ? 2 * kTileRing : 0)) * 8 <= 256,
                "mbarriers overflow their part of the control block");
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctrl + 256);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctrl + 260);
  int* bad_flag = reinterpret_cast<int*>(ctrl + 264);
  volatile int* s_ring = reinterpret_cast<volatile int*>(ctrl + 288);  // kTileRing tile numbers
  int* s_off = reinterpret_cast<int*>(ctrl + CTRL_BYTES);
  int* s_mt = s_off + (p.E + 1);
  // epilogue staging: one kStageWarpBytes block per epilogue warp, 16-byte aligned
  uint8_t* s_stage = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(s_mt + p.E + 1) + 15) & ~uintptr_t(15));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if constexpr (PAIR == 2) {
    // the pair's tcgen05 operations need a cluster of exactly two CTAs
    if (cluster_nctarank() != 2) {
      if (threadIdx.x == 0) atomicOr(p.status, MOE_DEVICE_ERR_LAUNCH);
      return;
    }
  }
  const uint32_t rank = PAIR == 2 ? cluster_ctarank() : 0u;  // 0 = leader of the pair
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < G::STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull0 + 8 * a, 1);
      mbar_init(tempty0 + 8 * a, 32 * NUM_EPI_WARPS * PAIR);
    }
    mbar_init(drain_bar, 1);
    if constexpr (kRing) {
      for (int i = 0; i < kTileRing; ++i) {
        mbar_init(ring_full0 + 8 * i, 1);
        mbar_init(ring_empty0 + 8 * i, 1 + NUM_EPI_WARPS);  // the MMA thread and one lane per epilogue warp
      }
    }
    *abort_flag = 0;
    *bad_flag = 0;
    fence_mbar_init();
    tma_prefetch_map(&mapA);
    tma_prefetch_map(&mapB);
    if constexpr (FUSED) {
      tma_prefetch_map(&mapA2);
      tma_prefetch_map(&mapB2);
    }
  }
  if (warp == 1) {
    if constexpr (PAIR == 2) {
      tmem_alloc_pair(smem_u32(tmem_slot), TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
      tmem_relinquish();
    }
  }
  griddep_wait();  // the CSR and operands of the kernels before are complete and visible
  for (int i = threadIdx.x; i <= p.E; i += NUM_THREADS) s_off[i] = p.offsets[i];
  __syncthreads();
  if (warp == 0) {
    // Validate the CSR and build the per-expert prefix of tile pieces.
    const int per = (p.E + 31) / 32;
    const int e0 = min(lane * per, p.E), e1 = min(e0 + per, p.E);
    int local = 0;
    bool bad = false;
    for (int e = e0; e < e1; ++e) {
      const int cnt = s_off[e + 1] - s_off[e];
      if (cnt < 0) bad = true;
      else local += (cnt + G::PIECE - 1) / G::PIECE;
    }
    int incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    int run = incl - local;
    for (int e = e0; e < e1; ++e) {
      s_mt[e] = run;
      const int cnt = s_off[e + 1] - s_off[e];
      if (cnt > 0) run += (cnt + G::PIECE - 1) / G::PIECE;
    }
    if (lane == 31) s_mt[p.E] = incl;
    if (lane == 0 && (s_off[0] != 0 || s_off[p.E] > p.R)) bad = true;
    if (__any_sync(0xffffffffu, bad) && lane == 0) *bad_flag = 1;
  }
  tc_fence_before_sync();
  if constexpr (PAIR == 2) {
    cluster_sync();  // both CTAs' barriers exist before either signals the other's
  } else {
    __syncthreads();
  }
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  const bool bad = *bad_flag != 0;
  if (bad && blockIdx.x == 0 && threadIdx.x == 0) atomicOr(p.status, MOE_DEVICE_ERR_CSR);
  const int total1 = bad ? 0 : s_mt[p.E] * p.n_tiles;
  const int total_tiles = total1 + (FUSED && !bad ? s_mt[p.E] * p2.n_tiles : 0);
  const int first_tile = blockIdx.x / PAIR;
  const int tile_stride = gridDim.x / PAIR;
  // down tiles of a piece wait for this many arrivals (one per epilogue warp
  // of each of the piece's gate_up tiles)
  const int arrivals_needed = NUM_EPI_WARPS * PAIR * p.n_tiles + p.extra_arrivals;
  const bool dyn = kRing && sched != nullptr;  // dynamic tile order

  if (warp == 0) {
    if (GATHER || lane == 0) {
      // ------------------------------------------------ TMA producer
      // Lane 0 waits on the barriers, draws tiles and issues every copy.
      // GATHER: the whole warp runs the loop, lane 0 still does all of the
      // above, and for a gate_up tile each lane also issues one
      // tile::gather4 per stage: the four rows 4*lane .. 4*lane+3 of the
      // tile, read from x by the routing permutation (row -> slot -> token),
      // into the same shared-memory image a 128-row box of the permuted copy
      // would give.
      auto bcast = [&](auto v) {
        if constexpr (GATHER) return __shfl_sync(0xffffffffu, v, 0);
        else return v;
      };
      int it = 0;
      bool ok = true;
      int t_next = first_tile;
      if (dyn && lane == 0) t_next = atomicAdd(sched, 1);
      t_next = bcast(t_next);
      for (int n = 0; ok; ++n) {
        const int t = t_next;
        if (dyn) {
          // hand tile number n to the consumers (the end marker too)
          bool stop = false;
          if (lane == 0) {
            const int slot = n % kTileRing;
            if (!mbar_wait(ring_empty0 + 8 * slot, (static_cast<uint32_t>(n / kTileRing) & 1u) ^ 1u, abort_flag,
                           kTimeoutNs)) {
              ok = false;
            } else {
              s_ring[slot] = t;
              mbar_arrive(ring_full0 + 8 * slot);
              if (t >= total_tiles) stop = true;
              else t_next = atomicAdd(sched, 1);  // in flight while this tile's copies are issued
            }
          }
          ok = bcast(ok);
          stop = bcast(stop);
          t_next = bcast(t_next);
          if (!ok || stop) break;
        } else {
          if (t >= total_tiles) break;
          t_next = t + tile_stride;
        }
        const bool ph2 = FUSED && t >= total1;
        const TileCoord tc = ph2 ? decode_tile(t - total1, p2.n_tiles, p.E, s_mt, s_off, G::PIECE)
                                 : decode_tile(t, p.n_tiles, p.E, s_mt, s_off, G::PIECE);
        // a CTA pair's piece of at most 128 rows runs M = 128: 64 rows in each CTA
        const bool pair_tail = PAIR == 2 && tc.rows <= BM;
        const int arow = (!ph2 && p.a_direct ? tc.row0 - s_off[tc.e] : tc.row0) +
                         static_cast<int>(rank) * (pair_tail ? HALF_ROWS : BM);
        const int nkb = ph2 ? p2.num_kb : p.num_kb;
        // a half tile (at most 64 rows, M = 64 MMAs) copies only 64 rows of A
        const bool half = (PAIR == 1 && tc.rows <= HALF_ROWS) || pair_tail;
        const uint32_t stage_tx = half ? G::STAGE_BYTES - HALF_A_BYTES : G::STAGE_BYTES;
        // A down tile whose piece is not complete yet issues the B copies of
        // its first stages (W_d does not depend on h) before it waits, on full
        // barriers armed with their bytes only (expect_tx, no arrival, so no
        // stage can complete), and their A copies after the wait.
        int pre = 0;  // stages of this tile whose B copy went out before the wait
        if constexpr (FUSED) {
          if (ph2) {
            bool got = true;
            if (lane == 0) {
              if (ld_acquire(arrivals + tc.piece) < arrivals_needed) {
                // (one CTA a tile only: a pair's leader counts both CTAs' bytes)
                for (; PAIR == 1 && pre < nkb && pre < G::STAGES; ++pre) {
                  const int s = (it + pre) % G::STAGES;
                  const uint32_t ph = static_cast<uint32_t>((it + pre) / G::STAGES) & 1u;
                  if (!mbar_wait(empty0 + 8 * s, ph ^ 1u, abort_flag, kTimeoutNs)) {
                    got = false;
                    break;
                  }
                  const uint32_t sb = sbase + s * G::STAGE_BYTES + A_BYTES;
                  mbar_expect_tx(full0 + 8 * s, 4 * B_BOX_BYTES);
                  load_down_b(sb, &mapB2, p2.b_one_box, full0 + 8 * s, pre * BK, tc);
                }
                if (got)
                  got = wait_arrivals(arrivals + tc.piece, arrivals_needed, abort_flag, p.status, p.err_bit,
                                      p.dep_timeout_ns);
                if (!got) {
                  // the stages armed so far complete once their B bytes land,
                  // so the abort drain below can wait for them
                  for (int j = 0; j < pre; ++j) mbar_arrive(full0 + 8 * ((it + j) % G::STAGES));
                  it += pre;
                }
              }
              if (got) fence_proxy_async_global();  // h stores (generic proxy) before the TMA reads of h
            }
            pre = bcast(pre);
            if (!bcast(got)) {
              ok = false;
              break;
            }
          }
        }
        // GATHER, gate_up tile: the tokens of this lane's four tile rows.
        // Rows past the expert's segment (and slots outside [0, R), which the
        // down epilogue flags) read the tile's first token; their results are
        // discarded.
        const bool gathered = GATHER && !ph2;
        int tok[4] = {0, 0, 0, 0};
        if constexpr (GATHER) {
          if (gathered) {
            const int s0 = p.perm[tc.row0];
            const int first = s0 >= 0 && s0 < p.R ? s0 / p.k : 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int r = 4 * lane + j;
              const int slot = r < tc.rows ? p.perm[tc.row0 + r] : -1;
              tok[j] = slot >= 0 && slot < p.R ? slot / p.k : first;
            }
          }
        }
        for (int kb = 0; kb < nkb; ++kb) {
          const int s = it % G::STAGES;
          const uint32_t ph = static_cast<uint32_t>(it / G::STAGES) & 1u;
          bool got = true;
          if (lane == 0 && kb >= pre) got = mbar_wait(empty0 + 8 * s, ph ^ 1u, abort_flag, kTimeoutNs);
          if (!bcast(got)) {
            ok = false;
            break;
          }
          const uint32_t sa = sbase + s * G::STAGE_BYTES;
          const uint32_t sb = sa + A_BYTES;
          // the leader's full barrier counts both CTAs' bytes
          const uint32_t fb = PAIR == 2 ? map_to_rank(full0 + 8 * s, 0) : full0 + 8 * s;
          const int kc = kb * BK;
          if (gathered) {
            // 32 (or, for a half tile, 16) lanes each copy four rows of A
            if (lane == 0) mbar_arrive_expect_tx(fb, stage_tx);
            __syncwarp();
            if (!half || lane < HALF_ROWS / 4)
              tma_gather4(sa + static_cast<uint32_t>(lane) * 512u, &mapA, fb, kc, tok[0], tok[1], tok[2], tok[3]);
            if (lane == 0) {
              if (p.b_one_box) {
                if constexpr (MODE == MODE_GATE_UP_CONCAT) tma_load_5d(sb, &mapB, fb, 0, kc, 2 * tc.n, 0, tc.e);
                else tma_load_4d(sb, &mapB, fb, 0, kc, 4 * tc.n, tc.e);
              } else if constexpr (MODE == MODE_GATE_UP_CONCAT) {
                const int c0 = tc.n * 128;
                tma_load_4d(sb, &mapB, fb, c0, 0, kc, tc.e);
                tma_load_4d(sb + B_BOX_BYTES, &mapB, fb, c0 + 64, 0, kc, tc.e);
                tma_load_4d(sb + 2 * B_BOX_BYTES, &mapB, fb, c0, 1, kc, tc.e);
                tma_load_4d(sb + 3 * B_BOX_BYTES, &mapB, fb, c0 + 64, 1, kc, tc.e);
              } else {
                const int c0 = tc.n * BN;
#pragma unroll
                for (int j = 0; j < 4; ++j) tma_load_3d(sb + j * B_BOX_BYTES, &mapB, fb, c0 + 64 * j, kc, tc.e);
              }
            }
          } else if (lane == 0) {
            if (FUSED && ph2 && PAIR == 2) {
              // down tile of a CTA pair: each CTA copies its rows of h (128,
              // or 64 in a pair tail) and its half of the tile's 256 columns
              // of W_d; the leader expects both CTAs' bytes
              if (leader) mbar_arrive_expect_tx(full0 + 8 * s, 2 * stage_tx);
              tma_load_2d_pair(sa, half ? &mapA2h : &mapA2, fb, kc, arow);
              if (p2.b_one_box) {
                tma_load_4d_pair(sb, &mapB2, fb, 0, kc, 4 * tc.n + 2 * static_cast<int>(rank), tc.e);
              } else {
                const int c0 = tc.n * BN + static_cast<int>(rank) * 128;
                tma_load_3d_pair(sb, &mapB2, fb, c0, kc, tc.e);
                tma_load_3d_pair(sb + B_BOX_BYTES, &mapB2, fb, c0 + 64, kc, tc.e);
              }
            } else if (FUSED && ph2) {
              // down tile: h rows of the piece, 256 columns of W_d (B already
              // in flight for the first `pre` stages)
              if (kb < pre) {
                mbar_arrive_expect_tx(fb, stage_tx - 4 * B_BOX_BYTES);
                tma_load_2d(sa, half ? &mapA2h : &mapA2, fb, kc, arow);
              } else {
                mbar_arrive_expect_tx(fb, stage_tx);
                tma_load_2d(sa, half ? &mapA2h : &mapA2, fb, kc, arow);
                load_down_b(sb, &mapB2, p2.b_one_box, fb, kc, tc);
              }
            } else if (PAIR == 1 && p.b_one_box) {
              // {64 columns, K, column block, (gate/up,) E} view: one copy lays
              // the four 64-column boxes out exactly as four copies would
              mbar_arrive_expect_tx(fb, stage_tx);
              tma_load_2d(sa, half ? &mapAh : &mapA, fb, kc, arow);
              if constexpr (MODE == MODE_GATE_UP_CONCAT) tma_load_5d(sb, &mapB, fb, 0, kc, 2 * tc.n, 0, tc.e);
              else tma_load_4d(sb, &mapB, fb, 0, kc, 4 * tc.n, tc.e);
            } else if constexpr (PAIR == 1) {
              mbar_arrive_expect_tx(fb, stage_tx);
              tma_load_2d(sa, half ? &mapAh : &mapA, fb, kc, arow);
              if constexpr (MODE == MODE_GATE_UP_CONCAT) {
                // 4-D view {D, 2 (gate/up), H, E}: two gate boxes then two up boxes.
                const int c0 = tc.n * 128;
                tma_load_4d(sb, &mapB, fb, c0, 0, kc, tc.e);
                tma_load_4d(sb + B_BOX_BYTES, &mapB, fb, c0 + 64, 0, kc, tc.e);
                tma_load_4d(sb + 2 * B_BOX_BYTES, &mapB, fb, c0, 1, kc, tc.e);
                tma_load_4d(sb + 3 * B_BOX_BYTES, &mapB, fb, c0 + 64, 1, kc, tc.e);
              } else {
                // 3-D view {N, K, E}: four consecutive 64-column boxes.
                const int c0 = tc.n * BN;
#pragma unroll
                for (int j = 0; j < 4; ++j) tma_load_3d(sb + j * B_BOX_BYTES, &mapB, fb, c0 + 64 * j, kc, tc.e);
              }
            } else {
              // The leader expects both CTAs' bytes on its own barrier; each
              // CTA loads its rows of A (128, or 64 in a tail) and its half of
              // the 256 columns.
              if (leader) mbar_arrive_expect_tx(full0 + 8 * s, 2 * stage_tx);
              tma_load_2d_pair(sa, half ? &mapAh : &mapA, fb, kc, arow);
              if (p.b_one_box) {
                // this CTA's two 64-column blocks in one copy (concatenated:
                // the gate and the up block of h columns 64*rank .. +63 of the tile)
                if constexpr (MODE == MODE_GATE_UP_CONCAT)
                  tma_load_5d_pair(sb, &mapB, fb, 0, kc, 2 * tc.n + static_cast<int>(rank), 0, tc.e);
                else
                  tma_load_4d_pair(sb, &mapB, fb, 0, kc, 4 * tc.n + 2 * static_cast<int>(rank), tc.e);
              } else if constexpr (MODE == MODE_GATE_UP_CONCAT) {
                // the gate and the up block of h columns c0 .. c0+63
                const int c0 = tc.n * 128 + 64 * static_cast<int>(rank);
                tma_load_4d_pair(sb, &mapB, fb, c0, 0, kc, tc.e);
                tma_load_4d_pair(sb + B_BOX_BYTES, &mapB, fb, c0, 1, kc, tc.e);
              } else {
                const int c0 = tc.n * BN + static_cast<int>(rank) * 128;
                tma_load_3d_pair(sb, &mapB, fb, c0, kc, tc.e);
                tma_load_3d_pair(sb + B_BOX_BYTES, &mapB, fb, c0 + 64, kc, tc.e);
              }
            }
          }
          ++it;
        }
      }
      if (lane == 0) {
        if (ok) {
          // Tail: wait until the MMAs have released every stage, so that no
          // tcgen05.commit arrival lands after this CTA exits.
          for (int i = 0; i < G::STAGES; ++i, ++it) {
            const int s = it % G::STAGES;
            const uint32_t ph = static_cast<uint32_t>(it / G::STAGES) & 1u;
            if (!mbar_wait(empty0 + 8 * s, ph ^ 1u, abort_flag, kTimeoutNs)) break;
          }
        } else if (leader) {
          // Aborted: let the copies already issued land before shared memory
          // is released (time-bounded, independent of the abort flag).
          for (int s = 0; s < G::STAGES; ++s) {
            if (it > s) {
              const int last = s + ((it - 1 - s) / G::STAGES) * G::STAGES;
              wait_time_only(full0 + 8 * s, static_cast<uint32_t>(last / G::STAGES) & 1u);
            }
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // --------------------------------------------------- MMA issuer
      int it = 0;
      bool ok = true;
      for (int ti = 0; ok; ++ti) {
        int t = first_tile + ti * tile_stride;
        if (dyn) {
          if (!ring_take(ring_full0, ring_empty0, s_ring, ti, abort_flag, true, &t)) {
            ok = false;
            break;
          }
        }
        if (t >= total_tiles) break;
        const int acc = ti & 1;
        const uint32_t aph = static_cast<uint32_t>(ti >> 1) & 1u;
        if (!mbar_wait(tempty0 + 8 * acc, aph ^ 1u, abort_flag, kTimeoutNs)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        const bool ph2 = FUSED && t >= total1;
        const int nkb = ph2 ? p2.num_kb : p.num_kb;
        uint32_t idesc = G::IDESC;
        {
          const TileCoord tc = ph2 ? decode_tile(t - total1, p2.n_tiles, p.E, s_mt, s_off, G::PIECE)
                                   : decode_tile(t, p.n_tiles, p.E, s_mt, s_off, G::PIECE);
          if (PAIR == 1 && tc.rows <= HALF_ROWS) idesc = IDESC_HALF;
          if (PAIR == 2 && tc.rows <= BM) idesc = IDESC_PAIR_TAIL;
        }
        for (int kb = 0; kb < nkb; ++kb) {
          const int s = it % G::STAGES;
          const uint32_t ph = static_cast<uint32_t>(it / G::STAGES) & 1u;
          if (!mbar_wait(full0 + 8 * s, ph, abort_flag, kTimeoutNs)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t sa = sbase + s * G::STAGE_BYTES;
          const uint32_t sb = sa + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk) {
            // A: K-major rows of 128 B, 8-row swizzle atoms 1024 B apart; a
            // 16-wide K step is 32 B along the row.
            const uint64_t a_desc = smem_desc_sw128(sa + kk * UMMA_K * 2, 16, 1024);
            // B: N-major; 64-column blocks B_BOX_BYTES apart (LBO), 8-row K
            // groups 1024 B apart (SBO); a 16-row K step is 2048 B.
            const uint64_t b_desc = smem_desc_sw128(sb + kk * UMMA_K * 128, B_BOX_BYTES, 1024);
            if constexpr (PAIR == 2) mma_bf16_ss_pair(d_tmem, a_desc, b_desc, idesc, (kb | kk) != 0 ? 1u : 0u);
            else mma_bf16_ss(d_tmem, a_desc, b_desc, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          if constexpr (PAIR == 2) mma_commit_pair(empty0 + 8 * s, 0x3);
          else mma_commit(empty0 + 8 * s);
          ++it;
        }
        if (!ok) break;
        if constexpr (PAIR == 2) mma_commit_pair(tfull0 + 8 * acc, 0x3);
        else mma_commit(tfull0 + 8 * acc);
      }
      if (!ok) {
        // Aborted: every MMA issued so far must finish before TMEM is freed.
        if constexpr (PAIR == 2) mma_commit_pair(drain_bar, 0x1);
        else mma_commit(drain_bar);
        wait_time_only(drain_bar, 0);
      }
    }
  } else {
    // ------------------------------------------------------ epilogue
    const int quad = warp & 3;  // this warp may access TMEM lanes 32*quad..+31
    const int part = (warp - 2) >> 2;  // which half of the tile's columns
    for (int ti = 0;; ++ti) {
      int t = first_tile + ti * tile_stride;
      if (dyn) {
        const bool took = ring_take(ring_full0, ring_empty0, s_ring, ti, abort_flag, lane == 0, &t);
        if (!__all_sync(0xffffffffu, took)) break;
      }
      if (t >= total_tiles) break;
      const bool ph2 = FUSED && t >= total1;
      TileCoord tc = ph2 ? decode_tile(t - total1, p2.n_tiles, p.E, s_mt, s_off, G::PIECE)
                         : decode_tile(t, p.n_tiles, p.E, s_mt, s_off, G::PIECE);
      int shape = kFull;
      if constexpr (PAIR == 1) {
        if (tc.rows <= HALF_ROWS) shape = kHalf;
      } else {
        // a piece of at most 128 rows: M = 128 over the pair, 64 rows each
        const int share = tc.rows <= BM ? HALF_ROWS : BM;
        if (tc.rows <= BM) shape = kPairTail;
        tc.row0 += static_cast<int>(rank) * share;
        tc.rows -= static_cast<int>(rank) * share;  // may be <= 0: nothing of this half is stored
      }
      const int acc = ti & 1;
      const uint32_t aph = static_cast<uint32_t>(ti >> 1) & 1u;
      const bool got = mbar_wait(tfull0 + 8 * acc, aph, abort_flag, kTimeoutNs);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after_sync();
      const uint32_t tacc = tmem_base + static_cast<uint32_t>(acc * BN) + (static_cast<uint32_t>(quad * 32) << 16);
      uint8_t* stage = s_stage + (warp - 2) * kStageWarpBytes;
      if (ph2) {
        epilogue_tile<MODE_DOWN, PAIR>(p2, tc, tacc, quad, part, lane, stage, shape);
      } else {
        epilogue_tile<MODE, PAIR>(p, tc, tacc, quad, part, lane, stage, shape);
        if constexpr (FUSED) {
          // publish this warp's h stores of the piece to the down tiles
          fence_proxy_async_global();
          __syncwarp();
          if (lane == 0) red_release_add(arrivals + tc.piece, 1);
        }
      }
      tc_fence_before_sync();
      if constexpr (PAIR == 2) mbar_arrive_cluster(map_to_rank(tempty0 + 8 * acc, 0));
      else mbar_arrive(tempty0 + 8 * acc);
    }
  }

  __syncthreads();
  griddep_launch_dependents();  // this CTA has no tiles left: the next kernel may begin launching
  if (threadIdx.x == 0 && *abort_flag) atomicOr(p.status, p.err_bit);
  if constexpr (PAIR == 2) {
    tc_fence_before_sync();
    cluster_sync();  // neither CTA leaves while the other may still signal it
  }
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    if constexpr (PAIR == 2) tmem_dealloc_pair(tmem_base, TMEM_COLS);
    else tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}

// The arguments of one encoding: a tensor map is a pure function of them, so
// an encoded map is reused while they are the same (the same buffers at the
// same shapes, call after call).
struct MapKey {
  const void* base;
  int rank;
  cuuint64_t dims[5];
  cuuint64_t strides[4];
  cuuint32_t box[5];
};

bool same_key(const MapKey& a, const MapKey& b) {
  if (a.base != b.base || a.rank != b.rank) return false;
  for (int i = 0; i < a.rank; ++i)
    if (a.dims[i] != b.dims[i] || a.box[i] != b.box[i]) return false;
  for (int i = 0; i + 1 < a.rank; ++i)
    if (a.strides[i] != b.strides[i]) return false;
  return true;
}

// A small per-thread cache of encoded maps, replaced round-robin.
constexpr int kMapCacheSize = 32;
struct MapCache {
  MapKey key[kMapCacheSize];
  CUtensorMap map[kMapCacheSize];
  int used = 0, next = 0;
};
thread_local MapCache t_maps;

bool encode_bf16_map(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims,
                     const cuuint64_t* strides_bytes, const cuuint32_t* box) {
  MapKey key = {};
  key.base = base;
  key.rank = rank;
  for (int i = 0; i < rank; ++i) {
    key.dims[i] = dims[i];
    key.box[i] = box[i];
  }
  for (int i = 0; i + 1 < rank; ++i) key.strides[i] = strides_bytes[i];
  MapCache& c = t_maps;
  for (int i = 0; i < c.used; ++i) {
    if (same_key(c.key[i], key)) {
      *map = c.map[i];
      return true;
    }
  }
  auto enc = encoder();
  if (enc == nullptr) return false;
  const cuuint32_t elem_strides[5] = {1, 1, 1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<cuuint32_t>(rank), const_cast<void*>(base),
                         dims, strides_bytes, box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  int slot;
  if (c.used < kMapCacheSize) {
    slot = c.used++;
  } else {
    slot = c.next;
    c.next = (c.next + 1) % kMapCacheSize;
  }
  c.key[slot] = key;
  c.map[slot] = *map;
  return true;
}

template <int PAIR>
constexpr size_t smem_bytes_for(int E) {
  return 1024 + static_cast<size_t>(Geo<PAIR>::STAGES) * Geo<PAIR>::STAGE_BYTES + CTRL_BYTES +
         2 * static_cast<size_t>(E + 1) * 4 + 16 + NUM_EPI_WARPS * kStageWarpBytes;
}

// Clusters of two of kernel `func` that can be resident at once, looked up
// once per device (occupancy depends on the device) and kernel.
int max_pair_clusters(const void* func, size_t smem, int num_sms) {
  struct Entry {
    int dev;
    const void* func;
    int n;
  };
  static std::mutex mu;
  static std::vector<Entry> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return num_sms / 2;
  std::lock_guard<std::mutex> lock(mu);
  for (const Entry& c : cache)
    if (c.dev == dev && c.func == func) return c.n;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(static_cast<unsigned>(num_sms & ~1));
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, func, &cfg) != cudaSuccess || n <= 0) return num_sms / 2;
  cache.push_back({dev, func, n});
  return n;
}

// The CTA-pair variant keeps the tensor pipe busier per clock (86-91% vs
// 76-79% of cycles on the Mixtral-shaped GEMMs) but these GEMMs run at the
// part's power limit, where it draws more power, runs at a lower clock and
// ends no faster; the single-CTA kernel is therefore the default.
// MOE_B200_CTA_PAIR=2 selects the pair variant (1 forces the default).
// One-copy B loads (default) or four 64-column copies per stage
// (MOE_B200_B_ONE_BOX=0).
// Row f1, the routed-row gather inside the gate_up GEMM
// (MOE_B200_FUSED_GATHER=1): the producer warp's lanes copy the tile's rows
// of x with tile::gather4 instead of a separate gather kernel writing the
// permuted copy Xp.  Single-CTA tiles only.
bool fused_gather_requested() { return switches().fused_gather; }

bool one_box_enabled() { return switches().b_one_box; }

int choose_pair(int /*R*/, int /*E*/) { return switches().cta_pair; }

template <int MODE, int PAIR, bool GATHER>
cudaError_t launch_with(const CUtensorMap& mapA, const CUtensorMap& mapB, const CUtensorMap& mapAh,
                        const GemmParams& p, int num_sms, cudaStream_t stream) {
  const int64_t max_pieces = p.R / Geo<PAIR>::PIECE + std::min(p.E, p.R);
  const int64_t max_tiles = max_pieces * p.n_tiles;
  const size_t smem = smem_bytes_for<PAIR>(p.E);
  cudaError_t err = opt_in_dynamic_smem(reinterpret_cast<const void*>(grouped_gemm_kernel<MODE, PAIR, false, GATHER>),
                                        static_cast<int>(smem_bytes_for<PAIR>(kMaxExperts)));
  if (err != cudaSuccess) return err;
  if constexpr (PAIR == 1) {
    const int grid = static_cast<int>(std::min<int64_t>(max_tiles, num_sms));
    grouped_gemm_kernel<MODE, 1, false, GATHER><<<grid, NUM_THREADS, smem, stream>>>(mapA, mapB, mapA, mapB, mapAh,
                                                                                      mapAh, p, p, nullptr, nullptr);
    return cudaGetLastError();
  } else {
    const int clusters = static_cast<int>(std::min<int64_t>(
        max_tiles, max_pair_clusters(reinterpret_cast<const void*>(grouped_gemm_kernel<MODE, 2, false, false>),
                                     smem_bytes_for<2>(kMaxExperts), num_sms)));
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters));
    cfg.blockDim = dim3(NUM_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // (the pair's tails of at most 128 rows copy 64 A rows per CTA through mapAh)
    return cudaLaunchKernelEx(&cfg, grouped_gemm_kernel<MODE, 2, false, false>, mapA, mapB, mapA, mapB, mapAh, mapAh, p,
                              p,
                              static_cast<int*>(nullptr), static_cast<int*>(nullptr));
  }
}

// Tensor maps and kernel parameters of one contraction.
// B tensor map that delivers a whole 64 K x 256 column stage tile in one copy:
// {64 columns, K, column blocks (, gate/up), E}, the column-block dimension
// 128 bytes apart, box {64, 64, blocks (, 2), 1}.  Its shared-memory image
// equals that of the four 64-column boxes of the plain view (the swizzle
// depends only on the shared address).  Requires the columns of one half to
// be a multiple of 64, so that every in-range coordinate stays inside the
// tensor; otherwise (or if the driver declines the view) false.
// `pair`: a CTA of a pair loads half of the 256 columns (2 blocks; the
// concatenated view then holds one of the gate/up halves per copy).
template <int MODE>
bool encode_one_box_b(const GroupedGemmArgs& a, CUtensorMap* map, bool pair) {
  const cuuint64_t H = a.H, D = a.D, E = a.E;
  if (MODE == MODE_GATE_UP_CONCAT) {
    if (D % 64 != 0) return false;
    const cuuint64_t dims[5] = {64, H, D / 64, 2, E};
    const cuuint64_t strides[4] = {2 * D * 2, 128, D * 2, H * 2 * D * 2};
    // one CTA: both 64-column blocks of the gate half, then of the up half;
    // a CTA of a pair: the gate and the up block of its 64 h columns
    const cuuint32_t box[5] = {64, BK, pair ? 1u : 2u, 2, 1};
    return encode_bf16_map(map, a.W, 5, dims, strides, box);
  } else if (MODE == MODE_GATE_UP_INTERLEAVED) {
    if ((2 * D) % 64 != 0) return false;
    const cuuint64_t dims[4] = {64, H, 2 * D / 64, E};
    const cuuint64_t strides[3] = {2 * D * 2, 128, H * 2 * D * 2};
    const cuuint32_t box[4] = {64, BK, pair ? 2u : 4u, 1};
    return encode_bf16_map(map, a.W, 4, dims, strides, box);
  } else {
    if (H % 64 != 0) return false;
    const cuuint64_t dims[4] = {64, D, H / 64, E};
    const cuuint64_t strides[3] = {H * 2, 128, D * H * 2};
    const cuuint32_t box[4] = {64, BK, pair ? 2u : 4u, 1};
    return encode_bf16_map(map, a.W, 4, dims, strides, box);
  }
}

template <int MODE>
cudaError_t prepare(const GroupedGemmArgs& a, CUtensorMap& mapA, CUtensorMap& mapAh, CUtensorMap& mapB, GemmParams& p,
                    bool pair) {
  const bool down = MODE == MODE_DOWN;
  const int K = down ? a.D : a.H;
  if (!down && a.gather) {
    // rows of x gathered by token index: one-row boxes, four rows per tile::gather4
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(a.T)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
    const cuuint32_t box[2] = {64, 1};
    if (!encode_bf16_map(&mapA, a.A, 2, dims, strides, box)) return cudaErrorInvalidValue;
    mapAh = mapA;
  } else {
    // with a_direct the A operand is x: T rows, indexed by the row within an expert
    const cuuint64_t rows = static_cast<cuuint64_t>(!down && a.a_direct ? a.T : a.R);
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), rows};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
    const cuuint32_t box[2] = {64, BM};
    if (!encode_bf16_map(&mapA, a.A, 2, dims, strides, box)) return cudaErrorInvalidValue;
    const cuuint32_t half_box[2] = {64, HALF_ROWS};
    if (!encode_bf16_map(&mapAh, a.A, 2, dims, strides, half_box)) return cudaErrorInvalidValue;
  }
  const cuuint64_t H = a.H, D = a.D, E = a.E;
  p.b_one_box = one_box_enabled() && encode_one_box_b<MODE>(a, &mapB, pair) ? 1 : 0;
  // Test hook for the single launch's bounded cross-CTA wait:
  // MOE_B200_TEST_STALL_DOWN_TILES_MS=<ms> makes every down tile wait for one
  // arrival more than will ever come, giving up after <ms>; the launch then
  // records MOE_DEVICE_ERR_TIMEOUT_GEMM1 | _GEMM2 and ends normally.
  p.extra_arrivals = 0;
  p.dep_timeout_ns = kTimeoutNs;
  if (const long ms = switches().test_stall_down_ms; ms > 0) {
    p.extra_arrivals = 1;
    p.dep_timeout_ns = static_cast<unsigned long long>(std::min(ms, 2000L)) * 1000000ull;
  }
  if (p.b_one_box) {
    // mapB already holds the one-copy view
  } else if (MODE == MODE_GATE_UP_CONCAT) {
    const cuuint64_t dims[4] = {D, 2, H, E};
    const cuuint64_t strides[3] = {D * 2, 2 * D * 2, H * 2 * D * 2};
    const cuuint32_t box[4] = {64, 1, BK, 1};
    if (!encode_bf16_map(&mapB, a.W, 4, dims, strides, box)) return cudaErrorInvalidValue;
  } else if (MODE == MODE_GATE_UP_INTERLEAVED) {
    const cuuint64_t dims[3] = {2 * D, H, E};
    const cuuint64_t strides[2] = {2 * D * 2, H * 2 * D * 2};
    const cuuint32_t box[3] = {64, BK, 1};
    if (!encode_bf16_map(&mapB, a.W, 3, dims, strides, box)) return cudaErrorInvalidValue;
  } else {
    const cuuint64_t dims[3] = {H, D, E};
    const cuuint64_t strides[2] = {H * 2, D * H * 2};
    const cuuint32_t box[3] = {64, BK, 1};
    if (!encode_bf16_map(&mapB, a.W, 3, dims, strides, box)) return cudaErrorInvalidValue;
  }
  p.offsets = a.offsets;
  p.a_direct = !down && a.a_direct ? 1 : 0;
  p.k = a.k;
  p.perm = a.perm;
  p.weights = a.weights;
  p.bias = a.bias;
  p.out = a.out;
  p.status = a.status;
  p.E = a.E;
  p.R = a.R;
  p.H = a.H;
  p.D = a.D;
  p.n_tiles = down ? (a.H + BN - 1) / BN : (a.D + 127) / 128;
  p.num_kb = (K + BK - 1) / BK;
  p.activation = a.activation;
  p.alpha = a.alpha;
  p.limit = a.limit;
  p.err_bit = down ? MOE_DEVICE_ERR_TIMEOUT_GEMM2 : MOE_DEVICE_ERR_TIMEOUT_GEMM1;
  return cudaSuccess;
}

template <int MODE>
cudaError_t launch_mode(const GroupedGemmArgs& a, cudaStream_t stream) {
  if (a.R == 0) return cudaSuccess;
  CUtensorMap mapA, mapAh, mapB;
  GemmParams p;
  const int pair = choose_pair(a.R, a.E);
  cudaError_t err = prepare<MODE>(a, mapA, mapAh, mapB, p, pair == 2);
  if (err != cudaSuccess) return err;
  if (pair == 2) return launch_with<MODE, 2, false>(mapA, mapB, mapAh, p, a.num_sms, stream);
  if constexpr (MODE != MODE_DOWN) {
    if (a.gather) return launch_with<MODE, 1, true>(mapA, mapB, mapAh, p, a.num_sms, stream);
  }
  return launch_with<MODE, 1, false>(mapA, mapB, mapAh, p, a.num_sms, stream);
}

// Rows per expert at which one bf16 weight byte carries as many FLOPs (2 per
// row per 2-byte weight) as the B200's measured bf16 peak per HBM byte
// (about 1.66 PFLOP/s over 6.5 TB/s).
constexpr int64_t kRidgeRowsPerExpert = 256;

template <int MODE, bool GATHER>
cudaError_t launch_fused(const GroupedGemmArgs& up, const GroupedGemmArgs& down, int* arrivals,
                         cudaStream_t stream) {
  if (up.R == 0) return cudaSuccess;
  CUtensorMap mapA, mapAh, mapB, mapA2, mapA2h, mapB2;
  GemmParams p, p2;
  cudaError_t err = prepare<MODE>(up, mapA, mapAh, mapB, p, false);
  if (err != cudaSuccess) return err;
  err = prepare<MODE_DOWN>(down, mapA2, mapA2h, mapB2, p2, false);
  if (err != cudaSuccess) return err;
  // a timeout anywhere in the fused launch is reported as both stages'
  p.err_bit = p2.err_bit = MOE_DEVICE_ERR_TIMEOUT_GEMM1 | MOE_DEVICE_ERR_TIMEOUT_GEMM2;
  const int64_t max_pieces = p.R / BM + std::min(p.E, p.R);
  const int64_t max_tiles = max_pieces * (p.n_tiles + p2.n_tiles);
  const size_t smem = smem_bytes_for<1>(p.E);
  err = opt_in_dynamic_smem(reinterpret_cast<const void*>(grouped_gemm_kernel<MODE, 1, true, GATHER>),
                            static_cast<int>(smem_bytes_for<1>(kMaxExperts)));
  if (err != cudaSuccess) return err;
  // Cooperative: the launch fails rather than run with CTAs that are not
  // resident, on which a down tile's wait could otherwise depend.  With
  // programmatic serialization (default) its CTAs may start while the gather
  // drains: barrier set-up and TMEM allocation overlap it, and every global
  // read waits in griddep_wait.
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(static_cast<unsigned>(std::min<int64_t>(max_tiles, up.num_sms)));
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() && switches().pdl_coop ? 2 : 1;
  // The last counter is the tile scheduler's (pieces use the ones before it).
  // Dynamic order pays where the weights stream from HBM (rows per expert
  // below the bf16 ridge point of about 256 FLOP/byte), the static order
  // where the tensor pipe bounds the launch; MOE_B200_TILE_SCHEDULE=dynamic
  // or =static overrides the choice.
  bool dynamic = up.R < kRidgeRowsPerExpert * up.E;
  if (switches().tile_schedule == 'd') dynamic = true;
  if (switches().tile_schedule == 's') dynamic = false;
  int* sched = dynamic ? arrivals + mega_ffn_counters(up.R, up.E) - 1 : nullptr;
  return cudaLaunchKernelEx(&cfg, grouped_gemm_kernel<MODE, 1, true, GATHER>, mapA, mapB, mapA2, mapB2, mapAh, mapA2h, p,
                            p2,
                            arrivals, sched);
}

// Both contractions in one launch on CTA pairs (tcgen05 cta_group::2):
// 256-row pieces, each CTA of a pair copying its rows of A and its half of
// B, static tile order.  Cooperative and clustered: the launch fails rather
// than run with clusters that are not all resident.
template <int MODE>
cudaError_t launch_fused_pair(const GroupedGemmArgs& up, const GroupedGemmArgs& down, int* arrivals,
                              cudaStream_t stream) {
  if (up.R == 0) return cudaSuccess;
  CUtensorMap mapA, mapAh, mapB, mapA2, mapA2h, mapB2;
  GemmParams p, p2;
  cudaError_t err = prepare<MODE>(up, mapA, mapAh, mapB, p, true);
  if (err != cudaSuccess) return err;
  err = prepare<MODE_DOWN>(down, mapA2, mapA2h, mapB2, p2, true);
  if (err != cudaSuccess) return err;
  p.err_bit = p2.err_bit = MOE_DEVICE_ERR_TIMEOUT_GEMM1 | MOE_DEVICE_ERR_TIMEOUT_GEMM2;
  const int64_t max_pieces = p.R / Geo<2>::PIECE + std::min(p.E, p.R);
  const int64_t max_tiles = max_pieces * (p.n_tiles + p2.n_tiles);
  const size_t smem = smem_bytes_for<2>(p.E);
  const void* kernel = reinterpret_cast<const void*>(grouped_gemm_kernel<MODE, 2, true, false>);
  err = opt_in_dynamic_smem(kernel, static_cast<int>(smem_bytes_for<2>(kMaxExperts)));
  if (err != cudaSuccess) return err;
  const int clusters = static_cast<int>(
      std::min<int64_t>(max_tiles, max_pair_clusters(kernel, smem_bytes_for<2>(kMaxExperts), up.num_sms)));
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[3];
  int n = 0;
  attr[n].id = cudaLaunchAttributeClusterDimension;
  attr[n].val.clusterDim.x = 2;
  attr[n].val.clusterDim.y = 1;
  attr[n].val.clusterDim.z = 1;
  ++n;
  if (switches().pair_coop) {
    attr[n].id = cudaLaunchAttributeCooperative;
    attr[n].val.cooperative = 1;
    ++n;
  }
  if (pdl_enabled() && switches().pdl_coop) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters));
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, grouped_gemm_kernel<MODE, 2, true, false>, mapA, mapB, mapA2, mapB2, mapAh,
                            mapA2h, p, p2, arrivals, static_cast<int*>(nullptr));
}

}  // namespace

bool tensor_map_encoder_available() { return encoder() != nullptr; }

bool fused_gather_enabled() { return fused_gather_requested() && choose_pair(0, 0) == 1; }

cudaError_t launch_gemm_gate_up(const GroupedGemmArgs& a, cudaStream_t stream) {
  return a.gate_up_format == 0 ? launch_mode<MODE_GATE_UP_CONCAT>(a, stream)
                               : launch_mode<MODE_GATE_UP_INTERLEAVED>(a, stream);
}

cudaError_t launch_gemm_down(const GroupedGemmArgs& a, cudaStream_t stream) {
  return launch_mode<MODE_DOWN>(a, stream);
}

int mega_ffn_counters(int R, int E) { return R / BM + std::min(E, R) + 1; }

cudaError_t launch_mega_ffn(const GroupedGemmArgs& up, const GroupedGemmArgs& down, int* arrivals,
                            cudaStream_t stream) {
  if (up.gather)
    return up.gate_up_format == 0 ? launch_fused<MODE_GATE_UP_CONCAT, true>(up, down, arrivals, stream)
                                  : launch_fused<MODE_GATE_UP_INTERLEAVED, true>(up, down, arrivals, stream);
  if (choose_pair(up.R, up.E) == 2)
    return up.gate_up_format == 0 ? launch_fused_pair<MODE_GATE_UP_CONCAT>(up, down, arrivals, stream)
                                  : launch_fused_pair<MODE_GATE_UP_INTERLEAVED>(up, down, arrivals, stream);
  return up.gate_up_format == 0 ? launch_fused<MODE_GATE_UP_CONCAT, false>(up, down, arrivals, stream)
                                : launch_fused<MODE_GATE_UP_INTERLEAVED, false>(up, down, arrivals, stream);
}

}  // namespace moe
