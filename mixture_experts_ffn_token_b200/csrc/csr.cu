// csr.cu -- stage 2 (moe_create_indices) plus the two bandwidth kernels
// around the grouped GEMMs (row gather and the k-way combine).
//
// moe_create_indices is named on the Mojo sink_gate_router_kernel page as the
// separate bucketing step (it needs every token's assignment, a grid-wide
// dependency); its outputs follow NeMo _permute_tokens_for_grouped_mm: the
// routed slots sorted by expert, the per-expert counts and their cumulative
// offsets.  Here the sort is a stable counting sort in three kernels:
//   count   each CTA histograms one chunk of 2048 slots in shared memory;
//   scan    one CTA turns the chunk histograms into per-expert offsets and
//           per-(chunk, expert) base positions;
//   scatter each CTA walks its chunk in slot order: every warp owns 128
//           consecutive slots, __match_any_sync groups equal experts inside a
//           32-slot step, a per-warp count table (scanned across warps) gives
//           the position of each slot, so the order inside an expert is the
//           slot order and no atomic decides any position.
#include <algorithm>
#include <cstdlib>
#include <mutex>
#include <vector>

#include "kernels.cuh"

namespace moe {
namespace {

constexpr int kCsrWarps = kCsrThreads / 32;
constexpr int kSlotsPerWarp = kCsrChunk / kCsrWarps;  // 128
static_assert(kSlotsPerWarp % 32 == 0, "slots per warp must be whole warp steps");

// A slot takes part unless its token is masked out (mask may be null).
__device__ __forceinline__ bool slot_live(const uint8_t* mask, int64_t s, int k) {
  return mask == nullptr || mask[s / k] != 0;
}

__global__ void __launch_bounds__(kCsrThreads) csr_count_kernel(const int32_t* __restrict__ idx, int R, int E,
                                                                int32_t* __restrict__ chunk_counts, int* status,
                                                                const uint8_t* __restrict__ mask, int k) {
  griddep_wait();  // the previous kernel's results are complete and visible
  griddep_launch_dependents();
  extern __shared__ int cnt[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kCsrChunk;
  const int64_t end = min(base + kCsrChunk, static_cast<int64_t>(R));
  // all of this thread's slots are loaded before the first is counted
  constexpr int kPerThread = kCsrChunk / kCsrThreads;
  int ev[kPerThread];
  uint32_t live = 0;  // bit q: slot q of this thread exists and its token is not masked
#pragma unroll
  for (int q = 0; q < kPerThread; ++q) {
    const int64_t s = base + threadIdx.x + static_cast<int64_t>(q) * kCsrThreads;
    const bool on = s < end && slot_live(mask, s, k);
    ev[q] = on ? idx[s] : 0;
    live |= on ? (1u << q) : 0u;
  }
  bool bad = false;
#pragma unroll
  for (int q = 0; q < kPerThread; ++q) {
    if (!((live >> q) & 1u)) continue;
    const int e = ev[q];
    if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
    else bad = true;
  }
  if (bad) atomicOr(status, MOE_DEVICE_ERR_EXPERT_INDEX);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) chunk_counts[static_cast<int64_t>(blockIdx.x) * E + e] = cnt[e];
}

// One CTA of 1024 threads; thread e owns expert e (E <= 1024).
__global__ void __launch_bounds__(1024) csr_scan_kernel(const int32_t* __restrict__ chunk_counts, int nchunks, int E,
                                                        int32_t* __restrict__ chunk_base,
                                                        int32_t* __restrict__ offsets) {
  griddep_wait();  // the previous kernel's results are complete and visible
  griddep_launch_dependents();
  __shared__ int warp_tot[32];
  const int e = threadIdx.x;
  const int lane = e & 31, warp = e >> 5;
  int total = 0;
  if (e < E) {
    for (int c = 0; c < nchunks; ++c) {
      const int64_t i = static_cast<int64_t>(c) * E + e;
      const int v = chunk_counts[i];
      chunk_base[i] = total;
      total += v;
    }
  }
  // exclusive scan of `total` over experts
  int incl = total;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int v = warp_tot[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, v, off);
      if (lane >= off) v += y;
    }
    warp_tot[lane] = v;  // inclusive prefix of warp totals
  }
  __syncthreads();
  const int excl = incl - total + (warp > 0 ? warp_tot[warp - 1] : 0);
  if (e < E) {
    offsets[e] = excl;
    for (int c = 0; c < nchunks; ++c) chunk_base[static_cast<int64_t>(c) * E + e] += excl;
  }
  if (e == E - 1) offsets[E] = excl + total;
}

__global__ void __launch_bounds__(kCsrThreads) csr_scatter_kernel(const int32_t* __restrict__ idx, int R, int E,
                                                                  const int32_t* __restrict__ chunk_base,
                                                                  int32_t* __restrict__ perm,
                                                                  int32_t* __restrict__ inv,
                                                                  const uint8_t* __restrict__ mask, int k) {
  griddep_wait();  // the previous kernel's results are complete and visible
  griddep_launch_dependents();
  extern __shared__ int wcnt[];  // [kCsrWarps][E]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < kCsrWarps * E; i += blockDim.x) wcnt[i] = 0;
  __syncthreads();
  const int64_t wbase = static_cast<int64_t>(blockIdx.x) * kCsrChunk + static_cast<int64_t>(warp) * kSlotsPerWarp;
  int* my = wcnt + warp * E;
  const uint32_t lt_mask = (1u << lane) - 1u;
  // this lane's slots, loaded once for both passes
  constexpr int kRounds = kSlotsPerWarp / 32;
  int ev[kRounds];
#pragma unroll
  for (int q = 0; q < kRounds; ++q) {
    const int64_t s = wbase + 32 * q + lane;
    ev[q] = s < R && slot_live(mask, s, k) ? idx[s] : -1;
  }
  // pass 1: per-warp histogram
#pragma unroll
  for (int q = 0; q < kRounds; ++q) {
    const int e = ev[q];
    const bool ok = e >= 0 && e < E;
    const uint32_t peers = __match_any_sync(0xffffffffu, ok ? e : E + lane);
    if (ok && (peers & lt_mask) == 0) my[e] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // exclusive scan over warps, per expert
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
    for (int w = 0; w < kCsrWarps; ++w) {
      const int v = wcnt[w * E + e];
      wcnt[w * E + e] = run;
      run += v;
    }
  }
  __syncthreads();
  // pass 2: positions in slot order
  const int32_t* cb = chunk_base + static_cast<int64_t>(blockIdx.x) * E;
#pragma unroll
  for (int q = 0; q < kRounds; ++q) {
    const int64_t s = wbase + 32 * q + lane;
    const int e = ev[q];
    const bool ok = e >= 0 && e < E;
    const uint32_t peers = __match_any_sync(0xffffffffu, ok ? e : E + lane);
    int base = 0;
    if (ok) base = cb[e] + my[e];
    __syncwarp();
    if (ok) {
      const int pos = base + __popc(peers & lt_mask);
      perm[pos] = static_cast<int32_t>(s);
      if (inv != nullptr) inv[s] = pos;
      if ((peers & lt_mask) == 0) my[e] += __popc(peers);
    }
    __syncwarp();
  }
}

// The whole counting sort in ONE cooperative launch, one CTA per chunk of
// kCsrChunk slots (used when the chunks fit on the GPU at once): each CTA
// builds the per-warp histograms of its chunk and publishes the chunk's
// counts; after a grid barrier every CTA reduces the (chunk x expert) count
// table itself -- it is small -- to the expert offsets and its own chunk's
// base positions, then places its slots exactly as csr_scatter_kernel does.
// The result is bit-identical to the three-kernel form.  *barrier must be
// zero at launch (the router kernel clears it, or the host); the wait is
// bounded (timeout_ns, and an iteration cap) and records
// MOE_DEVICE_ERR_TIMEOUT_CSR when it gives up, after which the CTA returns
// without writing offsets or positions.
constexpr uint64_t kCsrBarrierTimeoutNs = 1000000000ull;  // 1 s: far beyond any legitimate wait

__global__ void __launch_bounds__(kCsrThreads) csr_fused_kernel(const int32_t* __restrict__ idx, int R, int E,
                                                                int32_t* __restrict__ chunk_counts,
                                                                int32_t* __restrict__ offsets,
                                                                int32_t* __restrict__ perm, int32_t* __restrict__ inv,
                                                                int* status, int* barrier,
                                                                const uint8_t* __restrict__ mask, int k,
                                                                int extra_arrivals, unsigned long long timeout_ns) {
  griddep_wait();  // the previous kernel's results are complete and visible
  extern __shared__ int sm[];
  int* wcnt = sm;                  // [kCsrWarps][E]: per-warp counts, then their exclusive prefix over warps
  int* cb = sm + kCsrWarps * E;    // [E]: this chunk's first position per expert
  __shared__ int warp_tot[kCsrWarps];
  __shared__ int s_go;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < kCsrWarps * E; i += blockDim.x) wcnt[i] = 0;
  __syncthreads();
  const int64_t wbase = static_cast<int64_t>(blockIdx.x) * kCsrChunk + static_cast<int64_t>(warp) * kSlotsPerWarp;
  int* my = wcnt + warp * E;
  const uint32_t lt_mask = (1u << lane) - 1u;
  constexpr int kRounds = kSlotsPerWarp / 32;
  int ev[kRounds];
  bool bad = false;
#pragma unroll
  for (int q = 0; q < kRounds; ++q) {
    const int64_t s = wbase + 32 * q + lane;
    int e = -1;
    if (s < R && slot_live(mask, s, k)) {
      e = idx[s];
      if (e < 0 || e >= E) {
        bad = true;
        e = -1;
      }
    }
    ev[q] = e;
  }
  if (bad) atomicOr(status, MOE_DEVICE_ERR_EXPERT_INDEX);
  // per-warp histogram of the chunk
#pragma unroll
  for (int q = 0; q < kRounds; ++q) {
    const int e = ev[q];
    const uint32_t peers = __match_any_sync(0xffffffffu, e >= 0 ? e : E + lane);
    if (e >= 0 && (peers & lt_mask) == 0) my[e] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // exclusive prefix over warps per expert; the chunk's count is the total
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
    for (int w = 0; w < kCsrWarps; ++w) {
      const int v = wcnt[w * E + e];
      wcnt[w * E + e] = run;
      run += v;
    }
    chunk_counts[static_cast<int64_t>(blockIdx.x) * E + e] = run;
  }
  __syncthreads();
  // grid barrier: every chunk's counts are published before any CTA reads them
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(barrier, 1);
    const int target = static_cast<int>(gridDim.x) + extra_arrivals;
    bool ok = ld_acquire_gpu(barrier) >= target;
    if (!ok) {
      const uint64_t t0 = global_timer_ns();
      for (uint32_t it = 1; it < (1u << 26) && !ok; ++it) {
        __nanosleep(32);
        ok = ld_acquire_gpu(barrier) >= target;
        if (!ok && (it & 15u) == 0 && global_timer_ns() - t0 > timeout_ns) break;
      }
    }
    if (!ok) atomicOr(status, MOE_DEVICE_ERR_TIMEOUT_CSR);
    __threadfence();
    s_go = ok ? 1 : 0;
  }
  __syncthreads();
  if (!s_go) return;
  // every CTA: per expert, the slots of earlier chunks and the total; an
  // exclusive scan of the totals over experts gives the offsets (thread i
  // owns experts 2i and 2i+1)
  const int nchunks = static_cast<int>(gridDim.x);
  const int e0 = 2 * threadIdx.x, e1 = e0 + 1;
  int before0 = 0, before1 = 0, tot0 = 0, tot1 = 0;
  for (int c = 0; c < nchunks; ++c) {
    const int32_t* row = chunk_counts + static_cast<int64_t>(c) * E;
    const int v0 = e0 < E ? row[e0] : 0;
    const int v1 = e1 < E ? row[e1] : 0;
    if (c < static_cast<int>(blockIdx.x)) {
      before0 += v0;
      before1 += v1;
    }
    tot0 += v0;
    tot1 += v1;
  }
  const int local = tot0 + tot1;
  int incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int v = lane < kCsrWarps ? warp_tot[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, v, off);
      if (lane >= off) v += y;
    }
    if (lane < kCsrWarps) warp_tot[lane] = v;  // inclusive prefix of warp totals
  }
  __syncthreads();
  const int excl = incl - local + (warp > 0 ? warp_tot[warp - 1] : 0);
  if (e0 < E) {
    cb[e0] = excl + before0;
    if (blockIdx.x == 0) offsets[e0] = excl;
  }
  if (e1 < E) {
    cb[e1] = excl + tot0 + before1;
    if (blockIdx.x == 0) offsets[e1] = excl + tot0;
  }
  if (blockIdx.x == 0 && (e0 == E - 1 || e1 == E - 1)) offsets[E] = excl + local;
  __syncthreads();
  griddep_launch_dependents();
  // positions in slot order (as csr_scatter_kernel)
#pragma unroll
  for (int q = 0; q < kRounds; ++q) {
    const int64_t s = wbase + 32 * q + lane;
    const int e = ev[q];
    const uint32_t peers = __match_any_sync(0xffffffffu, e >= 0 ? e : E + lane);
    int base = 0;
    if (e >= 0) base = cb[e] + my[e];
    __syncwarp();
    if (e >= 0) {
      const int pos = base + __popc(peers & lt_mask);
      perm[pos] = static_cast<int32_t>(s);
      if (inv != nullptr) inv[s] = pos;
      if ((peers & lt_mask) == 0) my[e] += __popc(peers);
    }
    __syncwarp();
  }
}

}  // namespace

bool pdl_enabled() { return switches().pdl; }

cudaError_t opt_in_dynamic_smem(const void* func, int bytes) {
  struct Done {
    int dev;
    const void* func;
  };
  static std::mutex mu;
  static std::vector<Done> done;  // successful opt-ins only: a failure is retried
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  std::lock_guard<std::mutex> lock(mu);
  for (const Done& d : done)
    if (d.dev == dev && d.func == func) return cudaSuccess;
  err = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (err == cudaSuccess) done.push_back({dev, func});
  return err;
}

namespace {

constexpr int kCombineBatch = 8;   // rows a combine thread loads before summing
constexpr int kGatherUnroll = 4;   // 16-byte chunks a gather lane loads before storing

// One warp per gathered row: Xp[p, :] = x[perm[p] / k, :] (times
// scale[perm[p]] when scale is given), 16-byte vectors.
__global__ void __launch_bounds__(256) gather_rows_kernel(const __nv_bfloat16* __restrict__ x,
                                                          const int32_t* __restrict__ perm,
                                                          const int32_t* __restrict__ offsets, int E, int R, int k,
                                                          int H, const float* __restrict__ scale,
                                                          __nv_bfloat16* __restrict__ Xp, int* status,
                                                          int* __restrict__ zero, int n_zero) {
  griddep_wait();  // the previous kernel's results are complete and visible
  griddep_launch_dependents();
  // Clear the caller's counters (the single-launch FFN's per-piece arrival
  // counts) for the kernel that follows on the stream.
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_zero; i += gridDim.x * blockDim.x) zero[i] = 0;
  int total = offsets[E];
  if (total < 0 || total > R) {
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(status, MOE_DEVICE_ERR_CSR);
    total = total < 0 ? 0 : R;
  }
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int vec = H / 8;
  // The gathered rows stream through L2 (201 MB on the sink-shaped layer)
  // while every row of x is read k times in an order set by the experts: the
  // rows are stored as the first candidates for replacement, so that x stays
  // in L2 between its reads (sink: gather 46.0 -> 43.6 us, the FFN that
  // reads the rows unchanged).
  const uint64_t pol_first = l2_policy_evict_first();
  for (int64_t p = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; p < total; p += nwarps) {
    const int s = perm[p];
    if (s < 0 || s >= R) {
      if (lane == 0) atomicOr(status, MOE_DEVICE_ERR_CSR);
      continue;
    }
    const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(s / k) * H);
    uint4* dst = reinterpret_cast<uint4*>(Xp + p * H);
    // apply_router_weight_first: the routing weight scales the expert input
    const float f = scale != nullptr ? scale[s] : 1.f;
    // kGatherUnroll chunks per lane in flight before their stores
    for (int c0 = lane; c0 < vec; c0 += 32 * kGatherUnroll) {
      uint4 v[kGatherUnroll];
#pragma unroll
      for (int q = 0; q < kGatherUnroll; ++q)
        if (c0 + 32 * q < vec) v[q] = __ldg(src + c0 + 32 * q);
#pragma unroll
      for (int q = 0; q < kGatherUnroll; ++q) {
        if (c0 + 32 * q < vec) {
          uint4 o = v[q];
          if (scale != nullptr) {
            o.x = pack_bf16x2(bf16_lo(o.x) * f, bf16_hi(o.x) * f);
            o.y = pack_bf16x2(bf16_lo(o.y) * f, bf16_hi(o.y) * f);
            o.z = pack_bf16x2(bf16_lo(o.z) * f, bf16_hi(o.z) * f);
            o.w = pack_bf16x2(bf16_lo(o.w) * f, bf16_hi(o.w) * f);
          }
          st_v4_policy(dst + c0 + 32 * q, o, pol_first);
        }
      }
    }
  }
}

// out[t, :] = sum_j Y[t*k + j, :] (+ sum_i Ys[t*Ns + i, :] for shared
// experts) in fp32, j then i ascending, rounded to bf16; a masked token's row
// is zero.
__global__ void __launch_bounds__(256) combine_kernel(const __nv_bfloat16* __restrict__ Y, int T, int H, int k,
                                                      const __nv_bfloat16* __restrict__ Ys, int Ns,
                                                      const uint8_t* __restrict__ mask,
                                                      __nv_bfloat16* __restrict__ out) {
  griddep_wait();  // the previous kernel's results are complete and visible
  griddep_launch_dependents();
  const int vec = H / 8;
  const int64_t n = static_cast<int64_t>(T) * vec;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / vec;
    const int c = static_cast<int>(i - t * vec);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (mask == nullptr || mask[t] != 0) {
      const int terms = k + Ns;
      // up to kCombineBatch rows in flight per thread: all loads of a batch
      // are issued before the first add (the sum order stays j ascending)
      for (int j0 = 0; j0 < terms; j0 += kCombineBatch) {
        uint4 v[kCombineBatch];
#pragma unroll
        for (int q = 0; q < kCombineBatch; ++q) {
          const int j = j0 + q;
          if (j < terms) {
            const __nv_bfloat16* row = j < k ? Y + (t * k + j) * H : Ys + (t * Ns + (j - k)) * H;
            v[q] = __ldg(reinterpret_cast<const uint4*>(row) + c);
          }
        }
#pragma unroll
        for (int q = 0; q < kCombineBatch; ++q) {
          if (j0 + q < terms) {
            const uint32_t w[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
            for (int r = 0; r < 4; ++r) {
              acc[2 * r] += bf16_lo(w[r]);
              acc[2 * r + 1] += bf16_hi(w[r]);
            }
          }
        }
      }
    }
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    reinterpret_cast<uint4*>(out + t * H)[c] = o;
  }
}

// Shared experts as a grouped problem: expert i's segment is every token in
// order, offsets[i] = i*T, and row i*T + t is slot t*Ns + i of the [T, Ns]
// slot space (so slot / Ns is the token and the gates are indexed by slot).
__global__ void __launch_bounds__(256) shared_index_kernel(int T, int Ns, int32_t* __restrict__ offsets,
                                                           int32_t* __restrict__ perm, int* __restrict__ zero,
                                                           int n_zero) {
  griddep_wait();  // the previous kernel's results are complete and visible
  griddep_launch_dependents();
  // clear the shared pass's counters when it has no gather to do it
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_zero; i += gridDim.x * blockDim.x) zero[i] = 0;
  const int64_t n = static_cast<int64_t>(T) * Ns;
  for (int64_t p = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; p < n;
       p += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t i = p / T, t = p - i * T;
    perm[p] = static_cast<int32_t>(t * Ns + i);
  }
  if (blockIdx.x == 0 && threadIdx.x <= Ns) offsets[threadIdx.x] = threadIdx.x * T;
}

}  // namespace

cudaError_t launch_shared_index(int T, int Ns, int32_t* offsets, int32_t* perm, int num_sms, cudaStream_t stream,
                                int* zero, int n_zero) {
  const int64_t n = static_cast<int64_t>(T) * Ns;
  const int blocks = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((n + 255) / 256, num_sms * 4)));
  return launch_pdl(shared_index_kernel, dim3(blocks), dim3(256), 0, stream, T, Ns, offsets, perm, zero, n_zero);
}

cudaError_t launch_csr_count(const int32_t* idx, int R, int E, int32_t* chunk_counts, int* status,
                             const uint8_t* mask, int k, cudaStream_t stream) {
  const int nchunks = csr_num_chunks(R);
  if (nchunks == 0) return cudaSuccess;
  return launch_pdl(csr_count_kernel, dim3(nchunks), dim3(kCsrThreads), E * sizeof(int), stream, idx, R, E,
                    chunk_counts, status, mask, k);
}

cudaError_t launch_csr_scan(const int32_t* chunk_counts, int nchunks, int E, int32_t* chunk_base, int32_t* offsets,
                            cudaStream_t stream) {
  return launch_pdl(csr_scan_kernel, dim3(1), dim3(1024), 0, stream, chunk_counts, nchunks, E, chunk_base, offsets);
}

cudaError_t launch_csr_scatter(const int32_t* idx, int R, int E, const int32_t* chunk_base, int32_t* perm,
                               int32_t* inv, const uint8_t* mask, int k, cudaStream_t stream) {
  const int nchunks = csr_num_chunks(R);
  if (nchunks == 0) return cudaSuccess;
  const size_t smem = static_cast<size_t>(kCsrWarps) * E * sizeof(int);
  if (smem > 48 * 1024) {
    // once per device, for the largest expert count
    cudaError_t err = opt_in_dynamic_smem(reinterpret_cast<const void*>(csr_scatter_kernel),
                                          static_cast<int>(static_cast<size_t>(kCsrWarps) * kMaxExperts * sizeof(int)));
    if (err != cudaSuccess) return err;
  }
  return launch_pdl(csr_scatter_kernel, dim3(nchunks), dim3(kCsrThreads), smem, stream, idx, R, E, chunk_base, perm,
                    inv, mask, k);
}

bool csr_fused_enabled(int R, int num_sms) {
  if (!switches().csr_fused) return false;
  const int n = csr_num_chunks(R);
  return n > 0 && n <= num_sms;
}

cudaError_t launch_csr_fused(const int32_t* idx, int R, int E, int32_t* chunk_counts, int32_t* offsets, int32_t* perm,
                             int32_t* inv, int* status, int* barrier, const uint8_t* mask, int k,
                             cudaStream_t stream) {
  const int nchunks = csr_num_chunks(R);
  if (nchunks == 0) return cudaSuccess;
  const size_t smem = (static_cast<size_t>(kCsrWarps) + 1) * E * sizeof(int);
  if (smem > 48 * 1024) {
    // once per device, for the largest expert count
    cudaError_t err = opt_in_dynamic_smem(reinterpret_cast<const void*>(csr_fused_kernel),
                                          static_cast<int>((static_cast<size_t>(kCsrWarps) + 1) * kMaxExperts *
                                                           sizeof(int)));
    if (err != cudaSuccess) return err;
  }
  // cooperative: the launch fails rather than run CTAs that are not all
  // resident, which the grid barrier needs; with programmatic serialization
  // its CTAs may start while the router drains (they wait in griddep_wait)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(nchunks));
  cfg.blockDim = dim3(kCsrThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() && switches().pdl_coop ? 2 : 1;
  // Test hook for the bounded grid barrier: MOE_B200_TEST_STALL_CSR_MS=<ms>
  // makes every CTA wait for one arrival more than will ever come, giving
  // up after <ms>; the launch then records MOE_DEVICE_ERR_TIMEOUT_CSR and
  // ends normally.
  int extra = 0;
  unsigned long long timeout_ns = kCsrBarrierTimeoutNs;
  if (const long ms = switches().test_stall_csr_ms; ms > 0) {
    extra = 1;
    timeout_ns = static_cast<unsigned long long>(std::min(ms, 1000L)) * 1000000ull;
  }
  return cudaLaunchKernelEx(&cfg, csr_fused_kernel, idx, R, E, chunk_counts, offsets, perm, inv, status, barrier, mask,
                            k, extra, timeout_ns);
}

cudaError_t launch_gather(const __nv_bfloat16* x, const int32_t* perm, const int32_t* offsets, int E, int R, int k,
                          int H, const float* scale, __nv_bfloat16* Xp, int* status, int num_sms,
                          cudaStream_t stream, int* zero, int n_zero) {
  if (R == 0) return cudaSuccess;
  const int rows_per_block = 8;
  const int blocks = static_cast<int>(std::min<int64_t>((R + rows_per_block - 1) / rows_per_block,
                                                        static_cast<int64_t>(num_sms) * 16));
  return launch_pdl(gather_rows_kernel, dim3(blocks), dim3(256), 0, stream, x, perm, offsets, E, R, k, H, scale, Xp,
                    status, zero, n_zero);
}

cudaError_t launch_combine(const __nv_bfloat16* Y, int T, int H, int k, const __nv_bfloat16* Ys, int Ns,
                           const uint8_t* mask, __nv_bfloat16* out, int num_sms, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const int64_t n = static_cast<int64_t>(T) * (H / 8);
  const int blocks = static_cast<int>(std::min<int64_t>((n + 255) / 256, static_cast<int64_t>(num_sms) * 16));
  return launch_pdl(combine_kernel, dim3(blocks), dim3(256), 0, stream, Y, T, H, k, Ys, Ns, mask, out);
}

}  // namespace moe
