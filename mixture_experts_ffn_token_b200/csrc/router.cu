// router.cu -- stage 1: one warp per token.
//
// Softmax top-k router: the k largest logits, ties to the lowest expert
// index, ordered by descending logit; weights = softmax over the k selected
// logits (the StackedMoE page names the gate but not its body; this is the
// plain top-k softmax reading).
//
// Sigmoid-gate router with sink lanes (Mojo sink_gate_router_kernel page,
// description and Args): selection score sigmoid(z) + expert_bias (bias for
// selection only), top-k on that score, then a softmax over the log-sigmoid
// of the selected experts' RAW logits concatenated with the S always-on sink
// logits, times route_scale * global_scale.  The page computes this in log
// space so it stays finite where the sigmoids underflow; so does this kernel.
//
// Design: the page's kernel uses one block per token and one thread per
// expert with a block-level top-k.  Here one warp owns a token: each lane
// holds ceil(E/32) scores in registers, the k winners are found by k rounds
// of two warp reductions (ties -> lower index), and lanes 0..k+S-1 then
// hold one normalisation entry each, so the final softmax is one warp
// reduction.  The selection score is the fp32 value fl32(sigmoid(z)) + b
// (sigmoid evaluated in fp64 and rounded once), so the choice is decided in
// single precision exactly as the oracle decides it; the weights are
// evaluated in fp64 and rounded to fp32 on store.
#include <climits>

#include "kernels.cuh"

namespace moe {
namespace {

template <bool BF16>
__device__ __forceinline__ float load_logit(const void* logits, int64_t i) {
  if constexpr (BF16) {
    return __bfloat162float(static_cast<const __nv_bfloat16*>(logits)[i]);
  } else {
    return static_cast<const float*>(logits)[i];
  }
}

__device__ __forceinline__ double log_sigmoid(double z) { return fmin(z, 0.0) - log1p(exp(-fabs(z))); }

// Order-preserving unsigned image of a float score: a > b exactly when
// key(a) > key(b), with -0 taken as +0 (they compare equal) and NaN mapped to
// 0, below every number (-inf included), so a NaN score is never selected.
__device__ __forceinline__ uint32_t order_key(float v) {
  if (v != v) return 0u;
  const uint32_t b = __float_as_uint(v == 0.f ? 0.f : v);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Routes token t with the calling warp; returns this lane's selected expert
// (lanes 0..k-1, in selection order) and writes idx, w and sink_w.
template <int NPL, bool SINK, bool BF16>
__device__ __forceinline__ int route_token(const RouterArgs& a, int t, int lane) {
  const int64_t row = static_cast<int64_t>(t) * a.stride;
  uint32_t key[NPL];  // order_key of each score, 0 = not selectable
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const int e = lane + 32 * i;
    float kv = NAN;
    if (e < a.E) {
      const float z = load_logit<BF16>(a.logits, row + e);
      if constexpr (SINK) {
        const float sig = static_cast<float>(1.0 / (1.0 + exp(-static_cast<double>(z))));
        const float b = a.expert_bias != nullptr ? a.expert_bias[e] : 0.f;
        kv = __fadd_rn(sig, b);
      } else {
        kv = z;
      }
    }
    key[i] = order_key(kv);
  }

  // k rounds: the largest remaining key over the warp (one redux), then the
  // lowest expert index holding it (a second redux) -- ties go to the lowest
  // index, as the oracle decides them.
  uint32_t taken = 0;
  int my_e = 0;
  for (int j = 0; j < a.k; ++j) {
    uint32_t bv = 0;
    int bi = INT_MAX;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      // e grows with i, so a strict > keeps the lowest index among equal keys
      if (!((taken >> i) & 1u) && key[i] > bv) {
        bv = key[i];
        bi = lane + 32 * i;
      }
    }
    const uint32_t best = __reduce_max_sync(0xffffffffu, bv);
    const int cand = (best != 0u && bv == best) ? bi : INT_MAX;
    bi = static_cast<int>(__reduce_min_sync(0xffffffffu, static_cast<uint32_t>(cand)));
    // bi == INT_MAX only when no selectable score is left (NaN scores): the
    // index is then out of range and the CSR build flags it.
    if (bi < a.E && (bi & 31) == lane) taken |= 1u << (bi >> 5);
    if (lane == j) my_e = bi;
  }

  const int n_norm = a.k + (SINK ? a.S : 0);
  const bool active = lane < n_norm;
  double v = -INFINITY;
  if (lane < a.k) {
    const float z = my_e < a.E ? load_logit<BF16>(a.logits, row + my_e) : NAN;
    v = SINK ? log_sigmoid(static_cast<double>(z)) : static_cast<double>(z);
  } else if (SINK && active) {
    v = log_sigmoid(static_cast<double>(load_logit<BF16>(a.logits, row + a.E + (lane - a.k))));
  }
  double m = v;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, off));
  const double ex = active ? exp(v - m) : 0.0;
  double sum = ex;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  double w = ex / sum;
  if (SINK) {
    const double gs = a.global_scale != nullptr ? static_cast<double>(*a.global_scale) : 1.0;
    w *= static_cast<double>(a.route_scale) * gs;
  }
  if (lane < a.k) {
    a.idx[static_cast<int64_t>(t) * a.k + lane] = my_e;
    a.w[static_cast<int64_t>(t) * a.k + lane] = static_cast<float>(w);
  } else if (SINK && active) {
    a.sink_w[static_cast<int64_t>(t) * a.S + (lane - a.k)] = static_cast<float>(w);
  }
  return my_e;
}

template <int NPL, bool SINK, bool BF16>
__global__ void __launch_bounds__(128) router_kernel(const RouterArgs a) {
  griddep_wait();  // the previous kernel's results are complete and visible
  griddep_launch_dependents();
  if (a.status_reset != nullptr && blockIdx.x == 0 && threadIdx.x == 0) {
    a.status_reset[0] = 0;  // device status word
    a.status_reset[1] = 0;  // grid barrier of the one-launch CSR build that follows
  }
  const int lane = threadIdx.x & 31;
  const int t = static_cast<int>((static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5);
  if (t >= a.T) return;
  route_token<NPL, SINK, BF16>(a, t, lane);
}

// Small problems (R <= kSmallSlots, E <= kSmallExperts): routing and the
// whole CSR build in one CTA of kSmallWarps warps, replacing four launches.
// The CSR part is the counting sort of csr.cu with a single chunk: each warp
// owns a run of consecutive slots, a per-warp histogram scanned across warps
// and experts gives every slot its position, stable in slot order.
template <int NPL, bool SINK, bool BF16>
__global__ void __launch_bounds__(32 * kSmallWarps) route_csr_small_kernel(const RouterArgs a, int32_t* offsets,
                                                                           int32_t* perm, int* status,
                                                                           const uint8_t* mask) {
  griddep_wait();  // the previous kernel's results are complete and visible
  griddep_launch_dependents();
  extern __shared__ int sm[];
  int* s_idx = sm;                           // [R]
  int* wcnt = sm + kSmallSlots;              // [kSmallWarps][E]
  __shared__ int warp_tot[kSmallWarps];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int R = a.T * a.k, E = a.E;
  if (threadIdx.x == 0) *status = 0;
  for (int i = threadIdx.x; i < kSmallWarps * E; i += blockDim.x) wcnt[i] = 0;
  for (int t = warp; t < a.T; t += kSmallWarps) {
    const int e = route_token<NPL, SINK, BF16>(a, t, lane);
    // a masked token is routed (its weights are returned) but takes no slot
    if (lane < a.k) s_idx[t * a.k + lane] = (mask == nullptr || mask[t] != 0) ? e : -2;
  }
  __syncthreads();
  constexpr int kPerWarp = kSmallSlots / kSmallWarps;
  const int wbase = warp * kPerWarp;
  const uint32_t lt_mask = (1u << lane) - 1u;
  int* my = wcnt + warp * E;
  bool bad = false;
  for (int r = 0; r < kPerWarp; r += 32) {
    const int s = wbase + r + lane;
    const int e = s < R ? s_idx[s] : -1;
    const bool ok = e >= 0 && e < E;
    if (s < R && !ok && e != -2) bad = true;
    const uint32_t peers = __match_any_sync(0xffffffffu, ok ? e : E + lane);
    if (ok && (peers & lt_mask) == 0) my[e] += __popc(peers);
    __syncwarp();
  }
  if (bad) atomicOr(status, MOE_DEVICE_ERR_EXPERT_INDEX);
  __syncthreads();
  // per expert: exclusive prefix over warps, total, then exclusive scan over experts
  const int e = threadIdx.x;  // blockDim.x == 32 * kSmallWarps >= E
  int total = 0;
  if (e < E) {
    for (int w = 0; w < kSmallWarps; ++w) {
      const int v = wcnt[w * E + e];
      wcnt[w * E + e] = total;
      total += v;
    }
  }
  int incl = total;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int v = lane < kSmallWarps ? warp_tot[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, v, off);
      if (lane >= off) v += y;
    }
    if (lane < kSmallWarps) warp_tot[lane] = v;
  }
  __syncthreads();
  const int excl = incl - total + (warp > 0 ? warp_tot[warp - 1] : 0);
  if (e < E) {
    offsets[e] = excl;
    for (int w = 0; w < kSmallWarps; ++w) wcnt[w * E + e] += excl;
  }
  if (e == E - 1) offsets[E] = excl + total;
  __syncthreads();
  for (int r = 0; r < kPerWarp; r += 32) {
    const int s = wbase + r + lane;
    const int ee = s < R ? s_idx[s] : -1;
    const bool ok = ee >= 0 && ee < E;
    const uint32_t peers = __match_any_sync(0xffffffffu, ok ? ee : E + lane);
    int base = 0;
    if (ok) base = my[ee];
    __syncwarp();
    if (ok) {
      perm[base + __popc(peers & lt_mask)] = s;
      if ((peers & lt_mask) == 0) my[ee] += __popc(peers);
    }
    __syncwarp();
  }
}

template <int NPL>
cudaError_t launch_npl(const RouterArgs& a, cudaStream_t stream) {
  const int warps_per_block = 4;
  const dim3 grid((a.T + warps_per_block - 1) / warps_per_block);
  const dim3 block(32 * warps_per_block);
  if (a.sink) {
    if (a.logits_bf16) return launch_pdl(router_kernel<NPL, true, true>, grid, block, 0, stream, a);
    return launch_pdl(router_kernel<NPL, true, false>, grid, block, 0, stream, a);
  }
  if (a.logits_bf16) return launch_pdl(router_kernel<NPL, false, true>, grid, block, 0, stream, a);
  return launch_pdl(router_kernel<NPL, false, false>, grid, block, 0, stream, a);
}

template <int NPL>
cudaError_t launch_small_npl(const RouterArgs& a, int32_t* offsets, int32_t* perm, int* status,
                             const uint8_t* mask, cudaStream_t stream) {
  const size_t smem = (kSmallSlots + static_cast<size_t>(kSmallWarps) * a.E) * sizeof(int);
  const dim3 block(32 * kSmallWarps);
  const dim3 one(1);
  // the per-warp histograms need up to (2048 + 32 * 512) * 4 bytes, above
  // the default 48 KB: opted in once per device and kernel
  const int max_smem = static_cast<int>((kSmallSlots + static_cast<size_t>(kSmallWarps) * kSmallExperts) * sizeof(int));
  const void* kernel = a.sink ? (a.logits_bf16 ? reinterpret_cast<const void*>(route_csr_small_kernel<NPL, true, true>)
                                               : reinterpret_cast<const void*>(route_csr_small_kernel<NPL, true, false>))
                              : (a.logits_bf16 ? reinterpret_cast<const void*>(route_csr_small_kernel<NPL, false, true>)
                                               : reinterpret_cast<const void*>(route_csr_small_kernel<NPL, false, false>));
  const cudaError_t e = opt_in_dynamic_smem(kernel, max_smem);
  if (e != cudaSuccess) return e;
  if (a.sink) {
    if (a.logits_bf16)
      return launch_pdl(route_csr_small_kernel<NPL, true, true>, one, block, smem, stream, a, offsets, perm, status, mask);
    return launch_pdl(route_csr_small_kernel<NPL, true, false>, one, block, smem, stream, a, offsets, perm, status, mask);
  }
  if (a.logits_bf16)
    return launch_pdl(route_csr_small_kernel<NPL, false, true>, one, block, smem, stream, a, offsets, perm, status, mask);
  return launch_pdl(route_csr_small_kernel<NPL, false, false>, one, block, smem, stream, a, offsets, perm, status, mask);
}

}  // namespace

cudaError_t launch_route_csr_small(const RouterArgs& a, int32_t* offsets, int32_t* perm, int* status,
                                   const uint8_t* mask, cudaStream_t stream) {
  const int per_lane = (a.E + 31) / 32;
  if (per_lane <= 1) return launch_small_npl<1>(a, offsets, perm, status, mask, stream);
  if (per_lane <= 2) return launch_small_npl<2>(a, offsets, perm, status, mask, stream);
  if (per_lane <= 4) return launch_small_npl<4>(a, offsets, perm, status, mask, stream);
  if (per_lane <= 8) return launch_small_npl<8>(a, offsets, perm, status, mask, stream);
  return launch_small_npl<16>(a, offsets, perm, status, mask, stream);
}

cudaError_t launch_router(const RouterArgs& a, cudaStream_t stream) {
  if (a.T <= 0) return cudaSuccess;
  const int per_lane = (a.E + 31) / 32;
  if (per_lane <= 1) return launch_npl<1>(a, stream);
  if (per_lane <= 2) return launch_npl<2>(a, stream);
  if (per_lane <= 4) return launch_npl<4>(a, stream);
  if (per_lane <= 8) return launch_npl<8>(a, stream);
  if (per_lane <= 16) return launch_npl<16>(a, stream);
  return launch_npl<32>(a, stream);
}

}  // namespace moe
