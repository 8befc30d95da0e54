// kernels.cuh -- launchers of the sm_100a kernels, called by the C ABI
// (moe_api.cu).  Every launcher only enqueues work on `stream` and returns
// the launch status.
#pragma once

#include "common.cuh"

namespace moe {

// Runtime switches (environment variables, all optional):
//   MOE_B200_PDL=0             no programmatic dependent launch
//   MOE_B200_PDL_COOP=0        none on the two cooperative launches (CSR build, FFN)
//   MOE_B200_CSR_FUSED=0       the CSR build as three launches
//   MOE_B200_SINGLE_LAUNCH=0   the two grouped GEMMs as two launches
//   MOE_B200_CTA_PAIR=2        CTA-pair GEMM tiles (single launch unless
//                              MOE_B200_SINGLE_LAUNCH=0)
//   MOE_B200_PAIR_COOP=0       the single-launch pair without the cooperative
//                              attribute (its grid still comes from the
//                              cluster occupancy query; if some cluster is not
//                              resident, the bounded dependency waits report
//                              a timeout instead of hanging)
//   MOE_B200_B_ONE_BOX=0       four copies per B stage tile
//   MOE_B200_TILE_SCHEDULE=static|dynamic   tile order of the single launch
//   MOE_B200_FUSED_GATHER=1    the gate_up GEMM gathers its rows of x itself
//   MOE_B200_TEST_STALL_DOWN_TILES_MS, MOE_B200_TEST_STALL_CSR_MS   test hooks
//                              that make a bounded wait run out (see the kernels)
// Every API call takes one snapshot of them (refresh_switches) for all of
// its launches; switches() returns the calling thread's snapshot.
struct Switches {
  bool pdl = true;
  bool csr_fused = true;
  long test_stall_csr_ms = 0;
  bool fused_gather = false;
  bool b_one_box = true;
  int cta_pair = 1;
  long test_stall_down_ms = 0;
  char tile_schedule = 0;  // 's', 'd', or 0 (chosen by rows per expert)
  bool single_launch = true;
  bool pdl_coop = true;
  bool pair_coop = true;
};
void refresh_switches();
const Switches& switches();

// Launches `kernel` on `stream`, allowing it to overlap the tail of the
// kernel before it (programmatic dependent launch) unless
// MOE_B200_PDL=0; every kernel of this library calls griddep_wait() before
// touching global memory, so the overlap never changes what it reads.
bool pdl_enabled();

// Raises the dynamic shared-memory limit of kernel `func` to `bytes` on the
// current device the first time it is asked for that (device, kernel); once
// that has succeeded, later calls return without calling the runtime.  Every
// caller passes the kernel's largest possible size, so one opt-in serves all
// launches.  Thread-safe.
cudaError_t opt_in_dynamic_smem(const void* func, int bytes);

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// ------------------------------------------------------------------ router
struct RouterArgs {
  const void* logits;
  int logits_bf16;
  int64_t stride;
  int T, E, k, S;
  int sink;                  // 0 softmax top-k, 1 sigmoid + sink lanes
  const float* expert_bias;  // [E] or null
  const float* global_scale; // device [1] or null
  float route_scale;
  int32_t* idx;              // [T,k]
  float* w;                  // [T,k]
  float* sink_w;             // [T,S] or null
  int* status_reset;         // status_reset[0] (status) and [1] (CSR grid barrier) zeroed by the first thread, or null
};
cudaError_t launch_router(const RouterArgs& a, cudaStream_t stream);

// Routing plus the whole CSR build (offsets, permutation) in one CTA, for
// problems with at most kSmallSlots routed slots and kSmallExperts experts.
constexpr int kSmallWarps = 32;
constexpr int kSmallSlots = 2048;
constexpr int kSmallExperts = 512;
cudaError_t launch_route_csr_small(const RouterArgs& a, int32_t* offsets, int32_t* perm, int* status,
                                   const uint8_t* mask, cudaStream_t stream);

// ---------------------------------------------------------------------- CSR
constexpr int kCsrChunk = 2048;      // slots per CTA
constexpr int kCsrThreads = 512;     // 16 warps x 128 slots
inline int csr_num_chunks(int64_t R) { return static_cast<int>((R + kCsrChunk - 1) / kCsrChunk); }
// mask (may be null): slots of tokens whose mask byte is 0 take no place.
cudaError_t launch_csr_count(const int32_t* idx, int R, int E, int32_t* chunk_counts, int* status,
                             const uint8_t* mask, int k, cudaStream_t stream);
cudaError_t launch_csr_scan(const int32_t* chunk_counts, int nchunks, int E, int32_t* chunk_base,
                            int32_t* offsets, cudaStream_t stream);
cudaError_t launch_csr_scatter(const int32_t* idx, int R, int E, const int32_t* chunk_base, int32_t* perm,
                               int32_t* inv, const uint8_t* mask, int k, cudaStream_t stream);
// The three CSR kernels as one cooperative launch (one CTA per chunk), used
// when the chunks fit on the GPU at once (csr_num_chunks(R) <= num_sms) unless
// MOE_B200_CSR_FUSED=0; *barrier must be zero at launch.
bool csr_fused_enabled(int R, int num_sms);
cudaError_t launch_csr_fused(const int32_t* idx, int R, int E, int32_t* chunk_counts, int32_t* offsets, int32_t* perm,
                             int32_t* inv, int* status, int* barrier, const uint8_t* mask, int k,
                             cudaStream_t stream);
// shared slots: offsets[i] = i*T, perm[i*T + t] = t*Ns + i; also clears
// zero[0 .. n_zero) (may be null / 0).
cudaError_t launch_shared_index(int T, int Ns, int32_t* offsets, int32_t* perm, int num_sms, cudaStream_t stream,
                                int* zero = nullptr, int n_zero = 0);

// ----------------------------------------------------- gather and combine
// scale (may be null): per-slot factor applied to the gathered row.
// zero[0 .. n_zero) (may be null / 0) is cleared by the same launch.
cudaError_t launch_gather(const __nv_bfloat16* x, const int32_t* perm, const int32_t* offsets, int E, int R,
                          int k, int H, const float* scale, __nv_bfloat16* Xp, int* status, int num_sms,
                          cudaStream_t stream, int* zero = nullptr, int n_zero = 0);
// Ys (may be null, Ns = 0): shared-expert rows added after the routed ones;
// mask (may be null): masked tokens get zero rows.
cudaError_t launch_combine(const __nv_bfloat16* Y, int T, int H, int k, const __nv_bfloat16* Ys, int Ns,
                           const uint8_t* mask, __nv_bfloat16* out, int num_sms, cudaStream_t stream);

// ------------------------------------------------------------ grouped GEMM
struct GroupedGemmArgs {
  // routing (device)
  const int32_t* offsets;   // [E+1]
  const int32_t* perm;      // [R]
  const float* weights;     // [R] routing weight per slot (down GEMM), or null for 1
  int E, R, T, k;
  // problem
  int H, D;
  int gate_up_format;       // 0 concatenated, 1 interleaved
  int activation;           // 0 silu, 1 swigluoai, 2 gelu_tanh
  float alpha, limit;
  // operands (device)
  const __nv_bfloat16* A;   // Xp [R,H] (gate_up) or h [R,D] (down)
  // gate_up only: A is x [T,H] itself and a slot's A row is its row within
  // its expert's segment (the shared experts' slots, token order per expert)
  int a_direct = 0;
  // gate_up only: A is x [T,H] and the kernel gathers each tile's rows by the
  // permutation itself (token = perm[p] / k); no Xp is read
  int gather = 0;
  const __nv_bfloat16* W;   // [E,H,2D] (gate_up) or [E,D,H] (down)
  const __nv_bfloat16* bias;// [E,2D] / [E,H] or null
  __nv_bfloat16* out;       // h [R,D] (gate_up) or Y [R,H] slot rows (down)
  int* status;
  int num_sms;
};
cudaError_t launch_gemm_gate_up(const GroupedGemmArgs& a, cudaStream_t stream);
cudaError_t launch_gemm_down(const GroupedGemmArgs& a, cudaStream_t stream);

// Both contractions in one persistent cooperative launch: `up` describes the
// gate_up GEMM (A = Xp, out = h) and `down` the down GEMM (A = h, out = Y,
// which must not alias Xp).  A down tile of a 128-row piece waits (bounded)
// until every gate_up tile of that piece has stored its h columns, counted
// in arrivals[piece]; the counters must be zero at launch (launch_gather
// clears them) and hold at least mega_ffn_counters(R, E) entries: one per
// possible 128-row piece, and last the tile scheduler's counter.
int mega_ffn_counters(int R, int E);
cudaError_t launch_mega_ffn(const GroupedGemmArgs& up, const GroupedGemmArgs& down, int* arrivals,
                            cudaStream_t stream);

// Resolves cuTensorMapEncodeTiled through the runtime (no libcuda link).
bool tensor_map_encoder_available();

// Whether the gate_up GEMM gathers its rows of x itself in this process
// (MOE_B200_FUSED_GATHER=1 with single-CTA tiles; off by default).
bool fused_gather_enabled();

}  // namespace moe
