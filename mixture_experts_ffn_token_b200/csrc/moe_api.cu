// moe_api.cu -- the C ABI declared in include/moe.h: host-side validation,
// the workspace layout and the launch sequence of each entry point.
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "kernels.cuh"

using moe::kMaxExperts;
using moe::kMaxTopK;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool checked = false;
  bool supported = false;
  int num_sms = 0;
};
DeviceInfo g_devices[kMaxDevices];
std::mutex g_devices_mu;

// The current device must be compute capability 10.0 (the library's code is
// sm_100a only) and the driver must expose the tensor-map encoder.
moe_status_t current_device(int* num_sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_devices_mu);
  DeviceInfo& d = g_devices[dev];
  if (!d.checked) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return MOE_ERR_CUDA;
    d.supported = major == 10 && minor == 0 && moe::tensor_map_encoder_available();
    d.num_sms = sms;
    d.checked = true;
  }
  if (!d.supported) return MOE_ERR_UNSUPPORTED;
  *num_sms = d.num_sms;
  return MOE_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

moe_status_t validate_config(const moe_config_t* c) {
  if (c == nullptr) return MOE_ERR_INVALID_ARGUMENT;
  if (c->num_tokens < 0 || c->hidden_dim <= 0 || c->num_experts <= 0 || c->top_k <= 0 || c->moe_dim <= 0 ||
      c->num_sink < 0)
    return MOE_ERR_INVALID_ARGUMENT;
  if (c->top_k > c->num_experts) return MOE_ERR_INVALID_ARGUMENT;
  if (c->router != MOE_ROUTER_SOFTMAX_TOPK && c->router != MOE_ROUTER_SIGMOID_SINK) return MOE_ERR_INVALID_ARGUMENT;
  if (c->logits_dtype != MOE_DTYPE_BF16 && c->logits_dtype != MOE_DTYPE_F32) return MOE_ERR_INVALID_ARGUMENT;
  if (c->gate_up_format != MOE_GATE_UP_CONCATENATED && c->gate_up_format != MOE_GATE_UP_INTERLEAVED)
    return MOE_ERR_INVALID_ARGUMENT;
  if (c->activation != MOE_ACT_SILU && c->activation != MOE_ACT_SWIGLUOAI && c->activation != MOE_ACT_GELU_TANH)
    return MOE_ERR_INVALID_ARGUMENT;
  // GatedActivation: alpha must be 0 unless swigluoai; limit must be 0 for
  // gelu_tanh; a negative clamp bound is meaningless.
  if (!std::isfinite(c->alpha) || !std::isfinite(c->limit) || c->limit < 0.f) return MOE_ERR_INVALID_ARGUMENT;
  if (c->alpha != 0.f && c->activation != MOE_ACT_SWIGLUOAI) return MOE_ERR_INVALID_ARGUMENT;
  if (c->limit != 0.f && c->activation == MOE_ACT_GELU_TANH) return MOE_ERR_INVALID_ARGUMENT;
  if (c->has_bias != 0 && c->has_bias != 1) return MOE_ERR_INVALID_ARGUMENT;
  if (c->router == MOE_ROUTER_SOFTMAX_TOPK && c->num_sink != 0) return MOE_ERR_INVALID_ARGUMENT;
  if (c->logits_row_stride < static_cast<int64_t>(c->num_experts) + c->num_sink) return MOE_ERR_INVALID_ARGUMENT;
  if (c->router == MOE_ROUTER_SIGMOID_SINK && !std::isfinite(c->route_scale)) return MOE_ERR_INVALID_ARGUMENT;
  // What this library implements.
  if (c->num_experts > kMaxExperts || c->top_k > kMaxTopK) return MOE_ERR_UNSUPPORTED;
  if (c->hidden_dim % 8 != 0 || c->moe_dim % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if (c->router == MOE_ROUTER_SIGMOID_SINK) {
    // sink_gate_router_kernel: top-k plus sink lanes must be a power of two
    // no greater than the warp size.
    const int n = c->top_k + c->num_sink;
    if (n > 32 || (n & (n - 1)) != 0) return MOE_ERR_UNSUPPORTED;
  }
  const int64_t R = static_cast<int64_t>(c->num_tokens) * c->top_k;
  if (R > (int64_t(1) << 30)) return MOE_ERR_UNSUPPORTED;
  const int64_t pieces = R / 128 + c->num_experts;
  const int64_t ntiles = std::max<int64_t>((c->moe_dim + 127) / 128, (c->hidden_dim + 255) / 256);
  if (pieces * ntiles > (int64_t(1) << 30)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// The extensions of moe_forward_ex (token mask, router weight before the
// experts, shared experts), already validated.
struct Extras {
  const uint8_t* mask = nullptr;
  bool weight_first = false;
  int Ns = 0, Ds = 0;
  const void* s_gu_w = nullptr;
  const void* s_gu_b = nullptr;
  const void* s_d_w = nullptr;
  const void* s_d_b = nullptr;
};

struct WsLayout {
  size_t status, chunk_counts, chunk_base, offsets, perm, idx, w, sink, xp, h, y, arr, total;
  // shared experts: CSR of the [T, Ns] slot space, Xp_s, h_s, Y_s, counters
  size_t sh_offsets = 0, sh_perm = 0, sh_x = 0, sh_h = 0, sh_y = 0, sh_arr = 0;
};

// Whether the two contractions run as one launch (the default) or as two;
// MOE_B200_SINGLE_LAUNCH=0 selects two launches.
bool single_launch() { return moe::switches().single_launch; }

WsLayout ws_layout(const moe_config_t* c, const Extras* ex = nullptr) {
  const size_t T = static_cast<size_t>(c->num_tokens), H = c->hidden_dim, E = c->num_experts, D = c->moe_dim;
  const size_t R = T * c->top_k;
  const size_t nchunks = static_cast<size_t>(moe::csr_num_chunks(static_cast<int64_t>(R)));
  WsLayout L;
  size_t o = 0;
  L.status = o;
  o += 256;
  L.chunk_counts = o;
  o += align256(nchunks * E * 4);
  L.chunk_base = o;
  o += align256(nchunks * E * 4);
  L.offsets = o;
  o += align256((E + 1) * 4);
  L.perm = o;
  o += align256(R * 4);
  L.idx = o;
  o += align256(R * 4);
  L.w = o;
  o += align256(R * 4);
  L.sink = o;
  o += align256(T * static_cast<size_t>(c->num_sink) * 4);
  L.xp = o;  // Xp [R, H] for the gate_up GEMM, then Y [R, H] from the down GEMM
  o += align256(R * H * 2);
  L.h = o;
  o += align256(R * D * 2);
  L.y = o;  // Y [R, H] of the single-launch FFN (which still reads Xp while it writes Y)
  o += align256(R * H * 2);
  L.arr = o;
  o += align256(static_cast<size_t>(moe::mega_ffn_counters(static_cast<int>(R), static_cast<int>(E))) * 4);
  if (ex != nullptr && ex->Ns > 0) {
    const size_t Rs = T * static_cast<size_t>(ex->Ns);
    L.sh_offsets = o;
    o += align256((static_cast<size_t>(ex->Ns) + 1) * 4);
    L.sh_perm = o;
    o += align256(Rs * 4);
    L.sh_x = o;  // Xp_s [T*Ns, H] for the shared gate_up GEMM, then Y_s
    o += align256(Rs * H * 2);
    L.sh_h = o;
    o += align256(Rs * static_cast<size_t>(ex->Ds) * 2);
    L.sh_y = o;
    o += align256(Rs * H * 2);
    L.sh_arr = o;
    o += align256(static_cast<size_t>(moe::mega_ffn_counters(static_cast<int>(Rs), ex->Ns)) * 4);
  }
  L.total = o;
  return L;
}

template <typename T>
T* at(void* base, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(base) + off);
}

moe_status_t check_workspace(const moe_config_t* c, const void* ws, size_t bytes, WsLayout* L,
                             const Extras* ex = nullptr) {
  *L = ws_layout(c, ex);
  if (ws == nullptr || !aligned16(ws)) return MOE_ERR_INVALID_ARGUMENT;
  if (bytes < L->total) return MOE_ERR_WORKSPACE_TOO_SMALL;
  return MOE_OK;
}

moe_status_t check_bias(const moe_config_t* c, const void* gate_up_b, const void* down_b) {
  if (c->has_bias) return (gate_up_b != nullptr && down_b != nullptr) ? MOE_OK : MOE_ERR_INVALID_ARGUMENT;
  return (gate_up_b == nullptr && down_b == nullptr) ? MOE_OK : MOE_ERR_INVALID_ARGUMENT;
}

moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

moe::RouterArgs router_args(const moe_config_t* c, const void* logits, const float* bias, const float* gscale,
                            int32_t* idx, float* w, float* sink_w, int* status_reset) {
  moe::RouterArgs a;
  a.logits = logits;
  a.logits_bf16 = c->logits_dtype == MOE_DTYPE_BF16;
  a.stride = c->logits_row_stride;
  a.T = c->num_tokens;
  a.E = c->num_experts;
  a.k = c->top_k;
  a.S = c->num_sink;
  a.sink = c->router == MOE_ROUTER_SIGMOID_SINK;
  a.expert_bias = a.sink ? bias : nullptr;
  a.global_scale = a.sink ? gscale : nullptr;
  a.route_scale = c->route_scale;
  a.idx = idx;
  a.w = w;
  a.sink_w = sink_w;
  a.status_reset = status_reset;
  return a;
}

// Records ev[i] on the stream when events are requested.
// NVTX ranges (MOE_B200_NVTX=1): one per API call and one around the
// enqueue of each kernel, named "moe.<stage>", for a timeline profiler to
// line up with the kernels.  Off by default (no NVTX call is made).
bool nvtx_enabled() {
  static const bool on = [] {
    const char* env = std::getenv("MOE_B200_NVTX");
    return env != nullptr && env[0] == '1';
  }();
  return on;
}

struct NvtxRange {
  const bool on;
  explicit NvtxRange(const char* name) : on(nvtx_enabled()) {
    if (on) nvtxRangePushA(name);
  }
  ~NvtxRange() {
    if (on) nvtxRangePop();
  }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

struct Recorder {
  cudaEvent_t const* ev;
  cudaStream_t stream;
  void operator()(int i) const {
    if (ev == nullptr || ev[i] == nullptr) return;  // NULL slots are skipped
    // Under stream capture an event is recorded as an external event-record
    // node, so every replay of the graph records it (a plain record would
    // only become a dependency edge of the capture).
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
      cudaEventRecordWithFlags(ev[i], stream, cudaEventRecordExternal);
    else
      cudaEventRecord(ev[i], stream);
  }
};

// One grouped expert FFN pass: gather (x rows by perm, times scale[slot] if
// given) -> gate_up GEMM + activation -> down GEMM (+ bias, times
// weights[slot] if given) writing Y at slot rows.  With two launches Y
// overwrites Xp (the gate_up GEMM is done with it); the single launch
// writes Y to y_sep and counts arrivals in arr.  *y_out = where Y is.
// rec(base..base+2) before each stage (the down stage is empty when fused).
// a_direct: the gate_up GEMM reads x itself (a slot's A row is its row within
// its expert's segment, as for the shared experts' slots); no gather runs, so
// the caller has cleared arr.
moe_status_t enqueue_grouped_pass(const moe_config_t* c, int E, int k, int D, const void* x, const void* gate_up_w,
                                  const void* gate_up_b, const void* down_w, const void* down_b,
                                  const int32_t* offsets, const int32_t* perm, const float* scale,
                                  const float* weights, __nv_bfloat16* xp, __nv_bfloat16* h, __nv_bfloat16* y_sep,
                                  int* arr, __nv_bfloat16** y_out, int* status, int num_sms, cudaStream_t stream,
                                  const Recorder& rec, int base, bool a_direct = false) {
  const int T = c->num_tokens, H = c->hidden_dim;
  const int R = T * k;
  const bool fused = single_launch();
  // row f1: the gate_up GEMM gathers its rows of x itself (not when the
  // routing weight has to scale them first)
  const bool gather_in_gemm = !a_direct && scale == nullptr && moe::fused_gather_enabled();
  rec(base);
  if (gather_in_gemm) {
    // no gather kernel to clear the single launch's counters
    if (fused && R > 0 &&
        cudaMemsetAsync(arr, 0, static_cast<size_t>(moe::mega_ffn_counters(R, E)) * sizeof(int), stream) !=
            cudaSuccess)
      return MOE_ERR_CUDA;
  } else if (!a_direct) {
    const NvtxRange range("moe.gather");
    if (moe::launch_gather(static_cast<const __nv_bfloat16*>(x), perm, offsets, E, R, k, H, scale, xp, status,
                           num_sms, stream, fused ? arr : nullptr, fused ? moe::mega_ffn_counters(R, E) : 0) !=
        cudaSuccess)
      return MOE_ERR_CUDA;
  }
  moe::GroupedGemmArgs g;
  g.offsets = offsets;
  g.perm = perm;
  g.weights = weights;
  g.E = E;
  g.R = R;
  g.T = T;
  g.k = k;
  g.H = H;
  g.D = D;
  g.gate_up_format = c->gate_up_format;
  g.activation = c->activation;
  g.alpha = c->alpha;
  g.limit = c->limit;
  g.status = status;
  g.num_sms = num_sms;
  g.A = (a_direct || gather_in_gemm) ? static_cast<const __nv_bfloat16*>(x) : xp;
  g.a_direct = a_direct ? 1 : 0;
  g.gather = gather_in_gemm ? 1 : 0;
  g.W = static_cast<const __nv_bfloat16*>(gate_up_w);
  g.bias = static_cast<const __nv_bfloat16*>(gate_up_b);
  g.out = h;
  moe::GroupedGemmArgs g2 = g;
  g2.A = h;
  g2.W = static_cast<const __nv_bfloat16*>(down_w);
  g2.bias = static_cast<const __nv_bfloat16*>(down_b);
  g2.out = fused ? y_sep : xp;
  *y_out = g2.out;
  rec(base + 1);
  if (fused) {
    {
      const NvtxRange range("moe.mega_ffn");
      if (moe::launch_mega_ffn(g, g2, arr, stream) != cudaSuccess) return MOE_ERR_CUDA;
    }
    rec(base + 2);
    return MOE_OK;
  }
  {
    const NvtxRange range("moe.gemm_gate_up");
    if (moe::launch_gemm_gate_up(g, stream) != cudaSuccess) return MOE_ERR_CUDA;
  }
  rec(base + 2);
  {
    const NvtxRange range("moe.gemm_down");
    if (moe::launch_gemm_down(g2, stream) != cudaSuccess) return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

// Routed pass + combine (moe_grouped_ffn, and the tail of moe_forward
// without extensions).  ev (may be null): before gather, gate_up GEMM, down
// GEMM, combine, and after the combine.
moe_status_t enqueue_ffn(const moe_config_t* c, const void* x, const void* gate_up_w, const void* gate_up_b,
                         const void* down_w, const void* down_b, const int32_t* offsets, const int32_t* perm,
                         const float* weights, void* out, void* ws, const WsLayout& L, int num_sms,
                         cudaStream_t stream, cudaEvent_t const* ev) {
  const Recorder rec{ev, stream};
  __nv_bfloat16* xp = at<__nv_bfloat16>(ws, L.xp);
  __nv_bfloat16* y = nullptr;
  moe_status_t st = enqueue_grouped_pass(c, c->num_experts, c->top_k, c->moe_dim, x, gate_up_w, gate_up_b, down_w,
                                         down_b, offsets, perm, nullptr, weights, xp, at<__nv_bfloat16>(ws, L.h),
                                         at<__nv_bfloat16>(ws, L.y), at<int>(ws, L.arr), &y, at<int>(ws, L.status),
                                         num_sms, stream, rec, 0);
  if (st != MOE_OK) return st;
  rec(3);
  {
    const NvtxRange range("moe.combine");
    if (moe::launch_combine(y, c->num_tokens, c->hidden_dim, c->top_k, nullptr, 0, nullptr,
                            static_cast<__nv_bfloat16*>(out), num_sms, stream) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  rec(4);
  return MOE_OK;
}

// The CSR build: one cooperative launch when the chunks fit on the GPU at
// once, else count -> scan -> scatter.  The workspace's second int (right
// after the status word) is the one-launch form's grid barrier and must be
// zero here (the router clears both, or the caller's memset).
moe_status_t enqueue_csr(const moe_config_t* c, const int32_t* idx, int32_t* offsets, int32_t* perm, int32_t* inv,
                         void* ws, const WsLayout& L, int num_sms, cudaStream_t stream, cudaEvent_t const* ev,
                         const uint8_t* mask = nullptr) {
  const int R = c->num_tokens * c->top_k, E = c->num_experts, k = c->top_k;
  const Recorder rec{ev, stream};
  int* status = at<int>(ws, L.status);
  rec(0);
  if (moe::csr_fused_enabled(R, num_sms)) {
    {
      const NvtxRange range("moe.csr_fused");
      if (moe::launch_csr_fused(idx, R, E, at<int32_t>(ws, L.chunk_counts), offsets, perm, inv, status, status + 1,
                                mask, k, stream) != cudaSuccess)
        return MOE_ERR_CUDA;
    }
    rec(1);
    rec(2);
    return MOE_OK;
  }
  {
    const NvtxRange range("moe.csr_count");
    if (moe::launch_csr_count(idx, R, E, at<int32_t>(ws, L.chunk_counts), status, mask, k, stream) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  rec(1);
  {
    const NvtxRange range("moe.csr_scan");
    if (moe::launch_csr_scan(at<int32_t>(ws, L.chunk_counts), moe::csr_num_chunks(R), E, at<int32_t>(ws, L.chunk_base),
                             offsets, stream) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  rec(2);
  {
    const NvtxRange range("moe.csr_scatter");
    if (moe::launch_csr_scatter(idx, R, E, at<int32_t>(ws, L.chunk_base), perm, inv, mask, k, stream) !=
        cudaSuccess)
      return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

// Host-side checks of moe_extras_t against the configuration.
moe_status_t validate_extras(const moe_config_t* c, const moe_extras_t* e, Extras* out) {
  *out = Extras{};
  if (e == nullptr) return MOE_OK;
  if (e->apply_router_weight_first != 0 && e->apply_router_weight_first != 1) return MOE_ERR_INVALID_ARGUMENT;
  out->mask = e->token_mask;
  out->weight_first = e->apply_router_weight_first == 1;
  if (e->num_shared < 0) return MOE_ERR_INVALID_ARGUMENT;
  if (e->num_shared == 0) return MOE_OK;
  if (e->shared_dim <= 0) return MOE_ERR_INVALID_ARGUMENT;
  if (e->shared_dim % 8 != 0) return MOE_ERR_UNSUPPORTED;
  // sink router: the sink lanes are the gates of the shared experts
  if (c->router == MOE_ROUTER_SIGMOID_SINK && e->num_shared != c->num_sink) return MOE_ERR_INVALID_ARGUMENT;
  if (e->num_shared > moe::kMaxExperts) return MOE_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(c->num_tokens) * e->num_shared > (int64_t(1) << 30)) return MOE_ERR_UNSUPPORTED;
  if (c->num_tokens > 0) {
    if (e->shared_gate_up_w == nullptr || e->shared_down_w == nullptr) return MOE_ERR_INVALID_ARGUMENT;
    if (!aligned16(e->shared_gate_up_w) || !aligned16(e->shared_down_w)) return MOE_ERR_INVALID_ARGUMENT;
    if (check_bias(c, e->shared_gate_up_b, e->shared_down_b) != MOE_OK) return MOE_ERR_INVALID_ARGUMENT;
  }
  out->Ns = e->num_shared;
  out->Ds = e->shared_dim;
  out->s_gu_w = e->shared_gate_up_w;
  out->s_gu_b = e->shared_gate_up_b;
  out->s_d_w = e->shared_down_w;
  out->s_d_b = e->shared_down_b;
  return MOE_OK;
}

// moe_forward with or without extensions.  Event layouts: the plain timed
// call records MOE_NUM_STAGE_EVENTS (router, 3 x CSR, gather, gate_up, down,
// combine, end); with extensions MOE_NUM_STAGE_EVENTS_EX adds shared index,
// shared gather, shared gate_up and shared down before the combine.
moe_status_t forward_impl(const moe_config_t* cfg, const moe_extras_t* extras, const void* x, const void* logits,
                          const float* expert_bias, const float* global_scale, const void* gate_up_w,
                          const void* gate_up_b, const void* down_w, const void* down_b, void* out, int32_t* idx_out,
                          float* w_out, float* sink_out, void* ws, size_t ws_bytes, cudaStream_t stream,
                          cudaEvent_t const* ev) {
  moe::refresh_switches();  // one snapshot of the runtime switches for every launch of this call
  const NvtxRange api_range("moe_forward");
  moe_status_t st = validate_config(cfg);
  if (st != MOE_OK) return st;
  Extras ex;
  if ((st = validate_extras(cfg, extras, &ex)) != MOE_OK) return st;
  if (cfg->num_tokens == 0) return MOE_OK;  // nothing to read or write; empty tensors may have null pointers
  if (x == nullptr || logits == nullptr || gate_up_w == nullptr || down_w == nullptr || out == nullptr)
    return MOE_ERR_INVALID_ARGUMENT;
  if (!aligned16(x) || !aligned16(gate_up_w) || !aligned16(down_w) || !aligned16(out))
    return MOE_ERR_INVALID_ARGUMENT;
  if ((st = check_bias(cfg, gate_up_b, down_b)) != MOE_OK) return st;
  WsLayout L;
  if ((st = check_workspace(cfg, ws, ws_bytes, &L, &ex)) != MOE_OK) return st;
  int num_sms = 0;
  if ((st = current_device(&num_sms)) != MOE_OK) return st;
  const bool extended = extras != nullptr;
  const Recorder rec{ev, stream};
  const int T = cfg->num_tokens, k = cfg->top_k;

  int32_t* idx = idx_out != nullptr ? idx_out : at<int32_t>(ws, L.idx);
  float* w = w_out != nullptr ? w_out : at<float>(ws, L.w);
  float* sink = (sink_out != nullptr || cfg->num_sink == 0) ? sink_out : at<float>(ws, L.sink);
  int* status = at<int>(ws, L.status);
  rec(0);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* perm = at<int32_t>(ws, L.perm);
  const int64_t R = static_cast<int64_t>(T) * k;
  if (R <= moe::kSmallSlots && cfg->num_experts <= moe::kSmallExperts) {
    // small (decode-sized) problems: routing and the CSR build in one CTA;
    // the CSR stages then record back-to-back events
    const moe::RouterArgs ra = router_args(cfg, logits, expert_bias, global_scale, idx, w, sink, nullptr);
    {
      const NvtxRange range("moe.route_csr_small");
      if (moe::launch_route_csr_small(ra, offsets, perm, status, ex.mask, stream) != cudaSuccess) return MOE_ERR_CUDA;
    }
    for (int i = 1; i <= 3; ++i) rec(i);
  } else {
    const moe::RouterArgs ra = router_args(cfg, logits, expert_bias, global_scale, idx, w, sink, status);
    {
      const NvtxRange range("moe.router");
      if (moe::launch_router(ra, stream) != cudaSuccess) return MOE_ERR_CUDA;
    }
    if ((st = enqueue_csr(cfg, idx, offsets, perm, nullptr, ws, L, num_sms, stream, ev != nullptr ? ev + 1 : nullptr,
                          ex.mask)) != MOE_OK)
      return st;
  }
  if (!extended) return enqueue_ffn(cfg, x, gate_up_w, gate_up_b, down_w, down_b, offsets, perm, w, out, ws, L,
                                    num_sms, stream, ev != nullptr ? ev + 4 : nullptr);

  // routed pass: the weight scales the input (weight first) or the output
  __nv_bfloat16* xp = at<__nv_bfloat16>(ws, L.xp);
  __nv_bfloat16* y = nullptr;
  st = enqueue_grouped_pass(cfg, cfg->num_experts, k, cfg->moe_dim, x, gate_up_w, gate_up_b, down_w, down_b, offsets,
                            perm, ex.weight_first ? w : nullptr, ex.weight_first ? nullptr : w, xp,
                            at<__nv_bfloat16>(ws, L.h), at<__nv_bfloat16>(ws, L.y), at<int>(ws, L.arr), &y, status,
                            num_sms, stream, rec, 4);
  if (st != MOE_OK) return st;
  __nv_bfloat16* ys = nullptr;
  rec(7);
  if (ex.Ns > 0) {
    // shared experts: every token through each of them, gated by the sink
    // weights (sink router) or by 1
    int32_t* s_off = at<int32_t>(ws, L.sh_offsets);
    int32_t* s_perm = at<int32_t>(ws, L.sh_perm);
    // Shared expert i's slots are the tokens in order, so unless the gate
    // scales the input its gate_up GEMM reads x directly and no gather runs;
    // the index kernel then clears the pass's counters.
    const bool direct = !ex.weight_first;
    const int64_t Rs = static_cast<int64_t>(T) * ex.Ns;
    {
      const NvtxRange range("moe.shared_index");
      if (moe::launch_shared_index(T, ex.Ns, s_off, s_perm, num_sms, stream, direct ? at<int>(ws, L.sh_arr) : nullptr,
                                   direct ? moe::mega_ffn_counters(static_cast<int>(Rs), ex.Ns) : 0) != cudaSuccess)
        return MOE_ERR_CUDA;
    }
    const float* gates = cfg->router == MOE_ROUTER_SIGMOID_SINK ? sink : nullptr;
    st = enqueue_grouped_pass(cfg, ex.Ns, ex.Ns, ex.Ds, x, ex.s_gu_w, ex.s_gu_b, ex.s_d_w, ex.s_d_b, s_off, s_perm,
                              ex.weight_first ? gates : nullptr, ex.weight_first ? nullptr : gates,
                              at<__nv_bfloat16>(ws, L.sh_x), at<__nv_bfloat16>(ws, L.sh_h),
                              at<__nv_bfloat16>(ws, L.sh_y), at<int>(ws, L.sh_arr), &ys, status, num_sms, stream,
                              rec, 8, direct);
    if (st != MOE_OK) return st;
  } else {
    for (int i = 8; i <= 10; ++i) rec(i);
  }
  rec(11);
  {
    const NvtxRange range("moe.combine");
    if (moe::launch_combine(y, T, cfg->hidden_dim, k, ys, ex.Ns, ex.mask, static_cast<__nv_bfloat16*>(out), num_sms,
                            stream) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  rec(12);
  return MOE_OK;
}

}  // namespace

extern "C" {

const char* moe_status_string(moe_status_t status) {
  switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARGUMENT: return "MOE_ERR_INVALID_ARGUMENT";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_WORKSPACE_TOO_SMALL: return "MOE_ERR_WORKSPACE_TOO_SMALL";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_DEVICE_TIMEOUT: return "MOE_ERR_DEVICE_TIMEOUT";
  }
  return "MOE_ERR_UNKNOWN";
}

moe_status_t moe_single_launch_ffn(int32_t* enabled) {
  moe::refresh_switches();
  if (enabled == nullptr) return MOE_ERR_INVALID_ARGUMENT;
  *enabled = single_launch() ? 1 : 0;
  return MOE_OK;
}

moe_status_t moe_workspace_size(const moe_config_t* cfg, size_t* bytes) {
  const moe_status_t st = validate_config(cfg);
  if (st != MOE_OK) return st;
  if (bytes == nullptr) return MOE_ERR_INVALID_ARGUMENT;
  *bytes = ws_layout(cfg).total;
  return MOE_OK;
}

moe_status_t moe_route(const moe_config_t* cfg, const void* logits, const float* expert_bias,
                       const float* global_scale, int32_t* expert_indices, float* expert_weights,
                       float* sink_weights, moe_stream_t stream) {
  moe::refresh_switches();
  const NvtxRange api_range("moe_route");
  moe_status_t st = validate_config(cfg);
  if (st != MOE_OK) return st;
  if (cfg->num_tokens == 0) return MOE_OK;
  if (logits == nullptr || expert_indices == nullptr || expert_weights == nullptr) return MOE_ERR_INVALID_ARGUMENT;
  if (cfg->router == MOE_ROUTER_SIGMOID_SINK && cfg->num_sink > 0 && sink_weights == nullptr)
    return MOE_ERR_INVALID_ARGUMENT;
  int num_sms = 0;
  if ((st = current_device(&num_sms)) != MOE_OK) return st;
  const moe::RouterArgs ra =
      router_args(cfg, logits, expert_bias, global_scale, expert_indices, expert_weights, sink_weights, nullptr);
  return cuda_status(moe::launch_router(ra, reinterpret_cast<cudaStream_t>(stream)));
}

moe_status_t moe_create_indices(const moe_config_t* cfg, const int32_t* expert_indices, int32_t* expert_offsets,
                                int32_t* permutation, int32_t* inverse, void* workspace, size_t workspace_bytes,
                                moe_stream_t stream) {
  moe::refresh_switches();
  const NvtxRange api_range("moe_create_indices");
  moe_status_t st = validate_config(cfg);
  if (st != MOE_OK) return st;
  if (expert_offsets == nullptr) return MOE_ERR_INVALID_ARGUMENT;
  if (cfg->num_tokens > 0 && (expert_indices == nullptr || permutation == nullptr)) return MOE_ERR_INVALID_ARGUMENT;
  WsLayout L;
  if ((st = check_workspace(cfg, workspace, workspace_bytes, &L)) != MOE_OK) return st;
  int num_sms = 0;
  if ((st = current_device(&num_sms)) != MOE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // the status word and the CSR build's grid barrier start at zero
  if (cudaMemsetAsync(at<int>(workspace, L.status), 0, 2 * sizeof(int), s) != cudaSuccess) return MOE_ERR_CUDA;
  return enqueue_csr(cfg, expert_indices, expert_offsets, permutation, inverse, workspace, L, num_sms, s, nullptr);
}

moe_status_t moe_grouped_ffn(const moe_config_t* cfg, const void* x, const void* gate_up_w, const void* gate_up_b,
                             const void* down_w, const void* down_b, const int32_t* expert_offsets,
                             const int32_t* permutation, const float* expert_weights, void* out, void* workspace,
                             size_t workspace_bytes, moe_stream_t stream) {
  moe::refresh_switches();
  const NvtxRange api_range("moe_grouped_ffn");
  moe_status_t st = validate_config(cfg);
  if (st != MOE_OK) return st;
  if (cfg->num_tokens == 0) return MOE_OK;
  if (x == nullptr || gate_up_w == nullptr || down_w == nullptr || out == nullptr || expert_offsets == nullptr ||
      permutation == nullptr || expert_weights == nullptr)
    return MOE_ERR_INVALID_ARGUMENT;
  if (!aligned16(x) || !aligned16(gate_up_w) || !aligned16(down_w) || !aligned16(out))
    return MOE_ERR_INVALID_ARGUMENT;
  if ((st = check_bias(cfg, gate_up_b, down_b)) != MOE_OK) return st;
  WsLayout L;
  if ((st = check_workspace(cfg, workspace, workspace_bytes, &L)) != MOE_OK) return st;
  int num_sms = 0;
  if ((st = current_device(&num_sms)) != MOE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(at<int>(workspace, L.status), 0, sizeof(int), s) != cudaSuccess) return MOE_ERR_CUDA;
  return enqueue_ffn(cfg, x, gate_up_w, gate_up_b, down_w, down_b, expert_offsets, permutation, expert_weights, out,
                     workspace, L, num_sms, s, nullptr);
}

moe_status_t moe_forward(const moe_config_t* cfg, const void* x, const void* logits, const float* expert_bias,
                         const float* global_scale, const void* gate_up_w, const void* gate_up_b, const void* down_w,
                         const void* down_b, void* out, int32_t* expert_indices_out, float* expert_weights_out,
                         float* sink_weights_out, void* workspace, size_t workspace_bytes, moe_stream_t stream) {
  return forward_impl(cfg, nullptr, x, logits, expert_bias, global_scale, gate_up_w, gate_up_b, down_w, down_b, out,
                      expert_indices_out, expert_weights_out, sink_weights_out, workspace, workspace_bytes,
                      reinterpret_cast<cudaStream_t>(stream), nullptr);
}

moe_status_t moe_forward_timed(const moe_config_t* cfg, const void* x, const void* logits, const float* expert_bias,
                               const float* global_scale, const void* gate_up_w, const void* gate_up_b,
                               const void* down_w, const void* down_b, void* out, int32_t* expert_indices_out,
                               float* expert_weights_out, float* sink_weights_out, void* workspace,
                               size_t workspace_bytes, moe_stream_t stream, void* const* stage_events) {
  if (stage_events == nullptr) return MOE_ERR_INVALID_ARGUMENT;
  return forward_impl(cfg, nullptr, x, logits, expert_bias, global_scale, gate_up_w, gate_up_b, down_w, down_b, out,
                      expert_indices_out, expert_weights_out, sink_weights_out, workspace, workspace_bytes,
                      reinterpret_cast<cudaStream_t>(stream), reinterpret_cast<cudaEvent_t const*>(stage_events));
}

moe_status_t moe_workspace_size_ex(const moe_config_t* cfg, const moe_extras_t* extras, size_t* bytes) {
  moe_status_t st = validate_config(cfg);
  if (st != MOE_OK) return st;
  Extras ex;
  if ((st = validate_extras(cfg, extras, &ex)) != MOE_OK) return st;
  if (bytes == nullptr) return MOE_ERR_INVALID_ARGUMENT;
  *bytes = ws_layout(cfg, &ex).total;
  return MOE_OK;
}

moe_status_t moe_forward_ex(const moe_config_t* cfg, const moe_extras_t* extras, const void* x, const void* logits,
                            const float* expert_bias, const float* global_scale, const void* gate_up_w,
                            const void* gate_up_b, const void* down_w, const void* down_b, void* out,
                            int32_t* expert_indices_out, float* expert_weights_out, float* sink_weights_out,
                            void* workspace, size_t workspace_bytes, moe_stream_t stream, void* const* stage_events) {
  moe_extras_t none;
  std::memset(&none, 0, sizeof(none));
  return forward_impl(cfg, extras != nullptr ? extras : &none, x, logits, expert_bias, global_scale, gate_up_w,
                      gate_up_b, down_w, down_b, out, expert_indices_out, expert_weights_out, sink_weights_out,
                      workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream),
                      reinterpret_cast<cudaEvent_t const*>(stage_events));
}

moe_status_t moe_device_status(const void* workspace, int32_t* device_status, moe_stream_t stream) {
  if (workspace == nullptr || device_status == nullptr) return MOE_ERR_INVALID_ARGUMENT;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  *device_status = v;
  if (v & (MOE_DEVICE_ERR_TIMEOUT_GEMM1 | MOE_DEVICE_ERR_TIMEOUT_GEMM2 | MOE_DEVICE_ERR_TIMEOUT_CSR))
    return MOE_ERR_DEVICE_TIMEOUT;
  return MOE_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// moe_create_indices_noalloc: the same CSR build, with its scratch (the
// device status word and the per-chunk histogram and base tables) in one
// fixed-size array in device memory instead of a caller workspace.
namespace {

// Capacity: (number of 2048-slot chunks) x (experts) cells.  With 128
// experts that is up to 1,048,576 routed slots; with 1024 experts, 131,072.
constexpr size_t kNoAllocMaxCells = 65536;
constexpr size_t kNoAllocHeaderBytes = 256;  // the device status word lives here
constexpr size_t kNoAllocBytes = kNoAllocHeaderBytes + 2 * kNoAllocMaxCells * sizeof(int32_t);  // 512.25 KiB

// Every GPU that loads this library holds this array until the process
// exits.  Host code must not use its name as an address: the device address
// comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

void* g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mu;

// Device address of g_noalloc_scratch on the current device, looked up once
// per device (with that device current) on its first call.
moe_status_t noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" moe_status_t moe_create_indices_noalloc(const moe_config_t* cfg, const int32_t* expert_indices,
                                                   int32_t* expert_offsets, int32_t* permutation,
                                                   int32_t* inverse, moe_stream_t stream) {
  moe::refresh_switches();
  moe_status_t st = validate_config(cfg);
  if (st != MOE_OK) return st;
  if (expert_offsets == nullptr) return MOE_ERR_INVALID_ARGUMENT;
  if (cfg->num_tokens > 0 && (expert_indices == nullptr || permutation == nullptr)) return MOE_ERR_INVALID_ARGUMENT;
  const int64_t R = static_cast<int64_t>(cfg->num_tokens) * cfg->top_k;
  const size_t cells = static_cast<size_t>(moe::csr_num_chunks(R)) * static_cast<size_t>(cfg->num_experts);
  if (cells > kNoAllocMaxCells) return MOE_ERR_WORKSPACE_TOO_SMALL;
  int num_sms = 0;
  if ((st = current_device(&num_sms)) != MOE_OK) return st;
  void* base = nullptr;
  if ((st = noalloc_scratch(&base)) != MOE_OK) return st;
  WsLayout L = {};
  L.status = 0;
  L.chunk_counts = kNoAllocHeaderBytes;
  L.chunk_base = kNoAllocHeaderBytes + kNoAllocMaxCells * sizeof(int32_t);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // The histogram and base tables are fully rewritten by every call; only the
  // status word and the grid barrier word after it have to start at zero.
  if (cudaMemsetAsync(base, 0, 2 * sizeof(int32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
  return enqueue_csr(cfg, expert_indices, expert_offsets, permutation, inverse, base, L, num_sms, s, nullptr);
}
