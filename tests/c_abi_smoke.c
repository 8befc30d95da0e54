/* Plain-C use of the library through include/moe.h only (no Python): a
 * small MoE layer with device buffers from cudaMalloc.  It checks
 *   - argument errors come back as status codes before any launch,
 *   - moe_route -> moe_create_indices -> moe_grouped_ffn equals moe_forward
 *     bit for bit, and two moe_forward calls agree,
 *   - the device status word is clean,
 *   - the output is finite and not all zero.
 *   - moe_forward_timed, and moe_forward_ex without extensions, give
 *     moe_forward's bits; moe_forward_ex with a token mask zeroes the masked
 *     rows and leaves every other row's bits unchanged;
 *   - moe_single_launch_ffn answers 0 or 1, moe_workspace_size_ex(NULL)
 *     equals moe_workspace_size, and moe_create_indices_noalloc builds the
 *     same CSR as moe_create_indices.
 * Prints "ok" and exits 0 on success; the GPU test suite compiles and runs it. */
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "moe.h"

#define CHECK_CUDA(x)                                                         \
  do {                                                                        \
    cudaError_t e_ = (x);                                                     \
    if (e_ != cudaSuccess) {                                                  \
      fprintf(stderr, "%s:%d %s\n", __FILE__, __LINE__, cudaGetErrorString(e_)); \
      return 1;                                                               \
    }                                                                         \
  } while (0)

#define CHECK_MOE(x)                                                               \
  do {                                                                             \
    moe_status_t s_ = (x);                                                         \
    if (s_ != MOE_OK) {                                                            \
      fprintf(stderr, "%s:%d %s\n", __FILE__, __LINE__, moe_status_string(s_));   \
      return 1;                                                                    \
    }                                                                              \
  } while (0)

/* bf16 bits of a float (round to nearest even) */
static uint16_t to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

static float from_bf16(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* a small counter-based generator: uniform in [-1, 1) */
static float unif(uint64_t* s) {
  *s = *s * 6364136223846793005ull + 1442695040888963407ull;
  return (float)((*s >> 40) & 0xffffff) / 8388608.0f - 1.0f;
}

static int fill_bf16(void** dev, size_t n, float scale, uint64_t seed) {
  uint16_t* h = (uint16_t*)malloc(n * 2);
  for (size_t i = 0; i < n; ++i) h[i] = to_bf16(unif(&seed) * scale);
  CHECK_CUDA(cudaMalloc(dev, n * 2));
  CHECK_CUDA(cudaMemcpy(*dev, h, n * 2, cudaMemcpyHostToDevice));
  free(h);
  return 0;
}

int main(void) {
  const int T = 96, H = 256, E = 8, k = 2, D = 384;
  moe_config_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.num_tokens = T;
  cfg.hidden_dim = H;
  cfg.num_experts = E;
  cfg.top_k = k;
  cfg.moe_dim = D;
  cfg.router = MOE_ROUTER_SOFTMAX_TOPK;
  cfg.logits_dtype = MOE_DTYPE_F32;
  cfg.logits_row_stride = E;
  cfg.route_scale = 1.0f;
  cfg.gate_up_format = MOE_GATE_UP_CONCATENATED;
  cfg.activation = MOE_ACT_SILU;

  size_t ws_bytes = 0;
  CHECK_MOE(moe_workspace_size(&cfg, &ws_bytes));

  void *x, *wgu, *wd, *logits, *out, *out2, *ws;
  if (fill_bf16(&x, (size_t)T * H, 1.0f, 1)) return 1;
  if (fill_bf16(&wgu, (size_t)E * H * 2 * D, 0.05f, 2)) return 1;
  if (fill_bf16(&wd, (size_t)E * D * H, 0.05f, 3)) return 1;
  {
    float* hl = (float*)malloc((size_t)T * E * 4);
    uint64_t s = 4;
    for (int i = 0; i < T * E; ++i) hl[i] = 2.0f * unif(&s);
    CHECK_CUDA(cudaMalloc(&logits, (size_t)T * E * 4));
    CHECK_CUDA(cudaMemcpy(logits, hl, (size_t)T * E * 4, cudaMemcpyHostToDevice));
    free(hl);
  }
  CHECK_CUDA(cudaMalloc(&out, (size_t)T * H * 2));
  CHECK_CUDA(cudaMalloc(&out2, (size_t)T * H * 2));
  CHECK_CUDA(cudaMalloc(&ws, ws_bytes));

  /* argument errors: no launch, a status code */
  if (moe_forward(&cfg, NULL, logits, NULL, NULL, wgu, NULL, wd, NULL, out, NULL, NULL, NULL, ws, ws_bytes, 0) !=
      MOE_ERR_INVALID_ARGUMENT) {
    fprintf(stderr, "a NULL x was not rejected\n");
    return 1;
  }
  if (moe_forward(&cfg, x, logits, NULL, NULL, wgu, NULL, wd, NULL, out, NULL, NULL, NULL, ws, 16, 0) !=
      MOE_ERR_WORKSPACE_TOO_SMALL) {
    fprintf(stderr, "a short workspace was not rejected\n");
    return 1;
  }

  /* the whole layer */
  CHECK_MOE(moe_forward(&cfg, x, logits, NULL, NULL, wgu, NULL, wd, NULL, out, NULL, NULL, NULL, ws, ws_bytes, 0));
  int32_t dev_status = -1;
  CHECK_MOE(moe_device_status(ws, &dev_status, 0));
  if (dev_status != 0) {
    fprintf(stderr, "device status %#x\n", dev_status);
    return 1;
  }

  /* the same through the three stages */
  int32_t *idx, *offsets, *perm;
  float* w;
  CHECK_CUDA(cudaMalloc((void**)&idx, (size_t)T * k * 4));
  CHECK_CUDA(cudaMalloc((void**)&w, (size_t)T * k * 4));
  CHECK_CUDA(cudaMalloc((void**)&offsets, (size_t)(E + 1) * 4));
  CHECK_CUDA(cudaMalloc((void**)&perm, (size_t)T * k * 4));
  CHECK_MOE(moe_route(&cfg, logits, NULL, NULL, idx, w, NULL, 0));
  CHECK_MOE(moe_create_indices(&cfg, idx, offsets, perm, NULL, ws, ws_bytes, 0));
  CHECK_MOE(moe_grouped_ffn(&cfg, x, wgu, NULL, wd, NULL, offsets, perm, w, out2, ws, ws_bytes, 0));
  CHECK_CUDA(cudaDeviceSynchronize());

  uint16_t* h1 = (uint16_t*)malloc((size_t)T * H * 2);
  uint16_t* h2 = (uint16_t*)malloc((size_t)T * H * 2);
  CHECK_CUDA(cudaMemcpy(h1, out, (size_t)T * H * 2, cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(h2, out2, (size_t)T * H * 2, cudaMemcpyDeviceToHost));
  if (memcmp(h1, h2, (size_t)T * H * 2) != 0) {
    fprintf(stderr, "staged calls differ from moe_forward\n");
    return 1;
  }

  /* a second call gives the same bits */
  CHECK_MOE(moe_forward(&cfg, x, logits, NULL, NULL, wgu, NULL, wd, NULL, out2, NULL, NULL, NULL, ws, ws_bytes, 0));
  CHECK_CUDA(cudaDeviceSynchronize());
  CHECK_CUDA(cudaMemcpy(h2, out2, (size_t)T * H * 2, cudaMemcpyDeviceToHost));
  if (memcmp(h1, h2, (size_t)T * H * 2) != 0) {
    fprintf(stderr, "two moe_forward calls differ\n");
    return 1;
  }

  /* whether the two GEMMs run as one launch: a status and a 0/1 answer */
  int32_t single = -1;
  CHECK_MOE(moe_single_launch_ffn(&single));
  if (single != 0 && single != 1) {
    fprintf(stderr, "moe_single_launch_ffn gave %d\n", single);
    return 1;
  }

  /* moe_forward_timed: the same bits, and every stage interval non-negative */
  {
    cudaEvent_t ev[MOE_NUM_STAGE_EVENTS];
    for (int i = 0; i < MOE_NUM_STAGE_EVENTS; ++i) CHECK_CUDA(cudaEventCreate(&ev[i]));
    CHECK_MOE(moe_forward_timed(&cfg, x, logits, NULL, NULL, wgu, NULL, wd, NULL, out2, NULL, NULL, NULL, ws,
                                ws_bytes, 0, (void* const*)ev));
    CHECK_CUDA(cudaDeviceSynchronize());
    for (int i = 0; i + 1 < MOE_NUM_STAGE_EVENTS; ++i) {
      float ms = -1.0f;
      CHECK_CUDA(cudaEventElapsedTime(&ms, ev[i], ev[i + 1]));
      if (!(ms >= 0.0f)) {
        fprintf(stderr, "stage %d interval %f\n", i, ms);
        return 1;
      }
    }
    for (int i = 0; i < MOE_NUM_STAGE_EVENTS; ++i) CHECK_CUDA(cudaEventDestroy(ev[i]));
    CHECK_CUDA(cudaMemcpy(h2, out2, (size_t)T * H * 2, cudaMemcpyDeviceToHost));
    if (memcmp(h1, h2, (size_t)T * H * 2) != 0) {
      fprintf(stderr, "moe_forward_timed differs from moe_forward\n");
      return 1;
    }
  }

  /* moe_forward_ex: no extensions gives moe_forward's bits; a token mask
     zeroes the masked rows and leaves every other row's bits unchanged */
  {
    size_t ws_ex = 0;
    CHECK_MOE(moe_workspace_size_ex(&cfg, NULL, &ws_ex));
    if (ws_ex != ws_bytes) {
      fprintf(stderr, "moe_workspace_size_ex(NULL) %zu != moe_workspace_size %zu\n", ws_ex, ws_bytes);
      return 1;
    }
    CHECK_MOE(moe_forward_ex(&cfg, NULL, x, logits, NULL, NULL, wgu, NULL, wd, NULL, out2, NULL, NULL, NULL, ws,
                             ws_bytes, 0, NULL));
    CHECK_CUDA(cudaDeviceSynchronize());
    CHECK_CUDA(cudaMemcpy(h2, out2, (size_t)T * H * 2, cudaMemcpyDeviceToHost));
    if (memcmp(h1, h2, (size_t)T * H * 2) != 0) {
      fprintf(stderr, "moe_forward_ex without extensions differs from moe_forward\n");
      return 1;
    }
    uint8_t hmask[T];
    for (int t = 0; t < T; ++t) hmask[t] = (uint8_t)(t % 3 != 1);
    uint8_t* mask;
    CHECK_CUDA(cudaMalloc((void**)&mask, (size_t)T));
    CHECK_CUDA(cudaMemcpy(mask, hmask, (size_t)T, cudaMemcpyHostToDevice));
    moe_extras_t ex;
    memset(&ex, 0, sizeof(ex));
    ex.token_mask = mask;
    CHECK_MOE(moe_workspace_size_ex(&cfg, &ex, &ws_ex));
    void* ws2;
    CHECK_CUDA(cudaMalloc(&ws2, ws_ex));
    CHECK_MOE(moe_forward_ex(&cfg, &ex, x, logits, NULL, NULL, wgu, NULL, wd, NULL, out2, NULL, NULL, NULL, ws2,
                             ws_ex, 0, NULL));
    CHECK_CUDA(cudaDeviceSynchronize());
    CHECK_CUDA(cudaMemcpy(h2, out2, (size_t)T * H * 2, cudaMemcpyDeviceToHost));
    for (int t = 0; t < T; ++t) {
      const int same = memcmp(h1 + (size_t)t * H, h2 + (size_t)t * H, (size_t)H * 2) == 0;
      int zero = 1;
      for (int c = 0; c < H; ++c) zero &= from_bf16(h2[(size_t)t * H + c]) == 0.0f;
      if (hmask[t] ? !same : !zero) {
        fprintf(stderr, "token %d: masked rows must be zero, the others unchanged\n", t);
        return 1;
      }
    }
    CHECK_CUDA(cudaFree(ws2));
    CHECK_CUDA(cudaFree(mask));
  }

  /* moe_create_indices_noalloc: the same CSR without a workspace */
  {
    int32_t *off2, *perm2;
    CHECK_CUDA(cudaMalloc((void**)&off2, (size_t)(E + 1) * 4));
    CHECK_CUDA(cudaMalloc((void**)&perm2, (size_t)T * k * 4));
    CHECK_MOE(moe_create_indices_noalloc(&cfg, idx, off2, perm2, NULL, 0));
    CHECK_CUDA(cudaDeviceSynchronize());
    int32_t a[E + 1], b[E + 1];
    int32_t* pa = (int32_t*)malloc((size_t)T * k * 4);
    int32_t* pb = (int32_t*)malloc((size_t)T * k * 4);
    CHECK_CUDA(cudaMemcpy(a, offsets, (size_t)(E + 1) * 4, cudaMemcpyDeviceToHost));
    CHECK_CUDA(cudaMemcpy(b, off2, (size_t)(E + 1) * 4, cudaMemcpyDeviceToHost));
    CHECK_CUDA(cudaMemcpy(pa, perm, (size_t)T * k * 4, cudaMemcpyDeviceToHost));
    CHECK_CUDA(cudaMemcpy(pb, perm2, (size_t)T * k * 4, cudaMemcpyDeviceToHost));
    if (memcmp(a, b, sizeof(a)) != 0 || memcmp(pa, pb, (size_t)T * k * 4) != 0) {
      fprintf(stderr, "moe_create_indices_noalloc differs from moe_create_indices\n");
      return 1;
    }
    free(pa);
    free(pb);
    CHECK_CUDA(cudaFree(off2));
    CHECK_CUDA(cudaFree(perm2));
  }

  double sum = 0.0;
  int nonzero = 0;
  for (int i = 0; i < T * H; ++i) {
    const float v = from_bf16(h1[i]);
    if (!isfinite(v)) {
      fprintf(stderr, "non-finite output at %d\n", i);
      return 1;
    }
    sum += fabs(v);
    nonzero += v != 0.0f;
  }
  if (nonzero < T * H / 2) {
    fprintf(stderr, "output mostly zero (%d of %d nonzero)\n", nonzero, T * H);
    return 1;
  }
  printf("sum|out| = %.6f over %d values\nok\n", sum, T * H);
  free(h1);
  free(h2);
  return 0;
}
