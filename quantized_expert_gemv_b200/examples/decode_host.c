/* decode_host.c -- the library from plain C, no tensor framework:
 * fp32 expert weights (a seeded toy generator) are quantised on the device
 * (fmoe_quantize_groups), packed (fmoe_pack_experts_device), and one token
 * is carried through the layer from host memory a few times
 * (fmoe_layer_forward_host).  Prints the output norm of each step and the
 * device status; exits non-zero on any error or a non-finite output.
 *
 * Build (from the repository root, after the library is built):
 *   gcc -O2 -std=c11 -Iinclude -I/usr/local/cuda/include \
 *       quantized_expert_gemv_b200/examples/decode_host.c \
 *       -Lquantized_expert_gemv_b200 -lfmoe -L/usr/local/cuda/lib64 -lcudart \
 *       -Wl,-rpath,$PWD/quantized_expert_gemv_b200 -lm -o decode_host
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

#include <cuda_runtime.h>

#include "fmoe.h"

#define CHECK(call)                                                                   \
  do {                                                                                \
    int rc_ = (call);                                                                 \
    if (rc_ != FMOE_OK) {                                                             \
      fprintf(stderr, "%s: %s\n", #call, fmoe_error_string(rc_));                     \
      return 1;                                                                       \
    }                                                                                 \
  } while (0)
#define CUDA(call)                                                                    \
  do {                                                                                \
    cudaError_t e_ = (call);                                                          \
    if (e_ != cudaSuccess) {                                                          \
      fprintf(stderr, "%s: %s\n", #call, cudaGetErrorString(e_));                     \
      return 1;                                                                       \
    }                                                                                 \
  } while (0)

/* toy normal generator: 12 uniforms of a 64-bit LCG */
static uint64_t g_state = 0x2545F4914F6CDD1Dull;
static float toy_normal(void) {
  double s = 0.0;
  for (int i = 0; i < 12; ++i) {
    g_state = g_state * 6364136223846793005ull + 1442695040888963407ull;
    s += (double)(g_state >> 11) / 9007199254740992.0;
  }
  return (float)(s - 6.0);
}

static void* dev_alloc(size_t bytes) {
  void* p = NULL;
  return cudaMalloc(&p, bytes) == cudaSuccess ? p : NULL;
}

int main(void) {
  const int H = 1024, I = 256, E = 16, K = 4;
  fmoe_layer_desc d = {H, I, E, K, 4, 4, 64, 1e-6f};
  const size_t n_w = (size_t)3 * H * I;  /* weights per expert (gate, up, down) */
  cudaStream_t st;
  CUDA(cudaStreamCreate(&st));

  /* fp32 expert weights (E routed + 1 shared), quantised and packed on the device */
  const size_t n_all = n_w * (E + 1);
  float* h_w = (float*)malloc(n_all * sizeof(float));
  for (size_t i = 0; i < n_all; ++i) h_w[i] = 0.02f * toy_normal();
  float* d_w = (float*)dev_alloc(n_all * sizeof(float));
  uint8_t* d_q = (uint8_t*)dev_alloc(n_all);
  uint16_t* d_s = (uint16_t*)dev_alloc(n_all / 64 * 2);
  uint16_t* d_b = (uint16_t*)dev_alloc(n_all / 64 * 2);
  if (!h_w || !d_w || !d_q || !d_s || !d_b) return 1;
  CUDA(cudaMemcpy(d_w, h_w, n_all * sizeof(float), cudaMemcpyHostToDevice));
  CHECK(fmoe_quantize_groups(d_w, n_all / 64, 64, 4, d_q, d_s, d_b, st));
  const size_t rec = fmoe_packed_bytes(4, 1, H, I, 64);
  uint8_t* d_experts = (uint8_t*)dev_alloc(rec * E);
  uint8_t* d_shared = (uint8_t*)dev_alloc(rec);
  if (!d_experts || !d_shared) return 1;
  CHECK(fmoe_pack_experts_device(d_q, d_s, d_b, 4, E, H, I, 64, d_experts, rec * E, st));
  CHECK(fmoe_pack_experts_device(d_q + n_w * E, d_s + n_w * E / 64, d_b + n_w * E / 64, 4, 1, H, I, 64, d_shared,
                                 rec, st));

  /* router, shared gate, norm weight */
  float* h_r = (float*)malloc(((size_t)E + 2) * H * sizeof(float));
  for (size_t i = 0; i < ((size_t)E + 1) * H; ++i) h_r[i] = 0.02f * toy_normal();
  for (int i = 0; i < H; ++i) h_r[(size_t)(E + 1) * H + i] = 1.0f + 0.1f * toy_normal();
  float* d_r = (float*)dev_alloc(((size_t)E + 2) * H * sizeof(float));
  if (!h_r || !d_r) return 1;
  CUDA(cudaMemcpy(d_r, h_r, ((size_t)E + 2) * H * sizeof(float), cudaMemcpyHostToDevice));
  fmoe_layer_weights lw = {d, d_experts, d_shared, d_r, d_r + (size_t)E * H, d_r + (size_t)(E + 1) * H};

  /* workspace and the token's device block */
  const size_t ws_bytes = fmoe_workspace_bytes(&d, 1);
  void* d_ws = dev_alloc(ws_bytes);
  float* d_hx = (float*)dev_alloc((size_t)2 * H * sizeof(float));
  float* hx = NULL;
  if (!d_ws || !d_hx || cudaMallocHost((void**)&hx, (size_t)2 * H * sizeof(float)) != cudaSuccess) return 1;
  CHECK(fmoe_workspace_init(d_ws, ws_bytes, st));
  for (int i = 0; i < H; ++i) hx[i] = hx[H + i] = toy_normal();

  for (int step = 0; step < 4; ++step) {
    CHECK(fmoe_layer_forward_host(&lw, hx, hx, d_hx, 1, d_ws, ws_bytes, st));
    CUDA(cudaStreamSynchronize(st));
    double n = 0.0;
    for (int i = 0; i < H; ++i) n += (double)hx[H + i] * hx[H + i];
    if (!isfinite(n)) return 1;
    printf("step %d: |xn'| = %.6f\n", step, sqrt(n));
    for (int i = 0; i < H; ++i) hx[i] = hx[H + i];  /* the next step starts from this xn' */
  }
  uint32_t status = 0;
  CHECK(fmoe_read_status(&status, 1));
  printf("device status 0x%x\n", status);
  return status == 0 ? 0 : 1;
}
