/* A C11 caller (the CUDA runtime header needs C11) that runs the hot path on the GPU with no
 * Python: device memory from the CUDA runtime, then RoPE on k, the prefill (q rotated at load), the
 * append and a decode step, for a sliding and a full layer.  With every value row equal to 1 and
 * every gate logit 0, each output element is sigmoid(0) * (sum_j P_ij * 1) / (sum_j P_ij) = 0.5
 * whatever q and k are (softmax rows sum to 1); the kernels' bf16 P makes it 0.5 up to ~2^-8.
 * Prints one line per check; exits 1 on a failed call or a value off by more than 2e-2. */
#include <cuda_runtime_api.h>
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>
#include "spark_attn.h"

static unsigned short to_bf16(float x) {
  unsigned int u;
  memcpy(&u, &x, 4);
  return (unsigned short)((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
}

static float from_bf16(unsigned short h) {
  unsigned int u = (unsigned int)h << 16;
  float x;
  memcpy(&x, &u, 4);
  return x;
}

static void* dev_fill(size_t n, float (*f)(size_t)) {
  unsigned short* h = (unsigned short*)malloc(n * 2);
  void* d = NULL;
  size_t i;
  for (i = 0; i < n; ++i) h[i] = to_bf16(f(i));
  if (cudaMalloc(&d, n * 2) != cudaSuccess || cudaMemcpy(d, h, n * 2, cudaMemcpyHostToDevice) != cudaSuccess) {
    free(h);
    return NULL;
  }
  free(h);
  return d;
}

static float f_mixed(size_t i) { return (float)((int)((i * 2654435761u) >> 20) % 257 - 128) / 64.0f; }
static float f_one(size_t i) { (void)i; return 1.0f; }
static float f_zero(size_t i) { (void)i; return 0.0f; }

static int check_half(const void* dout, size_t n, const char* what) {
  unsigned short* h = (unsigned short*)malloc(n * 2);
  size_t i, bad = 0;
  float worst = 0.0f;
  cudaMemcpy(h, dout, n * 2, cudaMemcpyDeviceToHost);
  for (i = 0; i < n; ++i) {
    const float e = fabsf(from_bf16(h[i]) - 0.5f);
    if (!(e <= 2e-2f)) ++bad;
    if (e > worst) worst = e;
  }
  free(h);
  printf("%s: %zu outputs, worst |out - 0.5| %.5f, %zu off\n", what, n, worst, bad);
  return bad == 0;
}

int main(void) {
  const int B = 2, T = 700, cap_full = 1024;
  int ok = 1, kind;
  for (kind = 0; kind < 2 && ok; ++kind) {
    spark_layer_cfg cfg;
    const int cap = kind == SPARK_SLIDING ? SPARK_WINDOW : cap_full;
    const size_t nq = (size_t)B * T * 16 * 256, nk = (size_t)B * T * 4 * 256;
    void *q = dev_fill(nq, f_mixed), *k = dev_fill(nk, f_mixed), *v = dev_fill(nk, f_one);
    void *g = dev_fill((size_t)B * T * 16, f_zero), *out = NULL, *kc = NULL, *vc = NULL, *ws = NULL;
    void *qd = dev_fill((size_t)B * 16 * 256, f_mixed), *gd = dev_fill((size_t)B * 16, f_zero);
    void *kn = dev_fill((size_t)B * 4 * 256, f_mixed), *vn = dev_fill((size_t)B * 4 * 256, f_one);
    int* pos = NULL;
    int hpos0[2] = {0, 0}, hpos[2] = {T, T};
    size_t ws_bytes;
    spark_layer_cfg_for_kind(kind, &cfg);
    if (!q || !k || !v || !g || !qd || !gd || !kn || !vn) return 1;
    cudaMalloc(&out, nq * 2);
    cudaMalloc(&kc, (size_t)B * 4 * cap * 256 * 2);
    cudaMalloc(&vc, (size_t)B * 4 * cap * 256 * 2);
    cudaMalloc((void**)&pos, 2 * sizeof(int));
    cudaMemcpy(pos, hpos0, sizeof(hpos0), cudaMemcpyHostToDevice);
    /* prefill: RoPE on k, the attention with q rotated at load, the chunk appended */
    ok &= spark_rope_apply(k, B, T, 4, 0, 0, pos, &cfg, NULL) == SPARK_OK;
    ok &= spark_attn_prefill(out, q, k, v, g, NULL, NULL, 0, B, T, 0, 0, 0, 0, pos, &cfg, SPARK_ROPE_FUSED, NULL) ==
          SPARK_OK;
    ok &= spark_kv_append(kc, vc, cap, k, v, B, T, 0, 0, pos, &cfg, 0, NULL) == SPARK_OK;
    ok &= spark_check(NULL) == SPARK_OK;
    ok &= check_half(out, nq, kind == SPARK_SLIDING ? "prefill sliding" : "prefill full");
    /* decode of one more token at position T: append (RoPE fused on k), then attend */
    cudaMemcpy(pos, hpos, sizeof(hpos), cudaMemcpyHostToDevice);
    ws_bytes = spark_decode_workspace_bytes(B, cap, &cfg);
    cudaMalloc(&ws, ws_bytes > 0 ? ws_bytes : 16);
    ok &= spark_kv_append(kc, vc, cap, kn, vn, B, 1, 0, 0, pos, &cfg, SPARK_ROPE_FUSED, NULL) == SPARK_OK;
    ok &= spark_attn_decode(out, qd, 0, gd, kc, vc, cap, B, pos, &cfg, ws, ws_bytes, SPARK_ROPE_FUSED, NULL) ==
          SPARK_OK;
    ok &= spark_check(NULL) == SPARK_OK;
    ok &= check_half(out, (size_t)B * 16 * 256, kind == SPARK_SLIDING ? "decode sliding" : "decode full");
    if (!ok) printf("last error: %s\n", spark_last_error());
    cudaFree(q); cudaFree(k); cudaFree(v); cudaFree(g); cudaFree(out); cudaFree(kc); cudaFree(vc); cudaFree(ws);
    cudaFree(qd); cudaFree(gd); cudaFree(kn); cudaFree(vn); cudaFree(pos);
  }
  printf(ok ? "c caller ok\n" : "c caller FAILED\n");
  return ok ? 0 : 1;
}
