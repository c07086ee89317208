/*
 * forward_c.c -- the library driven from plain C through include/pkm.h alone: no
 * Python, no PyTorch. Builds a small random bf16 layer on the host, copies it to
 * device buffers from cudaMalloc, runs pkm_workspace_size, pkm_forward and
 * pkm_device_status, and checks what needs no oracle: every pick is a valid slot,
 * picks of a (token, head) are distinct and ordered by kept score, the weights of a
 * (token, head) sum to one, and out is finite.
 *
 *   forward_c        exit 0 on success, 1 on a failed check, 2 on an API error
 */
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "pkm.h"

static uint16_t to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  u += 0x7fffu + ((u >> 16) & 1u); /* round to nearest even */
  return (uint16_t)(u >> 16);
}

static float uniform(uint64_t* s) {
  *s = *s * 6364136223846793005ull + 1442695040888963407ull;
  return (float)((*s >> 40) & 0xffffff) / 16777216.0f - 0.5f;
}

#define CHECK_CUDA(x)                                                   \
  do {                                                                  \
    if ((x) != cudaSuccess) {                                           \
      fprintf(stderr, "CUDA error at %s:%d\n", __FILE__, __LINE__);     \
      return 2;                                                         \
    }                                                                   \
  } while (0)

int main(void) {
  const pkm_shape s = {200, 512, 4, 256, 256, 32, 512, PKM_BF16, 1e-5f};
  const int64_t B = s.B;
  const int F = s.H * s.dq, half = s.dq / 2;
  const size_t nx = (size_t)B * s.d_model, nw = (size_t)F * s.d_model;
  const size_t nc = (size_t)s.H * 2 * s.n * half, nv = (size_t)s.n * s.n * s.v;
  uint16_t* hx = malloc(nx * 2);
  uint16_t* hw = malloc(nw * 2);
  uint16_t* hc = malloc(nc * 2);
  uint16_t* hv = malloc(nv * 2);
  float* hbn = malloc(4 * (size_t)F * sizeof(float));
  if (!hx || !hw || !hc || !hv || !hbn) return 2;
  uint64_t seed = 12345;
  for (size_t i = 0; i < nx; ++i) hx[i] = to_bf16(2.f * uniform(&seed));
  for (size_t i = 0; i < nw; ++i) hw[i] = to_bf16(0.1f * uniform(&seed));
  for (size_t i = 0; i < nc; ++i) hc[i] = to_bf16(0.2f * uniform(&seed));
  for (size_t i = 0; i < nv; ++i) hv[i] = to_bf16(0.1f * uniform(&seed));
  for (int f = 0; f < F; ++f) {
    hbn[f] = 0.f;            /* mean  */
    hbn[F + f] = 1.f;        /* var   */
    hbn[2 * F + f] = 1.f;    /* gamma */
    hbn[3 * F + f] = 0.f;    /* beta  */
  }
  void *dx, *dw, *dc, *dv, *dbn, *dout, *didx, *dwt, *dws;
  const size_t picks = (size_t)B * s.H * s.k;
  const size_t ws_bytes = pkm_workspace_size(&s, 0);
  if (ws_bytes == 0) return 2;
  CHECK_CUDA(cudaMalloc(&dx, nx * 2));
  CHECK_CUDA(cudaMalloc(&dw, nw * 2));
  CHECK_CUDA(cudaMalloc(&dc, nc * 2));
  CHECK_CUDA(cudaMalloc(&dv, nv * 2));
  CHECK_CUDA(cudaMalloc(&dbn, 4 * (size_t)F * sizeof(float)));
  CHECK_CUDA(cudaMalloc(&dout, (size_t)B * s.v * sizeof(float)));
  CHECK_CUDA(cudaMalloc(&didx, picks * sizeof(int32_t)));
  CHECK_CUDA(cudaMalloc(&dwt, picks * sizeof(float)));
  CHECK_CUDA(cudaMalloc(&dws, ws_bytes));
  CHECK_CUDA(cudaMemcpy(dx, hx, nx * 2, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(dw, hw, nw * 2, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(dc, hc, nc * 2, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(dv, hv, nv * 2, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(dbn, hbn, 4 * (size_t)F * sizeof(float), cudaMemcpyHostToDevice));
  const float* bn = (const float*)dbn;
  int rc = pkm_forward(&s, dx, dw, bn, bn + F, bn + 2 * F, bn + 3 * F, dc, dv, (float*)dout,
                       (int32_t*)didx, (float*)dwt, NULL, dws, ws_bytes, NULL);
  if (rc != PKM_OK) {
    fprintf(stderr, "pkm_forward: %s\n", pkm_status_string(rc));
    return 2;
  }
  rc = pkm_device_status(dws, NULL);
  if (rc != PKM_OK) {
    fprintf(stderr, "device status: %s\n", pkm_status_string(rc));
    return 2;
  }
  int32_t* hidx = malloc(picks * sizeof(int32_t));
  float* hwt = malloc(picks * sizeof(float));
  float* hout = malloc((size_t)B * s.v * sizeof(float));
  if (!hidx || !hwt || !hout) return 2;
  CHECK_CUDA(cudaMemcpy(hidx, didx, picks * sizeof(int32_t), cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(hwt, dwt, picks * sizeof(float), cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(hout, dout, (size_t)B * s.v * sizeof(float), cudaMemcpyDeviceToHost));
  int bad = 0;
  for (int64_t th = 0; th < B * s.H; ++th) {
    double wsum = 0.0;
    for (int j = 0; j < s.k; ++j) {
      const int32_t slot = hidx[th * s.k + j];
      if (slot < 0 || slot >= s.n * s.n) ++bad;
      for (int l = 0; l < j; ++l)
        if (hidx[th * s.k + l] == slot) ++bad;
      /* weights are a softmax of scores kept best first: non-increasing */
      if (j > 0 && hwt[th * s.k + j] > hwt[th * s.k + j - 1] * (1.f + 1e-6f)) ++bad;
      wsum += hwt[th * s.k + j];
    }
    if (fabs(wsum - 1.0) > 1e-5) ++bad;
  }
  for (size_t i = 0; i < (size_t)B * s.v; ++i)
    if (!isfinite(hout[i])) ++bad;
  printf("forward_c: %lld tokens, %d failed checks\n", (long long)B, bad);
  cudaFree(dx); cudaFree(dw); cudaFree(dc); cudaFree(dv); cudaFree(dbn);
  cudaFree(dout); cudaFree(didx); cudaFree(dwt); cudaFree(dws);
  free(hx); free(hw); free(hc); free(hv); free(hbn); free(hidx); free(hwt); free(hout);
  return bad ? 1 : 0;
}
