/*
 * ddt_context_demo.c — the library used from two CUDA contexts of one device in
 * one process (plain C, driver API for the contexts).  The library remembers
 * two things per context: the address of the no-allocation entry point's
 * scratch array, and the dynamic shared-memory limit it sets on its kernels.
 * A context created after another must get its own lookups, not the first
 * context's.  Each context runs the same split-KV verify call through
 * ddt_verify_attn_noalloc and through ddt_verify_attn with a workspace; the four
 * outputs and log-sum-exps must agree bit for bit (same kernels, same split
 * count, same inputs), every request status must be OK and no fault flag set.
 * Every device pointer is checked to belong to the context it is used in before
 * anything is launched.  Exit status 0 when every check passes.
 */
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "ddt.h"

#define CHECK_CU(x)                                                                \
  do {                                                                             \
    CUresult r_ = (x);                                                             \
    if (r_ != CUDA_SUCCESS) {                                                      \
      fprintf(stderr, "%s:%d driver error %d\n", __FILE__, __LINE__, (int)r_);    \
      return 2;                                                                    \
    }                                                                              \
  } while (0)
#define CHECK_CUDA(x)                                                              \
  do {                                                                             \
    cudaError_t e_ = (x);                                                          \
    if (e_ != cudaSuccess) {                                                       \
      fprintf(stderr, "%s:%d %s\n", __FILE__, __LINE__, cudaGetErrorString(e_));  \
      return 2;                                                                    \
    }                                                                              \
  } while (0)
#define CHECK_DDT(x)                                                               \
  do {                                                                             \
    ddt_status s_ = (x);                                                           \
    if (s_ != DDT_OK) {                                                            \
      fprintf(stderr, "%s:%d %s\n", __FILE__, __LINE__, ddt_status_str(s_));       \
      return 3;                                                                    \
    }                                                                              \
  } while (0)

enum { B = 2, Q = 9, H = 64, DL = 512, DR = 64, CAP = 320, SPLITS = 2 };
#define N_QLAT ((size_t)B * Q * H * DL)
#define N_QROPE ((size_t)B * Q * H * DR)
#define N_CKV ((size_t)B * CAP * DL)
#define N_KR ((size_t)B * CAP * DR)
#define N_OUT ((size_t)B * Q * H * DL)
#define N_ROWS ((size_t)B * Q * H)

static uint16_t h_qlat[N_QLAT], h_qrope[N_QROPE], h_ckv[N_CKV], h_kr[N_KR];
static uint16_t h_out[2][2][N_OUT]; /* [context][entry point] */
static float h_lse[2][2][N_ROWS];

static uint16_t to_bf16(float f) { /* round to nearest even */
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

static void fill(uint16_t* v, size_t n, uint32_t* lcg, float amp) {
  for (size_t k = 0; k < n; ++k) {
    *lcg = *lcg * 1664525u + 1013904223u;
    v[k] = to_bf16((((float)(*lcg >> 8) / 16777216.0f) * 2.0f - 1.0f) * amp);
  }
}

/* 0 when p is memory of context ctx */
static int owned_by(const void* p, CUcontext ctx) {
  CUcontext c = NULL;
  if (cuPointerGetAttribute(&c, CU_POINTER_ATTRIBUTE_CONTEXT, (CUdeviceptr)(uintptr_t)p) !=
      CUDA_SUCCESS)
    return 1;
  return c == ctx ? 0 : 1;
}

/* The same split-KV call through both entry points in the current context. */
static int run_in_context(CUcontext ctx, int ci) {
  const int32_t prefix[B] = {300, 200};
  int32_t parents[B * Q];
  for (int b = 0; b < B; ++b)
    for (int i = 0; i < Q; ++i) parents[b * Q + i] = i == 0 ? -1 : (i - 1) / 2; /* binary tree */

  void *d_qlat, *d_qrope, *d_ckv, *d_kr, *d_out, *d_lse, *d_mask, *d_par, *d_pre, *d_st, *d_ws;
  CHECK_CUDA(cudaMalloc(&d_qlat, N_QLAT * 2));
  CHECK_CUDA(cudaMalloc(&d_qrope, N_QROPE * 2));
  CHECK_CUDA(cudaMalloc(&d_ckv, N_CKV * 2));
  CHECK_CUDA(cudaMalloc(&d_kr, N_KR * 2));
  CHECK_CUDA(cudaMalloc(&d_out, N_OUT * 2));
  CHECK_CUDA(cudaMalloc(&d_lse, N_ROWS * 4));
  CHECK_CUDA(cudaMalloc(&d_mask, (size_t)B * Q * 8));
  CHECK_CUDA(cudaMalloc(&d_par, sizeof parents));
  CHECK_CUDA(cudaMalloc(&d_pre, sizeof prefix));
  CHECK_CUDA(cudaMalloc(&d_st, B * 4));
  const void* mine[] = {d_qlat, d_qrope, d_ckv, d_kr, d_out, d_lse, d_mask, d_par, d_pre, d_st};
  for (size_t k = 0; k < sizeof mine / sizeof mine[0]; ++k)
    if (owned_by(mine[k], ctx)) {
      fprintf(stderr, "context %d: buffer %zu is not memory of this context\n", ci, k);
      return 5;
    }
  CHECK_CUDA(cudaMemcpy(d_qlat, h_qlat, N_QLAT * 2, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(d_qrope, h_qrope, N_QROPE * 2, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(d_ckv, h_ckv, N_CKV * 2, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(d_kr, h_kr, N_KR * 2, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(d_par, parents, sizeof parents, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(d_pre, prefix, sizeof prefix, cudaMemcpyHostToDevice));
  CHECK_DDT(ddt_build_mask((const int32_t*)d_par, B, Q, (uint64_t*)d_mask, NULL, NULL, NULL));

  ddt_attn_args a;
  memset(&a, 0, sizeof a);
  a.B = B;
  a.q_len = Q;
  a.num_heads = H;
  a.d_latent = DL;
  a.d_rope = DR;
  a.capacity = CAP;
  a.prefix_lens = (const int32_t*)d_pre;
  a.q_lat = d_qlat;
  a.q_rope = d_qrope;
  a.c_kv = d_ckv;
  a.k_rope = d_kr;
  a.ckv_batch_stride = (int64_t)CAP * DL;
  a.ckv_row_stride = DL;
  a.kr_batch_stride = (int64_t)CAP * DR;
  a.kr_row_stride = DR;
  a.mask = (const uint64_t*)d_mask;
  a.softmax_scale = 0.0721687836f;
  a.out_dtype = DDT_BF16;
  a.out = d_out;
  a.lse = (float*)d_lse;
  a.max_prefix = 300;
  a.num_splits = SPLITS;
  a.status = (int32_t*)d_st;

  for (int ep = 0; ep < 2; ++ep) {
    int32_t st[B] = {-1, -1};
    CHECK_CUDA(cudaMemset(d_out, 0xff, N_OUT * 2));
    CHECK_CUDA(cudaMemset(d_st, 0xff, B * 4));
    if (ep == 0) {
      CHECK_DDT(ddt_verify_attn_noalloc(&a, NULL));
    } else {
      const size_t ws = ddt_verify_attn_workspace_size(&a);
      if (ws == 0) return 6; /* two splits need partials */
      CHECK_CUDA(cudaMalloc(&d_ws, ws));
      if (owned_by(d_ws, ctx)) return 5;
      a.workspace = d_ws;
      a.workspace_bytes = ws;
      CHECK_DDT(ddt_verify_attn(&a, NULL));
    }
    CHECK_CUDA(cudaDeviceSynchronize());
    CHECK_CUDA(cudaMemcpy(h_out[ci][ep], d_out, N_OUT * 2, cudaMemcpyDeviceToHost));
    CHECK_CUDA(cudaMemcpy(h_lse[ci][ep], d_lse, N_ROWS * 4, cudaMemcpyDeviceToHost));
    CHECK_CUDA(cudaMemcpy(st, d_st, sizeof st, cudaMemcpyDeviceToHost));
    if (st[0] != DDT_REQ_OK || st[1] != DDT_REQ_OK) {
      fprintf(stderr, "context %d entry %d: statuses %d %d\n", ci, ep, st[0], st[1]);
      return 4;
    }
  }
  uint32_t faults = 0;
  CHECK_DDT(ddt_fault_flags(&faults, 1));
  if (faults) {
    fprintf(stderr, "context %d: fault flags %u\n", ci, faults);
    return 4;
  }
  void* all[] = {d_qlat, d_qrope, d_ckv, d_kr, d_out, d_lse, d_mask, d_par, d_pre, d_st, d_ws};
  for (size_t k = 0; k < sizeof all / sizeof all[0]; ++k) CHECK_CUDA(cudaFree(all[k]));
  return 0;
}

int main(void) {
  uint32_t lcg = 2024u;
  fill(h_qlat, N_QLAT, &lcg, 1.0f);
  fill(h_qrope, N_QROPE, &lcg, 1.0f);
  fill(h_ckv, N_CKV, &lcg, 1.0f);
  fill(h_kr, N_KR, &lcg, 1.0f);

  CHECK_CU(cuInit(0));
  CUdevice dev;
  CHECK_CU(cuDeviceGet(&dev, 0));
  CUcontext ctx[2];
  for (int ci = 0; ci < 2; ++ci) {
    CHECK_CU(cuCtxCreate(&ctx[ci], 0, dev)); /* current on this thread from here */
    const int rc = run_in_context(ctx[ci], ci);
    if (rc) return rc;
  }
  /* the first context again, after the second one was used */
  CHECK_CU(cuCtxSetCurrent(ctx[0]));
  {
    const int rc = run_in_context(ctx[0], 0);
    if (rc) return rc;
  }
  for (int ci = 0; ci < 2; ++ci) CHECK_CU(cuCtxDestroy(ctx[ci]));

  size_t diff = 0;
  for (int ci = 0; ci < 2; ++ci)
    for (int ep = 0; ep < 2; ++ep) {
      diff += memcmp(h_out[ci][ep], h_out[0][0], sizeof h_out[0][0]) != 0;
      diff += memcmp(h_lse[ci][ep], h_lse[0][0], sizeof h_lse[0][0]) != 0;
    }
  size_t nonfinite = 0;
  for (size_t k = 0; k < N_OUT; ++k) nonfinite += (h_out[0][0][k] & 0x7f80u) == 0x7f80u;
  printf("%s: two contexts x two entry points, %zu differing results, %zu non-finite outputs\n",
         ddt_version(), diff, nonfinite);
  return (diff == 0 && nonfinite == 0) ? 0 : 1;
}
