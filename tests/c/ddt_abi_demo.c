/*
 * ddt_abi_demo.c — the library driven from plain C (no Python, no torch): build
 * the visibility mask of a chain tree, run tree-verify attention with all-zero
 * queries, and walk the tree.  With q = 0 every visible key has score 0, so each
 * output row is the plain mean of the visible c_kv rows (a closed form the test
 * computes here in double), and the lse is ln(number of visible rows).
 * Exit status 0 when every check passes.
 */
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "ddt.h"

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

enum { B = 2, Q = 9, H = 64, DL = 512, DR = 64, CAP = 160 };

static uint16_t to_bf16(float f) { /* round to nearest even */
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}
static double from_bf16(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

int main(void) {
  const int32_t prefix[B] = {100, 37};
  static uint16_t ckv[B * CAP * DL], kr[B * CAP * DR];
  uint32_t lcg = 12345u;
  for (size_t k = 0; k < sizeof ckv / 2; ++k) {
    lcg = lcg * 1664525u + 1013904223u;
    ckv[k] = to_bf16(((float)(lcg >> 8) / 16777216.0f) * 2.0f - 1.0f);
  }
  for (size_t k = 0; k < sizeof kr / 2; ++k) kr[k] = to_bf16(0.25f);
  int32_t parents[B * Q];
  for (int b = 0; b < B; ++b)
    for (int i = 0; i < Q; ++i) parents[b * Q + i] = i - 1; /* a chain */

  void *d_qlat, *d_qrope, *d_ckv, *d_kr, *d_out, *d_lse, *d_mask, *d_par, *d_pre, *d_st;
  CHECK_CUDA(cudaMalloc(&d_qlat, (size_t)B * Q * H * DL * 2));
  CHECK_CUDA(cudaMalloc(&d_qrope, (size_t)B * Q * H * DR * 2));
  CHECK_CUDA(cudaMalloc(&d_ckv, sizeof ckv));
  CHECK_CUDA(cudaMalloc(&d_kr, sizeof kr));
  CHECK_CUDA(cudaMalloc(&d_out, (size_t)B * Q * H * DL * 4));
  CHECK_CUDA(cudaMalloc(&d_lse, (size_t)B * Q * H * 4));
  CHECK_CUDA(cudaMalloc(&d_mask, (size_t)B * Q * 8));
  CHECK_CUDA(cudaMalloc(&d_par, sizeof parents));
  CHECK_CUDA(cudaMalloc(&d_pre, sizeof prefix));
  CHECK_CUDA(cudaMalloc(&d_st, B * 4));
  CHECK_CUDA(cudaMemset(d_qlat, 0, (size_t)B * Q * H * DL * 2));
  CHECK_CUDA(cudaMemset(d_qrope, 0, (size_t)B * Q * H * DR * 2));
  CHECK_CUDA(cudaMemcpy(d_ckv, ckv, sizeof ckv, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(d_kr, kr, sizeof kr, cudaMemcpyHostToDevice));
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
  a.out_dtype = DDT_F32;
  a.out = d_out;
  a.lse = (float*)d_lse;
  a.max_prefix = 100;
  a.num_splits = 1; /* no workspace needed */
  a.status = (int32_t*)d_st;
  CHECK_DDT(ddt_verify_attn(&a, NULL));
  CHECK_CUDA(cudaDeviceSynchronize());

  float* out = (float*)malloc((size_t)B * Q * H * DL * 4);
  float lse[B * Q * H];
  int32_t st[B];
  CHECK_CUDA(cudaMemcpy(out, d_out, (size_t)B * Q * H * DL * 4, cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(lse, d_lse, sizeof lse, cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(st, d_st, sizeof st, cudaMemcpyDeviceToHost));
  double worst = 0.0, worst_lse = 0.0;
  for (int b = 0; b < B; ++b) {
    if (st[b] != DDT_REQ_OK) return 4;
    for (int i = 0; i < Q; ++i) {
      const int visible = prefix[b] + i + 1; /* the prefix and nodes 0..i of the chain */
      for (int d = 0; d < DL; ++d) {
        double mean = 0.0;
        for (int j = 0; j < visible; ++j) mean += from_bf16(ckv[((size_t)b * CAP + j) * DL + d]);
        mean /= visible;
        for (int h = 0; h < H; ++h) {
          const double e = fabs(out[(((size_t)b * Q + i) * H + h) * DL + d] - mean);
          if (e > worst) worst = e;
        }
      }
      for (int h = 0; h < H; ++h) {
        const double e = fabs(lse[(b * Q + i) * H + h] - log((double)visible));
        if (e > worst_lse) worst_lse = e;
      }
    }
  }

  /* the accept walk on the chain: targets follow nodes 1..4, then miss */
  int32_t tok[B * Q], tgt[B * Q], first[B * Q], sib[B * Q];
  for (int b = 0; b < B; ++b)
    for (int i = 0; i < Q; ++i) {
      tok[b * Q + i] = 1000 + i;
      tgt[b * Q + i] = i < 4 ? 1000 + i + 1 : 7;
      first[b * Q + i] = i + 1 < Q ? i + 1 : -1;
      sib[b * Q + i] = -1;
    }
  void *d_tok, *d_tgt, *d_first, *d_sib, *d_path, *d_alen;
  CHECK_CUDA(cudaMalloc(&d_tok, sizeof tok));
  CHECK_CUDA(cudaMalloc(&d_tgt, sizeof tgt));
  CHECK_CUDA(cudaMalloc(&d_first, sizeof first));
  CHECK_CUDA(cudaMalloc(&d_sib, sizeof sib));
  CHECK_CUDA(cudaMalloc(&d_path, sizeof tok));
  CHECK_CUDA(cudaMalloc(&d_alen, B * 4));
  CHECK_CUDA(cudaMemcpy(d_tok, tok, sizeof tok, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(d_tgt, tgt, sizeof tgt, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(d_first, first, sizeof first, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(d_sib, sib, sizeof sib, cudaMemcpyHostToDevice));
  CHECK_DDT(ddt_tree_accept((const int32_t*)d_tok, (const int32_t*)d_tgt,
                            (const int32_t*)d_first, (const int32_t*)d_sib, B, Q,
                            (int32_t*)d_path, (int32_t*)d_alen, NULL, NULL, NULL));
  int32_t alen[B];
  CHECK_CUDA(cudaMemcpy(alen, d_alen, sizeof alen, cudaMemcpyDeviceToHost));
  uint32_t faults = 0;
  CHECK_DDT(ddt_fault_flags(&faults, 1));

  printf("%s: out max-abs %.3g, lse max-abs %.3g, accept_len %d %d, faults %u\n", ddt_version(),
         worst, worst_lse, alen[0], alen[1], faults);
  free(out);
  return (worst <= 1e-4 && worst_lse <= 1e-4 && alen[0] == 5 && alen[1] == 5 && faults == 0) ? 0
                                                                                            : 1;
}
