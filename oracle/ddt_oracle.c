/*
 * ddt_oracle.c — plain, slow, obviously correct CPU oracle of the tree-verify
 * path.  TEST INFRASTRUCTURE ONLY: it is called by the tests, by the package's
 * smoke check and by the benchmark's CPU-baseline leg, never by the product
 * path.  It shares no code, header or constant with the CUDA library.
 *
 * Attention is done in double precision on inputs that are bfloat16 bit
 * patterns widened exactly; the tree build's weights are float32, the precision
 * the pages fix for them.  Each function follows the written definition of its
 * step, in the order of the definition, with no blocking or fusion.
 *
 * Sources (page title, section):
 *   [Race Conditions] "Race Conditions, Buffer Aliasing, and the Architecture of
 *       a Native DDTree Inference Engine"
 *   [Foundation] "Building the Foundation: Architecting a Native CUDA DDTree
 *       Inference Engine"
 *   [Verdict] "The Microsecond Verdict: Validating a DDTree Kernel Fix Under
 *       Time Pressure"
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC ddt_oracle.c -o libddt_oracle.so -lm
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Status codes, restated here (the oracle includes no library header). */
enum {
  ORC_OK = 0,
  ORC_BAD_PARENT = 1,
  ORC_BAD_INDEX = 2,
  ORC_WALK_LIMIT = 3,
  ORC_BAD_PREFIX = 4,
  ORC_BAD_LENGTH = 5
};

/* bfloat16 bit pattern -> double, exact (bf16 is the top half of a float). */
static double bf16_to_double(uint16_t bits) {
  uint32_t u = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

int oracle_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* Visibility.  [Foundation] "The Single-Threaded Heap Design": the tree      */
/* builder emits a visibility matrix over the tree nodes.  [Race Conditions]  */
/* "The Cache Compaction Problem": nodes are created after their parents, so  */
/* 0 <= parents[i] < i.  Node a is visible to node i iff a is i or one of     */
/* i's ancestors:  vis[i][i] = 1,  vis[i][a] = vis[parents[i]][a] (a != i).   */
/* ------------------------------------------------------------------------ */

/* Explicit Q x Q matrix of one tree.  Returns ORC_OK or ORC_BAD_PARENT; on
 * failure vis is all zero and depth all -1. */
int oracle_visibility(const int32_t* parents, int Q, uint8_t* vis, int32_t* depth) {
  int ok = (Q >= 1) && (parents[0] == -1);
  for (int i = 1; i < Q && ok; ++i)
    if (parents[i] < 0 || parents[i] >= i) ok = 0;
  memset(vis, 0, (size_t)Q * Q);
  if (!ok) {
    if (depth)
      for (int i = 0; i < Q; ++i) depth[i] = -1;
    return ORC_BAD_PARENT;
  }
  for (int i = 0; i < Q; ++i) {  /* ascending i: row parents[i] is complete */
    if (i > 0) {
      int p = parents[i];
      for (int a = 0; a < Q; ++a) vis[(size_t)i * Q + a] = vis[(size_t)p * Q + a];
    }
    vis[(size_t)i * Q + i] = 1;
    if (depth) depth[i] = (i == 0) ? 0 : depth[parents[i]] + 1;
  }
  return ORC_OK;
}

/* Packed bitmask: mask[(b*Q+i)*W + a/64] bit a%64 = vis_b[i][a].
 * Rows of a request with bad parents are all-zero, depths -1. */
void oracle_build_mask(const int32_t* parents, int B, int Q, uint64_t* mask,
                       int32_t* depth, int32_t* status) {
  int W = (Q + 63) / 64;
  uint8_t* vis = (uint8_t*)malloc((size_t)Q * Q);
  for (int b = 0; b < B; ++b) {
    int st = oracle_visibility(parents + (size_t)b * Q, Q, vis,
                               depth ? depth + (size_t)b * Q : NULL);
    if (status) status[b] = st;
    for (int i = 0; i < Q; ++i) {
      for (int w = 0; w < W; ++w) {
        uint64_t word = 0;
        for (int k = 0; k < 64; ++k) {
          int a = w * 64 + k;
          if (a < Q && vis[(size_t)i * Q + a]) word |= (uint64_t)1 << k;
        }
        mask[((size_t)b * Q + i) * W + w] = word;
      }
    }
  }
  free(vis);
}

/* ------------------------------------------------------------------------ */
/* Attention.  [Race Conditions] "The Mission: A Native DDTree Engine":       */
/* tree-verify MLA-absorb attention with visibility masking; "The Cache       */
/* Compaction Problem": the tree block is placed after the prefix, node a at  */
/* cache row P + a.  [Verdict] "The Timeout That Tells a Story": the latent   */
/* KV cache is shared by all heads.  Reading adopted (the pages print no      */
/* formula): absorbed MLA with key = [c_kv | k_rope], query = [q_lat |        */
/* q_rope], value = c_kv; every prefix row is visible; a tree row P + a is    */
/* visible to node i iff vis[i][a].                                           */
/*                                                                            */
/*   s_j = scale * (sum_d q_lat[d] c_kv[j][d] + sum_d q_rope[d] k_rope[j][d]) */
/*   m = max_visible s_j,  Z = sum_visible exp(s_j - m),  p_j = exp(s_j-m)/Z  */
/*   o[d] = sum_visible p_j c_kv[j][d],  lse = m + ln Z                       */
/* ------------------------------------------------------------------------ */

/* One query row.  q points at q_lat[b,i,h,:], qr at q_rope[b,i,h,:]; ckv/kr at
 * row 0 of request b.  vis_row = vis[i][:] (Q entries).  T = P + Q rows.
 * s is scratch of T doubles.  probs (optional, T entries) receives p_j with
 * exact zeros on masked rows. */
static void attn_one_row(const uint16_t* q, const uint16_t* qr, const uint16_t* ckv,
                         const uint16_t* kr, int64_t ckv_rs, int64_t kr_rs, int P, int Q,
                         int DL, int DR, double scale, const uint8_t* vis_row, double* s,
                         double* out, double* lse, double* probs) {
  int T = P + Q;
  double m = -INFINITY;
  for (int j = 0; j < T; ++j) {
    int visible = (j < P) ? 1 : vis_row[j - P];
    if (!visible) {
      s[j] = -INFINITY;
      continue;
    }
    const uint16_t* krow = ckv + (int64_t)j * ckv_rs;
    const uint16_t* rrow = kr + (int64_t)j * kr_rs;
    double dot = 0.0;
    for (int d = 0; d < DL; ++d) dot += bf16_to_double(q[d]) * bf16_to_double(krow[d]);
    for (int d = 0; d < DR; ++d) dot += bf16_to_double(qr[d]) * bf16_to_double(rrow[d]);
    s[j] = scale * dot;
    if (s[j] > m) m = s[j];
  }
  double Z = 0.0;
  for (int j = 0; j < T; ++j)
    if (s[j] != -INFINITY) Z += exp(s[j] - m);
  for (int d = 0; d < DL; ++d) out[d] = 0.0;
  for (int j = 0; j < T; ++j) {
    double p = (s[j] == -INFINITY) ? 0.0 : exp(s[j] - m) / Z;
    if (probs) probs[j] = p;
    if (p == 0.0) continue;
    const uint16_t* vrow = ckv + (int64_t)j * ckv_rs;
    for (int d = 0; d < DL; ++d) out[d] += p * bf16_to_double(vrow[d]);
  }
  *lse = m + log(Z);
}

/* Attention for a list of query rows.  rows[k] = (b*Q + i)*H + h.
 * Layouts: q_lat [B,Q,H,DL], q_rope [B,Q,H,DR] contiguous; cache row r of
 * request b at c_kv + b*ckv_bs + r*ckv_rs (elements), same for k_rope.
 * out [n_rows, DL], lse [n_rows]; probs NULL or [n_rows, probs_stride] with
 * probs_stride >= P_b + Q.  Returns 0, or -1 if a request's parents are bad
 * or a prefix is negative (those rows are filled with NaN). */
int oracle_attn_rows(const uint16_t* q_lat, const uint16_t* q_rope, const uint16_t* c_kv,
                     const uint16_t* k_rope, int64_t ckv_bs, int64_t ckv_rs, int64_t kr_bs,
                     int64_t kr_rs, const int32_t* prefix_lens, const int32_t* parents, int B,
                     int Q, int H, int DL, int DR, float softmax_scale, const int64_t* rows,
                     int64_t n_rows, double* out, double* lse, double* probs,
                     int64_t probs_stride, int nthreads) {
  int bad = 0;
  double scale = (double)softmax_scale;
  if (nthreads <= 0) nthreads = oracle_threads();
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads) reduction(| : bad)
#endif
  for (int64_t k = 0; k < n_rows; ++k) {
    int64_t row = rows[k];
    int b = (int)(row / ((int64_t)Q * H));
    int i = (int)((row / H) % Q);
    int h = (int)(row % H);
    int P = prefix_lens[b];
    uint8_t* vis = (uint8_t*)malloc((size_t)Q * Q);
    int st = oracle_visibility(parents + (size_t)b * Q, Q, vis, NULL);
    if (st != ORC_OK || P < 0) {
      for (int d = 0; d < DL; ++d) out[k * DL + d] = NAN;
      lse[k] = NAN;
      bad |= 1;
      free(vis);
      continue;
    }
    double* s = (double*)malloc(sizeof(double) * (size_t)(P + Q));
    const uint16_t* q = q_lat + (((int64_t)b * Q + i) * H + h) * DL;
    const uint16_t* qr = q_rope + (((int64_t)b * Q + i) * H + h) * DR;
    attn_one_row(q, qr, c_kv + (int64_t)b * ckv_bs, k_rope + (int64_t)b * kr_bs, ckv_rs, kr_rs,
                 P, Q, DL, DR, scale, vis + (size_t)i * Q, s, out + k * DL, lse + k,
                 probs ? probs + k * probs_stride : NULL);
    free(s);
    free(vis);
  }
  return bad ? -1 : 0;
}

/* ------------------------------------------------------------------------ */
/* Greedy accept.  [Verdict] "The Crash That Demanded a Fix": the walk        */
/* follows next_token / next_sibling pointers and is bounded by q_len; "What  */
/* Was Learned": greedy acceptance, bound `alen >= q_len`.  [Race Conditions] */
/* "The Cache Compaction Problem": the path starts at the root, node 0.       */
/* Steps, per request:                                                        */
/*   path[0]=0, alen=1, cur=0, examined=0                                     */
/*   loop: stop if alen >= Q; c = next_token[cur];                            */
/*         while c != -1: (c outside [0,Q) -> BAD_INDEX, stop)                */
/*                        examined += 1 (> Q -> WALK_LIMIT, stop)             */
/*                        if node_tokens[c] == target_tokens[cur]: accept c   */
/*                        c = next_sibling[c]                                 */
/*         none accepted -> stop; else path[alen++] = c, cur = c              */
/*   bonus = target_tokens[cur]; path[alen..Q) = -1                           */
/* ------------------------------------------------------------------------ */
void oracle_tree_accept(const int32_t* node_tokens, const int32_t* target_tokens,
                        const int32_t* next_token, const int32_t* next_sibling, int B, int Q,
                        int32_t* path, int32_t* accept_len, int32_t* bonus, int32_t* status) {
  for (int b = 0; b < B; ++b) {
    const int32_t* tok = node_tokens + (size_t)b * Q;
    const int32_t* tgt = target_tokens + (size_t)b * Q;
    const int32_t* first = next_token + (size_t)b * Q;
    const int32_t* sib = next_sibling + (size_t)b * Q;
    int32_t* pth = path + (size_t)b * Q;
    int alen = 1, cur = 0, examined = 0, st = ORC_OK;
    pth[0] = 0;
    while (alen < Q) {
      int c = first[cur];
      int found = -1;
      while (c != -1) {
        if (c < 0 || c >= Q) {
          st = ORC_BAD_INDEX;
          break;
        }
        examined += 1;
        if (examined > Q) {
          st = ORC_WALK_LIMIT;
          break;
        }
        if (tok[c] == tgt[cur]) {
          found = c;
          break;
        }
        c = sib[c];
      }
      if (st != ORC_OK || found == -1) break;
      pth[alen++] = found;
      cur = found;
    }
    for (int k = alen; k < Q; ++k) pth[k] = -1;
    accept_len[b] = alen;
    if (bonus) bonus[b] = tgt[cur];
    if (status) status[b] = st;
  }
}

/* ------------------------------------------------------------------------ */
/* Compaction.  [Race Conditions] "The Cache Compaction Problem": gather the  */
/* kept rows of the appended tree block into a contiguous prefix:             */
/*   new row P+i = old row P+keep[i] for i < alen (keep = path); other rows   */
/*   unchanged; new prefix = P + alen.                                        */
/* Done as the pages' two-step scheme: gather into scratch, then copy back.   */
/* Rows are bit patterns of width DL (c_kv) and DR (k_rope).                  */
/* ------------------------------------------------------------------------ */
void oracle_kv_compact(uint16_t* c_kv, uint16_t* k_rope, int64_t ckv_bs, int64_t ckv_rs,
                       int64_t kr_bs, int64_t kr_rs, int capacity, int DL, int DR,
                       const int32_t* prefix_lens, const int32_t* path,
                       const int32_t* accept_len, int B, int Q, int32_t* new_prefix_lens,
                       int32_t* status) {
  for (int b = 0; b < B; ++b) {
    int P = prefix_lens[b];
    int alen = accept_len[b];
    const int32_t* keep = path + (size_t)b * Q;
    int st = ORC_OK;
    if (alen < 1 || alen > Q) st = ORC_BAD_LENGTH;
    else if (P < 0 || P + Q > capacity) st = ORC_BAD_PREFIX;
    else
      for (int i = 0; i < alen; ++i)
        if (keep[i] < 0 || keep[i] >= Q) st = ORC_BAD_INDEX;
    if (status) status[b] = st;
    if (st != ORC_OK) {
      if (new_prefix_lens) new_prefix_lens[b] = P;
      continue;
    }
    uint16_t* s_ckv = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)alen * DL);
    uint16_t* s_kpe = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)alen * DR);
    uint16_t* ckv = c_kv + (int64_t)b * ckv_bs;
    uint16_t* kr = k_rope + (int64_t)b * kr_bs;
    for (int i = 0; i < alen; ++i) { /* step 1: gather into scratch */
      memcpy(s_ckv + (size_t)i * DL, ckv + (int64_t)(P + keep[i]) * ckv_rs, sizeof(uint16_t) * DL);
      memcpy(s_kpe + (size_t)i * DR, kr + (int64_t)(P + keep[i]) * kr_rs, sizeof(uint16_t) * DR);
    }
    for (int i = 0; i < alen; ++i) { /* step 2: copy back */
      memcpy(ckv + (int64_t)(P + i) * ckv_rs, s_ckv + (size_t)i * DL, sizeof(uint16_t) * DL);
      memcpy(kr + (int64_t)(P + i) * kr_rs, s_kpe + (size_t)i * DR, sizeof(uint16_t) * DR);
    }
    free(s_ckv);
    free(s_kpe);
    if (new_prefix_lens) new_prefix_lens[b] = P + alen;
  }
}

/* ------------------------------------------------------------------------ */
/* Tree build.  [Foundation] "The Single-Threaded Heap Design" (best-first     */
/* expansion of a draft tree from per-depth top-k log-probabilities, budget   */
/* and depth bounded), "Tie-Breaking and Numerical Precision" (equal weights  */
/* are taken in insertion order; float32 arithmetic), "Assumptions Underlying */
/* the Design" (4: the sibling weight is the parent-relative expression       */
/* logw - lp[depth-1][rank] + lp[depth-1][rank+1], in that order; 5: with     */
/* topk = 1 the candidates can run out before the budget).                    */
/*                                                                            */
/* Per request: lp[d][r], tok[d][r] for d < D, r < K (row d describes tree    */
/* depth d+1), and the root's token.  Node 0 is the root: depth 0, logw 0,    */
/* parent -1.  A candidate is (logw, depth d, rank r, parent).  The first     */
/* candidate is (0 + lp[0][0], 1, 0, 0).  While fewer than Q nodes exist and  */
/* a candidate remains: take the candidate of largest logw (among equals the  */
/* one inserted first); it becomes the next node n with that parent, depth,   */
/* logw and token tok[d-1][r].  Then insert, first                            */
/*   its first child  (logw + lp[d][0], d+1, 0, n)                 if d < D,  */
/* then                                                                       */
/*   its next sibling ((logw - lp[d-1][r]) + lp[d-1][r+1], d, r+1, parent)   */
/*                                                                 if r+1 < K.*/
/* logw arithmetic is binary32 with round-to-nearest, in the order shown.     */
/*                                                                            */
/* Retrieve pointers: next_token[i] = smallest child index of i, next_sibling */
/* [i] = next larger node index with the same parent (-1 where none).         */
/* Slots n_nodes <= i < Q (when candidates ran out) are padding: parent 0,    */
/* token -1, depth 1, logw -inf, linked into no list.  Every lp entry must be */
/* finite, else status BAD_LP and the tree is the root alone plus padding.    */
/* The candidate list is kept in insertion order (removal shifts the rest),   */
/* so the first maximum found by a scan is the earliest inserted one.         */
/* ------------------------------------------------------------------------ */
enum { ORC_BAD_LP = 6 };

typedef struct {
  float logw;
  int depth, rank, parent;
} orc_candidate;

void oracle_tree_build(const float* lp, const int32_t* tok, const int32_t* root_token, int B,
                       int D, int K, int Q, int32_t* parents, int32_t* node_tokens,
                       int32_t* depth, float* logw, int32_t* next_token, int32_t* next_sibling,
                       int32_t* n_nodes, int32_t* status) {
  orc_candidate* cand = (orc_candidate*)malloc(sizeof(orc_candidate) * (size_t)(2 * Q + 2));
  for (int b = 0; b < B; ++b) {
    const float* L = lp + (size_t)b * D * K;
    const int32_t* T = tok + (size_t)b * D * K;
    int32_t* par = parents + (size_t)b * Q;
    int32_t* ntk = node_tokens + (size_t)b * Q;
    int32_t* dep = depth + (size_t)b * Q;
    float* lw = logw + (size_t)b * Q;
    int32_t* first = next_token + (size_t)b * Q;
    int32_t* sib = next_sibling + (size_t)b * Q;
    int st = ORC_OK;
    for (int e = 0; e < D * K; ++e)
      if (!isfinite(L[e])) st = ORC_BAD_LP;

    par[0] = -1;
    ntk[0] = root_token[b];
    dep[0] = 0;
    lw[0] = 0.0f;
    int n = 1, ncand = 0;
    if (st == ORC_OK && Q > 1) {
      float root_w = 0.0f;
      cand[ncand++] = (orc_candidate){root_w + L[0], 1, 0, 0};
    }
    while (n < Q && ncand > 0) {
      int best = 0;
      for (int c = 1; c < ncand; ++c)
        if (cand[c].logw > cand[best].logw) best = c;
      orc_candidate x = cand[best];
      memmove(cand + best, cand + best + 1, sizeof(orc_candidate) * (size_t)(ncand - best - 1));
      ncand -= 1;
      const int node = n++;
      par[node] = x.parent;
      ntk[node] = T[(size_t)(x.depth - 1) * K + x.rank];
      dep[node] = x.depth;
      lw[node] = x.logw;
      if (x.depth < D) {
        float w = x.logw + L[(size_t)x.depth * K + 0];
        cand[ncand++] = (orc_candidate){w, x.depth + 1, 0, node};
      }
      if (x.rank + 1 < K) {
        float w = x.logw - L[(size_t)(x.depth - 1) * K + x.rank];
        w = w + L[(size_t)(x.depth - 1) * K + x.rank + 1];
        cand[ncand++] = (orc_candidate){w, x.depth, x.rank + 1, x.parent};
      }
    }
    for (int i = n; i < Q; ++i) {
      par[i] = 0;
      ntk[i] = -1;
      dep[i] = 1;
      lw[i] = -INFINITY;
    }
    for (int i = 0; i < Q; ++i) first[i] = sib[i] = -1;
    for (int i = 1; i < n; ++i) { /* children in ascending index */
      int p = par[i];
      if (first[p] == -1) {
        first[p] = i;
      } else {
        int c = first[p];
        while (sib[c] != -1) c = sib[c];
        sib[c] = i;
      }
    }
    if (n_nodes) n_nodes[b] = n;
    if (status) status[b] = st;
  }
  free(cand);
}
