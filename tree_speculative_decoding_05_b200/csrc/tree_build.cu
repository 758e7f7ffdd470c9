// tree_build.cu — best-first draft-tree construction on the GPU.
//
// Sources (page title, section):
//   [Foundation] "Building the Foundation: Architecting a Native CUDA DDTree
//       Inference Engine": "The Single-Threaded Heap Design" (one serial
//       best-first expansion per request, budget <= 64 and depth <= 15 small
//       enough for on-chip memory, the other threads of the block build the
//       visibility rows and retrieve pointers), "Tie-Breaking and Numerical
//       Precision" (equal weights in insertion order, float32 arithmetic),
//       "Assumptions Underlying the Design" (item 4: the sibling weight is the
//       parent-relative expression logw - lp[depth-1][rank] + lp[depth-1][rank+1]
//       evaluated in that order; item 5: candidates can run out before the
//       budget when topk is 1).
//
// The expansion (per request; rows d of lp / tok describe tree depth d+1):
//   node 0 = root (depth 0, logw 0, parent -1, the root token);
//   candidates start with (0 + lp[0][0], depth 1, rank 0, parent 0);
//   while fewer than q_len nodes and a candidate remains: the candidate of
//   largest logw (earliest inserted among equals) becomes the next node n with
//   token tok[d-1][r]; then insert its first child (logw + lp[d][0], d+1, 0, n)
//   if d < D, then its next sibling ((logw - lp[d-1][r]) + lp[d-1][r+1], d,
//   r+1, parent) if r+1 < K.
//
// B200 design.  The expansion is serial in its picks but each pick is a max
// over at most 2*q_len candidates, so one warp per request keeps the candidate
// list spread over its lanes: slot s lives in lane s % 32, register s / 32, and
// slots are handed out in insertion order, so the slot number is the tie-break
// key.  A register holds an order-preserving 32-bit key of the weight (larger
// weight, larger key; equal weights, equal keys; 0 = empty slot); the exact
// weight and the (depth, rank, parent) of each slot sit in shared memory.  A
// pick is a lane-local maximum over the lane's key registers (fully unrolled,
// so the keys never leave registers) and two warp-wide hardware reductions:
// the maximum key, then the smallest slot holding it — no heap, no shuffle tree
// and no memory access before the winner is known.  The kernel is instantiated
// per number of key registers and launched with the fewest that hold a build's
// 2 q_len - 1 slots, so the lane-local maximum and the key updates touch no
// register that can only hold zero (at q_len 33: 3 instead of 8).  The
// log-probs and tokens a build can touch (depth rows < min(D, q_len-1), ranks <
// min(K, q_len)) are staged in shared memory, loaded together and checked for
// finiteness on the way, and the other log-probs are only checked, so no pick
// waits on global memory.  The weights use explicitly rounded float32 adds and
// subtracts (__fadd_rn / __fsub_rn), which the compiler may neither contract
// nor reorder, so the result is bit-identical to any float32 evaluation of the
// same expressions.  A pick's only store is
// the new node's record (weight, depth, rank, parent), by lane 0.  After the
// expansion the lanes derive the retrieve pointers from the parents in one
// pass (a node's first child is the earliest node it parents, its next sibling
// the earliest later node with the same parent), then build, one node each,
// the tokens, the visibility words and the padding, and write everything
// coalesced.
#include <cuda_runtime.h>

#include <climits>
#include <cstdint>

#include "ddt.h"
#include "ddt_internal.h"

namespace ddt {

namespace tb {
// Dynamic shared memory bound: rows < q_len-1, ranks < q_len, float + int each.
constexpr int kMaxStageBytes = (DDT_MAX_Q_LEN - 1) * DDT_MAX_Q_LEN * 8;
// Candidate slots: at most 1 + 2 (q_len - 1) insertions; key registers per lane
// (the kernel is instantiated for 1 .. kMaxKeyRegs registers and launched with
// the fewest that hold 2 q_len - 1 slots).
constexpr int kMaxSlots = 2 * DDT_MAX_Q_LEN;
constexpr int kMaxKeyRegs = kMaxSlots / 32;
static_assert(kMaxSlots % 32 == 0, "whole key registers");
}  // namespace tb

// Order-preserving key of a weight: larger weight, larger key; -0 and +0 map to
// the same key; every key of a non-NaN weight is non-zero (0 marks an empty slot).
__device__ __forceinline__ uint32_t weight_key(float w) {
  uint32_t u = __float_as_uint(w);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Sets key register `reg` of a lane's candidate keys (reg is warp-uniform; the
// unrolled compare keeps every index a constant, so the array stays in registers).
template <int KR>
__device__ __forceinline__ void set_key(uint32_t (&ck)[KR], int reg, uint32_t key) {
#pragma unroll
  for (int j = 0; j < KR; ++j)
    if (j == reg) ck[j] = key;
}

template <int KR>
__global__ void __launch_bounds__(32) tree_build_kernel(
    const float* __restrict__ lp, const int32_t* __restrict__ tok,
    const int32_t* __restrict__ root_token, int D, int K, int q_len, int Dp, int Kp,
    int32_t* __restrict__ parents, int32_t* __restrict__ node_tokens, int32_t* __restrict__ depth,
    float* __restrict__ logw, int32_t* __restrict__ next_token,
    int32_t* __restrict__ next_sibling, uint64_t* __restrict__ mask,
    int32_t* __restrict__ n_nodes, int32_t* __restrict__ status) {
  extern __shared__ __align__(16) unsigned char tb_smem[];
  float* s_lp = reinterpret_cast<float*>(tb_smem);                   // [Dp][Kp]
  int32_t* s_tok = reinterpret_cast<int32_t*>(tb_smem) + Dp * Kp;   // [Dp][Kp]
  // per node: its weight's bits, and depth | rank << 8 | parent << 16 (root: parent -1)
  __shared__ uint2 s_node[DDT_MAX_Q_LEN];
  // per candidate slot: its weight's bits, and depth | rank << 8 | parent << 16
  __shared__ uint2 s_cand[tb::kMaxSlots];

  const int b = blockIdx.x;
  const int lane = threadIdx.x;
  const int64_t DK = static_cast<int64_t>(D) * K;
  const float* L = lp + b * DK;
  const int32_t* T = tok + b * DK;

  const int root = lane == 0 ? root_token[b] : 0;  // used after the expansion
  // Every log-prob must be finite (a NaN would make the arg-max order-dependent).
  // The entries a build can read (rows d < Dp, ranks r < Kp; Dp * Kp < 2^14, so
  // 32-bit indexes) are staged, their log-probs and tokens loaded together; then
  // the rest of each staged row (ranks Kp .. K-1) and the rows from Dp on are
  // only checked.
  bool bad = false;
#pragma unroll 4
  for (int e = lane; e < Dp * Kp; e += 32) {
    const int d = e / Kp, r = e - d * Kp;
    const float v = L[static_cast<int64_t>(d) * K + r];
    s_tok[e] = T[static_cast<int64_t>(d) * K + r];
    bad |= !isfinite(v);
    s_lp[e] = v;
  }
  if (K > Kp) {
    const int Kr = K - Kp;
    for (int64_t e = lane; e < static_cast<int64_t>(Dp) * Kr; e += 32) {
      const int64_t d = e / Kr;
      bad |= !isfinite(L[d * K + Kp + (e - d * Kr)]);
    }
  }
#pragma unroll 4
  for (int64_t e = static_cast<int64_t>(Dp) * K + lane; e < DK; e += 32) bad |= !isfinite(L[e]);
  bad = __any_sync(0xffffffffu, bad);
  if (lane == 0) s_node[0] = make_uint2(0u, 0xffff0000u);  // weight +0, depth 0, parent -1
  __syncwarp();

  // Candidate keys: slot s in lane s % 32, register s / 32 (0 = empty).  Every
  // register index below is a compile-time constant, so ck stays in registers.
  uint32_t ck[KR];
#pragma unroll
  for (int j = 0; j < KR; ++j) ck[j] = 0u;
  int n_slots = 0;
  // Inserts one candidate: its key in the slot's lane, weight and metadata by lane 0.
#define DDT_TB_INSERT(w_, meta_)                                   \
  do {                                                             \
    const int sl_ = n_slots++;                                     \
    const float wv_ = (w_);                                        \
    if (lane == (sl_ & 31)) set_key(ck, sl_ >> 5, weight_key(wv_)); \
    if (lane == 0)                                                 \
      s_cand[sl_] = make_uint2(__float_as_uint(wv_), (meta_));     \
  } while (0)
  if (!bad && q_len > 1) DDT_TB_INSERT(__fadd_rn(0.0f, s_lp[0]), 1 | (0 << 8) | (0 << 16));
  __syncwarp();

  int n = 1;
  while (n < q_len) {
    // Lane-local best: a lane's slots ascend with the register index, so a later
    // equal key never wins.
    uint32_t bk = 0u;
    uint32_t bs = 0xffffffffu;
#pragma unroll
    for (int j = 0; j < KR; ++j) {
      if (ck[j] > bk) {
        bk = ck[j];
        bs = static_cast<uint32_t>(j * 32 + lane);
      }
    }
    const uint32_t kmax = __reduce_max_sync(0xffffffffu, bk);
    if (kmax == 0u) break;  // no candidate left
    const uint32_t win = __reduce_min_sync(0xffffffffu, bk == kmax ? bs : 0xffffffffu);
    if (lane == static_cast<int>(win & 31u)) set_key(ck, static_cast<int>(win >> 5), 0u);
    const uint2 cand = s_cand[win];
    const float bw = __uint_as_float(cand.x);
    const int meta = static_cast<int>(cand.y);
    const int d = meta & 0xff, r = (meta >> 8) & 0xff, par = meta >> 16;
    const int node = n++;
    if (lane == 0) s_node[node] = cand;
    if (n == q_len) break;  // budget reached: nothing more will be picked
    if (d < D) DDT_TB_INSERT(__fadd_rn(bw, s_lp[d * Kp]), (d + 1) | (0 << 8) | (node << 16));
    if (r + 1 < K) {
      const float w = __fadd_rn(__fsub_rn(bw, s_lp[(d - 1) * Kp + r]), s_lp[(d - 1) * Kp + r + 1]);
      DDT_TB_INSERT(w, d | ((r + 1) << 8) | (par << 16));
    }
    __syncwarp();  // the new slots' weights and metadata are visible to every lane
  }
#undef DDT_TB_INSERT
  __syncwarp();

  // Retrieve pointers: node i's first child is the earliest node whose parent is
  // i, its next sibling the earliest later node with i's parent (nodes are
  // numbered in creation order).  Lane l holds nodes l, l + 32, ...; one
  // broadcast read of each node's parent serves every lane.
  constexpr int kNodesPerLane = (KR + 1) / 2;  // q_len <= 16 KR
  int my_par[kNodesPerLane], my_first[kNodesPerLane], my_sib[kNodesPerLane];
#pragma unroll
  for (int k = 0; k < kNodesPerLane; ++k) {
    const int i = lane + 32 * k;
    my_par[k] = i < n ? static_cast<int>(s_node[i].y) >> 16 : -2;
    my_first[k] = -1;
    my_sib[k] = -1;
  }
  for (int j = 1; j < n; ++j) {
    const int pj = static_cast<int>(s_node[j].y) >> 16;
#pragma unroll
    for (int k = 0; k < kNodesPerLane; ++k) {
      const int i = lane + 32 * k;
      if (pj == i && my_first[k] < 0) my_first[k] = j;
      if (j > i && pj == my_par[k] && my_sib[k] < 0) my_sib[k] = j;
    }
  }

  // Per node: padding, retrieve pointers, visibility words; coalesced writes.
  const int W = (q_len + 63) >> 6;
  const int64_t row0 = static_cast<int64_t>(b) * q_len;
#pragma unroll
  for (int k = 0; k < kNodesPerLane; ++k) {
    const int i = lane + 32 * k;
    if (i >= q_len) break;
    int p, t, dd, first = -1, sib = -1;
    float w;
    uint64_t w0 = 0, w1 = 0;
    if (i < n) {
      const uint2 rec = s_node[i];
      const int meta = static_cast<int>(rec.y);
      p = meta >> 16;
      dd = meta & 0xff;
      t = i == 0 ? root : s_tok[(dd - 1) * Kp + ((meta >> 8) & 0xff)];
      w = __uint_as_float(rec.x);
      first = my_first[k];
      sib = my_sib[k];  // -1 for the root, which is no one's child
      for (int a = i, steps = 0; a >= 0 && steps <= i;
           a = static_cast<int>(s_node[a].y) >> 16, ++steps) {
        if (a < 64) w0 |= 1ull << a;
        else w1 |= 1ull << (a - 64);
      }
    } else {
      p = 0;
      t = -1;
      dd = 1;
      w = -INFINITY;
      w0 = 1ull;
      if (i < 64) w0 |= 1ull << i;
      else w1 |= 1ull << (i - 64);
    }
    parents[row0 + i] = p;
    node_tokens[row0 + i] = t;
    next_token[row0 + i] = first;
    next_sibling[row0 + i] = sib;
    if (depth) depth[row0 + i] = dd;
    if (logw) logw[row0 + i] = w;
    if (mask) {
      uint64_t* m = mask + (row0 + i) * W;
      m[0] = w0;
      if (W > 1) m[1] = w1;
    }
  }
  if (lane == 0) {
    if (n_nodes) n_nodes[b] = n;
    if (status) status[b] = bad ? DDT_REQ_BAD_LP : DDT_REQ_OK;
  }
}

size_t tree_build_smem_bytes(int D, int K, int q_len) {
  const int Dp = D < q_len - 1 ? D : q_len - 1;
  const int Kp = K < q_len ? K : q_len;
  return static_cast<size_t>(Dp > 0 ? Dp : 0) * static_cast<size_t>(Kp) * 8;
}

cudaError_t launch_tree_build(const float* lp, const int32_t* tok, const int32_t* root_token,
                              int B, int D, int K, int q_len, int32_t* parents,
                              int32_t* node_tokens, int32_t* depth, float* logw,
                              int32_t* next_token, int32_t* next_sibling, uint64_t* mask,
                              int32_t* n_nodes, int32_t* status, cudaStream_t stream) {
  const int Dp = D < q_len - 1 ? D : q_len - 1;
  const int Kp = K < q_len ? K : q_len;
  const size_t smem = tree_build_smem_bytes(D, K, q_len);
  // the fewest key registers per lane that hold the 2 q_len - 1 candidate slots
  const int kr = (2 * q_len - 1 + 31) / 32;
  using Kernel = void (*)(const float*, const int32_t*, const int32_t*, int, int, int, int, int,
                          int32_t*, int32_t*, int32_t*, float*, int32_t*, int32_t*, uint64_t*,
                          int32_t*, int32_t*);
  static constexpr Kernel kKernels[tb::kMaxKeyRegs] = {
      tree_build_kernel<1>, tree_build_kernel<2>, tree_build_kernel<3>, tree_build_kernel<4>,
      tree_build_kernel<5>, tree_build_kernel<6>, tree_build_kernel<7>, tree_build_kernel<8>};
  static_assert(tb::kMaxKeyRegs == 8, "one instantiation per key-register count");
  if (kr < 1 || kr > tb::kMaxKeyRegs) return cudaErrorInvalidValue;
  const Kernel k = kKernels[kr - 1];
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(k), tb::kMaxStageBytes, 8 + kr - 1);
  if (e != cudaSuccess) return e;
  k<<<B, 32, smem, stream>>>(lp, tok, root_token, D, K, q_len, Dp > 0 ? Dp : 0, Kp, parents,
                             node_tokens, depth, logw, next_token, next_sibling, mask, n_nodes,
                             status);
  return cudaGetLastError();
}

}  // namespace ddt
