// companions.cu — the integer kernels of the tree-verify step: visibility mask,
// greedy tree accept, and KV-cache compaction.  All three are bit-exact by
// construction (pure integer / bit-copy work) and bounded on any input.
//
// Sources (page title, section):
//   [Race Conditions] "Race Conditions, Buffer Aliasing, and the Architecture of
//       a Native DDTree Inference Engine"
//   [Foundation] "Building the Foundation: Architecting a Native CUDA DDTree
//       Inference Engine"
//   [Verdict] "The Microsecond Verdict: Validating a DDTree Kernel Fix Under
//       Time Pressure"
#include <cuda_runtime.h>

#include <cstdint>

#include "ddt.h"
#include "ddt_internal.h"

namespace ddt {

// ---------------------------------------------------------------------------
// Visibility mask.  [Foundation] "The Single-Threaded Heap Design": the block's
// threads build the visibility matrix in parallel; [Race Conditions] "The
// Cache Compaction Problem": parents precede children.  One CTA per request,
// thread i builds row i by walking i's parent chain (at most i steps once the
// parents are validated, since parents[k] < k).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) build_mask_kernel(const int32_t* __restrict__ parents,
                                                         int q_len, uint64_t* __restrict__ mask,
                                                         int32_t* __restrict__ depth,
                                                         int32_t* __restrict__ status) {
  __shared__ int32_t s_par[DDT_MAX_Q_LEN];
  const int b = blockIdx.x;
  const int i = threadIdx.x;
  const int W = (q_len + 63) >> 6;
  int ok = 1;
  if (i < q_len) {
    const int32_t p = parents[static_cast<int64_t>(b) * q_len + i];
    s_par[i] = p;
    ok = (i == 0) ? (p == -1) : (p >= 0 && p < i);
  }
  const int all_ok = __syncthreads_and(ok);
  if (i >= q_len) return;
  uint64_t w0 = 0, w1 = 0;
  int d = -1;
  if (all_ok) {
    int a = i;
    d = 0;
    for (int step = 0; step <= i; ++step) {  // bounded: the chain strictly decreases
      if (a < 64) w0 |= 1ull << a;
      else w1 |= 1ull << (a - 64);
      if (a == 0) break;
      a = s_par[a];
      ++d;
    }
  }
  uint64_t* row = mask + (static_cast<int64_t>(b) * q_len + i) * W;
  row[0] = w0;
  if (W > 1) row[1] = w1;
  if (depth) depth[static_cast<int64_t>(b) * q_len + i] = d;
  if (status && i == 0) status[b] = all_ok ? DDT_REQ_OK : DDT_REQ_BAD_PARENT;
}

// ---------------------------------------------------------------------------
// Greedy accept.  [Verdict] "The Crash That Demanded a Fix" and "What Was
// Learned": follow the first-child / next-sibling retrieve pointers, accept the
// child whose draft token equals the target's greedy token, stop on a miss or
// once the path holds q_len nodes.  The pages' crash came from a walk over
// cyclic pointers; here every examined node counts against q_len, and pointers
// are range-checked before use, so the walk ends on any input.
// One warp per request: the warp stages the request's four arrays in shared
// memory, lane 0 walks, and the warp writes the padded path back.
// ---------------------------------------------------------------------------
constexpr int kAcceptWarps = 4;

// The walk itself, on one request's arrays in shared memory (one thread).
// path[0 .. alen) receives the accepted nodes (the caller pre-fills -1);
// returns the status, with alen and the last accepted node `cur`.
__device__ int accept_walk(const int32_t* tok, const int32_t* tgt, const int32_t* first,
                           const int32_t* sib, int q_len, int32_t* path, int& alen, int& cur) {
  int examined = 0, st = DDT_REQ_OK;
  alen = 1;
  cur = 0;
  path[0] = 0;
  while (alen < q_len) {
    int c = first[cur];
    int found = -1;
    while (c != -1) {
      if (c < 0 || c >= q_len) {
        st = DDT_REQ_BAD_INDEX;
        break;
      }
      if (++examined > q_len) {
        st = DDT_REQ_WALK_LIMIT;
        break;
      }
      if (tok[c] == tgt[cur]) {
        found = c;
        break;
      }
      c = sib[c];
    }
    if (st != DDT_REQ_OK || found == -1) break;
    path[alen++] = found;
    cur = found;
  }
  return st;
}

__global__ void __launch_bounds__(kAcceptWarps * 32) tree_accept_kernel(
    const int32_t* __restrict__ node_tokens, const int32_t* __restrict__ target_tokens,
    const int32_t* __restrict__ next_token, const int32_t* __restrict__ next_sibling, int B,
    int q_len, int32_t* __restrict__ path, int32_t* __restrict__ accept_len,
    int32_t* __restrict__ bonus_token, int32_t* __restrict__ status) {
  __shared__ int32_t s_tok[kAcceptWarps][DDT_MAX_Q_LEN];
  __shared__ int32_t s_tgt[kAcceptWarps][DDT_MAX_Q_LEN];
  __shared__ int32_t s_first[kAcceptWarps][DDT_MAX_Q_LEN];
  __shared__ int32_t s_sib[kAcceptWarps][DDT_MAX_Q_LEN];
  __shared__ int32_t s_path[kAcceptWarps][DDT_MAX_Q_LEN];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int b = blockIdx.x * kAcceptWarps + warp;
  if (b >= B) return;
  const int64_t base = static_cast<int64_t>(b) * q_len;
  for (int k = lane; k < q_len; k += 32) {
    s_tok[warp][k] = node_tokens[base + k];
    s_tgt[warp][k] = target_tokens[base + k];
    s_first[warp][k] = next_token[base + k];
    s_sib[warp][k] = next_sibling[base + k];
    s_path[warp][k] = -1;
  }
  __syncwarp();
  if (lane == 0) {
    int alen, cur;
    const int st = accept_walk(s_tok[warp], s_tgt[warp], s_first[warp], s_sib[warp], q_len,
                               s_path[warp], alen, cur);
    accept_len[b] = alen;
    if (bonus_token) bonus_token[b] = s_tgt[warp][cur];
    if (status) status[b] = st;
  }
  __syncwarp();
  for (int k = lane; k < q_len; k += 32) path[base + k] = s_path[warp][k];
}

// ---------------------------------------------------------------------------
// Compaction.  [Race Conditions] "The Cache Compaction Problem": row P+i takes
// old row P+keep[i].  A parallel in-place gather races when keep[j] = i' (row
// i' read by one thread while another writes it); the pages route the gather
// through scratch buffers.  Here a write can only clobber the same bytes of a
// row that some index reads, and a row's column ranges never alias, so each
// row (latent then rope, 72 vectors of 16 bytes) is cut into kCompactSlices
// column slices of kSliceVec vectors and one CTA owns one slice of one request:
// it reads that slice of every moving row into shared memory, synchronises, and
// only then writes it.  No write precedes a read of the same bytes, for any
// path, without scratch memory.  The slices of a request are one thread-block
// cluster; a cluster barrier after every CTA has read the request's prefix
// length lets the first slice publish the new prefix length even when
// new_prefix_lens aliases prefix_lens.  A slice stages at most 128 x 288 bytes
// (36 KB), so several CTAs share an SM and one request's reads overlap
// another's writes.  Rows that do not move (keep[i] == i) are not rewritten.
// ---------------------------------------------------------------------------
#ifndef DDT_COMPACT_THREADS
#define DDT_COMPACT_THREADS 256
#endif
#ifndef DDT_COMPACT_SLICES
#define DDT_COMPACT_SLICES 4
#endif
constexpr int kCompactThreads = DDT_COMPACT_THREADS;
constexpr int kLatVec = DDT_D_LATENT * 2 / 16;  // 16-byte vectors per latent row (64)
constexpr int kRopeVec = DDT_D_ROPE * 2 / 16;   // per rope row (8)
constexpr int kRowVec = kLatVec + kRopeVec;
constexpr int kCompactSlices = DDT_COMPACT_SLICES;  // a cluster: at most 8
constexpr int kSliceVec = kRowVec / kCompactSlices;  // 4 slices: 18 vectors = 288 bytes
static_assert(kSliceVec * kCompactSlices == kRowVec, "row slices cover the row");
static_assert(kSliceVec % 2 == 0, "a slice is whole 32-byte sectors");
static_assert(kCompactSlices <= 8, "the slices of a request form one portable cluster");

__device__ __forceinline__ void compact_cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
               "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Asynchronous 16-byte copy global -> shared (cp.async, L2 only): a thread can have
// all of its copies in flight at once instead of one load per loop iteration.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gmem_src) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// Moves slice `slice` (row vectors [slice * kSliceVec, + kSliceVec)) of rows
// P+keep[i] -> P+i (i < alen) of request b, both caches, through shared memory:
// the slice of every moving row is read before any is written.  Called by all
// kCompactThreads threads of the CTA; s_rows holds alen * kSliceVec vectors.
__device__ void compact_rows(uint16_t* __restrict__ c_kv, uint16_t* __restrict__ k_rope,
                             int64_t ckv_bs, int64_t ckv_rs, int64_t kr_bs, int64_t kr_rs, int b,
                             int P, int alen, const int32_t* s_keep, uint4* s_rows, int slice) {
  const uint4* ckv_b = reinterpret_cast<const uint4*>(c_kv + b * ckv_bs);
  const uint4* kr_b = reinterpret_cast<const uint4*>(k_rope + b * kr_bs);
  const int64_t ckv_rv = ckv_rs / 8, kr_rv = kr_rs / 8;  // row strides in 16-byte vectors
  const int total = alen * kSliceVec;
  const int v0 = slice * kSliceVec;
  // Phase 1: the slice of every moving row into shared memory, all copies in
  // flight together.
  for (int idx = threadIdx.x; idx < total; idx += kCompactThreads) {
    const int i = idx / kSliceVec, v = v0 + (idx - i * kSliceVec);
    if (s_keep[i] == i) continue;
    const int64_t src_row = P + s_keep[i];
    cp_async16(&s_rows[idx], (v < kLatVec) ? ckv_b + (src_row * ckv_rv + v)
                                           : kr_b + (src_row * kr_rv + (v - kLatVec)));
  }
  cp_async_wait_all();
  __syncthreads();
  // Phase 2: write the slice of rows P .. P+alen-1 (only those that move).
  uint4* ckv_w = reinterpret_cast<uint4*>(c_kv + b * ckv_bs);
  uint4* kr_w = reinterpret_cast<uint4*>(k_rope + b * kr_bs);
  for (int idx = threadIdx.x; idx < total; idx += kCompactThreads) {
    const int i = idx / kSliceVec, v = v0 + (idx - i * kSliceVec);
    if (s_keep[i] == i) continue;
    const int64_t dst_row = P + i;
    if (v < kLatVec) ckv_w[dst_row * ckv_rv + v] = s_rows[idx];
    else kr_w[dst_row * kr_rv + (v - kLatVec)] = s_rows[idx];
  }
}

// Grid: kCompactSlices CTAs per request, CTA b * kCompactSlices + s moving
// slice s of request b.  kInPlace (new_prefix_lens overlaps prefix_lens): the
// slices of a request are launched as one cluster and wait at a cluster barrier
// until all of them have read the prefix length that slice 0 then overwrites.
// Otherwise no CTA writes anything another reads, and the CTAs are independent
// (measured 5-13 % faster than clustered at 1024 requests x q_len 128).
template <bool kInPlace>
__global__ void __launch_bounds__(kCompactThreads)
    kv_compact_kernel(uint16_t* __restrict__ c_kv, uint16_t* __restrict__ k_rope, int64_t ckv_bs,
                      int64_t ckv_rs, int64_t kr_bs, int64_t kr_rs, int capacity,
                      const int32_t* prefix_lens, const int32_t* __restrict__ path,
                      const int32_t* __restrict__ accept_len, int q_len, int32_t* new_prefix_lens,
                      int32_t* __restrict__ status) {
  extern __shared__ uint4 s_rows[];  // [alen][kSliceVec]
  __shared__ int32_t s_keep[DDT_MAX_Q_LEN];
  static_assert(DDT_MAX_Q_LEN <= kCompactThreads, "one thread per path entry");
  const int b = blockIdx.x / kCompactSlices;
  const int slice = blockIdx.x % kCompactSlices;
  const int t = threadIdx.x;
  // The prefix length, the accepted length and the whole path row are loaded
  // together (one memory latency before the row copies can be addressed).
  const int P = prefix_lens[b];
  const int alen = accept_len[b];
  const int k = (t < q_len) ? path[static_cast<int64_t>(b) * q_len + t] : 0;
  int st = DDT_REQ_OK;
  if (alen < 1 || alen > q_len) st = DDT_REQ_BAD_LENGTH;
  else if (P < 0 || static_cast<int64_t>(P) + q_len > capacity) st = DDT_REQ_BAD_PREFIX;
  if (t < q_len) s_keep[t] = k;
  const int bad = (st == DDT_REQ_OK) && t < alen && (k < 0 || k >= q_len);
  if (__syncthreads_or(bad) && st == DDT_REQ_OK) st = DDT_REQ_BAD_INDEX;
  // Every slice has read P (and the same path, so the same verdict).
  if constexpr (kInPlace) compact_cluster_sync();
  if (st != DDT_REQ_OK) {
    if (threadIdx.x == 0 && slice == 0) {
      if (status) status[b] = st;
      if (new_prefix_lens) new_prefix_lens[b] = P;
    }
    return;
  }
  compact_rows(c_kv, k_rope, ckv_bs, ckv_rs, kr_bs, kr_rs, b, P, alen, s_keep, s_rows, slice);
  if (threadIdx.x == 0 && slice == 0) {
    if (status) status[b] = DDT_REQ_OK;
    if (new_prefix_lens) new_prefix_lens[b] = P + alen;
  }
}

// ---------------------------------------------------------------------------
// Accept fused with compaction.  [Race Conditions] "The Broader Significance"
// defers fusing the compaction gather to a later phase, keeping it a separate
// step.  Here the kCompactSlices CTAs of a request (one cluster) each walk the
// tree (thread 0, the same walk as tree_accept_kernel) and then move their
// slice of the accepted rows (the same staging as kv_compact_kernel), so the
// path never leaves the chip and one launch replaces two; the first slice
// publishes the walk's outputs.  The walk always yields 1 <= alen <= q_len and
// path entries in [0, q_len), so compaction can only fail on the prefix.
// ---------------------------------------------------------------------------
__global__ void __cluster_dims__(kCompactSlices, 1, 1) __launch_bounds__(kCompactThreads)
    accept_compact_kernel(const int32_t* __restrict__ node_tokens,
                          const int32_t* __restrict__ target_tokens,
                          const int32_t* __restrict__ next_token,
                          const int32_t* __restrict__ next_sibling, int q_len,
                          uint16_t* __restrict__ c_kv, uint16_t* __restrict__ k_rope,
                          int64_t ckv_bs, int64_t ckv_rs, int64_t kr_bs, int64_t kr_rs,
                          int capacity, const int32_t* prefix_lens, int32_t* __restrict__ path,
                          int32_t* __restrict__ accept_len, int32_t* __restrict__ bonus_token,
                          int32_t* __restrict__ accept_status, int32_t* new_prefix_lens,
                          int32_t* __restrict__ compact_status) {
  extern __shared__ uint4 s_rows[];  // [alen][kSliceVec]
  __shared__ int32_t s_tok[DDT_MAX_Q_LEN], s_tgt[DDT_MAX_Q_LEN], s_first[DDT_MAX_Q_LEN],
      s_sib[DDT_MAX_Q_LEN], s_path[DDT_MAX_Q_LEN];
  __shared__ int s_alen, s_state;
  const int b = blockIdx.x / kCompactSlices;
  const int slice = blockIdx.x % kCompactSlices;
  // Read by every thread of every slice before the cluster barrier below, so
  // new_prefix_lens may be prefix_lens itself.
  const int P = prefix_lens[b];
  const int64_t base = static_cast<int64_t>(b) * q_len;
  for (int k = threadIdx.x; k < q_len; k += kCompactThreads) {
    s_tok[k] = node_tokens[base + k];
    s_tgt[k] = target_tokens[base + k];
    s_first[k] = next_token[base + k];
    s_sib[k] = next_sibling[base + k];
    s_path[k] = -1;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int alen, cur;
    const int st = accept_walk(s_tok, s_tgt, s_first, s_sib, q_len, s_path, alen, cur);
    if (slice == 0) {
      accept_len[b] = alen;
      if (bonus_token) bonus_token[b] = s_tgt[cur];
      if (accept_status) accept_status[b] = st;
    }
    s_alen = alen;
    s_state = (P < 0 || static_cast<int64_t>(P) + q_len > capacity) ? DDT_REQ_BAD_PREFIX
                                                                     : DDT_REQ_OK;
  }
  __syncthreads();
  const int alen = s_alen;
  if (slice == 0)
    for (int k = threadIdx.x; k < q_len; k += kCompactThreads) path[base + k] = s_path[k];
  const int st = s_state;
  // Every slice has read P and its tree arrays.
  compact_cluster_sync();
  if (st != DDT_REQ_OK) {
    if (threadIdx.x == 0 && slice == 0) {
      if (compact_status) compact_status[b] = st;
      if (new_prefix_lens) new_prefix_lens[b] = P;
    }
    return;
  }
  compact_rows(c_kv, k_rope, ckv_bs, ckv_rs, kr_bs, kr_rs, b, P, alen, s_path, s_rows, slice);
  if (threadIdx.x == 0 && slice == 0) {
    if (compact_status) compact_status[b] = DDT_REQ_OK;
    if (new_prefix_lens) new_prefix_lens[b] = P + alen;
  }
}

// ---------------------------------------------------------------------------
// Tree-block write.  [Race Conditions] "The Cache Compaction Problem": the tree
// block's KV rows go into the cache right after the prefix, node i at row P+i
// (absolute positions offset by the prefix length).  One CTA per request copies
// the q_len rows (latent and rope) with 16-byte vectors.  Optionally, as the
// stand-in for the target model's greedy tokens, target_tokens[b,i] is taken
// from a per-depth continuation: cont[b, depth[b,i]] (the target's greedy token
// after the accepted prefix of that depth).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kCompactThreads) kv_write_block_kernel(
    uint16_t* __restrict__ c_kv, uint16_t* __restrict__ k_rope, int64_t ckv_bs, int64_t ckv_rs,
    int64_t kr_bs, int64_t kr_rs, int capacity, const int32_t* __restrict__ prefix_lens,
    const uint16_t* __restrict__ block_ckv, const uint16_t* __restrict__ block_krope, int q_len,
    const int32_t* __restrict__ depth, const int32_t* __restrict__ cont,
    int32_t* __restrict__ target_tokens, int32_t* __restrict__ status) {
  const int b = blockIdx.x;
  const int P = prefix_lens[b];
  const bool ok = P >= 0 && static_cast<int64_t>(P) + q_len <= capacity;
  const int64_t base = static_cast<int64_t>(b) * q_len;
  if (cont) {
    for (int i = threadIdx.x; i < q_len; i += kCompactThreads) {
      const int d = depth[base + i];
      target_tokens[base + i] = (d >= 0 && d < q_len) ? cont[base + d] : -1;
    }
  }
  if (threadIdx.x == 0 && status) status[b] = ok ? DDT_REQ_OK : DDT_REQ_BAD_PREFIX;
  if (!ok) return;
  const uint4* src_l = reinterpret_cast<const uint4*>(block_ckv) + base * kLatVec;
  const uint4* src_r = reinterpret_cast<const uint4*>(block_krope) + base * kRopeVec;
  uint4* ckv_w = reinterpret_cast<uint4*>(c_kv + b * ckv_bs);
  uint4* kr_w = reinterpret_cast<uint4*>(k_rope + b * kr_bs);
  const int64_t ckv_rv = ckv_rs / 8, kr_rv = kr_rs / 8;
  for (int idx = threadIdx.x; idx < q_len * kRowVec; idx += kCompactThreads) {
    const int i = idx / kRowVec, v = idx - i * kRowVec;
    const int64_t row = P + i;
    if (v < kLatVec) ckv_w[row * ckv_rv + v] = src_l[static_cast<int64_t>(i) * kLatVec + v];
    else kr_w[row * kr_rv + (v - kLatVec)] = src_r[static_cast<int64_t>(i) * kRopeVec + (v - kLatVec)];
  }
}

// ---------------------------------------------------------------------------
// Launchers
// ---------------------------------------------------------------------------
cudaError_t launch_build_mask(const int32_t* parents, int B, int q_len, uint64_t* mask,
                              int32_t* depth, int32_t* status, cudaStream_t stream) {
  build_mask_kernel<<<B, 128, 0, stream>>>(parents, q_len, mask, depth, status);
  return cudaGetLastError();
}

cudaError_t launch_tree_accept(const int32_t* node_tokens, const int32_t* target_tokens,
                               const int32_t* next_token, const int32_t* next_sibling, int B,
                               int q_len, int32_t* path, int32_t* accept_len, int32_t* bonus,
                               int32_t* status, cudaStream_t stream) {
  const int grid = (B + kAcceptWarps - 1) / kAcceptWarps;
  tree_accept_kernel<<<grid, kAcceptWarps * 32, 0, stream>>>(
      node_tokens, target_tokens, next_token, next_sibling, B, q_len, path, accept_len, bonus,
      status);
  return cudaGetLastError();
}

cudaError_t launch_kv_compact(uint16_t* c_kv, uint16_t* k_rope, int64_t ckv_bs, int64_t ckv_rs,
                              int64_t kr_bs, int64_t kr_rs, int capacity,
                              const int32_t* prefix_lens, const int32_t* path,
                              const int32_t* accept_len, int B, int q_len,
                              int32_t* new_prefix_lens, int32_t* status, cudaStream_t stream) {
  const size_t smem = static_cast<size_t>(q_len) * kSliceVec * sizeof(uint4);
  const int smem_max = static_cast<int>(DDT_MAX_Q_LEN * kSliceVec * sizeof(uint4));
  const uintptr_t np0 = reinterpret_cast<uintptr_t>(new_prefix_lens);
  const uintptr_t p0 = reinterpret_cast<uintptr_t>(prefix_lens);
  const uintptr_t bytes = static_cast<uintptr_t>(B) * sizeof(int32_t);
  const bool in_place = new_prefix_lens && np0 < p0 + bytes && p0 < np0 + bytes;
  if (!in_place) {
    cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kv_compact_kernel<false>),
                                      smem_max, 0);
    if (e != cudaSuccess) return e;
    kv_compact_kernel<false><<<B * kCompactSlices, kCompactThreads, smem, stream>>>(
        c_kv, k_rope, ckv_bs, ckv_rs, kr_bs, kr_rs, capacity, prefix_lens, path, accept_len,
        q_len, new_prefix_lens, status);
    return cudaGetLastError();
  }
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kv_compact_kernel<true>),
                                    smem_max, 2);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(B) * kCompactSlices);
  cfg.blockDim = dim3(kCompactThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kCompactSlices;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kv_compact_kernel<true>, c_kv, k_rope, ckv_bs, ckv_rs, kr_bs,
                         kr_rs, capacity, prefix_lens, path, accept_len, q_len, new_prefix_lens,
                         status);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_accept_compact(const int32_t* node_tokens, const int32_t* target_tokens,
                                  const int32_t* next_token, const int32_t* next_sibling, int B,
                                  int q_len, uint16_t* c_kv, uint16_t* k_rope, int64_t ckv_bs,
                                  int64_t ckv_rs, int64_t kr_bs, int64_t kr_rs, int capacity,
                                  const int32_t* prefix_lens, int32_t* path, int32_t* accept_len,
                                  int32_t* bonus, int32_t* accept_status, int32_t* new_prefix_lens,
                                  int32_t* compact_status, cudaStream_t stream) {
  const size_t smem = static_cast<size_t>(q_len) * kSliceVec * sizeof(uint4);
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(accept_compact_kernel),
                                    static_cast<int>(DDT_MAX_Q_LEN * kSliceVec * sizeof(uint4)), 4);
  if (e != cudaSuccess) return e;
  accept_compact_kernel<<<B * kCompactSlices, kCompactThreads, smem, stream>>>(
      node_tokens, target_tokens, next_token, next_sibling, q_len, c_kv, k_rope, ckv_bs, ckv_rs,
      kr_bs, kr_rs, capacity, prefix_lens, path, accept_len, bonus, accept_status,
      new_prefix_lens, compact_status);
  return cudaGetLastError();
}

cudaError_t launch_kv_write_block(uint16_t* c_kv, uint16_t* k_rope, int64_t ckv_bs,
                                  int64_t ckv_rs, int64_t kr_bs, int64_t kr_rs, int capacity,
                                  const int32_t* prefix_lens, const uint16_t* block_ckv,
                                  const uint16_t* block_krope, int B, int q_len,
                                  const int32_t* depth, const int32_t* cont,
                                  int32_t* target_tokens, int32_t* status, cudaStream_t stream) {
  kv_write_block_kernel<<<B, kCompactThreads, 0, stream>>>(
      c_kv, k_rope, ckv_bs, ckv_rs, kr_bs, kr_rs, capacity, prefix_lens, block_ckv, block_krope,
      q_len, depth, cont, target_tokens, status);
  return cudaGetLastError();
}

}  // namespace ddt
