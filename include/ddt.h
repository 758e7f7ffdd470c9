/*
 * ddt.h — C ABI of the DDTree tree-verify library for NVIDIA B200 (sm_100a).
 *
 * The calls below build a draft tree and verify it, one step of draft-tree
 * speculative decoding on a multi-head-latent-attention (MLA) model:
 *
 *   ddt_tree_build   best-first draft tree from per-depth top-k log-probabilities
 *   ddt_build_mask   per-node ancestor-or-self visibility bitmask from parents[]
 *   ddt_verify_attn  tree-verify MLA-absorb attention over the latent KV cache
 *   ddt_tree_accept  greedy longest-match walk of the draft tree
 *   ddt_kv_compact   gather of the accepted rows into the contiguous prefix
 *   ddt_accept_compact  the last two in one launch
 *   ddt_kv_write_block  the tree block's KV rows into the cache after the prefix
 *   ddt_decode_step  all of the above chained on the device for one decode step
 *
 * Sources (cited by page title and section):
 *   [Race Conditions]  "Race Conditions, Buffer Aliasing, and the Architecture of
 *                      a Native DDTree Inference Engine"
 *   [Foundation]       "Building the Foundation: Architecting a Native CUDA DDTree
 *                      Inference Engine"
 *   [Verdict]          "The Microsecond Verdict: Validating a DDTree Kernel Fix
 *                      Under Time Pressure"
 *
 * Conventions shared by every call
 *   - Every pointer argument is a DEVICE pointer owned by the caller.  No call
 *     allocates or frees device memory; scratch space that a call needs is
 *     passed in by the caller (see ddt_verify_attn_workspace_size).  One
 *     exception in footprint, not in calls: loading the library's device code
 *     on a GPU reserves the 32 MiB static scratch array of
 *     ddt_verify_attn_noalloc there until the process exits, whether or not
 *     that entry point is ever called.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and never synchronises the host.
 *   - Arguments that the host can check (sizes, null pointers, alignment,
 *     unsupported shapes) are checked before anything is launched; a failing
 *     check returns DDT_ERR_INVALID_ARG or DDT_ERR_UNSUPPORTED and launches
 *     nothing.
 *   - Errors that depend on device data (a malformed tree, an index out of
 *     range, a walk that exceeds its bound) are written to the per-request
 *     `status` output as one of the DDT_REQ_* codes below.  Kernels never trap,
 *     never read or write out of bounds because of such data, and always
 *     terminate.  The caller reads `status` after synchronising.
 *   - A launch failure reported by the CUDA runtime returns DDT_ERR_CUDA.
 *   - Supported shapes: 1 <= q_len <= 128 (so a mask row is W = ceil(q_len/64)
 *     <= 2 words), num_heads = 64, d_latent = 512, d_rope = 64.
 */
#ifndef DDT_H
#define DDT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Symbols of the shared library. */
#if defined(__GNUC__)
#define DDT_API __attribute__((visibility("default")))
#else
#define DDT_API
#endif

/* Opaque CUDA stream: identical to cudaStream_t / CUstream. */
struct CUstream_st;
typedef struct CUstream_st* ddt_stream_t;

typedef enum ddt_status {
  DDT_OK = 0,
  DDT_ERR_INVALID_ARG = 1, /* host-checkable argument error; nothing launched */
  DDT_ERR_UNSUPPORTED = 2, /* shape outside the supported set; nothing launched */
  DDT_ERR_CUDA = 3,        /* the CUDA runtime reported an error at launch */
  DDT_ERR_INPUT = 4        /* reserved for callers: a request's status was non-zero */
} ddt_status;

/* Per-request status codes written to `status[b]` by the kernels. */
#define DDT_REQ_OK 0
#define DDT_REQ_BAD_PARENT 1   /* parents[0] != -1, or parents[i] not in [0, i)    */
#define DDT_REQ_BAD_INDEX 2    /* a tree pointer or path entry is out of range     */
#define DDT_REQ_WALK_LIMIT 3   /* the tree walk examined more than q_len nodes     */
#define DDT_REQ_BAD_PREFIX 4   /* prefix_len < 0 or prefix_len + rows > capacity   */
#define DDT_REQ_BAD_LENGTH 5   /* accept_len not in [1, q_len]                     */
#define DDT_REQ_BAD_LP 6       /* a log-probability given to the tree build is not finite */

typedef enum ddt_dtype { DDT_F32 = 0, DDT_BF16 = 1 } ddt_dtype;

#define DDT_MAX_Q_LEN 128
#define DDT_NUM_HEADS 64
#define DDT_D_LATENT 512
#define DDT_D_ROPE 64

/* Mask words per node for a given q_len. */
#define DDT_MASK_WORDS(q_len) (((q_len) + 63) / 64)

/* ------------------------------------------------------------------------ */
/* ddt_tree_build                                                           */
/* ------------------------------------------------------------------------ */
/* Best-first construction of the draft tree of each request.
 *
 * Source: [Foundation] "The Single-Threaded Heap Design" (one serial best-first
 * expansion per request; budget <= 64 and depth <= 15 fit on chip; the other
 * threads build the visibility matrix and the retrieve pointers), "Tie-Breaking
 * and Numerical Precision" (equal weights in insertion order; float32), and
 * "Assumptions Underlying the Design" (item 4: the sibling weight expression;
 * item 5: candidates can run out before the budget, e.g. with topk = 1).
 *
 * Inputs per request b: lp[b,d,r] and tok[b,d,r] for d < D (depth_levels),
 * r < K (topk): the drafter's log-probabilities and tokens at tree depth d+1,
 * best first (the build does not require the order, but only with rows sorted
 * descending is it a best-first search); root_token[b].
 *
 * Expansion (the reading adopted where the pages are silent: a picked node
 * inserts its first child before its next sibling):
 *   node 0 = root: parent -1, depth 0, logw 0, token root_token[b]
 *   candidates = [(0 + lp[0,0], depth 1, rank 0, parent 0)]
 *   while nodes < q_len and candidates remain:
 *     take the candidate of largest logw (the earliest inserted among equals)
 *     -> node n: parent, depth d, logw, token tok[d-1, r]
 *     if d < D:     insert (logw + lp[d,0], d+1, 0, n)
 *     if r+1 < K:   insert ((logw - lp[d-1,r]) + lp[d-1,r+1], d, r+1, parent)
 *   All logw arithmetic is float32, rounded to nearest, in exactly this order.
 *
 * Outputs, int32 [B, q_len] unless noted:
 *   parents, node_tokens; depth (or NULL); logw float [B, q_len] (or NULL);
 *   next_token[i] = smallest child index of i, next_sibling[i] = the next larger
 *   index with the same parent (-1 where none) — the retrieve pointers that
 *   ddt_tree_accept walks; mask uint64 [B, q_len, W] (or NULL) as ddt_build_mask
 *   would compute it from parents; n_nodes int32 [B] (or NULL); status int32
 *   [B] (or NULL).
 * Node slots n_nodes <= i < q_len (candidates ran out) are padding: parent 0,
 * token -1, depth 1, logw -inf, visibility {0, i}, in no child list, so no walk
 * reaches them.  A non-finite lp entry sets DDT_REQ_BAD_LP and leaves the root
 * alone (n_nodes = 1) with padding.
 * Errors: B < 0, depth_levels < 1, topk < 1 -> DDT_ERR_INVALID_ARG; q_len
 * outside [1,128] -> DDT_ERR_UNSUPPORTED; lp, tok, root_token, parents,
 * node_tokens, next_token or next_sibling NULL with B > 0 -> DDT_ERR_INVALID_ARG.
 * B = 0 is a no-op. */
DDT_API ddt_status ddt_tree_build(const float* lp, const int32_t* tok, const int32_t* root_token,
                          int32_t B, int32_t depth_levels, int32_t topk, int32_t q_len,
                          int32_t* parents, int32_t* node_tokens, int32_t* depth, float* logw,
                          int32_t* next_token, int32_t* next_sibling, uint64_t* mask,
                          int32_t* n_nodes, int32_t* status, ddt_stream_t stream);

/* ------------------------------------------------------------------------ */
/* ddt_build_mask                                                           */
/* ------------------------------------------------------------------------ */
/* Visibility of tree nodes, built from the parent array.
 *
 * Source: [Foundation] "The Single-Threaded Heap Design" (the block's other
 * threads build the visibility matrix in parallel next to the serial heap) and
 * [Race Conditions] "The Cache Compaction Problem" (best-first creation order:
 * a child's index is larger than its parent's).
 *
 * Definition: node a is visible to node i iff a is i or an ancestor of i.
 *   mask[(b*q_len + i)*W + a/64] bit (a%64) = 1  iff  a in anc*(i),
 *   anc*(0) = {0},  anc*(i) = {i} U anc*(parents[i]).
 *   depth[b*q_len + i] = 0 for the root, depth[parent] + 1 otherwise.
 *
 * parents  int32 [B, q_len]  parents[b,0] = -1 and 0 <= parents[b,i] < i.
 * mask     uint64 [B, q_len, W], W = DDT_MASK_WORDS(q_len); every word written.
 * depth    int32 [B, q_len] or NULL.
 * status   int32 [B] or NULL: DDT_REQ_OK, or DDT_REQ_BAD_PARENT, in which case
 *          that request's mask words are all 0 and its depths are all -1.
 * Errors: B < 0, q_len outside [1,128], parents or mask NULL with B > 0 ->
 *         DDT_ERR_INVALID_ARG / DDT_ERR_UNSUPPORTED.  B = 0 is a no-op. */
DDT_API ddt_status ddt_build_mask(const int32_t* parents, int32_t B, int32_t q_len,
                          uint64_t* mask, int32_t* depth, int32_t* status,
                          ddt_stream_t stream);

/* ------------------------------------------------------------------------ */
/* ddt_verify_attn                                                          */
/* ------------------------------------------------------------------------ */
/* Tree-verify MLA-absorb attention.
 *
 * Source: [Race Conditions] "The Mission: A Native DDTree Engine" (a tree-verify
 * MLA-absorb attention kernel with visibility masking) and "The Cache Compaction
 * Problem" (the tree block sits after the prefix: absolute cache positions are
 * offset by the prefix length); [Verdict] "The Timeout That Tells a Story" (one
 * latent KV cache shared by all 64 attention heads).  The pages never write the
 * formula down; the reading adopted (absorbed MLA: the 512-wide latent c_kv is
 * both the key's latent part and the value) is:
 *
 *   For request b with prefix P = prefix_lens[b], node i, head h, and cache row
 *   j < P + q_len (the tree block occupies rows P .. P+q_len-1, node a at P+a):
 *     visible(j)  = j < P  or  bit (j-P) of mask[b,i]
 *     s_j = softmax_scale * ( q_lat[b,i,h,:] . c_kv[b,j,:] + q_rope[b,i,h,:] . k_rope[b,j,:] )
 *     p_j = exp(s_j - m) / Z over visible j  (m = max visible s_j, Z = sum exp(s_j - m))
 *     out[b,i,h,:] = sum_j p_j c_kv[b,j,:]
 *     lse[b,i,h]   = m + ln Z        (natural log of the scaled scores)
 *
 * Layout: q_lat bf16 [B, q_len, 64, 512] and q_rope bf16 [B, q_len, 64, 64],
 * both contiguous.  Cache rows of request b: c_kv + b*ckv_batch_stride +
 * r*ckv_row_stride (elements, bf16, 512 contiguous values per row), and the same
 * for k_rope (64 values per row).  Strides must be multiples of 8 elements
 * (16 bytes) and all base pointers 16-byte aligned.  out is [B, q_len, 64, 512]
 * contiguous, fp32 or bf16 (round to nearest even).  lse is fp32 [B, q_len, 64].
 *
 * Work split: rows are taken two tree nodes (128 query rows) at a time by a
 * pair of CTAs; long caches are split across SMs into num_splits KV ranges whose
 * partial results are merged with their log-sum-exp.  Splitting needs the
 * caller's workspace: ddt_verify_attn_workspace_size(args) bytes, 256-byte
 * aligned.  With workspace NULL or too small the call uses one split. */
typedef struct ddt_attn_args {
  int32_t B;          /* requests, >= 0                                        */
  int32_t q_len;      /* tree nodes per request, 1..128                         */
  int32_t num_heads;  /* must be 64                                             */
  int32_t d_latent;   /* must be 512                                            */
  int32_t d_rope;     /* must be 64                                             */
  int32_t capacity;   /* cache rows per request; prefix_lens[b] + q_len <= capacity */
  const int32_t* prefix_lens; /* int32 [B]                                      */
  const void* q_lat;  /* bf16 [B, q_len, 64, 512]                               */
  const void* q_rope; /* bf16 [B, q_len, 64, 64]                                */
  const void* c_kv;   /* bf16 cache, see strides                                */
  const void* k_rope; /* bf16 cache, see strides                                */
  int64_t ckv_batch_stride, ckv_row_stride; /* elements                         */
  int64_t kr_batch_stride, kr_row_stride;   /* elements                         */
  const uint64_t* mask; /* uint64 [B, q_len, W] from ddt_build_mask              */
  float softmax_scale; /* > 0 and finite (e.g. 1/sqrt(576)); otherwise the call
                          returns DDT_ERR_INVALID_ARG                            */
  int32_t out_dtype;  /* ddt_dtype                                              */
  void* out;          /* [B, q_len, 64, 512]                                    */
  float* lse;         /* fp32 [B, q_len, 64] or NULL                            */
  int32_t max_prefix; /* host-known upper bound on prefix_lens (plans splits)   */
  int32_t num_splits; /* 0 = choose automatically; otherwise 1..64             */
  void* workspace;    /* scratch for split partials, or NULL                    */
  size_t workspace_bytes;
  int32_t* status;    /* int32 [B] or NULL: DDT_REQ_OK or DDT_REQ_BAD_PREFIX    */
} ddt_attn_args;

/* Bytes of workspace the call will use for these arguments (0 if no split).
 * Reads only the sizes (B, q_len, heads, dims, capacity, max_prefix,
 * num_splits); pointers may still be unset.  Invalid sizes give 0. */
DDT_API size_t ddt_verify_attn_workspace_size(const ddt_attn_args* args);

/* Number of KV splits the call will use for these arguments (same inputs as
 * ddt_verify_attn_workspace_size; invalid sizes give 1). */
DDT_API int32_t ddt_verify_attn_num_splits(const ddt_attn_args* args);

DDT_API ddt_status ddt_verify_attn(const ddt_attn_args* args, ddt_stream_t stream);

/* ddt_verify_attn for callers that cannot allocate device memory.
 *
 * The pages describe no counterpart of this call; it exists for users of the
 * library.  Some callers may not call cudaMalloc at all: a plugin inside a host
 * framework that owns all device memory after start-up, or a latency-critical
 * decode loop that cannot take the device synchronisation an allocation may
 * cause.  Such callers cannot hand ddt_verify_attn the workspace its split-KV
 * path needs.  This call computes exactly what ddt_verify_attn computes, with
 * args->workspace and args->workspace_bytes ignored: split partials go to a
 * fixed scratch array inside the library (ddt_verify_attn_noalloc_scratch_bytes()
 * bytes, 32 MiB, held on every GPU that loads the library until the process
 * exits).  It allocates nothing.
 *   - The first call in a CUDA context (normally the device's primary
 *     context) looks the array's address up (this may load the library's
 *     device code on that device); make it before any stream capture on that
 *     device.  The address is remembered per context (by the driver's unique
 *     context ID), so a reset or replaced context gets a fresh lookup.
 *   - All calls on a device share the array and it keeps the last call's
 *     contents; nothing in it needs to start at zero.  Calls that overlap on
 *     the GPU race on it: order them (one stream, or events).
 *   - num_splits = 0 picks the largest useful split count whose partials fit
 *     the array (a single split needs none).  A forced num_splits whose
 *     partials do not fit is rejected with DDT_ERR_UNSUPPORTED before any
 *     launch.  Other errors are those of ddt_verify_attn. */
DDT_API ddt_status ddt_verify_attn_noalloc(const ddt_attn_args* args, ddt_stream_t stream);

/* Size in bytes of the scratch array used by ddt_verify_attn_noalloc. */
DDT_API size_t ddt_verify_attn_noalloc_scratch_bytes(void);

/* ------------------------------------------------------------------------ */
/* ddt_verify_attn_split_tail                                               */
/* ------------------------------------------------------------------------ */
/* The same attention as ddt_verify_attn, computed the way the pages planned
 * their production engine: a dense pass over the prefix rows [0, P) (every
 * node sees all of them; split across SMs like the split-KV plan), a small pass
 * over the tree block [P, P+q_len) with the visibility mask, and an LSE merge of
 * the partials:  lse = ln(e^lse_prefix + e^lse_tree),
 * out = e^(lse_prefix - lse) out_prefix + e^(lse_tree - lse) out_tree.
 * Source: [Foundation] "Assumptions Underlying the Design" (item 2: a library
 * kernel for the long prefix, the custom kernel only for the small tree tail)
 * and [Verdict] "The Timeout That Tells a Story".  It exists to measure that
 * design against the single fused pass of ddt_verify_attn; results agree with
 * it within the attention tolerance (the summation order differs).
 * Arguments as for ddt_verify_attn, except that the workspace is required:
 * at least ddt_verify_attn_split_tail_workspace_size(args) bytes, 256-byte
 * aligned, else DDT_ERR_INVALID_ARG and nothing is launched.  num_splits, when
 * positive, forces the number of prefix splits. */
DDT_API size_t ddt_verify_attn_split_tail_workspace_size(const ddt_attn_args* args);
DDT_API ddt_status ddt_verify_attn_split_tail(const ddt_attn_args* args, ddt_stream_t stream);

/* ------------------------------------------------------------------------ */
/* ddt_tree_accept                                                          */
/* ------------------------------------------------------------------------ */
/* Greedy acceptance of the longest draft path that the target agrees with.
 *
 * Source: [Verdict] "The Crash That Demanded a Fix" (follow the next_token /
 * next_sibling retrieve pointers; bound the walk by q_len), "What Was Learned"
 * (greedy acceptance; the bound `alen >= q_len`), and [Race Conditions] "The
 * Cache Compaction Problem" (the accepted path starts at the root, node 0).
 *
 * Walk, per request:
 *   path[0] = 0, alen = 1, cur = 0, examined = 0
 *   while alen < q_len:
 *     c = next_token[cur]                      (first child of cur, -1 if none)
 *     while c != -1 and node_tokens[c] != target_tokens[cur]:
 *       c = next_sibling[c]                    (next child of the same parent)
 *     (every node c examined counts; more than q_len -> DDT_REQ_WALK_LIMIT)
 *     if c == -1: stop
 *     path[alen++] = c, cur = c
 *   bonus_token = target_tokens[cur];  path[alen .. q_len) = -1
 * target_tokens[cur] is the target model's greedy token after node cur.
 * A pointer outside [-1, q_len) stops the walk with DDT_REQ_BAD_INDEX.  On any
 * status the accepted prefix so far is kept and bonus is target_tokens[cur].
 *
 * node_tokens, target_tokens, next_token, next_sibling: int32 [B, q_len].
 * path int32 [B, q_len]; accept_len, bonus_token, status: int32 [B]
 * (bonus_token and status may be NULL). */
DDT_API ddt_status ddt_tree_accept(const int32_t* node_tokens, const int32_t* target_tokens,
                           const int32_t* next_token, const int32_t* next_sibling,
                           int32_t B, int32_t q_len, int32_t* path, int32_t* accept_len,
                           int32_t* bonus_token, int32_t* status, ddt_stream_t stream);

/* ------------------------------------------------------------------------ */
/* ddt_kv_compact                                                           */
/* ------------------------------------------------------------------------ */
/* Gather of the accepted rows of the tree block into the contiguous prefix.
 *
 * Source: [Race Conditions] "The Cache Compaction Problem": new row P+i takes
 * old row P+keep[i] for i < alen (keep = path, keep[i] >= i).  A parallel
 * in-place gather races when keep[j] = i' for some j < i' (row i' is read by
 * one thread while another overwrites it); the pages gather into scratch and
 * copy back.  This call reads every kept row into on-chip memory before the
 * first write, so it is race-free for any path, needs no scratch, and rows of
 * the cache other than P .. P+alen-1 are not written.
 *
 *   for i < accept_len[b]:  row[P+i] <- old row[P+path[b,i]]   (both caches)
 *   new_prefix_lens[b] = P + accept_len[b]
 *
 * c_kv / k_rope: bf16 caches with the strides of ddt_verify_attn (elements,
 * multiples of 8, 16-byte aligned bases); rows are 512 / 64 values.
 * path int32 [B, q_len] (entries read for i < accept_len only), accept_len
 * int32 [B], prefix_lens int32 [B], new_prefix_lens int32 [B] or NULL (it may
 * be prefix_lens itself, updated in place).
 * status int32 [B] or NULL: DDT_REQ_BAD_LENGTH, DDT_REQ_BAD_INDEX (a path entry
 * outside [0, q_len)) or DDT_REQ_BAD_PREFIX (P < 0 or P + q_len > capacity);
 * a request with a non-zero status is left unchanged and its new prefix equals
 * its old one. */
DDT_API ddt_status ddt_kv_compact(void* c_kv, void* k_rope, int64_t ckv_batch_stride,
                          int64_t ckv_row_stride, int64_t kr_batch_stride,
                          int64_t kr_row_stride, int32_t capacity,
                          const int32_t* prefix_lens, const int32_t* path,
                          const int32_t* accept_len, int32_t B, int32_t q_len,
                          int32_t* new_prefix_lens, int32_t* status,
                          ddt_stream_t stream);

/* ------------------------------------------------------------------------ */
/* ddt_accept_compact                                                       */
/* ------------------------------------------------------------------------ */
/* ddt_tree_accept followed by ddt_kv_compact of its path, in one launch.
 *
 * Source: [Race Conditions] "The Cache Compaction Problem" (the gather of the
 * accepted rows) and "The Broader Significance" (fusing that gather is deferred
 * there to a later phase), and the walk of ddt_tree_accept.  Results are exactly those of the two calls
 * in sequence: path, accept_len, bonus_token and accept_status as
 * ddt_tree_accept writes them, then the cache rows, new_prefix_lens and
 * compact_status as ddt_kv_compact writes them for that path (which can only
 * report DDT_REQ_BAD_PREFIX, since the walk's path is always in range).
 * new_prefix_lens may be prefix_lens itself (updated in place); bonus_token,
 * accept_status, new_prefix_lens and compact_status may be NULL.  Arguments and
 * errors as for the two calls. */
DDT_API ddt_status ddt_accept_compact(const int32_t* node_tokens, const int32_t* target_tokens,
                              const int32_t* next_token, const int32_t* next_sibling,
                              int32_t B, int32_t q_len, void* c_kv, void* k_rope,
                              int64_t ckv_batch_stride, int64_t ckv_row_stride,
                              int64_t kr_batch_stride, int64_t kr_row_stride, int32_t capacity,
                              const int32_t* prefix_lens, int32_t* path, int32_t* accept_len,
                              int32_t* bonus_token, int32_t* accept_status,
                              int32_t* new_prefix_lens, int32_t* compact_status,
                              ddt_stream_t stream);

/* ------------------------------------------------------------------------ */
/* ddt_kv_write_block                                                       */
/* ------------------------------------------------------------------------ */
/* Writes the tree block's KV rows into the cache right after the prefix.
 *
 * Source: [Race Conditions] "The Cache Compaction Problem" (the tree's KV goes
 * into the cache at the offset of the prefix; node i is row P+i).
 *
 *   for i < q_len:  c_kv row P+i <- block_ckv[b,i,:],  k_rope row P+i <- block_krope[b,i,:]
 *
 * block_ckv bf16 [B, q_len, 512] and block_krope bf16 [B, q_len, 64], both
 * contiguous and 16-byte aligned; caches and strides as for ddt_verify_attn.
 * status int32 [B] or NULL: DDT_REQ_BAD_PREFIX (P < 0 or P + q_len > capacity,
 * nothing written for that request).  Errors as for ddt_kv_compact. */
DDT_API ddt_status ddt_kv_write_block(void* c_kv, void* k_rope, int64_t ckv_batch_stride,
                              int64_t ckv_row_stride, int64_t kr_batch_stride,
                              int64_t kr_row_stride, int32_t capacity,
                              const int32_t* prefix_lens, const void* block_ckv,
                              const void* block_krope, int32_t B, int32_t q_len,
                              int32_t* status, ddt_stream_t stream);

/* ------------------------------------------------------------------------ */
/* ddt_decode_step                                                          */
/* ------------------------------------------------------------------------ */
/* One speculative decode step chained on the device, for every request:
 *   1. ddt_tree_build   from this step's draft (lp, tok) and root_token
 *   2. ddt_kv_write_block of this step's tree-block rows at the prefix, and the
 *      target's greedy token after each node, target_tokens[b,i] =
 *      target_continuation[b, depth[b,i]]
 *   3. ddt_verify_attn  with the tree's mask
 *   4. ddt_accept_compact, writing the bonus token into root_token and the new
 *      prefix length into attn.prefix_lens (both are the state of the next step)
 * Source: [Race Conditions] "The Mission: A Native DDTree Engine" and "The Cache
 * Compaction Problem" (build, verify, accept, compact, in that order, with the
 * tree block written at the prefix offset), [Verdict] "What Was Learned"
 * (chaining the tree builder's output into the accept walk).
 *
 * The model's own work (the drafter, the target model's KV rows, queries and
 * greedy tokens) is outside this library: its results arrive as inputs — lp and
 * tok [B, D, K], the tree block's KV rows, the absorbed queries (attn.q_lat,
 * attn.q_rope), and target_continuation int32 [B, q_len], where entry d is the
 * target's greedy token after the accepted path of depth d.  Under greedy
 * verification that token does not depend on which path of that depth was
 * taken once the path matches the target, so a per-depth continuation gives
 * every node on a matching path its exact target token.
 *
 * The call only launches kernels (four, or five with split-KV), in order, on
 * `stream`; it neither allocates nor synchronises, so it can be captured in a
 * CUDA graph.  attn.max_prefix sizes the split-KV plan (any prefix is handled;
 * a bound near the real prefixes plans best).  The step writes through
 * attn.mask (the tree's visibility words), attn.c_kv / attn.k_rope (the tree
 * block, then the compaction), attn.prefix_lens (the new prefix) and
 * attn.status (the verify status).
 * status int32 [4, B] or NULL: rows = tree build, block write, accept,
 * compaction.  Every output array is caller-owned and [B, q_len] unless noted. */
typedef struct ddt_decode_args {
  ddt_attn_args attn;                 /* verify; prefix_lens is updated in place */
  int32_t depth_levels, topk;         /* D, K of the draft */
  const float* lp;                    /* [B, D, K] */
  const int32_t* tok;                 /* [B, D, K] */
  int32_t* root_token;                /* [B]: this step's root; the bonus token after */
  const void* block_ckv;              /* bf16 [B, q_len, 512] */
  const void* block_krope;            /* bf16 [B, q_len, 64] */
  const int32_t* target_continuation; /* [B, q_len] */
  int32_t* parents;
  int32_t* node_tokens;
  int32_t* depth;
  int32_t* next_token;
  int32_t* next_sibling;
  int32_t* n_nodes;                   /* [B] or NULL */
  int32_t* target_tokens;
  int32_t* path;
  int32_t* accept_len;                /* [B] */
  int32_t* status;                    /* [4, B] or NULL */
} ddt_decode_args;

DDT_API ddt_status ddt_decode_step(const ddt_decode_args* args, ddt_stream_t stream);

/* Human-readable name of a status code (static storage). */
DDT_API const char* ddt_status_str(ddt_status status);

/* Diagnostic: the library's device fault word, a bit set of
 *   1 = a kernel gave up waiting on a barrier (bounded wait expired).
 * Reading it synchronises the device; with reset != 0 it is cleared.  A clean
 * run leaves it 0. */
#define DDT_FAULT_WAIT_TIMEOUT 1u
DDT_API ddt_status ddt_fault_flags(uint32_t* flags, int32_t reset);

/* Self-test of the kernels' bounded waits (no counterpart on the pages; the
 * library's own failure detection).  Launches one thread that waits, for at most
 * timeout_us microseconds, on a barrier that nothing will ever complete.  The
 * wait gives up as every wait in the library does on a stalled barrier: it sets
 * DDT_FAULT_WAIT_TIMEOUT in the fault word (read with ddt_fault_flags), writes 1
 * to *gave_up (device int32, or NULL) and returns, leaving the context usable.
 * timeout_us must be in [1, 1000000], else DDT_ERR_INVALID_ARG. */
DDT_API ddt_status ddt_selftest_bounded_wait(uint32_t timeout_us, int32_t* gave_up,
                                     ddt_stream_t stream);

/* Library version string (static storage). */
DDT_API const char* ddt_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DDT_H */
