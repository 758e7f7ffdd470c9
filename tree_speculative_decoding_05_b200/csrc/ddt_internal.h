// ddt_internal.h — launcher declarations shared by the library's translation
// units (not part of the public C ABI).
#pragma once

#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "ddt.h"

// Rows of the latent cache per KV tile of the verify kernel (128, or 256 for the
// wide-tile build); the host-side split plan counts tiles of this size.
#ifndef DDT_VERIFY_TILE_KEYS
#define DDT_VERIFY_TILE_KEYS 128
#endif

namespace ddt {

constexpr int kVerifyTileKeys = DDT_VERIFY_TILE_KEYS;

cudaError_t launch_tree_build(const float* lp, const int32_t* tok, const int32_t* root_token,
                              int B, int D, int K, int q_len, int32_t* parents,
                              int32_t* node_tokens, int32_t* depth, float* logw,
                              int32_t* next_token, int32_t* next_sibling, uint64_t* mask,
                              int32_t* n_nodes, int32_t* status, cudaStream_t stream);

cudaError_t launch_build_mask(const int32_t* parents, int B, int q_len, uint64_t* mask,
                              int32_t* depth, int32_t* status, cudaStream_t stream);

cudaError_t launch_tree_accept(const int32_t* node_tokens, const int32_t* target_tokens,
                               const int32_t* next_token, const int32_t* next_sibling, int B,
                               int q_len, int32_t* path, int32_t* accept_len, int32_t* bonus,
                               int32_t* status, cudaStream_t stream);

cudaError_t launch_kv_compact(uint16_t* c_kv, uint16_t* k_rope, int64_t ckv_bs, int64_t ckv_rs,
                              int64_t kr_bs, int64_t kr_rs, int capacity,
                              const int32_t* prefix_lens, const int32_t* path,
                              const int32_t* accept_len, int B, int q_len,
                              int32_t* new_prefix_lens, int32_t* status, cudaStream_t stream);

cudaError_t launch_accept_compact(const int32_t* node_tokens, const int32_t* target_tokens,
                                  const int32_t* next_token, const int32_t* next_sibling, int B,
                                  int q_len, uint16_t* c_kv, uint16_t* k_rope, int64_t ckv_bs,
                                  int64_t ckv_rs, int64_t kr_bs, int64_t kr_rs, int capacity,
                                  const int32_t* prefix_lens, int32_t* path, int32_t* accept_len,
                                  int32_t* bonus, int32_t* accept_status, int32_t* new_prefix_lens,
                                  int32_t* compact_status, cudaStream_t stream);

cudaError_t launch_kv_write_block(uint16_t* c_kv, uint16_t* k_rope, int64_t ckv_bs,
                                  int64_t ckv_rs, int64_t kr_bs, int64_t kr_rs, int capacity,
                                  const int32_t* prefix_lens, const uint16_t* block_ckv,
                                  const uint16_t* block_krope, int B, int q_len,
                                  const int32_t* depth, const int32_t* cont,
                                  int32_t* target_tokens, int32_t* status, cudaStream_t stream);

// Split plan of the verify kernel.
int verify_num_splits(const ddt_attn_args& a, int sm_count);
size_t verify_workspace_bytes(const ddt_attn_args& a, int num_splits);

// Launch the verify kernel (and the split merge when num_splits > 1) with the
// given split count and partial buffers (may be null when num_splits == 1).
ddt_status launch_verify_attn(const ddt_attn_args& a, int num_splits, float* part_o,
                              float* part_lse, cudaStream_t stream);

// The prefix / tree-block split of the same attention: a pass over the prefix
// rows in prefix_splits splits, a pass over the tree block, and an LSE merge of
// the prefix_splits + 1 partials (part_o / part_lse hold that many).
ddt_status launch_verify_attn_split_tail(const ddt_attn_args& a, int prefix_splits,
                                         float* part_o, float* part_lse, cudaStream_t stream);

int device_sm_count();

// Sets the dynamic shared-memory limit of `func` once per CUDA context (`slot`
// names the function, 0 .. 15).
cudaError_t ensure_smem_limit(const void* func, int bytes, int slot);

// Unique ID of the calling thread's current CUDA context (0 if there is none or
// the driver cannot say).  IDs are never reused within a process.
unsigned long long current_context_id();

}  // namespace ddt
