// ddt_internal.h — launcher declarations shared by the library's translation
// units (not part of the public C ABI).
#pragma once

#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "ddt.h"

namespace ddt {

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

// Split plan of the verify kernel.
int verify_num_splits(const ddt_attn_args& a, int sm_count);
size_t verify_workspace_bytes(const ddt_attn_args& a, int num_splits);

// Launch the verify kernel (and the split merge when num_splits > 1) with the
// given split count and partial buffers (may be null when num_splits == 1).
ddt_status launch_verify_attn(const ddt_attn_args& a, int num_splits, float* part_o,
                              float* part_lse, cudaStream_t stream);

int device_sm_count();

// Sets the dynamic shared-memory limit of `func` on the current device once.
cudaError_t ensure_smem_limit(const void* func, int bytes, int slot);

}  // namespace ddt
