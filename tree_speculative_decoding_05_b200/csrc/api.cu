// api.cu — the extern "C" entry points of libddt: host-side argument checks,
// then one launch per call on the caller's stream.  No entry point allocates
// device memory or synchronises the host.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <mutex>

#include "ddt.h"
#include "ddt_internal.h"

namespace ddt {

namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxSlots = 16;
constexpr int kMaxContexts = 64;
static_assert(kMaxSlots <= 32, "one bit per slot");

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shared cache row checks of ddt_verify_attn and ddt_kv_compact.
bool cache_strides_ok(int B, int capacity, int64_t ckv_bs, int64_t ckv_rs, int64_t kr_bs,
                      int64_t kr_rs) {
  if (ckv_rs < DDT_D_LATENT || kr_rs < DDT_D_ROPE) return false;
  if ((ckv_rs % 8) || (kr_rs % 8) || (ckv_bs % 8) || (kr_bs % 8)) return false;
  if (B > 1 && (ckv_bs < static_cast<int64_t>(capacity) * ckv_rs ||
                kr_bs < static_cast<int64_t>(capacity) * kr_rs))
    return false;
  return true;
}

}  // namespace

int device_sm_count() {
  static std::atomic<int> counts[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  int n = counts[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    counts[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

namespace {

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

struct DriverFns {
  CtxGetCurrentFn get_current = nullptr;
  CtxGetIdFn get_id = nullptr;
};

const DriverFns& driver_fns() {
  static DriverFns fns;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fns.get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fns.get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  return fns;
}

}  // namespace

unsigned long long current_context_id() {
  const DriverFns& f = driver_fns();
  if (!f.get_current || !f.get_id) return 0;
  CUcontext ctx = nullptr;
  if (f.get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  unsigned long long id = 0;
  if (f.get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// A function attribute belongs to the function as loaded in one context (a
// context that is reset or replaced loads the module afresh), so what has been
// set is remembered per context ID: one bit per slot.
cudaError_t ensure_smem_limit(const void* func, int bytes, int slot) {
  static std::mutex mu;
  static unsigned long long ctx_id[kMaxContexts] = {};
  static uint32_t done[kMaxContexts] = {};
  static int next = 0;
  const unsigned long long id = current_context_id();
  if (id == 0 || slot < 0 || slot >= kMaxSlots)  // nothing to key a cache on
    return cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  std::lock_guard<std::mutex> lock(mu);
  int i = 0;
  while (i < kMaxContexts && ctx_id[i] != id) ++i;
  if (i < kMaxContexts && ((done[i] >> slot) & 1u)) return cudaSuccess;
  const cudaError_t e =
      cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  if (i == kMaxContexts) {  // a context not seen yet takes the oldest entry
    i = next;
    next = (next + 1) % kMaxContexts;
    ctx_id[i] = id;
    done[i] = 0;
  }
  done[i] |= 1u << slot;
  return cudaSuccess;
}

// Split plan of the verify kernel (host side).
int verify_num_splits(const ddt_attn_args& a, int sm_count) {
  if (a.num_splits > 0) return a.num_splits;
  const int n_pairs = (a.q_len + 1) / 2;
  const int64_t items = static_cast<int64_t>(a.B) * n_pairs;
  const int64_t pairs_avail = sm_count / 2 > 0 ? sm_count / 2 : 1;
  const int max_tiles = (a.max_prefix + a.q_len + kVerifyTileKeys - 1) / kVerifyTileKeys;
  const double rows128 = kVerifyTileKeys / 128.0;  // a tile's work in 128-row units
  // Estimated time in units of one 128-row tile: waves of work items x (tiles per
  // item + a fixed cost per item: its Q load, pipeline fill and epilogue), plus,
  // with several splits, writing and merging the partials.  The two constants (4
  // units per item, 0.75 per split) are fitted to measured split sweeps (one
  // request with a 32768-row prefix: 4 splits 149 us, 8: 162, 13: 169, 16: 203).
  auto cost = [&](int s) {
    const int64_t waves = (items * s + pairs_avail - 1) / pairs_avail;
    const int per = (max_tiles + s - 1) / s;
    return static_cast<double>(waves) * (per * rows128 + 4.0) + (s > 1 ? 0.75 * s : 0.0);
  };
  int best = 1;
  double best_cost = cost(1);
  for (int s = 2; s <= 32 && s <= max_tiles; ++s) {
    const double c = cost(s);
    if (c < best_cost) {
      best = s;
      best_cost = c;
    }
  }
  return best;
}

size_t verify_workspace_bytes(const ddt_attn_args& a, int num_splits) {
  if (num_splits <= 1) return 0;
  const size_t rows = static_cast<size_t>(a.B) * a.q_len * 64;
  return static_cast<size_t>(num_splits) * rows * (512 + 1) * sizeof(float);
}

}  // namespace ddt

using namespace ddt;

extern "C" {

const char* ddt_version(void) { return "ddt 0.1.0 (sm_100a)"; }

const char* ddt_status_str(ddt_status s) {
  switch (s) {
    case DDT_OK: return "ok";
    case DDT_ERR_INVALID_ARG: return "invalid argument";
    case DDT_ERR_UNSUPPORTED: return "unsupported shape";
    case DDT_ERR_CUDA: return "CUDA error";
    case DDT_ERR_INPUT: return "malformed request data";
  }
  return "unknown status";
}

ddt_status ddt_build_mask(const int32_t* parents, int32_t B, int32_t q_len, uint64_t* mask,
                          int32_t* depth, int32_t* status, ddt_stream_t stream) {
  if (B < 0) return DDT_ERR_INVALID_ARG;
  if (q_len < 1 || q_len > DDT_MAX_Q_LEN) return DDT_ERR_UNSUPPORTED;
  if (B == 0) return DDT_OK;
  if (!parents || !mask) return DDT_ERR_INVALID_ARG;
  if (launch_build_mask(parents, B, q_len, mask, depth, status,
                        reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DDT_ERR_CUDA;
  return DDT_OK;
}

ddt_status ddt_tree_build(const float* lp, const int32_t* tok, const int32_t* root_token,
                          int32_t B, int32_t depth_levels, int32_t topk, int32_t q_len,
                          int32_t* parents, int32_t* node_tokens, int32_t* depth, float* logw,
                          int32_t* next_token, int32_t* next_sibling, uint64_t* mask,
                          int32_t* n_nodes, int32_t* status, ddt_stream_t stream) {
  if (B < 0 || depth_levels < 1 || topk < 1) return DDT_ERR_INVALID_ARG;
  if (q_len < 1 || q_len > DDT_MAX_Q_LEN) return DDT_ERR_UNSUPPORTED;
  if (B == 0) return DDT_OK;
  if (!lp || !tok || !root_token || !parents || !node_tokens || !next_token || !next_sibling)
    return DDT_ERR_INVALID_ARG;
  if (launch_tree_build(lp, tok, root_token, B, depth_levels, topk, q_len, parents, node_tokens,
                        depth, logw, next_token, next_sibling, mask, n_nodes, status,
                        reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DDT_ERR_CUDA;
  return DDT_OK;
}

ddt_status ddt_tree_accept(const int32_t* node_tokens, const int32_t* target_tokens,
                           const int32_t* next_token, const int32_t* next_sibling, int32_t B,
                           int32_t q_len, int32_t* path, int32_t* accept_len,
                           int32_t* bonus_token, int32_t* status, ddt_stream_t stream) {
  if (B < 0) return DDT_ERR_INVALID_ARG;
  if (q_len < 1 || q_len > DDT_MAX_Q_LEN) return DDT_ERR_UNSUPPORTED;
  if (B == 0) return DDT_OK;
  if (!node_tokens || !target_tokens || !next_token || !next_sibling || !path || !accept_len)
    return DDT_ERR_INVALID_ARG;
  if (launch_tree_accept(node_tokens, target_tokens, next_token, next_sibling, B, q_len, path,
                         accept_len, bonus_token, status,
                         reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DDT_ERR_CUDA;
  return DDT_OK;
}

ddt_status ddt_kv_compact(void* c_kv, void* k_rope, int64_t ckv_batch_stride,
                          int64_t ckv_row_stride, int64_t kr_batch_stride, int64_t kr_row_stride,
                          int32_t capacity, const int32_t* prefix_lens, const int32_t* path,
                          const int32_t* accept_len, int32_t B, int32_t q_len,
                          int32_t* new_prefix_lens, int32_t* status, ddt_stream_t stream) {
  if (B < 0 || capacity < 0) return DDT_ERR_INVALID_ARG;
  if (q_len < 1 || q_len > DDT_MAX_Q_LEN) return DDT_ERR_UNSUPPORTED;
  if (B == 0) return DDT_OK;
  if (!c_kv || !k_rope || !prefix_lens || !path || !accept_len) return DDT_ERR_INVALID_ARG;
  if (!aligned16(c_kv) || !aligned16(k_rope)) return DDT_ERR_INVALID_ARG;
  if (!cache_strides_ok(B, capacity, ckv_batch_stride, ckv_row_stride, kr_batch_stride,
                        kr_row_stride))
    return DDT_ERR_INVALID_ARG;
  if (launch_kv_compact(static_cast<uint16_t*>(c_kv), static_cast<uint16_t*>(k_rope),
                        ckv_batch_stride, ckv_row_stride, kr_batch_stride, kr_row_stride, capacity,
                        prefix_lens, path, accept_len, B, q_len, new_prefix_lens, status,
                        reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DDT_ERR_CUDA;
  return DDT_OK;
}

ddt_status ddt_accept_compact(const int32_t* node_tokens, const int32_t* target_tokens,
                              const int32_t* next_token, const int32_t* next_sibling, int32_t B,
                              int32_t q_len, void* c_kv, void* k_rope, int64_t ckv_batch_stride,
                              int64_t ckv_row_stride, int64_t kr_batch_stride,
                              int64_t kr_row_stride, int32_t capacity,
                              const int32_t* prefix_lens, int32_t* path, int32_t* accept_len,
                              int32_t* bonus_token, int32_t* accept_status,
                              int32_t* new_prefix_lens, int32_t* compact_status,
                              ddt_stream_t stream) {
  if (B < 0 || capacity < 0) return DDT_ERR_INVALID_ARG;
  if (q_len < 1 || q_len > DDT_MAX_Q_LEN) return DDT_ERR_UNSUPPORTED;
  if (B == 0) return DDT_OK;
  if (!node_tokens || !target_tokens || !next_token || !next_sibling || !c_kv || !k_rope ||
      !prefix_lens || !path || !accept_len)
    return DDT_ERR_INVALID_ARG;
  if (!aligned16(c_kv) || !aligned16(k_rope)) return DDT_ERR_INVALID_ARG;
  if (!cache_strides_ok(B, capacity, ckv_batch_stride, ckv_row_stride, kr_batch_stride,
                        kr_row_stride))
    return DDT_ERR_INVALID_ARG;
  if (launch_accept_compact(node_tokens, target_tokens, next_token, next_sibling, B, q_len,
                            static_cast<uint16_t*>(c_kv), static_cast<uint16_t*>(k_rope),
                            ckv_batch_stride, ckv_row_stride, kr_batch_stride, kr_row_stride,
                            capacity, prefix_lens, path, accept_len, bonus_token, accept_status,
                            new_prefix_lens, compact_status,
                            reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DDT_ERR_CUDA;
  return DDT_OK;
}

// Sizes and plan parameters only (what the split plan and workspace size need).
static ddt_status check_attn_shape(const ddt_attn_args* a) {
  if (!a) return DDT_ERR_INVALID_ARG;
  if (a->B < 0 || a->capacity < 0 || a->max_prefix < 0) return DDT_ERR_INVALID_ARG;
  if (a->q_len < 1 || a->q_len > DDT_MAX_Q_LEN || a->num_heads != DDT_NUM_HEADS ||
      a->d_latent != DDT_D_LATENT || a->d_rope != DDT_D_ROPE)
    return DDT_ERR_UNSUPPORTED;
  if (a->num_splits < 0 || a->num_splits > 64) return DDT_ERR_INVALID_ARG;
  return DDT_OK;
}

static ddt_status check_attn_args(const ddt_attn_args* a) {
  const ddt_status shape = check_attn_shape(a);
  if (shape != DDT_OK) return shape;
  if (a->out_dtype != DDT_F32 && a->out_dtype != DDT_BF16) return DDT_ERR_INVALID_ARG;
  if (a->B == 0) return DDT_OK;
  if (!a->prefix_lens || !a->q_lat || !a->q_rope || !a->c_kv || !a->k_rope || !a->mask || !a->out)
    return DDT_ERR_INVALID_ARG;
  if (!aligned16(a->q_lat) || !aligned16(a->q_rope) || !aligned16(a->c_kv) ||
      !aligned16(a->k_rope) || !aligned16(a->out))
    return DDT_ERR_INVALID_ARG;
  if (a->capacity < a->q_len) return DDT_ERR_INVALID_ARG;
  if (!cache_strides_ok(a->B, a->capacity, a->ckv_batch_stride, a->ckv_row_stride,
                        a->kr_batch_stride, a->kr_row_stride))
    return DDT_ERR_INVALID_ARG;
  // A positive, finite scale (and log2(e) times it): the kernel applies it after
  // taking the maximum of the raw scores, which needs scale > 0.
  const float scale_log2 = a->softmax_scale * 1.4426950408889634f;
  if (!(a->softmax_scale > 0.0f) || !(scale_log2 <= 3.402823466e38f)) return DDT_ERR_INVALID_ARG;
  return DDT_OK;
}

int32_t ddt_verify_attn_num_splits(const ddt_attn_args* a) {
  if (check_attn_shape(a) != DDT_OK || a->B == 0) return 1;
  return verify_num_splits(*a, device_sm_count());
}

size_t ddt_verify_attn_workspace_size(const ddt_attn_args* a) {
  if (check_attn_shape(a) != DDT_OK || a->B == 0) return 0;
  return verify_workspace_bytes(*a, verify_num_splits(*a, device_sm_count()));
}

ddt_status ddt_verify_attn(const ddt_attn_args* a, ddt_stream_t stream) {
  const ddt_status st = check_attn_args(a);
  if (st != DDT_OK || a->B == 0) return st;
  int splits = verify_num_splits(*a, device_sm_count());
  const size_t need = verify_workspace_bytes(*a, splits);
  float* part_o = nullptr;
  float* part_lse = nullptr;
  if (splits > 1) {
    if (!a->workspace || a->workspace_bytes < need ||
        (reinterpret_cast<uintptr_t>(a->workspace) & 255u)) {
      splits = 1;
    } else {
      part_o = static_cast<float*>(a->workspace);
      part_lse = part_o + static_cast<size_t>(splits) * a->B * a->q_len * 64 * 512;
    }
  }
  return launch_verify_attn(*a, splits, part_o, part_lse, reinterpret_cast<cudaStream_t>(stream));
}

size_t ddt_verify_attn_split_tail_workspace_size(const ddt_attn_args* a) {
  if (check_attn_shape(a) != DDT_OK || a->B == 0) return 0;
  return verify_workspace_bytes(*a, verify_num_splits(*a, device_sm_count()) + 1);
}

ddt_status ddt_verify_attn_split_tail(const ddt_attn_args* a, ddt_stream_t stream) {
  const ddt_status st = check_attn_args(a);
  if (st != DDT_OK || a->B == 0) return st;
  const int splits = verify_num_splits(*a, device_sm_count());
  const size_t need = verify_workspace_bytes(*a, splits + 1);
  if (!a->workspace || a->workspace_bytes < need ||
      (reinterpret_cast<uintptr_t>(a->workspace) & 255u))
    return DDT_ERR_INVALID_ARG;
  float* part_o = static_cast<float*>(a->workspace);
  float* part_lse = part_o + static_cast<size_t>(splits + 1) * a->B * a->q_len * 64 * 512;
  return launch_verify_attn_split_tail(*a, splits, part_o, part_lse,
                                       reinterpret_cast<cudaStream_t>(stream));
}

ddt_status ddt_kv_write_block(void* c_kv, void* k_rope, int64_t ckv_batch_stride,
                              int64_t ckv_row_stride, int64_t kr_batch_stride,
                              int64_t kr_row_stride, int32_t capacity,
                              const int32_t* prefix_lens, const void* block_ckv,
                              const void* block_krope, int32_t B, int32_t q_len,
                              int32_t* status, ddt_stream_t stream) {
  if (B < 0 || capacity < 0) return DDT_ERR_INVALID_ARG;
  if (q_len < 1 || q_len > DDT_MAX_Q_LEN) return DDT_ERR_UNSUPPORTED;
  if (B == 0) return DDT_OK;
  if (!c_kv || !k_rope || !prefix_lens || !block_ckv || !block_krope) return DDT_ERR_INVALID_ARG;
  if (!aligned16(c_kv) || !aligned16(k_rope) || !aligned16(block_ckv) || !aligned16(block_krope))
    return DDT_ERR_INVALID_ARG;
  if (!cache_strides_ok(B, capacity, ckv_batch_stride, ckv_row_stride, kr_batch_stride,
                        kr_row_stride))
    return DDT_ERR_INVALID_ARG;
  if (launch_kv_write_block(static_cast<uint16_t*>(c_kv), static_cast<uint16_t*>(k_rope),
                            ckv_batch_stride, ckv_row_stride, kr_batch_stride, kr_row_stride,
                            capacity, prefix_lens, static_cast<const uint16_t*>(block_ckv),
                            static_cast<const uint16_t*>(block_krope), B, q_len, nullptr, nullptr,
                            nullptr, status, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DDT_ERR_CUDA;
  return DDT_OK;
}

ddt_status ddt_decode_step(const ddt_decode_args* d, ddt_stream_t stream) {
  if (!d) return DDT_ERR_INVALID_ARG;
  const ddt_attn_args& a = d->attn;
  ddt_status st = check_attn_args(&a);
  if (st != DDT_OK) return st;
  if (d->depth_levels < 1 || d->topk < 1) return DDT_ERR_INVALID_ARG;
  if (a.B == 0) return DDT_OK;
  if (!d->lp || !d->tok || !d->root_token || !d->block_ckv || !d->block_krope ||
      !d->target_continuation || !d->parents || !d->node_tokens || !d->depth ||
      !d->next_token || !d->next_sibling || !d->target_tokens || !d->path || !d->accept_len)
    return DDT_ERR_INVALID_ARG;
  if (!aligned16(d->block_ckv) || !aligned16(d->block_krope)) return DDT_ERR_INVALID_ARG;
  const int B = a.B, Q = a.q_len;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int32_t* row[4] = {nullptr, nullptr, nullptr, nullptr};
  if (d->status)
    for (int k = 0; k < 4; ++k) row[k] = d->status + static_cast<int64_t>(k) * B;
  uint64_t* mask = const_cast<uint64_t*>(a.mask);
  if (launch_tree_build(d->lp, d->tok, d->root_token, B, d->depth_levels, d->topk, Q, d->parents,
                        d->node_tokens, d->depth, nullptr, d->next_token, d->next_sibling, mask,
                        d->n_nodes, row[0], s) != cudaSuccess)
    return DDT_ERR_CUDA;
  uint16_t* ckv = static_cast<uint16_t*>(const_cast<void*>(a.c_kv));
  uint16_t* kr = static_cast<uint16_t*>(const_cast<void*>(a.k_rope));
  if (launch_kv_write_block(ckv, kr, a.ckv_batch_stride, a.ckv_row_stride, a.kr_batch_stride,
                            a.kr_row_stride, a.capacity, a.prefix_lens,
                            static_cast<const uint16_t*>(d->block_ckv),
                            static_cast<const uint16_t*>(d->block_krope), B, Q, d->depth,
                            d->target_continuation, d->target_tokens, row[1], s) != cudaSuccess)
    return DDT_ERR_CUDA;
  st = ddt_verify_attn(&a, stream);
  if (st != DDT_OK) return st;
  if (launch_accept_compact(d->node_tokens, d->target_tokens, d->next_token, d->next_sibling, B,
                            Q, ckv, kr, a.ckv_batch_stride, a.ckv_row_stride, a.kr_batch_stride,
                            a.kr_row_stride, a.capacity, a.prefix_lens, d->path, d->accept_len,
                            d->root_token, row[2], const_cast<int32_t*>(a.prefix_lens), row[3],
                            s) != cudaSuccess)
    return DDT_ERR_CUDA;
  return DDT_OK;
}

}  // extern "C"
