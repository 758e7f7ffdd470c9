// noalloc.cu — ddt_verify_attn_noalloc: tree-verify attention for callers that
// cannot allocate device memory.
//
// Some callers of this library must not call cudaMalloc or any allocating
// routine: a plugin living inside a host framework that owns every byte of
// device memory after start-up, or a latency-critical decode loop that cannot
// afford the implicit device synchronisation an allocation may bring.  The
// split-KV path of ddt_verify_attn needs scratch space for its partial
// results, which such callers cannot provide.  This entry point takes that
// scratch from a fixed array in the library's own device memory instead.
//
// Facts a user should know:
//   * The array is a file-scope static device array of kScratchBytes (32 MiB).
//     Every GPU on which the library's device code is loaded holds it until the
//     process exits.
//   * The first call on a device looks up the array's device address
//     (cudaGetSymbolAddress, which may load the library's device code on that
//     device); make that first call before any stream capture on the device.
//   * All calls on a device share the one array, and it keeps whatever the last
//     call left in it.  Nothing in it needs to start at zero: every split
//     writes all of its partial rows before the merge reads them, and empty
//     splits are skipped.  Calls that overlap on the GPU (different streams
//     without ordering between them) race on the array; order them.
//   * A request whose split partials do not fit is handled as follows: with
//     num_splits = 0 (automatic) the call uses the largest split count that
//     fits (one split needs no scratch at all); a caller-forced num_splits
//     whose partials exceed the array is rejected with DDT_ERR_UNSUPPORTED
//     before anything is launched.
//   * It allocates nothing: no cudaMalloc, cudaFree or allocating library call.
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <mutex>

#include "ddt.h"

namespace {

constexpr size_t kScratchBytes = static_cast<size_t>(32) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_verify_scratch[kScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once per
// device, with that device current).
ddt_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DDT_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return DDT_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_verify_scratch) != cudaSuccess || p == nullptr)
      return DDT_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return DDT_OK;
}

}  // namespace

extern "C" DDT_API size_t ddt_verify_attn_noalloc_scratch_bytes(void) { return kScratchBytes; }

extern "C" DDT_API ddt_status ddt_verify_attn_noalloc(const ddt_attn_args* args,
                                                      ddt_stream_t stream) {
  if (!args) return DDT_ERR_INVALID_ARG;
  ddt_attn_args a = *args;
  a.workspace = nullptr;
  a.workspace_bytes = 0;
  size_t need = ddt_verify_attn_workspace_size(&a);
  if (need > kScratchBytes) {
    if (args->num_splits > 0) return DDT_ERR_UNSUPPORTED;  // forced split count too large
    // Automatic plan: the largest split count below the planned one that fits.
    int32_t s = ddt_verify_attn_num_splits(&a) - 1;
    for (; s >= 2; --s) {
      a.num_splits = s;
      need = ddt_verify_attn_workspace_size(&a);
      if (need <= kScratchBytes) break;
    }
    if (s < 2) {
      a.num_splits = 1;
      need = 0;
    }
  }
  if (need > 0) {
    void* p = nullptr;
    const ddt_status st = scratch_address(&p);
    if (st != DDT_OK) return st;
    a.workspace = p;
    a.workspace_bytes = kScratchBytes;
  }
  return ddt_verify_attn(&a, stream);
}
