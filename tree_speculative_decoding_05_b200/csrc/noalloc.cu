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
//   * The first call in a CUDA context (normally a device's primary context)
//     looks up the array's device address there (cudaGetSymbolAddress, which
//     may load the library's device code on that device); make that first call
//     before any stream capture on the device.  The address is remembered per
//     context, keyed by the driver's unique context ID, so a context that is
//     reset (cudaDeviceReset) or replaced gets a fresh lookup instead of a
//     stale address.
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
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <mutex>

#include "ddt.h"
#include "ddt_internal.h"

namespace {

using ddt::current_context_id;

constexpr size_t kScratchBytes = static_cast<size_t>(32) << 20;
constexpr int kMaxContexts = 64;

static __device__ __align__(256) unsigned char g_verify_scratch[kScratchBytes];

std::mutex g_scratch_mu;
unsigned long long g_ctx_id[kMaxContexts] = {};
void* g_ctx_ptr[kMaxContexts] = {};
int g_ctx_next = 0;

// Device address of the scratch array in the current context: looked up with
// cudaGetSymbolAddress once per context and remembered under the context's
// unique ID.  Without a usable ID (no current context yet, or a driver that
// cannot report one) the address is looked up again on every call.
ddt_status scratch_address(void** out) {
  unsigned long long id = current_context_id();
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (id != 0) {
    for (int i = 0; i < kMaxContexts; ++i)
      if (g_ctx_id[i] == id) {
        *out = g_ctx_ptr[i];
        return DDT_OK;
      }
  }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_verify_scratch) != cudaSuccess || p == nullptr)
    return DDT_ERR_CUDA;
  if (id == 0) id = current_context_id();  // the lookup may have made the context current
  if (id != 0) {
    g_ctx_id[g_ctx_next] = id;
    g_ctx_ptr[g_ctx_next] = p;
    g_ctx_next = (g_ctx_next + 1) % kMaxContexts;
  }
  *out = p;
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
