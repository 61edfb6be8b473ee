// Allocation-free decode entry point: the split-KV partial results live in a
// file-scope device array of fixed size instead of a caller-provided
// workspace.  Everything else is the ordinary mla_decode path.
#include <cudaTypedefs.h>

#include <mutex>

#include "mla_decode.h"
#include "mla_kernels.cuh"

namespace {

// Every GPU that loads the library holds this array until the process exits.
static __device__ __align__(256) unsigned char g_mla_noalloc_scratch[MLA_NOALLOC_SCRATCH_BYTES];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <typename F>
F driver_entry(const char* name) {
  void* ptr = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &ptr, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<F>(ptr);
}

// Unique id of the context current on this thread (0 if none or unknown).
// A context created after a cudaDeviceReset, or one the caller made current
// through the driver API, has a new id even where its handle is reused.
unsigned long long current_context_id() {
  static const CtxGetCurrentFn get_current = driver_entry<CtxGetCurrentFn>("cuCtxGetCurrent");
  static const CtxGetIdFn get_id = driver_entry<CtxGetIdFn>("cuCtxGetId");
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of the array in the current context.  In host code the
// array's name is only a stand-in for the symbol, never a device pointer:
// the address is looked up with cudaGetSymbolAddress, once per context, and
// kept with the context's id (a reset or another context looks it up again).
void* scratch_address() {
  constexpr int kSlots = 64;
  static std::mutex mu;
  static unsigned long long ids[kSlots];
  static void* ptrs[kSlots];
  static int next = 0;
  unsigned long long id = current_context_id();
  if (id != 0) {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < kSlots; ++i)
      if (ids[i] == id) return ptrs[i];
  }
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_mla_noalloc_scratch) != cudaSuccess || ptr == nullptr) return nullptr;
  if (id == 0) id = current_context_id();     // the lookup may have made the primary context current
  if (id != 0) {
    std::lock_guard<std::mutex> lock(mu);
    ids[next] = id;
    ptrs[next] = ptr;
    next = (next + 1) % kSlots;
  }
  return ptr;
}

}  // namespace

extern "C" int mla_decode_noalloc(const mla_decode_args* args, void* stream) {
  if (args == nullptr) return MLA_ERR_INVALID_ARG;
  size_t need = 0;
  const int st = mla_workspace_bytes(args->batch, args->s_q, args->h_q, args->indices ? args->topk : 0,
                                     args->num_parts, &need);
  if (st != MLA_OK) return st;
  if (need > MLA_NOALLOC_SCRATCH_BYTES) return MLA_ERR_WORKSPACE;
  void* scratch = scratch_address();
  if (scratch == nullptr) return MLA_ERR_CUDA;
  mla_decode_args a = *args;
  a.workspace = scratch;
  a.workspace_bytes = MLA_NOALLOC_SCRATCH_BYTES;
  return mla_decode(&a, stream);
}
