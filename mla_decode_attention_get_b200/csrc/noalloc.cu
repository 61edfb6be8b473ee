// Allocation-free decode entry point: the split-KV partial results live in a
// file-scope device array of fixed size instead of a caller-provided
// workspace.  Everything else is the ordinary mla_decode path.
#include <atomic>

#include "mla_decode.h"
#include "mla_kernels.cuh"

namespace {

// Every GPU that loads the library holds this array until the process exits.
static __device__ __align__(256) unsigned char g_mla_noalloc_scratch[MLA_NOALLOC_SCRATCH_BYTES];

// Device address of the array, looked up once per device.  In host code the
// array's name is only a stand-in for the symbol, never a device pointer.
void* scratch_address() {
  static std::atomic<void*> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  void* ptr = cache[dev].load(std::memory_order_acquire);
  if (ptr != nullptr) return ptr;
  if (cudaGetSymbolAddress(&ptr, g_mla_noalloc_scratch) != cudaSuccess || ptr == nullptr) return nullptr;
  cache[dev].store(ptr, std::memory_order_release);
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
