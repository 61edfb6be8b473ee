// Internal interface between the C-ABI layer (mla_api.cu) and the kernels.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include <utility>

namespace mla {

constexpr int kPage = 64;
constexpr int kDqk = 576;
constexpr int kDv = 512;
constexpr int kChunks = kDqk / 64;      // 64-dim (128-byte) column blocks of a cache row
constexpr int kFp8Row = 656;
constexpr int kMdWords = 8;
constexpr int kFixedSplitCost = 5;

// Row tile of the decode: the number of (token, head) query rows one CTA
// handles, the M of every tensor-core MMA; units with fewer rows leave the
// rest of the tile as zero padding.
constexpr int kTileRows = 64;

// Largest query-row count of one unit: the combine kernel's grid covers a
// unit's rows 4 to a CTA in its y dimension (at most 65535).
constexpr int kMaxRowsPerUnit = 4 * 65535;

struct DecodeParams {
  const uint16_t* q;          // bf16 bits [batch, s_q, h_q, 576]
  int64_t q_batch_stride;     // elements between batch entries
  const uint8_t* kv;          // cache base (bytes)
  int64_t kv_block_stride;    // bytes between pages
  int num_blocks;
  const int* block_table;
  int bt_stride;
  int bt_width;
  const int* seqlens;
  const int* indices;         // sparse path, else nullptr
  int topk;
  const int* tile_md;
  const int* num_splits;
  int num_parts;
  int num_units;
  uint16_t* out;              // bf16 bits
  float* lse;
  float* ws_o;                // [splits, rows_per_unit, 512]
  float* ws_lse;              // [splits, rows_per_unit]
  int* err;
  int batch, s_q, h_q;
  int rows_per_unit;
  float scale_log2;           // softmax_scale * log2(e)
  int causal;
  uint64_t wait_ns;           // give-up limit of the pipeline waits (drains keep kWaitTimeoutNs)
};

// Launch with programmatic stream serialization: the kernel may start while
// the preceding kernel of the stream drains; it calls grid_dependency_wait()
// before touching memory that kernel reads or writes.
// As launch_dependent, with clusters of cluster_y CTAs along y (1: none).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_dependent_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                            unsigned cluster_y, cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  int n = 1;
  if (cluster_y > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 1;
    attr[1].val.clusterDim.y = cluster_y;
    attr[1].val.clusterDim.z = 1;
    n = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                    cudaStream_t stream, Args&&... args) {
  return launch_dependent_cluster(kernel, grid, block, smem, 1u, stream, std::forward<Args>(args)...);
}

// Launchers (return cudaSuccess or the launch error).
cudaError_t launch_metadata(const int* seqlens, int batch, int s_q, int topk, int num_units, int num_parts,
                            int* tile_md, int* num_splits, int* err, cudaStream_t stream);

// The bf16 cache (TMA page loads through tmap_kv) and the FP8 cache.
cudaError_t launch_decode(const DecodeParams& p, const CUtensorMap& tmap_kv, int row_tiles, cudaStream_t stream);
cudaError_t launch_decode_fp8(const DecodeParams& p, int row_tiles, cudaStream_t stream);

cudaError_t launch_combine(const DecodeParams& p, cudaStream_t stream);

cudaError_t launch_fp8_cache_write(const uint16_t* k_new, int64_t row_stride, int n, const int* slot_mapping,
                                   uint8_t* cache, int64_t block_stride, int num_blocks, int* err,
                                   cudaStream_t stream);

}  // namespace mla
