// C ABI of the MLA decode library: argument validation, the split plan's
// sizes, TMA tensor-map encoding, and the kernel launches.  Declarations and
// the meaning of every argument are in include/mla_decode.h.
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdint>
#include <cmath>
#include <cstring>

#include "mla_decode.h"
#include "mla_kernels.cuh"
#include "ptx_sm100.cuh"

namespace {

using mla::kDqk;
using mla::kDv;
using mla::kPage;

struct Plan {
  int units;          // sequences (dense) or (sequence, token) pairs (sparse)
  int rows_per_unit;  // s_q * h_q (dense) or h_q (sparse)
  int row_tiles;      // 64-row tiles per unit (one CTA each per partition)
};

int make_plan(int batch, int s_q, int h_q, int h_kv, int topk, Plan* pl) {
  if (batch < 1 || s_q < 1 || h_q < 1 || topk < 0) return MLA_ERR_INVALID_ARG;
  if (h_kv != 1) return MLA_ERR_UNSUPPORTED;
  const long long rows = static_cast<long long>(s_q) * h_q;
  const long long units = topk > 0 ? static_cast<long long>(batch) * s_q : batch;
  if (units > (1 << 24)) return MLA_ERR_INVALID_ARG;
  const long long rows_per_unit = topk > 0 ? h_q : rows;
  // the combine kernel's grid spans a unit's rows in its y dimension
  if (rows_per_unit > mla::kMaxRowsPerUnit) return MLA_ERR_UNSUPPORTED;
  pl->units = static_cast<int>(units);
  pl->rows_per_unit = static_cast<int>(rows_per_unit);
  pl->row_tiles = (pl->rows_per_unit + mla::kTileRows - 1) / mla::kTileRows;
  return MLA_OK;
}

int device_sm_count(int* out) {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  if (dev >= 0 && dev < 64) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) { *out = c; return MLA_OK; }
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return MLA_ERR_CUDA;
  if (dev >= 0 && dev < 64) cache[dev].store(n, std::memory_order_relaxed);
  *out = n;
  return MLA_OK;
}

size_t lse_region_bytes(const Plan& pl, int num_parts) {
  const size_t splits = static_cast<size_t>(pl.units) + static_cast<size_t>(num_parts);
  return (splits * pl.rows_per_unit * sizeof(float) + 255) & ~size_t(255);
}

size_t workspace_need(const Plan& pl, int num_parts) {
  const size_t splits = static_cast<size_t>(pl.units) + static_cast<size_t>(num_parts);
  const size_t o_bytes = splits * pl.rows_per_unit * kDv * sizeof(float);
  return o_bytes + lse_region_bytes(pl, num_parts);
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static std::atomic<PFN_cuTensorMapEncodeTiled_v12000> fn{nullptr};
  PFN_cuTensorMapEncodeTiled_v12000 f = fn.load();
  if (f) return f;
  void* ptr = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || ptr == nullptr)
    return nullptr;
  f = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  fn.store(f);
  return f;
}

// bf16 3-D map with 128-byte swizzle: dims {576, d1, d2}, byte strides {s1, s2}, box {64, box1, 1}.
bool encode_bf16_map(CUtensorMap* map, const void* base, uint64_t d1, uint64_t d2, uint64_t s1, uint64_t s2,
                     uint32_t box1) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kDqk), d1, d2};
  const cuuint64_t strides[2] = {s1, s2};
  const cuuint32_t box[3] = {64, box1, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Give-up limit of the kernels' pipeline waits for the calls that follow
// (mla_set_pipeline_wait_limit); 0 = the default.
std::atomic<uint64_t> g_wait_limit_ns{0};

// Validates a decode call and fills the kernel parameters.
int prepare(const mla_decode_args* a, Plan* pl, mla::DecodeParams* kp) {
  if (a == nullptr) return MLA_ERR_INVALID_ARG;
  int st = make_plan(a->batch, a->s_q, a->h_q, a->h_kv, a->indices ? a->topk : 0, pl);
  if (st != MLA_OK) return st;
  if (a->d_v != kDv) return MLA_ERR_UNSUPPORTED;
  if (a->indices != nullptr && !a->is_fp8) return MLA_ERR_UNSUPPORTED;  // bf16 sparse
  if (a->indices != nullptr && a->topk < 1) return MLA_ERR_INVALID_ARG;
  if (!a->q || !a->k_cache || !a->block_table || !a->cache_seqlens || !a->tile_md || !a->num_splits || !a->out ||
      !a->lse || !a->err_word || !a->workspace)
    return MLA_ERR_INVALID_ARG;
  if (a->num_parts < 1 || a->num_blocks < 1 || a->block_table_width < 1 ||
      a->block_table_stride < a->block_table_width)
    return MLA_ERR_INVALID_ARG;
  const int64_t page_bytes = a->is_fp8 ? int64_t(kPage) * mla::kFp8Row : int64_t(kPage) * kDqk * 2;
  if (!aligned(a->q, 16) || !aligned(a->k_cache, 16) || !aligned(a->out, 16) || !aligned(a->lse, 4) ||
      !aligned(a->workspace, 256) || !aligned(a->err_word, 4))
    return MLA_ERR_INVALID_ARG;
  if (a->k_block_stride < page_bytes || a->k_block_stride % 16 != 0) return MLA_ERR_INVALID_ARG;
  const int64_t rows = int64_t(a->s_q) * a->h_q;
  if (a->q_batch_stride < rows * kDqk || a->q_batch_stride % 8 != 0) return MLA_ERR_INVALID_ARG;
  if (!std::isfinite(a->softmax_scale) || !(a->softmax_scale > 0.f)) return MLA_ERR_INVALID_ARG;
  if (a->workspace_bytes < workspace_need(*pl, a->num_parts)) return MLA_ERR_WORKSPACE;

  std::memset(kp, 0, sizeof(*kp));
  kp->q = static_cast<const uint16_t*>(a->q);
  kp->q_batch_stride = a->q_batch_stride;
  kp->kv = static_cast<const uint8_t*>(a->k_cache);
  kp->kv_block_stride = a->k_block_stride;
  kp->num_blocks = a->num_blocks;
  kp->block_table = a->block_table;
  kp->bt_stride = a->block_table_stride;
  kp->bt_width = a->block_table_width;
  kp->seqlens = a->cache_seqlens;
  kp->indices = a->indices;
  kp->topk = a->indices ? a->topk : 0;
  kp->tile_md = a->tile_md;
  kp->num_splits = a->num_splits;
  kp->num_parts = a->num_parts;
  kp->num_units = pl->units;
  kp->out = static_cast<uint16_t*>(a->out);
  kp->lse = a->lse;
  const size_t splits = static_cast<size_t>(pl->units) + static_cast<size_t>(a->num_parts);
  kp->ws_o = static_cast<float*>(a->workspace);
  kp->ws_lse = kp->ws_o + splits * pl->rows_per_unit * kDv;
  kp->err = a->err_word;
  kp->batch = a->batch;
  kp->s_q = a->s_q;
  kp->h_q = a->h_q;
  kp->rows_per_unit = pl->rows_per_unit;
  kp->scale_log2 = a->softmax_scale * 1.4426950408889634f;
  kp->causal = a->causal ? 1 : 0;
  const uint64_t lim = g_wait_limit_ns.load(std::memory_order_relaxed);
  kp->wait_ns = lim ? lim : mla::kWaitTimeoutNs;
  return MLA_OK;
}

}  // namespace

extern "C" {

int mla_metadata_shape(int batch, int s_q, int h_q, int h_kv, int topk, int num_sm_parts, int* num_parts_out,
                       int* num_splits_len_out) {
  if (!num_parts_out || !num_splits_len_out) return MLA_ERR_INVALID_ARG;
  Plan pl;
  int st = make_plan(batch, s_q, h_q, h_kv, topk, &pl);
  if (st != MLA_OK) return st;
  int parts = num_sm_parts;
  if (parts <= 0) {
    int sms = 0;
    st = device_sm_count(&sms);
    if (st != MLA_OK) return st;
    // one CTA per SM: a partition per SM and row tile
    parts = sms / pl.row_tiles;
    if (parts < 1) parts = 1;
  }
  if (parts > (1 << 16)) return MLA_ERR_INVALID_ARG;
  *num_parts_out = parts;
  *num_splits_len_out = pl.units + 1;
  return MLA_OK;
}

int mla_get_metadata(const int32_t* cache_seqlens, int batch, int s_q, int h_q, int h_kv, int topk, int num_parts,
                     int32_t* tile_md, int32_t* num_splits, void* stream) {
  Plan pl;
  int st = make_plan(batch, s_q, h_q, h_kv, topk, &pl);
  if (st != MLA_OK) return st;
  if (!cache_seqlens || !tile_md || !num_splits || num_parts < 1 || num_parts > (1 << 16)) return MLA_ERR_INVALID_ARG;
  const cudaError_t e = mla::launch_metadata(cache_seqlens, batch, s_q, topk, pl.units, num_parts, tile_md,
                                             num_splits, nullptr, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

int mla_workspace_bytes(int batch, int s_q, int h_q, int topk, int num_parts, size_t* bytes) {
  if (!bytes || num_parts < 1) return MLA_ERR_INVALID_ARG;
  Plan pl;
  const int st = make_plan(batch, s_q, h_q, 1, topk, &pl);
  if (st != MLA_OK) return st;
  *bytes = workspace_need(pl, num_parts);
  return MLA_OK;
}

int mla_decode_attention(const mla_decode_args* a, void* stream) {
  Plan pl;
  mla::DecodeParams kp;
  int st = prepare(a, &pl, &kp);
  if (st != MLA_OK) return st;
  CUtensorMap tkv;
  std::memset(&tkv, 0, sizeof(tkv));
  if (!a->is_fp8 && !encode_bf16_map(&tkv, a->k_cache, uint64_t(kPage), uint64_t(a->num_blocks),
                                     uint64_t(kDqk) * 2, uint64_t(a->k_block_stride), kPage))
    return MLA_ERR_CUDA;
  const cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const cudaError_t e =
      a->is_fp8 ? mla::launch_decode_fp8(kp, pl.row_tiles, cs) : mla::launch_decode(kp, tkv, pl.row_tiles, cs);
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

int mla_decode_combine(const mla_decode_args* a, void* stream) {
  Plan pl;
  mla::DecodeParams kp;
  const int st = prepare(a, &pl, &kp);
  if (st != MLA_OK) return st;
  const cudaError_t e = mla::launch_combine(kp, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

int mla_decode(const mla_decode_args* a, void* stream) {
  const int st = mla_decode_attention(a, stream);
  if (st != MLA_OK) return st;
  return mla_decode_combine(a, stream);
}

int mla_fp8_cache_write(const void* k_new, int64_t k_row_stride, int32_t n, const int32_t* slot_mapping,
                        void* kv_cache, int64_t k_block_stride, int32_t num_blocks, int32_t* err_word,
                        void* stream) {
  if (n < 0 || num_blocks < 1) return MLA_ERR_INVALID_ARG;
  if (n == 0) return MLA_OK;
  if (!k_new || !slot_mapping || !kv_cache || !err_word) return MLA_ERR_INVALID_ARG;
  if (!aligned(k_new, 16) || !aligned(kv_cache, 16) || !aligned(slot_mapping, 4) || !aligned(err_word, 4))
    return MLA_ERR_INVALID_ARG;
  if (k_row_stride < kDqk || k_row_stride % 8 != 0) return MLA_ERR_INVALID_ARG;
  if (k_block_stride < int64_t(kPage) * mla::kFp8Row || k_block_stride % 16 != 0) return MLA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(num_blocks) * kPage > INT32_MAX) return MLA_ERR_INVALID_ARG;
  const cudaError_t e = mla::launch_fp8_cache_write(static_cast<const uint16_t*>(k_new), k_row_stride, n, slot_mapping,
                                                    static_cast<uint8_t*>(kv_cache), k_block_stride, num_blocks,
                                                    err_word, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

int mla_set_pipeline_wait_limit(uint64_t ns) {
  g_wait_limit_ns.store(ns, std::memory_order_relaxed);
  return MLA_OK;
}

const char* mla_status_string(int status) {
  switch (status) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG: invalid argument";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED: unsupported configuration";
    case MLA_ERR_WORKSPACE: return "MLA_ERR_WORKSPACE: workspace too small";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA: CUDA call failed";
    default: return "MLA_ERR_UNKNOWN";
  }
}

}  // extern "C"
