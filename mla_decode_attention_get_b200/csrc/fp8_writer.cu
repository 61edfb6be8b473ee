// FP8 cache writer: quantise new key rows (bf16, 576 dims) into the FP8
// cache row format and store them at their cache slots.
//
// Row format: FlashMLA walkthrough (sao.pub), section "二、核心功能与架构",
// KV-cache format list -- 512 e4m3 NoPE values, one float32 scale per 128 of
// them, then the 64 RoPE values unquantised as bf16 (656 bytes).  The pages
// fix the format, not how scales are chosen; this writer takes the plainest
// reading: per 128-value group scale = max|x| / 448 (float32), code = e4m3
// round-to-nearest-even of x / scale (IEEE float32 division), saturating at
// +-448; an all-zero group gets scale 0 and codes 0; RoPE is copied.
//
// One warp per row: lane l converts NoPE dims [16 l, 16 l + 16), which lie
// in group l / 8, so a group's max is a reduction over its 8 lanes.  Every
// store is a 16-B vector store; a row is 41 such stores, 16-B aligned.
#include <cuda_fp8.h>

#include "mla_kernels.cuh"

namespace mla {
namespace {

constexpr int kWriterWarps = 8;   // rows per CTA

__global__ void __launch_bounds__(32 * kWriterWarps)
    fp8_cache_write_kernel(const uint16_t* k_new, int64_t row_stride, int n, const int* slot_mapping,
                           uint8_t* cache, int64_t block_stride, int num_blocks, int* err) {
  const int lane = threadIdx.x & 31;
  const int i = blockIdx.x * kWriterWarps + (threadIdx.x >> 5);
  if (i >= n) return;
  const int slot = slot_mapping[i];
  if (slot == -1) return;
  if (slot < 0 || slot >= num_blocks * kPage) {
    if (lane == 0) atomicOr(err, 1);              // MLA_DEVERR_BLOCK_TABLE: a slot outside the cache
    return;
  }
  const uint16_t* src = k_new + static_cast<int64_t>(i) * row_stride;
  uint8_t* dst = cache + static_cast<int64_t>(slot / kPage) * block_stride + (slot % kPage) * kFp8Row;

  const uint4* s4 = reinterpret_cast<const uint4*>(src) + 2 * lane;
  const uint4 a = s4[0], b = s4[1];
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  float x[16];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    x[2 * k] = __uint_as_float(w[k] << 16);           // bf16 -> float32, exact
    x[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
  }
  float amax = 0.f;
#pragma unroll
  for (int k = 0; k < 16; ++k) amax = fmaxf(amax, fabsf(x[k]));
#pragma unroll
  for (int off = 1; off < 8; off <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const float scale = __fdiv_rn(amax, 448.f);

  uint32_t c[4] = {0u, 0u, 0u, 0u};
  if (amax > 0.f) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float2 q = make_float2(__fdiv_rn(x[2 * k], scale), __fdiv_rn(x[2 * k + 1], scale));
      const uint32_t pair = __nv_cvt_float2_to_fp8x2(q, __NV_SATFINITE, __NV_E4M3);   // .x in the low byte
      c[k >> 1] |= pair << (16 * (k & 1));
    }
  }
  *reinterpret_cast<uint4*>(dst + 16 * lane) = make_uint4(c[0], c[1], c[2], c[3]);

  // the four group scales (lanes 0, 8, 16, 24 hold them) in one 16-B store
  const float s1 = __shfl_sync(0xffffffffu, scale, 8);
  const float s2 = __shfl_sync(0xffffffffu, scale, 16);
  const float s3 = __shfl_sync(0xffffffffu, scale, 24);
  if (lane == 0) *reinterpret_cast<float4*>(dst + 512) = make_float4(scale, s1, s2, s3);
  // RoPE: 128 bytes copied by lanes 0-7
  if (lane < 8) *reinterpret_cast<uint4*>(dst + 528 + 16 * lane) = reinterpret_cast<const uint4*>(src + 512)[lane];
}

}  // namespace

cudaError_t launch_fp8_cache_write(const uint16_t* k_new, int64_t row_stride, int n, const int* slot_mapping,
                                   uint8_t* cache, int64_t block_stride, int num_blocks, int* err,
                                   cudaStream_t stream) {
  const int grid = (n + kWriterWarps - 1) / kWriterWarps;
  fp8_cache_write_kernel<<<grid, 32 * kWriterWarps, 0, stream>>>(k_new, row_stride, n, slot_mapping, cache,
                                                                 block_stride, num_blocks, err);
  return cudaGetLastError();
}

}  // namespace mla
