// LSE-weighted combine of split-KV partial results.
//
// The pages return (o, lse) from the decode and split the KV range through
// num_splits ("Was ist FlashMLA?", sections "2. MLA-Metadaten abrufen" and
// "3. MLA-Decodierung ausführen") without spelling out the merge.  Each split
// s of a row holds its normalised output O_s and log-sum-exp lse_s over a
// disjoint key subset, so the exact merge is
//   lse = M + ln sum_s exp(lse_s - M),  M = max_s lse_s,
//   out = sum_s exp(lse_s - lse) * O_s.
// Rows of units with one split were finished by the decode kernel; units
// with no split (empty key set) get out = 0, lse = -inf here.
#include <cuda_bf16.h>

#include "mla_kernels.cuh"
#include "ptx_sm100.cuh"

namespace mla {
namespace {

constexpr int kRowsPerCta = 4;  // one warp per row

__global__ void __launch_bounds__(32 * kRowsPerCta) combine_kernel(const DecodeParams p) {
  grid_dependency_wait();        // the attention kernel's partials and outputs
  grid_launch_dependents();
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int u = blockIdx.x;
  const int R = p.rows_per_unit;
  const int r = blockIdx.y * kRowsPerCta + warp;
  if (r >= R) return;
  const int s0 = p.num_splits[u];
  const int n = p.num_splits[u + 1] - s0;
  if (n == 1) return;

  int b, tok, h;
  if (p.indices != nullptr) { b = u / p.s_q; tok = u % p.s_q; h = r; }
  else { b = u; tok = r / p.h_q; h = r % p.h_q; }
  uint2* orow = reinterpret_cast<uint2*>(p.out + (static_cast<int64_t>(u) * R + r) * kDv);
  float* lse_out = p.lse + (static_cast<int64_t>(b) * p.h_q + h) * p.s_q + tok;

  // lane k holds the log-sum-exp of splits k, k + 32, ...
  float mx = -INFINITY;
  float l_reg[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int sidx = lane + 32 * i;
    l_reg[i] = sidx < n ? p.ws_lse[static_cast<int64_t>(s0 + sidx) * R + r] : -INFINITY;
    mx = fmaxf(mx, l_reg[i]);
  }
  for (int sidx = lane + 128; sidx < n; sidx += 32) mx = fmaxf(mx, p.ws_lse[static_cast<int64_t>(s0 + sidx) * R + r]);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));

  if (n <= 0 || mx == -INFINITY) {
#pragma unroll
    for (int k = 0; k < 4; ++k) orow[lane + 32 * k] = make_uint2(0, 0);
    if (lane == 0) *lse_out = -INFINITY;
    return;
  }
  float sum = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) sum += expf(l_reg[i] - mx);
  for (int sidx = lane + 128; sidx < n; sidx += 32) sum += expf(p.ws_lse[static_cast<int64_t>(s0 + sidx) * R + r] - mx);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  const float lse = mx + logf(sum);
  float w_reg[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) w_reg[i] = expf(l_reg[i] - lse);

  float4 acc[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
  auto weight = [&](int sidx) -> float {
    if (sidx < 128) {
      float w = w_reg[0];
#pragma unroll
      for (int i = 1; i < 4; ++i) w = (sidx >> 5) == i ? w_reg[i] : w;
      return __shfl_sync(0xffffffffu, w, sidx & 31);
    }
    return expf(p.ws_lse[static_cast<int64_t>(s0 + sidx) * R + r] - lse);
  };
  int sidx = 0;
  for (; sidx + 1 < n; sidx += 2) {
    const float wa = weight(sidx), wb = weight(sidx + 1);
    const float4* a4 = reinterpret_cast<const float4*>(p.ws_o + (static_cast<int64_t>(s0 + sidx) * R + r) * kDv);
    const float4* b4 = reinterpret_cast<const float4*>(p.ws_o + (static_cast<int64_t>(s0 + sidx + 1) * R + r) * kDv);
    float4 va[4], vb[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) { va[k] = a4[lane + 32 * k]; vb[k] = b4[lane + 32 * k]; }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      acc[k].x += wa * va[k].x + wb * vb[k].x;
      acc[k].y += wa * va[k].y + wb * vb[k].y;
      acc[k].z += wa * va[k].z + wb * vb[k].z;
      acc[k].w += wa * va[k].w + wb * vb[k].w;
    }
  }
  if (sidx < n) {
    const float wa = weight(sidx);
    const float4* a4 = reinterpret_cast<const float4*>(p.ws_o + (static_cast<int64_t>(s0 + sidx) * R + r) * kDv);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float4 v = a4[lane + 32 * k];
      acc[k].x += wa * v.x;
      acc[k].y += wa * v.y;
      acc[k].z += wa * v.z;
      acc[k].w += wa * v.w;
    }
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const __nv_bfloat162 lo = __floats2bfloat162_rn(acc[k].x, acc[k].y);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(acc[k].z, acc[k].w);
    orow[lane + 32 * k] = make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
  }
  if (lane == 0) *lse_out = lse;
}

}  // namespace

cudaError_t launch_combine(const DecodeParams& p, cudaStream_t stream) {
  dim3 grid(p.num_units, (p.rows_per_unit + kRowsPerCta - 1) / kRowsPerCta);
  return launch_dependent(combine_kernel, grid, dim3(32 * kRowsPerCta), 0, stream, p);
}

}  // namespace mla
