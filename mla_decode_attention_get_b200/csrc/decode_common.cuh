// Device-side helpers shared by the decode kernels: the partition a CTA
// walks (from the scheduler's tile metadata), per-unit index arithmetic and
// the page cursor.
#pragma once

#include "mla_kernels.cuh"
#include "ptx_sm100.cuh"

namespace mla {
namespace dec {

constexpr int kPageBytes = kPage * kDqk * 2;  // 73728: 64 tokens x 576 bf16
constexpr int kChunkBytes = kPage * 128;      // 8192: 64 rows x 64 dims (one 128-B swizzle column)
constexpr int kPrefetchPages = 4;             // block-table entries read ahead of the TMA loads
constexpr float kRescaleThreshold = 8.0f;     // log2 units
constexpr float kLn2 = 0.69314718055994530942f;
constexpr int kErrBlockTable = 1, kErrIndex = 2, kErrTimeout = 4, kErrSeqlen = 8, kErrInternal = 16;

__device__ __forceinline__ int unit_tiles(const DecodeParams& p, int u) {
  if (p.indices != nullptr) return (p.topk + kPage - 1) / kPage;
  const int L = p.seqlens[u];
  return L > 0 ? (L + kPage - 1) / kPage : 0;
}

// The (unit, page range) segments of this CTA's partition, in order.
struct Partition {
  int u0, j0, u1, j1, first_split;
};

__device__ __forceinline__ Partition load_partition(const DecodeParams& p, int part_idx) {
  const int* md = p.tile_md + part_idx * kMdWords;
  Partition r;
  r.u0 = min(max(md[0], 0), p.num_units);
  r.j0 = max(md[1], 0);
  r.u1 = min(max(md[2], 0), p.num_units);
  r.j1 = max(md[3], 0);
  r.first_split = md[4];
  return r;
}

template <typename F>
__device__ __forceinline__ void for_each_segment(const DecodeParams& p, const Partition& part, F&& f) {
  for (int u = part.u0; u <= part.u1 && u < p.num_units; ++u) {
    const int n = unit_tiles(p, u);
    const int jb = (u == part.u0) ? part.j0 : 0;
    const int je = (u == part.u1) ? min(part.j1, n) : n;
    if (jb >= je) continue;
    if (!f(u, jb, je)) return;
  }
}

__device__ __forceinline__ void raise_abort(volatile int* abort_flag, int* err) {
  if (!*abort_flag) {
    *abort_flag = 1;
    atomicOr(err, kErrTimeout);
  }
}

// Index arithmetic of a work unit.
struct UnitInfo {
  int b, token;      // token: query token of a sparse unit, -1 on the dense path
  int L;
};

__device__ __forceinline__ UnitInfo unit_info(const DecodeParams& p, int u) {
  UnitInfo x;
  if (p.indices != nullptr) {
    x.b = u / p.s_q;
    x.token = u % p.s_q;
  } else {
    x.b = u;
    x.token = -1;
  }
  x.L = max(p.seqlens[x.b], 0);
  return x;
}

__device__ __forceinline__ int page_of(const DecodeParams& p, int b, int j) {
  return j < p.bt_width ? p.block_table[static_cast<int64_t>(b) * p.bt_stride + j] : -1;
}

// Walks the pages of a partition in order: unit u, page j of [jb, je), global
// page index t, segment index seg.
struct Cursor {
  int u, j, je, t, seg;
  bool valid;
};

__device__ __forceinline__ bool segment_bounds(const DecodeParams& p, const Partition& part, int u, int& jb,
                                               int& je) {
  const int n = unit_tiles(p, u);
  jb = (u == part.u0) ? part.j0 : 0;
  je = (u == part.u1) ? min(part.j1, n) : n;
  return jb < je;
}

__device__ __forceinline__ void cursor_seek(const DecodeParams& p, const Partition& part, Cursor& c, int u_from) {
  for (int u = u_from; u <= part.u1 && u < p.num_units; ++u) {
    int jb, je;
    if (segment_bounds(p, part, u, jb, je)) {
      c.u = u;
      c.j = jb;
      c.je = je;
      c.valid = true;
      return;
    }
  }
  c.valid = false;
}

__device__ __forceinline__ Cursor cursor_begin(const DecodeParams& p, const Partition& part) {
  Cursor c;
  c.t = 0;
  c.seg = 0;
  cursor_seek(p, part, c, part.u0);
  return c;
}

__device__ __forceinline__ void cursor_next(const DecodeParams& p, const Partition& part, Cursor& c) {
  ++c.t;
  if (++c.j < c.je) return;
  ++c.seg;
  cursor_seek(p, part, c, c.u + 1);
}

// Element offset in q of row `tile_row0` of a unit (rows are (token, head)
// pairs, token-major; a sparse unit is one token).
__device__ __forceinline__ int64_t q_tile_offset(const DecodeParams& p, const UnitInfo& ui, int tile_row0) {
  const int row0 = (ui.token >= 0 ? ui.token * p.h_q : 0) + tile_row0;
  return static_cast<int64_t>(ui.b) * p.q_batch_stride + static_cast<int64_t>(row0) * kDqk;
}

}  // namespace dec
}  // namespace mla
