// MLA decode attention over a paged KV cache on sm_100a (tcgen05 + TMEM + TMA).
//
// What it computes (per query row = (token, head), h_kv = 1): logits
// s_t = scale * q . K_t over the 576 cache dims of every visible key t,
// out = sum_t softmax(s)_t * K_t[:512] and lse = ln sum_t exp(s_t)
// ("Was ist FlashMLA?" (topnet.top), section "3. MLA-Decodierung ausführen":
// o_i, lse_i = flash_mla_with_kvcache(q, kvcache, block_table,
// cache_seqlens, dv, metadata, num_splits, causal)).  The sparse variant
// attends only to the cache positions an indices tensor names, reading FP8
// rows (512 e4m3 + 4 fp32 scales + 64 bf16 RoPE) -- FlashMLA walkthrough
// (sao.pub), section "二、核心功能与架构".
//
// Design (one CTA = one scheduler partition x one tile of N <= 64 query rows):
//  * Keys sit on the tensor-core M dimension ("swap AB"): for each 64-token
//    page, S^T[64 keys, N rows] = K_page[64, 576] . Q^T is one M=64
//    tcgen05.mma chain with S^T in TMEM; then O^T[512, N] += V^T . P^T as four
//    M=128 MMAs (V^T is read MN-major straight from the same swizzled page
//    tile, so V costs no extra load).  O^T lives in TMEM for the whole
//    segment: 4N columns, plus two N-column S^T buffers.
//  * Warp 0 streams pages with TMA (3-D tensor map, 128-byte swizzle, one
//    page = 9 boxes of 64 tokens x 64 dims) into a 2-stage ring; warp 1
//    issues the MMAs; warps 2-5 run the online softmax (one key per TMEM
//    lane, warp-wide max via redux.sync, exp2 with the scale folded in, P^T
//    written as bf16 into a swizzled K-major tile) and the epilogue.  On the
//    FP8 sparse path warps 6-9 gather the indexed rows and dequantise them
//    into the same bf16 page layout.
//  * The running max is only moved when a tile's max exceeds it by more than
//    2^8; the final division by the row sum uses the same stale max, so the
//    result is exact.
//  * Every wait is bounded; on timeout the CTA raises MLA_DEVERR_TIMEOUT,
//    drains its own copies and MMAs, frees TMEM and returns.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "mla_kernels.cuh"
#include "ptx_sm100.cuh"

namespace mla {
namespace {

constexpr int kStages = 2;
constexpr int kPageBytes = kPage * kDqk * 2;  // 73728: 64 tokens x 576 bf16
constexpr int kChunkBytes = kPage * 128;      // 8192: 64 tokens x 64 dims
constexpr float kRescaleThreshold = 8.0f;     // log2 units
constexpr float kLn2 = 0.69314718055994530942f;
constexpr int kErrBlockTable = 1, kErrIndex = 2, kErrTimeout = 4, kErrSeqlen = 8, kErrInternal = 16;

constexpr int kWarpLoad = 0, kWarpMma = 1, kWarpSoftmax0 = 2, kWarpDequant0 = 6;

template <int N>
struct Smem {
  static constexpr int q_chunk = N * 128;                    // one 64-dim block of N query rows
  static constexpr int q_off = 0;
  static constexpr int kv_off = q_off + kChunks * q_chunk;   // multiple of 1024
  static constexpr int p_off = kv_off + kStages * kPageBytes;
  static constexpr int red_off = p_off + N * 128;
  static constexpr int red_bytes = 2 * 4 * N * 4;
  static constexpr int bar_off = red_off + red_bytes;
  // kv_full[S], kv_empty[S], s_full[2], s_empty[2], q_full, q_empty, p_full, p_empty, done, sm_sync
  static constexpr int n_bars = 2 * kStages + 4 + 6;
  static constexpr int info_off = bar_off + n_bars * 8;
  static constexpr int info_bytes = kStages * 16;            // per stage: int nvalid; uint16 mask[4]
  static constexpr int misc_off = info_off + info_bytes;     // tmem base, abort flag
  static constexpr int total = misc_off + 16;
  static_assert(kv_off % 1024 == 0 && p_off % 1024 == 0, "tiles must stay 1024-B aligned");
  static_assert(total <= 232448, "shared memory budget");
};

template <int N>
constexpr uint32_t tmem_cols() {
  return (6 * N) <= 128 ? 128u : ((6 * N) <= 256 ? 256u : 512u);
}

struct StageInfo {
  int nvalid;
  uint16_t mask[4];
  int pad;
};

struct Bars {
  uint64_t* kv_full;
  uint64_t* kv_empty;
  uint64_t* s_full;
  uint64_t* s_empty;
  uint64_t* q_full;
  uint64_t* q_empty;
  uint64_t* p_full;
  uint64_t* p_empty;
  uint64_t* done;
  uint64_t* sm_sync;
};

__device__ __forceinline__ int unit_tiles(const DecodeParams& p, int u) {
  if (p.indices != nullptr) return (p.topk + kPage - 1) / kPage;
  const int L = p.seqlens[u];
  return L > 0 ? (L + kPage - 1) / kPage : 0;
}

// The (unit, page range) segments of this CTA's partition, in order.
struct Partition {
  int u0, j0, u1, j1, first_split;
};

__device__ __forceinline__ Partition load_partition(const DecodeParams& p) {
  const int* md = p.tile_md + blockIdx.x * kMdWords;
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

// ---------------------------------------------------------------------------
// Warp 0: TMA loads of the query tile (once per segment) and of cache pages.
template <int N, bool FP8>
__device__ void load_role(const DecodeParams& p, const Partition& part, const CUtensorMap* tmap_q,
                          const CUtensorMap* tmap_kv, uint8_t* smem, Bars bars, StageInfo* info,
                          volatile int* abort_flag) {
  using L = Smem<N>;
  const uint64_t pol_kv = l2_policy_evict_first();
  const uint64_t pol_q = l2_policy_evict_last();
  const int row0 = blockIdx.y * N;
  int t = 0, seg = 0;
  int last_t[kStages] = {-1, -1};
  int q_last = -1;  // segment index of the last query-tile load issued
  bool ok = true;

  auto load_q = [&](const UnitInfo& ui) -> bool {
    if (!mbar_wait(bars.q_empty, (seg & 1) ^ 1, abort_flag)) return false;
    mbar_arrive_expect_tx(bars.q_full, kChunks * L::q_chunk);
    const int y = (ui.token >= 0 ? ui.token * p.h_q : 0) + row0;
#pragma unroll 1
    for (int c = 0; c < kChunks; ++c)
      tma_load_3d(smem + L::q_off + c * L::q_chunk, tmap_q, bars.q_full, 64 * c, y, ui.b, pol_q);
    q_last = seg;
    return true;
  };

  for_each_segment(p, part, [&](int u, int jb, int je) -> bool {
    const UnitInfo ui = unit_info(p, u);
    if (FP8) {
      if (!load_q(ui)) { ok = false; return false; }
      ++seg;
      return true;
    }
    for (int j = jb; j < je; ++j) {
      const int s = t % kStages;
      if (!mbar_wait(&bars.kv_empty[s], ((t / kStages) & 1) ^ 1, abort_flag)) { ok = false; return false; }
      int nv = min(kPage, ui.L - kPage * j);
      int phys = -1;
      if (j < p.bt_width) phys = p.block_table[static_cast<int64_t>(ui.b) * p.bt_stride + j];
      if (j >= p.bt_width || phys < 0 || phys >= p.num_blocks) {
        atomicOr(p.err, kErrBlockTable);
        nv = 0;
      }
      info[s].nvalid = nv;
      if (nv > 0) {
        mbar_arrive_expect_tx(&bars.kv_full[s], kPageBytes);
        uint8_t* dst = smem + L::kv_off + s * kPageBytes;
#pragma unroll 1
        for (int c = 0; c < kChunks; ++c)
          tma_load_3d(dst + c * kChunkBytes, tmap_kv, &bars.kv_full[s], 64 * c, 0, phys, pol_kv);
        last_t[s] = t;
      } else {
        mbar_arrive(&bars.kv_full[s]);
      }
      if (j == jb) {
        if (!load_q(ui)) { ok = false; return false; }
      }
      ++t;
    }
    ++seg;
    return true;
  });

  if (!ok) {
    raise_abort(abort_flag, p.err);
    // Drain this warp's own copies before the CTA tears down.
    const uint64_t t0 = globaltimer_ns();
    for (int s = 0; s < kStages; ++s) {
      if (last_t[s] < 0) continue;
      while (!mbar_try_wait(&bars.kv_full[s], (last_t[s] / kStages) & 1) &&
             globaltimer_ns() - t0 < kWaitTimeoutNs) {
      }
    }
    if (q_last >= 0) {
      while (!mbar_try_wait(bars.q_full, q_last & 1) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Warps 6-9 (FP8 sparse path): gather the rows the indices name, dequantise
// NoPE (e4m3 x per-128 scale) and copy RoPE into the bf16 swizzled page tile.
template <int N>
__device__ void dequant_role(const DecodeParams& p, const Partition& part, uint8_t* smem, Bars bars,
                             StageInfo* info, volatile int* abort_flag, int dq) {
  using L = Smem<N>;
  const int lane = threadIdx.x & 31;
  int t = 0;
  bool ok = true;
  for_each_segment(p, part, [&](int u, int jb, int je) -> bool {
    const UnitInfo ui = unit_info(p, u);
    const int* idx_row = p.indices + static_cast<int64_t>(u) * p.topk;
    for (int j = jb; j < je; ++j) {
      const int s = t % kStages;
      if (!mbar_wait(&bars.kv_empty[s], ((t / kStages) & 1) ^ 1, abort_flag)) { ok = false; return false; }
      uint8_t* stage = smem + L::kv_off + s * kPageBytes;
      uint32_t mask = 0;
#pragma unroll 1
      for (int kb = 0; kb < 4; ++kb) {
        const uint8_t* rows[4];
        bool valid[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int k = 16 * dq + 4 * kb + e;
          const int pos_i = kPage * j + k;
          const int pos = pos_i < p.topk ? idx_row[pos_i] : -1;
          bool v = pos >= 0 && pos < ui.L;
          if (!v && pos != -1 && lane == 0) atomicOr(p.err, kErrIndex);
          int phys = -1;
          if (v) {
            const int page = pos >> 6;
            phys = page < p.bt_width ? p.block_table[static_cast<int64_t>(ui.b) * p.bt_stride + page] : -1;
            if (phys < 0 || phys >= p.num_blocks) {
              if (lane == 0) atomicOr(p.err, kErrBlockTable);
              v = false;
            }
          }
          valid[e] = v;
          rows[e] = v ? p.kv + static_cast<int64_t>(phys) * p.kv_block_stride + (pos & 63) * kFp8Row : nullptr;
        }
        uint4 nope[4], rope[4];
        float scale[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          nope[e] = make_uint4(0, 0, 0, 0);
          rope[e] = make_uint4(0, 0, 0, 0);
          scale[e] = 0.f;
          if (valid[e]) {
            nope[e] = __ldg(reinterpret_cast<const uint4*>(rows[e] + 16 * lane));
            scale[e] = __ldg(reinterpret_cast<const float*>(rows[e] + 512 + 4 * (lane >> 3)));
            if (lane < 8) rope[e] = __ldg(reinterpret_cast<const uint4*>(rows[e] + 528 + 16 * lane));
          }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int k = 16 * dq + 4 * kb + e;   // token row of the tile
          const int sw = k & 7;
          // NoPE dims [16*lane, 16*lane + 16): block c = lane / 4, 16-B chunks 2*(lane%4) and +1
          uint32_t w[4] = {nope[e].x, nope[e].y, nope[e].z, nope[e].w};
          uint32_t o[8];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w[i] & 0xFFFFu), __NV_E4M3);
            const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w[i] >> 16), __NV_E4M3);
            const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&lo));
            const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&hi));
            const __nv_bfloat162 pa = __floats2bfloat162_rn(a.x * scale[e], a.y * scale[e]);
            const __nv_bfloat162 pb = __floats2bfloat162_rn(b.x * scale[e], b.y * scale[e]);
            o[2 * i] = *reinterpret_cast<const uint32_t*>(&pa);
            o[2 * i + 1] = *reinterpret_cast<const uint32_t*>(&pb);
          }
          const int c = lane >> 2;
          const int ch0 = 2 * (lane & 3);
          uint8_t* rowp = stage + c * kChunkBytes + k * 128;
          *reinterpret_cast<uint4*>(rowp + (((ch0) ^ sw) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
          *reinterpret_cast<uint4*>(rowp + (((ch0 + 1) ^ sw) << 4)) = make_uint4(o[4], o[5], o[6], o[7]);
          if (lane < 8) {
            uint8_t* rp = stage + 8 * kChunkBytes + k * 128;
            *reinterpret_cast<uint4*>(rp + ((lane ^ sw) << 4)) = rope[e];
          }
          if (valid[e]) mask |= 1u << (4 * kb + e);
        }
      }
      if (lane == 0) info[s].mask[dq] = static_cast<uint16_t>(mask);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.kv_full[s]);
      ++t;
    }
    return true;
  });
  if (!ok) raise_abort(abort_flag, p.err);
}

__device__ __forceinline__ int stage_nvalid(const StageInfo& si, bool fp8) {
  if (!fp8) return si.nvalid;
  return __popc(si.mask[0]) + __popc(si.mask[1]) + __popc(si.mask[2]) + __popc(si.mask[3]);
}

// ---------------------------------------------------------------------------
// Warp 1 (one lane): QK^T and PV MMAs.
template <int N, bool FP8>
__device__ void mma_role(const DecodeParams& p, const Partition& part, uint8_t* smem, Bars bars,
                         const StageInfo* info, uint32_t tmem_base, volatile int* abort_flag) {
  using L = Smem<N>;
  constexpr uint32_t idesc_qk = idesc_bf16_f32(64, N, false, false);
  constexpr uint32_t idesc_pv = idesc_bf16_f32(128, N, true, false);
  const uint32_t q_addr = smem_u32(smem + L::q_off);
  const uint32_t kv_addr = smem_u32(smem + L::kv_off);
  const uint32_t p_addr = smem_u32(smem + L::p_off);
  const uint32_t tmem_s[2] = {tmem_base + 4 * N, tmem_base + 5 * N};

  int t = 0, seg = 0;
  int pv_t = -1, pv_nv = 0, pv_seg = -1, pv_stage = 0, o_seg = -1;
  bool ok = true;

  auto issue_pv = [&]() -> bool {
    if (!mbar_wait(bars.p_full, pv_t & 1, abort_flag)) return false;
    tc_fence_after();
    if (pv_nv > 0) {
      const bool acc0 = (o_seg == pv_seg);
      const uint32_t stage = kv_addr + pv_stage * kPageBytes;
#pragma unroll
      for (int jb = 0; jb < 4; ++jb) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint64_t a = sdesc_sw128(stage + (2 * jb) * kChunkBytes + k * 2048, kChunkBytes, 1024);
          const uint64_t b = sdesc_sw128(p_addr + k * 32, 16, 1024);
          umma_bf16(tmem_base + jb * N, a, b, idesc_pv, (acc0 || k > 0) ? 1u : 0u);
        }
      }
      o_seg = pv_seg;
    }
    umma_commit(&bars.kv_empty[pv_stage]);
    umma_commit(bars.p_empty);
    return true;
  };

  for_each_segment(p, part, [&](int u, int jb, int je) -> bool {
    (void)u;
    for (int j = jb; j < je; ++j) {
      const int s = t % kStages;
      const int sb = t & 1;
      if (!mbar_wait(&bars.kv_full[s], (t / kStages) & 1, abort_flag)) { ok = false; return false; }
      if (j == jb && !mbar_wait(bars.q_full, seg & 1, abort_flag)) { ok = false; return false; }
      if (!mbar_wait(&bars.s_empty[sb], ((t >> 1) & 1) ^ 1, abort_flag)) { ok = false; return false; }
      tc_fence_after();
      const int nv = stage_nvalid(info[s], FP8);
      if (nv > 0) {
        const uint32_t stage = kv_addr + s * kPageBytes;
#pragma unroll 1
        for (int c = 0; c < kChunks; ++c) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t a = sdesc_sw128(stage + c * kChunkBytes + k * 32, 16, 1024);
            const uint64_t b = sdesc_sw128(q_addr + c * L::q_chunk + k * 32, 16, 1024);
            umma_bf16(tmem_s[sb], a, b, idesc_qk, (c | k) != 0 ? 1u : 0u);
          }
        }
      }
      umma_commit(&bars.s_full[sb]);
      if (j == je - 1) umma_commit(bars.q_empty);
      if (pv_t >= 0 && !issue_pv()) { ok = false; return false; }
      pv_t = t;
      pv_nv = nv;
      pv_seg = seg;
      pv_stage = s;
      ++t;
    }
    ++seg;
    return true;
  });
  if (ok && pv_t >= 0) ok = issue_pv();
  if (!ok) raise_abort(abort_flag, p.err);
  // Wait until every MMA this warp issued has completed.
  umma_commit(bars.done);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bars.done, 0) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
  }
}

// ---------------------------------------------------------------------------
// Warps 2-5: online softmax per page and the per-segment epilogue.
template <int N, bool FP8>
__device__ void softmax_role(const DecodeParams& p, const Partition& part, uint8_t* smem, Bars bars,
                             const StageInfo* info, uint32_t tmem_base, volatile int* abort_flag) {
  using L = Smem<N>;
  const int lane = threadIdx.x & 31;
  const int q4 = (threadIdx.x >> 5) & 3;            // TMEM lane quadrant of this warp
  const uint32_t lane_off = static_cast<uint32_t>(32 * q4) << 16;
  const bool key_lane = lane < 16;                  // M=64 accumulators use lanes 0-15 of each quadrant
  const int key = 16 * q4 + lane;
  const uint32_t tmem_s[2] = {tmem_base + 4 * N, tmem_base + 5 * N};
  float* red_base = reinterpret_cast<float*>(smem + L::red_off);
  uint8_t* p_tile = smem + L::p_off;
  const int row0 = blockIdx.y * N;
  const int R = p.rows_per_unit;

  float m_run[N], l_run[N];
  int t = 0, seg = 0, sync_uses = 0;
  bool ok = true;

  auto group_sync = [&]() -> bool {
    __syncwarp();
    if (lane == 0) mbar_arrive(bars.sm_sync);
    const bool r = mbar_wait(bars.sm_sync, sync_uses & 1, abort_flag);
    ++sync_uses;
    return r;
  };

  for_each_segment(p, part, [&](int u, int jb, int je) -> bool {
    const UnitInfo ui = unit_info(p, u);
    if (!FP8 && lane == 0 && q4 == 0 && p.seqlens[ui.b] < 0) atomicOr(p.err, kErrSeqlen);
#pragma unroll
    for (int c = 0; c < N; ++c) {
      m_run[c] = -INFINITY;
      l_run[c] = 0.f;
    }
    bool any_pv = false;
    // causal limit: key position must be <= L - s_q + token(row)
    const bool causal = !FP8 && p.causal != 0;
    for (int j = jb; j < je; ++j) {
      const int s = t % kStages;
      const int sb = t & 1;
      if (!mbar_wait(&bars.kv_full[s], (t / kStages) & 1, abort_flag)) { ok = false; return false; }
      if (!mbar_wait(&bars.s_full[sb], (t >> 1) & 1, abort_flag)) { ok = false; return false; }
      tc_fence_after();
      const int nv = stage_nvalid(info[s], FP8);
      bool kvalid;
      if (FP8) {
        const uint32_t m16 = info[s].mask[q4];
        kvalid = key_lane && ((m16 >> lane) & 1u);
      } else {
        kvalid = key_lane && key < nv;
      }
      const int kpos = kPage * j + key;
      const bool causal_pg = causal && (kPage * j + kPage - 1 > ui.L - p.s_q);
      float* red = red_base + (t & 1) * 4 * N;

      auto logit = [&](float raw, int c) -> float {
        bool v = kvalid;
        if (causal_pg) {
          const int tok = (row0 + c) / p.h_q;
          v = v && (kpos <= ui.L - p.s_q + tok);
        }
        return v ? raw * p.scale_log2 : -INFINITY;
      };

      // pass 1: per-row maxima of this page
      if (nv > 0) {
#pragma unroll
        for (int g = 0; g < N / 16; ++g) {
          float v[16];
          tmem_ld16(tmem_s[sb] + lane_off + 16 * g, v);
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const float mx = warp_max_f32(logit(v[c], 16 * g + c));
            if (lane == 0) red[q4 * N + 16 * g + c] = mx;
          }
        }
      }
      if (!group_sync()) { ok = false; return false; }

      // new maxima; rescale only when some row's max grew by more than 2^8
      bool need = false;
      if (nv > 0) {
#pragma unroll
        for (int c = 0; c < N; ++c) {
          const float tm = fmaxf(fmaxf(red[c], red[N + c]), fmaxf(red[2 * N + c], red[3 * N + c]));
          need |= tm > m_run[c] + kRescaleThreshold;
        }
      }
      if (t > 0 && !mbar_wait(bars.p_empty, (t - 1) & 1, abort_flag)) { ok = false; return false; }
      tc_fence_after();
      if (need) {
        if (any_pv) {
#pragma unroll 1
          for (int jb4 = 0; jb4 < 4; ++jb4) {
#pragma unroll
            for (int g = 0; g < N / 16; ++g) {
              float v[16];
              const uint32_t addr = tmem_base + lane_off + jb4 * N + 16 * g;
              tmem_ld16(addr, v);
#pragma unroll
              for (int c = 0; c < 16; ++c) {
                const int cc = 16 * g + c;
                const float tm = fmaxf(fmaxf(red[cc], red[N + cc]), fmaxf(red[2 * N + cc], red[3 * N + cc]));
                const float mn = fmaxf(m_run[cc], tm);
                v[c] *= (mn == -INFINITY) ? 1.f : fast_exp2(m_run[cc] - mn);
              }
              tmem_st16(addr, v);
            }
          }
        }
#pragma unroll
        for (int c = 0; c < N; ++c) {
          const float tm = fmaxf(fmaxf(red[c], red[N + c]), fmaxf(red[2 * N + c], red[3 * N + c]));
          const float mn = fmaxf(m_run[c], tm);
          l_run[c] *= (mn == -INFINITY) ? 1.f : fast_exp2(m_run[c] - mn);
          m_run[c] = mn;
        }
      }

      // pass 2: P = exp2(s - m) as bf16 into the K-major swizzled P^T tile
      if (nv > 0) {
#pragma unroll
        for (int g = 0; g < N / 16; ++g) {
          float v[16];
          tmem_ld16(tmem_s[sb] + lane_off + 16 * g, v);
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int cc = 16 * g + c;
            const float x = logit(v[c], cc);
            const float m_safe = m_run[cc] == -INFINITY ? 0.f : m_run[cc];
            const float pr = key_lane ? fast_exp2(x - m_safe) : 0.f;
            const __nv_bfloat16 pb = __float2bfloat16_rn(pr);
            l_run[cc] += pr;
            if (key_lane) {
              uint8_t* dst = p_tile + cc * 128 + ((((key >> 3) ^ (cc & 7)) << 4)) + (key & 7) * 2;
              *reinterpret_cast<__nv_bfloat16*>(dst) = pb;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.s_empty[sb]);

      // a partial last page may hold non-finite padding: zero its unused V rows
      if (!FP8 && nv > 0 && nv < kPage) {
        uint8_t* stage = smem + L::kv_off + s * kPageBytes;
        const int nrow = kPage - nv;
        const int tid = (q4 << 5) | lane;
        for (int idx = tid; idx < nrow * 8 * 8; idx += 128) {
          const int r = nv + idx / 64;
          const int rem = idx % 64;
          const int c = rem / 8, ch = rem % 8;
          *reinterpret_cast<uint4*>(stage + c * kChunkBytes + r * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.p_full);
      if (nv > 0) any_pv = true;

      if (j == je - 1) {
        // ------------------------------------------------ epilogue of the segment
        if (!mbar_wait(bars.p_empty, t & 1, abort_flag)) { ok = false; return false; }
        tc_fence_after();
        float* redl = red_base + ((t + 1) & 1) * 4 * N;
#pragma unroll
        for (int c = 0; c < N; ++c) {
          float x = l_run[c];
#pragma unroll
          for (int off = 16; off >= 1; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
          if (lane == 0) redl[q4 * N + c] = x;
        }
        if (!group_sync()) { ok = false; return false; }
        const int nsplit = p.num_splits[u + 1] - p.num_splits[u];
        const int split_idx = (u == part.u0 && jb == part.j0) ? part.first_split : p.num_splits[u];
        bool split = nsplit > 1;
        if (split && (split_idx < 0 || split_idx >= p.num_units + p.num_parts)) {
          // metadata from another plan: never write outside the workspace
          if (lane == 0 && q4 == 0) atomicOr(p.err, kErrInternal);
          split = false;
        }
#pragma unroll 1
        for (int jb4 = 0; jb4 < 4; ++jb4) {
          const int dim = 128 * jb4 + 32 * q4 + lane;
#pragma unroll
          for (int g = 0; g < N / 16; ++g) {
            float v[16];
            tmem_ld16(tmem_base + lane_off + jb4 * N + 16 * g, v);
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const int cc = 16 * g + c;
              const int r = row0 + cc;
              if (r >= R) continue;
              const float l = redl[cc] + redl[N + cc] + redl[2 * N + cc] + redl[3 * N + cc];
              const float val = (any_pv && l > 0.f) ? v[c] / l : 0.f;
              if (split) {
                p.ws_o[(static_cast<int64_t>(split_idx) * R + r) * kDv + dim] = val;
              } else {
                const __nv_bfloat16 ob = __float2bfloat16_rn(val);
                p.out[(static_cast<int64_t>(u) * R + r) * kDv + dim] = *reinterpret_cast<const uint16_t*>(&ob);
              }
            }
          }
        }
        {
          const int k = (q4 << 5) | lane;   // this thread writes the lse of tile row k
#pragma unroll
          for (int c = 0; c < N; ++c) {
            if (c != k) continue;
            const int r = row0 + c;
            if (r >= R) continue;
            const float l = redl[c] + redl[N + c] + redl[2 * N + c] + redl[3 * N + c];
            const float lse = (any_pv && l > 0.f) ? (m_run[c] + log2f(l)) * kLn2 : -INFINITY;
            if (split) {
              p.ws_lse[static_cast<int64_t>(split_idx) * R + r] = lse;
            } else {
              int b, tok, h;
              if (FP8) { b = ui.b; tok = ui.token; h = r; }
              else { b = ui.b; tok = r / p.h_q; h = r % p.h_q; }
              p.lse[(static_cast<int64_t>(b) * p.h_q + h) * p.s_q + tok] = lse;
            }
          }
        }
        tc_fence_before();
        if (!group_sync()) { ok = false; return false; }
      }
      ++t;
    }
    ++seg;
    return true;
  });
  if (!ok) raise_abort(abort_flag, p.err);
}

// ---------------------------------------------------------------------------
template <int N, bool FP8>
__global__ void __launch_bounds__(FP8 ? 320 : 192, 1)
    mla_decode_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmap_q,
                      const __grid_constant__ CUtensorMap tmap_kv) {
  using L = Smem<N>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L::bar_off);
  Bars bars;
  bars.kv_full = bar;
  bars.kv_empty = bar + kStages;
  bars.s_full = bar + 2 * kStages;
  bars.s_empty = bar + 2 * kStages + 2;
  bars.q_full = bar + 2 * kStages + 4;
  bars.q_empty = bar + 2 * kStages + 5;
  bars.p_full = bar + 2 * kStages + 6;
  bars.p_empty = bar + 2 * kStages + 7;
  bars.done = bar + 2 * kStages + 8;
  bars.sm_sync = bar + 2 * kStages + 9;
  StageInfo* info = reinterpret_cast<StageInfo*>(smem + L::info_off);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::misc_off);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::misc_off + 4);

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    if ((smem_u32(smem) & 1023u) != 0) {
      *abort_flag = 1;
      atomicOr(p.err, kErrInternal);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars.kv_full[s], FP8 ? 4 : 1);
      mbar_init(&bars.kv_empty[s], 1);
      info[s].nvalid = 0;
      for (int w = 0; w < 4; ++w) info[s].mask[w] = 0;
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.s_full[i], 1);
      mbar_init(&bars.s_empty[i], 4);
    }
    mbar_init(bars.q_full, 1);
    mbar_init(bars.q_empty, 1);
    mbar_init(bars.p_full, 4);
    mbar_init(bars.p_empty, 1);
    mbar_init(bars.done, 1);
    mbar_init(bars.sm_sync, 4);
    fence_barrier_init();
  }
  if (warp == kWarpLoad && lane == 0 && !FP8) {
    prefetch_tensormap(&tmap_q);
    prefetch_tensormap(&tmap_kv);
  }
  if (warp == kWarpMma) {
    tmem_alloc(tmem_slot, tmem_cols<N>());
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const Partition part = load_partition(p);

  if (!*abort_flag) {
    if (warp == kWarpLoad) {
      if (lane == 0) load_role<N, FP8>(p, part, &tmap_q, &tmap_kv, smem, bars, info, abort_flag);
    } else if (warp == kWarpMma) {
      if (lane == 0) mma_role<N, FP8>(p, part, smem, bars, info, tmem_base, abort_flag);
    } else if (warp < kWarpDequant0) {
      softmax_role<N, FP8>(p, part, smem, bars, info, tmem_base, abort_flag);
    } else if (FP8) {
      dequant_role<N>(p, part, smem, bars, info, abort_flag, warp - kWarpDequant0);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWarpMma) {
    __syncwarp();
    tmem_dealloc(tmem_base, tmem_cols<N>());
  }
}

template <int N, bool FP8>
cudaError_t launch_one(const DecodeParams& p, const CUtensorMap& tq, const CUtensorMap& tkv, int row_tiles,
                       cudaStream_t stream) {
  constexpr int smem = Smem<N>::total;
  // The shared-memory opt-in is per device; remember which devices have it.
  static unsigned long long configured = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(__atomic_load_n(&configured, __ATOMIC_ACQUIRE) & bit)) {
    e = cudaFuncSetAttribute(mla_decode_kernel<N, FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    __atomic_fetch_or(&configured, bit, __ATOMIC_RELEASE);
  }
  dim3 grid(p.num_parts, row_tiles);
  mla_decode_kernel<N, FP8><<<grid, FP8 ? 320 : 192, smem, stream>>>(p, tq, tkv);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeParams& p, const CUtensorMap& tmap_q, const CUtensorMap& tmap_kv,
                          int tile_rows, bool fp8, int row_tiles, cudaStream_t stream) {
  switch (tile_rows) {
    case 16: return fp8 ? launch_one<16, true>(p, tmap_q, tmap_kv, row_tiles, stream)
                        : launch_one<16, false>(p, tmap_q, tmap_kv, row_tiles, stream);
    case 32: return fp8 ? launch_one<32, true>(p, tmap_q, tmap_kv, row_tiles, stream)
                        : launch_one<32, false>(p, tmap_q, tmap_kv, row_tiles, stream);
    case 64: return fp8 ? launch_one<64, true>(p, tmap_q, tmap_kv, row_tiles, stream)
                        : launch_one<64, false>(p, tmap_q, tmap_kv, row_tiles, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace mla
