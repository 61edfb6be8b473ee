// MLA decode attention for units of more than 64 query rows on sm_100a: a
// cluster of two CTAs shares one 128-row tile, one CTA per half of the work.
//
// What it computes is the same as the single-CTA kernel (logits over the 576
// cache dims, softmax, output over the first 512 dims, log-sum-exp;
// "Was ist FlashMLA?" (topnet.top), section "3. MLA-Decodierung ausführen"),
// for the dense BF16 cache.
//
// Why two CTAs: with 128 query rows per MMA (the full-rate tcgen05 shape) the
// fp32 output tile O[128 x 512] fills all 512 TMEM columns of an SM, leaving
// no room for the logits.  So the work is split by function:
//  * the score CTA (cluster rank 0) keeps the query tile Q[128 x 576] in TMEM
//    (columns 128-415, two bf16 per column) and two logit buffers
//    S[128 x 64] (columns 0-127); it streams whole 576-dim pages, issues
//    S = Q K^T (36 x M128 N64 K16, A read from TMEM), runs the online softmax
//    (one thread per row) and publishes, per page, P = exp2(s - m) as bf16
//    in the swizzled K-major layout the tensor core reads, the factor alpha
//    by which each O row must be rescaled before P V is added, and on a
//    segment's last page 1 / l;
//  * the value CTA (rank 1) keeps O in TMEM, streams the first 512 dims of
//    the same pages, copies each published P tile into shared memory and
//    issues O += P V (2 x 4 x M128 N256 K16, V read MN-major), applies the
//    rescales and writes the output.
// P travels through a small ring in global memory (L2): the measured
// distributed-shared-memory rate between the two SMs (about 4 B per clock)
// is far below the 16 KB per page the hand-off needs, while L2 takes it in
// stride.  The two CTAs signal each other with mbarrier arrivals across the
// cluster (release / acquire at cluster scope).
//
// Every wait is bounded; a CTA that gives up raises MLA_DEVERR_TIMEOUT, sets
// its peer's abort flag, drains its own copies and MMAs and meets the peer at
// the final cluster barrier, so neither CTA's shared memory goes away while
// the other may still signal it.
#include <cuda_bf16.h>

#include "decode_common.cuh"
#include "mla_kernels.cuh"
#include "ptx_sm100.cuh"

namespace mla {
namespace {

using namespace dec;

constexpr int kRows = 128;                      // query rows of a tile = M of every MMA
constexpr int kStagesK = 3;                     // score CTA: whole pages
constexpr int kStagesV = 3;                     // value CTA: 512-dim part of pages
constexpr int kVPageBytes = kPage * kDv * 2;    // 65536
constexpr int kPTileBytes = kRows * 128;        // 16384: [128 rows x 64 keys] bf16
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemQCol = 128;             // score CTA: Q in columns 128..415

constexpr int kWarpLoad = 0, kWarpMma = 1, kWarpRow0 = 2;

// Global ring entry: P tile | alpha[128] | inv_l[128].
constexpr int kAlphaOff = kPTileBytes;
constexpr int kInvLOff = kAlphaOff + kRows * 4;

struct Smem {
  // score CTA: page ring
  static constexpr int k_off = 0;
  // value CTA: V ring and two P buffers (one ring entry each)
  static constexpr int v_off = 0;
  static constexpr int pb_off = v_off + kStagesV * kVPageBytes;
  static constexpr int bar_off = pb_off + 2 * kPairSlotBytes;
  static constexpr int n_bars = 32;
  static constexpr int info_off = bar_off + n_bars * 8;  // int nvalid per stage
  static constexpr int misc_off = info_off + 16;          // tmem base, abort flag
  static constexpr int total = misc_off + 16;
  static_assert(kStagesK * kPageBytes <= bar_off, "score ring overlaps the barriers");
  static_assert(pb_off % 1024 == 0 && kPairSlotBytes % 1024 == 0, "P tiles must stay 1024-B aligned");
  static_assert(total <= 232448, "shared memory budget");
};

// Barrier slots (each CTA uses its own subset).
enum : int {
  // score CTA
  kBarKFull = 0,                   // [kStagesK]
  kBarKEmpty = kBarKFull + kStagesK,
  kBarSFull = kBarKEmpty + kStagesK,   // [2]
  kBarSEmpty = kBarSFull + 2,          // [2]
  kBarQFull = kBarSEmpty + 2,
  kBarSlotFree = kBarQFull + 1,        // [kPairSlots], arrived by the value CTA
  kBarDoneA = kBarSlotFree + kPairSlots,
  // value CTA
  kBarVFull = 0,                   // [kStagesV]
  kBarVEmpty = kBarVFull + kStagesV,
  kBarPbFull = kBarVEmpty + kStagesV,  // [2]
  kBarPbEmpty = kBarPbFull + 2,        // [2]
  kBarOReady = kBarPbEmpty + 2,        // [2]
  kBarPvDone = kBarOReady + 2,
  kBarSlotReady = kBarPvDone + 1,      // [kPairSlots], arrived by the score CTA
  kBarDoneB = kBarSlotReady + kPairSlots,
};
static_assert(kBarDoneA < Smem::n_bars && kBarDoneB < Smem::n_bars, "barrier slots");

struct Ctx {
  DecodeParams p;
  Partition part;
  uint8_t* smem;
  uint64_t* bar;
  int* nvalid;                 // per stage
  volatile int* abort_flag;
  uint32_t peer_abort;         // cluster address of the peer's abort flag
  uint8_t* ring;               // this cluster's global ring
  int row0;                    // first row of the tile within a unit
};

__device__ __forceinline__ void pair_abort(const Ctx& c) {
  if (!*c.abort_flag) {
    *c.abort_flag = 1;
    atomicOr(c.p.err, kErrTimeout);
  }
  st_shared_cluster_u32(c.peer_abort, 1u);
}

// Valid keys of page j of unit u (0 when its block-table entry is bad).
__device__ __forceinline__ int page_keys(const DecodeParams& p, const UnitInfo& ui, int j, int* phys_out) {
  const int phys = page_of(p, ui.b, j);
  if (phys_out) *phys_out = phys;
  if (phys < 0 || phys >= p.num_blocks) return 0;
  return min(kPage, ui.L - kPage * j);
}

// ===========================================================================
// Score CTA
// ===========================================================================

// Warp 0, one lane: whole pages into the ring, L2 warmed a few pages ahead.
__device__ __forceinline__ void score_load(const Ctx& c, const CUtensorMap* tmap_kv) {
  const DecodeParams& p = c.p;
  const uint64_t pol = l2_policy_evict_first();
  const uint32_t q_bytes = static_cast<uint32_t>(min(kRows, p.rows_per_unit - c.row0)) * kDqk * 2;
  int t = 0;
  int last_t[kStagesK];
#pragma unroll
  for (int s = 0; s < kStagesK; ++s) last_t[s] = -1;
  bool ok = true;
  int ring[kPrefetchPages];
  for_each_segment(p, c.part, [&](int u, int jb, int je) -> bool {
    if (u + 1 <= c.part.u1 && u + 1 < p.num_units) {
      int jb2, je2;
      if (segment_bounds(p, c.part, u + 1, jb2, je2))
        bulk_prefetch_l2(p.q + q_tile_offset(p, unit_info(p, u + 1), c.row0), q_bytes);
    }
    const UnitInfo ui = unit_info(p, u);
    const int jn = min(je, jb + kPrefetchPages);
    for (int j = jb; j < jn; ++j) ring[j % kPrefetchPages] = page_of(p, ui.b, j);
    for (int j = jb; j < jn; ++j) {
      const int phys = ring[j % kPrefetchPages];
      if (phys >= 0 && phys < p.num_blocks) {
#pragma unroll 1
        for (int ch = 0; ch < kChunks; ++ch) tma_prefetch_3d(tmap_kv, 64 * ch, 0, phys);
      }
    }
    for (int j = jb; j < je; ++j) {
      const int s = t % kStagesK;
      if (!mbar_wait(&c.bar[kBarKEmpty + s], ((t / kStagesK) & 1) ^ 1, c.abort_flag)) { ok = false; return false; }
      const int phys = ring[j % kPrefetchPages];
      int nv = min(kPage, ui.L - kPage * j);
      if (phys < 0 || phys >= p.num_blocks) {
        atomicOr(p.err, kErrBlockTable);
        nv = 0;
      }
      c.nvalid[s] = nv;
      if (nv > 0) {
        mbar_arrive_expect_tx(&c.bar[kBarKFull + s], kPageBytes);
        uint8_t* dst = c.smem + Smem::k_off + s * kPageBytes;
#pragma unroll 1
        for (int ch = 0; ch < kChunks; ++ch)
          tma_load_3d(dst + ch * kChunkBytes, tmap_kv, &c.bar[kBarKFull + s], 64 * ch, 0, phys, pol);
        last_t[s] = t;
      } else {
        mbar_arrive(&c.bar[kBarKFull + s]);
      }
      if (j + kPrefetchPages < je) {
        const int jj = j + kPrefetchPages;
        const int ph = page_of(p, ui.b, jj);
        ring[jj % kPrefetchPages] = ph;
        if (ph >= 0 && ph < p.num_blocks) {
#pragma unroll 1
          for (int ch = 0; ch < kChunks; ++ch) tma_prefetch_3d(tmap_kv, 64 * ch, 0, ph);
        }
      }
      ++t;
    }
    return true;
  });
  if (!ok) {
    pair_abort(c);
    const uint64_t t0 = globaltimer_ns();
    for (int s = 0; s < kStagesK; ++s) {
      if (last_t[s] < 0) continue;
      while (!mbar_try_wait(&c.bar[kBarKFull + s], (last_t[s] / kStagesK) & 1) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
      }
    }
  }
}

// Warp 1 (whole warp, one elected lane issues): S = Q K^T per page.
__device__ __forceinline__ void score_mma(const Ctx& c, uint32_t tmem_base) {
  const DecodeParams& p = c.p;
  constexpr uint32_t idesc = idesc_bf16_f32(kRows, kPage, false, false);
  const uint32_t tmem_q = tmem_base + kTmemQCol;
  uint64_t k_desc[kStagesK];
#pragma unroll
  for (int s = 0; s < kStagesK; ++s) k_desc[s] = sdesc_sw128(smem_u32(c.smem + Smem::k_off + s * kPageBytes), 16, 1024);
  const int lane = threadIdx.x & 31;
  auto ready = [&](uint64_t* b, uint32_t parity) -> bool {
    bool r = lane == 0 ? mbar_wait(b, parity, c.abort_flag) : false;
    return __shfl_sync(0xffffffffu, r ? 1 : 0, 0) != 0;
  };
  bool ok = true;
  Cursor q = cursor_begin(p, c.part);
  while (q.valid) {
    const int s = q.t % kStagesK;
    const int sb = q.t & 1;
    const bool first = (q.j == (q.u == c.part.u0 ? c.part.j0 : 0));
    if (!ready(&c.bar[kBarKFull + s], (q.t / kStagesK) & 1)) { ok = false; break; }
    if (first && !ready(&c.bar[kBarQFull], q.seg & 1)) { ok = false; break; }
    if (!ready(&c.bar[kBarSEmpty + sb], ((q.t >> 1) & 1) ^ 1)) { ok = false; break; }
    tc_fence_after();
    if (c.nvalid[s] > 0) {
      const uint64_t kd = k_desc[s];
      const uint32_t d = tmem_base + sb * kPage;
#pragma unroll
      for (int ch = 0; ch < kChunks; ++ch) {
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma_bf16_ts_elect(d, tmem_q + 32 * ch + 8 * k, kd + ((ch * kChunkBytes + k * 32) >> 4), idesc,
                             (ch | k) != 0 ? 1u : 0u);
      }
    }
    umma_commit_elect(&c.bar[kBarSFull + sb]);
    umma_commit_elect(&c.bar[kBarKEmpty + s]);
    cursor_next(p, c.part, q);
  }
  if (!ok && lane == 0) pair_abort(c);
  umma_commit_elect(&c.bar[kBarDoneA]);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(&c.bar[kBarDoneA], 0) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
  }
  __syncwarp();
}

// Query tile row r of unit `ui` into TMEM lane r (columns 128..415).
__device__ __forceinline__ void score_write_q(const Ctx& c, const UnitInfo& ui, uint32_t tq_lane, int r) {
  const DecodeParams& p = c.p;
  const bool valid = c.row0 + r < p.rows_per_unit;
  const uint4* src = reinterpret_cast<const uint4*>(p.q + q_tile_offset(p, ui, c.row0) + static_cast<int64_t>(r) * kDqk);
#pragma unroll 1
  for (int ch = 0; ch < kChunks; ++ch) {
    uint4 buf[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) buf[i] = valid ? __ldg(src + 8 * ch + i) : make_uint4(0, 0, 0, 0);
    uint32_t v[32];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[4 * i] = buf[i].x; v[4 * i + 1] = buf[i].y; v[4 * i + 2] = buf[i].z; v[4 * i + 3] = buf[i].w;
    }
    tmem_st_32x32b_x32u(tq_lane + 32 * ch, v);
  }
}

// Warps 2-5: query tiles, online softmax (one thread per row), publication of
// P / alpha / 1/l, and the log-sum-exp output.
__device__ __forceinline__ void score_softmax(const Ctx& c, uint32_t tmem_base) {
  const DecodeParams& p = c.p;
  const int lane = threadIdx.x & 31;
  const int q4 = (threadIdx.x >> 5) & 3;           // TMEM lane quadrant of this warp
  const int r = 32 * q4 + lane;                    // tile row = TMEM lane
  const int R = p.rows_per_unit;
  const int grow = c.row0 + r;
  const bool row_valid = grow < R;
  const float scale_log2 = p.scale_log2;
  const int h_q = p.h_q, s_q = p.s_q;
  const int tok = grow / h_q;
  const bool causal = p.causal != 0;
  const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(32 * q4) << 16);

  auto stage_q = [&](int u_from) {
    for (int u = u_from; u <= c.part.u1 && u < p.num_units; ++u) {
      int jb, je;
      if (segment_bounds(p, c.part, u, jb, je)) {
        score_write_q(c, unit_info(p, u), lane_base + kTmemQCol, r);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&c.bar[kBarQFull]);
        return;
      }
    }
  };
  stage_q(c.part.u0);

  const uint32_t peer = cluster_ctarank() ^ 1u;
  int t = 0;
  bool ok = true;
  for_each_segment(p, c.part, [&](int u, int jb, int je) -> bool {
    const UnitInfo ui = unit_info(p, u);
    if (lane == 0 && q4 == 0 && p.seqlens[ui.b] < 0) atomicOr(p.err, kErrSeqlen);
    float m_run = -INFINITY, l_run = 0.f;
    const int lim = ui.L - s_q + tok + 1;          // causal: keys < lim are visible
    for (int j = jb; j < je; ++j) {
      const int sb = t & 1;
      const int nv = page_keys(p, ui, j, nullptr);
      if (!mbar_wait(&c.bar[kBarSFull + sb], (t >> 1) & 1, c.abort_flag)) { ok = false; return false; }
      tc_fence_after();
      float x[64];
      if (nv > 0) tmem_ld_32x32b_x64(lane_base + sb * kPage, x);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.bar[kBarSEmpty + sb]);
      const bool last = (j == je - 1);

      float tmax = -INFINITY;
      if (nv > 0) {
        int nk = nv;
        if (causal) nk = min(nk, max(lim - kPage * j, 0));
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          x[i] = i < nk ? x[i] * scale_log2 : -INFINITY;
          tmax = fmaxf(tmax, x[i]);
        }
      }
      const bool need = tmax > m_run + kRescaleThreshold;
      const float m_new = need ? fmaxf(m_run, tmax) : m_run;
      const float alpha = (m_new == m_run) ? 1.f : fast_exp2(m_run - m_new);   // m_run = -inf -> 0
      l_run *= alpha;
      m_run = m_new;
      const float m_safe = m_run == -INFINITY ? 0.f : m_run;
      uint32_t pk[32];
      if (nv > 0) {
        float lsum = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float a = fast_exp2(x[2 * i] - m_safe);
          const float b = fast_exp2(x[2 * i + 1] - m_safe);
          lsum += a + b;
          pk[i] = pack_bf16x2(a, b);
        }
        l_run += lsum;
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) pk[i] = 0u;
      }

      // publish into ring slot t % kPairSlots once the value CTA has copied
      // out what it held before
      const int slot = t % kPairSlots;
      if (!mbar_wait_cluster(&c.bar[kBarSlotFree + slot], ((t / kPairSlots) & 1) ^ 1, c.abort_flag)) {
        ok = false;
        return false;
      }
      uint8_t* e = c.ring + static_cast<size_t>(slot) * kPairSlotBytes;
      uint4* prow = reinterpret_cast<uint4*>(e + r * 128);
#pragma unroll
      for (int ch = 0; ch < 8; ++ch)
        prow[ch ^ (r & 7)] = make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
      reinterpret_cast<float*>(e + kAlphaOff)[r] = alpha;
      float lse = -INFINITY;
      if (last) {
        const bool has = l_run > 0.f;
        reinterpret_cast<float*>(e + kInvLOff)[r] = has ? 1.f / l_run : 0.f;
        lse = has ? (m_run + log2f(l_run)) * kLn2 : -INFINITY;
      }
      fence_proxy_async_global();
      __syncwarp();
      if (lane == 0)
        mbar_arrive_remote(mapa_shared(smem_u32(&c.bar[kBarSlotReady + slot]), peer));

      if (last && row_valid) {
        const int nsplit = p.num_splits[u + 1] - p.num_splits[u];
        const int split_idx = (u == c.part.u0 && jb == c.part.j0) ? c.part.first_split : p.num_splits[u];
        const bool split = nsplit > 1 && split_idx >= 0 && split_idx < p.num_units + p.num_parts;
        if (nsplit > 1 && !split) atomicOr(p.err, kErrInternal);
        else if (split) p.ws_lse[static_cast<int64_t>(split_idx) * R + grow] = lse;
        else p.lse[(static_cast<int64_t>(ui.b) * h_q + grow % h_q) * s_q + tok] = lse;
      }
      // every QK of this segment has been consumed: the next query tile may
      // take the TMEM columns of this one
      if (last) stage_q(u + 1);
      ++t;
    }
    return true;
  });
  if (!ok) pair_abort(c);
}

// ===========================================================================
// Value CTA
// ===========================================================================

// Warp 0, one lane: the 512-dim part of every page into the V ring.
__device__ __forceinline__ void value_load(const Ctx& c, const CUtensorMap* tmap_kv) {
  const DecodeParams& p = c.p;
  const uint64_t pol = l2_policy_evict_first();
  int last_t[kStagesV];
#pragma unroll
  for (int s = 0; s < kStagesV; ++s) last_t[s] = -1;
  bool ok = true;
  Cursor v = cursor_begin(p, c.part);
  while (v.valid) {
    const int s = v.t % kStagesV;
    if (!mbar_wait(&c.bar[kBarVEmpty + s], ((v.t / kStagesV) & 1) ^ 1, c.abort_flag)) { ok = false; break; }
    int phys;
    const int nv = page_keys(p, unit_info(p, v.u), v.j, &phys);
    c.nvalid[s] = nv;
    if (nv > 0) {
      mbar_arrive_expect_tx(&c.bar[kBarVFull + s], kVPageBytes);
      uint8_t* dst = c.smem + Smem::v_off + s * kVPageBytes;
#pragma unroll 1
      for (int ch = 0; ch < kDv / 64; ++ch)
        tma_load_3d(dst + ch * kChunkBytes, tmap_kv, &c.bar[kBarVFull + s], 64 * ch, 0, phys, pol);
      last_t[s] = v.t;
    } else {
      mbar_arrive(&c.bar[kBarVFull + s]);
    }
    cursor_next(p, c.part, v);
  }
  if (!ok) {
    pair_abort(c);
    const uint64_t t0 = globaltimer_ns();
    for (int s = 0; s < kStagesV; ++s) {
      if (last_t[s] < 0) continue;
      while (!mbar_try_wait(&c.bar[kBarVFull + s], (last_t[s] / kStagesV) & 1) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
      }
    }
  }
}

// Warp 1 (whole warp, one elected lane issues): O += P V per page.
__device__ __forceinline__ void value_mma(const Ctx& c, uint32_t tmem_base) {
  const DecodeParams& p = c.p;
  constexpr uint32_t idesc = idesc_bf16_f32(kRows, 256, false, true);
  uint64_t v_desc[kStagesV], p_desc[2];
#pragma unroll
  for (int s = 0; s < kStagesV; ++s) v_desc[s] = sdesc_sw128(smem_u32(c.smem + Smem::v_off + s * kVPageBytes), kChunkBytes, 1024);
#pragma unroll
  for (int b = 0; b < 2; ++b) p_desc[b] = sdesc_sw128(smem_u32(c.smem + Smem::pb_off + b * kPairSlotBytes), 16, 1024);
  const int lane = threadIdx.x & 31;
  auto ready = [&](uint64_t* b, uint32_t parity) -> bool {
    bool r = lane == 0 ? mbar_wait(b, parity, c.abort_flag) : false;
    return __shfl_sync(0xffffffffu, r ? 1 : 0, 0) != 0;
  };
  bool ok = true;
  int o_seg = -1;
  Cursor v = cursor_begin(p, c.part);
  while (v.valid) {
    const int s = v.t % kStagesV;
    const int b = v.t & 1;
    if (!ready(&c.bar[kBarVFull + s], (v.t / kStagesV) & 1)) { ok = false; break; }
    if (!ready(&c.bar[kBarPbFull + b], (v.t >> 1) & 1)) { ok = false; break; }
    if (!ready(&c.bar[kBarOReady + b], (v.t >> 1) & 1)) { ok = false; break; }
    tc_fence_after();
    if (c.nvalid[s] > 0) {
      const bool acc0 = (o_seg == v.seg);
      const uint64_t vd = v_desc[s];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma_bf16_elect(tmem_base + h * 256, p_desc[b] + ((k * 32) >> 4),
                          vd + ((4 * h * kChunkBytes + k * 2048) >> 4), idesc, (acc0 || k > 0) ? 1u : 0u);
      }
      o_seg = v.seg;
    }
    umma_commit_elect(&c.bar[kBarVEmpty + s]);
    umma_commit_elect(&c.bar[kBarPbEmpty + b]);
    umma_commit_elect(&c.bar[kBarPvDone]);
    cursor_next(p, c.part, v);
  }
  if (!ok && lane == 0) pair_abort(c);
  umma_commit_elect(&c.bar[kBarDoneB]);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(&c.bar[kBarDoneB], 0) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
  }
  __syncwarp();
}

// Warps 2-5: copy each published P tile in (warp 2, lane 0), apply the O
// rescales, zero the padding rows of a partial page's V, and write the
// output of every segment (one thread per row).
__device__ __forceinline__ void value_rows(const Ctx& c, uint32_t tmem_base) {
  const DecodeParams& p = c.p;
  const int lane = threadIdx.x & 31;
  const int q4 = (threadIdx.x >> 5) & 3;
  const int r = 32 * q4 + lane;
  const int R = p.rows_per_unit;
  const int grow = c.row0 + r;
  const bool row_valid = grow < R;
  const bool issuer = (threadIdx.x >> 5) == kWarpRow0 && lane == 0;
  const uint32_t o_lane = tmem_base + (static_cast<uint32_t>(32 * q4) << 16);
  const uint32_t peer = cluster_ctarank() ^ 1u;
  int last_copy = -1;
  bool ok = true;

  // Copy ring entry `tc` into P buffer tc & 1 (issuer only).
  auto issue_copy = [&](int tc) -> bool {
    const int b = tc & 1;
    const int slot = tc % kPairSlots;
    if (!mbar_wait(&c.bar[kBarPbEmpty + b], ((tc >> 1) & 1) ^ 1, c.abort_flag)) return false;
    if (!mbar_wait_cluster(&c.bar[kBarSlotReady + slot], (tc / kPairSlots) & 1, c.abort_flag)) return false;
    fence_proxy_async_global();
    mbar_arrive_expect_tx(&c.bar[kBarPbFull + b], kPairSlotBytes);
    bulk_load_g2s(c.smem + Smem::pb_off + b * kPairSlotBytes, c.ring + static_cast<size_t>(slot) * kPairSlotBytes,
                  kPairSlotBytes, &c.bar[kBarPbFull + b]);
    last_copy = tc;
    return true;
  };

  Cursor v = cursor_begin(p, c.part);
  if (issuer && v.valid && !issue_copy(0)) ok = false;
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;

  UnitInfo ui{};
  int seg = -1, seg_jb = 0;
  bool any_pv = false;
  while (ok && v.valid) {
    const int t = v.t;
    const int u = v.u;
    if (v.seg != seg) {
      seg = v.seg;
      seg_jb = v.j;
      ui = unit_info(p, u);
      any_pv = false;
    }
    const int b = t & 1;
    const int s = t % kStagesV;
    const int nv = page_keys(p, ui, v.j, nullptr);
    const bool last = (v.j == v.je - 1);
    Cursor nx = v;
    cursor_next(p, c.part, nx);

    if (!mbar_wait(&c.bar[kBarPbFull + b], (t >> 1) & 1, c.abort_flag)) { ok = false; break; }
    // the ring entry now sits in shared memory: hand it back
    if (issuer) mbar_arrive_remote(mapa_shared(smem_u32(&c.bar[kBarSlotFree + t % kPairSlots]), peer));
    const uint8_t* pb = c.smem + Smem::pb_off + b * kPairSlotBytes;
    const float alpha = reinterpret_cast<const float*>(pb + kAlphaOff)[r];
    const float inv_l = last ? reinterpret_cast<const float*>(pb + kInvLOff)[r] : 0.f;
    if (__any_sync(0xffffffffu, any_pv && alpha != 1.f)) {
      // O must hold every earlier PV of the segment before it is rescaled
      // (PV(t - 2) has completed: the copy of this page waited for it)
      if (!mbar_wait(&c.bar[kBarPvDone], (t - 1) & 1, c.abort_flag)) { ok = false; break; }
      tc_fence_after();
#pragma unroll 1
      for (int c0 = 0; c0 < kDv; c0 += 32) {
        float o[32];
        tmem_ld_32x32b_x32(o_lane + c0, o);
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] *= alpha;
        tmem_st_32x32b_x32(o_lane + c0, o);
      }
    }
    if (nv > 0 && nv < kPage) {
      // a partial page may hold non-finite padding: zero its unused V rows
      if (!mbar_wait(&c.bar[kBarVFull + s], (t / kStagesV) & 1, c.abort_flag)) { ok = false; break; }
      uint8_t* stage = c.smem + Smem::v_off + s * kVPageBytes;
      const int tid = (q4 << 5) | lane;
      for (int idx = tid; idx < (kPage - nv) * 8 * 8; idx += 128) {
        const int rr = nv + idx / 64;
        const int rem = idx % 64;
        st_shared_v4(smem_u32(stage + (rem / 8) * kChunkBytes + rr * 128 + (rem % 8) * 16), make_uint4(0, 0, 0, 0));
      }
      fence_proxy_async_smem();
    }
    if (nv > 0) any_pv = true;
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&c.bar[kBarOReady + b]);

    if (last) {
      // ------------------------------------------------ epilogue of the segment
      // (the next segment's first PV overwrites O; it waits for this warp's
      // next o_ready arrival, which comes after these reads)
      // pv_done completes once per page and only parities are observable: at
      // this point PV(t - 1) may still be running, so wait for it first (else
      // the parity of PV(t) would alias the phase before PV(t - 1))
      if (t > 0 && !mbar_wait(&c.bar[kBarPvDone], (t - 1) & 1, c.abort_flag)) { ok = false; break; }
      if (!mbar_wait(&c.bar[kBarPvDone], t & 1, c.abort_flag)) { ok = false; break; }
      tc_fence_after();
      const bool has = any_pv && inv_l > 0.f;
      const float inv = has ? inv_l : 0.f;
      const int nsplit = p.num_splits[u + 1] - p.num_splits[u];
      const int split_idx = (u == c.part.u0 && seg_jb == c.part.j0) ? c.part.first_split : p.num_splits[u];
      const bool split = nsplit > 1 && split_idx >= 0 && split_idx < p.num_units + p.num_parts;
      const bool skip = nsplit > 1 && !split;      // plan from another call: reported by the score CTA
#pragma unroll 1
      for (int c0 = 0; c0 < kDv; c0 += 32) {
        float o[32];
        tmem_ld_32x32b_x32(o_lane + c0, o);
        if (!row_valid || skip) continue;
        if (!has) {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0.f;
        }
        if (split) {
          float4* dst = reinterpret_cast<float4*>(p.ws_o + (static_cast<int64_t>(split_idx) * R + grow) * kDv + c0);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(o[4 * i] * inv, o[4 * i + 1] * inv, o[4 * i + 2] * inv, o[4 * i + 3] * inv);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(p.out + (static_cast<int64_t>(u) * R + grow) * kDv + c0);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_uint4(pack_bf16x2(o[8 * i] * inv, o[8 * i + 1] * inv),
                                pack_bf16x2(o[8 * i + 2] * inv, o[8 * i + 3] * inv),
                                pack_bf16x2(o[8 * i + 4] * inv, o[8 * i + 5] * inv),
                                pack_bf16x2(o[8 * i + 6] * inv, o[8 * i + 7] * inv));
        }
      }
      tc_fence_before();
    }
    if (nx.valid) {
      if (issuer && !issue_copy(t + 1)) ok = false;
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    }
    v = nx;
  }
  if (!ok) {
    pair_abort(c);
    if (issuer && last_copy >= 0) {
      // drain this lane's own bulk copy
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(&c.bar[kBarPbFull + (last_copy & 1)], (last_copy >> 1) & 1) &&
             globaltimer_ns() - t0 < kWaitTimeoutNs) {
      }
    }
  }
}

// ===========================================================================

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    mla_decode_pair_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmap_kv) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool score = rank == 0;

  Ctx c;
  c.p = p;
  c.smem = smem;
  c.bar = reinterpret_cast<uint64_t*>(smem + Smem::bar_off);
  c.nvalid = reinterpret_cast<int*>(smem + Smem::info_off);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Smem::misc_off);
  int* abort_word = reinterpret_cast<int*>(smem + Smem::misc_off + 4);
  c.abort_flag = abort_word;
  c.peer_abort = mapa_shared(smem_u32(abort_word), rank ^ 1u);
  c.row0 = static_cast<int>(blockIdx.y) * kRows;
  const int part_idx = static_cast<int>(blockIdx.x) >> 1;
  const int cluster_id = static_cast<int>(blockIdx.y) * p.num_parts + part_idx;
  c.ring = p.ws_pring + static_cast<size_t>(cluster_id) * kPairSlots * kPairSlotBytes;

  const bool misaligned = (smem_u32(smem) & 1023u) != 0;
  if (threadIdx.x == 0) {
    *abort_word = misaligned ? 1 : 0;
    if (score) {
      for (int s = 0; s < kStagesK; ++s) {
        mbar_init(&c.bar[kBarKFull + s], 1);
        mbar_init(&c.bar[kBarKEmpty + s], 1);
        c.nvalid[s] = 0;
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(&c.bar[kBarSFull + i], 1);
        mbar_init(&c.bar[kBarSEmpty + i], 4);
      }
      mbar_init(&c.bar[kBarQFull], 4);
      for (int i = 0; i < kPairSlots; ++i) mbar_init(&c.bar[kBarSlotFree + i], 1);
      mbar_init(&c.bar[kBarDoneA], 1);
    } else {
      for (int s = 0; s < kStagesV; ++s) {
        mbar_init(&c.bar[kBarVFull + s], 1);
        mbar_init(&c.bar[kBarVEmpty + s], 1);
        c.nvalid[s] = 0;
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(&c.bar[kBarPbFull + i], 1);
        mbar_init(&c.bar[kBarPbEmpty + i], 1);
        mbar_init(&c.bar[kBarOReady + i], 4);
      }
      mbar_init(&c.bar[kBarPvDone], 1);
      for (int i = 0; i < kPairSlots; ++i) mbar_init(&c.bar[kBarSlotReady + i], 4);
      mbar_init(&c.bar[kBarDoneB], 1);
    }
    fence_barrier_init();
  }
  if (warp == kWarpLoad && lane == 0) prefetch_tensormap(&tmap_kv);
  if (warp == kWarpMma) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  cluster_sync_all();          // both CTAs' barriers exist before any remote arrival
  tc_fence_after();
  grid_dependency_wait();
  grid_launch_dependents();
  if (misaligned && threadIdx.x == 0) atomicOr(p.err, kErrInternal);
  const uint32_t tmem_base = *tmem_slot;
  c.part = load_partition(p, part_idx);

  if (!*c.abort_flag) {
    if (score) {
      if (warp == kWarpLoad) {
        if (lane == 0) score_load(c, &tmap_kv);
      } else if (warp == kWarpMma) {
        score_mma(c, tmem_base);
      } else {
        score_softmax(c, tmem_base);
      }
    } else {
      if (warp == kWarpLoad) {
        if (lane == 0) value_load(c, &tmap_kv);
      } else if (warp == kWarpMma) {
        value_mma(c, tmem_base);
      } else {
        value_rows(c, tmem_base);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();          // neither CTA leaves while the other may still signal it
  tc_fence_after();
  if (warp == kWarpMma) {
    __syncwarp();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

int pair_cluster_capacity() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < 64 && cached[dev] > 0) return cached[dev];
  if (cudaFuncSetAttribute(mla_decode_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Smem::total) !=
      cudaSuccess)
    return 0;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (sms / 2), 1, 1);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = Smem::total;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, mla_decode_pair_kernel, &cfg) != cudaSuccess || n <= 0) {
    (void)cudaGetLastError();
    n = sms / 2;
  }
  if (dev >= 0 && dev < 64) cached[dev] = n;
  return n;
}

cudaError_t launch_decode_pair(const DecodeParams& p, const CUtensorMap& tmap_kv, int row_tiles, cudaStream_t stream) {
  static unsigned long long configured = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(__atomic_load_n(&configured, __ATOMIC_ACQUIRE) & bit)) {
    e = cudaFuncSetAttribute(mla_decode_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Smem::total);
    if (e != cudaSuccess) return e;
    __atomic_fetch_or(&configured, bit, __ATOMIC_RELEASE);
  }
  return launch_dependent(mla_decode_pair_kernel, dim3(2 * p.num_parts, row_tiles), dim3(kThreads), Smem::total,
                          stream, p, tmap_kv);
}

}  // namespace mla
