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
//    the same pages, reads each published P tile into shared memory and
//    issues O += P V (2 x 4 x M128 N256 K16, V read MN-major), applies the
//    rescales and writes the output.
// P travels through a small ring in global memory (L2): the measured
// distributed-shared-memory rate between the two SMs (about 4 B per clock)
// is far below the 16 KB per page the hand-off needs, while L2 takes it in
// stride.  Writes and reads of the ring are plain (generic-proxy) coalesced
// stores and loads.  The ring holds two groups of kPairGroup pages; the
// score CTA releases a group once its last page is stored (every softmax
// thread fences its own stores at cluster scope, then one mbarrier arrival
// per warp across the cluster), because such a fence costs about a
// microsecond however little is pending.  The value CTA's row warps hand a
// group back through a signal warp of their own (their loads have completed
// when they signal, so the cluster-scope arrival stays off their path).
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

#ifdef MLA_TRACE
// Opt-in hand-off trace (built only with -DMLA_TRACE): %globaltimer stamps of
// the events of every page of the first kPairTraceCtas / 2 clusters of row
// tile 0, indexed [CTA][event][page].
constexpr int kPairTraceCtas = 4, kPairTraceEvents = 16, kPairTracePages = 256;
__device__ unsigned long long g_pair_trace[kPairTraceCtas][kPairTraceEvents][kPairTracePages];
#define PAIR_TRACE(ev, idx)                                                                     \
  do {                                                                                          \
    if (blockIdx.x < kPairTraceCtas && blockIdx.y == 0 && (idx) >= 0 && (idx) < kPairTracePages) \
      g_pair_trace[blockIdx.x][ev][idx] = globaltimer_ns();                                     \
  } while (0)
#else
#define PAIR_TRACE(ev, idx) \
  do {                      \
  } while (0)
#endif

namespace {

using namespace dec;

constexpr int kRows = 128;                      // query rows of a tile = M of every MMA
constexpr int kStagesK = 3;                     // score CTA: whole pages
constexpr int kStagesV = 3;                     // value CTA: 512-dim part of pages
constexpr int kVPageBytes = kPage * kDv * 2;    // 65536
constexpr int kPTileBytes = kRows * 128;        // 16384: [128 rows x 64 keys] bf16
constexpr int kThreads = 224;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemQCol = 128;             // score CTA: Q in columns 128..415

constexpr int kWarpLoad = 0, kWarpMma = 1, kWarpSignal = 6;   // warp 6: value CTA only

// Global ring entry: P tile | alpha[128] | inv_l[128].
constexpr int kAlphaOff = kPTileBytes;
constexpr int kInvLOff = kAlphaOff + kRows * 4;

struct Smem {
  // score CTA: page ring, then per-warp staging (16 rows x 128 B) that turns
  // a warp's row-per-thread P into 512-B coalesced stores
  static constexpr int k_off = 0;
  static constexpr int stage_off = k_off + kStagesK * kPageBytes;
  // value CTA: V ring and two P buffers (one ring entry each)
  static constexpr int v_off = 0;
  static constexpr int pb_off = v_off + kStagesV * kVPageBytes;
  static constexpr int bar_off = pb_off + 2 * kPairSlotBytes;
  static constexpr int n_bars = 32;
  static constexpr int info_off = bar_off + n_bars * 8;  // int nvalid per stage
  static constexpr int misc_off = info_off + 16;          // tmem base, abort flag
  static constexpr int total = misc_off + 16;
  static_assert(stage_off + 4 * 16 * 128 <= bar_off, "score ring and staging overlap the barriers");
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
  kBarSlotFree = kBarQFull + 1,        // [2] per group of the ring, arrived by the value CTA's signal warp
  kBarDoneA = kBarSlotFree + 2,
  // value CTA
  kBarVFull = 0,                   // [kStagesV]
  kBarVEmpty = kBarVFull + kStagesV,
  kBarPbEmpty = kBarVEmpty + kStagesV, // [2] P buffer b free = PV of the last page using it done
  kBarOReady = kBarPbEmpty + 2,        // [2]
  kBarSlotReady = kBarOReady + 2,      // [2] per group, arrived by the score CTA's 4 softmax warps
  kBarSlotRead = kBarSlotReady + 2,    // [2] per group, the 4 row warps have read it
  kBarDoneB = kBarSlotRead + 2,
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

// Warp 0, one lane: whole pages into the ring (block-table entries read ahead).
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
    // (no L2 prefetch of pages here: with both CTAs of the pair streaming
    // the same pages it measured slower)
    const int jn = min(je, jb + kPrefetchPages);
    for (int j = jb; j < jn; ++j) ring[j % kPrefetchPages] = page_of(p, ui.b, j);
    for (int j = jb; j < je; ++j) {
      const int s = t % kStagesK;
      if (!mbar_wait(&c.bar[kBarKEmpty + s], ((t / kStagesK) & 1) ^ 1, c.abort_flag)) { ok = false; return false; }
      PAIR_TRACE(0, t);
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
        ring[jj % kPrefetchPages] = page_of(p, ui.b, jj);   // block-table entries read ahead
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
    if (lane == 0) PAIR_TRACE(1, q.t);
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
//
// Publication of page t: the warp's 32 P rows go out through a 2 KB staging
// tile as 512-B coalesced stores; the release to the value CTA (lane 0, after
// __syncwarp, at cluster scope) is issued one page later, once the stores
// have long been acknowledged, so it never stalls the softmax.
__device__ __forceinline__ void score_softmax(const Ctx& c, uint32_t tmem_base) {
  const DecodeParams& p = c.p;
  const int lane = threadIdx.x & 31;
  const int q4 = (threadIdx.x >> 5) & 3;           // TMEM lane quadrant of this warp
  const int r = 32 * q4 + lane;                    // tile row = TMEM lane
  const int R = p.rows_per_unit;
  const int grow = c.row0 + r;
  const bool row_valid = grow < R;
  const float scale_log2 = p.scale_log2;           // > 0 (checked on the host)
  const int h_q = p.h_q, s_q = p.s_q;
  const int tok = grow / h_q;
  const bool causal = p.causal != 0;
  const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(32 * q4) << 16);
  const uint32_t stage = smem_u32(c.smem + Smem::stage_off + q4 * 2048);

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
  // Release the group of ring entries that page t closes to the value CTA.
  // Every thread fences its own stores at cluster scope (a single lane's
  // release does not cover the other lanes' global stores); the fence costs
  // about a microsecond whatever is pending, so it is paid once per group.
  auto release = [&](int t) {
    if (lane == 0 && q4 == 0) PAIR_TRACE(7, t);
    asm volatile("fence.acq_rel.cluster;" ::: "memory");
    __syncwarp();
    if (lane == 0) mbar_arrive_remote(mapa_shared(smem_u32(&c.bar[kBarSlotReady + (t / kPairGroup) % 2]), peer));
    if (lane == 0 && q4 == 0) PAIR_TRACE(8, t);
  };
  int t = 0;
  bool ok = true;
  for_each_segment(p, c.part, [&](int u, int jb, int je) -> bool {
    const UnitInfo ui = unit_info(p, u);
    if (lane == 0 && q4 == 0 && p.seqlens[ui.b] < 0) atomicOr(p.err, kErrSeqlen);
    float m_run = -INFINITY, l_run = 0.f;
    const int lim = ui.L - s_q + tok + 1;          // causal: keys < lim are visible
    int phys_next = page_of(p, ui.b, jb);          // block-table entries are read one page ahead
    for (int j = jb; j < je; ++j) {
      const int sb = t & 1;
      const int phys = phys_next;
      if (j + 1 < je) phys_next = page_of(p, ui.b, j + 1);
      const int nv = (phys >= 0 && phys < p.num_blocks) ? min(kPage, ui.L - kPage * j) : 0;
      if (!mbar_wait(&c.bar[kBarSFull + sb], (t >> 1) & 1, c.abort_flag)) { ok = false; return false; }
      if (lane == 0 && q4 == 0) PAIR_TRACE(2, t);
      tc_fence_after();
      float x[64];
      if (nv > 0) tmem_ld_32x32b_x64(lane_base + sb * kPage, x);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.bar[kBarSEmpty + sb]);
      const bool last = (j == je - 1);

      // keys [0, nk) of the page are visible to this row
      int nk = nv;
      if (causal) nk = min(nk, max(lim - kPage * j, 0));
      const bool partial = __any_sync(0xffffffffu, nk < kPage);
      float rmax = -INFINITY;
      if (partial) {
#pragma unroll
        for (int i = 0; i < 64; ++i) rmax = fmaxf(rmax, i < nk ? x[i] : -INFINITY);
      } else {
#pragma unroll
        for (int i = 0; i < 64; ++i) rmax = fmaxf(rmax, x[i]);
      }
      const float tmax = rmax * scale_log2;         // -inf when no key is visible
      const bool need = tmax > m_run + kRescaleThreshold;
      const float m_new = need ? fmaxf(m_run, tmax) : m_run;
      const float alpha = (m_new == m_run) ? 1.f : fast_exp2(m_run - m_new);   // m_run = -inf -> 0
      l_run *= alpha;
      m_run = m_new;
      const float neg_m = m_run == -INFINITY ? 0.f : -m_run;
      uint32_t pk[32];
      float lsum = 0.f;
      if (partial) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float a = 2 * i < nk ? fast_exp2(fmaf(x[2 * i], scale_log2, neg_m)) : 0.f;
          const float b = 2 * i + 1 < nk ? fast_exp2(fmaf(x[2 * i + 1], scale_log2, neg_m)) : 0.f;
          lsum += a + b;
          pk[i] = pack_bf16x2(a, b);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float a = fast_exp2(fmaf(x[2 * i], scale_log2, neg_m));
          const float b = fast_exp2(fmaf(x[2 * i + 1], scale_log2, neg_m));
          lsum += a + b;
          pk[i] = pack_bf16x2(a, b);
        }
      }
      l_run += lsum;

      // publish into ring slot t % kPairSlots; a group's first page waits
      // until the value CTA has read the group the slots held before
      const int slot = t % kPairSlots;
      const int grp = t / kPairGroup;
      if (lane == 0 && q4 == 0) PAIR_TRACE(3, t);
      if (t % kPairGroup == 0 &&
          !mbar_wait_cluster(&c.bar[kBarSlotFree + grp % 2], ((grp / 2) & 1) ^ 1, c.abort_flag)) {
        ok = false;
        return false;
      }
      if (lane == 0 && q4 == 0) PAIR_TRACE(4, t);
      uint8_t* e = c.ring + static_cast<size_t>(slot) * kPairSlotBytes;
      uint8_t* wrows = e + q4 * 32 * 128;           // this warp's 32 rows (4 KB, contiguous)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        // rows 16h..16h+15 of the warp through the staging tile (same swizzle
        // as the tensor-core layout, so both sides are conflict-free)
        if ((lane >> 4) == h) {
          const uint32_t srow = stage + (lane & 15) * 128;
#pragma unroll
          for (int ch = 0; ch < 8; ++ch)
            st_shared_v4(srow + ((ch ^ (r & 7)) << 4),
                         make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]));
        }
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint4 v;
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                       : "r"(stage + k * 512 + lane * 16));
          *reinterpret_cast<uint4*>(wrows + h * 2048 + k * 512 + lane * 16) = v;
        }
        __syncwarp();
      }
      reinterpret_cast<float*>(e + kAlphaOff)[r] = alpha;
      float lse = -INFINITY;
      if (last) {
        const bool has = l_run > 0.f;
        reinterpret_cast<float*>(e + kInvLOff)[r] = has ? 1.f / l_run : 0.f;
        lse = has ? (m_run + log2f(l_run)) * kLn2 : -INFINITY;
      }


      if (last && row_valid) {
        const int nsplit = p.num_splits[u + 1] - p.num_splits[u];
        const int split_idx = (u == c.part.u0 && jb == c.part.j0) ? c.part.first_split : p.num_splits[u];
        const bool split = nsplit > 1 && split_idx >= 0 && split_idx < p.num_units + p.num_parts;
        if (nsplit > 1 && !split) atomicOr(p.err, kErrInternal);
        else if (split) p.ws_lse[static_cast<int64_t>(split_idx) * R + grow] = lse;
        else p.lse[(static_cast<int64_t>(ui.b) * h_q + grow % h_q) * s_q + tok] = lse;
      }
      if (t % kPairGroup == kPairGroup - 1) release(t);
      // every QK of this segment has been consumed: the next query tile may
      // take the TMEM columns of this one
      if (last) stage_q(u + 1);
      if (last && lane == 0 && q4 == 0) PAIR_TRACE(6, t);
      ++t;
    }
    return true;
  });
  if (ok && t % kPairGroup != 0) release(t - 1);    // the partition's last, partial group
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
    PAIR_TRACE(0, v.t);
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
    if (!ready(&c.bar[kBarOReady + b], (v.t >> 1) & 1)) { ok = false; break; }
    if (lane == 0) PAIR_TRACE(1, v.t);
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
    cursor_next(p, c.part, v);
  }
  if (!ok && lane == 0) pair_abort(c);
  umma_commit_elect(&c.bar[kBarDoneB]);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(&c.bar[kBarDoneB], 0) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
  }
  __syncwarp();
}

// Warps 2-5: take each published ring entry in (every warp its own 32 P rows,
// 512-B coalesced loads, into the P buffer the MMA reads), apply the O
// rescales, zero the padding rows of a partial page's V, and write the output
// of every segment (one thread per row).
__device__ __forceinline__ void value_rows(const Ctx& c, uint32_t tmem_base) {
  const DecodeParams& p = c.p;
  const int lane = threadIdx.x & 31;
  const int q4 = (threadIdx.x >> 5) & 3;
  const int r = 32 * q4 + lane;
  const int R = p.rows_per_unit;
  const int grow = c.row0 + r;
  const bool row_valid = grow < R;
  const uint32_t o_lane = tmem_base + (static_cast<uint32_t>(32 * q4) << 16);
  bool ok = true;

  Cursor v = cursor_begin(p, c.part);
  UnitInfo ui{};
  int seg = -1, seg_jb = 0, phys_next = -1;
  bool any_pv = false;
  while (v.valid) {
    const int t = v.t;
    const int u = v.u;
    if (v.seg != seg) {
      seg = v.seg;
      seg_jb = v.j;
      ui = unit_info(p, u);
      any_pv = false;
      phys_next = page_of(p, ui.b, v.j);
    }
    const int b = t & 1;
    const int s = t % kStagesV;
    const int slot = t % kPairSlots;
    const int phys = phys_next;                     // block-table entries are read one page ahead
    if (v.j + 1 < v.je) phys_next = page_of(p, ui.b, v.j + 1);
    const int nv = (phys >= 0 && phys < p.num_blocks) ? min(kPage, ui.L - kPage * v.j) : 0;
    const bool last = (v.j == v.je - 1);

    // ring entry t: its group was published by the score CTA (acquire at cluster scope)
    const int grp = t / kPairGroup;
    if (t % kPairGroup == 0 &&
        !mbar_wait_cluster(&c.bar[kBarSlotReady + grp % 2], (grp / 2) & 1, c.abort_flag)) {
      ok = false;
      break;
    }
    if (lane == 0 && q4 == 0) PAIR_TRACE(10, t);
    const uint8_t* e = c.ring + static_cast<size_t>(slot) * kPairSlotBytes;
    const uint8_t* wrows = e + q4 * 32 * 128;
    uint4 pv[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) pv[k] = ld_global_cg_v4(wrows + k * 512 + lane * 16);
    const float alpha = ld_global_cg_f32(e + kAlphaOff + 4 * r);
    const float inv_l = last ? ld_global_cg_f32(e + kInvLOff + 4 * r) : 0.f;
    // P buffer b is free once PV(t - 2) has completed
    if (!mbar_wait(&c.bar[kBarPbEmpty + b], ((t >> 1) & 1) ^ 1, c.abort_flag)) { ok = false; break; }
    const uint32_t pb_base = smem_u32(c.smem + Smem::pb_off + b * kPairSlotBytes);
    const uint32_t pb = pb_base + q4 * 32 * 128;
#pragma unroll
    for (int k = 0; k < 8; ++k) st_shared_v4(pb + k * 512 + lane * 16, pv[k]);
    // storing alpha and 1/l as well makes every load of the entry complete
    // before the entry is handed back below
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(pb_base + kAlphaOff + 4 * r), "f"(alpha) : "memory");
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(pb_base + kInvLOff + 4 * r), "f"(inv_l) : "memory");
    fence_proxy_async_smem();
    Cursor nx = v;
    cursor_next(p, c.part, nx);
    // the group has been read: the signal warp hands it back
    if (t % kPairGroup == kPairGroup - 1 || !nx.valid) {
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.bar[kBarSlotRead + grp % 2]);
    }

    if (__any_sync(0xffffffffu, any_pv && alpha != 1.f)) {
      // O must hold every earlier PV of the segment before it is rescaled:
      // pb_empty[(t - 1) & 1] completes with PV(t - 1) (and, the MMAs
      // completing in order, with every PV before it); its previous use,
      // PV(t - 3), has completed, and PV(t + 1) cannot start before this
      // warp's o_ready, so the parity is unambiguous
      if (!mbar_wait(&c.bar[kBarPbEmpty + ((t - 1) & 1)], ((t - 1) >> 1) & 1, c.abort_flag)) { ok = false; break; }
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
      uint8_t* vst = c.smem + Smem::v_off + s * kVPageBytes;
      const int tid = (q4 << 5) | lane;
      for (int idx = tid; idx < (kPage - nv) * 8 * 8; idx += 128) {
        const int rr = nv + idx / 64;
        const int rem = idx % 64;
        st_shared_v4(smem_u32(vst + (rem / 8) * kChunkBytes + rr * 128 + (rem % 8) * 16), make_uint4(0, 0, 0, 0));
      }
      fence_proxy_async_smem();
    }
    if (nv > 0) any_pv = true;
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&c.bar[kBarOReady + b]);
    if (lane == 0 && q4 == 0) PAIR_TRACE(11, t);

    if (last) {
      // ------------------------------------------------ epilogue of the segment
      // (the next segment's first PV overwrites O; it waits for this warp's
      // next o_ready arrival, which comes after these reads)
      // pb_empty[b] completes with PV(t) (its previous use, PV(t - 2), has
      // completed: this page's P buffer was free; PV(t + 2) cannot start
      // before this warp's next arrivals), and PV(t) completing implies
      // every earlier PV has
      if (!mbar_wait(&c.bar[kBarPbEmpty + b], (t >> 1) & 1, c.abort_flag)) { ok = false; break; }
      tc_fence_after();
      if (lane == 0 && q4 == 0) PAIR_TRACE(12, t);
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
      if (lane == 0 && q4 == 0) PAIR_TRACE(13, t);
    }
    v = nx;
  }
  if (!ok) pair_abort(c);
}

// Warp 6, one lane: each ring entry the row warps have read is handed back to
// the score CTA (release at cluster scope, ordering the reads before the
// score CTA's next stores into it).
__device__ __forceinline__ void value_signal(const Ctx& c) {
  const uint32_t peer = cluster_ctarank() ^ 1u;
  Cursor v = cursor_begin(c.p, c.part);
  while (v.valid) {
    Cursor nx = v;
    cursor_next(c.p, c.part, nx);
    if (v.t % kPairGroup == kPairGroup - 1 || !nx.valid) {
      const int grp = v.t / kPairGroup;
      if (!mbar_wait(&c.bar[kBarSlotRead + grp % 2], (grp / 2) & 1, c.abort_flag)) {
        pair_abort(c);
        return;
      }
      mbar_arrive_remote(mapa_shared(smem_u32(&c.bar[kBarSlotFree + grp % 2]), peer));
    }
    v = nx;
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
      for (int i = 0; i < 2; ++i) mbar_init(&c.bar[kBarSlotFree + i], 1);
      mbar_init(&c.bar[kBarDoneA], 1);
    } else {
      for (int s = 0; s < kStagesV; ++s) {
        mbar_init(&c.bar[kBarVFull + s], 1);
        mbar_init(&c.bar[kBarVEmpty + s], 1);
        c.nvalid[s] = 0;
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(&c.bar[kBarPbEmpty + i], 1);
        mbar_init(&c.bar[kBarOReady + i], 4);
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(&c.bar[kBarSlotReady + i], 4);
        mbar_init(&c.bar[kBarSlotRead + i], 4);
      }
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
      } else if (warp < kWarpSignal) {
        score_softmax(c, tmem_base);
      }
    } else {
      if (warp == kWarpLoad) {
        if (lane == 0) value_load(c, &tmap_kv);
      } else if (warp == kWarpMma) {
        value_mma(c, tmem_base);
      } else if (warp == kWarpSignal) {
        if (lane == 0) value_signal(c);
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

#ifdef MLA_TRACE
extern "C" __attribute__((visibility("default"))) int mla_pair_trace_copy(void* host_dst, size_t bytes) {
  if (bytes > sizeof(g_pair_trace)) bytes = sizeof(g_pair_trace);
  return cudaMemcpyFromSymbol(host_dst, g_pair_trace, bytes) == cudaSuccess ? 0 : 4;
}
extern "C" __attribute__((visibility("default"))) int mla_pair_trace_clear() {
  static unsigned long long zeros[kPairTraceCtas][kPairTraceEvents][kPairTracePages];
  return cudaMemcpyToSymbol(g_pair_trace, zeros, sizeof(zeros)) == cudaSuccess ? 0 : 4;
}
#endif

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
