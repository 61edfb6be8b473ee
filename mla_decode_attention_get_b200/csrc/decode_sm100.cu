// MLA decode attention over a paged KV cache on sm_100a (tcgen05 + TMEM + TMA).
//
// What it computes (per query row = (token, head), h_kv = 1): logits
// s_t = scale * q . K_t over the 576 cache dims of every visible key t,
// out = sum_t softmax(s)_t * K_t[:512] and lse = ln sum_t exp(s_t)
// ("Was ist FlashMLA?" (topnet.top), section "3. MLA-Decodierung ausführen":
// o_i, lse_i = flash_mla_with_kvcache(q, kvcache, block_table,
// cache_seqlens, dv, metadata, num_splits, causal)), over the bf16 cache.
// The FP8 cache (dense and sparse) has its own kernel, decode_fp8_sm100.cu.
//
// Design (one CTA = one scheduler partition x one tile of 64 query rows):
//  * Every MMA has M = 64 query rows.  Per 64-token page:
//      S[64 rows, 64 keys]  = Q[64, 576] . K_page[64, 576]^T   36 x (K = 16)
//      O[64 rows, 512 dims] += P[64, 64] . V_page[64, 512]       2 halves x 4 x (K = 16)
//    V is read MN-major straight from the same swizzled page tile, so V costs
//    no extra load.  The M = 64 accumulator layout fills 16 of the 32 lanes of
//    each TMEM quadrant: O sits in lanes 0-15 (all 512 columns); lanes 16-31
//    hold the two S buffers (columns 0-63, 64-127) and the query tile Q
//    (columns 128-415, two bf16 per column), which QK reads straight from TMEM
//    as its A operand.  With Q out of shared memory the page ring has 3 stages.
//  * P of a page is written into the page's own RoPE box (64 rows x 128 B,
//    the geometry of the swizzled P tile) once QK of the page has completed;
//    PV of the page reads it before the stage is refilled.  So the softmax of
//    the next page never waits for PV of this one: O is waited on only to
//    rescale it and in a segment's epilogue.
//  * Row r of the tile belongs to threads (r % 16) and (r % 16) + 16 of
//    softmax warp r / 16: with 16-lane TMEM accesses each of the pair holds
//    half of the row's 64 logits (and, in the epilogue, half of its O row), so
//    the row max / sum need one shuffle and no cross-warp synchronisation.
//  * Warp 0 streams pages with TMA (3-D tensor map, 128-byte swizzle, one page
//    = 9 boxes of 64 tokens x 64 dims) into the ring and warms L2 a few pages
//    (and the next query tile) ahead; warp 1 issues the MMAs; warps 2-5 write
//    each segment's query tile into TMEM, run the online softmax and the
//    epilogue.
//  * The running max only moves when a page's max exceeds it by more than
//    2^8 (per row); the final division by the row sum uses the same stale
//    max, so the result is exact.
//  * Every wait is bounded; on timeout the CTA raises MLA_DEVERR_TIMEOUT,
//    drains its own copies and MMAs, frees TMEM and returns.
#include <cuda_bf16.h>

#include "decode_common.cuh"
#include "mla_kernels.cuh"
#include "ptx_sm100.cuh"

namespace mla {

#ifdef MLA_TRACE
// Opt-in pipeline trace (built only with -DMLA_TRACE): clock64() stamps of the
// hand-offs of every page in the first kTraceCtas CTAs of row tile 0.
constexpr int kTraceCtas = 4, kTraceEvents = 16, kTracePages = 256;
__device__ unsigned long long g_mla_trace[kTraceCtas][kTraceEvents][kTracePages];
// globaltimer at the start and end of every CTA (x + 1024 * y), and its SM
__device__ unsigned long long g_mla_trace_span[3][4096];
#define MLA_TRACE_EV(ev, idx)                                                                   \
  do {                                                                                          \
    if (blockIdx.x < kTraceCtas && blockIdx.y == 0 && (idx) >= 0 && (idx) < kTracePages)        \
      g_mla_trace[blockIdx.x][ev][idx] = clock64();                                             \
  } while (0)
#define MLA_TRACE_SPAN(which)                                                                   \
  do {                                                                                          \
    const unsigned id = blockIdx.x + 1024u * blockIdx.y;                                        \
    if (id < 4096u) {                                                                           \
      g_mla_trace_span[which][id] = globaltimer_ns();                                           \
      unsigned smid;                                                                            \
      asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));                                         \
      g_mla_trace_span[2][id] = smid;                                                           \
    }                                                                                           \
  } while (0)
#else
#define MLA_TRACE_SPAN(which) \
  do {                        \
  } while (0)
#define MLA_TRACE_EV(ev, idx) \
  do {                        \
  } while (0)
#endif

namespace {

using namespace dec;

constexpr int kRows = kTileRows;              // query rows per CTA = M of every MMA
constexpr int kStages = 3;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemQCol = 128;           // Q tile columns 128..415 in lanes 16-31
constexpr int kPChunk = kChunks - 1;          // the RoPE chunk of a stage, reused for the page's P tile
// A stage is refilled in two parts: its chunks 0-3 (dims 0-255), which only
// QK^T and the first half of PV read, as soon as that half has completed,
// and chunks 4-8 (dims 256-575, P in chunk 8) once all of PV has.
constexpr int kLoChunks = 4;
static_assert(kLoChunks < kPChunk, "P lives in the part released last");

constexpr int kWarpLoad = 0, kWarpMma = 1, kWarpEnd = 6;   // warps 2-5: softmax
constexpr int kThreads = 32 * kWarpEnd;

struct Smem {
  // page ring; once QK of a page has completed, the page's RoPE chunk holds
  // its P tile ([64 rows x 64 keys], the same 128-B swizzled geometry)
  static constexpr int kv_off = 0;
  static constexpr int bar_off = kv_off + kStages * kPageBytes;
  // kv_full[S], kv_empty_lo[S], s_full[2], s_empty[2], q_full, p_full[S],
  // done, kv_empty[S]
  static constexpr int n_bars = 4 * kStages + 6;
  static constexpr int info_off = bar_off + n_bars * 8;
  static constexpr int info_bytes = kStages * 16;                // per stage: valid keys of the page
  static constexpr int misc_off = info_off + info_bytes;         // tmem base, abort flag
  static constexpr int total = misc_off + 16;
  static_assert(kv_off % 1024 == 0 && kPageBytes % 1024 == 0 && kChunkBytes % 1024 == 0,
                "tiles must stay 1024-B aligned");
  static_assert(total <= 232448, "shared memory budget");
};

struct StageInfo {
  int nvalid;
  int pad[3];
};

struct Bars {
  uint64_t* kv_full;      // per stage: both parts of the page landed (two arrivals)
  uint64_t* kv_empty_lo;  // per stage: chunks 0-3 free (first half of PV completed)
  uint64_t* kv_empty;     // per stage: the whole stage free (PV completed)
  uint64_t* s_full;
  uint64_t* s_empty;
  uint64_t* q_full;
  uint64_t* p_full;     // per stage: P of the stage's page written (4 softmax warps)
  uint64_t* done;
};

// Rows of this CTA's tile that exist in the unit (the rest is zero padding).
__device__ __forceinline__ int tile_valid_rows(const DecodeParams& p) {
  return min(kRows, p.rows_per_unit - static_cast<int>(blockIdx.y) * kRows);
}

__device__ __forceinline__ int64_t q_tile_offset(const DecodeParams& p, const UnitInfo& ui) {
  return q_tile_offset(p, ui, static_cast<int>(blockIdx.y) * kRows);
}

// One of a few values by a run-time index, without an indexed array (which
// would live in local memory).
__device__ __forceinline__ int pick(int i, int a, int b, int c, int d = 0) {
  return i == 0 ? a : (i == 1 ? b : (i == 2 ? c : d));
}

// The last page the load warp issued into each stage (-1: none), so that a
// CTA that gives up can wait for its own copies before it exits.
struct Issued {
  int t0 = -1, t1 = -1, t2 = -1;
  __device__ __forceinline__ void set(int s, int t) {
    if (s == 0) t0 = t;
    else if (s == 1) t1 = t;
    else t2 = t;
  }
  __device__ __forceinline__ int get(int s) const { return pick(s, t0, t1, t2); }
};
static_assert(kStages == 3, "Issued holds three stages");

// ---------------------------------------------------------------------------
// Warp 0 (one lane): TMA loads of cache pages, each in two parts (chunks 0-3
// once the stage's first PV half has completed, chunks 4-8 once all of PV
// has), their block-table entries read kPrefetchPages pages ahead, and an L2
// prefetch of the next segment's query tile.  (Warming the pages themselves
// in L2 ahead of their loads, 1 to 4 pages ahead, measured slower than not
// warming them at all.)
__device__ __forceinline__ void load_role(const DecodeParams& p, const Partition& part, const CUtensorMap* tmap_kv,
                                          uint8_t* smem, Bars bars, StageInfo* info, volatile int* abort_flag,
                                          Issued& issued) {
  const uint64_t pol_kv = l2_policy_evict_first();
  const uint32_t q_bytes = static_cast<uint32_t>(tile_valid_rows(p)) * kDqk * 2;
  int t = 0;
  bool ok = true;

  // Physical pages of the next kPrefetchPages pages, read ahead so that a
  // page's TMA load never waits on the block table (four scalars: an indexed
  // array would live in local memory).
  static_assert(kPrefetchPages == 4, "the page ring holds four entries");
  int r0 = -1, r1 = -1, r2 = -1, r3 = -1;
  auto ring_set = [&](int j, int phys) {
    const int i = j % kPrefetchPages;
    if (i == 0) r0 = phys;
    else if (i == 1) r1 = phys;
    else if (i == 2) r2 = phys;
    else r3 = phys;
  };
  auto ring_get = [&](int j) { return pick(j % kPrefetchPages, r0, r1, r2, r3); };

  for_each_segment(p, part, [&](int u, int jb, int je) -> bool {
    // warm the query tile of the following segment
    if (u + 1 <= part.u1 && u + 1 < p.num_units) {
      int jb2, je2;
      if (segment_bounds(p, part, u + 1, jb2, je2))
        bulk_prefetch_l2(p.q + q_tile_offset(p, unit_info(p, u + 1)), q_bytes);
    }
    {
      const UnitInfo ui = unit_info(p, u);
      // read the first pages' table entries together
      const int jn = min(je, jb + kPrefetchPages);
      for (int j = jb; j < jn; ++j) ring_set(j, page_of(p, ui.b, j));
      for (int j = jb; j < je; ++j) {
        const int s = t % kStages;
        const uint32_t free_parity = ((t / kStages) & 1) ^ 1;
        if (!mbar_wait(&bars.kv_empty_lo[s], free_parity, abort_flag, p.wait_ns)) { ok = false; return false; }
        MLA_TRACE_EV(0, t);
        int nv = min(kPage, ui.L - kPage * j);
        const int phys = ring_get(j);
        if (phys < 0 || phys >= p.num_blocks) {
          atomicOr(p.err, kErrBlockTable);
          nv = 0;
        }
        // (the stage's previous page is done with its info: the MMA warp read
        // it before QK^T, the softmax before writing the P that PV read)
        info[s].nvalid = nv;
        uint8_t* dst = smem + Smem::kv_off + s * kPageBytes;
        // kv_full takes two arrivals per page, one per part
        if (nv > 0) {
          mbar_arrive_expect_tx(&bars.kv_full[s], kLoChunks * kChunkBytes);
#pragma unroll 1
          for (int c = 0; c < kLoChunks; ++c)
            tma_load_3d(dst + c * kChunkBytes, tmap_kv, &bars.kv_full[s], 64 * c, 0, phys, pol_kv);
          issued.set(s, t);
        } else {
          mbar_arrive(&bars.kv_full[s]);
        }
        if (!mbar_wait(&bars.kv_empty[s], free_parity, abort_flag, p.wait_ns)) {
          // the page's second arrival, so that the drain at exit sees its
          // first part land
          mbar_arrive(&bars.kv_full[s]);
          ok = false;
          return false;
        }
        if (nv > 0) {
          mbar_arrive_expect_tx(&bars.kv_full[s], (kChunks - kLoChunks) * kChunkBytes);
#pragma unroll 1
          for (int c = kLoChunks; c < kChunks; ++c)
            tma_load_3d(dst + c * kChunkBytes, tmap_kv, &bars.kv_full[s], 64 * c, 0, phys, pol_kv);
        } else {
          mbar_arrive(&bars.kv_full[s]);
        }
        if (j + kPrefetchPages < je) ring_set(j + kPrefetchPages, page_of(p, ui.b, j + kPrefetchPages));
        ++t;
      }
      return true;
    }
  });

  if (!ok) raise_abort(abort_flag, p.err);
}

// ---------------------------------------------------------------------------
// Warp 1 (whole warp, one elected lane issues): the QK^T and PV MMAs.  Lane 0
// tests the barriers and broadcasts, so control flow stays warp-uniform and
// the MMA operands stay uniform.  Two cursors walk the pages: QK(t)
// is issued once page t has landed and its S buffer is free; PV(t) once the
// softmax has written P(t).  Whichever is ready goes first (PV preferred, as
// it releases the page's stage), so a late page never holds back the PV of
// the previous one.
__device__ __forceinline__ void mma_role(const DecodeParams& p, const Partition& part, uint8_t* smem, Bars bars,
                                         const StageInfo* info, uint32_t tmem_base, volatile int* abort_flag) {
  // S = Q K^T and O += P V (V MN-major)
  constexpr uint32_t idesc_qk = idesc_bf16_f32(kRows, kPage, false, false);
  constexpr uint32_t idesc_pv = idesc_bf16_f32(kRows, 256, false, true);
  const uint32_t tmem_q = tmem_base + (16u << 16) + kTmemQCol;   // A operand of QK (lanes 16-31)
  // descriptors of stage 0; a stage's own add its offset to the 16-B address field
  const uint32_t ring = smem_u32(smem + Smem::kv_off);
  const uint64_t k_desc0 = sdesc_sw128(ring, 16, 1024);
  const uint64_t v_desc0 = sdesc_sw128(ring, kChunkBytes, 1024);
  const uint64_t p_desc0 = sdesc_sw128(ring + kPChunk * kChunkBytes, 16, 1024);
  const uint32_t tmem_s0 = tmem_base + (16u << 16);    // S buffers: lanes 16-31 of each quadrant

  Cursor qk = cursor_begin(p, part);
  Cursor pv = qk;
  int o_seg = -1;
  // valid keys of the page in each stage (scalars: an indexed array would
  // live in local memory)
  int nv0 = 0, nv1 = 0, nv2 = 0;
  bool ok = true;
  uint64_t t_idle = globaltimer_ns();
  uint32_t spins = 0;

  const int lane = threadIdx.x & 31;
  auto ready = [&](uint64_t* bar, uint32_t parity) -> bool {
    return __shfl_sync(0xffffffffu, lane == 0 ? (mbar_test_wait(bar, parity) ? 1 : 0) : 0, 0) != 0;
  };

  while (pv.valid) {
    bool progressed = false;
    // PV(pv.t): after QK(pv.t) was issued and the softmax wrote P(pv.t)
    if (pv.t < qk.t && ready(&bars.p_full[pv.t % kStages], (pv.t / kStages) & 1)) {
      if (lane == 0) MLA_TRACE_EV(3, pv.t);
      tc_fence_after();
      const int s = pv.t % kStages;
      if (pick(s, nv0, nv1, nv2) > 0) {
        const bool acc0 = (o_seg == pv.seg);
        const uint64_t vd = v_desc0 + ((s * kPageBytes) >> 4);
        const uint64_t pd = p_desc0 + ((s * kPageBytes) >> 4);
        static_assert(kLoChunks == 4, "the first PV half reads chunks 0-3");
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            umma_bf16_elect(tmem_base + h * 256, pd + ((k * 32) >> 4),
                            vd + ((4 * h * kChunkBytes + k * 2048) >> 4), idesc_pv, (acc0 || k > 0) ? 1u : 0u);
          }
          // chunks 0-3 of the stage are free once the first half (and QK^T,
          // issued before it) has completed
          if (h == 0) umma_commit_elect(&bars.kv_empty_lo[s]);
        }
        o_seg = pv.seg;
      } else {
        umma_commit_elect(&bars.kv_empty_lo[s]);
      }
      // the stage (K, V and P of the page) is free once PV has completed
      umma_commit_elect(&bars.kv_empty[s]);
      if (lane == 0) MLA_TRACE_EV(14, pv.t);
      cursor_next(p, part, pv);
      progressed = true;
    }
    // QK(qk.t): page landed, query tile of its segment loaded, S buffer free
    if (qk.valid) {
      const int s = qk.t % kStages;
      const int sb = qk.t & 1;
      const bool first = (qk.j == (qk.u == part.u0 ? part.j0 : 0));
      if (ready(&bars.kv_full[s], (qk.t / kStages) & 1) && (!first || ready(bars.q_full, qk.seg & 1)) &&
          ready(&bars.s_empty[sb], ((qk.t >> 1) & 1) ^ 1)) {
        if (lane == 0) MLA_TRACE_EV(2, qk.t);
        tc_fence_after();
        const int nv = info[s].nvalid;
        if (s == 0) nv0 = nv;
        else if (s == 1) nv1 = nv;
        else nv2 = nv;
        if (nv > 0) {
          const uint64_t kd = k_desc0 + ((s * kPageBytes) >> 4);
          const uint32_t d = tmem_s0 + sb * kPage;
#pragma unroll
          for (int c = 0; c < kChunks; ++c) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              // K elements [64c + 16k, +16) of Q = TMEM columns [32c + 8k, +8)
              umma_bf16_ts_elect(d, tmem_q + 32 * c + 8 * k, kd + ((c * kChunkBytes + k * 32) >> 4), idesc_qk,
                                 (c | k) != 0 ? 1u : 0u);
            }
          }
        }
        umma_commit_elect(&bars.s_full[sb]);
        if (lane == 0) MLA_TRACE_EV(12, qk.t);
        cursor_next(p, part, qk);
        progressed = true;
      }
    }
    if (progressed) {
      spins = 0;
      t_idle = globaltimer_ns();
    } else if ((++spins & 255u) == 0) {
      const bool give_up = *abort_flag || globaltimer_ns() - t_idle > p.wait_ns;
      if (__shfl_sync(0xffffffffu, give_up ? 1 : 0, 0)) {
        ok = false;
        break;
      }
    }
  }
  if (!ok && lane == 0) raise_abort(abort_flag, p.err);
  // Wait until every MMA this warp issued has completed.
  umma_commit_elect(bars.done);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bars.done, 0) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
  }
  __syncwarp();
}

// ---------------------------------------------------------------------------
// Warps 2-5 (whole warps): the query tile of a unit into TMEM lanes 16-31 as
// packed bf16 pairs.  Thread (r, half) writes row r's dims
// [128 c + 64 half, +64) for c = 0..3 and RoPE dims [512 + 32 half, +32).
__device__ __forceinline__ void write_q_tile(const DecodeParams& p, const UnitInfo& ui, uint32_t tq_lane, int r,
                                             int half) {
  const bool valid = r < tile_valid_rows(p);
  const uint4* src = reinterpret_cast<const uint4*>(p.q + q_tile_offset(p, ui) + static_cast<int64_t>(r) * kDqk);
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    uint4 buf[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) buf[i] = valid ? __ldg(src + 16 * c + 8 * half + i) : make_uint4(0, 0, 0, 0);
    uint32_t v[32];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[4 * i] = buf[i].x; v[4 * i + 1] = buf[i].y; v[4 * i + 2] = buf[i].z; v[4 * i + 3] = buf[i].w;
    }
    tmem_st_16x32bx2_x32u(tq_lane + 64 * c, v);
  }
  uint32_t w[16];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 x = valid ? __ldg(src + 64 + 4 * half + i) : make_uint4(0, 0, 0, 0);
    w[4 * i] = x.x; w[4 * i + 1] = x.y; w[4 * i + 2] = x.z; w[4 * i + 3] = x.w;
  }
  tmem_st_16x32bx2_x16(tq_lane + 256, w);
}

// ---------------------------------------------------------------------------
// Warps 2-5: online softmax per page and the per-segment epilogue.
__device__ __forceinline__ void softmax_role(const DecodeParams& p, const Partition& part, uint8_t* smem,
                                             Bars bars, const StageInfo* info, uint32_t tmem_base,
                                             volatile int* abort_flag) {
  const int lane = threadIdx.x & 31;
  const int q4 = (threadIdx.x >> 5) & 3;            // TMEM lane quadrant of this warp
  const int half = lane >> 4;                        // which half of the row's keys / dims
  const int r = 16 * q4 + (lane & 15);               // tile row of this thread
  const int R = p.rows_per_unit;
  const int grow = blockIdx.y * kRows + r;           // row within the unit
  const bool row_valid = grow < R;
  // A warp whose 16 rows are all padding keeps the barrier protocol but does
  // no math: the O rows its P rows feed are never read.
  const bool warp_live = static_cast<int>(blockIdx.y) * kRows + 16 * q4 < R;
  const float scale_log2 = p.scale_log2;
  const int h_q = p.h_q, s_q = p.s_q;
  const int tok_dense = grow / h_q;                  // dense path: the row's query token
  const bool causal = p.causal != 0;
  const uint32_t s_taddr = tmem_base + (static_cast<uint32_t>(32 * q4 + 16) << 16);
  const uint32_t o_taddr = tmem_base + (static_cast<uint32_t>(32 * q4) << 16);
  const uint32_t p_row0 = smem_u32(smem + Smem::kv_off + kPChunk * kChunkBytes) + r * 128;
  const int key0 = 32 * half;                        // first key (and dim offset) of this thread's half
  const uint32_t tq_lane = tmem_base + (static_cast<uint32_t>(32 * q4 + 16) << 16) + kTmemQCol;

  // The query tile of the unit that follows u in this partition, if any, goes
  // into TMEM once every QK of the current segment has been consumed.
  auto stage_next_q = [&](int u_from) {
    for (int u = u_from; u <= part.u1 && u < p.num_units; ++u) {
      int jb, je;
      if (segment_bounds(p, part, u, jb, je)) {
        write_q_tile(p, unit_info(p, u), tq_lane, r, half);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars.q_full);
        return;
      }
    }
  };
  stage_next_q(part.u0);

  int t = 0;
  bool ok = true;

  for_each_segment(p, part, [&](int u, int jb, int je) -> bool {
    const UnitInfo ui = unit_info(p, u);
    if (lane == 0 && q4 == 0 && p.seqlens[ui.b] < 0) atomicOr(p.err, kErrSeqlen);
    float m_run = -INFINITY, l_run = 0.f;
    bool any_pv = false;
    const int lim = ui.L - s_q + tok_dense + 1;      // causal: keys t < lim are visible
    for (int j = jb; j < je; ++j) {
      const int s = t % kStages;
      const int sb = t & 1;
      if (!mbar_wait(&bars.kv_full[s], (t / kStages) & 1, abort_flag, p.wait_ns)) { ok = false; return false; }
      if (!mbar_wait(&bars.s_full[sb], (t >> 1) & 1, abort_flag, p.wait_ns)) { ok = false; return false; }
      if (lane == 0 && q4 == 2) MLA_TRACE_EV(4, t);
      tc_fence_after();
      const int nv = info[s].nvalid;
      const bool work = nv > 0 && warp_live;
      float x[32];
      if (work) tmem_ld_16x32bx2_x32(s_taddr + sb * kPage, x);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.s_empty[sb]);

      float tmax = -INFINITY;
      if (work) {
        const int nk = min(max(nv - key0, 0), 32);
        uint32_t vmask = nk >= 32 ? 0xFFFFFFFFu : ((1u << nk) - 1u);
        if (causal && kPage * j + key0 + 31 >= lim) {
          const int nc = min(max(lim - kPage * j - key0, 0), 32);
          vmask &= nc >= 32 ? 0xFFFFFFFFu : ((1u << nc) - 1u);
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          x[i] = ((vmask >> i) & 1u) ? x[i] * scale_log2 : -INFINITY;
          tmax = fmaxf(tmax, x[i]);
        }
      }
      tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 16));
      const bool need = tmax > m_run + kRescaleThreshold;
      if (lane == 0 && q4 == 2) MLA_TRACE_EV(11, t);

      if (lane == 0 && q4 == 2) MLA_TRACE_EV(6, t);
      if (__any_sync(0xffffffffu, need)) {
        const float m_new = need ? fmaxf(m_run, tmax) : m_run;
        const float alpha = (m_new == m_run) ? 1.f : fast_exp2(m_run - m_new);   // m_run = -inf -> 0
        l_run *= alpha;
        m_run = m_new;
        if (__any_sync(0xffffffffu, any_pv && alpha != 1.f)) {
          // O holds every PV of the segment once PV(t-1), which frees its
          // stage, has completed (any_pv implies t > 0)
          const int tp = t - 1;
          if (!mbar_wait(&bars.kv_empty[tp % kStages], (tp / kStages) & 1, abort_flag, p.wait_ns)) { ok = false; return false; }
          tc_fence_after();
          if (lane == 0 && q4 == 2) MLA_TRACE_EV(9, t);
#pragma unroll 1
          for (int c0 = 0; c0 < kDv; c0 += 64) {
            float v[32];
            tmem_ld_16x32bx2_x32(o_taddr + c0, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= alpha;
            tmem_st_16x32bx2_x32(o_taddr + c0, v);
          }
        }
      }

      // P = exp2(s - m) as bf16: this thread's 64-B half of
      // row r of the K-major swizzled P tile in the page's RoPE chunk, whose
      // last reader, QK of this page, has completed
      const float m_safe = m_run == -INFINITY ? 0.f : m_run;
      const uint32_t p_row = p_row0 + s * kPageBytes;
      uint32_t pk[16];
      if (work) {
        float lsum = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float a = fast_exp2(x[2 * i] - m_safe);
          const float b = fast_exp2(x[2 * i + 1] - m_safe);
          lsum += a + b;
          pk[i] = pack_bf16x2(a, b);
        }
        l_run += lsum;
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = 0u;
      }
      if (warp_live) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int chunk = 4 * half + c;
          st_shared_v4(p_row + ((chunk ^ (r & 7)) << 4),
                       make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]));
        }
      }
      if (lane == 0 && q4 == 2) MLA_TRACE_EV(13, t);

      // a partial last page may hold non-finite padding: zero its unused V rows
      if (nv > 0 && nv < kPage) {
        uint8_t* stage = smem + Smem::kv_off + s * kPageBytes;
        const int nrow = kPage - nv;
        const int tid = (q4 << 5) | lane;
        for (int idx = tid; idx < nrow * 8 * 8; idx += 128) {
          const int rr = nv + idx / 64;
          const int rem = idx % 64;
          const int c = rem / 8, ch = rem % 8;
          st_shared_v4(smem_u32(stage + c * kChunkBytes + rr * 128 + ch * 16), make_uint4(0, 0, 0, 0));
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.p_full[s]);
      if (lane == 0 && q4 == 2) MLA_TRACE_EV(7, t);
      if (nv > 0) any_pv = true;

      if (j == je - 1) stage_next_q(u + 1);
      if (j == je - 1 && warp_live) {
        // ------------------------------------------------ epilogue of the segment
        if (!mbar_wait(&bars.kv_empty[s], (t / kStages) & 1, abort_flag, p.wait_ns)) { ok = false; return false; }   // PV(t) done
        tc_fence_after();
        const float l = l_run + __shfl_xor_sync(0xffffffffu, l_run, 16);
        const bool has = any_pv && l > 0.f;
        const float inv = has ? 1.f / l : 0.f;
        const float lse = has ? (m_run + log2f(l)) * kLn2 : -INFINITY;
        const int nsplit = p.num_splits[u + 1] - p.num_splits[u];
        const int split_idx = (u == part.u0 && jb == part.j0) ? part.first_split : p.num_splits[u];
        bool split = nsplit > 1;
        if (split && (split_idx < 0 || split_idx >= p.num_units + p.num_parts)) {
          // metadata from another plan: never write outside the workspace
          if (lane == 0 && q4 == 0) atomicOr(p.err, kErrInternal);
          split = false;
        }
#pragma unroll 1
        for (int c0 = 0; c0 < kDv; c0 += 64) {
          float v[32];
          tmem_ld_16x32bx2_x32(o_taddr + c0, v);
          if (!row_valid) continue;
          const int d0 = c0 + key0;      // this thread's 32 dims
          if (split) {
            float4* dst = reinterpret_cast<float4*>(p.ws_o + (static_cast<int64_t>(split_idx) * R + grow) * kDv + d0);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(v[4 * i] * inv, v[4 * i + 1] * inv, v[4 * i + 2] * inv, v[4 * i + 3] * inv);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(p.out + (static_cast<int64_t>(u) * R + grow) * kDv + d0);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(pack_bf16x2(v[8 * i] * inv, v[8 * i + 1] * inv),
                                  pack_bf16x2(v[8 * i + 2] * inv, v[8 * i + 3] * inv),
                                  pack_bf16x2(v[8 * i + 4] * inv, v[8 * i + 5] * inv),
                                  pack_bf16x2(v[8 * i + 6] * inv, v[8 * i + 7] * inv));
          }
        }
        if (row_valid && half == 0) {
          if (split) {
            p.ws_lse[static_cast<int64_t>(split_idx) * R + grow] = lse;
          } else {
            p.lse[(static_cast<int64_t>(ui.b) * h_q + grow % h_q) * s_q + tok_dense] = lse;
          }
        }
        tc_fence_before();
        if (lane == 0 && q4 == 2) MLA_TRACE_EV(8, t);
      }
      ++t;
    }
    return true;
  });
  if (!ok) raise_abort(abort_flag, p.err);
}

// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 1)
    mla_decode_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmap_kv) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + Smem::bar_off);
  Bars bars;
  bars.kv_full = bar;
  bars.kv_empty_lo = bar + kStages;
  bars.s_full = bar + 2 * kStages;
  bars.s_empty = bar + 2 * kStages + 2;
  bars.q_full = bar + 2 * kStages + 4;
  bars.p_full = bar + 2 * kStages + 5;
  bars.done = bar + 3 * kStages + 5;
  bars.kv_empty = bar + 3 * kStages + 6;
  StageInfo* info = reinterpret_cast<StageInfo*>(smem + Smem::info_off);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Smem::misc_off);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Smem::misc_off + 4);

  const bool misaligned = (smem_u32(smem) & 1023u) != 0;
  if (threadIdx.x == 0) {
    *abort_flag = misaligned ? 1 : 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars.kv_full[s], 2);
      mbar_init(&bars.kv_empty_lo[s], 1);
      mbar_init(&bars.kv_empty[s], 1);
      mbar_init(&bars.p_full[s], 4);
      info[s].nvalid = 0;
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.s_full[i], 1);
      mbar_init(&bars.s_empty[i], 4);
    }
    mbar_init(bars.q_full, 4);
    mbar_init(bars.done, 1);
    fence_barrier_init();
  }
  if (warp == kWarpLoad && lane == 0) prefetch_tensormap(&tmap_kv);
  if (warp == kWarpMma) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // everything above overlaps the tail of the preceding kernel; the plan and
  // the caller's buffers are only touched from here on
  grid_dependency_wait();
  grid_launch_dependents();
  if (misaligned && threadIdx.x == 0) atomicOr(p.err, kErrInternal);
  const uint32_t tmem_base = *tmem_slot;
  const Partition part = load_partition(p, blockIdx.x);
  if (threadIdx.x == 0) MLA_TRACE_EV(10, 0);
  if (threadIdx.x == 0) MLA_TRACE_SPAN(0);

  Issued issued;
  if (!*abort_flag) {
    if (warp == kWarpLoad) {
      if (lane == 0) load_role(p, part, &tmap_kv, smem, bars, info, abort_flag, issued);
    } else if (warp == kWarpMma) {
      mma_role(p, part, smem, bars, info, tmem_base, abort_flag);
    } else {
      softmax_role(p, part, smem, bars, info, tmem_base, abort_flag);
    }
  }
  tc_fence_before();
  __syncthreads();
  // A CTA that gave up may still have page copies of its own in flight (the
  // load lane may have issued every page before another role gave up): the
  // load lane waits for them, bounded, before the shared memory is released.
  if (warp == kWarpLoad && lane == 0 && *abort_flag) {
    const uint64_t t0 = globaltimer_ns();
    for (int s = 0; s < kStages; ++s) {
      const int lt = issued.get(s);
      if (lt < 0) continue;
      while (!mbar_try_wait(&bars.kv_full[s], (lt / kStages) & 1) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) MLA_TRACE_EV(10, 1);
  if (threadIdx.x == 0) MLA_TRACE_SPAN(1);
  tc_fence_after();
  if (warp == kWarpMma) {
    __syncwarp();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

cudaError_t launch_one(const DecodeParams& p, const CUtensorMap& tkv, int row_tiles, cudaStream_t stream) {
  constexpr int smem = Smem::total;
  // The shared-memory opt-in is per device; remember which devices have it.
  static unsigned long long configured = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(__atomic_load_n(&configured, __ATOMIC_ACQUIRE) & bit)) {
    e = cudaFuncSetAttribute(mla_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    __atomic_fetch_or(&configured, bit, __ATOMIC_RELEASE);
  }
  return launch_dependent(mla_decode_kernel, dim3(p.num_parts, row_tiles), dim3(kThreads), smem, stream, p, tkv);
}

}  // namespace

#ifdef MLA_TRACE
extern "C" __attribute__((visibility("default"))) int mla_trace_copy(void* host_dst, size_t bytes) {
  if (bytes > sizeof(g_mla_trace)) bytes = sizeof(g_mla_trace);
  return cudaMemcpyFromSymbol(host_dst, g_mla_trace, bytes) == cudaSuccess ? 0 : 4;
}
extern "C" __attribute__((visibility("default"))) int mla_trace_span_copy(void* host_dst, size_t bytes) {
  if (bytes > sizeof(g_mla_trace_span)) bytes = sizeof(g_mla_trace_span);
  return cudaMemcpyFromSymbol(host_dst, g_mla_trace_span, bytes) == cudaSuccess ? 0 : 4;
}
extern "C" __attribute__((visibility("default"))) int mla_trace_clear() {
  static unsigned long long zeros[kTraceCtas][kTraceEvents][kTracePages];
  return cudaMemcpyToSymbol(g_mla_trace, zeros, sizeof(zeros)) == cudaSuccess ? 0 : 4;
}
#endif

cudaError_t launch_decode(const DecodeParams& p, const CUtensorMap& tmap_kv, int row_tiles, cudaStream_t stream) {
  return launch_one(p, tmap_kv, row_tiles, stream);
}

}  // namespace mla
