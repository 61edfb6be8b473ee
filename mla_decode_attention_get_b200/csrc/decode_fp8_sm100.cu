// MLA decode attention over the FP8 paged KV cache on sm_100a (tcgen05 +
// TMEM), sparse (the positions an indices tensor names) or dense (the block
// table walked page by page).
//
// What it computes is the bf16 path's result on the dequantised cache: a
// cache row is 512 e4m3 codes, four fp32 scales (one per 128-code group) and
// 64 bf16 RoPE values (FlashMLA walkthrough (sao.pub), section
// "二、核心功能与架构"); key dim d < 512 is code[d] * scale[d / 128], and
// dims 512..575 are the RoPE values.  Logits s_t = scale * q . K_t, out =
// sum_t softmax(s)_t * K_t[:512], lse = ln sum_t exp(s_t) ("Was ist
// FlashMLA?" (topnet.top), section "3. MLA-Decodierung ausführen").
//
// Exactness of the logits.  The tensor core never sees a scaled value:
//  * the gather warps convert the e4m3 codes to f16 (exact) and copy the
//    RoPE values as bf16 (exact);
//  * the query's 512 latent dims go to f16 after a per-row power-of-two
//    scaling 2^-e_r that keeps them inside the f16 range (exact for every
//    value within 2^24 of the row's largest), its RoPE dims stay bf16;
//  * QK^T accumulates one fp32 partial per 128-dim group (and one for RoPE)
//    in its own TMEM buffer, and the softmax warps form
//      s_t = scale * (2^e_r * sum_g scale[t][g] * partial_g + partial_rope)
//    in fp32.  The only rounding left is the fp32 arithmetic.
//  * PV needs the scales inside the products.  Once QK^T of a tile has
//    completed, the gather warps rewrite the tile's codes in place as
//    V'[t][d] = code[t][d] * scale[t][g] * 2^-E_g (f16, g = d / 128; the
//    values only feed the output, so their 2^-11 rounding is harmless), and
//    PV accumulates P . V'.  E_g is a per-CTA, per-segment power of two that
//    follows the largest scale of the group seen so far (raised lazily; O's
//    group columns are rescaled by the exact power of two when it moves), so
//    V' stays inside the f16 range whatever the scales' magnitude.  The
//    epilogue multiplies back by 2^E_g.
//
// Design (one CTA = one scheduler partition x one tile of 64 query rows):
//  * Warp 0 warms L2 with the next segment's query tile; warp 1 issues the
//    MMAs; warps 2-5 stage the query tile in TMEM, run the softmax and the
//    epilogue; warps 6-13 gather and convert the cache rows of each 64-key
//    tile into a three-stage ring, and six of them rewrite V' one tile behind.
//  * A stage holds 9 swizzled 64-key x 64-dim chunks (8 of f16 codes, 1 of
//    bf16 RoPE); the RoPE chunk holds the tile's P (f16) once QK^T of the
//    tile has completed.
//  * TMEM (M = 64 layout: 16 lanes of each 32-lane quadrant): O in lanes
//    0-15 (512 columns); lanes 16-31 hold a ring of three partial-S slots
//    (columns 0-191), the query's latent dims (192-447) and its RoPE dims
//    (448-479).  QK^T of a tile is five parts (latent groups 0-3, RoPE), each
//    into the next slot once the softmax has read the slot's previous part,
//    so the MMAs of one tile overlap the softmax of the one before.
//  * Every wait is bounded; on timeout the CTA raises MLA_DEVERR_TIMEOUT,
//    drains its own MMAs, frees TMEM and returns.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "decode_common.cuh"
#include "mla_kernels.cuh"
#include "ptx_sm100.cuh"

namespace mla {

#ifdef MLA_TRACE
// Opt-in pipeline trace (built only with -DMLA_TRACE): clock64() stamps of the
// hand-offs of every tile in the first kFp8TraceCtas CTAs of row tile 0.
constexpr int kFp8TraceCtas = 4, kFp8TraceEvents = 64, kFp8TraceTiles = 256;
__device__ unsigned long long g_fp8_trace[kFp8TraceCtas][kFp8TraceEvents][kFp8TraceTiles];
// Per CTA (all of them): %globaltimer at entry, after the set-up and the
// dependency wait, and at exit, and the SM it ran on.
constexpr int kFp8SpanCtas = 1024;
__device__ unsigned long long g_fp8_span[kFp8SpanCtas][4];
#define FP8_SPAN(k)                                                              \
  do {                                                                           \
    const unsigned cta = blockIdx.y * gridDim.x + blockIdx.x;                    \
    if (threadIdx.x == 0 && cta < kFp8SpanCtas) {                                \
      g_fp8_span[cta][k] = globaltimer_ns();                                     \
      if ((k) == 0) {                                                            \
        unsigned sm;                                                             \
        asm volatile("mov.u32 %0, %%smid;" : "=r"(sm));                          \
        g_fp8_span[cta][3] = sm;                                                 \
      }                                                                          \
    }                                                                            \
  } while (0)
#define FP8_TRACE(ev, idx)                                                                      \
  do {                                                                                          \
    if (blockIdx.x < kFp8TraceCtas && blockIdx.y == 0 && (idx) >= 0 && (idx) < kFp8TraceTiles)  \
      g_fp8_trace[blockIdx.x][ev][idx] = clock64();                                             \
  } while (0)
#else
#define FP8_TRACE(ev, idx) \
  do {                     \
  } while (0)
#define FP8_SPAN(k) \
  do {              \
  } while (0)
#endif

namespace {

using namespace dec;

constexpr int kRows = kTileRows;               // query rows per CTA = M of every MMA
constexpr int kStages = 3;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColQ = 192;                // query latent dims (f16 pairs), lanes 16-31
constexpr uint32_t kColQRope = 448;            // query RoPE dims (bf16 pairs), lanes 16-31
constexpr int kRopeChunk = kChunks - 1;        // chunk 8: RoPE; then P of the tile
constexpr int kStageBytes = kPageBytes;        // 73728
// The scales of a stage: [group][key] fp32, so that a softmax thread reads the
// group-g scales of its 32 keys as eight 16-byte loads.
constexpr int kScaleFloats = 4 * kPage;        // per stage
// QK^T of a tile is five parts (latent groups 0-3, then RoPE), each written
// into the next slot of a ring of partial-S buffers in TMEM.
constexpr int kParts = 5;
constexpr int kSlots = 3;
constexpr int kRescaleGroupLog2 = 7;           // raise E_g once a scale reaches 2^(E_g + 7)

constexpr int kWarpQPrefetch = 0, kWarpMma = 1, kWarpSoftmax0 = 2, kWarpGather0 = 6;
constexpr int kGatherWarps = 8;                // warp gw converts keys [8 gw, 8 gw + 8)
// The V' rewrite is left to the gather warps whose schedulers do not hold the
// MMA warp (the softmax warp that shares a scheduler with the MMA warp is the
// slowest one, and a quarter of a gather warp's instructions are the
// rewrite): gather warps 2 and 6 (scheduler 0, whose prefetch warp is idle)
// take 8 keys each, gather warps 0, 4 (scheduler 2) and 1, 5 (scheduler 3) 12.
constexpr int kRewriteWarps = 6;
struct RewriteKeys {
  int first, count;
};
__host__ __device__ constexpr RewriteKeys rewrite_keys(int gw) {
  return gw == 2 ? RewriteKeys{0, 8} : gw == 6 ? RewriteKeys{8, 8} : gw == 0 ? RewriteKeys{16, 12}
         : gw == 4 ? RewriteKeys{28, 12} : gw == 1 ? RewriteKeys{40, 12} : gw == 5 ? RewriteKeys{52, 12}
                   : RewriteKeys{0, 0};
}
static_assert(rewrite_keys(0).count + rewrite_keys(1).count + rewrite_keys(2).count + rewrite_keys(3).count +
                      rewrite_keys(4).count + rewrite_keys(5).count + rewrite_keys(6).count +
                      rewrite_keys(7).count == kPage &&
                  rewrite_keys(5).first + rewrite_keys(5).count == kPage,
              "the rewriting warps cover the 64 keys once");
constexpr int kThreads = 32 * (kWarpGather0 + kGatherWarps);

struct StageInfo {
  float4 gmax[kGatherWarps];                   // per gather warp: largest |scale| of each group
  uint8_t mask[kGatherWarps];                  // valid keys of the warp's 8
  uint8_t pad[8];
};

struct Smem {
  static constexpr int stage_off = 0;
  static constexpr int scales_off = stage_off + kStages * kStageBytes;      // [stage][group][key] float
  static constexpr int info_off = scales_off + kStages * kScaleFloats * 4;
  static constexpr int bar_off = (info_off + kStages * static_cast<int>(sizeof(StageInfo)) + 7) & ~7;
  // kv_full, kv_empty, p_full, qk_done, v_ready (per stage), slot_full, slot_empty (per slot),
  // q_full, done
  static constexpr int n_bars = 5 * kStages + 2 * kSlots + 2;
  static constexpr int misc_off = bar_off + n_bars * 8;                     // tmem base, abort flag
  static constexpr int total = misc_off + 16;
  static_assert(kStageBytes % 1024 == 0 && kChunkBytes % 1024 == 0, "tiles must stay 1024-B aligned");
  static_assert(total <= 232448, "shared memory budget");
};

struct Bars {
  uint64_t* kv_full;    // [stage] tile converted (8 gather warps)
  uint64_t* kv_empty;   // [stage] PV of the stage's tile completed (commit)
  uint64_t* p_full;     // [stage] P of the stage's tile written (4 softmax warps)
  uint64_t* qk_done;    // [stage] both QK^T passes of the stage's tile completed (commit)
  uint64_t* v_ready;    // [stage] V' of the stage's tile written (6 rewriting gather warps)
  uint64_t* slot_full;  // [slot] a part of QK^T completed into the slot (commit)
  uint64_t* slot_empty; // [slot] the slot was read (4 softmax warps)
  uint64_t* q_full;     // query tile of the next segment in TMEM (4 softmax warps)
  uint64_t* done;
};

__device__ __forceinline__ int tile_valid_rows(const DecodeParams& p) {
  return min(kRows, p.rows_per_unit - static_cast<int>(blockIdx.y) * kRows);
}

__device__ __forceinline__ uint8_t* stage_ptr(uint8_t* smem, int s) { return smem + Smem::stage_off + s * kStageBytes; }

__device__ __forceinline__ int scale_index(int s, int g, int k) { return (s * 4 + g) * kPage + k; }

// Position in the ring of partial-S slots; the MMA warp and the softmax warps
// step through it in the same order (five parts per tile).
struct Ring {
  int slot = 0;
  uint32_t phase = 0;
  __device__ __forceinline__ void next() {
    if (++slot == kSlots) {
      slot = 0;
      phase ^= 1u;
    }
  }
};

// 2^n for n in [-126, 127] (a normal fp32 number).
__device__ __forceinline__ float pow2i(int n) { return __int_as_float((127 + n) << 23); }

// floor(log2 x) of a positive finite x, clamped to [-126, 126].
__device__ __forceinline__ int exp2_floor(float x) {
  const int e = static_cast<int>((__float_as_uint(x) >> 23) & 0xFFu) - 127;   // subnormal -> -127
  return min(max(e, -126), 126);
}

// One of four values by a run-time index, without an indexed array (which
// would live in local memory).
template <typename T>
__device__ __forceinline__ T pick4(int g, T a, T b, T c, T d) {
  return g == 0 ? a : (g == 1 ? b : (g == 2 ? c : d));
}

// The per-segment exponents E_g of the four scale groups.  Every thread that
// feeds it the same tiles in the same order holds the same values: E_g is set
// by the first tile with a nonzero scale in the group and raised once a
// tile's largest |scale| reaches 2^(E_g + 7), so that scale * 2^-E_g < 2^7.
struct GroupExp {
  int e0, e1, e2, e3;
  uint32_t set;          // bit g: E_g has been set in this segment

  __device__ __forceinline__ void reset() {
    e0 = e1 = e2 = e3 = 0;
    set = 0;
  }
  __device__ __forceinline__ int e(int g) const { return pick4(g, e0, e1, e2, e3); }

  // Raise or set E_g from the group's largest |scale| in a tile; returns
  // 2^(E_old - E_new) (1 where E_g did not move).
  __device__ __forceinline__ float step(int& eg, int g, float gm) {
    if (!(gm > 0.f && gm <= 3.4e38f)) return 1.f;
    const int x = exp2_floor(gm);
    if (!(set & (1u << g))) {
      eg = x;                // the group's columns of O are still zero
      set |= 1u << g;
      return 1.f;
    }
    if (x < eg + kRescaleGroupLog2) return 1.f;
    const float beta = pow2i(eg) * pow2i(-x);
    eg = x;
    return beta;
  }

  // The tile's largest |scale| per group, from its gather warps' maxima.
  __device__ __forceinline__ static float4 tile_max(const StageInfo& si) {
    float4 m = si.gmax[0];
#pragma unroll
    for (int w = 1; w < kGatherWarps; ++w) {
      const float4 x = si.gmax[w];
      m = make_float4(fmaxf(m.x, x.x), fmaxf(m.y, x.y), fmaxf(m.z, x.z), fmaxf(m.w, x.w));
    }
    return m;
  }
  // Update from a tile's per-group maxima; beta_g = 2^(E_old - E_new).
  // Returns whether some E_g moved.
  __device__ __forceinline__ bool update(const float4 m, float4& beta) {
    beta.x = step(e0, 0, m.x);
    beta.y = step(e1, 1, m.y);
    beta.z = step(e2, 2, m.z);
    beta.w = step(e3, 3, m.w);
    return beta.x != 1.f || beta.y != 1.f || beta.z != 1.f || beta.w != 1.f;
  }
};

// ---------------------------------------------------------------------------
// Warp 0 (one lane): warm L2 with the query tile of every segment after the
// first, a segment ahead.
__device__ __forceinline__ void q_prefetch_role(const DecodeParams& p, const Partition& part) {
  const uint32_t q_bytes = static_cast<uint32_t>(tile_valid_rows(p)) * kDqk * 2;
  for_each_segment(p, part, [&](int u, int, int) -> bool {
    if (u + 1 <= part.u1 && u + 1 < p.num_units) {
      int jb2, je2;
      if (segment_bounds(p, part, u + 1, jb2, je2))
        bulk_prefetch_l2(p.q + q_tile_offset(p, unit_info(p, u + 1), static_cast<int>(blockIdx.y) * kRows), q_bytes);
    }
    return true;
  });
}

// ---------------------------------------------------------------------------
// Warps 6-13: gather the rows of each 64-key tile (the indexed positions, or
// the page's rows on the dense path) and write them into the stage: codes as
// f16 (exact), RoPE as bf16 (copied), the four scales per key, each warp's
// largest |scale| per group and its valid-key mask.  Warp gw owns keys
// [8 gw, 8 gw + 8); lane l (< 8) resolves key 8 gw + l (index -> block table
// -> row).  While tile t converts, the table entries of tile t+2 and the
// indices of tile t+3 are in flight (the rows are not warmed in L2 ahead:
// that measured no faster).  Lane
// l converts codes [8 l, 8 l + 8) and [256 + 8 l, 256 + 8 l + 8) and, for
// l < 16, copies RoPE dims [512 + 4 l, +4) of each of the warp's 8 rows.
// After converting tile t the rewriting warps rewrite tile t-1 as V' (they
// wait for its QK^T to complete): lane l of a warp that rewrites keys
// [first, first + count) scales key first + 8 h + l / 4 (h = 0, 1, while
// below first + count), group l % 4 (128 codes, 16 x 16 B), by its scale x
// 2^-E_g.  So PV of tile t-1 can run while tile t+1
// converts, and the stage it frees is the one tile t+2 needs.
__device__ __forceinline__ void gather_role(const DecodeParams& p, const Partition& part, uint8_t* smem, Bars bars,
                                            volatile int* abort_flag, int gw) {
  const int lane = threadIdx.x & 31;
  const int kl = lane & 7;
  bool ok = true;
  StageInfo* info = reinterpret_cast<StageInfo*>(smem + Smem::info_off);
  float* scales = reinterpret_cast<float*>(smem + Smem::scales_off);

  const bool sparse = p.indices != nullptr;
  auto fetch_pos = [&](const Cursor& c) -> int {
    if (!c.valid) return -1;
    const int pos_i = kPage * c.j + 8 * gw + kl;
    if (!sparse) return pos_i;
    const bool in = pos_i < p.topk;
    return ld_nc_s32_if(p.indices + (in ? static_cast<int64_t>(c.u) * p.topk + pos_i : 0), in, -1);
  };
  auto row_ptr = [&](int phys, int pos) -> const uint8_t* {
    return p.kv + static_cast<int64_t>(phys) * p.kv_block_stride + (pos & 63) * kFp8Row;
  };
  struct Pending {
    int pos, L, page_entry;
  };
  auto start_resolve = [&](const Cursor& c, int pos) -> Pending {
    Pending r{pos, 0, -1};
    if (!c.valid) return r;
    const int b = sparse ? c.u / p.s_q : c.u;
    r.L = ld_nc_s32_if(p.seqlens + b, true, 0);
    const int j = pos >> 6;
    const bool in = pos >= 0 && j < p.bt_width;
    r.page_entry = ld_nc_s32_if(p.block_table + (in ? static_cast<int64_t>(b) * p.bt_stride + j : 0), in, -1);
    return r;
  };
  auto finish_resolve = [&](const Cursor& c, const Pending& r, int& phys) -> bool {
    phys = -1;
    if (!c.valid) return false;
    bool v = r.pos >= 0 && r.pos < r.L;
    if (!v && r.pos != -1 && sparse && lane < 8) atomicOr(p.err, kErrIndex);
    if (v) {
      phys = r.page_entry;
      if (phys < 0 || phys >= p.num_blocks) {
        if (lane < 8) atomicOr(p.err, kErrBlockTable);
        v = false;
      }
    }
    return v;
  };

  // V' of tile tr (cursor rwc), one tile behind the conversion
  const RewriteKeys rwk = rewrite_keys(gw);
  const bool rewriter = rwk.count > 0;
  Cursor rwc = cursor_begin(p, part);
  int tr = 0, rw_seg = -1;
  GroupExp gexp;
  gexp.reset();
  auto rewrite = [&]() -> bool {
    const int s = tr % kStages;
    if (!mbar_wait(&bars.qk_done[s], (tr / kStages) & 1, abort_flag, p.wait_ns)) return false;
    if (rwc.seg != rw_seg) {
      gexp.reset();
      rw_seg = rwc.seg;
    }
    float4 beta;
    gexp.update(GroupExp::tile_max(info[s]), beta);
    const int e = lane >> 2, qq = lane & 3;
    const float gsc = pow2i(-gexp.e(qq));
#pragma unroll 1
    for (int h = 0; h < 2; ++h) {
      if (8 * h + e >= rwk.count) continue;
      const int k = rwk.first + 8 * h + e;
      const float f32 = scales[scale_index(s, qq, k)] * gsc;
      const uint32_t f = pack_f16x2(f32, f32);
      uint8_t* row = stage_ptr(smem, s) + k * 128;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint4* base = reinterpret_cast<uint4*>(row + (2 * qq + cc) * kChunkBytes);
        // a quarter warp (two keys x four groups) touches eight different 16-B banks
        uint4 v[8];
#pragma unroll
        for (int uu = 0; uu < 8; ++uu) v[uu] = base[(uu + 2 * qq + e) & 7];
#pragma unroll
        for (int uu = 0; uu < 8; ++uu)
          base[(uu + 2 * qq + e) & 7] =
              make_uint4(hmul2_f16(v[uu].x, f), hmul2_f16(v[uu].y, f), hmul2_f16(v[uu].z, f), hmul2_f16(v[uu].w, f));
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars.v_ready[s]);
    cursor_next(p, part, rwc);
    ++tr;
    return true;
  };

  Cursor cur = cursor_begin(p, part);
  Cursor nxt = cur;
  cursor_next(p, part, nxt);
  Cursor nxt2 = nxt;
  cursor_next(p, part, nxt2);
  int pos_c = fetch_pos(cur);
  int phys_c = -1;
  bool valid_c = finish_resolve(cur, start_resolve(cur, pos_c), phys_c);
  int pos_n = fetch_pos(nxt);
  Pending pend_n = start_resolve(nxt, pos_n);
  int pos_nn = fetch_pos(nxt2);
  int t = 0;
  while (cur.valid) {
    const int s = t % kStages;
    int phys_n = -1;
    const bool valid_n = finish_resolve(nxt, pend_n, phys_n);
    const Pending pend_nn = start_resolve(nxt2, pos_nn);
    Cursor nxt3 = nxt2;
    cursor_next(p, part, nxt3);
    const int pos_nnn = fetch_pos(nxt3);
    float gm0 = 0.f, gm1 = 0.f;   // lanes < 16: groups 0, 2; lanes >= 16: groups 1, 3
    {
      // the tile's rows are loaded before the
      // stage is free, so their latency overlaps the wait
      uint2 n0[8], n1[8], rp[8];
      float s0[8], s1[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int phys = __shfl_sync(0xffffffffu, phys_c, e);
        const int pos = __shfl_sync(0xffffffffu, pos_c, e);
        const bool v = __shfl_sync(0xffffffffu, valid_c ? 1 : 0, e) != 0;
        n0[e] = n1[e] = rp[e] = make_uint2(0, 0);
        s0[e] = s1[e] = 0.f;
        if (v) {
          const uint8_t* row = row_ptr(phys, pos);
          n0[e] = __ldg(reinterpret_cast<const uint2*>(row + 8 * lane));
          n1[e] = __ldg(reinterpret_cast<const uint2*>(row + 256 + 8 * lane));
          s0[e] = __ldg(reinterpret_cast<const float*>(row + 512 + 4 * (lane >> 4)));
          s1[e] = __ldg(reinterpret_cast<const float*>(row + 520 + 4 * (lane >> 4)));
          if (lane < 16) rp[e] = __ldg(reinterpret_cast<const uint2*>(row + 528 + 8 * lane));
        }
      }
      if (lane == 0 && gw == 0) FP8_TRACE(0, t);
      if (!mbar_wait(&bars.kv_empty[s], ((t / kStages) & 1) ^ 1, abort_flag, p.wait_ns)) { ok = false; break; }
      if (lane == 0 && gw == 0) FP8_TRACE(1, t);
      uint8_t* stage = stage_ptr(smem, s);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int k = 8 * gw + e;   // token row of the tile
        const int sw = k & 7;
        const uint32_t slot = static_cast<uint32_t>(((lane & 7) ^ sw) << 4);
        const uint32_t rowa = smem_u32(stage + k * 128);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const uint2 codes = half ? n1[e] : n0[e];
          const uint32_t w[2] = {codes.x, codes.y};
          uint32_t o[4];
          e4m3x4_to_f16x4(w[0], o[0], o[1]);
          e4m3x4_to_f16x4(w[1], o[2], o[3]);
          const int chunk = 4 * half + (lane >> 3);
          st_shared_v4(rowa + chunk * kChunkBytes + slot, make_uint4(o[0], o[1], o[2], o[3]));
        }
        if (lane < 16) {
          const uint32_t unit = static_cast<uint32_t>(((lane >> 1) ^ sw) << 4) + (lane & 1) * 8;
          asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(rowa + kRopeChunk * kChunkBytes + unit),
                       "r"(rp[e].x), "r"(rp[e].y)
                       : "memory");
        }
        // the key's four scales: lane 0 holds groups 0 and 2, lane 16 groups 1 and 3
        if ((lane & 15) == 0) {
          scales[scale_index(s, lane >> 4, k)] = s0[e];
          scales[scale_index(s, 2 + (lane >> 4), k)] = s1[e];
        }
        gm0 = fmaxf(gm0, fabsf(s0[e]));
        gm1 = fmaxf(gm1, fabsf(s1[e]));
      }
    }
    const uint32_t mask = __ballot_sync(0xffffffffu, valid_c) & 0xFFu;
    if (lane == 0) info[s].mask[gw] = static_cast<uint8_t>(mask);
    if ((lane & 15) == 0) {
      float* gm = reinterpret_cast<float*>(&info[s].gmax[gw]);
      gm[lane >> 4] = gm0;
      gm[2 + (lane >> 4)] = gm1;
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars.kv_full[s]);
    if (lane == 0 && (gw == 0 || gw == 7)) FP8_TRACE(gw == 0 ? 2 : 14, t);
    cur = nxt;
    nxt = nxt2;
    nxt2 = nxt3;
    pos_c = pos_n;
    phys_c = phys_n;
    valid_c = valid_n;
    pos_n = pos_nn;
    pend_n = pend_nn;
    pos_nn = pos_nnn;
    ++t;
    if (rewriter && t - tr > 1 && !rewrite()) { ok = false; break; }
  }
  while (ok && rewriter && rwc.valid) {
    if (!rewrite()) ok = false;
  }
  if (!ok && lane == 0) raise_abort(abort_flag, p.err);
}

__device__ __forceinline__ int stage_nvalid(const StageInfo& si) {
  int n = 0;
#pragma unroll
  for (int w = 0; w < kGatherWarps; ++w) n += __popc(si.mask[w]);
  return n;
}

// ---------------------------------------------------------------------------
// Warp 1 (whole warp, one elected lane issues): the MMAs, in a fixed order per
// tile t, each step after a (bounded, sleeping) wait for its inputs:
//   QK^T(t), five parts   latent groups 0-3 (8 MMAs each, f16 codes) and RoPE
//                         (4 MMAs, bf16), each into the next slot of the
//                         three-slot ring once the softmax has read the
//                         slot's previous part; the first part also waits for
//                         the tile and (at a segment start) the query tile;
//   PV(t-1)               P and V' of t-1 written;
//   PV(t)                 only at the end of a segment, whose epilogue waits
//                         on it.
// So the first three parts of tile t run while the softmax finishes tile t-1,
// and PV(t-1) while it reads the parts of tile t.
__device__ __forceinline__ void mma_role(const DecodeParams& p, const Partition& part, uint8_t* smem, Bars bars,
                                         uint32_t tmem_base, volatile int* abort_flag) {
  constexpr uint32_t idesc_qk = idesc_f16_f32(kRows, kPage, false, false);
  constexpr uint32_t idesc_rope = idesc_bf16_f32(kRows, kPage, false, false);
  constexpr uint32_t idesc_pv = idesc_f16_f32(kRows, 256, false, true);
  const StageInfo* info = reinterpret_cast<const StageInfo*>(smem + Smem::info_off);
  const uint32_t tmem_hi = tmem_base + (16u << 16);      // lanes 16-31 of each quadrant
  const uint32_t ring_base = smem_u32(smem + Smem::stage_off);
  const uint64_t k_desc0 = sdesc_sw128(ring_base, 16, 1024);
  const uint64_t v_desc0 = sdesc_sw128(ring_base, kChunkBytes, 1024);
  const uint64_t p_desc0 = sdesc_sw128(ring_base + kRopeChunk * kChunkBytes, 16, 1024);

  auto qk_chunk = [&](uint32_t d, uint64_t kd, uint32_t a_col, int c, uint32_t idesc, bool first_chunk) {
#pragma unroll
    for (int k = 0; k < 4; ++k)
      umma_bf16_ts_elect(d, tmem_hi + a_col + 8 * k, kd + ((c * kChunkBytes + k * 32) >> 4), idesc,
                         (!first_chunk || k > 0) ? 1u : 0u);
  };
  // PV(t): O += P . V' of the stage's tile (both 256-column halves)
  int o_seg = -1;
  auto pv_tile = [&](int t, int seg, int nv) -> bool {
    const int s = t % kStages;
    FP8_TRACE(41, t);
    if (!mbar_wait(&bars.p_full[s], (t / kStages) & 1, abort_flag, p.wait_ns)) return false;
    FP8_TRACE(42, t);
    if (!mbar_wait(&bars.v_ready[s], (t / kStages) & 1, abort_flag, p.wait_ns)) return false;
    tc_fence_after();
    FP8_TRACE(5, t);
    if (nv > 0) {
      const bool acc0 = (o_seg == seg);
      const uint64_t vd = v_desc0 + ((s * kStageBytes) >> 4);
      const uint64_t pd = p_desc0 + ((s * kStageBytes) >> 4);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma_bf16_elect(tmem_base + h * 256, pd + ((k * 32) >> 4),
                          vd + ((4 * h * kChunkBytes + k * 2048) >> 4), idesc_pv, (acc0 || k > 0) ? 1u : 0u);
      }
      o_seg = seg;
    }
    umma_commit_elect(&bars.kv_empty[s]);   // the stage is free once PV has completed
    return true;
  };

  Cursor c = cursor_begin(p, part);
  bool ok = true;
  bool have_prev = false;   // a tile whose PV is still to issue
  int prev_t = 0, prev_seg = 0, prev_nv = 0;
  Ring ring;
  while (c.valid) {
    const int t = c.t;
    const int s = t % kStages;
    const bool first = (c.j == (c.u == part.u0 ? part.j0 : 0));
    const bool last = (c.j + 1 == c.je);
    if (!mbar_wait(&bars.kv_full[s], (t / kStages) & 1, abort_flag, p.wait_ns) ||
        (first && !mbar_wait(bars.q_full, c.seg & 1, abort_flag, p.wait_ns))) {
      ok = false;
      break;
    }
    const int nv = stage_nvalid(info[s]);
    const uint64_t kd = k_desc0 + ((s * kStageBytes) >> 4);
#pragma unroll 1
    for (int i = 0; i < kParts; ++i) {
      FP8_TRACE(16 + 5 * i, t);
      if (!mbar_wait(&bars.slot_empty[ring.slot], ring.phase ^ 1u, abort_flag, p.wait_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (i == 0) FP8_TRACE(3, t);
      if (i == kParts - 1) FP8_TRACE(4, t);
      const uint32_t d = tmem_hi + 64 * ring.slot;
      if (nv > 0) {
        if (i < 4) {
          qk_chunk(d, kd, kColQ + 32 * (2 * i), 2 * i, idesc_qk, true);
          qk_chunk(d, kd, kColQ + 32 * (2 * i + 1), 2 * i + 1, idesc_qk, false);
        } else {
          qk_chunk(d, kd, kColQRope, kRopeChunk, idesc_rope, true);
        }
      }
      umma_commit_elect(&bars.slot_full[ring.slot]);
      FP8_TRACE(17 + 5 * i, t);
      ring.next();
    }
    if (!ok) break;
    umma_commit_elect(&bars.qk_done[s]);     // the codes may now become V'
    // PV of the previous tile, and of this one at the end of its segment
    if (have_prev && !pv_tile(prev_t, prev_seg, prev_nv)) { ok = false; break; }
    have_prev = true;
    prev_t = t;
    prev_seg = c.seg;
    prev_nv = nv;
    if (last) {
      if (!pv_tile(t, c.seg, nv)) { ok = false; break; }
      have_prev = false;
    }
    cursor_next(p, part, c);
  }
  if (ok && have_prev && !pv_tile(prev_t, prev_seg, prev_nv)) ok = false;
  const int lane = threadIdx.x & 31;
  if (!ok && lane == 0) raise_abort(abort_flag, p.err);
  // Wait until every MMA this warp issued has completed.
  umma_commit_elect(bars.done);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bars.done, 0) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
  }
  __syncwarp();
}

// ---------------------------------------------------------------------------
// Warps 2-5: the query tile of a unit into TMEM lanes 16-31.  Thread
// (r, half) owns row r's latent dims [128 c + 64 half, +64) for c = 0..3 and
// RoPE dims [512 + 32 half, +32).  The latent dims are scaled by 2^-e_r (e_r
// from the row's largest |q|, shared by the thread pair) and rounded to f16;
// the RoPE dims are stored as bf16.  Returns 2^e_r.
__device__ __forceinline__ float write_q_tile(const DecodeParams& p, const UnitInfo& ui, uint32_t tq, int r,
                                              int half) {
  const bool valid = r < tile_valid_rows(p);
  const uint4* src = reinterpret_cast<const uint4*>(
      p.q + q_tile_offset(p, ui, static_cast<int>(blockIdx.y) * kRows) + static_cast<int64_t>(r) * kDqk);
  float amax = 0.f;
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint4 x = valid ? __ldg(src + 16 * c + 8 * half + i) : make_uint4(0, 0, 0, 0);
      const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int j = 0; j < 4; ++j)
        amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w[j] << 16)), fabsf(__uint_as_float(w[j] & 0xFFFF0000u))));
    }
  }
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 16));
  // q * 2^-e stays below 2^15 in magnitude
  int e = 0;
  if (amax > 0.f && amax <= 3.4e38f) e = min(max(ilogbf(amax) - 14, -100), 113);
  const float f = ldexpf(1.f, -e);
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    uint4 buf[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) buf[i] = valid ? __ldg(src + 16 * c + 8 * half + i) : make_uint4(0, 0, 0, 0);
    uint32_t v[32];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t w[4] = {buf[i].x, buf[i].y, buf[i].z, buf[i].w};
#pragma unroll
      for (int j = 0; j < 4; ++j)
        v[4 * i + j] = pack_f16x2(__uint_as_float(w[j] << 16) * f, __uint_as_float(w[j] & 0xFFFF0000u) * f);
    }
    tmem_st_16x32bx2_x32u(tq + kColQ + 64 * c, v);
  }
  uint32_t w[16];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 x = valid ? __ldg(src + 64 + 4 * half + i) : make_uint4(0, 0, 0, 0);
    w[4 * i] = x.x; w[4 * i + 1] = x.y; w[4 * i + 2] = x.z; w[4 * i + 3] = x.w;
  }
  tmem_st_16x32bx2_x16(tq + kColQRope, w);
  return ldexpf(1.f, e);
}

// ---------------------------------------------------------------------------
// Warps 2-5: per tile, the logits from the partial sums, the online softmax
// and P; per segment, the epilogue.
__device__ __forceinline__ void softmax_role(const DecodeParams& p, const Partition& part, uint8_t* smem, Bars bars,
                                             uint32_t tmem_base, volatile int* abort_flag) {
  const int lane = threadIdx.x & 31;
  const int q4 = (threadIdx.x >> 5) & 3;            // TMEM lane quadrant of this warp
  const int half = lane >> 4;                        // which half of the row's keys / dims
  const int r = 16 * q4 + (lane & 15);               // tile row of this thread
  const int R = p.rows_per_unit;
  const int grow = blockIdx.y * kRows + r;           // row within the unit
  const bool row_valid = grow < R;
  const bool warp_live = static_cast<int>(blockIdx.y) * kRows + 16 * q4 < R;
  const float scale_log2 = p.scale_log2;
  const int h_q = p.h_q, s_q = p.s_q;
  const int tok_dense = grow / h_q;
  const bool sparse = p.indices != nullptr;
  const bool causal = !sparse && p.causal != 0;
  const StageInfo* info = reinterpret_cast<const StageInfo*>(smem + Smem::info_off);
  const float* scales = reinterpret_cast<const float*>(smem + Smem::scales_off);
  const uint32_t s_taddr = tmem_base + (static_cast<uint32_t>(32 * q4 + 16) << 16);
  const uint32_t o_taddr = tmem_base + (static_cast<uint32_t>(32 * q4) << 16);
  const int key0 = 32 * half;                        // first key (and dim offset) of this thread's half
  const uint32_t tq = s_taddr;                        // query tile: same lanes as the partial sums

  float rho_next = 1.f;
  auto stage_next_q = [&](int u_from) {
    for (int u = u_from; u <= part.u1 && u < p.num_units; ++u) {
      int jb, je;
      if (segment_bounds(p, part, u, jb, je)) {
        rho_next = write_q_tile(p, unit_info(p, u), tq, r, half);
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
  Ring ring;

  for_each_segment(p, part, [&](int u, int jb, int je) -> bool {
    const UnitInfo ui = unit_info(p, u);
    if (!sparse && lane == 0 && q4 == 0 && p.seqlens[ui.b] < 0) atomicOr(p.err, kErrSeqlen);
    const float rho = rho_next;
    float m_run = -INFINITY, l_run = 0.f;
    bool any_pv = false;
    GroupExp gexp;
    gexp.reset();
    const int lim = ui.L - s_q + tok_dense + 1;      // causal: keys t < lim are visible
    for (int j = jb; j < je; ++j) {
      const int s = t % kStages;
      if (!mbar_wait(&bars.kv_full[s], (t / kStages) & 1, abort_flag, p.wait_ns)) { ok = false; return false; }
      // the tile's valid-key count, masks and per-group scale maxima, read
      // while the first parts of QK^T run
      const int nv = stage_nvalid(info[s]);
      const bool work = nv > 0 && warp_live;
      const uint32_t vmask = static_cast<uint32_t>(info[s].mask[4 * half]) |
                             (static_cast<uint32_t>(info[s].mask[4 * half + 1]) << 8) |
                             (static_cast<uint32_t>(info[s].mask[4 * half + 2]) << 16) |
                             (static_cast<uint32_t>(info[s].mask[4 * half + 3]) << 24);
      const float4 gmax = GroupExp::tile_max(info[s]);
      const float* sck = scales + scale_index(s, 0, key0);   // group g of this half's keys: sck[g * kPage + i]
      // the five parts of QK^T, each from its ring slot:
      //   x = (sum_g scale[k][g] * S_g) * 2^e_r + S_rope  (= q.k; the softmax
      //   scale enters with the row max and the exponent)
      float x[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) x[i] = 0.f;
#pragma unroll 1
      for (int i = 0; i < kParts; ++i) {
        if (lane == 0 && q4 == 2) FP8_TRACE(18 + 5 * i, t);
        if (lane == 0 && i == 0) FP8_TRACE(47 + q4, t);
        if (!mbar_wait(&bars.slot_full[ring.slot], ring.phase, abort_flag, p.wait_ns)) { ok = false; return false; }
        tc_fence_after();
        if (lane == 0 && q4 == 2) FP8_TRACE(19 + 5 * i, t);
        if (lane == 0 && q4 == 2 && i == 0) FP8_TRACE(6, t);
        if (lane == 0 && q4 == 2 && i == kParts - 1) FP8_TRACE(8, t);
        float y[32];
        if (work) tmem_ld_16x32bx2_x32(s_taddr + 64 * ring.slot, y);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.slot_empty[ring.slot]);
        if (lane == 0 && i == 0) FP8_TRACE(43 + q4, t);
        ring.next();
        if (work) {
          if (i < 4) {
            const float4* sg = reinterpret_cast<const float4*>(sck + i * kPage);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float4 v = sg[q];
              x[4 * q] = fmaf(y[4 * q], v.x, x[4 * q]);
              x[4 * q + 1] = fmaf(y[4 * q + 1], v.y, x[4 * q + 1]);
              x[4 * q + 2] = fmaf(y[4 * q + 2], v.z, x[4 * q + 2]);
              x[4 * q + 3] = fmaf(y[4 * q + 3], v.w, x[4 * q + 3]);
            }
          } else {
#pragma unroll
            for (int q = 0; q < 32; ++q) x[q] = fmaf(x[q], rho, y[q]);
          }
        }
        if (lane == 0 && q4 == 2 && i == 2) FP8_TRACE(7, t);
        if (lane == 0 && q4 == 2) FP8_TRACE(20 + 5 * i, t);
      }
      if (lane == 0 && q4 == 2) FP8_TRACE(9, t);

      float tmax = -INFINITY;
      if (work) {
        uint32_t m = vmask;
        if (causal && kPage * j + key0 + 31 >= lim) {
          const int nc = min(max(lim - kPage * j - key0, 0), 32);
          m &= nc >= 32 ? 0xFFFFFFFFu : ((1u << nc) - 1u);
        }
        if (m != 0xFFFFFFFFu) {
#pragma unroll
          for (int i = 0; i < 32; ++i) x[i] = ((m >> i) & 1u) ? x[i] : -INFINITY;
        }
        // pairwise, so that the chain is five deep instead of 32
        float mx[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) mx[i] = fmaxf(x[i], x[i + 16]);
#pragma unroll
        for (int w = 8; w >= 1; w >>= 1) {
#pragma unroll
          for (int i = 0; i < w; ++i) mx[i] = fmaxf(mx[i], mx[i + w]);
        }
        tmax = mx[0] * scale_log2;   // log2 units (scale_log2 > 0 keeps the max)
      }
      tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 16));
      const bool need = tmax > m_run + kRescaleThreshold;
      float alpha = 1.f;
      if (__any_sync(0xffffffffu, need)) {
        const float m_new = need ? fmaxf(m_run, tmax) : m_run;
        alpha = (m_new == m_run) ? 1.f : fast_exp2(m_run - m_new);   // m_run = -inf -> 0
        l_run *= alpha;
        m_run = m_new;
      }
      if (lane == 0 && q4 == 2) FP8_TRACE(12, t);
      // group exponents (the same in every thread, and in the gather warps
      // that scale V' with them)
      float4 beta;
      const bool moved = gexp.update(gmax, beta);
      if (lane == 0 && q4 == 2) FP8_TRACE(13, t);
      if (__any_sync(0xffffffffu, any_pv && (alpha != 1.f || moved))) {
        // O holds every PV of the segment once PV(t-1), which frees its
        // stage, has completed (any_pv implies t > 0)
        const int tp = t - 1;
        if (!mbar_wait(&bars.kv_empty[tp % kStages], (tp / kStages) & 1, abort_flag, p.wait_ns)) { ok = false; return false; }
        tc_fence_after();
        if (warp_live) {
#pragma unroll 1
          for (int c0 = 0; c0 < kDv; c0 += 64) {
            const float fct = alpha * pick4(c0 >> 7, beta.x, beta.y, beta.z, beta.w);
            float v[32];
            tmem_ld_16x32bx2_x32(o_taddr + c0, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= fct;
            tmem_st_16x32bx2_x32(o_taddr + c0, v);
          }
        }
      }

      if (lane == 0 && q4 == 2) FP8_TRACE(10, t);
      // P = exp2(s - m) as f16: this thread's 64-B half of row r of the
      // K-major swizzled P tile in the stage's RoPE chunk, whose last reader,
      // the RoPE part of this tile's QK^T, has completed.  (P <= 2^8: the
      // lazy max.)
      const float m_safe = m_run == -INFINITY ? 0.f : m_run;
      uint8_t* stage = stage_ptr(smem, s);
      if (warp_live) {
        uint32_t pk[16];
        if (work) {
          float ps[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float a = fast_exp2(fmaf(x[2 * i], scale_log2, -m_safe));
            const float b = fast_exp2(fmaf(x[2 * i + 1], scale_log2, -m_safe));
            ps[i] = a + b;
            pk[i] = pack_f16x2(a, b);
          }
#pragma unroll
          for (int w = 8; w >= 1; w >>= 1) {
#pragma unroll
            for (int i = 0; i < w; ++i) ps[i] += ps[i + w];
          }
          l_run += ps[0];
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = 0u;
        }
        const uint32_t prow = smem_u32(stage + kRopeChunk * kChunkBytes) + r * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int chunk = 4 * half + c;
          st_shared_v4(prow + ((chunk ^ (r & 7)) << 4),
                       make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]));
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.p_full[s]);
      if (lane == 0) FP8_TRACE(51 + q4, t);
      if (lane == 0 && q4 == 2) FP8_TRACE(11, t);
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
          if (lane == 0 && q4 == 0) atomicOr(p.err, kErrInternal);
          split = false;
        }
#pragma unroll 1
        for (int c0 = 0; c0 < kDv; c0 += 64) {
          float v[32];
          tmem_ld_16x32bx2_x32(o_taddr + c0, v);
          if (!row_valid) continue;
          const float fct = inv * pow2i(gexp.e(c0 >> 7));
          const int d0 = c0 + key0;
          if (split) {
            float4* dst = reinterpret_cast<float4*>(p.ws_o + (static_cast<int64_t>(split_idx) * R + grow) * kDv + d0);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(v[4 * i] * fct, v[4 * i + 1] * fct, v[4 * i + 2] * fct, v[4 * i + 3] * fct);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(p.out + (static_cast<int64_t>(u) * R + grow) * kDv + d0);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(pack_bf16x2(v[8 * i] * fct, v[8 * i + 1] * fct),
                                  pack_bf16x2(v[8 * i + 2] * fct, v[8 * i + 3] * fct),
                                  pack_bf16x2(v[8 * i + 4] * fct, v[8 * i + 5] * fct),
                                  pack_bf16x2(v[8 * i + 6] * fct, v[8 * i + 7] * fct));
          }
        }
        if (row_valid && half == 0) {
          if (split) {
            p.ws_lse[static_cast<int64_t>(split_idx) * R + grow] = lse;
          } else {
            int b, tok, h;
            if (sparse) { b = ui.b; tok = ui.token; h = grow; }
            else { b = ui.b; tok = tok_dense; h = grow % h_q; }
            p.lse[(static_cast<int64_t>(b) * h_q + h) * s_q + tok] = lse;
          }
        }
        tc_fence_before();
      }
      ++t;
    }
    return true;
  });
  if (!ok) raise_abort(abort_flag, p.err);
}

// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 1)
    mla_decode_fp8_kernel(const DecodeParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  FP8_SPAN(0);

  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + Smem::bar_off);
  Bars bars;
  bars.kv_full = bar;
  bars.kv_empty = bar + kStages;
  bars.p_full = bar + 2 * kStages;
  bars.qk_done = bar + 3 * kStages;
  bars.v_ready = bar + 4 * kStages;
  bars.slot_full = bar + 5 * kStages;
  bars.slot_empty = bar + 5 * kStages + kSlots;
  bars.q_full = bar + 5 * kStages + 2 * kSlots;
  bars.done = bar + 5 * kStages + 2 * kSlots + 1;
  StageInfo* info = reinterpret_cast<StageInfo*>(smem + Smem::info_off);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Smem::misc_off);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Smem::misc_off + 4);

  const bool misaligned = (smem_u32(smem) & 1023u) != 0;
  if (threadIdx.x == 0) {
    *abort_flag = misaligned ? 1 : 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars.kv_full[s], kGatherWarps);
      mbar_init(&bars.kv_empty[s], 1);
      mbar_init(&bars.p_full[s], 4);
      mbar_init(&bars.qk_done[s], 1);
      mbar_init(&bars.v_ready[s], kRewriteWarps);
      for (int w = 0; w < kGatherWarps; ++w) {
        info[s].mask[w] = 0;
        info[s].gmax[w] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    for (int r = 0; r < kSlots; ++r) {
      mbar_init(&bars.slot_full[r], 1);
      mbar_init(&bars.slot_empty[r], 4);
    }
    mbar_init(bars.q_full, 4);
    mbar_init(bars.done, 1);
    fence_barrier_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  grid_dependency_wait();
  grid_launch_dependents();
  if (misaligned && threadIdx.x == 0) atomicOr(p.err, kErrInternal);
  const uint32_t tmem_base = *tmem_slot;
  const Partition part = load_partition(p, blockIdx.x);
  if (threadIdx.x == 0) FP8_TRACE(15, 0);
  FP8_SPAN(1);

  if (!*abort_flag) {
    if (warp == kWarpQPrefetch) {
      if (lane == 0) q_prefetch_role(p, part);
    } else if (warp == kWarpMma) {
      mma_role(p, part, smem, bars, tmem_base, abort_flag);
    } else if (warp >= kWarpSoftmax0 && warp < kWarpGather0) {
      softmax_role(p, part, smem, bars, tmem_base, abort_flag);
    } else {
      gather_role(p, part, smem, bars, abort_flag, warp - kWarpGather0);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) FP8_TRACE(15, 1);
  FP8_SPAN(2);
  tc_fence_after();
  if (warp == kWarpMma) {
    __syncwarp();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

#ifdef MLA_TRACE
extern "C" __attribute__((visibility("default"))) int mla_trace_fp8_copy(void* host_dst, size_t bytes) {
  if (bytes > sizeof(g_fp8_trace)) bytes = sizeof(g_fp8_trace);
  return cudaMemcpyFromSymbol(host_dst, g_fp8_trace, bytes) == cudaSuccess ? 0 : 4;
}
extern "C" __attribute__((visibility("default"))) int mla_trace_fp8_span_copy(void* host_dst, size_t bytes) {
  if (bytes > sizeof(g_fp8_span)) bytes = sizeof(g_fp8_span);
  return cudaMemcpyFromSymbol(host_dst, g_fp8_span, bytes) == cudaSuccess ? 0 : 4;
}
#endif

cudaError_t launch_decode_fp8(const DecodeParams& p, int row_tiles, cudaStream_t stream) {
  constexpr int smem = Smem::total;
  static unsigned long long configured = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(__atomic_load_n(&configured, __ATOMIC_ACQUIRE) & bit)) {
    e = cudaFuncSetAttribute(mla_decode_fp8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    __atomic_fetch_or(&configured, bit, __ATOMIC_RELEASE);
  }
  // The row tiles of a partition read the same rows: as one cluster they
  // share a GPC and its side of L2.  Only when every cluster fits at once.
  static int fits[64] = {};
  unsigned cy = 1;
  if (row_tiles == 2 && dev >= 0 && dev < 64) {
    if (fits[dev] == 0) {
      cudaLaunchConfig_t q = {};
      q.gridDim = dim3(p.num_parts, row_tiles);
      q.blockDim = dim3(kThreads);
      q.dynamicSmemBytes = smem;
      cudaLaunchAttribute a[1];
      a[0].id = cudaLaunchAttributeClusterDimension;
      a[0].val.clusterDim.x = 1;
      a[0].val.clusterDim.y = 2;
      a[0].val.clusterDim.z = 1;
      q.attrs = a;
      q.numAttrs = 1;
      int clusters = 0;
      fits[dev] = (cudaOccupancyMaxActiveClusters(&clusters, mla_decode_fp8_kernel, &q) == cudaSuccess) ? clusters : -1;
    }
    if (fits[dev] >= p.num_parts) cy = 2;
  }
  return launch_dependent_cluster(mla_decode_fp8_kernel, dim3(p.num_parts, row_tiles), dim3(kThreads), smem, cy,
                                  stream, p);
}

}  // namespace mla
