// Split-KV tile-scheduler metadata ("Was ist FlashMLA?", section
// "2. MLA-Metadaten abrufen": computed once per decode step, reused by every
// layer).  The pages give the call, not the algorithm; the plan here is this
// library's own:
//
//   unit u (a sequence, or a (sequence, token) pair on the sparse path) has
//   n_u pages and costs c_u = n_u + kFixedSplitCost (0 if n_u == 0);
//   boundary p of P partitions sits at cost position x_p = floor(p*T/P),
//   which maps to (unit, page) = (u, max(0, x - C_u - kFixedSplitCost)) for
//   the unit whose cost interval [C_u, C_u + c_u) holds x, and to (U, 0) at
//   x = T.
//
// One CTA computes it in parallel: a block scan of the costs, a binary search
// per boundary, and two scans that turn the distinct interior cut points into
// split counts and split indices.
#include "mla_kernels.cuh"
#include "ptx_sm100.cuh"

namespace mla {
namespace {

constexpr int kMdThreads = 512;

__device__ __forceinline__ int unit_pages(const int* seqlens, int u, int s_q, int topk) {
  if (topk > 0) return (topk + kPage - 1) / kPage;
  const int L = seqlens[u];
  return L > 0 ? (L + kPage - 1) / kPage : 0;
}

// Block-wide exclusive scan of one value per thread; also returns the total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* buf, int& total) {
  const int tid = threadIdx.x;
  buf[tid] = v;
  __syncthreads();
  for (int off = 1; off < kMdThreads; off <<= 1) {
    int add = tid >= off ? buf[tid - off] : 0;
    __syncthreads();
    buf[tid] += add;
    __syncthreads();
  }
  total = buf[kMdThreads - 1];
  const int incl = buf[tid];
  __syncthreads();
  return incl - v;
}

__global__ void __launch_bounds__(kMdThreads, 1)
    metadata_kernel(const int* __restrict__ seqlens, int s_q, int topk, int U, int P, int* __restrict__ md,
                    int* __restrict__ ns) {
  __shared__ int buf[kMdThreads];
  const int tid = threadIdx.x;
  grid_dependency_wait();        // the previous decode may still read num_splits
  grid_launch_dependents();

  // 1. exclusive prefix of unit costs -> ns[0..U-1] (temporarily), ns[U] = T.
  int carry = 0;
  for (int base = 0; base < U; base += kMdThreads) {
    const int u = base + tid;
    const int n = u < U ? unit_pages(seqlens, u, s_q, topk) : 0;
    const int c = n > 0 ? n + kFixedSplitCost : 0;
    int chunk_total;
    const int ex = block_exclusive_scan(c, buf, chunk_total);
    if (u < U) ns[u] = carry + ex;
    carry += chunk_total;
  }
  if (tid == 0) ns[U] = carry;
  __syncthreads();
  const long long T = carry;

  // 2. boundaries: begin of partition p in md[p][0..1], end in md[p-1][2..3].
  for (int p = tid; p <= P; p += kMdThreads) {
    const long long x = (static_cast<long long>(p) * T) / P;
    int bu = U, bj = 0;
    if (x < T) {
      int lo = 0, hi = U - 1;  // largest u with ns[u] <= x
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (static_cast<long long>(ns[mid]) <= x) lo = mid; else hi = mid - 1;
      }
      bu = lo;
      const long long j = x - ns[lo] - kFixedSplitCost;
      bj = j > 0 ? static_cast<int>(j) : 0;
    }
    if (p < P) { md[p * kMdWords + 0] = bu; md[p * kMdWords + 1] = bj; }
    if (p > 0) { md[(p - 1) * kMdWords + 2] = bu; md[(p - 1) * kMdWords + 3] = bj; }
  }
  __syncthreads();

  // 3. flag distinct interior cut points; inclusive prefix F_p -> md[p][5].
  carry = 0;
  for (int base = 0; base < P; base += kMdThreads) {
    const int p = base + tid;
    int flag = 0;
    if (p >= 1 && p < P) {
      const int u = md[p * kMdWords + 0], j = md[p * kMdWords + 1];
      const int pu = md[(p - 1) * kMdWords + 0], pj = md[(p - 1) * kMdWords + 1];
      flag = (u < U && j > 0 && (u != pu || j != pj)) ? 1 : 0;
    }
    int chunk_total;
    const int ex = block_exclusive_scan(flag, buf, chunk_total);
    if (p < P) md[p * kMdWords + 5] = carry + ex + flag;
    carry += chunk_total;
  }
  __syncthreads();

  // 4. num_splits[u] = (non-empty units before u) + (cut flags of units before u).
  //    Cuts of units < u sit at partitions p < lb(u) = first p with u_p >= u.
  int ne_carry = 0;
  for (int base = 0; base <= U; base += kMdThreads) {
    const int u = base + tid;
    const int nonempty = (u < U && unit_pages(seqlens, u, s_q, topk) > 0) ? 1 : 0;
    int chunk_total;
    const int ne_before = ne_carry + block_exclusive_scan(nonempty, buf, chunk_total);
    ne_carry += chunk_total;
    if (u <= U) {
      int lo = 0, hi = P;  // first p in [0, P] with u_p >= u (u_P is U)
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        const int um = mid < P ? md[mid * kMdWords + 0] : U;
        if (um >= u) hi = mid; else lo = mid + 1;
      }
      const int cuts_before = lo > 0 ? md[(lo - 1) * kMdWords + 5] : 0;
      ns[u] = ne_before + cuts_before;
    }
    __syncthreads();
  }
  __syncthreads();

  // 5. first split index of each partition: NE(u_p) + F_p, i.e.
  //    ns[u_p] - (cuts of units before u_p) + F_p.
  for (int p = tid; p < P; p += kMdThreads) {
    const int u = md[p * kMdWords + 0];
    int first;
    if (u >= U) {
      first = ns[U];
    } else {
      int lo = 0, hi = P;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        const int um = mid < P ? md[mid * kMdWords + 0] : U;
        if (um >= u) hi = mid; else lo = mid + 1;
      }
      const int cuts_before = lo > 0 ? md[(lo - 1) * kMdWords + 5] : 0;
      first = ns[u] - cuts_before + md[p * kMdWords + 5];
    }
    md[p * kMdWords + 4] = first;
  }
  __syncthreads();
  for (int p = tid; p < P; p += kMdThreads) {
    md[p * kMdWords + 5] = 0;
    md[p * kMdWords + 6] = 0;
    md[p * kMdWords + 7] = 0;
  }
}

// Shared-memory variant for plans whose arrays fit on chip (the common case):
// the same plan, with the prefix arrays and boundaries kept in shared memory
// and warp-shuffle scans, so the binary searches never touch global memory.
constexpr int kMdFastThreads = 1024;
constexpr int kMdFastMaxInts = 48 * 1024;   // 192 KB of shared memory

// Exclusive block scan of one value per thread (kMdFastThreads threads);
// returns the exclusive prefix and the block total.
__device__ __forceinline__ int block_scan_fast(int v, int* warp_sums, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sums[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, off);
      if (lane >= off) w += y;
    }
    warp_sums[lane] = w;
  }
  __syncthreads();
  const int before = warp > 0 ? warp_sums[warp - 1] : 0;
  total = warp_sums[31];
  __syncthreads();
  return before + x - v;
}

__global__ void __launch_bounds__(kMdFastThreads, 1)
    metadata_smem_kernel(const int* __restrict__ seqlens, int s_q, int topk, int U, int P, int* __restrict__ md,
                         int* __restrict__ ns) {
  extern __shared__ int sh[];
  __shared__ int warp_sums[32];
  int* C = sh;                 // [U + 1] exclusive cost prefix
  int* NE = C + (U + 1);       // [U + 1] non-empty units before u
  int* bu = NE + (U + 1);      // [P + 1] boundary unit
  int* bj = bu + (P + 1);      // [P + 1] boundary page
  int* F = bj + (P + 1);       // [P + 1] inclusive prefix of cut flags
  const int tid = threadIdx.x;
  grid_dependency_wait();        // the previous decode may still read num_splits
  grid_launch_dependents();

  int carry_c = 0, carry_n = 0;
  for (int base = 0; base < U; base += kMdFastThreads) {
    const int u = base + tid;
    const int n = u < U ? unit_pages(seqlens, u, s_q, topk) : 0;
    int tc, tn;
    const int ec = block_scan_fast(n > 0 ? n + kFixedSplitCost : 0, warp_sums, tc);
    const int en = block_scan_fast(n > 0 ? 1 : 0, warp_sums, tn);
    if (u < U) { C[u] = carry_c + ec; NE[u] = carry_n + en; }
    carry_c += tc;
    carry_n += tn;
  }
  if (tid == 0) { C[U] = carry_c; NE[U] = carry_n; }
  __syncthreads();
  const long long T = carry_c;

  for (int p = tid; p <= P; p += kMdFastThreads) {
    const long long x = (static_cast<long long>(p) * T) / P;
    int b_u = U, b_j = 0;
    if (x < T) {
      int lo = 0, hi = U - 1;  // largest u with C[u] <= x
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (static_cast<long long>(C[mid]) <= x) lo = mid; else hi = mid - 1;
      }
      b_u = lo;
      const long long j = x - C[lo] - kFixedSplitCost;
      b_j = j > 0 ? static_cast<int>(j) : 0;
    }
    bu[p] = b_u;
    bj[p] = b_j;
  }
  __syncthreads();

  int carry = 0;
  for (int base = 0; base < P; base += kMdFastThreads) {
    const int p = base + tid;
    int flag = 0;
    if (p >= 1 && p < P) flag = (bu[p] < U && bj[p] > 0 && (bu[p] != bu[p - 1] || bj[p] != bj[p - 1])) ? 1 : 0;
    int tf;
    const int ef = block_scan_fast(flag, warp_sums, tf);
    if (p < P) F[p] = carry + ef + flag;
    carry += tf;
  }
  __syncthreads();

  // num_splits[u] = NE(u) + (cut flags of units before u)
  for (int u = tid; u <= U; u += kMdFastThreads) {
    int lo = 0, hi = P;  // first p in [0, P] with bu[p] >= u
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (bu[mid] >= u) hi = mid; else lo = mid + 1;
    }
    ns[u] = NE[u] + (lo > 0 ? F[lo - 1] : 0);
  }
  for (int p = tid; p < P; p += kMdFastThreads) {
    const int u = bu[p];
    int* row = md + p * kMdWords;
    row[0] = u;
    row[1] = bj[p];
    row[2] = bu[p + 1];
    row[3] = bj[p + 1];
    row[4] = u < U ? NE[u] + F[p] : NE[U] + F[P - 1];
    row[5] = 0;
    row[6] = 0;
    row[7] = 0;
  }
}

}  // namespace

cudaError_t launch_metadata(const int* seqlens, int batch, int s_q, int topk, int num_units, int num_parts,
                            int* tile_md, int* num_splits, int* err, cudaStream_t stream) {
  (void)batch;
  (void)err;
  const long long ints = 2LL * (num_units + 1) + 3LL * (num_parts + 1);
  if (ints <= kMdFastMaxInts) {
    const size_t bytes = static_cast<size_t>(ints) * sizeof(int);
    if (bytes > 48 * 1024) {
      static unsigned long long configured = 0;
      int dev = 0;
      cudaError_t e = cudaGetDevice(&dev);
      if (e != cudaSuccess) return e;
      const unsigned long long bit = 1ull << (dev & 63);
      if (!(__atomic_load_n(&configured, __ATOMIC_ACQUIRE) & bit)) {
        e = cudaFuncSetAttribute(metadata_smem_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kMdFastMaxInts * static_cast<int>(sizeof(int)));
        if (e != cudaSuccess) return e;
        __atomic_fetch_or(&configured, bit, __ATOMIC_RELEASE);
      }
    }
    return launch_dependent(metadata_smem_kernel, dim3(1), dim3(kMdFastThreads), bytes, stream, seqlens, s_q, topk,
                            num_units, num_parts, tile_md, num_splits);
  }
  return launch_dependent(metadata_kernel, dim3(1), dim3(kMdThreads), 0, stream, seqlens, s_q, topk, num_units,
                          num_parts, tile_md, num_splits);
}

}  // namespace mla
