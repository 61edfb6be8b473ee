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

}  // namespace

cudaError_t launch_metadata(const int* seqlens, int batch, int s_q, int topk, int num_units, int num_parts,
                            int* tile_md, int* num_splits, int* err, cudaStream_t stream) {
  (void)batch;
  (void)err;
  metadata_kernel<<<1, kMdThreads, 0, stream>>>(seqlens, s_q, topk, num_units, num_parts, tile_md, num_splits);
  return cudaGetLastError();
}

}  // namespace mla
