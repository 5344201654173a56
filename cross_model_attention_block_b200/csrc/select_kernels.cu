// Selection of kept blocks and CSR assembly (MapFlow article, 163.com, section
// on the three system components: blocks are kept by cumulative attention
// probability; the number kept varies per layer and position).
//
// Per query block: order the key blocks by mass descending with ties to the
// lower index (bitonic sort in shared memory), take float64 prefix sums in that
// order, keep the shortest prefix whose sum reaches tau * total.  Counts are
// scanned into row pointers; kept key blocks are written ascending.
#include <algorithm>

#include "mf_device.cuh"
#include "mf_internal.h"

namespace mf {

constexpr int kSelThreads = 256;
constexpr int kSelMax = 512;  // key blocks per query block

__global__ void k_qb_map(int64_t nqb, int nseq, const int32_t* __restrict__ cu_qb,
                         int32_t* __restrict__ qb_seq, int32_t* __restrict__ qb_idx) {
  for (int64_t g = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; g < nqb;
       g += int64_t(gridDim.x) * blockDim.x) {
    int s = upper_index(cu_qb, nseq, g);
    qb_seq[g] = s;
    qb_idx[g] = int(g - cu_qb[s]);
  }
}

// a precedes b: larger mass first, then lower index
__device__ __forceinline__ bool precedes(float ma, int ia, float mb, int ib) {
  return ma > mb || (ma == mb && ia < ib);
}

__global__ void __launch_bounds__(kSelThreads) k_select(
    const float* __restrict__ mass, const int64_t* __restrict__ cu_blk,
    const int32_t* __restrict__ qb_seq, const int32_t* __restrict__ qb_idx, double tau,
    int64_t qb_lo, int32_t* __restrict__ counts, uint8_t* __restrict__ keep) {
  __shared__ float mv[kSelMax];
  __shared__ int kv[kSelMax];
  __shared__ int kstar_s;
  const int64_t gqb = qb_lo + blockIdx.x;
  const int tid = threadIdx.x;
  const int s = qb_seq[gqb], qb = qb_idx[gqb];
  const int n = qb + 1;
  const int64_t blk0 = cu_blk[s] + int64_t(qb) * (qb + 1) / 2;
  int n2 = 1;
  while (n2 < n) n2 <<= 1;
  for (int t = tid; t < n2; t += kSelThreads) {
    mv[t] = t < n ? mass[blk0 + t] : -1.0f;  // masses are >= 0: padding sorts last
    kv[t] = t;
  }
  __syncthreads();
  for (int k = 2; k <= n2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int t = tid; t < n2; t += kSelThreads) {
        int u = t ^ j;
        if (u > t) {
          bool up = (t & k) == 0;  // this pair ends in "precedes" order
          bool t_first = precedes(mv[t], kv[t], mv[u], kv[u]);
          if (up != t_first) {
            float fm = mv[t]; mv[t] = mv[u]; mv[u] = fm;
            int fi = kv[t]; kv[t] = kv[u]; kv[u] = fi;
          }
        }
      }
      __syncthreads();
    }
  }
  if (tid == 0) {
    int kstar = n;
    if (tau < 1.0) {
      double T = 0.0;
      for (int k = 0; k < n; ++k) T += double(mv[k]);
      double c = 0.0;
      for (int k = 0; k < n; ++k) {
        c += double(mv[k]);
        if (c >= tau * T) { kstar = k + 1; break; }
      }
    }
    kstar_s = kstar;
    counts[gqb] = kstar;
  }
  __syncthreads();
  // (a NaN mass could leave padding among the first n entries: never index with it)
  for (int t = tid; t < n; t += kSelThreads)
    if (kv[t] < n) keep[blk0 + kv[t]] = uint8_t(t < kstar_s ? 1 : 0);
}

// Exclusive scan of counts into row_ptr (int64), one CTA.
__global__ void __launch_bounds__(1024) k_scan(const int32_t* __restrict__ counts, int64_t n,
                                               int64_t* __restrict__ row_ptr) {
  __shared__ int64_t part[1024];
  const int tid = threadIdx.x;
  const int64_t chunk = (n + 1023) / 1024;
  const int64_t lo = min(n, tid * chunk), hi = min(n, lo + chunk);
  int64_t sum = 0;
  for (int64_t i = lo; i < hi; ++i) sum += counts[i];
  part[tid] = sum;
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {
    int64_t v = tid >= off ? part[tid - off] : 0;
    __syncthreads();
    part[tid] += v;
    __syncthreads();
  }
  int64_t run = part[tid] - sum;  // exclusive prefix of this chunk
  for (int64_t i = lo; i < hi; ++i) {
    row_ptr[i] = run;
    run += counts[i];
  }
  if (tid == 1023) row_ptr[n] = part[1023];
}

// Ascending column indices and the block -> entry map (-1 when not kept).
__global__ void k_fill(const int64_t* __restrict__ row_ptr, const uint8_t* __restrict__ keep,
                       const int64_t* __restrict__ cu_blk, const int32_t* __restrict__ qb_seq,
                       const int32_t* __restrict__ qb_idx, int64_t capacity, int64_t qb_lo,
                       int32_t* __restrict__ col_idx, int32_t* __restrict__ slot,
                       unsigned* status) {
  const int64_t gqb = qb_lo + blockIdx.x;
  if (threadIdx.x != 0) return;
  const int s = qb_seq[gqb], qb = qb_idx[gqb];
  const int64_t blk0 = cu_blk[s] + int64_t(qb) * (qb + 1) / 2;
  int64_t e = row_ptr[gqb];
  bool over = false;
  for (int kb = 0; kb <= qb; ++kb) {
    int32_t sl = -1;
    if (keep[blk0 + kb]) {
      if (e < capacity) {
        col_idx[e] = kb;
        sl = int32_t(e);
      } else {
        over = true;
      }
      ++e;
    }
    slot[blk0 + kb] = sl;
  }
  if (over) atomicOr(status, kStatusCapacity);
}

void launch_qb_map(int64_t nqb, int nseq, const int32_t* cu_qb, int32_t* qb_seq,
                   int32_t* qb_idx, int grid, cudaStream_t st) {
  k_qb_map<<<grid, 256, 0, st>>>(nqb, nseq, cu_qb, qb_seq, qb_idx);
}

void launch_scan(const int32_t* counts, int64_t n, int64_t* row_ptr, cudaStream_t st) {
  k_scan<<<1, 1024, 0, st>>>(counts, n, row_ptr);
}

cudaError_t launch_select(const mf_attn_desc& d, const Sizes& sz, const QbRange& r,
                          const Meta& m, const float* mass, double tau, const mf_csr_cache& c,
                          int32_t* counts, uint8_t* keep, int32_t* slot, cudaStream_t st) {
  if (sz.nqb == 0) return cudaSuccess;
  int g = int(std::min<int64_t>((sz.nqb + 255) / 256, 1024));
  k_qb_map<<<g, 256, 0, st>>>(sz.nqb, d.nseq, m.cu_qb, c.qb_seq, c.qb_idx);
  const unsigned n = unsigned(r.qb_hi - r.qb_lo);
  if (n < sz.nqb) {  // rows outside the range stay empty
    cudaError_t e = cudaMemsetAsync(counts, 0, sizeof(int32_t) * size_t(sz.nqb), st);
    if (e != cudaSuccess) return e;
  }
  if (n > 0)
    k_select<<<n, kSelThreads, 0, st>>>(mass, m.cu_blk, c.qb_seq, c.qb_idx, tau, r.qb_lo,
                                        counts, keep);
  k_scan<<<1, 1024, 0, st>>>(counts, sz.nqb, c.row_ptr);
  if (n > 0)
    k_fill<<<n, 32, 0, st>>>(c.row_ptr, keep, m.cu_blk, c.qb_seq, c.qb_idx, c.nnz_capacity,
                             r.qb_lo, c.col_idx, slot, status_word());
  return cudaGetLastError();
}

}  // namespace mf
