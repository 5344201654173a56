// Round-level selection and extraction over a given CSR.
//
// Round Attention page ("方法详解"): in a multi-turn context, the attention of
// a watershed layer decides, per conversation round, which earlier rounds
// matter; the kept rounds then serve the later layers.  Here that decision is
// a second selection policy over the block cache: rounds start on block
// boundaries, a query round keeps its own blocks plus the fewest earlier
// rounds, heaviest first (ties to the lower round), whose mass with its own
// reaches tau * T.  The round masses are sums of the watershed layer's block
// masses (fp64, in a fixed order).  Every query block of a round keeps the
// blocks of the kept rounds up to its own position.  mf_extract then writes
// the probability blocks of any CSR (this one, or another layer's) for a
// layer's own Q, K and lse.
#include <algorithm>

#include "mf_device.cuh"
#include "mf_internal.h"

namespace mf {

constexpr int kRoundThreads = 256;
constexpr int kMaxRoundsPerSeq = 512;  // a round holds at least one block

// Sequence of every round and the first round of every sequence.
__global__ void k_round_meta(int nseq, const int32_t* __restrict__ cu_seqlens, int nrounds,
                             const int32_t* __restrict__ starts, int32_t* __restrict__ r_seq,
                             int32_t* __restrict__ r_first) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  int s = 0;
  for (int r = 0; r < nrounds; ++r) {
    while (s + 1 < nseq && cu_seqlens[s + 1] <= starts[r]) ++s;
    r_seq[r] = s;
  }
  int r = 0;
  for (int q = 0; q <= nseq; ++q) {
    while (r < nrounds && r_seq[r] < q) ++r;
    r_first[q] = r;
  }
}

// First key block of round r within its sequence, and past its last block.
__device__ __forceinline__ int round_b0(const int32_t* starts, int r, int seq0, int B) {
  return (starts[r] - seq0) / B;
}
__device__ __forceinline__ int round_b1(const int32_t* starts, int r, int seq0, int B) {
  return (starts[r + 1] - seq0 + B - 1) / B;
}

// One CTA per query round: round masses, order, cut, keep flags and the row
// counts of the round's query blocks.
__global__ void __launch_bounds__(kRoundThreads) k_select_rounds(
    const float* __restrict__ mass, const int64_t* __restrict__ cu_blk,
    const int32_t* __restrict__ cu_qb, const int32_t* __restrict__ cu_seqlens,
    const int32_t* __restrict__ starts, const int32_t* __restrict__ r_seq,
    const int32_t* __restrict__ r_first, int B, double tau, int max_r,
    uint8_t* __restrict__ flags, int32_t* __restrict__ counts) {
  __shared__ double mv[kMaxRoundsPerSeq];
  __shared__ int kv[kMaxRoundsPerSeq];
  __shared__ uint8_t keep[kMaxRoundsPerSeq];
  const int rq = blockIdx.x, tid = threadIdx.x;
  const int s = r_seq[rq];
  const int f = r_first[s];
  const int q = rq - f;  // local index of the query round
  const int seq0 = cu_seqlens[s];
  const int qb0 = round_b0(starts, rq, seq0, B), qb1 = round_b1(starts, rq, seq0, B);
  const int64_t cb = cu_blk[s];
  // mass of key round r: block masses of the round's query blocks over the
  // key round's blocks (causal), summed in float64 query block by query block
  for (int r = tid; r <= q; r += kRoundThreads) {
    const int kb0 = round_b0(starts, f + r, seq0, B), kb1 = round_b1(starts, f + r, seq0, B);
    double m = 0.0;
    for (int qb = qb0; qb < qb1; ++qb) {
      const int64_t row = cb + int64_t(qb) * (qb + 1) / 2;
      for (int kb = kb0; kb < min(kb1, qb + 1); ++kb) m += double(mass[row + kb]);
    }
    mv[r] = m;
    kv[r] = r;
    keep[r] = 0;
  }
  // bitonic sort of the earlier rounds 0..q-1: mass descending, index ascending
  int n2 = 1;
  while (n2 < q) n2 <<= 1;
  for (int t = q + tid; t < n2; t += kRoundThreads) {
    if (t == q) continue;  // mv[q] is the own round: keep it in place
    mv[t] = -1.0;          // masses are >= 0: padding sorts last
    kv[t] = t;
  }
  __syncthreads();
  double own = mv[q];
  __syncthreads();
  if (q < n2 && tid == 0) {
    // the own round's slot joins the sort as padding; its mass is kept in `own`
    mv[q] = -1.0;
    kv[q] = q;
  }
  __syncthreads();
  for (int k = 2; k <= n2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int t = tid; t < n2; t += kRoundThreads) {
        const int u = t ^ j;
        if (u > t) {
          const bool up = (t & k) == 0;
          const bool t_first = mv[t] > mv[u] || (mv[t] == mv[u] && kv[t] < kv[u]);
          if (up != t_first) {
            const double fm = mv[t]; mv[t] = mv[u]; mv[u] = fm;
            const int fi = kv[t]; kv[t] = kv[u]; kv[u] = fi;
          }
        }
      }
      __syncthreads();
    }
  }
  __shared__ int kstar_s;
  if (tid == 0) {
    int kstar = q;
    if (tau < 1.0) {
      double T = own;
      for (int k = 0; k < q; ++k) T += mv[k];
      double c = own;
      kstar = 0;
      while (c < tau * T && kstar < q) c += mv[kstar++];
    }
    kstar_s = kstar;
  }
  __syncthreads();
  for (int t = tid; t < kstar_s; t += kRoundThreads)
    if (kv[t] < q) keep[kv[t]] = 1;
  if (tid == 0) keep[q] = 1;
  __syncthreads();
  uint8_t* fl = flags + int64_t(rq) * max_r;
  for (int r = tid; r <= q; r += kRoundThreads) fl[r] = keep[r];
  // row counts: every block of a kept earlier round, and the own round up to qb
  __shared__ int before;
  if (tid == 0) {
    int n = 0;
    for (int r = 0; r < q; ++r)
      if (keep[r])
        n += round_b1(starts, f + r, seq0, B) - round_b0(starts, f + r, seq0, B);
    before = n;
  }
  __syncthreads();
  for (int qb = qb0 + tid; qb < qb1; qb += kRoundThreads)
    counts[cu_qb[s] + qb] = before + (qb - qb0 + 1);
}

// CSR columns of every query block: the kept rounds' blocks up to its own.
__global__ void k_round_fill(const int64_t* __restrict__ row_ptr, const int32_t* __restrict__ qb_seq,
                             const int32_t* __restrict__ qb_idx,
                             const int32_t* __restrict__ cu_seqlens,
                             const int32_t* __restrict__ starts,
                             const int32_t* __restrict__ r_first,
                             const uint8_t* __restrict__ flags, int B, int max_r,
                             int64_t capacity, int32_t* __restrict__ col_idx, unsigned* status) {
  const int64_t g = blockIdx.x;
  if (threadIdx.x != 0) return;
  const int s = qb_seq[g], qb = qb_idx[g];
  const int seq0 = cu_seqlens[s];
  const int f = r_first[s], nr = r_first[s + 1] - f;
  // the query round: the last round starting at or before the block
  int q = 0;
  while (q + 1 < nr && starts[f + q + 1] - seq0 <= qb * B) ++q;
  const uint8_t* fl = flags + int64_t(f + q) * max_r;
  int64_t e = row_ptr[g];
  bool over = false;
  int r = 0;
  for (int kb = 0; kb <= qb; ++kb) {
    while (r + 1 < nr && starts[f + r + 1] - seq0 <= kb * B) ++r;
    if (fl[r]) {
      if (e < capacity) col_idx[e] = kb; else over = true;
      ++e;
    }
  }
  if (over) atomicOr(status, kStatusCapacity);
}

// Block -> cache entry map of a CSR (-1 elsewhere, set by the caller's memset).
__global__ void k_csr_slots(const int64_t* __restrict__ row_ptr, const int32_t* __restrict__ col_idx,
                            const int32_t* __restrict__ qb_seq, const int32_t* __restrict__ qb_idx,
                            const int64_t* __restrict__ cu_blk, int64_t nqb, int64_t capacity,
                            int32_t* __restrict__ slot, unsigned* status) {
  const int64_t g = blockIdx.x;
  if (g >= nqb) return;
  const int s = qb_seq[g], qb = qb_idx[g];
  const int64_t row = cu_blk[s] + int64_t(qb) * (qb + 1) / 2;
  const int64_t e0 = row_ptr[g], e1 = min(row_ptr[g + 1], capacity);
  for (int64_t e = e0 + threadIdx.x; e < e1; e += blockDim.x) {
    const int kb = col_idx[e];
    if (kb < 0 || kb > qb) {  // not a causal block of this query block
      atomicOr(status, kStatusBadCache);
      continue;
    }
    slot[row + kb] = int32_t(e);
  }
}

cudaError_t launch_select_rounds(const mf_attn_desc& d, const Sizes& sz, const Meta& m,
                                 const float* mass, int nrounds, const int32_t* starts,
                                 int max_r, double tau, const mf_csr_cache& c,
                                 int32_t* r_seq, int32_t* r_first, uint8_t* flags,
                                 int32_t* counts, cudaStream_t st) {
  if (sz.nqb == 0 || nrounds == 0) return cudaSuccess;
  k_round_meta<<<1, 32, 0, st>>>(d.nseq, d.cu_seqlens, nrounds, starts, r_seq, r_first);
  int g = int(std::min<int64_t>((sz.nqb + 255) / 256, 1024));
  launch_qb_map(sz.nqb, d.nseq, m.cu_qb, c.qb_seq, c.qb_idx, g, st);
  k_select_rounds<<<unsigned(nrounds), kRoundThreads, 0, st>>>(
      mass, m.cu_blk, m.cu_qb, d.cu_seqlens, starts, r_seq, r_first, d.B, tau, max_r, flags,
      counts);
  launch_scan(counts, sz.nqb, c.row_ptr, st);
  k_round_fill<<<unsigned(sz.nqb), 32, 0, st>>>(c.row_ptr, c.qb_seq, c.qb_idx, d.cu_seqlens,
                                                starts, r_first, flags, d.B, max_r,
                                                c.nnz_capacity, c.col_idx, status_word());
  return cudaGetLastError();
}

cudaError_t launch_csr_slots(const Sizes& sz, const Meta& m, const mf_csr_cache& c,
                             int32_t* slot, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(slot, 0xff, sizeof(int32_t) * size_t(sz.nblocks), st);
  if (e != cudaSuccess || sz.nqb == 0) return e;
  k_csr_slots<<<unsigned(sz.nqb), 128, 0, st>>>(c.row_ptr, c.col_idx, c.qb_seq, c.qb_idx,
                                                m.cu_blk, sz.nqb, c.nnz_capacity, slot,
                                                status_word());
  return cudaGetLastError();
}

}  // namespace mf
