// Scalar (CUDA-core, fp32 arithmetic) kernels of the MapFlow path.
//
// These are the float32 path of the library (the bf16 tensor-core kernels
// cannot meet a 1e-4 relative error bound) and serve every shape the
// tensor-core kernels do not cover.  One thread owns one query row.
//
// Definitions follow the MapFlow article (163.com, section on the three system
// components): block statistics of the causal attention map computed without
// the dense matrix, extraction of the kept blocks, and the fused head mix
// multiplied into the receiver's V.
#include <cuda_bf16.h>
#include <math_constants.h>

#include <algorithm>

#include "mf_device.cuh"
#include "mf_internal.h"

namespace mf {

// ---------------------------------------------------------------- metadata

__global__ void k_meta(int nseq, const int32_t* __restrict__ cu_seqlens, int B, int64_t qb_lo,
                       int64_t qb_hi, int32_t* cu_qb, int64_t* cu_blk, int32_t* cu_tile,
                       int32_t* tiles) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  int32_t q = 0, t = 0, tmax = 0;
  int64_t b = 0;
  cu_qb[0] = 0;
  cu_blk[0] = 0;
  cu_tile[0] = 0;
  for (int s = 0; s < nseq; ++s) {
    int L = cu_seqlens[s + 1] - cu_seqlens[s];
    int n = (L + B - 1) / B;
    int nt = (L + 127) / 128;
    q += n;
    b += int64_t(n) * (n + 1) / 2;
    t += nt;
    tmax = max(tmax, nt);
    cu_qb[s + 1] = q;
    cu_blk[s + 1] = b;
    cu_tile[s + 1] = t;
  }
  // 128-row tiles ordered by tile index descending (longest causal rows
  // first), only those holding a query block of [qb_lo, qb_hi)
  const int per = 128 / B;  // query blocks per tile
  int w = 0;
  for (int tt = tmax - 1; tt >= 0; --tt)
    for (int s = 0; s < nseq; ++s)
      if (tt < cu_tile[s + 1] - cu_tile[s]) {
        const int64_t a = cu_qb[s] + int64_t(tt) * per;                 // first query block
        const int64_t e = min(int64_t(cu_qb[s + 1]), a + per);           // past the last
        if (a >= qb_hi || e <= qb_lo) continue;
        tiles[2 * w] = s;
        tiles[2 * w + 1] = tt;
        ++w;
      }
}

cudaError_t launch_meta(int nseq, const int32_t* cu_seqlens, int B, int64_t qb_lo,
                        int64_t qb_hi, const Meta& m, cudaStream_t st) {
  k_meta<<<1, 32, 0, st>>>(nseq, cu_seqlens, B, qb_lo, qb_hi, m.cu_qb, m.cu_blk, m.cu_tile,
                           m.tiles);
  return cudaGetLastError();
}

// ------------------------------------------------------------- block stats

constexpr int kKeyTile = 32;

// Logit of row i (local) against key j (local), given q . k.
__device__ __forceinline__ float logit(float dot, float scale, int i, int j, float band_bias,
                                       int band_width) {
  float s = dot * scale;
  int delta = i - j;
  if (delta < band_width) s += band_bias;  // caller guarantees delta >= 0
  return s;
}

// Two passes per (query block, head): pass 1 the row log-sum-exp, pass 2 the
// per-key-block probability mass summed over the block's rows.
template <typename T, int D>
__global__ void __launch_bounds__(128) k_stats_simt(
    const T* __restrict__ Q, const T* __restrict__ K, const int32_t* __restrict__ cu_seqlens,
    const int32_t* __restrict__ cu_qb, const int64_t* __restrict__ cu_blk, int nseq, int Hs,
    int B, float scale, float band_bias, int band_width, int64_t ntok, int64_t nblocks,
    int64_t qb_lo, float* __restrict__ lse_out, float* __restrict__ part) {
  __shared__ float ks[kKeyTile][D + 1];
  __shared__ float red[4];
  const int64_t gqb = qb_lo + blockIdx.x;
  const int h = blockIdx.y, tid = threadIdx.x;
  const int s = upper_index(cu_qb, nseq, gqb);
  const int qb = int(gqb - cu_qb[s]);
  const int seq0 = cu_seqlens[s];
  const int L = cu_seqlens[s + 1] - seq0;
  const int i = qb * B + tid;
  const bool valid = i < L;
  const int kend = min(L, (qb + 1) * B);

  float q[D];
#pragma unroll
  for (int c = 0; c < D; ++c)
    q[c] = valid ? to_f32(Q[(int64_t(seq0 + i) * Hs + h) * D + c]) : 0.f;

  auto load_tile = [&](int j0) {
    __syncthreads();
    for (int idx = tid; idx < kKeyTile * D; idx += blockDim.x) {
      int jj = idx / D, c = idx % D;
      int j = j0 + jj;
      ks[jj][c] = (j < kend) ? to_f32(K[(int64_t(seq0 + j) * Hs + h) * D + c]) : 0.f;
    }
    __syncthreads();
  };

  // pass 1: online max / sum
  float m = -CUDART_INF_F, l = 0.f;
  for (int j0 = 0; j0 < kend; j0 += kKeyTile) {
    load_tile(j0);
    if (valid) {
      for (int jj = 0; jj < kKeyTile; ++jj) {
        int j = j0 + jj;
        if (j > i) break;
        float dot = 0.f;
#pragma unroll
        for (int c = 0; c < D; ++c) dot = fmaf(q[c], ks[jj][c], dot);
        float x = logit(dot, scale, i, j, band_bias, band_width);
        if (x > m) {
          l = l * expf(m - x) + 1.f;
          m = x;
        } else {
          l += expf(x - m);
        }
      }
    }
  }
  const float lse = valid ? m + logf(l) : 0.f;
  if (valid) lse_out[int64_t(h) * ntok + seq0 + i] = lse;

  // pass 2: mass per key block
  const int64_t blk0 = cu_blk[s] + int64_t(qb) * (qb + 1) / 2;
  for (int kb = 0; kb <= qb; ++kb) {
    float acc = 0.f;
    for (int j0 = kb * B; j0 < min(kend, (kb + 1) * B); j0 += kKeyTile) {
      load_tile(j0);
      if (valid) {
        for (int jj = 0; jj < kKeyTile; ++jj) {
          int j = j0 + jj;
          if (j > i || j >= (kb + 1) * B) break;
          float dot = 0.f;
#pragma unroll
          for (int c = 0; c < D; ++c) dot = fmaf(q[c], ks[jj][c], dot);
          acc += expf(logit(dot, scale, i, j, band_bias, band_width) - lse);
        }
      }
    }
    acc = warp_sum(acc);
    __syncthreads();
    if ((tid & 31) == 0) red[tid >> 5] = acc;
    __syncthreads();
    if (tid == 0) {
      float t = 0.f;
      for (int w = 0; w < int(blockDim.x >> 5); ++w) t += red[w];
      part[int64_t(h) * nblocks + blk0 + kb] = t;
    }
  }
}

cudaError_t launch_stats_simt(const mf_attn_desc& d, const Sizes& sz, const QbRange& r,
                              const Meta& m, const void* Q, const void* K, float* lse,
                              float* part, cudaStream_t st) {
  if (r.qb_hi <= r.qb_lo) return cudaSuccess;
  dim3 grid(unsigned(r.qb_hi - r.qb_lo), unsigned(d.Hs));
  const float scale = 1.0f / sqrtf(float(d.d));
#define MF_STATS(T, DD)                                                                  \
  k_stats_simt<T, DD><<<grid, d.B, 0, st>>>(                                             \
      static_cast<const T*>(Q), static_cast<const T*>(K), d.cu_seqlens, m.cu_qb, m.cu_blk, \
      d.nseq, d.Hs, d.B, scale, d.band_bias, d.band_width, sz.ntok, sz.nblocks, r.qb_lo, lse, \
      part)
  if (d.dt == MF_F32) {
    if (d.d == 64) MF_STATS(float, 64); else MF_STATS(float, 128);
  } else {
    if (d.d == 64) MF_STATS(__nv_bfloat16, 64); else MF_STATS(__nv_bfloat16, 128);
  }
#undef MF_STATS
  return cudaGetLastError();
}

// mass[b] = sum_h part[h][b], float64 in head order, for b in [blk_lo, blk_hi).
__global__ void k_mass_reduce(const float* __restrict__ part, int Hs, int64_t nblocks,
                              int64_t blk_lo, int64_t blk_hi, float* __restrict__ mass) {
  for (int64_t b = blk_lo + blockIdx.x * int64_t(blockDim.x) + threadIdx.x; b < blk_hi;
       b += int64_t(gridDim.x) * blockDim.x) {
    double t = 0.0;
    for (int h = 0; h < Hs; ++h) t += double(part[int64_t(h) * nblocks + b]);
    mass[b] = float(t);
  }
}

cudaError_t launch_mass_reduce(const float* part, int Hs, int64_t nblocks, int64_t blk_lo,
                               int64_t blk_hi, float* mass, cudaStream_t st) {
  if (blk_hi <= blk_lo) return cudaSuccess;
  int grid = int(std::min<int64_t>((blk_hi - blk_lo + 255) / 256, 148 * 8));
  k_mass_reduce<<<grid, 256, 0, st>>>(part, Hs, nblocks, blk_lo, blk_hi, mass);
  return cudaGetLastError();
}

// ----------------------------------------------------------------- extract

template <typename T, int D>
__global__ void __launch_bounds__(128) k_extract_simt(
    const T* __restrict__ Q, const T* __restrict__ K, const float* __restrict__ lse_in,
    const int32_t* __restrict__ cu_seqlens, const int32_t* __restrict__ qb_seq,
    const int32_t* __restrict__ qb_idx, const int64_t* __restrict__ row_ptr,
    const int32_t* __restrict__ col_idx, int64_t capacity, int Hs, int B, float scale,
    float band_bias, int band_width, int64_t ntok, int64_t qb_lo, T* __restrict__ values) {
  __shared__ float ks[kKeyTile][D + 1];
  const int64_t gqb = qb_lo + blockIdx.x;
  const int h = blockIdx.y, tid = threadIdx.x;
  const int s = qb_seq[gqb], qb = qb_idx[gqb];
  const int seq0 = cu_seqlens[s];
  const int L = cu_seqlens[s + 1] - seq0;
  const int i = qb * B + tid;
  const bool valid = i < L;
  float q[D];
#pragma unroll
  for (int c = 0; c < D; ++c)
    q[c] = valid ? to_f32(Q[(int64_t(seq0 + i) * Hs + h) * D + c]) : 0.f;
  const float lse = valid ? lse_in[int64_t(h) * ntok + seq0 + i] : 0.f;
  const int64_t e0 = row_ptr[gqb], e1 = min(row_ptr[gqb + 1], capacity);
  for (int64_t e = e0; e < e1; ++e) {
    const int kb = col_idx[e];
    for (int j0 = kb * B; j0 < (kb + 1) * B; j0 += kKeyTile) {
      __syncthreads();
      for (int idx = tid; idx < kKeyTile * D; idx += blockDim.x) {
        int jj = idx / D, c = idx % D;
        int j = j0 + jj;
        ks[jj][c] = (j < L) ? to_f32(K[(int64_t(seq0 + j) * Hs + h) * D + c]) : 0.f;
      }
      __syncthreads();
      for (int jj = 0; jj < kKeyTile; ++jj) {
        int j = j0 + jj;
        float p = 0.f;
        if (valid && j <= i) {
          float dot = 0.f;
#pragma unroll
          for (int c = 0; c < D; ++c) dot = fmaf(q[c], ks[jj][c], dot);
          p = expf(logit(dot, scale, i, j, band_bias, band_width) - lse);
        }
        values[value_offset(e, tid, h, j - kb * B, B, Hs)] = from_f32<T>(p);
      }
    }
  }
}

cudaError_t launch_extract_simt(const mf_attn_desc& d, const Sizes& sz, const QbRange& r,
                                const void* Q, const void* K, const float* lse,
                                const mf_csr_cache& c, cudaStream_t st) {
  if (r.qb_hi <= r.qb_lo) return cudaSuccess;
  dim3 grid(unsigned(r.qb_hi - r.qb_lo), unsigned(d.Hs));
  const float scale = 1.0f / sqrtf(float(d.d));
#define MF_EXTRACT(T, DD)                                                                 \
  k_extract_simt<T, DD><<<grid, d.B, 0, st>>>(                                            \
      static_cast<const T*>(Q), static_cast<const T*>(K), lse, d.cu_seqlens, c.qb_seq,    \
      c.qb_idx, c.row_ptr, c.col_idx, c.nnz_capacity, d.Hs, d.B, scale, d.band_bias,      \
      d.band_width, sz.ntok, r.qb_lo, static_cast<T*>(c.values))
  if (d.dt == MF_F32) {
    if (d.d == 64) MF_EXTRACT(float, 64); else MF_EXTRACT(float, 128);
  } else {
    if (d.d == 64) MF_EXTRACT(__nv_bfloat16, 64); else MF_EXTRACT(__nv_bfloat16, 128);
  }
#undef MF_EXTRACT
  return cudaGetLastError();
}

// --------------------------------------------------------------- mapped AV

constexpr int kAvThreads = 256;
constexpr int kAvMaxOut = 16;  // outputs per thread: Hr * d <= 4096
constexpr int kAvKeys = 32;

template <typename T>
__device__ __forceinline__ const T* v_row(const T* V, const int32_t* page_table, int page_size,
                                          int max_pages, int s, int seq0, int j, int Hkv, int d) {
  if (page_table == nullptr) return V + (int64_t(seq0 + j) * Hkv) * d;
  int page = page_table[int64_t(s) * max_pages + j / page_size];
  return V + (int64_t(page) * page_size + (j % page_size)) * Hkv * d;
}

// One CTA per (query block, row in block): O[row] for all receiver heads.
template <typename T>
__global__ void __launch_bounds__(kAvThreads) k_mapped_av_simt(
    const T* __restrict__ values, const int64_t* __restrict__ row_ptr,
    const int32_t* __restrict__ col_idx, int64_t capacity, const int32_t* __restrict__ qb_seq,
    const int32_t* __restrict__ qb_idx, const int32_t* __restrict__ cu_seqlens,
    const T* __restrict__ W, const T* __restrict__ V, const int32_t* __restrict__ page_table,
    int page_size, int max_pages, int Hs, int Hr, int Hkv, int d, int B, int64_t qb_lo,
    T* __restrict__ O) {
  extern __shared__ float sm[];
  float* Ws = sm;             // [Hr][Hs]
  float* Ms = sm + Hr * Hs;   // [Hr][kAvKeys]
  const int64_t gqb = qb_lo + blockIdx.x;
  const int il = blockIdx.y, tid = threadIdx.x;
  const int s = qb_seq[gqb], qb = qb_idx[gqb];
  const int seq0 = cu_seqlens[s];
  const int L = cu_seqlens[s + 1] - seq0;
  const int i = qb * B + il;
  if (i >= L) return;
  for (int idx = tid; idx < Hr * Hs; idx += kAvThreads) Ws[idx] = to_f32(W[idx]);
  float acc[kAvMaxOut];
#pragma unroll
  for (int o = 0; o < kAvMaxOut; ++o) acc[o] = 0.f;
  const int gsz = Hr / Hkv;
  const int64_t e1 = min(row_ptr[gqb + 1], capacity);
  for (int64_t e = row_ptr[gqb]; e < e1; ++e) {
    const int kb = col_idx[e];
    for (int j0 = 0; j0 < B; j0 += kAvKeys) {
      __syncthreads();
      for (int idx = tid; idx < Hr * kAvKeys; idx += kAvThreads) {
        int r = idx / kAvKeys, jj = idx % kAvKeys;
        float mv = 0.f;
        for (int h = 0; h < Hs; ++h)
          mv = fmaf(Ws[r * Hs + h], to_f32(values[value_offset(e, il, h, j0 + jj, B, Hs)]), mv);
        Ms[r * kAvKeys + jj] = mv;
      }
      __syncthreads();
#pragma unroll
      for (int o = 0; o < kAvMaxOut; ++o) {
        int out = tid + o * kAvThreads;
        if (out < Hr * d) {
          int r = out / d, c = out % d, g = r / gsz;
          float a = acc[o];
          for (int jj = 0; jj < kAvKeys; ++jj) {
            int j = kb * B + j0 + jj;
            if (j >= L) break;
            const T* vr = v_row(V, page_table, page_size, max_pages, s, seq0, j, Hkv, d);
            a = fmaf(Ms[r * kAvKeys + jj], to_f32(vr[g * d + c]), a);
          }
          acc[o] = a;
        }
      }
    }
  }
#pragma unroll
  for (int o = 0; o < kAvMaxOut; ++o) {
    int out = tid + o * kAvThreads;
    if (out < Hr * d) O[int64_t(seq0 + i) * Hr * d + out] = from_f32<T>(acc[o]);
  }
}

cudaError_t launch_mapped_av_simt(const mf_csr_cache& c, const mf_attn_desc& d,
                                  const Sizes& sz, int Hr, const void* W,
                                  const mf_v_desc& v, void* O, int64_t qb_lo, int64_t qb_hi,
                                  cudaStream_t st) {
  if (qb_hi <= qb_lo) return cudaSuccess;
  dim3 grid(unsigned(qb_hi - qb_lo), unsigned(d.B));
  size_t smem = sizeof(float) * (size_t(Hr) * d.Hs + size_t(Hr) * kAvKeys);
#define MF_AV(T)                                                                        \
  k_mapped_av_simt<T><<<grid, kAvThreads, smem, st>>>(                                  \
      static_cast<const T*>(c.values), c.row_ptr, c.col_idx, c.nnz_capacity, c.qb_seq,   \
      c.qb_idx,                                                                         \
      d.cu_seqlens, static_cast<const T*>(W), static_cast<const T*>(v.V), v.page_table, \
      v.page_size, v.max_pages_per_seq, d.Hs, Hr, v.Hkv, v.d, d.B, qb_lo, static_cast<T*>(O))
  if (d.dt == MF_F32) MF_AV(float); else MF_AV(__nv_bfloat16);
#undef MF_AV
  return cudaGetLastError();
}

}  // namespace mf
