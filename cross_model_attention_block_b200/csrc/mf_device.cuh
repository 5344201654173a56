// Small device helpers shared by the libmapflow kernels.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace mf {

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Largest s in [0, n) with a[s] <= v, for a non-decreasing a[0..n] (a[0] <= v).
template <typename I>
__device__ __forceinline__ int upper_index(const I* a, int n, int64_t v) {
  int lo = 0, hi = n;  // invariant: a[lo] <= v, answer in [lo, hi)
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (static_cast<int64_t>(a[mid]) <= v) lo = mid; else hi = mid;
  }
  return lo;
}

// Element offset of (entry e, head h, row i, key j) in the CSR value array.
// Layout [nnz][B/16 key groups][B/8 row slices][2 halves][Hs][64]: one
// (entry, key group, row slice) -- 8 rows x 16 keys, all heads -- is one
// contiguous stage of the fused kernel, stored exactly as the 128-byte-swizzled
// MN-major operand of its head-mixing MMA: pair m = (i%8)*16 + j%16, half
// m/64, and inside a 128-byte line (head h) the 16-byte chunk (m%64)/8 sits at
// chunk ((m%64)/8) ^ (h%8).
__device__ __forceinline__ int64_t value_offset(int64_t e, int i, int h, int j, int B, int Hs) {
  const int64_t line = ((((e * (B >> 4) + (j >> 4)) * (B >> 3) + (i >> 3)) * 2 + ((i & 7) >> 2)) *
                            Hs + h);
  const int chunk = (((i & 3) << 1) | ((j >> 3) & 1)) ^ (h & 7);
  return line * 64 + chunk * 8 + (j & 7);
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace mf
