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

// Position of key (j % 16) inside its stored 16-key group for head h: the two
// 8-key halves are swapped when bit 2 of h is set.  Spreads the eight heads
// read together by a transposing shared-memory load over all banks.
__device__ __forceinline__ int key_slot(int j16, int h) { return j16 ^ (((h >> 2) & 1) << 3); }

// Element offset of (entry e, row i, head h, key j) in the CSR value array
// [nnz][B/16][B][Hs][16].
__device__ __forceinline__ int64_t value_offset(int64_t e, int i, int h, int j, int B, int Hs) {
  return (((e * (B >> 4) + (j >> 4)) * B + i) * Hs + h) * 16 + key_slot(j & 15, h);
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
