// Tensor-core (tcgen05 + TMA) kernels over the causal sender logits, bf16, d = 128.
//
// MapFlow article (163.com, section on the three system components): the
// sender's attention map is compressed in stages -- block-level statistics
// first, then extraction of the kept blocks -- never forming the dense N x N
// matrix.  Both stages walk the causal QK^T of one (head, 128-row query tile)
// pair tile by tile; they differ only in what the epilogue does with a tile.
//
//  * Block statistics (k_stats_wide, one pass): online row max and sum give
//    the row log-sum-exp; each key block's partial sum is kept as a log value
//    a = m + log2(sum_j 2^(x_j - m)) in TMEM columns 256.., so that after the
//    last tile mass contribution = 2^(a - lse2) needs no second QK^T pass.
//  * Extraction (k_extract_wide): for every kept block of the tile,
//    P = 2^(x - lse2) rounded to bf16 and written in the cache layout.
//
// Roles (640 threads): warp 0 issues TMA loads (Q once, K tiles through a
// 3-stage ring), warp 1 owns TMEM and issues tcgen05.mma from one thread into
// one of two 128-column S buffers, warps 4..19 run the epilogue as four
// warpgroups: the two groups of a tile parity split the tile's columns, one
// query row per thread, so the next tile's MMA overlaps this tile's epilogue
// and four groups keep exponentials in flight.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math_constants.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "mf_sm100.cuh"

namespace mf {
using namespace sm100;

namespace qk {

constexpr int kTile = 128;
constexpr int kD = 128;
constexpr int kMaxBlocksPerSeq = 512;  // a sequence holds at most 512 blocks
constexpr uint32_t kTileBytes = kTile * kD * 2;  // 32 KB: two [128][64] swizzled halves
constexpr uint32_t kHalfBytes = kTileBytes / 2;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAcol = 256;  // first TMEM column of the per-key-block log partials
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct Params {
  const int32_t* cu_seqlens;
  const int32_t* tiles;    // [ntiles][2] = (sequence, 128-row tile), heaviest first
  const int64_t* cu_blk;   // [nseq+1]
  const int32_t* cu_qb;    // [nseq+1]
  int ntiles;
  int Hs;
  int head_group;  // extraction: heads per CTA group (head innermost)
  int B;
  int band_width;
  float scale2;            // log2(e) / sqrt(d)
  float bias2;             // band_bias * log2(e)
  int64_t ntok;
  int64_t nblocks;
  float* lse;              // stats: out [Hs][ntok] (natural log); extract: in
  float* part;             // stats: out [Hs][nblocks]
  const int32_t* slot;     // extract: block -> cache entry or -1
  __nv_bfloat16* values;   // extract: out
  int64_t qb_lo, qb_hi;    // global query blocks whose rows and blocks are written
  unsigned* status;
};

// Does key tile kt hold a kept block of this query tile?  `slots` is the
// CTA's copy of the block -> entry map (-1: not kept or not causal).
template <int BB>
__device__ __forceinline__ bool tile_needed(const int32_t (*slots)[kMaxBlocksPerSeq], int kt) {
  if (BB == 128) return slots[0][kt] >= 0;
  return slots[0][2 * kt] >= 0 || slots[0][2 * kt + 1] >= 0 || slots[1][2 * kt] >= 0 ||
         slots[1][2 * kt + 1] >= 0;
}

// Lane l ends up holding sum over the warp of v[l] (v has 32 entries).
__device__ __forceinline__ float transpose_reduce32(float* v, int lane) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int k = 0; k < s; ++k) {
      float send = upper ? v[k] : v[k + s];
      float keep = upper ? v[k + s] : v[k];
      v[k] = keep + __shfl_xor_sync(0xffffffffu, send, s);
    }
  }
  return v[0];
}

// ------------------------------------------------- statistics, four groups
//
// The one-pass statistics with four epilogue warpgroups: the two groups of a
// tile parity split its columns (group g takes the tiles kt % 2 == g % 2 and
// the 64-column half g / 2), so sixteen warps per SM keep exponentials in
// flight while the MMA warp fills the other S buffer.  Each group keeps its own running (max, sum)
// per row; the four are merged once at the end.  B = 64: a half is one key
// block, stored as is.  B = 128: the second half hands its (reference, sum)
// to the first through shared memory, double-buffered and signalled with
// mbarriers (a full and a consumed barrier per buffer), so neither group of
// the pair waits for the other in the common case.  FMAX of every 8
// exponentials run on the FMA pipe (exp2_fma2), the rest on MUFU.
constexpr int kWideThreads = 640;  // warps 0-3 roles, 4-19 epilogue (four warpgroups)
// Exponentials of every 8 that the statistics compute on the FMA pipe (the
// rest on MUFU).  Measured on the 32K-token workload: 0 -> 8.0 ms, 2 -> 7.6,
// 4 -> 8.2.
constexpr int kStatsFmaExp = 2;

struct SmemWide {
  uint8_t q[kTileBytes];
  uint8_t k[3][kTileBytes];
  float red[4][4][32];
  float2 xch[4][4][32];    // [quarter][group][lane]: each group's row (max, sum)
  float2 half[2][2][128];  // B = 128: [tile parity][buffer][row] second half's (ref, sum)
  uint64_t q_full;
  uint64_t k_full[3];
  uint64_t k_empty[3];
  uint64_t s_full[2];
  uint64_t s_empty[2];
  uint64_t h_full[2][2];   // B = 128 hand-over: written by the second half
  uint64_t h_free[2][2];   // read by the first half
  uint64_t drain;
  uint32_t tmem_base;
};

// The four epilogue warps of one TMEM lane quarter (named barriers 2..5).
__device__ __forceinline__ void quarter_sync(int quarter) {
  asm volatile("bar.sync %0, 128;" ::"r"(2 + quarter) : "memory");
}

// AND over the 512 epilogue threads (named barrier 1).
__device__ __forceinline__ bool wide_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 512, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(uint32_t(v))
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void wide_sync() { asm volatile("bar.sync 1, 512;" ::: "memory"); }

template <int BB, int FMAX>
__global__ void __launch_bounds__(kWideThreads, 1)
    k_stats_wide(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const Params p) {
  constexpr int kStg = 3;
  extern __shared__ uint8_t smem_raw[];
  SmemWide& sm = *reinterpret_cast<SmemWide*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x / p.ntiles;
  const int w = blockIdx.x % p.ntiles;
  const int s = p.tiles[2 * w], t = p.tiles[2 * w + 1];
  const int seq0 = p.cu_seqlens[s];
  const int L = p.cu_seqlens[s + 1] - seq0;
  const int nqb_s = p.cu_qb[s + 1] - p.cu_qb[s];
  const int row0 = t * kTile;

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    for (int i = 0; i < kStg; ++i) {
      mbar_init(&sm.k_full[i], 1);
      mbar_init(&sm.k_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.s_empty[i], 256);  // both groups of the tile parity
      for (int b = 0; b < 2; ++b) {
        mbar_init(&sm.h_full[i][b], 128);
        mbar_init(&sm.h_free[i][b], 128);
      }
    }
    mbar_init(&sm.drain, 1);
    fence_barrier_init();
  }
  const int64_t gq0 = p.cu_qb[s];
  auto in_range = [&](int qb) { return gq0 + qb >= p.qb_lo && gq0 + qb < p.qb_hi; };
  if (warp == 1) tmem_alloc(&sm.tmem_base, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      mbar_expect_tx(&sm.q_full, kTileBytes);
      tma_load_2d(sm.q, &tmQ, &sm.q_full, h * kD, seq0 + row0);
      tma_load_2d(sm.q + kHalfBytes, &tmQ, &sm.q_full, h * kD + 64, seq0 + row0);
      for (int kt = 0; kt <= t; ++kt) {
        const int st = kt % kStg;
        if (!mbar_wait(&sm.k_empty[st], ((kt / kStg) & 1) ^ 1, p.status)) break;
        mbar_expect_tx(&sm.k_full[st], kTileBytes);
        tma_load_2d(sm.k[st], &tmK, &sm.k_full[st], h * kD, seq0 + kt * kTile);
        tma_load_2d(sm.k[st] + kHalfBytes, &tmK, &sm.k_full[st], h * kD + 64,
                    seq0 + kt * kTile);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, 128, 0, 0);
      const uint32_t q_addr = smem_u32(sm.q);
      bool ok = mbar_wait(&sm.q_full, 0, p.status);
      for (int kt = 0; ok && kt <= t; ++kt) {
        const int st = kt % kStg, sb = kt & 1;
        if (!mbar_wait(&sm.k_full[st], (kt / kStg) & 1, p.status)) break;
        if (!mbar_wait(&sm.s_empty[sb], ((kt >> 1) & 1) ^ 1, p.status)) break;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sm.k[st]);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
          mma_bf16_ss(tmem + sb * 128, smem_desc(q_addr + off, 16, 1024, kSwizzle128),
                      smem_desc(k_addr + off, 16, 1024, kSwizzle128), idesc, kk > 0);
        }
        mma_commit(&sm.k_empty[st]);
        mma_commit(&sm.s_full[sb]);
      }
      mma_commit(&sm.drain);
      mbar_wait(&sm.drain, 0, p.status);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int eg = (warp - 4) >> 2;  // group 0..3
    const int par = eg & 1;          // tiles kt % 2 == par, S buffer par
    const int hc = eg >> 1;          // columns 64 * hc .. 64 * hc + 63
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int ri = row0 + r;
    const bool valid = ri < L;
    const uint32_t lane_addr = tmem + (uint32_t(quarter * 32) << 16);
    const int W = p.band_width;
    float m_run = -CUDART_INF_F, l_run = 0.f;
    bool ok = true;
    for (int kt = par, u = 0; kt <= t; kt += 2, ++u) {
      const int sb = par;
      if (!mbar_wait(&sm.s_full[sb], (kt >> 1) & 1, p.status)) { ok = false; break; }
      tc_fence_after();
      float v[64];
      tmem_ld32(lane_addr + sb * 128 + hc * 64, v);
      tmem_ld32(lane_addr + sb * 128 + hc * 64 + 32, v + 32);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&sm.s_empty[sb]);
      const int kbase = kt * kTile + hc * 64;
      const bool band_tile = row0 - (kt * kTile + kTile - 1) < W;
      const bool plain = !band_tile && kt != t;
      const float sc = plain ? p.scale2 : 1.f;
      if (!plain) {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const int j = kbase + c;
          float x = v[c] * p.scale2;
          if (ri - j < W) x += p.bias2;
          if (j > ri) x = -CUDART_INF_F;
          v[c] = x;
        }
      }
      float mx[8];
#pragma unroll
      for (int k = 0; k < 8; ++k)
        mx[k] = fmaxf(fmax3(fmax3(fmax3(v[k], v[8 + k], v[16 + k]), v[24 + k], v[32 + k]),
                            v[40 + k], v[48 + k]),
                      v[56 + k]);
      const float mt =
          fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) * sc;
      const float m_new = valid ? fmaxf(m_run, mt) : 0.f;
      const float m_use = m_new == -CUDART_INF_F ? 0.f : m_new;
      float2 acc[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[k] = make_float2(0.f, 0.f);
      const float2 sc2 = make_float2(sc, sc), nm2 = make_float2(-m_use, -m_use);
#pragma unroll
      for (int c = 0; c < 64; c += 8)
#pragma unroll
        for (int k = 0; k < 8; k += 2) {
          const float2 x = ffma2(make_float2(v[c + k], v[c + k + 1]), sc2, nm2);
          const float2 e = (k >= 8 - FMAX) ? exp2_fma2(x) : make_float2(ex2(x.x), ex2(x.y));
          acc[k >> 1] = fadd2(acc[k >> 1], e);
        }
      const float sh = ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) +
                       ((acc[2].x + acc[2].y) + (acc[3].x + acc[3].y));
      l_run = l_run * ex2(m_run - m_use) + sh;
      m_run = m_new;
      if (BB == 64) {
        const float a = valid ? m_new + lg2(sh) : -CUDART_INF_F;
        tmem_st1(lane_addr + kAcol + 2 * kt + hc, a);
      } else {
        const int b = u & 1;
        const uint32_t ph = (u >> 1) & 1;
        if (hc == 1) {
          // the first half has read this buffer's previous hand-over
          if (!mbar_wait(&sm.h_free[par][b], ph ^ 1, p.status)) { ok = false; break; }
          sm.half[par][b][r] = make_float2(m_use, sh);
          mbar_arrive(&sm.h_full[par][b]);
        } else {
          if (!mbar_wait(&sm.h_full[par][b], ph, p.status)) { ok = false; break; }
          const float2 o = sm.half[par][b][r];
          mbar_arrive(&sm.h_free[par][b]);
          const float M = fmaxf(m_use, o.x);
          const float tot = sh * ex2(m_use - M) + o.y * ex2(o.x - M);
          const float a = valid ? M + lg2(tot) : -CUDART_INF_F;
          tmem_st1(lane_addr + kAcol + kt, a);
        }
      }
    }
    ok = wide_all(ok);
    if (ok) {
      // row log-sum-exp from the four groups' (max, sum)
      sm.xch[quarter][eg][lane] = make_float2(m_run, l_run);
      quarter_sync(quarter);
      float M = -CUDART_INF_F;
#pragma unroll
      for (int g = 0; g < 4; ++g) M = fmaxf(M, sm.xch[quarter][g][lane].x);
      const float Mu = M == -CUDART_INF_F ? 0.f : M;
      float l = 0.f;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const float2 o = sm.xch[quarter][g][lane];
        l += o.y * ex2(o.x - Mu);
      }
      const float lse2 = valid ? M + lg2(l) : 0.f;
      if (valid && eg == 0 && in_range(ri / BB)) p.lse[int64_t(h) * p.ntok + seq0 + ri] = lse2 * kLn2;
      tmem_wait_st();
      tc_fence_before();
      wide_sync();  // every group's log partials are in TMEM
      tc_fence_after();
      // block masses: chunks of 32 key blocks, one per group in turn
      const int nkb = (t + 1) * (kTile / BB);
      const int64_t cb = p.cu_blk[s];
      for (int c2 = 0; c2 < nkb; c2 += 128) {
        const int c0 = c2 + eg * 32;
        float a[32];
        tmem_ld32(lane_addr + kAcol + min(c0, 256 - 32), a);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) a[k] = (valid && c0 + k < nkb) ? ex2(a[k] - lse2) : 0.f;
        const float tot = transpose_reduce32(a, lane);
        wide_sync();
        sm.red[eg][quarter][lane] = tot;
        wide_sync();
        if (quarter == 0 && c0 < nkb) {
          const int kb = c0 + lane;
          if (BB == 128) {
            const float m = (sm.red[eg][0][lane] + sm.red[eg][1][lane]) +
                            (sm.red[eg][2][lane] + sm.red[eg][3][lane]);
            if (kb <= t && in_range(t))
              p.part[int64_t(h) * p.nblocks + cb + int64_t(t) * (t + 1) / 2 + kb] = m;
          } else {
            const int qa = 2 * t, qbb = 2 * t + 1;
            const float m0 = sm.red[eg][0][lane] + sm.red[eg][1][lane];
            const float m1 = sm.red[eg][2][lane] + sm.red[eg][3][lane];
            if (kb <= qa && in_range(qa))
              p.part[int64_t(h) * p.nblocks + cb + int64_t(qa) * (qa + 1) / 2 + kb] = m0;
            if (qbb < nqb_s && kb <= qbb && in_range(qbb))
              p.part[int64_t(h) * p.nblocks + cb + int64_t(qbb) * (qbb + 1) / 2 + kb] = m1;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------- extraction, four groups
//
// Extraction with four epilogue warpgroups: as in k_stats_wide, the two
// groups of a tile parity (counted over the kept tiles only) split the
// tile's columns, so each group extracts one 64-key chunk per tile into its
// own 16 KB staging buffer.  A warp's 32 rows make 8 consecutive 128-byte
// lines of every 16-key group in the cache; the warp stages its 4 x 8 lines
// as one 4 KB run, stores them with one TMA store per tile and waits only for
// its own previous store: no barrier inside the group.  The run is laid out
// in the store's 128-byte swizzle (16-byte chunk ^ line % 8), which spreads
// the 8 lanes of a shared-memory store phase over all 32 banks; the layout in
// the cache is unchanged.  CTAs take heads in groups of up to kHeadGroup, the
// head innermost, so the heads' 128-byte pieces of a cache line (adjacent in
// the cache layout) are written at about the same time; the group is cut so
// that its K (every sequence's keys of those heads) fits kHeadGroupL2 bytes
// and stays in L2 while the tiles run (one head when a single head's K does
// not fit, the order of one head after another).
constexpr int kHeadGroup = 8;
constexpr double kHeadGroupL2 = 72.0 * 1024 * 1024;

struct SmemWideX {
  uint8_t q[kTileBytes];
  uint8_t k[3][kTileBytes];
  uint8_t out[4][kHalfBytes];
  int32_t slots[2][kMaxBlocksPerSeq];
  uint64_t q_full;
  uint64_t k_full[3];
  uint64_t k_empty[3];
  uint64_t s_full[2];
  uint64_t s_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
};

template <int BB>
__global__ void __launch_bounds__(kWideThreads, 1)
    k_extract_wide(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const Params p) {
  constexpr int kStg = 3;
  extern __shared__ uint8_t smem_raw[];
  SmemWideX& sm = *reinterpret_cast<SmemWideX*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // heads in groups of head_group, the head innermost: the CTAs writing
  // neighbouring 128-byte pieces of a cache line run at about the same time
  const int per = p.ntiles * p.head_group;
  const int hg = blockIdx.x / per;
  const int gsz = min(p.head_group, p.Hs - hg * p.head_group);
  const int rem = blockIdx.x - hg * per;
  const int h = hg * p.head_group + rem % gsz;
  const int w = rem / gsz;
  const int s = p.tiles[2 * w], t = p.tiles[2 * w + 1];
  const int seq0 = p.cu_seqlens[s];
  const int L = p.cu_seqlens[s + 1] - seq0;
  const int nqb_s = p.cu_qb[s + 1] - p.cu_qb[s];
  const int row0 = t * kTile;

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    for (int i = 0; i < kStg; ++i) {
      mbar_init(&sm.k_full[i], 1);
      mbar_init(&sm.k_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.s_empty[i], 256);  // both groups of the tile parity
    }
    mbar_init(&sm.drain, 1);
    fence_barrier_init();
  }
  const int64_t gq0 = p.cu_qb[s];
  auto in_range = [&](int qb) { return gq0 + qb >= p.qb_lo && gq0 + qb < p.qb_hi; };
  {
    const int64_t cb = p.cu_blk[s];
    for (int i = threadIdx.x; i < 2 * kMaxBlocksPerSeq; i += kWideThreads) {
      const int a = i / kMaxBlocksPerSeq, kb = i % kMaxBlocksPerSeq;
      const int qb = (BB == 128) ? (a == 0 ? t : -1) : 2 * t + a;
      sm.slots[a][kb] = (qb >= 0 && qb < nqb_s && kb <= qb && in_range(qb))
                            ? p.slot[cb + int64_t(qb) * (qb + 1) / 2 + kb]
                            : -1;
    }
  }
  if (warp == 1) tmem_alloc(&sm.tmem_base, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      mbar_expect_tx(&sm.q_full, kTileBytes);
      tma_load_2d(sm.q, &tmQ, &sm.q_full, h * kD, seq0 + row0);
      tma_load_2d(sm.q + kHalfBytes, &tmQ, &sm.q_full, h * kD + 64, seq0 + row0);
      int n = 0;
      for (int kt = 0; kt <= t; ++kt) {
        if (!tile_needed<BB>(sm.slots, kt)) continue;
        const int st = n % kStg;
        if (!mbar_wait(&sm.k_empty[st], ((n / kStg) & 1) ^ 1, p.status)) break;
        mbar_expect_tx(&sm.k_full[st], kTileBytes);
        tma_load_2d(sm.k[st], &tmK, &sm.k_full[st], h * kD, seq0 + kt * kTile);
        tma_load_2d(sm.k[st] + kHalfBytes, &tmK, &sm.k_full[st], h * kD + 64,
                    seq0 + kt * kTile);
        ++n;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, 128, 0, 0);
      const uint32_t q_addr = smem_u32(sm.q);
      bool ok = mbar_wait(&sm.q_full, 0, p.status);
      int n = 0;
      for (int kt = 0; ok && kt <= t; ++kt) {
        if (!tile_needed<BB>(sm.slots, kt)) continue;
        const int st = n % kStg, sb = n & 1;
        if (!mbar_wait(&sm.k_full[st], (n / kStg) & 1, p.status)) break;
        if (!mbar_wait(&sm.s_empty[sb], ((n >> 1) & 1) ^ 1, p.status)) break;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sm.k[st]);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
          mma_bf16_ss(tmem + sb * 128, smem_desc(q_addr + off, 16, 1024, kSwizzle128),
                      smem_desc(k_addr + off, 16, 1024, kSwizzle128), idesc, kk > 0);
        }
        mma_commit(&sm.k_empty[st]);
        mma_commit(&sm.s_full[sb]);
        ++n;
      }
      mma_commit(&sm.drain);
      mbar_wait(&sm.drain, 0, p.status);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int eg = (warp - 4) >> 2;  // group 0..3
    const int par = eg & 1;          // needed tiles n % 2 == par, S buffer par
    const int hc = eg >> 1;          // columns 64 * hc .. 64 * hc + 63
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int ri = row0 + r;
    const bool valid = ri < L;
    const uint32_t lane_addr = tmem + (uint32_t(quarter * 32) << 16);
    const int W = p.band_width;
    const float lse2 = valid ? p.lse[int64_t(h) * p.ntok + seq0 + ri] * kLog2e : 0.f;
    const int rb = r & (BB - 1);                          // row within the block
    const int lrow = ((rb >> 3) << 1) + ((rb & 7) >> 2);  // line of this row, key group 0
    const int cbase = (rb & 3) << 1;                       // chunk of keys 0-7
    // The warp's 32 rows fill 8 consecutive lines of every 16-key group of its
    // (row block's) staging area: it writes and stores them on its own.
    const int a = (BB == 128) ? 0 : (quarter >> 1);               // row block (B = 64)
    const int wl = (BB == 128) ? 8 * quarter : 8 * (quarter & 1);  // first line per key group
    uint8_t* stage = sm.out[eg] + quarter * 4096;  // the warp's 4 key groups x 8 lines
    // the kept map (tens of GB) is written once: its lines leave L2 first, so
    // the K tiles that later query tiles re-read stay
    const uint64_t keep_out = l2_evict_first();
    int n = 0;
    for (int kt = 0; kt <= t; ++kt) {
      if (!tile_needed<BB>(sm.slots, kt)) continue;
      if ((n & 1) != par) { ++n; continue; }
      const int sb = par;
      const bool got = mbar_wait(&sm.s_full[sb], (n >> 1) & 1, p.status);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      float v[64];
      tmem_ld32(lane_addr + sb * 128 + hc * 64, v);
      tmem_ld32(lane_addr + sb * 128 + hc * 64 + 32, v + 32);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&sm.s_empty[sb]);
      const int kbase = kt * kTile + hc * 64;
      const bool band_tile = row0 - (kt * kTile + kTile - 1) < W;
      const bool plain = !band_tile && kt != t;
      const float sc = plain ? p.scale2 : 1.f;
      if (!plain) {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const int j = kbase + c;
          float x = v[c] * p.scale2;
          if (ri - j < W) x += p.bias2;
          if (j > ri) x = -CUDART_INF_F;
          v[c] = x;
        }
      }
      const int kb = (BB == 128) ? kt : 2 * kt + hc;
      const int e = sm.slots[a][kb];
      if (e >= 0) {
        // the warp's previous stores are done reading its lines
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
#pragma unroll
        for (int kgl = 0; kgl < 4; ++kgl) {
          uint8_t* line = stage + (kgl * 8 + (lrow & 7)) * 128;
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t w4[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int col = kgl * 16 + c * 8 + 2 * k;
              const float2 x = ffma2(make_float2(v[col], v[col + 1]), make_float2(sc, sc),
                                     make_float2(-lse2, -lse2));
              __nv_bfloat162 pr =
                  __floats2bfloat162_rn(valid ? ex2(x.x) : 0.f, valid ? ex2(x.y) : 0.f);
              w4[k] = *reinterpret_cast<uint32_t*>(&pr);
            }
            *reinterpret_cast<uint4*>(line + ((((cbase | c) ^ (h & 7)) ^ (lrow & 7)) << 4)) =
                make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_5d_hint(&tmV, stage, 0, h, wl, (BB == 128) ? hc * 4 : 0, int32_t(e),
                            keep_out);
          bulk_commit();
        }
      }
      ++n;
    }
    if (lane == 0) bulk_wait_all<0>();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------------- host side

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                 const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                 const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                 CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// One thread waits, with the kernels' bounded wait, on an mbarrier whose
// phase nothing completes: the wait gives up after limit_ns and raises the
// timeout bit of the status word (diagnostic entry point for the failure path).
__global__ void k_selftest_timeout(uint64_t limit_ns, unsigned* status) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_barrier_init();
  mbar_wait_for(&bar, 0, status, limit_ns);  // expected to return false
}

// y = 2^x by the FMA-pipe exponential, grid-stride (diagnostic entry point):
// pairs through exp2_fma2 (the form the statistics kernel uses), a last odd
// element through exp2_fma.
__global__ void k_exp2_fma_eval(const float* __restrict__ x, float* y, int64_t n) {
  for (int64_t i = 2 * (int64_t(blockIdx.x) * blockDim.x + threadIdx.x); i < n;
       i += 2 * int64_t(gridDim.x) * blockDim.x) {
    if (i + 1 < n) {
      const float2 r = exp2_fma2(make_float2(x[i], x[i + 1]));
      y[i] = r.x;
      y[i + 1] = r.y;
    } else {
      y[i] = exp2_fma(x[i]);
    }
  }
}

}  // namespace qk

static qk::EncodeTiled encode_fn() {
  static qk::EncodeTiled fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<qk::EncodeTiled>(p);
  });
  return fn;
}

// 2-D bf16 tensor map over rows x cols (cols contiguous), box {64, box_rows},
// 128-byte swizzle.
cudaError_t make_tmap_2d_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                              uint32_t box_cols, uint32_t box_rows, bool swizzle128) {
  qk::EncodeTiled enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_tmap_bf16(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
                           const uint64_t* strides_bytes, const uint32_t* box, int swizzle_bytes) {
  qk::EncodeTiled enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  cuuint64_t d[5], st[4];
  cuuint32_t bx[5], estr[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
    estr[i] = 1;
    if (i + 1 < rank) st[i] = strides_bytes[i];
  }
  CUtensorMapSwizzle sw = swizzle_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                          : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                          : swizzle_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                : CU_TENSOR_MAP_SWIZZLE_NONE;
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, cuuint32_t(rank), const_cast<void*>(base),
                   d, st, bx, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t launch_stats_tc(const mf_attn_desc& d, const Sizes& sz, const QbRange& r,
                            const Meta& m, const void* Q, const void* K, float* lse,
                            float* part, cudaStream_t st) {
  if (r.ntiles == 0) return cudaSuccess;
  CUtensorMap tq, tk;
  const uint64_t cols = uint64_t(d.Hs) * d.d;
  cudaError_t e = make_tmap_2d_bf16(&tq, Q, uint64_t(sz.ntok), cols, 64, qk::kTile, true);
  if (e != cudaSuccess) return e;
  e = make_tmap_2d_bf16(&tk, K, uint64_t(sz.ntok), cols, 64, qk::kTile, true);
  if (e != cudaSuccess) return e;
  qk::Params p{};
  p.cu_seqlens = d.cu_seqlens;
  p.tiles = m.tiles;
  p.cu_blk = m.cu_blk;
  p.cu_qb = m.cu_qb;
  p.ntiles = int(r.ntiles);
  p.Hs = d.Hs;
  p.B = d.B;
  p.band_width = d.band_width;
  p.scale2 = qk::kLog2e / sqrtf(float(d.d));
  p.bias2 = d.band_bias * qk::kLog2e;
  p.ntok = sz.ntok;
  p.nblocks = sz.nblocks;
  p.lse = lse;
  p.part = part;
  p.qb_lo = r.qb_lo;
  p.qb_hi = r.qb_hi;
  p.status = status_word();
  const size_t smem = sizeof(qk::SmemWide) + 1024;
  const unsigned grid = unsigned(r.ntiles) * unsigned(d.Hs);
#define MF_QKW(BB)                                                                        \
  do {                                                                                    \
    e = cudaFuncSetAttribute(qk::k_stats_wide<BB, qk::kStatsFmaExp>,                      \
                             cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));     \
    if (e != cudaSuccess) return e;                                                       \
    qk::k_stats_wide<BB, qk::kStatsFmaExp><<<grid, qk::kWideThreads, smem, st>>>(tq, tk, p); \
  } while (0)
  if (d.B == 128) MF_QKW(128); else MF_QKW(64);
#undef MF_QKW
  return cudaGetLastError();
}

cudaError_t launch_extract_tc(const mf_attn_desc& d, const Sizes& sz, const QbRange& r,
                              const Meta& m, const void* Q, const void* K, const float* lse,
                              const int32_t* slot, void* values, int64_t capacity,
                              cudaStream_t st) {
  if (r.ntiles == 0 || capacity < 1) return cudaSuccess;
  CUtensorMap tq, tk, tv;
  const uint64_t cols = uint64_t(d.Hs) * d.d;
  cudaError_t e = make_tmap_2d_bf16(&tq, Q, uint64_t(sz.ntok), cols, 64, qk::kTile, true);
  if (e != cudaSuccess) return e;
  e = make_tmap_2d_bf16(&tk, K, uint64_t(sz.ntok), cols, 64, qk::kTile, true);
  if (e != cudaSuccess) return e;
  // one store writes one warp's rows of an (entry, head): 8 lines of each of
  // the 4 key groups of a 64-key chunk, from a staging run in the 128-byte
  // swizzle; the lines are split as (line in its key group, key group)
  const uint64_t nl = uint64_t(d.B) * uint64_t(d.B) / 64;
  const uint64_t lpg = uint64_t(d.B) / 4;  // lines of one 16-key group
  const uint64_t dims[5] = {64, uint64_t(d.Hs), lpg, nl / lpg, uint64_t(capacity)};
  const uint64_t strides[4] = {128, uint64_t(d.Hs) * 128, lpg * uint64_t(d.Hs) * 128,
                               nl * uint64_t(d.Hs) * 128};
  const uint32_t box[5] = {64, 1, 8, 4, 1};
  e = make_tmap_bf16(&tv, values, 5, dims, strides, box, 128);
  if (e != cudaSuccess) return e;
  qk::Params p{};
  p.cu_seqlens = d.cu_seqlens;
  p.tiles = m.tiles;
  p.cu_blk = m.cu_blk;
  p.cu_qb = m.cu_qb;
  p.ntiles = int(r.ntiles);
  p.Hs = d.Hs;
  {
    const double k_head = double(sz.ntok) * double(d.d) * 2.0;  // K bytes of one head
    const int fit = int(std::min(double(qk::kHeadGroup), qk::kHeadGroupL2 / k_head));
    p.head_group = std::max(1, std::min(d.Hs, fit));
  }
  p.B = d.B;
  p.band_width = d.band_width;
  p.scale2 = qk::kLog2e / sqrtf(float(d.d));
  p.bias2 = d.band_bias * qk::kLog2e;
  p.ntok = sz.ntok;
  p.nblocks = sz.nblocks;
  p.lse = const_cast<float*>(lse);
  p.slot = slot;
  p.values = static_cast<__nv_bfloat16*>(values);
  p.qb_lo = r.qb_lo;
  p.qb_hi = r.qb_hi;
  p.status = status_word();
  const size_t smem = sizeof(qk::SmemWideX) + 1024;
  const unsigned grid = unsigned(r.ntiles) * unsigned(d.Hs);
#define MF_QKX(BB)                                                                            \
  do {                                                                                        \
    e = cudaFuncSetAttribute(qk::k_extract_wide<BB>,                                          \
                             cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));         \
    if (e != cudaSuccess) return e;                                                           \
    qk::k_extract_wide<BB><<<grid, qk::kWideThreads, smem, st>>>(tq, tk, tv, p);              \
  } while (0)
  if (d.B == 128) MF_QKX(128); else MF_QKX(64);
#undef MF_QKX
  return cudaGetLastError();
}

cudaError_t launch_exp2_fma_eval(const float* x, float* y, int64_t n, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const int64_t blocks = std::min<int64_t>((n + 255) / 256, 148 * 8);
  qk::k_exp2_fma_eval<<<unsigned(blocks), 256, 0, st>>>(x, y, n);
  return cudaGetLastError();
}

cudaError_t launch_selftest_timeout(uint64_t limit_ns, cudaStream_t st) {
  qk::k_selftest_timeout<<<1, 32, 0, st>>>(limit_ns, status_word());
  return cudaGetLastError();
}

}  // namespace mf
