// Tensor-core (tcgen05 + TMA) kernels over the causal sender logits, bf16, d = 128.
//
// MapFlow article (163.com, section on the three system components): the
// sender's attention map is compressed in stages -- block-level statistics
// first, then extraction of the kept blocks -- never forming the dense N x N
// matrix.  Both stages walk the causal QK^T of one (head, 128-row query tile)
// pair tile by tile; they differ only in what the epilogue does with a tile.
//
//  * Block statistics (one pass): online row max and sum give the row
//    log-sum-exp; each key block's partial sum is kept as a log value
//    a = m + log2(sum_j 2^(x_j - m)) in TMEM columns 256.., so that after the
//    last tile mass contribution = 2^(a - lse2) needs no second QK^T pass.
//  * Extraction: for every kept block of the tile, P = 2^(x - lse2) rounded to
//    bf16 and written in the cache layout.
//
// Roles (384 threads): warp 0 issues TMA loads, warp 1 owns TMEM and issues
// tcgen05.mma from one thread, warps 4..11 run the epilogue as two
// warpgroups that take turns on the tiles (group n % 2 reads S buffer n % 2),
// one query row per thread.  S = Q K^T for a 128 x 128 tile
// lands in one of two TMEM buffers (columns 0..255) so the next tile's MMA
// overlaps this tile's epilogue; K tiles stream through a 3-stage ring.
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
constexpr int kStages = 3;
constexpr int kMaxBlocksPerSeq = 512;  // a sequence holds at most 512 blocks
constexpr int kThreads = 384;  // warps 0-3 roles, 4-11 epilogue (two per lane quarter)
constexpr uint32_t kTileBytes = kTile * kD * 2;  // 32 KB: two [128][64] swizzled halves
constexpr uint32_t kHalfBytes = kTileBytes / 2;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAcol = 256;  // first TMEM column of the per-key-block log partials
// Share of the statistics exponentials computed by exp2_fma (k of every 8).
// Measured on B200 with the 32K-token workload: 2/8 -> 7.96 ms, 3/8 -> 8.31,
// 4/8 -> 8.89, against 7.6-8.0 ms with none: the epilogue is bound by
// instruction issue, not by the MUFU unit, so the extra FMA-pipe instructions
// cost more than they save.  Kept selectable; off.
constexpr int kFmaExp = 0;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

enum Mode { kStats = 0, kExtract = 1 };

struct Smem {
  uint8_t q[kTileBytes];
  uint8_t k[kStages][kTileBytes];
  // extraction: two staging tiles for TMA stores, each either two [128][64]
  // (B = 128) or four [64][64] (B = 64) bf16 sub-tiles, 128-byte swizzled
  uint8_t out[2][kTileBytes];
  float red[2][4][32];
  float2 xch[4][64];  // per-row (max, sum) exchange between the two warpgroups
  // extraction: cache entry of (row block a of this query tile, key block kb),
  // -1 where the block is not kept or not causal; read by every role instead
  // of the global block -> entry map
  int32_t slots[2][kMaxBlocksPerSeq];
  uint64_t q_full;
  uint64_t k_full[kStages];
  uint64_t k_empty[kStages];
  uint64_t s_full[2];
  uint64_t s_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
};

struct Params {
  const int32_t* cu_seqlens;
  const int32_t* tiles;    // [ntiles][2] = (sequence, 128-row tile), heaviest first
  const int64_t* cu_blk;   // [nseq+1]
  const int32_t* cu_qb;    // [nseq+1]
  int ntiles;
  int Hs;
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

// Does key tile kt hold a kept block of this query tile (extract) -- every
// causal key tile counts for the statistics.  `slots` is the CTA's copy of
// the block -> entry map (-1: not kept or not causal).
template <int MODE, int BB>
__device__ __forceinline__ bool tile_needed(const int32_t (*slots)[kMaxBlocksPerSeq], int kt) {
  if (MODE == kStats) return true;
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

__device__ __forceinline__ void named_sync_epilogue() {
  asm volatile("bar.sync 1, 256;" ::: "memory");
}

// One epilogue warpgroup (named barriers 6, 7).
__device__ __forceinline__ void group_sync(int wg) {
  asm volatile("bar.sync %0, 128;" ::"r"(6 + wg) : "memory");
}

// AND of a predicate over one epilogue warpgroup (named barriers 6, 7).
__device__ __forceinline__ bool group_all(int wg, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(uint32_t(v)), "r"(6 + wg)
      : "memory");
  return r != 0;
}

// The two epilogue warps of one TMEM lane quarter (named barriers 2..5).
__device__ __forceinline__ void pair_sync(int quarter) {
  asm volatile("bar.sync %0, 64;" ::"r"(2 + quarter) : "memory");
}

// AND of a predicate over the 256 epilogue threads (named barrier 1).
__device__ __forceinline__ bool epilogue_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 256, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(uint32_t(v))
      : "memory");
  return r != 0;
}

template <int MODE, int BB>
__global__ void __launch_bounds__(kThreads, 1)
    k_qk(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
         const __grid_constant__ CUtensorMap tmV, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
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
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sm.k_full[i], 1);
      mbar_init(&sm.k_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.s_empty[i], 128);
    }
    mbar_init(&sm.drain, 1);
    fence_barrier_init();
  }
  // global index of this sequence's query block 0; a query block outside
  // [qb_lo, qb_hi) is computed with its tile but nothing of it is written
  const int64_t gq0 = p.cu_qb[s];
  auto in_range = [&](int qb) { return gq0 + qb >= p.qb_lo && gq0 + qb < p.qb_hi; };
  if (MODE == kExtract) {
    const int64_t cb = p.cu_blk[s];
    for (int i = threadIdx.x; i < 2 * kMaxBlocksPerSeq; i += kThreads) {
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
        if (!tile_needed<MODE, BB>(sm.slots, kt)) continue;
        const int st = n % kStages;
        if (!mbar_wait(&sm.k_empty[st], ((n / kStages) & 1) ^ 1, p.status)) break;
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
        if (!tile_needed<MODE, BB>(sm.slots, kt)) continue;
        const int st = n % kStages, sb = n & 1;
        if (!mbar_wait(&sm.k_full[st], (n / kStages) & 1, p.status)) break;
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
      // every MMA issued above has completed once this arrives
      mma_commit(&sm.drain);
      mbar_wait(&sm.drain, 0, p.status);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    // Two warpgroups take turns: group wg handles the tiles n with n % 2 == wg
    // (S buffer wg), so one group's TMEM reads and exponentials overlap the
    // other's.  One query row per thread, the 128 columns in two 64-column
    // chunks.  Key blocks of different tiles are disjoint, so the groups only
    // merge their row (max, sum) once, at the end.
    const int wg = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // tile row
    const int ri = row0 + r;            // row within the sequence
    const bool valid = ri < L;
    const uint32_t lane_addr = tmem + (uint32_t(quarter * 32) << 16);
    const int W = p.band_width;
    const bool leader = (threadIdx.x & 127) == 0;  // lane 0 of the group's first warp
    float m_run = -CUDART_INF_F, l_run = 0.f;  // this group's online max and sum
    float lse2 = 0.f;
    if (MODE == kExtract) lse2 = valid ? p.lse[int64_t(h) * p.ntok + seq0 + ri] * kLog2e : 0.f;
    const int64_t cb = p.cu_blk[s];
    int n = 0;
    bool ok = true;
    for (int kt = 0; kt <= t; ++kt) {
      if (!tile_needed<MODE, BB>(sm.slots, kt)) continue;
      if ((n & 1) != wg) { ++n; continue; }
      const int sb = wg;
      bool got = mbar_wait(&sm.s_full[sb], (n >> 1) & 1, p.status);
      // the loop takes named barriers (extraction staging): leave it together
      got = group_all(wg, got);
      if (!got) { ok = false; break; }
      tc_fence_after();
      const int kbase0 = kt * kTile;
      const bool band_tile = row0 - (kbase0 + kTile - 1) < W;
      const bool diag = kt == t;
      const bool plain = !band_tile && !diag;
      const float sc = plain ? p.scale2 : 1.f;
      uint8_t* obuf = sm.out[wg];
      if (MODE == kExtract) {
        if (leader) bulk_wait_read<0>();  // this group's previous stores are done reading
        group_sync(wg);
      }
      float cm = 0.f, cs = 0.f;  // chunk 0 (max, sum) for a 128-key block
#pragma unroll 1
      for (int ch = 0; ch < 2; ++ch) {
        float v[64];
        tmem_ld32(lane_addr + sb * 128 + ch * 64, v);
        tmem_ld32(lane_addr + sb * 128 + ch * 64 + 32, v + 32);
        tmem_wait_ld();
        if (ch == 1) {
          tc_fence_before();
          mbar_arrive(&sm.s_empty[sb]);
        }
        // Logits in log2 units: x = s * scale2 (+ bias2 in the band), -inf
        // above the diagonal.  Tiles away from the band and the diagonal
        // ("plain", most of them) keep raw s and fold the scale into one FMA.
        const int kbase = kbase0 + ch * 64;  // key of v[0]
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
        if (MODE == kStats) {
          // row max over the chunk with three-input maxima in eight
          // independent chains, then eight independent partial sums
          float mx[8];
#pragma unroll
          for (int k = 0; k < 8; ++k)
            mx[k] = fmaxf(fmax3(fmax3(fmax3(v[k], v[8 + k], v[16 + k]), v[24 + k], v[32 + k]),
                                v[40 + k], v[48 + k]),
                          v[56 + k]);
          const float mt =
              fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) *
              sc;
          const float m_new = valid ? fmaxf(m_run, mt) : 0.f;
          // only masked keys seen so far (m = -inf): sum nothing
          const float m_use = m_new == -CUDART_INF_F ? 0.f : m_new;
          // pairs of columns on the packed f32x2 pipe: one instruction scales
          // and shifts two logits, one adds two exponentials
          float2 acc[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) acc[k] = make_float2(0.f, 0.f);
          const float2 sc2 = make_float2(sc, sc), nm2 = make_float2(-m_use, -m_use);
#pragma unroll
          for (int c = 0; c < 64; c += 8)
#pragma unroll
            for (int k = 0; k < 8; k += 2) {
              const float2 x = ffma2(make_float2(v[c + k], v[c + k + 1]), sc2, nm2);
              // kFmaExp of every 8 exponentials may run on the FMA pipe
              const float e0 = (k >= 8 - kFmaExp) ? exp2_fma(x.x) : ex2(x.x);
              const float e1 = (k + 1 >= 8 - kFmaExp) ? exp2_fma(x.y) : ex2(x.y);
              acc[k >> 1] = fadd2(acc[k >> 1], make_float2(e0, e1));
            }
          const float sh = ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) +
                           ((acc[2].x + acc[2].y) + (acc[3].x + acc[3].y));
          l_run = l_run * ex2(m_run - m_use) + sh;
          m_run = m_new;
          if (BB == 64) {
            // each chunk is one key block
            const float a = valid ? m_new + lg2(sh) : -CUDART_INF_F;
            tmem_st1(lane_addr + kAcol + 2 * kt + ch, a);
          } else if (ch == 0) {
            cm = m_new;
            cs = sh;
          } else {
            // the 128-key block: both chunks relative to the newer max
            const float tot = cs * ex2(cm - m_use) + sh;
            const float a = valid ? m_new + lg2(tot) : -CUDART_INF_F;
            tmem_st1(lane_addr + kAcol + kt, a);
          }
        } else {
          // Extraction into the group's staging tile, in the cache's own layout
          // for this head: one 128-byte line per (key group, 8-row slice,
          // half), 16-byte chunks permuted by h % 8.  B = 128: the tile is one
          // block (256 lines), this chunk fills key groups 4*ch..; B = 64:
          // sub-block (row half, key half = ch) holds 64 lines at
          // 8 KB * (2 * rowhalf + ch).  A row writes only into kept blocks of
          // its own query block (which must exist).
          const int rb = r & (BB - 1);                          // row within the block
          const int lrow = ((rb >> 3) << 1) + ((rb & 7) >> 2);  // line of this row, key group 0
          const int cbase = (rb & 3) << 1;                       // chunk of keys 0-7
          const int kb = (BB == 128) ? kt : 2 * kt + ch;
          if (sm.slots[(BB == 128) ? 0 : (r >> 6)][kb] >= 0) {  // kept (so causal, row exists)
            uint8_t* sub = obuf + ((BB == 128) ? 0 : ((r >> 6) * 2 + ch) * 8192);
#pragma unroll
            for (int kgl = 0; kgl < 4; ++kgl) {
              const int kg = (BB == 128) ? ch * 4 + kgl : kgl;
              uint8_t* line = sub + (kg * (BB / 4) + lrow) * 128;
#pragma unroll
              for (int c = 0; c < 2; ++c) {
                uint32_t w4[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  const int col = kgl * 16 + c * 8 + 2 * k;
                  const float2 x = ffma2(make_float2(v[col], v[col + 1]), make_float2(sc, sc),
                                         make_float2(-lse2, -lse2));
                  __nv_bfloat162 pr = __floats2bfloat162_rn(valid ? ex2(x.x) : 0.f,
                                                            valid ? ex2(x.y) : 0.f);
                  w4[k] = *reinterpret_cast<uint32_t*>(&pr);
                }
                *reinterpret_cast<uint4*>(line + (((cbase | c) ^ (h & 7)) << 4)) =
                    make_uint4(w4[0], w4[1], w4[2], w4[3]);
              }
            }
          }
        }
      }
      if (MODE == kExtract) {
        fence_proxy_async_smem();
        group_sync(wg);
        if (leader) {
#pragma unroll
          for (int a = 0; a < kTile / BB; ++a) {
#pragma unroll
            for (int b = 0; b < kTile / BB; ++b) {
              const int kbb = kt * (kTile / BB) + b;
              const int e = sm.slots[a][kbb];  // -1: not kept, not causal or no such row block
              if (e < 0) continue;
              const uint8_t* sub = obuf + ((BB == 128) ? 0 : (a * 2 + b) * 8192);
              tma_store_4d(&tmV, sub, 0, h, 0, int32_t(e));
            }
          }
          bulk_commit();
        }
      }
      ++n;
    }
    if (MODE == kExtract && leader) bulk_wait_all<0>();
    ok = epilogue_all(ok);  // uniform, so every thread takes the named barriers below
    if (MODE == kStats && ok) {
      // row log-sum-exp from the two groups' (max, sum)
      {
        float2* xs = sm.xch[quarter];
        xs[wg * 32 + lane] = make_float2(m_run, l_run);
        pair_sync(quarter);
        const float2 o = xs[(wg ^ 1) * 32 + lane];
        const float M = fmaxf(m_run, o.x);
        const float Mu = M == -CUDART_INF_F ? 0.f : M;
        const float l = l_run * ex2(m_run - Mu) + o.y * ex2(o.x - Mu);
        lse2 = valid ? M + lg2(l) : 0.f;
      }
      if (valid && wg == 0 && in_range(ri / BB)) p.lse[int64_t(h) * p.ntok + seq0 + ri] = lse2 * kLn2;
      tmem_wait_st();
      tc_fence_before();
      named_sync_epilogue();  // both groups' log partials are in TMEM
      tc_fence_after();
      // block masses: chunks of 32 key blocks, even chunks to group 0, odd to group 1
      const int nkb = (t + 1) * (kTile / BB);
      for (int c2 = 0; c2 < nkb; c2 += 64) {
        const int c0 = c2 + wg * 32;
        float a[32];
        tmem_ld32(lane_addr + kAcol + min(c0, 256 - 32), a);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k)
          a[k] = (valid && c0 + k < nkb) ? ex2(a[k] - lse2) : 0.f;
        const float tot = transpose_reduce32(a, lane);
        named_sync_epilogue();
        sm.red[wg][quarter][lane] = tot;
        named_sync_epilogue();
        if (quarter == 0 && c0 < nkb) {
          const int kb = c0 + lane;
          if (BB == 128) {
            const float m = (sm.red[wg][0][lane] + sm.red[wg][1][lane]) +
                            (sm.red[wg][2][lane] + sm.red[wg][3][lane]);
            if (kb <= t && in_range(t))
              p.part[int64_t(h) * p.nblocks + cb + int64_t(t) * (t + 1) / 2 + kb] = m;
          } else {
            const int qa = 2 * t, qbb = 2 * t + 1;
            const float m0 = sm.red[wg][0][lane] + sm.red[wg][1][lane];
            const float m1 = sm.red[wg][2][lane] + sm.red[wg][3][lane];
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

// y = exp2_fma(x), grid-stride (diagnostic entry point).
__global__ void k_exp2_fma_eval(const float* __restrict__ x, float* y, int64_t n) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += int64_t(gridDim.x) * blockDim.x)
    y[i] = exp2_fma(x[i]);
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

static cudaError_t launch_qk(int mode, const mf_attn_desc& d, const Sizes& sz, const QbRange& r,
                             const Meta& m, const void* Q, const void* K, float* lse,
                             float* part, const int32_t* slot, void* values, int64_t capacity,
                             cudaStream_t st) {
  if (r.ntiles == 0) return cudaSuccess;
  CUtensorMap tq, tk;
  const uint64_t cols = uint64_t(d.Hs) * d.d;
  cudaError_t e = make_tmap_2d_bf16(&tq, Q, uint64_t(sz.ntok), cols, 64, qk::kTile, true);
  if (e != cudaSuccess) return e;
  e = make_tmap_2d_bf16(&tk, K, uint64_t(sz.ntok), cols, 64, qk::kTile, true);
  if (e != cudaSuccess) return e;
  // the cache values viewed as (64 elements of a line, head, line (key group,
  // 8-row slice, half) of an entry, entry): one store writes all lines of one
  // (entry, head) -- extraction only
  CUtensorMap tv;
  memset(&tv, 0, sizeof(tv));
  if (mode == qk::kExtract) {
    if (capacity < 1) return cudaSuccess;
    const uint64_t nl = uint64_t(d.B) * uint64_t(d.B) / 64;  // lines per (entry, head)
    const uint64_t dims[4] = {64, uint64_t(d.Hs), nl, uint64_t(capacity)};
    const uint64_t strides[3] = {128, uint64_t(d.Hs) * 128, nl * uint64_t(d.Hs) * 128};
    const uint32_t box[4] = {64, 1, uint32_t(nl), 1};
    e = make_tmap_bf16(&tv, values, 4, dims, strides, box, 0);
    if (e != cudaSuccess) return e;
  }
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
  p.slot = slot;
  p.values = static_cast<__nv_bfloat16*>(values);
  p.qb_lo = r.qb_lo;
  p.qb_hi = r.qb_hi;
  p.status = status_word();
  const size_t smem = sizeof(qk::Smem) + 1024;
  const unsigned grid = unsigned(r.ntiles) * unsigned(d.Hs);
#define MF_QK(MODE, BB)                                                                       \
  do {                                                                                        \
    e = cudaFuncSetAttribute(qk::k_qk<MODE, BB>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                             int(smem));                                                      \
    if (e != cudaSuccess) return e;                                                           \
    qk::k_qk<MODE, BB><<<grid, qk::kThreads, smem, st>>>(tq, tk, tv, p);                      \
  } while (0)
  if (mode == qk::kStats) {
    if (d.B == 128) MF_QK(qk::kStats, 128); else MF_QK(qk::kStats, 64);
  } else {
    if (d.B == 128) MF_QK(qk::kExtract, 128); else MF_QK(qk::kExtract, 64);
  }
#undef MF_QK
  return cudaGetLastError();
}

cudaError_t launch_stats_tc(const mf_attn_desc& d, const Sizes& sz, const QbRange& r,
                            const Meta& m, const void* Q, const void* K, float* lse,
                            float* part, cudaStream_t st) {
  return launch_qk(qk::kStats, d, sz, r, m, Q, K, lse, part, nullptr, nullptr, 0, st);
}

cudaError_t launch_extract_tc(const mf_attn_desc& d, const Sizes& sz, const QbRange& r,
                              const Meta& m, const void* Q, const void* K, const float* lse,
                              const int32_t* slot, void* values, int64_t capacity,
                              cudaStream_t st) {
  return launch_qk(qk::kExtract, d, sz, r, m, Q, K, const_cast<float*>(lse), nullptr, slot,
                   values, capacity, st);
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
