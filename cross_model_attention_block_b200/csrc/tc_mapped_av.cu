// Fused map-mix x V on B200 (bf16, d = 128), both products on tcgen05.
//
// MapFlow article (163.com, section on the three system components, third
// component): the fused kernel reads the kept sparse blocks, forms the linear
// combination of sender heads into receiver heads on chip, and multiplies the
// result straight into the receiver's own V, accumulating the output, so the
// receiver's dense attention matrix is never formed in memory:
//
//   O_r[i,:] = sum_{kb kept} sum_{j in kb} (sum_h W[r,h] P_h[i,j]) V_{g(r)}[j,:]
//
// One CTA owns an 8-row slice of one query block and all Hr receiver heads,
// so every map byte is read from HBM once.  Kept key blocks are walked in
// stages of up to two 16-key groups (one where shared memory cannot hold two
// 32-key slots); per 16-key group a stage moves two contiguous chunks with
// plain bulk copies: the map slab (8 rows x 16 keys x Hs heads, stored by the
// cache in exactly the operand layout of the mixing MMA) and the V image of
// those 16 keys (prepared once per call by k_v_format).  Per 16-key group:
//   1. mix MMA   Mix[128 pairs x Hr] = Map[128 pairs x Hs] . W^T[Hs x Hr]
//      (tcgen05, M = 128 (row, key) pairs, K = Hs padded to a multiple of 16
//      with zero W rows; four stage accumulators in TMEM);
//   2. convert   eight warps read Mix from TMEM, round to bf16 and store it as
//      M^T_g[keys x 8 rows * G heads], the MN-major operand of step 3;
//   3. O MMAs    O^T_g[128 d x 8G] += V_g^T[128 x 16] . M^T_g[16 x 8G] for every
//      GQA group g (O^T of all groups resident in TMEM for the whole CTA).
// Two warps issue the MMAs, each from one elected lane, into disjoint
// accumulators: the mix warp runs ahead (gated by the map slab and by the
// converters releasing a mix buffer), the O warp takes each stage from the
// converters through a named barrier.  Descriptors are built once and only
// their address field moves.
//
// Why not mma.sync for the mix: on this part a legacy mma.sync takes a few
// thousand cycles from issue to result unless hundreds are in flight; with
// one stage's worth of work per warp that serialised the whole pipeline.
#include <cuda.h>
#include <cuda_bf16.h>

#include <cstring>

#include "mf_sm100.cuh"

namespace mf {
using namespace sm100;

namespace av {

constexpr int kRows = 8;   // query rows per CTA
constexpr int kKeys = 16;  // keys per 16-key group (a stage holds one or two)
constexpr int kD = 128;
constexpr int kThreads = 384;  // warps 0-3 roles, 4-11 converters (two per lane quarter)
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxMapStages = 8;
// Mix accumulators in TMEM: mix(n + kMixBufs) is issued as soon as stage n has
// been converted, so kMixBufs stages of MMA latency overlap the conversion.
constexpr int kMixBufs = 4;

struct Params {
  const int64_t* row_ptr;
  const int32_t* col_idx;
  const int32_t* qb_seq;
  const int32_t* qb_idx;
  const int32_t* cu_seqlens;
  const int32_t* cu_g;        // [nseq+1] prefix of ceil(L_s / 16)
  const uint8_t* vimg;        // [groups][4096 * Hkv] V operand images
  const __nv_bfloat16* values;
  const __nv_bfloat16* W;     // [Hr][Hs]
  __nv_bfloat16* O;           // [ntok][Hr][d]
  int64_t capacity;
  int64_t qb_hi;  // CTAs cover the global query blocks [qb_hi - grid / slices, qb_hi)
  int Hs, Hs_pad, Hr, Hkv, G, B;
  uint32_t map_bytes;       // Hs * 256: one 16-key group's slab
  uint32_t map_slot;        // KG slabs + 1 KB guard, 1 KB aligned
  uint32_t v_bytes;         // 4096 * Hkv: one 16-key group's V image
  uint32_t v_slot;          // KG images
  uint32_t mt_group_stride, mt_bytes, w_bytes;
  uint32_t off_v, off_map, off_mt, off_w, off_kb, off_bar;
  int map_stages, vm_stages;
  unsigned* status;
};

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Named barriers 1 and 2 (by stage parity) hand stage n from the converters
// to the O warp: both sides bar.sync once per stage, so neither can run a
// phase ahead, also when a timed-out wait makes the rest of the walk a no-op.
constexpr int kBarMt = 1;
constexpr int kConverterWarps = 8;
constexpr int kHandOff = kConverterWarps * 32 + 32;  // named-barrier count: converters + O warp

// bar.sync is warp-aligned: a warp that reaches it split (after a spin wait
// or a one-lane branch) would be counted once per piece, so converge first.
__device__ __forceinline__ void named_sync(int id, int count) {
  __syncwarp();
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred P;\n\telect.sync _|P, 0xffffffff;\n\tselp.b32 %0, 1, 0, P;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

// Ring position: slot and the parity of its current use, advanced without
// division (stage counters never feed a divide in the issue path).
struct Ring {
  int slot = 0;
  uint32_t phase = 0;
  int size;
  __device__ explicit Ring(int n) : size(n) {}
  __device__ void next() {
    if (++slot == size) {
      slot = 0;
      phase ^= 1u;
    }
  }
};

// 16-key groups of key block kb that hold keys of the sequence.
__device__ __forceinline__ int key_groups_of(int kb, int B, int L) {
  const int rem = L - kb * B;
  return rem <= 0 ? 0 : min(B, rem + kKeys - 1) / kKeys;
}

// A stage is up to KG consecutive 16-key groups of one kept entry of the
// CTA's query block (the last stage of an entry may hold fewer); every role
// walks the same list, read from the kept-block list in shared memory.
template <int KG>
struct Stages {
  const int32_t* kb_list;
  int nE, B, L;
  int e = -1, kb = 0, kg0 = 0, nkg = 0;
  __device__ Stages(const int32_t* list, int n, int b, int l) : kb_list(list), nE(n), B(b), L(l) {}
  __device__ bool next() {
    kg0 += KG;
    while (kg0 >= nkg) {
      if (++e >= nE) return false;
      kb = kb_list[e];
      nkg = key_groups_of(kb, B, L);
      kg0 = 0;
    }
    return true;
  }
  __device__ int nk() const { return min(KG, nkg - kg0); }  // groups in this stage
};

template <int HR, int G, int KG>
__global__ void __launch_bounds__(kThreads, 1) k_mapped_av(const Params p) {
  constexpr int HKV = HR / G;
  constexpr int NO = kRows * G;          // O MMA N per group
  constexpr uint32_t kMixCol = 8u * HR;  // first TMEM column of the mix accumulators
  constexpr uint32_t kMixCols = KG * HR;  // one stage's mix accumulator (KG M-tiles)
  static_assert(kMixCol + kMixBufs * kMixCols <= kTmemCols, "O^T and mix accumulators exceed TMEM");
  static_assert((kMixBufs & (kMixBufs - 1)) == 0, "kMixBufs must be a power of two");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int MS = p.map_stages, VS = p.vm_stages;
  uint64_t* map_full = reinterpret_cast<uint64_t*>(base + p.off_bar);  // [MS]
  uint64_t* map_empty = map_full + MS;                                  // [MS]
  // V ring: one barrier pair per 16-key half of a slot, so a half is refilled
  // as soon as the O products that read it are done
  uint64_t* v_full = map_empty + MS;                                    // [VS][KG]
  uint64_t* vm_empty = v_full + VS * KG;                                // [VS][KG]
  uint64_t* mix_full = vm_empty + VS * KG;                              // [kMixBufs]
  uint64_t* mix_empty = mix_full + kMixBufs;                            // [kMixBufs]
  uint64_t* final_bar = mix_empty + kMixBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(final_bar + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* s_kb = reinterpret_cast<int32_t*>(base + p.off_kb);  // kept key blocks of the row

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slices = p.B / kRows;
  const int64_t gqb = p.qb_hi - 1 - blockIdx.x / slices;  // longest rows first
  const int slice = blockIdx.x % slices;
  const int s = p.qb_seq[gqb], qb = p.qb_idx[gqb];
  const int seq0 = p.cu_seqlens[s];
  const int L = p.cu_seqlens[s + 1] - seq0;
  const int i0 = qb * p.B + slice * kRows;  // first row (in the sequence)
  if (i0 >= L) return;                      // the whole slice is past the sequence end
  const int64_t e0 = p.row_ptr[gqb];
  int nE = int(max(int64_t(0), min(p.row_ptr[gqb + 1], p.capacity) - e0));
  if (nE > qb + 1) {  // a causal row holds at most qb + 1 key blocks
    if (threadIdx.x == 0) atomicOr(p.status, kStatusBadCache);
    nE = qb + 1;
  }

  for (int e = threadIdx.x; e < nE; e += kThreads) s_kb[e] = p.col_idx[e0 + e];
  if (threadIdx.x == 0) {
    for (int i = 0; i < MS; ++i) {
      mbar_init(&map_full[i], 1);
      mbar_init(&map_empty[i], 1);
    }
    for (int i = 0; i < VS * KG; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&vm_empty[i], 1);
    }
    for (int i = 0; i < kMixBufs; ++i) {
      mbar_init(&mix_full[i], 1);
      mbar_init(&mix_empty[i], kConverterWarps);
    }
    mbar_init(final_bar, 1);
    *abort = 0;
    fence_barrier_init();
  }
  // W^T as the K-major operand [Hr rows][Hs_pad], core matrices of 8 rows x 16
  // bytes, K chunks 128 bytes apart, row groups Hs_pad * 16 bytes apart; zero
  // past Hs.  The map ring is zeroed: the padded K step of the mix reads past
  // a slab (into the next slab or the 1 KB guard), where it must meet finite
  // values for the zero rows of W^T to cancel them.
  {
    uint8_t* wt = base + p.off_w;
    for (int idx = threadIdx.x; idx < HR * p.Hs_pad; idx += kThreads) {
      const int r = idx / p.Hs_pad, h = idx % p.Hs_pad;
      const __nv_bfloat16 w = h < p.Hs ? p.W[r * p.Hs + h] : __float2bfloat16_rn(0.f);
      *reinterpret_cast<__nv_bfloat16*>(wt + (r >> 3) * (p.Hs_pad * 16) + (h >> 3) * 128 +
                                        (r & 7) * 16 + (h & 7) * 2) = w;
    }
    uint4* ring = reinterpret_cast<uint4*>(base + p.off_map);
    for (uint32_t k = threadIdx.x; k < uint32_t(MS) * p.map_slot / 16u; k += kThreads)
      ring[k] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sbase = smem_u32(base);
  const int S8 = p.B / 8, S16 = p.B / kKeys;
  // a wait that gave up makes every later wait of the CTA give up at once, so
  // the named-barrier hand-offs below still run to the end without blocking
  auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (*abort) return false;
    if (mbar_wait(bar, parity, p.status)) return true;
    *abort = 1;
    return false;
  };

  if (warp == 0) {
    // ------------------------------------------------------- map producer
    if (lane == 0) {
      Ring ring(MS);
      Stages<KG> st(s_kb, nE, p.B, L);
      while (st.next()) {
        if (!wait(&map_empty[ring.slot], ring.phase ^ 1u)) break;
        const int nk = st.nk();
        mbar_expect_tx(&map_full[ring.slot], uint32_t(nk) * p.map_bytes);
        for (int h = 0; h < nk; ++h) {
          const int64_t line0 = (((e0 + st.e) * S16 + st.kg0 + h) * S8 + slice) * 2 * p.Hs;
          bulk_load(base + p.off_map + ring.slot * p.map_slot + h * p.map_bytes,
                    p.values + line0 * 64, p.map_bytes, &map_full[ring.slot]);
        }
        ring.next();
      }
    }
  } else if (warp == 2) {
    // --------------------------------------------------------- V producer
    if (lane == 0) {
      Ring ring(VS);
      Stages<KG> st(s_kb, nE, p.B, L);
      const int64_t g0 = p.cu_g[s];
      bool live = true;
      while (live && st.next()) {
        const int nk = st.nk();
        const int64_t grp = g0 + int64_t(st.kb) * S16 + st.kg0;
        for (int h = 0; h < KG; ++h) {
          uint64_t* full = &v_full[ring.slot * KG + h];
          if (!wait(&vm_empty[ring.slot * KG + h], ring.phase ^ 1u)) {
            live = false;
            break;
          }
          // a half past the stage's groups still completes its phase (no bytes)
          mbar_expect_tx(full, h < nk ? p.v_bytes : 0u);
          if (h < nk)
            bulk_load(base + p.off_v + ring.slot * p.v_slot + h * p.v_bytes,
                      p.vimg + (grp + h) * p.v_bytes, p.v_bytes, full);
        }
        ring.next();
      }
    }
  } else if (warp == 1 || warp == 3) {
    // ------------------------------------------------- O warp / mix warp
    // Two issuing warps with disjoint accumulators: warp 1 issues the O
    // products (accumulating O^T), warp 3 the head mix (into the four mix
    // buffers), each from one elected lane while the warp walks the stages
    // converged.  Descriptors are built once, per MMA only the start-address
    // field moves (added in 16-byte units, never carrying out of its 14
    // bits), and ring positions advance without division.  The mix warp runs
    // up to kMixBufs stages ahead, gated by the map slab and by the
    // converters releasing the buffer; the O warp takes each stage from the
    // converters through the named barrier.
    // Operands of tcgen05.mma live in uniform registers: derive every base
    // from values the compiler can see are warp-uniform.
    const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
    const uint32_t sb = __shfl_sync(0xffffffffu, sbase, 0);
    Stages<KG> st(s_kb, nE, p.B, L);
    if (warp == 3) {
      const uint32_t idesc_mix = idesc_bf16(128, HR, 1, 0);  // A MN-major, B K-major
      const int ksteps = p.Hs_pad / 16;                     // 1..4
      const uint64_t mix_a0 = smem_desc(sb + p.off_map, p.Hs * 128, 1024, kSwizzle128);
      const uint64_t mix_b0 = smem_desc(sb + p.off_w, 128, p.Hs_pad * 16, kSwizzleNone);
      const uint32_t map_step = p.map_slot >> 4, map_half = p.map_bytes >> 4;
      Ring mring(MS);
      int m = 0;
      while (st.next()) {
        const int db = m & (kMixBufs - 1);
        if (elect_one()) {
          // the map slab arrives by bulk copy (async proxy, ordered by its
          // mbarrier); the converters' TMEM reads of the buffer's previous
          // stage are ordered by mix_empty and the fence
          const bool ok = wait(&map_full[mring.slot], mring.phase) &&
                          wait(&mix_empty[db], (uint32_t(m / kMixBufs) & 1u) ^ 1u);
          tc_fence_after();
          if (ok) {
            const uint64_t a = mix_a0 + uint64_t(mring.slot) * map_step;
            const uint32_t d = tm + kMixCol + uint32_t(db) * kMixCols;
            const int nk = st.nk();
#pragma unroll
            for (int h = 0; h < KG; ++h)
              if (h < nk)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                  if (kk < ksteps)
                    mma_bf16_ss(d + h * HR, a + h * map_half + kk * (2048 >> 4),
                                mix_b0 + kk * (256 >> 4), idesc_mix, kk > 0);
            mma_commit(&map_empty[mring.slot]);
            mma_commit(&mix_full[db]);
          }
        }
        __syncwarp();
        mring.next();
        ++m;
      }
    } else {
      const uint32_t idesc_o = idesc_bf16(128, NO, 1, 1);  // A, B MN-major
      const uint64_t o_a0 = smem_desc(sb + p.off_v, 2048, 1024, kSwizzle128);
      const uint64_t o_b0 = smem_desc(sb + p.off_mt, 128, KG * 256, kSwizzleNone);
      const uint32_t v_step = p.v_slot >> 4, v_half = p.v_bytes >> 4,
                     mt_step = p.mt_bytes >> 4, mtg_step = p.mt_group_stride >> 4;
      Ring vring(VS);
      int n = 0;
      while (st.next()) {
        named_sync(kBarMt + (n & 1), kHandOff);  // stage n's M^T is written
        tc_fence_after();
        if (elect_one()) {
          const uint64_t a = o_a0 + uint64_t(vring.slot) * v_step;
          const uint64_t b = o_b0 + uint64_t(vring.slot) * mt_step;
          const int nk = st.nk();
#pragma unroll
          for (int h = 0; h < KG; ++h) {
            // each half of the V slot is waited for, consumed and released on
            // its own; a half past the stage's groups only passes its phase
            if (wait(&v_full[vring.slot * KG + h], vring.phase) && h < nk) {
#pragma unroll
              for (int g = 0; g < HKV; ++g)
                mma_bf16_ss(tm + g * NO, a + h * v_half + g * (4096 >> 4),
                            b + uint64_t(g) * mtg_step + h * (256 >> 4), idesc_o,
                            n > 0 || h > 0);
            }
            mma_commit(&vm_empty[vring.slot * KG + h]);
          }
        }
        __syncwarp();
        vring.next();
        ++n;
      }
      if (elect_one()) mma_commit(final_bar);
      __syncwarp();
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ converters
    // One thread per mix-accumulator lane = (row, key) pair of each M-tile;
    // the two warps of a lane quarter split the receiver heads (columns).
    constexpr int HH = HR / 2;  // heads per converter warp
    const int q = warp & 3;     // TMEM lane quarter: pairs 32q .. 32q+31
    const int hh = (warp - 4) >> 2;
    const int m = q * 32 + lane;
    const int r8 = m >> 4, k16 = m & 15;
    const uint32_t lane_addr = tmem + (uint32_t(q * 32) << 16);
    const bool row_ok = i0 + r8 < L;
    uint8_t* mt0 = base + p.off_mt + (k16 >> 3) * 128 + (k16 & 7) * 16 +
                   (hh * (HH / G)) * p.mt_group_stride;
    Ring vring(VS);
    Stages<KG> st(s_kb, nE, p.B, L);
    int n = 0;
    while (st.next()) {
      const int db = n & (kMixBufs - 1);
      if (wait(&mix_full[db], uint32_t(n / kMixBufs) & 1u)) {
        tc_fence_after();
        // the M^T slot is free once all of O(n - VS) is done: its last half's commit
        if (wait(&vm_empty[vring.slot * KG + KG - 1], vring.phase ^ 1u)) {
          const int nk = st.nk();
          uint8_t* mt = mt0 + vring.slot * p.mt_bytes;
#pragma unroll
          for (int h = 0; h < KG; ++h) {
            if (h < nk) {
              float v[HH];
              const uint32_t col = lane_addr + kMixCol + db * kMixCols + h * HR + hh * HH;
              if constexpr (HH == 16) {
                tmem_ld16(col, v);
              } else {
                tmem_ld8(col, v);
              }
              tmem_wait_ld();
              if (h + 1 == nk) {  // the stage's mix buffer is read: release it
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&mix_empty[db]);
              }
              const int key = st.kb * p.B + (st.kg0 + h) * kKeys + k16;
              const bool keep = key < L && row_ok;  // select, never multiply stale values
#pragma unroll
              for (int r = 0; r < HH; r += 2) {
                const int g = r / G, rl = r % G;  // group relative to this warp's first
                const int nn = r8 * G + rl;       // MMA N index of (row r8, head)
                *reinterpret_cast<uint32_t*>(mt + h * 256 + g * p.mt_group_stride +
                                             (nn >> 3) * (KG * 256) + ((nn & 7) << 1)) =
                    keep ? pack_bf16(v[r], v[r + 1]) : 0u;
              }
            }
          }
          fence_proxy_async_smem();
        }
      }
      tc_fence_before();
      named_sync(kBarMt + (n & 1), kHandOff);  // hand stage n to the O warp
      vring.next();
      ++n;
    }
    // ------------------------------------------------------------ epilogue
    // O^T of the GQA groups g with g % 2 == hh (TMEM lane = d), stored to O.
    const int c = q * 32 + lane;  // d index
    const bool ok = wait(final_bar, 0);
    tc_fence_after();
#pragma unroll 1
    for (int g = hh; g < HKV; g += 2) {
#pragma unroll
      for (int c0 = 0; c0 < NO; c0 += 16) {
        float o[16];
        tmem_ld16(lane_addr + g * NO + c0, o);
        tmem_wait_ld();
        if (!ok || n == 0) {
#pragma unroll
          for (int k = 0; k < 16; ++k) o[k] = 0.f;
        }
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const int nn = c0 + k;
          const int i = nn / G, rl = nn % G;
          const int row = i0 + i;
          if (row < L)
            p.O[(int64_t(seq0 + row) * HR + g * G + rl) * kD + c] = __float2bfloat16_rn(o[k]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// Prefix sums of 16-key groups per sequence.
__global__ void k_group_meta(int nseq, const int32_t* __restrict__ cu_seqlens, int32_t* cu_g) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  int32_t g = 0;
  cu_g[0] = 0;
  for (int s = 0; s < nseq; ++s) {
    g += (cu_seqlens[s + 1] - cu_seqlens[s] + 15) / 16;
    cu_g[s + 1] = g;
  }
}

// V regrouped per (sequence, 16-key group) into the image the O MMA reads as
// its A operand: chunk (group g, d half) of 16 keys x 64 d, rows of 128 bytes,
// 16-byte chunk index XOR key % 8 (128-byte swizzle).  Keys past the sequence
// end are zero.  One CTA per image.
__global__ void __launch_bounds__(256) k_v_format(
    const __nv_bfloat16* __restrict__ V, const int32_t* __restrict__ page_table, int page_size,
    int max_pages, const int32_t* __restrict__ cu_seqlens, const int32_t* __restrict__ cu_g,
    int nseq, int Hkv, uint8_t* __restrict__ out) {
  const int64_t grp = blockIdx.x;
  const int s = upper_index(cu_g, nseq, grp);
  const int kg = int(grp - cu_g[s]);
  const int seq0 = cu_seqlens[s];
  const int L = cu_seqlens[s + 1] - seq0;
  const int chunks_per_key = Hkv * 16;  // 16-byte chunks of one key row (Hkv x 128 x 2 B)
  const uint32_t img = 4096u * uint32_t(Hkv);
  uint8_t* dst = out + grp * int64_t(img);
  for (int q = threadIdx.x; q < kKeys * chunks_per_key; q += blockDim.x) {
    const int k = q / chunks_per_key, cc = q % chunks_per_key;
    const int j = kg * kKeys + k;
    uint4 val = make_uint4(0, 0, 0, 0);
    if (j < L) {
      int64_t row;
      if (page_table) {
        const int page = page_table[int64_t(s) * max_pages + j / page_size];
        row = int64_t(page) * page_size + (j % page_size);
      } else {
        row = seq0 + j;
      }
      val = reinterpret_cast<const uint4*>(V + row * int64_t(Hkv) * kD)[cc];
    }
    const int g = cc >> 4, dch = cc & 15;  // group, 16-byte chunk of the 128 d
    const int half = dch >> 3, c8 = dch & 7;
    const uint32_t o = uint32_t((2 * g + half) * 2048 + k * 128 + ((c8 ^ (k & 7)) << 4));
    *reinterpret_cast<uint4*>(dst + o) = val;
  }
}

}  // namespace av

// ------------------------------------------------------------------- host side

namespace {
// Shared-memory plan of the fused kernel for one shape: stage width (KG
// 16-key groups), ring depths and region offsets, written into p.  Returns
// KG, or 0 when nothing fits.  p.Hs_pad and p.G must be set.
int plan_layout(av::Params& p, int Hs, int Hr, int Hkv, size_t& smem) {
  p.map_bytes = 256u * uint32_t(Hs);
  p.v_bytes = 4096u * uint32_t(Hkv);
  p.w_bytes = (uint32_t(Hr) * uint32_t(p.Hs_pad) * 2u + 127u) & ~127u;
  const uint32_t kb_bytes = 512u * 4u;  // kept key blocks of one row (L <= 512 B)
  const size_t budget = 227u * 1024u - 1024u - 512u - p.w_bytes - kb_bytes;
  // Stages of 32 keys (two 16-key groups) when two V / M^T slots and two map
  // slots fit: half the per-stage waits, commits and hand-offs of 16-key
  // stages.  Otherwise 16-key stages with the deepest rings that fit.
  int kg = 0, ms = 0, vs = 0;
  for (int cand_kg = 2; cand_kg >= 1 && ms == 0; --cand_kg) {
    const uint32_t map_slot = (uint32_t(cand_kg) * p.map_bytes + 1024u + 1023u) & ~1023u;
    const uint32_t mtg = uint32_t(cand_kg) * 256u * uint32_t(p.G) + 16u;
    const uint32_t mt_bytes = (uint32_t(Hkv) * mtg + 127u) & ~127u;
    const uint32_t v_slot = uint32_t(cand_kg) * p.v_bytes;
    for (int cand_vs = (cand_kg == 2 ? 2 : 4); cand_vs >= 2 && ms == 0; --cand_vs) {
      const size_t fixed = size_t(cand_vs) * (v_slot + mt_bytes);
      for (int cand_ms = av::kMaxMapStages; cand_ms >= 2; --cand_ms)
        if (fixed + size_t(cand_ms) * map_slot <= budget) {
          kg = cand_kg;
          ms = cand_ms;
          vs = cand_vs;
          p.map_slot = map_slot;
          p.mt_group_stride = mtg;
          p.mt_bytes = mt_bytes;
          p.v_slot = v_slot;
          break;
        }
    }
  }
  if (ms == 0) return 0;
  p.map_stages = ms;
  p.vm_stages = vs;
  p.off_v = 0;
  p.off_map = vs * p.v_slot;
  p.off_mt = p.off_map + ms * p.map_slot;
  p.off_w = p.off_mt + vs * p.mt_bytes;
  p.off_kb = p.off_w + p.w_bytes;
  p.off_bar = (p.off_kb + kb_bytes + 7u) & ~7u;
  smem =
      size_t(p.off_bar) + (2 * ms + 2 * vs * kg + 2 * av::kMixBufs + 1) * 8 + 32 + 1024;
  return kg;
}
}  // namespace

bool mapped_av_tc_supported(const mf_attn_desc& d, int Hr, const mf_v_desc& v) {
  if (d.dt != MF_BF16 || d.d != 128 || v.d != 128) return false;
  if (d.Hs % 8 != 0 || d.Hs > 64) return false;
  if ((Hr != 16 && Hr != 32) || v.Hkv < 1 || Hr % v.Hkv != 0) return false;
  const int G = Hr / v.Hkv;
  return G == 2 || G == 4 || G == 8;
}

size_t mapped_av_tc_workspace(int nseq, int64_t key_groups, int Hkv) {
  const size_t meta = (size_t(nseq + 1) * 4 + 255) & ~size_t(255);
  return meta + size_t(key_groups) * 4096u * size_t(Hkv) + 1024;
}

cudaError_t launch_mapped_av_tc(const mf_csr_cache& c, const mf_attn_desc& d, const Sizes& sz,
                                int Hr, const void* W, const mf_v_desc& v, void* O, void* ws,
                                int64_t key_groups, int64_t qb_lo, int64_t qb_hi,
                                cudaStream_t st) {
  if (c.nnz_capacity < 1 || qb_hi <= qb_lo || key_groups == 0) return cudaSuccess;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  int32_t* cu_g = reinterpret_cast<int32_t*>(wsb);
  const size_t meta = (size_t(d.nseq + 1) * 4 + 255) & ~size_t(255);
  uint8_t* vimg = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(wsb + meta) + 1023) &
                                             ~uintptr_t(1023));
  av::k_group_meta<<<1, 32, 0, st>>>(d.nseq, d.cu_seqlens, cu_g);
  av::k_v_format<<<unsigned(key_groups), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(v.V), v.page_table, v.page_table ? v.page_size : 16,
      v.max_pages_per_seq, d.cu_seqlens, cu_g, d.nseq, v.Hkv, vimg);

  av::Params p{};
  p.row_ptr = c.row_ptr;
  p.col_idx = c.col_idx;
  p.qb_seq = c.qb_seq;
  p.qb_idx = c.qb_idx;
  p.cu_seqlens = d.cu_seqlens;
  p.cu_g = cu_g;
  p.vimg = vimg;
  p.values = static_cast<const __nv_bfloat16*>(c.values);
  p.W = static_cast<const __nv_bfloat16*>(W);
  p.O = static_cast<__nv_bfloat16*>(O);
  p.capacity = c.nnz_capacity;
  p.qb_hi = qb_hi;
  p.Hs = d.Hs;
  p.Hs_pad = (d.Hs + 15) / 16 * 16;
  p.Hr = Hr;
  p.Hkv = v.Hkv;
  p.G = Hr / v.Hkv;
  p.B = d.B;
  p.status = status_word();
  size_t smem = 0;
  const int kg = plan_layout(p, d.Hs, Hr, v.Hkv, smem);
  if (kg == 0) return cudaErrorInvalidConfiguration;
  const unsigned grid = unsigned(qb_hi - qb_lo) * unsigned(d.B / av::kRows);
  cudaError_t e = cudaSuccess;
#define MF_AV(HR, G, KG)                                                                    \
  do {                                                                                      \
    e = cudaFuncSetAttribute(av::k_mapped_av<HR, G, KG>,                                    \
                             cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));       \
    if (e != cudaSuccess) return e;                                                         \
    av::k_mapped_av<HR, G, KG><<<grid, av::kThreads, smem, st>>>(p);                        \
  } while (0)
#define MF_AV_G(HR, KG)                                                                     \
  do {                                                                                      \
    if (p.G == 2) MF_AV(HR, 2, KG); else if (p.G == 4) MF_AV(HR, 4, KG); else MF_AV(HR, 8, KG); \
  } while (0)
  if (Hr == 32) {
    if (kg == 2) MF_AV_G(32, 2); else MF_AV_G(32, 1);
  } else {
    if (kg == 2) MF_AV_G(16, 2); else MF_AV_G(16, 1);
  }
#undef MF_AV_G
#undef MF_AV
  return cudaGetLastError();
}

bool mapped_av_tc_plan(int Hs, int Hr, int Hkv, int32_t out[8]) {
  av::Params p{};
  p.Hs_pad = (Hs + 15) / 16 * 16;
  p.G = Hr / Hkv;
  size_t smem = 0;
  const int kg = plan_layout(p, Hs, Hr, Hkv, smem);
  if (kg == 0) return false;
  out[0] = kg;
  out[1] = p.map_stages;
  out[2] = p.vm_stages;
  out[3] = int32_t(smem);
  out[4] = int32_t(p.off_map);
  out[5] = int32_t(p.off_mt);
  out[6] = int32_t(p.off_w);
  out[7] = int32_t(p.off_bar);
  return true;
}

}  // namespace mf
