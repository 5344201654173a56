// Fused map-mix x V on B200 (bf16, d = 128).
//
// MapFlow article (163.com, section on the three system components, third
// component): the fused kernel reads the kept sparse blocks, forms the linear
// combination of sender heads into receiver heads on chip, and multiplies the
// result straight into the receiver's own V, accumulating the output, so the
// receiver's dense attention matrix is never formed in memory:
//
//   O_r[i,:] = sum_{kb kept} sum_{j in kb} (sum_h W[r,h] P_h[i,j]) V_{g(r)}[j,:]
//
// One CTA owns a 16-row slice of one query block and all Hr receiver heads, so
// every map byte is read from HBM once.  The kept key blocks are walked in
// stages of 16 keys:
//  * warp 0 (one thread) TMA-loads the map slab [16 rows][Hs][16 keys] with one
//    4-D box (hardware 32-byte swizzle) and V [16 keys][Hkv][128] with one 3-D
//    box (128-byte swizzle; with paged V the 16 keys are one page);
//  * warps 4..7 mix: mma.sync m16n8k16 with the map slab as A (keys x heads,
//    loaded transposed by ldmatrix) and W^T held in registers as B, giving the
//    mixed map M (16 keys x Hr heads per row), written as bf16 into the
//    MN-major B operand of the next product;
//  * warp 1 (one thread) issues, per GQA group g, one tcgen05.mma
//    O^T_g[128 x 16G] += V_g^T[128 x 16] M^T_g[16 x 16G] (M = d = 128, N = 16
//    rows x G heads), with O^T for all groups resident in the 512 TMEM columns;
//  * at the end warps 4..7 read O^T from TMEM (lane = d) and store O.
#include <cuda.h>
#include <cuda_bf16.h>

#include <cstring>

#include "mf_sm100.cuh"

namespace mf {
using namespace sm100;

namespace av {

constexpr int kRows = 16;      // query rows per CTA
constexpr int kKeys = 16;      // keys per stage (= MMA K)
constexpr int kD = 128;
constexpr int kMaxStages = 3;
constexpr int kThreads = 256;
constexpr uint32_t kTmemCols = 512;

struct Params {
  const int64_t* row_ptr;
  const int32_t* col_idx;
  const int32_t* qb_seq;
  const int32_t* qb_idx;
  const int32_t* cu_seqlens;
  const int32_t* page_table;  // NULL: contiguous V
  const __nv_bfloat16* W;     // [Hr][Hs]
  __nv_bfloat16* O;           // [ntok][Hr][d]
  int64_t capacity;
  int64_t nqb;
  int Hs, Hr, Hkv, G, B;
  int page_size, max_pages;
  // shared-memory layout (bytes from the 1024-aligned base)
  uint32_t off_v, off_map, off_mt, v_bytes, map_bytes, mt_bytes, mt_group_stride;
  uint32_t off_bar;
  int stages;  // pipeline depth (2 or 3, whatever fits in shared memory)
  unsigned* status;
};

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& a0, uint32_t& a1, uint32_t& a2,
                                          uint32_t& a3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(a0), "=r"(a1), "=r"(a2), "=r"(a3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x2_t(uint32_t addr, uint32_t& a0, uint32_t& a1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
               : "=r"(a0), "=r"(a1)
               : "r"(addr));
}

__device__ __forceinline__ void mma16816(float* c, uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma1688(float* c, uint32_t a0, uint32_t a1, uint32_t b0) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(b0));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Address of 16-byte chunk c (keys 8c..8c+7) of line (row i, head h) in the
// map slab: lines of 32 bytes, 32-byte swizzle (chunk bit flips on line bit 2).
__device__ __forceinline__ uint32_t map_addr(uint32_t base, int line, int c) {
  return base + line * 32 + ((c ^ ((line >> 2) & 1)) << 4);
}

// Stage walk: (entry e, key group kg) pairs of this query block, skipping key
// groups that start past the sequence end.
struct Walk {
  int64_t e, e1;
  int kg, nkg, kb;
  int B, L;
  const int32_t* col_idx;
  __device__ bool next() {
    while (true) {
      if (kg + 1 < nkg) { ++kg; return true; }
      ++e;
      if (e >= e1) return false;
      kb = col_idx[e];
      int rem = L - kb * B;
      nkg = (min(rem, B) + kKeys - 1) / kKeys;
      kg = -1;
      if (nkg <= 0) { nkg = 0; continue; }
    }
  }
};

__device__ __forceinline__ Walk make_walk(const Params& p, int64_t gqb, int L) {
  Walk w;
  w.e = p.row_ptr[gqb] - 1;
  w.e1 = min(p.row_ptr[gqb + 1], p.capacity);
  w.kg = 0;
  w.nkg = 0;
  w.kb = 0;
  w.B = p.B;
  w.L = L;
  w.col_idx = p.col_idx;
  return w;
}

__global__ void __launch_bounds__(kThreads, 1)
    k_mapped_av(const __grid_constant__ CUtensorMap tmMap, const __grid_constant__ CUtensorMap tmV,
                const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int kStages = p.stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(base + p.off_bar);  // [stages]
  uint64_t* mt_ready = full + kStages;                              // [stages]
  uint64_t* done = mt_ready + kStages;                              // [stages]
  uint64_t* final_bar = done + kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(final_bar + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slices = p.B / kRows;
  const int64_t gqb = p.nqb - 1 - blockIdx.x / slices;  // longest rows first
  const int slice = blockIdx.x % slices;
  const int s = p.qb_seq[gqb], qb = p.qb_idx[gqb];
  const int seq0 = p.cu_seqlens[s];
  const int L = p.cu_seqlens[s + 1] - seq0;
  const int i0 = qb * p.B + slice * kRows;  // first row (in the sequence)
  if (i0 >= L) return;                      // the whole slice is past the sequence end

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&mt_ready[i], 4);
      mbar_init(&done[i], 1);
    }
    mbar_init(final_bar, 1);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sbase = smem_u32(base);
  const int N = kRows * p.G;  // MMA N per group

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmMap);
      tma_prefetch_desc(&tmV);
      Walk wk = make_walk(p, gqb, L);
      int n = 0;
      while (wk.next()) {
        const int st = n % kStages;
        if (!mbar_wait(&done[st], ((n / kStages) & 1) ^ 1, p.status)) break;
        // exact bytes of the two boxes: 16 keys x Hs x 16 rows, 16 keys x Hkv x 128
        mbar_expect_tx(&full[st], uint32_t(512 * p.Hs) + uint32_t(4096 * p.Hkv));
        // map slab: keys 16kg.., all heads, rows 16*slice.., entry e
        asm volatile(
            "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
            " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(sbase + p.off_map + st * p.map_bytes),
            "l"(reinterpret_cast<uint64_t>(&tmMap)), "r"(smem_u32(&full[st])),
            "r"(wk.kg * kKeys), "r"(0), "r"(slice * kRows), "r"(int32_t(wk.e))
            : "memory");
        // V rows of these 16 keys
        const int j = wk.kb * p.B + wk.kg * kKeys;  // key (in the sequence)
        int row;
        if (p.page_table) {
          const int page = p.page_table[int64_t(s) * p.max_pages + j / p.page_size];
          row = page * p.page_size + (j % p.page_size);
        } else {
          row = seq0 + j;
        }
        tma_load_3d(base + p.off_v + st * p.v_bytes, &tmV, &full[st], 0, row, 0);
        ++n;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, N, 1, 1);
      Walk wk = make_walk(p, gqb, L);
      int n = 0;
      while (wk.next()) {
        const int st = n % kStages;
        const uint32_t ph = (n / kStages) & 1;
        if (!mbar_wait(&full[st], ph, p.status)) break;
        if (!mbar_wait(&mt_ready[st], ph, p.status)) break;
        tc_fence_after();
        const uint32_t va = sbase + p.off_v + st * p.v_bytes;
        const uint32_t mb = sbase + p.off_mt + st * p.mt_bytes;
        for (int g = 0; g < p.Hkv; ++g) {
          // A = V_g^T: MN-major, 128-byte swizzle, d halves 2 KB apart, 8-key groups 1 KB apart
          const uint64_t adesc = smem_desc(va + g * 4096, 2048, 1024, kSwizzle128);
          // B = M^T_g: MN-major, no swizzle, n-chunks 256 B apart, 8-key groups 128 B apart
          const uint64_t bdesc = smem_desc(mb + g * p.mt_group_stride, 128, 256, kSwizzleNone);
          mma_bf16_ss(tmem + g * N, adesc, bdesc, idesc, n > 0);
        }
        mma_commit(&done[st]);
        ++n;
      }
      mma_commit(final_bar);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ mix warps
    const int mw = warp - 4;  // rows 4mw .. 4mw+3 of the slice
    const int nks16 = p.Hs / 16;
    const bool has8 = (p.Hs & 15) != 0;
    const int ntile = p.Hr / 8;
    // W^T fragments (B operand): B[k = h][n = r], thread: n = lane/4, k = 2(lane%4)+{0,1}(+8)
    uint32_t wb[4][5][2];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int ks = 0; ks < 5; ++ks)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int r = nt * 8 + lane / 4;
          const int h = ks * 16 + hh * 8 + 2 * (lane % 4);
          float w0 = 0.f, w1 = 0.f;
          if (nt < ntile && h < p.Hs) {
            w0 = __bfloat162float(p.W[r * p.Hs + h]);
            w1 = __bfloat162float(p.W[r * p.Hs + h + 1]);
          }
          wb[nt][ks][hh] = pack_bf16(w0, w1);
        }
    Walk wk = make_walk(p, gqb, L);
    int n = 0;
    while (wk.next()) {
      const int st = n % kStages;
      const uint32_t ph = (n / kStages) & 1;
      if (!mbar_wait(&full[st], ph, p.status)) break;
      const uint32_t mp = sbase + p.off_map + st * p.map_bytes;
      uint8_t* mt = base + p.off_mt + st * p.mt_bytes;
      const int kvalid = min(kKeys, L - (wk.kb * p.B + wk.kg * kKeys));  // keys < L
#pragma unroll 1
      for (int ii = 0; ii < 4; ++ii) {
        const int i = mw * 4 + ii;  // row in the slice
        float acc[4][4];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
          for (int k = 0; k < 4; ++k) acc[nt][k] = 0.f;
        // ldmatrix rows: lanes 0-7 heads h0+l keys 0-7, 8-15 heads h0+l keys 8-15,
        // 16-23 heads h0+8+l keys 0-7, 24-31 heads h0+8+l keys 8-15
        const int lh = (lane & 7) + ((lane >> 4) << 3);
        const int lc = (lane >> 3) & 1;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          if (ks < nks16) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4_t(map_addr(mp, i * p.Hs + ks * 16 + lh, lc), a0, a1, a2, a3);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
              if (nt < ntile) mma16816(acc[nt], a0, a1, a2, a3, wb[nt][ks][0], wb[nt][ks][1]);
          }
        }
        if (has8) {
          uint32_t a0, a1;
          ldsm_x2_t(map_addr(mp, i * p.Hs + nks16 * 16 + (lane & 7), (lane >> 3) & 1), a0, a1);
#pragma unroll
          for (int nt = 0; nt < 4; ++nt)
            if (nt < ntile) {
              // the k8 step uses the first register of the last 16-head fragment slot
              uint32_t b = (nks16 == 0) ? wb[nt][0][0]
                         : (nks16 == 1) ? wb[nt][1][0]
                         : (nks16 == 2) ? wb[nt][2][0]
                         : (nks16 == 3) ? wb[nt][3][0] : wb[nt][4][0];
              mma1688(acc[nt], a0, a1, b);
            }
        }
        // D fragment: keys j = lane/4 (+8), heads r = 8nt + 2(lane%4) + {0,1}
        const int j0 = lane >> 2;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
          if (nt >= ntile) continue;
          const int r = nt * 8 + 2 * (lane & 3);
          const int g = r / p.G, rl = r % p.G;
          const int nn = i * p.G + rl;  // MMA N index of (row i, head r)
          uint8_t* gb = mt + g * p.mt_group_stride + (nn >> 3) * 256 + ((nn & 7) << 1);
          const float z0 = j0 < kvalid ? 1.f : 0.f, z1 = j0 + 8 < kvalid ? 1.f : 0.f;
          *reinterpret_cast<uint32_t*>(gb + (j0 >> 3) * 128 + (j0 & 7) * 16) =
              pack_bf16(acc[nt][0] * z0, acc[nt][1] * z0);
          *reinterpret_cast<uint32_t*>(gb + ((j0 + 8) >> 3) * 128 + ((j0 + 8) & 7) * 16) =
              pack_bf16(acc[nt][2] * z1, acc[nt][3] * z1);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&mt_ready[st]);
      ++n;
    }
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int c = quarter * 32 + lane;  // d index = TMEM lane
    bool ok = mbar_wait(final_bar, 0, p.status);
    tc_fence_after();
    const uint32_t lane_addr = tmem + (uint32_t(quarter * 32) << 16);
    for (int g = 0; g < p.Hkv; ++g) {
      for (int c0 = 0; c0 < N; c0 += 32) {
        float v[32];
        tmem_ld32(lane_addr + g * N + c0, v);
        tmem_wait_ld();
        if (!ok || n == 0) {
#pragma unroll
          for (int k = 0; k < 32; ++k) v[k] = 0.f;
        }
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const int nn = c0 + k;
          const int i = nn / p.G, rl = nn % p.G;
          const int row = i0 + i;
          if (row < L)
            p.O[(int64_t(seq0 + row) * p.Hr + g * p.G + rl) * kD + c] = __float2bfloat16_rn(v[k]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace av

// ------------------------------------------------------------------- host side

bool mapped_av_tc_supported(const mf_attn_desc& d, int Hr, const mf_v_desc& v) {
  if (d.dt != MF_BF16 || d.d != 128 || v.d != 128) return false;
  if (d.Hs % 8 != 0 || d.Hs > 64) return false;
  if (Hr > 32 || Hr % 8 != 0 || v.Hkv < 1 || Hr % v.Hkv != 0) return false;
  const int G = Hr / v.Hkv;
  return G == 2 || G == 4 || G == 8;
}

cudaError_t launch_mapped_av_tc(const mf_csr_cache& c, const mf_attn_desc& d, const Sizes& sz,
                                int Hr, const void* W, const mf_v_desc& v, void* O,
                                cudaStream_t st) {
  if (c.nnz_capacity < 1 || sz.nqb == 0) return cudaSuccess;
  av::Params p{};
  p.row_ptr = c.row_ptr;
  p.col_idx = c.col_idx;
  p.qb_seq = c.qb_seq;
  p.qb_idx = c.qb_idx;
  p.cu_seqlens = d.cu_seqlens;
  p.page_table = v.page_table;
  p.W = static_cast<const __nv_bfloat16*>(W);
  p.O = static_cast<__nv_bfloat16*>(O);
  p.capacity = c.nnz_capacity;
  p.nqb = sz.nqb;
  p.Hs = d.Hs;
  p.Hr = Hr;
  p.Hkv = v.Hkv;
  p.G = Hr / v.Hkv;
  p.B = d.B;
  p.page_size = v.page_table ? v.page_size : 16;
  p.max_pages = v.max_pages_per_seq;
  p.status = status_word();
  // shared memory: V stages (1024-aligned), map stages, mixed-map stages, barriers
  p.v_bytes = 4096u * uint32_t(v.Hkv);
  p.map_bytes = ((512u * uint32_t(d.Hs)) + 1023u) & ~1023u;
  p.mt_group_stride = 512u * uint32_t(p.G) + 16u;
  p.mt_bytes = (uint32_t(v.Hkv) * p.mt_group_stride + 127u) & ~127u;
  const uint32_t per_stage = p.v_bytes + p.map_bytes + p.mt_bytes;
  int nst = 3;
  if (size_t(nst) * per_stage + 2048 > 227u * 1024u) nst = 2;
  p.stages = nst;
  p.off_v = 0;
  p.off_map = nst * p.v_bytes;
  p.off_mt = p.off_map + nst * p.map_bytes;
  p.off_bar = (p.off_mt + nst * p.mt_bytes + 7u) & ~7u;
  const size_t smem = size_t(p.off_bar) + (3 * nst + 1) * 8 + 16 + 1024;
  if (smem > 227u * 1024u) return cudaErrorInvalidConfiguration;

  CUtensorMap tmap, tv;
  {
    // values [cap][Hs][B][B] viewed as (key j, head h, row i, entry e)
    const uint64_t B = uint64_t(d.B);
    const uint64_t dims[4] = {B, uint64_t(d.Hs), B, uint64_t(c.nnz_capacity)};
    const uint64_t strides[3] = {B * B * 2, B * 2, uint64_t(d.Hs) * B * B * 2};
    const uint32_t box[4] = {16, uint32_t(d.Hs), 16, 1};
    cudaError_t e = make_tmap_bf16(&tmap, c.values, 4, dims, strides, box, 32);
    if (e != cudaSuccess) return e;
  }
  {
    // V rows (tokens or pool rows) viewed as (d half, row, (group, half) chunk)
    const uint64_t rows = v.page_table ? uint64_t(v.npages) * v.page_size : uint64_t(sz.ntok);
    const uint64_t dims[3] = {64, rows, uint64_t(2 * v.Hkv)};
    const uint64_t strides[2] = {uint64_t(v.Hkv) * 128 * 2, 128};
    const uint32_t box[3] = {64, 16, uint32_t(2 * v.Hkv)};
    cudaError_t e = make_tmap_bf16(&tv, v.V, 3, dims, strides, box, 128);
    if (e != cudaSuccess) return e;
  }
  cudaError_t e = cudaFuncSetAttribute(av::k_mapped_av,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const unsigned grid = unsigned(sz.nqb) * unsigned(d.B / av::kRows);
  av::k_mapped_av<<<grid, av::kThreads, smem, st>>>(tmap, tv, p);
  return cudaGetLastError();
}

}  // namespace mf
