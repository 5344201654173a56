// Internal host-side interface between the translation units of libmapflow.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

#include "../../include/mapflow.h"

namespace mf {

// Bits of the per-device status word.
enum : unsigned { kStatusTimeout = 1u, kStatusCapacity = 2u, kStatusBadCache = 4u };

// Device address of the status word of the current device.
unsigned* status_word();

// Sets the text mf_last_error() returns to this thread.
void set_last_error(const char* msg);

// Per-context block layout, device arrays computed from cu_seqlens.
struct Meta {
  int32_t* cu_qb;    // [nseq+1] prefix of ceil(L_s/B)
  int64_t* cu_blk;   // [nseq+1] prefix of C_s
  int32_t* cu_tile;  // [nseq+1] prefix of ceil(L_s/128)
  int32_t* tiles;    // [ntiles][2] (sequence, 128-row tile), longest causal rows first
};

// Host-side sizes of a context.
struct Sizes {
  int64_t ntok = 0;
  int64_t nqb = 0;
  int64_t nblocks = 0;
  int64_t ntiles = 0;  // 128-row tiles
  int32_t max_len = 0;
};

// A range of global query blocks [qb_lo, qb_hi) of a context: the 128-row
// tiles that hold at least one of its query blocks, and the range of block
// indices [blk_lo, blk_hi) of its blocks (contiguous in the mass layout).
struct QbRange {
  int64_t qb_lo = 0, qb_hi = 0;
  int64_t blk_lo = 0, blk_hi = 0;
  int64_t ntiles = 0;
};

// Bump allocator over a caller workspace (256-byte aligned pieces).
struct Carve {
  char* base;
  size_t used = 0;
  explicit Carve(void* p) : base(static_cast<char*>(p)) {}
  template <typename T>
  T* take(size_t count) {
    used = (used + 255) & ~size_t(255);
    T* p = base ? reinterpret_cast<T*>(base + used) : nullptr;
    used += count * sizeof(T);
    return p;
  }
};

// ---- launchers (return cudaGetLastError of the launch) ----
// The tile list holds the tiles of the query blocks [qb_lo, qb_hi) only.
cudaError_t launch_meta(int nseq, const int32_t* cu_seqlens, int B, int64_t qb_lo,
                        int64_t qb_hi, const Meta& m, cudaStream_t st);

// Tensor-core kernels (bf16, d = 128), over the query blocks of a range: they
// write lse rows, partial masses and cache entries of those blocks only.
cudaError_t launch_stats_tc(const mf_attn_desc& d, const Sizes& sz, const QbRange& r,
                            const Meta& m, const void* Q, const void* K, float* lse,
                            float* part, cudaStream_t st);
cudaError_t launch_extract_tc(const mf_attn_desc& d, const Sizes& sz, const QbRange& r,
                              const Meta& m, const void* Q, const void* K, const float* lse,
                              const int32_t* slot, void* values, int64_t capacity,
                              cudaStream_t st);

// Tensor map of a bf16 tensor (rank <= 5; strides of dims 1.. in bytes;
// swizzle_bytes 0, 32, 64 or 128).
cudaError_t make_tmap_bf16(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
                           const uint64_t* strides_bytes, const uint32_t* box, int swizzle_bytes);

bool mapped_av_tc_supported(const mf_attn_desc& d, int Hr, const mf_v_desc& v);
// Workspace of the tensor-core fused kernel: per-sequence 16-key-group prefix
// sums and V regrouped per 16 keys into operand images (4096 * Hkv bytes each).
size_t mapped_av_tc_workspace(int nseq, int64_t key_groups, int Hkv);
// Both fused-kernel launchers cover the global query blocks [qb_lo, qb_hi).
cudaError_t launch_mapped_av_tc(const mf_csr_cache& c, const mf_attn_desc& d, const Sizes& sz,
                                int Hr, const void* W, const mf_v_desc& v, void* O, void* ws,
                                int64_t key_groups, int64_t qb_lo, int64_t qb_hi,
                                cudaStream_t st);

// Shared-memory plan of the tensor-core fused kernel for a shape: {KG, map
// stages, V stages, dynamic smem bytes, offsets of map, M^T, W^T, barriers}.
bool mapped_av_tc_plan(int Hs, int Hr, int Hkv, int32_t out[8]);
cudaError_t launch_exp2_fma_eval(const float* x, float* y, int64_t n, cudaStream_t st);
cudaError_t launch_selftest_timeout(uint64_t limit_ns, cudaStream_t st);
cudaError_t launch_stats_simt(const mf_attn_desc& d, const Sizes& sz, const QbRange& r,
                              const Meta& m, const void* Q, const void* K, float* lse,
                              float* part, cudaStream_t st);
// mass[b] = sum_h part[h][b] for the blocks b in [blk_lo, blk_hi).
cudaError_t launch_mass_reduce(const float* part, int Hs, int64_t nblocks, int64_t blk_lo,
                               int64_t blk_hi, float* mass, cudaStream_t st);

// Selection of the query blocks of a range; the CSR rows of every other query
// block are left empty.
cudaError_t launch_select(const mf_attn_desc& d, const Sizes& sz, const QbRange& r,
                          const Meta& m, const float* mass, double tau, const mf_csr_cache& c,
                          int32_t* counts, uint8_t* keep, int32_t* slot, cudaStream_t st);

// Global query block -> (sequence, index) map; exclusive int64 scan of counts.
void launch_qb_map(int64_t nqb, int nseq, const int32_t* cu_qb, int32_t* qb_seq,
                   int32_t* qb_idx, int grid, cudaStream_t st);
void launch_scan(const int32_t* counts, int64_t n, int64_t* row_ptr, cudaStream_t st);

// Round-level selection: CSR rows of every query block from the kept rounds
// of its query round (r_seq [nrounds], r_first [nseq+1], flags
// [nrounds][max_r], counts [nqb] are workspace).
cudaError_t launch_select_rounds(const mf_attn_desc& d, const Sizes& sz, const Meta& m,
                                 const float* mass, int nrounds, const int32_t* starts,
                                 int max_r, double tau, const mf_csr_cache& c,
                                 int32_t* r_seq, int32_t* r_first, uint8_t* flags,
                                 int32_t* counts, cudaStream_t st);
// Block -> entry map of a filled CSR (slot [nblocks], -1 where not kept).
cudaError_t launch_csr_slots(const Sizes& sz, const Meta& m, const mf_csr_cache& c,
                             int32_t* slot, cudaStream_t st);

cudaError_t launch_extract_simt(const mf_attn_desc& d, const Sizes& sz, const QbRange& r,
                                const void* Q, const void* K, const float* lse,
                                const mf_csr_cache& c, cudaStream_t st);

cudaError_t launch_mapped_av_simt(const mf_csr_cache& c, const mf_attn_desc& d,
                                  const Sizes& sz, int Hr, const void* W,
                                  const mf_v_desc& v, void* O, int64_t qb_lo, int64_t qb_hi,
                                  cudaStream_t st);

}  // namespace mf
