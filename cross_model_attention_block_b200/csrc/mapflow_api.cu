// Host side of libmapflow: argument checks, workspace layout, dispatch to the
// kernels, the device status word and the host prefix-hash index.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <unordered_map>
#include <vector>

#include "mf_internal.h"

namespace mf {

__device__ unsigned g_status_word;

namespace {
thread_local std::string t_last_error;
std::mutex g_status_mu;
unsigned* g_status_ptr[64] = {nullptr};

mf_status fail(mf_status st, const std::string& msg) {
  t_last_error = msg;
  return st;
}

mf_status cuda_fail(cudaError_t e, const char* where) {
  return fail(MF_ERR_CUDA, std::string(where) + ": " + cudaGetErrorString(e));
}
}  // namespace

void set_last_error(const char* msg) { t_last_error = msg; }

unsigned* status_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_status_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = static_cast<unsigned*>(p);
  }
  return g_status_ptr[dev];
}

// ------------------------------------------------------------ validation

static mf_status sizes_of(int32_t nseq, const int32_t* cu, int32_t B, Sizes* out) {
  if (nseq < 1 || cu == nullptr) return fail(MF_ERR_INVALID_ARG, "nseq < 1 or cu_seqlens_host is NULL");
  if (B != 64 && B != 128) return fail(MF_ERR_UNSUPPORTED, "block size B must be 64 or 128");
  if (cu[0] != 0) return fail(MF_ERR_INVALID_ARG, "cu_seqlens_host[0] must be 0");
  Sizes s;
  for (int i = 0; i < nseq; ++i) {
    int64_t L = int64_t(cu[i + 1]) - cu[i];
    if (L < 0) return fail(MF_ERR_INVALID_ARG, "cu_seqlens_host must be non-decreasing");
    if (L > int64_t(512) * B)
      return fail(MF_ERR_UNSUPPORTED, "sequence longer than 512 blocks");
    int64_t n = (L + B - 1) / B;
    s.nqb += n;
    s.nblocks += n * (n + 1) / 2;
    s.ntiles += (L + 127) / 128;
    if (L > s.max_len) s.max_len = int32_t(L);
  }
  s.ntok = cu[nseq];
  *out = s;
  return MF_OK;
}

static mf_status check_desc(const mf_attn_desc* d, Sizes* sz) {
  if (!d) return fail(MF_ERR_INVALID_ARG, "desc is NULL");
  if (!d->cu_seqlens) return fail(MF_ERR_INVALID_ARG, "cu_seqlens (device) is NULL");
  mf_status st = sizes_of(d->nseq, d->cu_seqlens_host, d->B, sz);
  if (st != MF_OK) return st;
  if (d->Hs < 1 || d->Hs > 64) return fail(MF_ERR_UNSUPPORTED, "Hs must be in [1, 64]");
  if (d->d != 64 && d->d != 128) return fail(MF_ERR_UNSUPPORTED, "head dim d must be 64 or 128");
  if (d->dt != MF_BF16 && d->dt != MF_F32) return fail(MF_ERR_INVALID_ARG, "unknown dtype");
  if (d->band_width < 0) return fail(MF_ERR_INVALID_ARG, "band_width < 0");
  if (!std::isfinite(d->band_bias)) return fail(MF_ERR_INVALID_ARG, "band_bias not finite");
  return MF_OK;
}

static size_t meta_bytes(Carve& c, int nseq, int64_t ntiles, Meta* m) {
  Meta mm;
  mm.cu_qb = c.take<int32_t>(nseq + 1);
  mm.cu_blk = c.take<int64_t>(nseq + 1);
  mm.cu_tile = c.take<int32_t>(nseq + 1);
  mm.tiles = c.take<int32_t>(2 * size_t(ntiles) + 2);
  if (m) *m = mm;
  return c.used;
}

// Tiles and block span of the global query blocks [lo, hi) (host arithmetic
// on cu_seqlens_host; the same tile rule as k_meta).
static QbRange range_of(const mf_attn_desc& d, const Sizes& sz, int64_t lo, int64_t hi) {
  QbRange r;
  r.qb_lo = lo;
  r.qb_hi = hi;
  r.blk_lo = r.blk_hi = sz.nblocks;
  const int per = 128 / d.B;
  int64_t q0 = 0, b0 = 0;
  bool first = true;
  for (int s = 0; s < d.nseq; ++s) {
    const int64_t L = int64_t(d.cu_seqlens_host[s + 1]) - d.cu_seqlens_host[s];
    const int64_t n = (L + d.B - 1) / d.B;
    const int64_t a = std::max(lo - q0, int64_t(0)), e = std::min(hi - q0, n);
    if (a < e) {
      r.ntiles += (e - 1) / per - a / per + 1;
      if (first) {
        r.blk_lo = b0 + a * (a + 1) / 2;
        first = false;
      }
      r.blk_hi = b0 + e * (e + 1) / 2;
    }
    q0 += n;
    b0 += n * (n + 1) / 2;
  }
  if (first) r.blk_lo = r.blk_hi = 0;
  return r;
}

static mf_status check_range(const Sizes& sz, int64_t lo, int64_t hi) {
  if (lo < 0 || lo > hi || hi > sz.nqb)
    return fail(MF_ERR_INVALID_ARG, "query-block range outside [0, nqb_total]");
  return MF_OK;
}

// bf16 with d = 128 runs on the tcgen05 kernels; float32 (1e-4 relative
// accuracy) and d = 64 run on the scalar kernels.
static bool use_tc(const mf_attn_desc& d) { return d.dt == MF_BF16 && d.d == 128; }

static bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255) == 0; }

// ------------------------------------------------------------- stats

static size_t stats_ws(const mf_attn_desc& d, const Sizes& sz, void* base, Meta* m,
                       float** part) {
  Carve c(base);
  meta_bytes(c, d.nseq, sz.ntiles, m);
  float* p = c.take<float>(size_t(d.Hs) * size_t(sz.nblocks));
  if (part) *part = p;
  return c.used + 256;
}

static size_t select_ws(const mf_attn_desc& d, const Sizes& sz, void* base, Meta* m,
                        int32_t** counts, uint8_t** keep, int32_t** slot) {
  Carve c(base);
  meta_bytes(c, d.nseq, sz.ntiles, m);
  int32_t* a = c.take<int32_t>(size_t(sz.nqb) + 1);
  uint8_t* b = c.take<uint8_t>(size_t(sz.nblocks) + 1);
  int32_t* s = c.take<int32_t>(size_t(sz.nblocks) + 1);
  if (counts) *counts = a;
  if (keep) *keep = b;
  if (slot) *slot = s;
  return c.used + 256;
}

}  // namespace mf

using namespace mf;

extern "C" {

const char* mf_version(void) { return "mapflow-b200 0.1 (sm_100a)"; }

const char* mf_last_error(void) { return t_last_error.c_str(); }

mf_status mf_layout_sizes(int32_t nseq, const int32_t* cu_seqlens_host, int32_t B,
                          int64_t* nqb_total, int64_t* nblocks_total) {
  Sizes sz;
  mf_status st = sizes_of(nseq, cu_seqlens_host, B, &sz);
  if (st != MF_OK) return st;
  if (nqb_total) *nqb_total = sz.nqb;
  if (nblocks_total) *nblocks_total = sz.nblocks;
  return MF_OK;
}

size_t mf_block_stats_workspace(const mf_attn_desc* desc) {
  Sizes sz;
  if (check_desc(desc, &sz) != MF_OK) return 0;
  return stats_ws(*desc, sz, nullptr, nullptr, nullptr);
}

mf_status mf_block_stats(const mf_attn_desc* desc, const void* Q, const void* K, float* lse,
                         float* mass, void* ws, size_t ws_bytes, mf_stream_t stream) {
  Sizes sz;
  mf_status st = check_desc(desc, &sz);
  if (st != MF_OK) return st;
  return mf_block_stats_range(desc, Q, K, lse, mass, 0, sz.nqb, ws, ws_bytes, stream);
}

// A NULL pointer is accepted for a buffer that is empty at the sizes given.
static bool present(const void* p, int64_t elements) { return p != nullptr || elements == 0; }

mf_status mf_block_stats_range(const mf_attn_desc* desc, const void* Q, const void* K,
                               float* lse, float* mass, int64_t qb_begin, int64_t qb_end,
                               void* ws, size_t ws_bytes, mf_stream_t stream) {
  Sizes sz;
  mf_status st = check_desc(desc, &sz);
  if (st != MF_OK) return st;
  if (!present(Q, sz.ntok) || !present(K, sz.ntok) || !present(lse, sz.ntok) ||
      !present(mass, sz.nblocks))
    return fail(MF_ERR_INVALID_ARG, "Q, K, lse or mass is NULL");
  st = check_range(sz, qb_begin, qb_end);
  if (st != MF_OK) return st;
  const mf_attn_desc& d = *desc;
  if (!ws || !aligned256(ws) || ws_bytes < stats_ws(d, sz, nullptr, nullptr, nullptr))
    return fail(MF_ERR_WORKSPACE, "workspace missing, not 256-byte aligned or too small");
  if (!status_word()) return fail(MF_ERR_CUDA, "no CUDA device");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Meta m;
  float* part = nullptr;
  stats_ws(d, sz, ws, &m, &part);
  const QbRange r = range_of(d, sz, qb_begin, qb_end);
  cudaError_t e = launch_meta(d.nseq, d.cu_seqlens, d.B, r.qb_lo, r.qb_hi, m, s);
  if (e != cudaSuccess) return cuda_fail(e, "meta");
  if (r.qb_hi == r.qb_lo) return MF_OK;
  // the one-pass statistics keep one TMEM column per key block: 256 at most
  // (mf_path_info reports the same choice)
  const bool tc_stats = use_tc(d) && (sz.max_len + d.B - 1) / d.B <= 256;
  e = tc_stats ? launch_stats_tc(d, sz, r, m, Q, K, lse, part, s)
                : launch_stats_simt(d, sz, r, m, Q, K, lse, part, s);
  if (e != cudaSuccess) return cuda_fail(e, "block stats");
  e = launch_mass_reduce(part, d.Hs, sz.nblocks, r.blk_lo, r.blk_hi, mass, s);
  if (e != cudaSuccess) return cuda_fail(e, "mass reduce");
  return MF_OK;
}

size_t mf_select_extract_workspace(const mf_attn_desc* desc) {
  Sizes sz;
  if (check_desc(desc, &sz) != MF_OK) return 0;
  return select_ws(*desc, sz, nullptr, nullptr, nullptr, nullptr, nullptr);
}

static mf_status check_cache(const mf_csr_cache* c, const mf_attn_desc& d, const Sizes& sz) {
  if (!c) return fail(MF_ERR_INVALID_ARG, "cache is NULL");
  if (!c->row_ptr || !present(c->col_idx, c->nnz_capacity) || !present(c->qb_seq, sz.nqb) ||
      !present(c->qb_idx, sz.nqb) || !present(c->values, c->nnz_capacity))
    return fail(MF_ERR_INVALID_ARG, "cache has a NULL array");
  if (c->Hs != d.Hs || c->B != d.B || c->dt != d.dt)
    return fail(MF_ERR_INVALID_ARG, "cache Hs/B/dtype differ from the descriptor");
  if (c->nqb_total != sz.nqb)
    return fail(MF_ERR_INVALID_ARG, "cache nqb_total differs from the context layout");
  if (c->nnz_capacity < 0) return fail(MF_ERR_INVALID_ARG, "negative nnz_capacity");
  return MF_OK;
}

mf_status mf_select_extract(const mf_attn_desc* desc, const void* Q, const void* K,
                            const float* lse, const float* mass, double tau,
                            mf_csr_cache* out, void* ws, size_t ws_bytes, mf_stream_t stream) {
  Sizes sz;
  mf_status st = check_desc(desc, &sz);
  if (st != MF_OK) return st;
  return mf_select_extract_range(desc, Q, K, lse, mass, tau, out, 0, sz.nqb, ws, ws_bytes,
                                 stream);
}

mf_status mf_select_extract_range(const mf_attn_desc* desc, const void* Q, const void* K,
                                  const float* lse, const float* mass, double tau,
                                  mf_csr_cache* out, int64_t qb_begin, int64_t qb_end, void* ws,
                                  size_t ws_bytes, mf_stream_t stream) {
  Sizes sz;
  mf_status st = check_desc(desc, &sz);
  if (st != MF_OK) return st;
  const mf_attn_desc& d = *desc;
  if (!present(Q, sz.ntok) || !present(K, sz.ntok) || !present(lse, sz.ntok) ||
      !present(mass, sz.nblocks))
    return fail(MF_ERR_INVALID_ARG, "Q, K, lse or mass is NULL");
  if (!(tau > 0.0) || !std::isfinite(tau)) return fail(MF_ERR_INVALID_ARG, "tau must be > 0");
  st = check_cache(out, d, sz);
  if (st != MF_OK) return st;
  st = check_range(sz, qb_begin, qb_end);
  if (st != MF_OK) return st;
  if (!ws || !aligned256(ws) ||
      ws_bytes < select_ws(d, sz, nullptr, nullptr, nullptr, nullptr, nullptr))
    return fail(MF_ERR_WORKSPACE, "workspace missing, not 256-byte aligned or too small");
  if (!status_word()) return fail(MF_ERR_CUDA, "no CUDA device");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Meta m;
  int32_t* counts = nullptr;
  uint8_t* keep = nullptr;
  int32_t* slot = nullptr;
  select_ws(d, sz, ws, &m, &counts, &keep, &slot);
  const QbRange r = range_of(d, sz, qb_begin, qb_end);
  cudaError_t e = launch_meta(d.nseq, d.cu_seqlens, d.B, r.qb_lo, r.qb_hi, m, s);
  if (e != cudaSuccess) return cuda_fail(e, "meta");
  if (sz.nqb == 0) {
    e = cudaMemsetAsync(out->row_ptr, 0, sizeof(int64_t), s);
    return e == cudaSuccess ? MF_OK : cuda_fail(e, "row_ptr");
  }
  e = launch_select(d, sz, r, m, mass, tau, *out, counts, keep, slot, s);
  if (e != cudaSuccess) return cuda_fail(e, "select");
  e = use_tc(d) ? launch_extract_tc(d, sz, r, m, Q, K, lse, slot, out->values,
                                    out->nnz_capacity, s)
                : launch_extract_simt(d, sz, r, Q, K, lse, *out, s);
  if (e != cudaSuccess) return cuda_fail(e, "extract");
  return MF_OK;
}

// ------------------------------------------------------- rounds, extraction

// Checks a round layout against the context: starts ascending from 0 to ntok,
// every non-empty sequence starts a round, every round starts on a block
// boundary of its sequence and ends inside it.  *max_r: most rounds of one
// sequence.
static mf_status check_rounds(const mf_attn_desc& d, int32_t nrounds, const int32_t* st,
                              int* max_r) {
  if (nrounds < 1 || !st) return fail(MF_ERR_INVALID_ARG, "no rounds, or round_starts_host is NULL");
  const int32_t* cu = d.cu_seqlens_host;
  if (st[0] != 0 || st[nrounds] != cu[d.nseq])
    return fail(MF_ERR_INVALID_ARG, "round starts must run from 0 to the token count");
  int s = 0, in_seq = 0;
  *max_r = 0;
  for (int r = 0; r < nrounds; ++r) {
    if (st[r + 1] <= st[r]) return fail(MF_ERR_INVALID_ARG, "round starts must increase");
    while (s < d.nseq && cu[s + 1] <= st[r]) {
      ++s;
      in_seq = 0;
    }
    if (in_seq == 0 && st[r] != cu[s])
      return fail(MF_ERR_INVALID_ARG, "a sequence does not start a round");
    if ((st[r] - cu[s]) % d.B != 0)
      return fail(MF_ERR_INVALID_ARG, "a round does not start on a block boundary");
    if (st[r + 1] > cu[s + 1]) return fail(MF_ERR_INVALID_ARG, "a round crosses a sequence end");
    *max_r = std::max(*max_r, ++in_seq);
  }
  return MF_OK;
}

static size_t rounds_ws(const mf_attn_desc& d, const Sizes& sz, int nrounds, int max_r,
                        void* base, Meta* m, int32_t** r_seq, int32_t** r_first,
                        uint8_t** flags, int32_t** counts) {
  Carve c(base);
  meta_bytes(c, d.nseq, sz.ntiles, m);
  int32_t* a = c.take<int32_t>(size_t(nrounds));
  int32_t* b = c.take<int32_t>(size_t(d.nseq) + 1);
  uint8_t* f = c.take<uint8_t>(size_t(nrounds) * size_t(max_r));
  int32_t* n = c.take<int32_t>(size_t(sz.nqb) + 1);
  if (r_seq) *r_seq = a;
  if (r_first) *r_first = b;
  if (flags) *flags = f;
  if (counts) *counts = n;
  return c.used + 256;
}

static size_t extract_ws(const mf_attn_desc& d, const Sizes& sz, void* base, Meta* m,
                         int32_t** slot) {
  Carve c(base);
  meta_bytes(c, d.nseq, sz.ntiles, m);
  int32_t* s = c.take<int32_t>(size_t(sz.nblocks) + 1);
  if (slot) *slot = s;
  return c.used + 256;
}

static mf_status check_av(const mf_csr_cache* cache, const mf_attn_desc* desc, int32_t Hr,
                          const mf_v_desc* v, Sizes* sz) {
  mf_status st = check_desc(desc, sz);
  if (st != MF_OK) return st;
  const mf_attn_desc& d = *desc;
  st = check_cache(cache, d, *sz);
  if (st != MF_OK) return st;
  if (!v || !present(v->V, sz->ntok)) return fail(MF_ERR_INVALID_ARG, "V is NULL");
  if (v->d != d.d) return fail(MF_ERR_INVALID_ARG, "V head dim differs from the descriptor");
  if (v->Hkv < 1 || Hr < 1 || Hr % v->Hkv != 0)
    return fail(MF_ERR_INVALID_ARG, "Hr must be a positive multiple of Hkv");
  if (int64_t(Hr) * d.d > 4096) return fail(MF_ERR_UNSUPPORTED, "Hr * d above 4096");
  if (v->page_table) {
    if (v->page_size < 16 || v->page_size % 16 != 0)
      return fail(MF_ERR_INVALID_ARG, "page_size must be a positive multiple of 16");
    if (int64_t(v->max_pages_per_seq) * v->page_size < sz->max_len)
      return fail(MF_ERR_INVALID_ARG, "max_pages_per_seq * page_size below a sequence length");
    if (v->npages < 1) return fail(MF_ERR_INVALID_ARG, "npages < 1");
  }
  return MF_OK;
}

// 16-key groups of a context: sum_s ceil(L_s / 16).
static int64_t key_groups(const mf_attn_desc& d) {
  int64_t g = 0;
  for (int s = 0; s < d.nseq; ++s) g += (int64_t(d.cu_seqlens_host[s + 1]) - d.cu_seqlens_host[s] + 15) / 16;
  return g;
}

size_t mf_mapped_av_workspace(const mf_csr_cache* cache, const mf_attn_desc* desc, int32_t Hr,
                              const mf_v_desc* v) {
  Sizes sz;
  if (check_av(cache, desc, Hr, v, &sz) != MF_OK) return 0;
  if (!mapped_av_tc_supported(*desc, Hr, *v)) return 256;
  return mapped_av_tc_workspace(desc->nseq, key_groups(*desc), v->Hkv);
}

mf_status mf_mapped_av(const mf_csr_cache* cache, const mf_attn_desc* desc, int32_t Hr,
                       const void* W, const mf_v_desc* v, void* O, void* ws, size_t ws_bytes,
                       mf_stream_t stream) {
  if (!cache) return fail(MF_ERR_INVALID_ARG, "cache is NULL");
  return mf_mapped_av_range(cache, desc, Hr, W, v, O, 0, cache->nqb_total, ws, ws_bytes,
                            stream);
}

mf_status mf_mapped_av_range(const mf_csr_cache* cache, const mf_attn_desc* desc, int32_t Hr,
                             const void* W, const mf_v_desc* v, void* O, int64_t qb_begin,
                             int64_t qb_end, void* ws, size_t ws_bytes, mf_stream_t stream) {
  Sizes sz;
  mf_status st = check_av(cache, desc, Hr, v, &sz);
  if (st != MF_OK) return st;
  const mf_attn_desc& d = *desc;
  if (!W || !present(O, sz.ntok)) return fail(MF_ERR_INVALID_ARG, "W or O is NULL");
  st = check_range(sz, qb_begin, qb_end);
  if (st != MF_OK) return st;
  const bool tc = mapped_av_tc_supported(d, Hr, *v);
  if (tc && (!ws || !aligned256(ws) ||
             ws_bytes < mapped_av_tc_workspace(d.nseq, key_groups(d), v->Hkv)))
    return fail(MF_ERR_WORKSPACE, "workspace missing, not 256-byte aligned or too small");
  if (!status_word()) return fail(MF_ERR_CUDA, "no CUDA device");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (sz.nqb == 0) return MF_OK;
  cudaError_t e = tc ? launch_mapped_av_tc(*cache, d, sz, Hr, W, *v, O, ws, key_groups(d),
                                           qb_begin, qb_end, s)
                     : launch_mapped_av_simt(*cache, d, sz, Hr, W, *v, O, qb_begin, qb_end, s);
  if (e != cudaSuccess) return cuda_fail(e, "mapped av");
  return MF_OK;
}

size_t mf_select_rounds_workspace(const mf_attn_desc* desc, int32_t nrounds,
                                  const int32_t* round_starts_host) {
  Sizes sz;
  if (check_desc(desc, &sz) != MF_OK) return 0;
  int max_r = 0;
  if (check_rounds(*desc, nrounds, round_starts_host, &max_r) != MF_OK) return 0;
  return rounds_ws(*desc, sz, nrounds, max_r, nullptr, nullptr, nullptr, nullptr, nullptr,
                   nullptr);
}

mf_status mf_select_rounds(const mf_attn_desc* desc, const float* mass, int32_t nrounds,
                           const int32_t* round_starts, const int32_t* round_starts_host,
                           double tau, mf_csr_cache* out, void* ws, size_t ws_bytes,
                           mf_stream_t stream) {
  Sizes sz;
  mf_status st = check_desc(desc, &sz);
  if (st != MF_OK) return st;
  const mf_attn_desc& d = *desc;
  if (!mass || !round_starts) return fail(MF_ERR_INVALID_ARG, "mass or round_starts is NULL");
  if (!(tau > 0.0) || !std::isfinite(tau)) return fail(MF_ERR_INVALID_ARG, "tau must be > 0");
  int max_r = 0;
  st = check_rounds(d, nrounds, round_starts_host, &max_r);
  if (st != MF_OK) return st;
  st = check_cache(out, d, sz);
  if (st != MF_OK) return st;
  const size_t need = rounds_ws(d, sz, nrounds, max_r, nullptr, nullptr, nullptr, nullptr,
                                nullptr, nullptr);
  if (!ws || !aligned256(ws) || ws_bytes < need)
    return fail(MF_ERR_WORKSPACE, "workspace missing, not 256-byte aligned or too small");
  if (!status_word()) return fail(MF_ERR_CUDA, "no CUDA device");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Meta m;
  int32_t *r_seq = nullptr, *r_first = nullptr, *counts = nullptr;
  uint8_t* flags = nullptr;
  rounds_ws(d, sz, nrounds, max_r, ws, &m, &r_seq, &r_first, &flags, &counts);
  cudaError_t e = launch_meta(d.nseq, d.cu_seqlens, d.B, 0, sz.nqb, m, s);
  if (e != cudaSuccess) return cuda_fail(e, "meta");
  if (sz.nqb == 0) {
    e = cudaMemsetAsync(out->row_ptr, 0, sizeof(int64_t), s);
    return e == cudaSuccess ? MF_OK : cuda_fail(e, "row_ptr");
  }
  e = launch_select_rounds(d, sz, m, mass, nrounds, round_starts, max_r, tau, *out, r_seq,
                           r_first, flags, counts, s);
  if (e != cudaSuccess) return cuda_fail(e, "select rounds");
  return MF_OK;
}

size_t mf_extract_workspace(const mf_attn_desc* desc) {
  Sizes sz;
  if (check_desc(desc, &sz) != MF_OK) return 0;
  return extract_ws(*desc, sz, nullptr, nullptr, nullptr);
}

mf_status mf_extract(const mf_attn_desc* desc, const void* Q, const void* K, const float* lse,
                     const mf_csr_cache* cache, void* ws, size_t ws_bytes, mf_stream_t stream) {
  Sizes sz;
  mf_status st = check_desc(desc, &sz);
  if (st != MF_OK) return st;
  const mf_attn_desc& d = *desc;
  if (!present(Q, sz.ntok) || !present(K, sz.ntok) || !present(lse, sz.ntok))
    return fail(MF_ERR_INVALID_ARG, "Q, K or lse is NULL");
  st = check_cache(cache, d, sz);
  if (st != MF_OK) return st;
  if (!ws || !aligned256(ws) || ws_bytes < extract_ws(d, sz, nullptr, nullptr, nullptr))
    return fail(MF_ERR_WORKSPACE, "workspace missing, not 256-byte aligned or too small");
  if (!status_word()) return fail(MF_ERR_CUDA, "no CUDA device");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Meta m;
  int32_t* slot = nullptr;
  extract_ws(d, sz, ws, &m, &slot);
  const QbRange r = range_of(d, sz, 0, sz.nqb);
  cudaError_t e = launch_meta(d.nseq, d.cu_seqlens, d.B, r.qb_lo, r.qb_hi, m, s);
  if (e != cudaSuccess) return cuda_fail(e, "meta");
  if (sz.nqb == 0) return MF_OK;
  if (use_tc(d)) {
    e = launch_csr_slots(sz, m, *cache, slot, s);
    if (e != cudaSuccess) return cuda_fail(e, "csr slots");
    e = launch_extract_tc(d, sz, r, m, Q, K, lse, slot, cache->values, cache->nnz_capacity, s);
  } else {
    e = launch_extract_simt(d, sz, r, Q, K, lse, *cache, s);
  }
  if (e != cudaSuccess) return cuda_fail(e, "extract");
  return MF_OK;
}

mf_status mf_path_info(const mf_attn_desc* desc, int32_t Hr, const mf_v_desc* v,
                       uint32_t* flags) {
  if (!flags) return fail(MF_ERR_INVALID_ARG, "flags is NULL");
  Sizes sz;
  mf_status st = check_desc(desc, &sz);
  if (st != MF_OK) return st;
  const mf_attn_desc& d = *desc;
  uint32_t f = 0;
  if (use_tc(d) && (sz.max_len + d.B - 1) / d.B <= 256) f |= MF_PATH_STATS_TC;
  if (use_tc(d)) f |= MF_PATH_EXTRACT_TC;
  if (v) {
    if (v->Hkv < 1 || Hr < 1 || Hr % v->Hkv != 0)
      return fail(MF_ERR_INVALID_ARG, "Hr must be a positive multiple of Hkv");
    if (mapped_av_tc_supported(d, Hr, *v)) f |= MF_PATH_AV_TC;
  }
  *flags = f;
  return MF_OK;
}

mf_status mf_mapped_av_plan(int32_t Hs, int32_t Hr, int32_t Hkv, int32_t* out) {
  if (!out) return fail(MF_ERR_INVALID_ARG, "out is NULL");
  if (Hs < 8 || Hs > 64 || Hs % 8 != 0 || (Hr != 16 && Hr != 32) || Hkv < 1 || Hr % Hkv != 0 ||
      (Hr / Hkv != 2 && Hr / Hkv != 4 && Hr / Hkv != 8))
    return fail(MF_ERR_UNSUPPORTED, "shape outside the tensor-core fused kernel");
  if (!mapped_av_tc_plan(Hs, Hr, Hkv, out)) return fail(MF_ERR_UNSUPPORTED, "no plan fits");
  return MF_OK;
}

mf_status mf_exp2_fma_eval(const float* x, float* y, int64_t n, mf_stream_t stream) {
  if (n < 0 || (n > 0 && (!x || !y))) return fail(MF_ERR_INVALID_ARG, "n < 0 or NULL array");
  const cudaError_t e = launch_exp2_fma_eval(x, y, n, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MF_OK : cuda_fail(e, "exp2_fma_eval launch");
}

mf_status mf_selftest_timeout(int32_t limit_ms, mf_stream_t stream) {
  if (limit_ms < 1 || limit_ms > 2000) return fail(MF_ERR_INVALID_ARG, "limit_ms must be in [1, 2000]");
  const cudaError_t e =
      launch_selftest_timeout(uint64_t(limit_ms) * 1000000ull, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MF_OK : cuda_fail(e, "selftest_timeout launch");
}

mf_status mf_sync_status(mf_stream_t stream) {
  unsigned* p = status_word();
  if (!p) return fail(MF_ERR_CUDA, "no CUDA device");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  unsigned v = 0;
  e = cudaMemcpy(&v, p, sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  if (v != 0) {
    unsigned zero = 0;
    e = cudaMemcpy(p, &zero, sizeof(zero), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "status clear");
  }
  if (v & kStatusTimeout) return fail(MF_ERR_TIMEOUT, "a device-side bounded wait gave up");
  if (v & kStatusCapacity) return fail(MF_ERR_CAPACITY, "kept blocks exceed nnz_capacity");
  if (v & kStatusBadCache)
    return fail(MF_ERR_INVALID_ARG, "a cache row holds more entries than its query block has key blocks");
  return MF_OK;
}

}  // extern "C"
