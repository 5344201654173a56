// Host-memory tier of the block cache: offload a device cache to host memory,
// fetch the rows of a range of query blocks back into a device cache.
//
// MapFlow article (163.com, section on the three system components, second
// component): cached sender states are indexed by a prefix hash, and the
// receiver's retrieval of the cached blocks overlaps its recomputation of its
// first layers.  A cache that outlives the sender's request and serves
// several receivers lives here in (pinned) host memory; a receiver fetches a
// mapped layer's rows range by range on a copy stream while its compute
// stream recomputes the early layers, and runs the fused kernel on each range
// once it has landed.  Only cudaMemcpyAsync is used (one call per array).
#include <cuda_runtime.h>

#include <string>

#include "mf_internal.h"

namespace {

mf_status fail(mf_status st, const char* msg) {
  mf::set_last_error(msg);
  return st;
}

size_t elem_bytes(mf_dtype dt) { return dt == MF_F32 ? 4 : 2; }

mf_status same_layout(const mf_csr_cache* a, const mf_csr_cache* b) {
  if (!a || !b) return fail(MF_ERR_INVALID_ARG, "cache is NULL");
  // an array may be NULL only where it is empty (no entries, no query blocks)
  for (const mf_csr_cache* c : {a, b}) {
    const bool rows = c->nqb_total == 0, entries = c->nnz_capacity == 0;
    if (!c->row_ptr || (!c->qb_seq && !rows) || (!c->qb_idx && !rows) ||
        (!c->col_idx && !entries) || (!c->values && !entries))
      return fail(MF_ERR_INVALID_ARG, "cache has a NULL array");
  }
  if (a->nqb_total != b->nqb_total || a->Hs != b->Hs || a->B != b->B || a->dt != b->dt)
    return fail(MF_ERR_INVALID_ARG, "caches differ in nqb_total, Hs, B or dtype");
  if (a->nqb_total < 0 || a->nnz_capacity < 0 || b->nnz_capacity < 0 || a->Hs < 1 ||
      (a->B != 64 && a->B != 128) || (a->dt != MF_BF16 && a->dt != MF_F32))
    return fail(MF_ERR_INVALID_ARG, "cache sizes out of range");
  return MF_OK;
}

mf_status copy(void* dst, const void* src, size_t n, cudaStream_t s) {
  if (n == 0) return MF_OK;
  const cudaError_t e = cudaMemcpyAsync(dst, src, n, cudaMemcpyDefault, s);
  if (e != cudaSuccess) {
    mf::set_last_error((std::string("cudaMemcpyAsync: ") + cudaGetErrorString(e)).c_str());
    return MF_ERR_CUDA;
  }
  return MF_OK;
}

// Copies rows [a, b) of src into dst at the same positions (both layouts
// equal; entries e0 .. e1 of those rows).
mf_status copy_rows(const mf_csr_cache* src, mf_csr_cache* dst, int64_t a, int64_t b,
                    int64_t e0, int64_t e1, cudaStream_t s) {
  const size_t entry = size_t(src->B) * size_t(src->B) * size_t(src->Hs) * elem_bytes(src->dt);
  mf_status st = copy(dst->row_ptr + a, src->row_ptr + a, sizeof(int64_t) * size_t(b - a + 1), s);
  if (st == MF_OK) st = copy(dst->qb_seq + a, src->qb_seq + a, sizeof(int32_t) * size_t(b - a), s);
  if (st == MF_OK) st = copy(dst->qb_idx + a, src->qb_idx + a, sizeof(int32_t) * size_t(b - a), s);
  if (st == MF_OK)
    st = copy(dst->col_idx + e0, src->col_idx + e0, sizeof(int32_t) * size_t(e1 - e0), s);
  if (st == MF_OK)
    st = copy(static_cast<char*>(dst->values) + size_t(e0) * entry,
              static_cast<const char*>(src->values) + size_t(e0) * entry,
              entry * size_t(e1 - e0), s);
  return st;
}

}  // namespace

extern "C" {

mf_status mf_cache_offload(const mf_csr_cache* dev_src, mf_csr_cache* host_dst,
                           mf_stream_t stream) {
  mf_status st = same_layout(dev_src, host_dst);
  if (st != MF_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t n = dev_src->nqb_total;
  int64_t nnz = 0;
  cudaError_t e = cudaStreamSynchronize(s);
  if (e == cudaSuccess)
    e = cudaMemcpy(&nnz, dev_src->row_ptr + n, sizeof(int64_t), cudaMemcpyDefault);
  if (e != cudaSuccess) return fail(MF_ERR_CUDA, "reading the cache's entry count failed");
  if (nnz < 0 || nnz > dev_src->nnz_capacity)
    return fail(MF_ERR_CAPACITY, "the device cache holds more entries than its capacity");
  if (nnz > host_dst->nnz_capacity)
    return fail(MF_ERR_CAPACITY, "the host cache's capacity is below the entry count");
  return copy_rows(dev_src, host_dst, 0, n, 0, nnz, s);
}

mf_status mf_cache_fetch(const mf_csr_cache* host_src, mf_csr_cache* dev_dst, int64_t qb_begin,
                         int64_t qb_end, mf_stream_t stream) {
  mf_status st = same_layout(host_src, dev_dst);
  if (st != MF_OK) return st;
  if (qb_begin < 0 || qb_begin > qb_end || qb_end > host_src->nqb_total)
    return fail(MF_ERR_INVALID_ARG, "query-block range outside [0, nqb_total]");
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, host_src->row_ptr) == cudaSuccess &&
      attr.type == cudaMemoryTypeDevice)
    return fail(MF_ERR_INVALID_ARG, "the source cache's row_ptr must be host memory");
  cudaGetLastError();  // an unregistered host pointer may leave an error behind
  if (qb_begin == qb_end) return MF_OK;
  const int64_t e0 = host_src->row_ptr[qb_begin], e1 = host_src->row_ptr[qb_end];
  if (e0 < 0 || e1 < e0 || e1 > host_src->nnz_capacity)
    return fail(MF_ERR_INVALID_ARG, "the source cache's row pointers are inconsistent");
  if (e1 > dev_dst->nnz_capacity)
    return fail(MF_ERR_CAPACITY, "the device cache's capacity is below the rows' entries");
  return copy_rows(host_src, dev_dst, qb_begin, qb_end, e0, e1,
                   reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
