/*
 * mapflow.h -- C ABI of libmapflow.so, the MapFlow hot path on B200 (sm_100a).
 *
 * MapFlow ("Accelerating Cross-Model LLM Inference via Attention Map Reuse",
 * PKU-DAIR; 163.com article, section on the three system components) reuses a
 * sender model's attention map in a receiver model.  The map is compressed to
 * regular 2-D blocks kept by cumulative attention probability, in stages that
 * never form the dense N x N matrix (block statistics, then extraction of the
 * kept blocks).  A fused kernel reads the kept blocks, combines sender heads
 * into receiver heads with a learned linear map W on chip, and multiplies the
 * result into the receiver's own V.  A prefix-hash index lets a receiver find
 * the cached state of a shared context.
 *
 * Conventions for every entry point:
 *  - Plain pointers and sizes only.  "device" pointers are CUDA global memory
 *    of the current device; "host" pointers are CPU memory.
 *  - The caller owns every buffer.  The library never allocates device memory;
 *    scratch space comes from a caller-provided workspace whose size the
 *    matching *_workspace() query returns (bytes, 256-byte aligned start).
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and is asynchronous.  Argument errors are found on the host
 *    before anything is enqueued and return a status; nothing is enqueued
 *    then.  Launch failures return MF_ERR_CUDA.  Conditions found on the
 *    device (a bounded wait that gave up, a CSR capacity overflow) set a
 *    per-device status word that mf_sync_status() reads and clears.
 *  - The text of the last error of the calling thread: mf_last_error().
 *  - A buffer that is empty at the descriptor's sizes may be NULL: Q, K, lse,
 *    V and O when ntok = 0; mass when there are no causal blocks; a cache's
 *    col_idx and values when nnz_capacity = 0, its qb_seq and qb_idx when
 *    nqb_total = 0.  Every other NULL pointer is MF_ERR_INVALID_ARG.
 *
 * Notation: ntok packed tokens over nseq sequences (cu_seqlens prefix sums);
 * Hs sender heads; Hr receiver heads; Hkv receiver KV heads; d head dim;
 * B block size.  Sequence s has L_s tokens, nqb_s = ceil(L_s / B) query
 * blocks and C_s = nqb_s (nqb_s + 1) / 2 causal blocks; blocks are aligned to
 * the start of each sequence and no token attends across sequences.
 */
#ifndef MAPFLOW_H
#define MAPFLOW_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* mf_stream_t; /* same object as cudaStream_t */

typedef enum {
  MF_OK = 0,
  MF_ERR_INVALID_ARG = 1,  /* null pointer, inconsistent sizes */
  MF_ERR_UNSUPPORTED = 2,  /* a shape the library has no kernel for */
  MF_ERR_WORKSPACE = 3,    /* workspace missing, misaligned or too small */
  MF_ERR_CUDA = 4,         /* a CUDA runtime call or a launch failed */
  MF_ERR_TIMEOUT = 5,      /* a device-side bounded wait gave up */
  MF_ERR_NOT_FOUND = 6,    /* prefix index lookup found no match */
  MF_ERR_CAPACITY = 7      /* kept blocks exceed the CSR capacity */
} mf_status;

typedef enum { MF_BF16 = 0, MF_F32 = 1 } mf_dtype;

/* One sender layer's context.
 * Logits (article: attention map of the sender, causal):
 *   s_h[i,j] = q_i.k_j / sqrt(d) + band_bias * [0 <= i-j < band_width], j <= i.
 * Q, K: device, [ntok][Hs][d] of dtype dt, row-major (token, head, dim).
 * Supported: B in {64,128}, d in {64,128}, 1 <= Hs <= 64, L_s <= 512 * B.
 * The bf16 tensor-core kernels need d = 128. */
typedef struct {
  int32_t nseq;
  const int32_t* cu_seqlens;      /* device [nseq+1], cu_seqlens[0] = 0 */
  const int32_t* cu_seqlens_host; /* host [nseq+1], the same values */
  int32_t Hs, d, B;
  float band_bias;
  int32_t band_width;
  mf_dtype dt;
} mf_attn_desc;

/* Block-sparse attention-map cache, CSR by query block (article: kept 2-D
 * blocks, a variable number per layer and position).  All pointers are
 * device memory owned by the caller; mf_select_extract fills them.
 *  row_ptr [nqb_total+1] int64: kept blocks of global query block q are
 *          entries row_ptr[q] .. row_ptr[q+1]-1.  Global query blocks are
 *          numbered sequence by sequence.
 *  col_idx [nnz_capacity] int32: key-block index within the sequence,
 *          ascending within a row.
 *  qb_seq, qb_idx [nqb_total] int32: sequence and in-sequence index of each
 *          global query block.
 *  values: kept probability blocks P_h[i,j] = exp(s_h[i,j] - lse_h[i]) for
 *          j <= i (0 above the diagonal and beyond the sequence end), of
 *          dtype dt.  Layout [nnz][B/16][B/8][2][Hs][64]: entry e, key group
 *          j/16, row slice i/8, half (i%8)/4, head h, then 64 elements of the
 *          pairs m = (i%4)*16 + j%16 in which the 8-element chunk m/8 is
 *          stored at chunk (m/8) ^ (h%8) (element m%8 inside it).  One
 *          (entry, key group, row slice) is Hs * 128 contiguous elements:
 *          the unit the fused kernel reads.
 *  cu_seqlens, nseq: the context the cache was built from (device). */
typedef struct {
  int64_t nqb_total;
  int64_t nnz_capacity;
  int64_t* row_ptr;
  int32_t* col_idx;
  int32_t* qb_seq;
  int32_t* qb_idx;
  void* values;
  int32_t Hs, B;
  mf_dtype dt;
  int32_t nseq;
  const int32_t* cu_seqlens;
} mf_csr_cache;

/* Receiver V (article: the receiver keeps its own V; PagedAttention and
 * varlen packing are supported).
 *  page_table == NULL: V is [ntok][Hkv][d] (packed like Q).
 *  otherwise V is a page pool [npages][page_size][Hkv][d] and
 *  page_table[s * max_pages_per_seq + p] is the pool page holding tokens
 *  p*page_size .. of sequence s; the pool holds npages pages.  page_size
 *  must be a multiple of 16.  Rows past a sequence's end are never read. */
typedef struct {
  const void* V;
  const int32_t* page_table;
  int32_t page_size;
  int32_t max_pages_per_seq;
  int64_t npages;           /* pages in the pool (paged only) */
  int32_t Hkv, d;
} mf_v_desc;

/* Library version string. */
const char* mf_version(void);

/* Text of the last error returned to this thread ("" if none). */
const char* mf_last_error(void);

/* Sizes of the block layout for a context (host only).
 * nqb_total = sum_s ceil(L_s/B); nblocks_total = sum_s C_s.  The mass array
 * of mf_block_stats has nblocks_total entries; nblocks_total is also the
 * CSR capacity that can never overflow. */
mf_status mf_layout_sizes(int32_t nseq, const int32_t* cu_seqlens_host, int32_t B,
                          int64_t* nqb_total, int64_t* nblocks_total);

/* Stage 1, block statistics (article: block-level statistics first, with no
 * dense N x N matrix).
 *  lse  [Hs][ntok] float (device, out): natural-log log-sum-exp of each
 *       causal row, lse_h[i] = log sum_{j<=i} exp(s_h[i,j]).
 *  mass [nblocks_total] float (device, out): block (s, qb, kb), kb <= qb, at
 *       index cu_blocks[s] + qb (qb+1)/2 + kb, where cu_blocks is the prefix
 *       sum of C_s; mass = sum_h sum_{i in qb} sum_{j in kb, j<=i}
 *       exp(s_h[i,j] - lse_h[i]).  Per-head partial sums are added in
 *       float64 in head order, so results do not depend on scheduling.
 *  ws: device workspace of at least mf_block_stats_workspace(desc) bytes. */
size_t mf_block_stats_workspace(const mf_attn_desc* desc);
mf_status mf_block_stats(const mf_attn_desc* desc, const void* Q, const void* K,
                         float* lse, float* mass, void* ws, size_t ws_bytes,
                         mf_stream_t stream);

/* As mf_block_stats, restricted to the global query blocks [qb_begin,
 * qb_end) (global order: sequence by sequence): only the lse rows of those
 * query blocks and the masses of their blocks (a contiguous span of the mass
 * array) are written; the rest of lse and mass is left as it was.  Every
 * query block's statistics depend only on its own rows and the keys before
 * them, so a context split into ranges -- one per GPU, or several per GPU --
 * gives, entry for entry, the result of one call (article, first and third
 * components: block statistics per position; chunked prefill).  Q and K must
 * hold the whole context.  Arguments, workspace and errors as
 * mf_block_stats, plus MF_ERR_INVALID_ARG unless
 * 0 <= qb_begin <= qb_end <= nqb_total. */
mf_status mf_block_stats_range(const mf_attn_desc* desc, const void* Q, const void* K,
                               float* lse, float* mass, int64_t qb_begin, int64_t qb_end,
                               void* ws, size_t ws_bytes, mf_stream_t stream);

/* Block statistics without a caller workspace.  The article has no
 * counterpart: this exists for callers that cannot allocate device memory,
 * such as a serving engine that gave all free HBM to its KV-cache pool, or a
 * host program with a fixed memory plan and no device allocator.
 *  Same inputs, outputs and results as mf_block_stats; the scratch comes from
 *  one array the library keeps in device memory (8 MiB, held by every GPU that
 *  loads the library until the process exits).  A context needing more than
 *  mf_block_stats_noalloc_max_workspace() bytes (see
 *  mf_block_stats_workspace) is rejected with MF_ERR_WORKSPACE and a message.
 *  Allocates nothing (no cudaMalloc, cudaFree or allocating library call).
 *  The first call on a device looks up the array's device address
 *  (cudaGetSymbolAddress) with that device current; make that first call
 *  before any stream capture.
 *  Every call shares the one array and leaves its contents behind; no part
 *  of it needs to start at zero, since each call writes every scratch word it
 *  reads.  Calls that overlap on the GPU (other streams, or other host
 *  threads using the same device) race on the array: serialize them. */
size_t mf_block_stats_noalloc_max_workspace(void);
mf_status mf_block_stats_noalloc(const mf_attn_desc* desc, const void* Q, const void* K,
                                 float* lse, float* mass, mf_stream_t stream);

/* Stage 2, selection and extraction (article: keep the important blocks by
 * cumulative attention probability; extract only the kept blocks).
 * Per global query block: order key blocks by mass descending, ties to the
 * lower index; take float64 prefix sums c_k in that order, T = c_last; keep
 * the first k* = min{k : c_k >= tau * T} blocks (all blocks if tau >= 1);
 * write them ascending into the CSR and write their probability blocks.
 *  out: caller-filled descriptor (pointers, nqb_total, nnz_capacity, Hs, B,
 *       dt, nseq, cu_seqlens); Hs/B/dt must match desc.
 *  Overflowing nnz_capacity sets the device status (MF_ERR_CAPACITY via
 *  mf_sync_status); entries past the capacity are dropped and the
 *  results are incomplete. */
size_t mf_select_extract_workspace(const mf_attn_desc* desc);
mf_status mf_select_extract(const mf_attn_desc* desc, const void* Q, const void* K,
                            const float* lse, const float* mass, double tau,
                            mf_csr_cache* out, void* ws, size_t ws_bytes,
                            mf_stream_t stream);

/* As mf_select_extract, restricted to the global query blocks [qb_begin,
 * qb_end): selection and extraction run on those query blocks only (lse and
 * mass are read only there), and every other row of the CSR is left empty
 * (row_ptr covers all nqb_total rows).  The kept sets and probability blocks
 * of the range are those of one full call; the cache holds entries of the
 * range only, so nnz_capacity can be the range's causal blocks.  A process
 * that owns several ranges keeps one cache per range; mf_mapped_av_range over
 * the same range reads it.  Arguments, workspace and errors as
 * mf_select_extract, plus MF_ERR_INVALID_ARG unless
 * 0 <= qb_begin <= qb_end <= nqb_total. */
mf_status mf_select_extract_range(const mf_attn_desc* desc, const void* Q, const void* K,
                                  const float* lse, const float* mass, double tau,
                                  mf_csr_cache* out, int64_t qb_begin, int64_t qb_end,
                                  void* ws, size_t ws_bytes, mf_stream_t stream);

/* Extraction for a given CSR: writes the probability blocks of every entry
 * of `cache` (row_ptr, col_idx, qb_seq and qb_idx filled, e.g. by
 * mf_select_extract of another layer or by mf_select_rounds) from this
 * layer's Q, K and lse (article, first component: the kept blocks are
 * extracted after the block statistics; Round Attention page, "方法详解": the
 * rounds kept at the watershed layer serve the later layers).  Values as in
 * mf_select_extract.  An entry whose key block is not a causal block of its
 * query block is skipped and sets the device status (MF_ERR_INVALID_ARG via
 * mf_sync_status).  Arguments and errors as mf_select_extract; the workspace
 * is at least mf_extract_workspace(desc) bytes. */
size_t mf_extract_workspace(const mf_attn_desc* desc);
mf_status mf_extract(const mf_attn_desc* desc, const void* Q, const void* K, const float* lse,
                     const mf_csr_cache* cache, void* ws, size_t ws_bytes, mf_stream_t stream);

/* Round-level selection, a second selection policy over the same cache
 * (Round Attention page, "方法详解": in a multi-turn context the attention
 * of a watershed layer picks, for every conversation round, the earlier
 * rounds that matter).  The context is split into nrounds rounds:
 * round_starts [nrounds+1] int32 (device) and round_starts_host (host, the
 * same values) are packed token offsets, from 0 to ntok; every non-empty
 * sequence starts a round, every round starts on a block boundary of its
 * sequence (offset from the sequence start a multiple of B) and ends inside
 * it.  With mass the watershed layer's block masses (mf_block_stats), the
 * mass of key round r for query round q is the float64 sum of the block
 * masses of q's query blocks over r's key blocks (causal).  Query round q
 * keeps its own round and the fewest earlier rounds, in order of mass
 * descending with ties to the lower round, whose masses with its own reach
 * tau * T (T: q's mass over rounds 0..q, float64); tau >= 1 keeps every
 * round.  Every query block of q keeps the blocks of the kept rounds up to
 * its own (ascending).  Fills row_ptr, col_idx, qb_seq, qb_idx of `out`;
 * the values are written by mf_extract, once per layer that uses the
 * selection.  Overflowing nnz_capacity sets the device status
 * (MF_ERR_CAPACITY).  Errors: MF_ERR_INVALID_ARG (rounds that break the rules
 * above, tau <= 0, NULL pointers), MF_ERR_WORKSPACE (workspace smaller than
 * mf_select_rounds_workspace, which returns 0 for an invalid layout). */
size_t mf_select_rounds_workspace(const mf_attn_desc* desc, int32_t nrounds,
                                  const int32_t* round_starts_host);
mf_status mf_select_rounds(const mf_attn_desc* desc, const float* mass, int32_t nrounds,
                           const int32_t* round_starts, const int32_t* round_starts_host,
                           double tau, mf_csr_cache* out, void* ws, size_t ws_bytes,
                           mf_stream_t stream);

/* Stage 3, fused map-mix x V (article: the fused kernel reads the sparse
 * blocks, combines heads on chip and multiplies straight into the receiver's
 * V, accumulating the output):
 *   O_r[i,:] = sum_{kb kept for qb(i)} sum_{j in kb}
 *              (sum_h W[r,h] P_h[i,j]) V_{g(r)}[j,:],  g(r) = floor(r*Hkv/Hr).
 *  desc: the sender context (cu_seqlens, Hs, B, dt as in the cache).
 *  W [Hr][Hs] of dtype dt (device); O [ntok][Hr][d] of dtype dt (device, out;
 *  every row of every sequence is written).  No renormalisation of the kept
 *  map.  Hr must be a multiple of Hkv.
 *  ws: device workspace of at least mf_mapped_av_workspace(...) bytes; it
 *  holds V regrouped per 16 keys in the tensor cores' operand layout. */
size_t mf_mapped_av_workspace(const mf_csr_cache* cache, const mf_attn_desc* desc,
                              int32_t Hr, const mf_v_desc* v);
mf_status mf_mapped_av(const mf_csr_cache* cache, const mf_attn_desc* desc,
                       int32_t Hr, const void* W, const mf_v_desc* v, void* O,
                       void* ws, size_t ws_bytes, mf_stream_t stream);

/* As mf_mapped_av, restricted to the global query blocks [qb_begin, qb_end)
 * (global order: sequence by sequence, as row_ptr): only the O rows of those
 * blocks are written, the rest of O is left as it was.  Uses:
 *  - chunked prefill: a context processed in consecutive ranges gives, row for
 *    row, the same O as one call (article, third component: the kernel works
 *    with chunked prefill);
 *  - prefix-partial reuse: when mf_index_lookup finds that a receiver's
 *    context shares its first `matched` blocks with a cached sender context,
 *    the sender's cache run over those blocks is exact for the receiver's
 *    rows there (a causal row attends only to keys of the shared prefix);
 *    the receiver computes its remaining rows itself.
 *  Arguments, workspace and errors as mf_mapped_av, plus MF_ERR_INVALID_ARG
 *  unless 0 <= qb_begin <= qb_end <= nqb_total. */
mf_status mf_mapped_av_range(const mf_csr_cache* cache, const mf_attn_desc* desc,
                             int32_t Hr, const void* W, const mf_v_desc* v, void* O,
                             int64_t qb_begin, int64_t qb_end, void* ws, size_t ws_bytes,
                             mf_stream_t stream);

/* ---- host-memory tier of the cache (article, second component: the
 * receiver's retrieval of cached blocks overlaps its recomputation of its
 * first layers).  A cache that outlives the sender's request lives in host
 * memory (pinned, for copies that overlap kernels); a receiver fetches the
 * rows it needs into a device cache on a copy stream.  Both caches have the
 * same layout (nqb_total, Hs, B, dt) and every entry sits at the same index
 * in both, so a device cache filled range by range serves mf_mapped_av_range
 * over each fetched range.  Only cudaMemcpyAsync is used; the library
 * allocates nothing. */

/* Copies a whole device cache (rows and entries row_ptr[nqb_total] of them)
 * into host buffers.  Synchronizes `stream` first and reads the entry count
 * with a blocking copy; the array copies are then enqueued on `stream`.
 * Errors: MF_ERR_INVALID_ARG (layouts differ, NULL arrays), MF_ERR_CAPACITY
 * (host capacity below the entry count), MF_ERR_CUDA. */
mf_status mf_cache_offload(const mf_csr_cache* dev_src, mf_csr_cache* host_dst,
                           mf_stream_t stream);

/* Enqueues on `stream` the copies of the rows of global query blocks
 * [qb_begin, qb_end) of a host cache into a device cache: row_ptr[qb_begin ..
 * qb_end], qb_seq and qb_idx of those rows, and their entries (col_idx,
 * values).  host_src's arrays are host memory (row_ptr is read on the host);
 * dev_dst's are device memory.  Errors: MF_ERR_INVALID_ARG (layouts differ,
 * a bad range, a device row_ptr in host_src), MF_ERR_CAPACITY (the rows'
 * entries exceed dev_dst's capacity), MF_ERR_CUDA. */
mf_status mf_cache_fetch(const mf_csr_cache* host_src, mf_csr_cache* dev_dst, int64_t qb_begin,
                         int64_t qb_end, mf_stream_t stream);

/* Diagnostic, not on the hot path: y[i] = 2^x[i] by the FMA-pipe
 * exponential of the block-statistics kernel, which computes 2 of every 8 of
 * its exponentials this way (the rest on MUFU): x = j + f, j = round(x); 2^f
 * from a degree-4 polynomial with relative minimax error 2.7e-6 on
 * [-1/2, 1/2]; 2^j added to the exponent; two lanes per packed f32x2
 * instruction (pairs of elements; a last odd element by the scalar form).
 * Meant for x <= 0; x below -125 is clamped to -125.  x, y: device float
 * arrays of n elements (they may be the same array).  Lets tests hold it
 * against CUDA's exp2f.  Errors: MF_ERR_INVALID_ARG (n < 0, or a NULL array
 * with n > 0), MF_ERR_CUDA (launch failure). */
mf_status mf_exp2_fma_eval(const float* x, float* y, int64_t n, mf_stream_t stream);

/* Which kernels the calls above run for a shape (host only; nothing is
 * launched).  Every stage has a tensor-core kernel and a scalar (CUDA-core,
 * float32 arithmetic) kernel that gives the same results more slowly:
 *  MF_PATH_STATS_TC   mf_block_stats runs the one-pass tensor-core kernel:
 *                     bf16, d = 128 and every sequence at most 256 key blocks
 *                     (L_s <= 256 * B); otherwise the scalar two-pass kernel;
 *  MF_PATH_EXTRACT_TC mf_select_extract extracts on the tensor cores: bf16,
 *                     d = 128;
 *  MF_PATH_AV_TC      mf_mapped_av runs the tensor-core fused kernel: bf16,
 *                     d = 128, Hs a multiple of 8, Hr 16 or 32, Hr / Hkv in
 *                     {2, 4, 8} (v may be NULL: this bit is then left 0).
 * Errors: as the calls' own argument checks (MF_ERR_INVALID_ARG,
 * MF_ERR_UNSUPPORTED), MF_ERR_INVALID_ARG for a NULL flags. */
enum { MF_PATH_STATS_TC = 1, MF_PATH_EXTRACT_TC = 2, MF_PATH_AV_TC = 4 };
mf_status mf_path_info(const mf_attn_desc* desc, int32_t Hr, const mf_v_desc* v,
                       uint32_t* flags);

/* Diagnostic, host only: the shared-memory plan the tensor-core fused kernel
 * uses for a shape (bf16, d = 128; Hs a multiple of 8 up to 64, Hr 16 or 32,
 * Hr / Hkv in {2, 4, 8}).  out[8] (host): 16-key groups per stage (1 or 2),
 * map ring slots, V ring slots, dynamic shared memory in bytes, and the
 * byte offsets of the map ring, the mixed-map ring, W^T and the barriers.
 * Errors: MF_ERR_INVALID_ARG (NULL out), MF_ERR_UNSUPPORTED (other shapes). */
mf_status mf_mapped_av_plan(int32_t Hs, int32_t Hr, int32_t Hkv, int32_t* out);

/* Diagnostic, for tests of the failure path: launches one kernel whose
 * bounded wait (the same one every tensor-core kernel uses) waits on an
 * mbarrier phase that nothing completes, gives up after limit_ms and raises
 * the timeout bit of the device status word, so the next mf_sync_status
 * returns MF_ERR_TIMEOUT.  Nothing faults; the context stays usable.
 * limit_ms in [1, 2000].  Errors: MF_ERR_INVALID_ARG, MF_ERR_CUDA. */
mf_status mf_selftest_timeout(int32_t limit_ms, mf_stream_t stream);

/* Waits for `stream`, then reads and clears the device status word of the
 * current device: MF_OK; MF_ERR_TIMEOUT (a bounded wait gave up);
 * MF_ERR_CAPACITY (kept blocks overflowed a CSR capacity); MF_ERR_INVALID_ARG
 * (the fused kernel met a cache row holding more entries than its query block
 * has key blocks, and clamped it). */
mf_status mf_sync_status(mf_stream_t stream);

/* ---- host-side prefix index (article: states are indexed by a prefix hash
 * that includes the preceding context; one sender state can serve several
 * receivers).  The index stores cache descriptors, not copies: the caller
 * keeps the buffers alive.  Not thread-safe per index object. */

/* Chained 128-bit hash per block of B tokens: block k hashes the previous
 * block's hash and its own tokens (two independent 64-bit FNV-1a chains).
 * out [ceil(n/B)][2] (host).  A partial last block is hashed over the tokens
 * it has. */
mf_status mf_prefix_hash(const int32_t* tokens, int64_t n, int32_t B, uint64_t seed,
                         uint64_t* out);

mf_status mf_index_create(void** index);
void mf_index_destroy(void* index);

/* Registers every prefix 1..nblocks of a context (hashes [nblocks][2]) for
 * sequence `seq` of `cache` at `sender_layer`.  A key already present is
 * replaced (the newest insert wins). */
mf_status mf_index_insert(void* index, const uint64_t* hashes, int64_t nblocks,
                          int32_t sender_layer, int32_t seq, const mf_csr_cache* cache);

/* Longest registered prefix of the query context (hashes [nblocks][2]) at
 * `sender_layer`: fills *cache, *seq and *matched_blocks, or returns
 * MF_ERR_NOT_FOUND (outputs untouched). */
mf_status mf_index_lookup(void* index, const uint64_t* hashes, int64_t nblocks,
                          int32_t sender_layer, mf_csr_cache* cache, int32_t* seq,
                          int64_t* matched_blocks);

/* Number of entries (prefix keys) held by the index. */
int64_t mf_index_size(void* index);

#ifdef __cplusplus
}
#endif

#endif /* MAPFLOW_H */
