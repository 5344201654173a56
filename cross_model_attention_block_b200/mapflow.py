"""ctypes binding of libmapflow.so (argument marshalling only).

Every step of the path runs in the library's CUDA kernels; this module only
turns torch tensors into pointers, allocates caller-owned outputs and
workspaces with torch, and passes torch's current stream.  There is no CPU
fallback: if the shared library is missing, loading raises.

Names follow the C ABI in include/mapflow.h.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# the in-tree build; MAPFLOW_LIB names another build of the same library
LIB_PATH = os.environ.get("MAPFLOW_LIB") or os.path.join(_HERE, "libmapflow.so")

MF_OK, MF_ERR_INVALID_ARG, MF_ERR_UNSUPPORTED, MF_ERR_WORKSPACE = 0, 1, 2, 3
MF_ERR_CUDA, MF_ERR_TIMEOUT, MF_ERR_NOT_FOUND, MF_ERR_CAPACITY = 4, 5, 6, 7
MF_BF16, MF_F32 = 0, 1

EXPORTED = [
    "mf_version", "mf_last_error", "mf_layout_sizes", "mf_block_stats_workspace",
    "mf_block_stats", "mf_block_stats_range", "mf_select_extract_workspace",
    "mf_select_extract", "mf_select_extract_range", "mf_extract_workspace", "mf_extract",
    "mf_select_rounds_workspace", "mf_select_rounds", "mf_cache_offload", "mf_cache_fetch",
    "mf_mapped_av_workspace", "mf_mapped_av", "mf_mapped_av_range", "mf_block_stats_noalloc",
    "mf_block_stats_noalloc_max_workspace",
    "mf_mapped_av_plan", "mf_path_info", "mf_exp2_fma_eval", "mf_selftest_timeout", "mf_sync_status", "mf_prefix_hash",
    "mf_index_create",
    "mf_index_destroy",
    "mf_index_insert", "mf_index_lookup", "mf_index_size",
]


class AttnDesc(C.Structure):
    _fields_ = [("nseq", C.c_int32), ("cu_seqlens", C.c_void_p),
                ("cu_seqlens_host", C.c_void_p), ("Hs", C.c_int32), ("d", C.c_int32),
                ("B", C.c_int32), ("band_bias", C.c_float), ("band_width", C.c_int32),
                ("dt", C.c_int)]


class CsrCache(C.Structure):
    _fields_ = [("nqb_total", C.c_int64), ("nnz_capacity", C.c_int64),
                ("row_ptr", C.c_void_p), ("col_idx", C.c_void_p), ("qb_seq", C.c_void_p),
                ("qb_idx", C.c_void_p), ("values", C.c_void_p), ("Hs", C.c_int32),
                ("B", C.c_int32), ("dt", C.c_int), ("nseq", C.c_int32),
                ("cu_seqlens", C.c_void_p)]


class VDesc(C.Structure):
    _fields_ = [("V", C.c_void_p), ("page_table", C.c_void_p), ("page_size", C.c_int32),
                ("max_pages_per_seq", C.c_int32), ("npages", C.c_int64), ("Hkv", C.c_int32),
                ("d", C.c_int32)]


class MapflowError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"mapflow status {status}: {msg}")
        self.status = status


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libmapflow.so and declare its signatures (no GPU needed)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with `python -m cross_model_attention_block_b200.build`")
    L = C.CDLL(path)
    P, I32, I64, SZ = C.c_void_p, C.c_int32, C.c_int64, C.c_size_t
    sig = {
        "mf_version": (C.c_char_p, []),
        "mf_last_error": (C.c_char_p, []),
        "mf_layout_sizes": (C.c_int, [I32, P, I32, P, P]),
        "mf_block_stats_workspace": (SZ, [P]),
        "mf_block_stats": (C.c_int, [P, P, P, P, P, P, SZ, P]),
        "mf_block_stats_range": (C.c_int, [P, P, P, P, P, I64, I64, P, SZ, P]),
        "mf_select_extract_workspace": (SZ, [P]),
        "mf_select_extract": (C.c_int, [P, P, P, P, P, C.c_double, P, P, SZ, P]),
        "mf_select_extract_range": (C.c_int, [P, P, P, P, P, C.c_double, P, I64, I64, P, SZ,
                                              P]),
        "mf_extract_workspace": (SZ, [P]),
        "mf_extract": (C.c_int, [P, P, P, P, P, P, SZ, P]),
        "mf_select_rounds_workspace": (SZ, [P, I32, P]),
        "mf_select_rounds": (C.c_int, [P, P, I32, P, P, C.c_double, P, P, SZ, P]),
        "mf_cache_offload": (C.c_int, [P, P, P]),
        "mf_cache_fetch": (C.c_int, [P, P, I64, I64, P]),
        "mf_mapped_av_workspace": (SZ, [P, P, I32, P]),
        "mf_mapped_av": (C.c_int, [P, P, I32, P, P, P, P, SZ, P]),
        "mf_mapped_av_range": (C.c_int, [P, P, I32, P, P, P, I64, I64, P, SZ, P]),
        "mf_block_stats_noalloc_max_workspace": (SZ, []),
        "mf_block_stats_noalloc": (C.c_int, [P, P, P, P, P, P]),
        "mf_mapped_av_plan": (C.c_int, [I32, I32, I32, P]),
        "mf_path_info": (C.c_int, [P, I32, P, P]),
        "mf_exp2_fma_eval": (C.c_int, [P, P, I64, P]),
        "mf_selftest_timeout": (C.c_int, [I32, P]),
        "mf_sync_status": (C.c_int, [P]),
        "mf_prefix_hash": (C.c_int, [P, I64, I32, C.c_uint64, P]),
        "mf_index_create": (C.c_int, [P]),
        "mf_index_destroy": (None, [P]),
        "mf_index_insert": (C.c_int, [P, P, I64, I32, I32, P]),
        "mf_index_lookup": (C.c_int, [P, P, I64, I32, P, P, P]),
        "mf_index_size": (I64, [P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


def _check(status):
    if status != MF_OK:
        raise MapflowError(status, load_library().mf_last_error().decode())


def _stream():
    # without a CUDA device only the library's argument checks can run (they
    # return before anything is enqueued); NULL then stands for the stream
    if not torch.cuda.is_available():
        return C.c_void_p(None)
    return C.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _dtype_code(dt):
    if dt == torch.bfloat16:
        return MF_BF16
    if dt == torch.float32:
        return MF_F32
    raise ValueError(f"unsupported dtype {dt}")


def _workspace(nbytes, device):
    buf = torch.empty(int(nbytes) + 256, dtype=torch.uint8, device=device)
    off = (-buf.data_ptr()) % 256
    return buf, buf.data_ptr() + off


@dataclass
class Context:
    """A packed varlen sender context and its attention settings."""

    cu_seqlens: torch.Tensor        # int32 [nseq+1] on the device
    cu_seqlens_host: np.ndarray     # int32 [nseq+1]
    Hs: int
    d: int
    B: int
    band_bias: float
    band_width: int
    dtype: torch.dtype

    @classmethod
    def make(cls, lengths, Hs, d, B, band_bias, band_width, dtype, device="cuda"):
        cu = np.zeros(len(lengths) + 1, dtype=np.int32)
        cu[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
        return cls(torch.from_numpy(cu).to(device), cu, Hs, d, B, float(band_bias),
                   int(band_width), dtype)

    @property
    def nseq(self):
        return len(self.cu_seqlens_host) - 1

    @property
    def ntok(self):
        return int(self.cu_seqlens_host[-1])

    def desc(self) -> AttnDesc:
        self._host = np.ascontiguousarray(self.cu_seqlens_host, dtype=np.int32)
        return AttnDesc(self.nseq, self.cu_seqlens.data_ptr(),
                        self._host.ctypes.data, self.Hs, self.d, self.B,
                        self.band_bias, self.band_width, _dtype_code(self.dtype))

    def layout_sizes(self):
        return layout_sizes(self.cu_seqlens_host, self.B)

    def range_blocks(self, qb_begin, qb_end):
        """Causal blocks of the global query blocks [qb_begin, qb_end): the
        CSR capacity a cache of that range can never overflow."""
        n = 0
        q0 = 0
        for L in np.diff(self.cu_seqlens_host):
            nq = (int(L) + self.B - 1) // self.B
            a, b = max(qb_begin - q0, 0), min(qb_end - q0, nq)
            if a < b:
                n += b * (b + 1) // 2 - a * (a + 1) // 2
            q0 += nq
        return n


def layout_sizes(cu_seqlens_host, B):
    """(nqb_total, nblocks_total) of a context."""
    L = load_library()
    cu = np.ascontiguousarray(cu_seqlens_host, dtype=np.int32)
    a, b = C.c_int64(), C.c_int64()
    _check(L.mf_layout_sizes(len(cu) - 1, cu.ctypes.data, B, C.byref(a), C.byref(b)))
    return a.value, b.value


def block_stats(ctx: Context, Q, K, lse=None, mass=None, qb_range=None):
    """Stage 1: lse [Hs, ntok] float32 and block masses [nblocks] float32.
    `qb_range` = (begin, end) restricts the call to those global query
    blocks: only their lse rows and block masses are written."""
    L = load_library()
    d = ctx.desc()
    _, nblocks = ctx.layout_sizes()
    dev = Q.device
    if lse is None:
        lse = torch.empty((ctx.Hs, ctx.ntok), dtype=torch.float32, device=dev)
    if mass is None:
        mass = torch.empty((max(nblocks, 1),), dtype=torch.float32, device=dev)
    nbytes = L.mf_block_stats_workspace(C.byref(d))
    if nbytes == 0:
        _check(MF_ERR_INVALID_ARG)
    ws, wsp = _workspace(nbytes, dev)
    if qb_range is None:
        _check(L.mf_block_stats(C.byref(d), _ptr(Q), _ptr(K), _ptr(lse), _ptr(mass),
                                C.c_void_p(wsp), nbytes, _stream()))
    else:
        _check(L.mf_block_stats_range(C.byref(d), _ptr(Q), _ptr(K), _ptr(lse), _ptr(mass),
                                      int(qb_range[0]), int(qb_range[1]), C.c_void_p(wsp),
                                      nbytes, _stream()))
    ctx._stats_ws = ws  # keep the workspace alive until the stream has used it
    return lse, mass


class Cache:
    """Caller-owned buffers of one CSR block cache (device memory, or pinned
    host memory for the host tier)."""

    def __init__(self, ctx: Context, capacity=None, device="cuda", pin=False):
        nqb, nblocks = ctx.layout_sizes()
        cap = nblocks if capacity is None else int(capacity)
        self.ctx = ctx
        self.nqb = nqb
        self.capacity = cap
        self.row_ptr = torch.empty(nqb + 1, dtype=torch.int64, device=device)
        self.col_idx = torch.empty(max(cap, 1), dtype=torch.int32, device=device)
        self.qb_seq = torch.empty(max(nqb, 1), dtype=torch.int32, device=device)
        self.qb_idx = torch.empty(max(nqb, 1), dtype=torch.int32, device=device)
        nvals = max(cap, 1) * ctx.B * ctx.B * ctx.Hs
        self.values = torch.empty(nvals, dtype=ctx.dtype, device=device)
        if pin:
            for name in ("row_ptr", "col_idx", "qb_seq", "qb_idx", "values"):
                setattr(self, name, getattr(self, name).pin_memory())

    def struct(self) -> CsrCache:
        return CsrCache(self.nqb, self.capacity, self.row_ptr.data_ptr(),
                        self.col_idx.data_ptr(), self.qb_seq.data_ptr(),
                        self.qb_idx.data_ptr(), self.values.data_ptr(), self.ctx.Hs,
                        self.ctx.B, _dtype_code(self.ctx.dtype), self.ctx.nseq,
                        self.ctx.cu_seqlens.data_ptr())

    @property
    def nnz(self):
        return int(self.row_ptr[-1].item())

    def values_view(self):
        """values in stored order [capacity, B/16 key groups, B/8 row slices, 2 halves,
        Hs, 8 chunks, 8] (see the C header for the chunk permutation)."""
        B, Hs = self.ctx.B, self.ctx.Hs
        return self.values[: self.capacity * B * B * Hs].view(
            self.capacity, B // 16, B // 8, 2, Hs, 8, 8)


def select_extract(ctx: Context, Q, K, lse, mass, tau, cache: Cache | None = None,
                   qb_range=None):
    """Stage 2: kept blocks per query block (CSR) and their probability blocks.
    `qb_range` = (begin, end) restricts the call to those global query blocks;
    the CSR rows of every other query block are empty."""
    L = load_library()
    d = ctx.desc()
    if cache is None:
        cache = Cache(ctx, device=Q.device)
    cs = cache.struct()
    nbytes = L.mf_select_extract_workspace(C.byref(d))
    if nbytes == 0:
        _check(MF_ERR_INVALID_ARG)
    ws, wsp = _workspace(nbytes, Q.device)
    if qb_range is None:
        _check(L.mf_select_extract(C.byref(d), _ptr(Q), _ptr(K), _ptr(lse), _ptr(mass),
                                   float(tau), C.byref(cs), C.c_void_p(wsp), nbytes, _stream()))
    else:
        _check(L.mf_select_extract_range(C.byref(d), _ptr(Q), _ptr(K), _ptr(lse), _ptr(mass),
                                         float(tau), C.byref(cs), int(qb_range[0]),
                                         int(qb_range[1]), C.c_void_p(wsp), nbytes,
                                         _stream()))
    cache._ws = ws  # keep the workspace alive until the stream has used it
    return cache


def extract(ctx: Context, Q, K, lse, cache: Cache):
    """Probability blocks of every entry of a filled CSR (this layer's Q, K, lse)."""
    L = load_library()
    d = ctx.desc()
    nbytes = L.mf_extract_workspace(C.byref(d))
    if nbytes == 0:
        _check(MF_ERR_INVALID_ARG)
    ws, wsp = _workspace(nbytes, Q.device)
    cs = cache.struct()
    _check(L.mf_extract(C.byref(d), _ptr(Q), _ptr(K), _ptr(lse), C.byref(cs), C.c_void_p(wsp),
                        nbytes, _stream()))
    cache._ws = ws
    return cache


def select_rounds(ctx: Context, mass, round_starts, tau, cache: Cache | None = None):
    """Round-level selection from the watershed layer's block masses: the CSR
    of every query block (values are written by `extract`, per layer).
    round_starts: packed token offsets of the rounds, 0 .. ntok."""
    L = load_library()
    d = ctx.desc()
    st = np.ascontiguousarray(round_starts, dtype=np.int32)
    nr = len(st) - 1
    dev = mass.device
    st_dev = torch.from_numpy(st).to(dev)
    if cache is None:
        cache = Cache(ctx, device=dev)
    nbytes = L.mf_select_rounds_workspace(C.byref(d), nr, st.ctypes.data)
    if nbytes == 0:
        _check(L.mf_select_rounds(C.byref(d), _ptr(mass), nr, _ptr(st_dev), st.ctypes.data,
                                  float(tau), None, None, 0, _stream()))
        _check(MF_ERR_INVALID_ARG)
    ws, wsp = _workspace(nbytes, dev)
    cs = cache.struct()
    _check(L.mf_select_rounds(C.byref(d), _ptr(mass), nr, _ptr(st_dev), st.ctypes.data,
                              float(tau), C.byref(cs), C.c_void_p(wsp), nbytes, _stream()))
    cache._round_ws = (ws, st_dev)
    return cache


def cache_offload(dev_cache: Cache, host_cache: Cache):
    """Copy a device cache into a (pinned) host cache of the same layout."""
    _check(load_library().mf_cache_offload(C.byref(dev_cache.struct()),
                                           C.byref(host_cache.struct()), _stream()))
    return host_cache


def cache_fetch(host_cache: Cache, dev_cache: Cache, qb_range):
    """Enqueue the copies of a range of rows of a host cache into a device
    cache on the current stream."""
    _check(load_library().mf_cache_fetch(C.byref(host_cache.struct()),
                                         C.byref(dev_cache.struct()), int(qb_range[0]),
                                         int(qb_range[1]), _stream()))
    return dev_cache


def mapped_av(cache: Cache, Hr, W, V, Hkv, page_table=None, page_size=16, O=None,
              workspace=None, qb_range=None):
    """Stage 3: O [ntok, Hr, d] = (W-mixed kept map) x V (fused).

    `workspace` may be a uint8 device tensor reused across calls (grown when
    too small); by default one is allocated per call.  `qb_range` =
    (begin, end) restricts the call to those global query blocks (chunked
    prefill, prefix reuse): only their rows of O are written."""
    L = load_library()
    ctx = cache.ctx
    d = ctx.desc()
    if O is None:
        O = torch.empty((ctx.ntok, Hr, ctx.d), dtype=ctx.dtype, device=W.device)
    maxp = 0 if page_table is None else int(page_table.shape[1])
    npages = 0 if page_table is None else int(V.shape[0])
    vd = VDesc(V.data_ptr(), 0 if page_table is None else page_table.data_ptr(),
               page_size, maxp, npages, Hkv, ctx.d)
    cs = cache.struct()
    nbytes = L.mf_mapped_av_workspace(C.byref(cs), C.byref(d), int(Hr), C.byref(vd))
    if nbytes == 0:
        _check(MF_ERR_INVALID_ARG)
    if workspace is not None and workspace.numel() >= nbytes + 256:
        ws = workspace
        wsp = ws.data_ptr() + (-ws.data_ptr()) % 256
    else:
        ws, wsp = _workspace(nbytes, W.device)
    if qb_range is None:
        _check(L.mf_mapped_av(C.byref(cs), C.byref(d), int(Hr), _ptr(W), C.byref(vd), _ptr(O),
                              C.c_void_p(wsp), nbytes, _stream()))
    else:
        _check(L.mf_mapped_av_range(C.byref(cs), C.byref(d), int(Hr), _ptr(W), C.byref(vd),
                                    _ptr(O), int(qb_range[0]), int(qb_range[1]),
                                    C.c_void_p(wsp), nbytes, _stream()))
    cache._av_ws = ws  # keep the workspace alive until the stream has used it
    return O


def mapped_av_plan(Hs, Hr, Hkv):
    """The fused kernel's shared-memory plan for a shape (host only): dict."""
    out = np.zeros(8, dtype=np.int32)
    _check(load_library().mf_mapped_av_plan(int(Hs), int(Hr), int(Hkv), out.ctypes.data))
    keys = ("groups_per_stage", "map_stages", "v_stages", "smem_bytes", "off_map", "off_mt",
            "off_w", "off_bar")
    return dict(zip(keys, (int(v) for v in out)))


MF_PATH_STATS_TC, MF_PATH_EXTRACT_TC, MF_PATH_AV_TC = 1, 2, 4


def path_info(ctx: Context, Hr=None, Hkv=None):
    """Which kernels the three calls run for a shape (host only): dict of
    bools for the statistics, extraction and fused stages."""
    d = ctx.desc()
    vd = None
    if Hr is not None:
        vd = VDesc(0, 0, 16, 0, 0, int(Hkv), ctx.d)
    f = C.c_uint32()
    _check(load_library().mf_path_info(C.byref(d), int(Hr or 0),
                                       None if vd is None else C.byref(vd), C.byref(f)))
    return {"stats_tc": bool(f.value & MF_PATH_STATS_TC),
            "extract_tc": bool(f.value & MF_PATH_EXTRACT_TC),
            "mapped_av_tc": bool(f.value & MF_PATH_AV_TC)}


def exp2_fma_eval(x):
    """2^x by the statistics kernel's FMA-pipe exponential (float32 CUDA tensor)."""
    L = load_library()
    if x.dtype != torch.float32 or not x.is_cuda:
        _check(MF_ERR_INVALID_ARG)
    x = x.contiguous()
    y = torch.empty_like(x)
    _check(L.mf_exp2_fma_eval(_ptr(x), _ptr(y), x.numel(), _stream()))
    return y


def selftest_timeout(limit_ms=20):
    """Make one bounded device wait give up (nothing completes its barrier)."""
    _check(load_library().mf_selftest_timeout(int(limit_ms), _stream()))


def sync_status():
    """Wait for the current stream; raise on a device-side status."""
    _check(load_library().mf_sync_status(_stream()))


def prefix_hash(tokens, B, seed=0):
    """Chained 128-bit per-block prefix hashes, uint64 [ceil(n/B), 2]."""
    L = load_library()
    t = np.ascontiguousarray(tokens, dtype=np.int32)
    nb = (len(t) + B - 1) // B
    out = np.zeros((max(nb, 1), 2), dtype=np.uint64)
    _check(L.mf_prefix_hash(t.ctypes.data if len(t) else None, len(t), B, C.c_uint64(seed),
                            out.ctypes.data))
    return out[:nb]


class PrefixIndex:
    """Host prefix-hash index of cache descriptors (C ABI object)."""

    def __init__(self):
        self._L = load_library()
        h = C.c_void_p()
        _check(self._L.mf_index_create(C.byref(h)))
        self._h = h

    def close(self):
        if self._h:
            self._L.mf_index_destroy(self._h)
            self._h = None

    __del__ = close

    def __len__(self):
        return int(self._L.mf_index_size(self._h))

    def insert(self, hashes, sender_layer, seq, cache_struct: CsrCache):
        h = np.ascontiguousarray(hashes, dtype=np.uint64)
        _check(self._L.mf_index_insert(self._h, h.ctypes.data, len(h), sender_layer, seq,
                                       C.byref(cache_struct)))

    def lookup(self, hashes, sender_layer):
        """(CsrCache, seq, matched_blocks) or None when nothing matches."""
        h = np.ascontiguousarray(hashes, dtype=np.uint64)
        out = CsrCache()
        seq, matched = C.c_int32(), C.c_int64()
        st = self._L.mf_index_lookup(self._h, h.ctypes.data if len(h) else None, len(h),
                                     sender_layer, C.byref(out), C.byref(seq),
                                     C.byref(matched))
        if st == MF_ERR_NOT_FOUND:
            return None
        _check(st)
        return out, seq.value, matched.value
