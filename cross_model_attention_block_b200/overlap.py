"""Receiver prefill with the cache fetch overlapped with the early-layer
recompute (host scheduling of C-ABI calls on two CUDA streams).

MapFlow article (163.com, section on the three system components, second
component): the receiver finds the sender's cached blocks through the
prefix-hash index, and their retrieval overlaps its recomputation of its first
layers.  Here the cached state sits in the host-memory tier (pinned); for a
receiver whose first layers are recomputed and whose later layers are mapped:

* the copy stream fetches every mapped layer's cache, range of query blocks by
  range, into a device cache (mf_cache_fetch) and records an event per range;
* the compute stream runs the recompute layers, then, per mapped layer and
  range, waits for that range's event and runs the fused kernel over it
  (mf_mapped_av_range).

`serial=True` issues the same calls in order on one stream, the baseline the
overlap is measured against.  Every call writes the same O rows either way.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import mapflow as mfb


@dataclass
class MappedLayer:
    """One mapped receiver layer: where its sender cache lives, and its own
    head map W [Hr, Hs], V and output O."""

    host_cache: mfb.Cache
    dev_cache: mfb.Cache
    W: torch.Tensor
    V: torch.Tensor
    O: torch.Tensor


def chunk_ranges(nqb: int, chunks: int):
    """[0, nqb) cut into `chunks` consecutive ranges of near-equal length."""
    chunks = max(1, min(chunks, nqb)) if nqb else 1
    return [(nqb * c // chunks, nqb * (c + 1) // chunks) for c in range(chunks)
            if nqb * (c + 1) // chunks > nqb * c // chunks]


def prefill(recompute, mapped, Hr: int, Hkv: int, chunks: int = 8, serial: bool = False,
            copy_stream: torch.cuda.Stream | None = None):
    """Run a receiver prefill: `recompute` (callables, the receiver's own
    first layers) and the `mapped` layers (MappedLayer) over their fetched
    caches.  Returns the events recorded after each fetched range (copy
    stream) so callers can time the fetch."""
    compute = torch.cuda.current_stream()
    if not mapped:
        for f in recompute:
            f()
        return []
    nqb = mapped[0].dev_cache.nqb
    ranges = chunk_ranges(nqb, chunks)
    fetched = []
    if serial:
        for m in mapped:
            for r in ranges:
                mfb.cache_fetch(m.host_cache, m.dev_cache, r)
                ev = torch.cuda.Event(enable_timing=True)
                ev.record(compute)
                fetched.append(ev)
        for f in recompute:
            f()
        for m in mapped:
            for r in ranges:
                mfb.mapped_av(m.dev_cache, Hr, m.W, m.V, Hkv, O=m.O, qb_range=r,
                              workspace=getattr(m.dev_cache, "_av_ws", None))
        return fetched
    copy = copy_stream or torch.cuda.Stream()
    copy.wait_stream(compute)  # inputs written earlier on the compute stream
    with torch.cuda.stream(copy):
        for m in mapped:
            for r in ranges:
                mfb.cache_fetch(m.host_cache, m.dev_cache, r)
                ev = torch.cuda.Event(enable_timing=True)
                ev.record(copy)
                fetched.append(ev)
    for f in recompute:
        f()
    k = 0
    for m in mapped:
        for r in ranges:
            compute.wait_event(fetched[k])
            k += 1
            mfb.mapped_av(m.dev_cache, Hr, m.W, m.V, Hkv, O=m.O, qb_range=r,
                          workspace=getattr(m.dev_cache, "_av_ws", None))
    # the device caches are read on the compute stream from here on
    compute.wait_stream(copy)
    return fetched
