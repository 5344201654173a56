"""MapFlow hot path on B200: block-sparse attention-map compression and the
fused map-mix x V kernel, behind the C-ABI library libmapflow.so.

Submodules are imported on demand: ``synth`` (seeded inputs) needs no GPU and
no compiled code; ``mapflow`` (the ctypes binding) loads libmapflow.so and
fails loudly when it is missing.
"""
