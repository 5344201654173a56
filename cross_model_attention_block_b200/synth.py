"""Seeded synthetic inputs for the MapFlow hot path.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic, so that the CUDA path and the CPU oracle can share it.

Workloads (MapFlow, "Accelerating Cross-Model LLM Inference via Attention Map
Reuse", 163.com article, section on the three system components): a sender
model's causal attention map over a context is compressed once and reused by a
receiver that keeps its own V.  The pages use real models and conversation
datasets; these seeded generators stand in for them:

* Q, K ~ 1.5 * N(0, 1) per sender head; the keys of the first four tokens of
  every sequence get +3 * (unit mean-query direction) of that head and
  sequence, computed in fp32 before rounding (attention sinks).
* V ~ N(0, 1) per receiver KV head; W ~ N(0, 1/Hs) (receiver x sender heads).
* Generation order per layer: for every sequence Q then K (sender), then V
  and W (receiver); numpy PCG64 streams, fp32 normals, rounded to the
  workload dtype by round-to-nearest-even.
* Varlen batches draw log-uniform lengths and a random page permutation from
  their own stream.
* Multi-turn contexts (the Round Attention page's conversations) draw round
  lengths in whole blocks, uniform in [2, 16] blocks, from their own stream
  (seed 3) until the sequence is covered; the last round is cut to fit.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

SINK_TOKENS = 4
SINK_GAIN = 3.0
QK_GAIN = 1.5
PAGE_SIZE = 16


@dataclass
class Workload:
    """One synthetic problem: sizes, selection threshold and bias settings."""

    name: str
    lengths: list
    Hs: int
    Hr: int
    Hkv: int
    d: int
    B: int
    tau: float
    band_bias: float
    band_width: int
    dtype: str  # "f32" or "bf16"
    seed: int = 0
    paged: bool = False
    sender_layers: int = 1
    # receivers: list of (name, n_layers, layer_table)
    receivers: list = field(default_factory=list)
    # multi-turn contexts: round start offsets per sequence (token offsets
    # within the sequence, then its length), and the watershed sender layer
    rounds: list = field(default_factory=list)
    watershed: int = 0

    @property
    def ntok(self) -> int:
        return int(sum(self.lengths))

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


def _varlen_lengths(n: int, lo: int, hi: int, seed: int):
    rng = np.random.default_rng(seed)
    u = rng.uniform(math.log(lo), math.log(hi), size=n)
    return [int(math.floor(math.exp(x))) for x in u], rng


def workloads() -> dict:
    """The synthetic workloads, keyed by a descriptive name."""
    w = {}
    w["tiny_f32_n512"] = Workload(
        "tiny_f32_n512", [512], Hs=4, Hr=2, Hkv=2, d=64, B=64, tau=0.9,
        band_bias=0.0, band_width=256, dtype="f32", seed=0)
    w["mid_bf16_n8192"] = Workload(
        "mid_bf16_n8192", [8192], Hs=32, Hr=32, Hkv=8, d=128, B=64, tau=0.95,
        band_bias=2.0, band_width=256, dtype="bf16", seed=0)
    w["large_bf16_n32768"] = Workload(
        "large_bf16_n32768", [32768], Hs=40, Hr=32, Hkv=8, d=128, B=128,
        tau=0.95, band_bias=2.0, band_width=256, dtype="bf16", seed=0)
    # the 32K workload's shape (heads, B = 128) at 8,192 tokens: small enough for
    # counter captures of the B = 128 kernels (a few GB on the device)
    w["large_shape_bf16_n8192"] = Workload(
        "large_shape_bf16_n8192", [8192], Hs=40, Hr=32, Hkv=8, d=128, B=128,
        tau=0.95, band_bias=2.0, band_width=256, dtype="bf16", seed=0)
    # one sender state (8 layers) consumed by two receivers; receiver layer l
    # of an L-layer receiver reads sender layer floor(l * 8 / L)
    r1 = [(l * 8) // 6 for l in range(6)]
    r2 = [(l * 8) // 4 for l in range(4)]
    w["multi_receiver_n16384"] = Workload(
        "multi_receiver_n16384", [16384], Hs=40, Hr=32, Hkv=8, d=128, B=64,
        tau=0.9, band_bias=2.0, band_width=256, dtype="bf16", seed=0,
        sender_layers=8, receivers=[("r1", 6, r1), ("r2", 4, r2)])
    w["multi_turn_rounds_n8192"] = Workload(
        "multi_turn_rounds_n8192", [8192], Hs=32, Hr=32, Hkv=8, d=128, B=64, tau=0.8,
        band_bias=2.0, band_width=256, dtype="bf16", seed=0, sender_layers=4,
        rounds=[round_starts(8192, 64, seed=3)], watershed=1)
    lens, _ = _varlen_lengths(64, 1024, 16384, seed=1)
    w["varlen_paged_64seq"] = Workload(
        "varlen_paged_64seq", lens, Hs=32, Hr=32, Hkv=8, d=128, B=64,
        tau=0.95, band_bias=2.0, band_width=256, dtype="bf16", seed=0,
        paged=True)
    return w


def round_starts(L: int, B: int, seed: int, lo_blocks: int = 2, hi_blocks: int = 16):
    """Round start offsets of one sequence of L tokens, then L: each round a
    whole number of blocks drawn uniformly in [lo_blocks, hi_blocks]."""
    rng = np.random.default_rng(seed)
    starts = [0]
    while starts[-1] < L:
        n = int(rng.integers(lo_blocks, hi_blocks + 1))
        starts.append(min(L, starts[-1] + n * B))
    return starts


def cu_seqlens(lengths) -> np.ndarray:
    out = np.zeros(len(lengths) + 1, dtype=np.int32)
    out[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    return out


def _round(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x))
    return t if dtype == "f32" else t.to(torch.bfloat16)


def sender_qk(lengths, Hs: int, d: int, dtype: str, rng: np.random.Generator,
              qk_gain: float = QK_GAIN, sink_gain: float = SINK_GAIN):
    """Q, K as [ntok, Hs, d] tensors of the workload dtype (CPU)."""
    qs, ks = [], []
    for L in lengths:
        q = rng.standard_normal((L, Hs, d), dtype=np.float32) * np.float32(qk_gain)
        k = rng.standard_normal((L, Hs, d), dtype=np.float32) * np.float32(qk_gain)
        if sink_gain != 0.0 and L > 0:  # an empty sequence has no sink
            u = q.mean(axis=0, dtype=np.float32)                      # [Hs, d]
            u = u / np.linalg.norm(u, axis=1, keepdims=True).astype(np.float32)
            ns = min(SINK_TOKENS, L)
            k[:ns] += np.float32(sink_gain) * u[None, :, :]
        qs.append(_round(q, dtype))
        ks.append(_round(k, dtype))
    return torch.cat(qs, 0).contiguous(), torch.cat(ks, 0).contiguous()


def receiver_vw(ntok: int, Hr: int, Hkv: int, Hs: int, d: int, dtype: str,
                rng: np.random.Generator):
    """V as [ntok, Hkv, d] and W as [Hr, Hs], of the workload dtype (CPU)."""
    v = rng.standard_normal((ntok, Hkv, d), dtype=np.float32)
    w = rng.standard_normal((Hr, Hs), dtype=np.float32) * np.float32(1.0 / math.sqrt(Hs))
    return _round(v, dtype), _round(w, dtype)


def page_rng(w: Workload) -> np.random.Generator:
    """The varlen stream (seed 1) positioned just after the length draws."""
    _, rng = _varlen_lengths(len(w.lengths), 1024, 16384, seed=1)
    return rng


def paged_v(V: torch.Tensor, lengths, rng: np.random.Generator,
            page_size: int = PAGE_SIZE):
    """Scatter contiguous V into a page pool under a random permutation.

    Returns (pool [npages, page_size, Hkv, d], page_table int32 [nseq, maxp]).
    Unused table entries hold -1; unused rows of a last page are zero.
    """
    npg = [(L + page_size - 1) // page_size for L in lengths]
    total = int(sum(npg))
    perm = rng.permutation(total).astype(np.int32)
    Hkv, d = V.shape[1], V.shape[2]
    pool = torch.zeros((total, page_size, Hkv, d), dtype=V.dtype)
    maxp = max(npg)
    table = np.full((len(lengths), maxp), -1, dtype=np.int32)
    logical = 0
    start = 0
    for s, L in enumerate(lengths):
        for p in range(npg[s]):
            phys = int(perm[logical])
            table[s, p] = phys
            lo = start + p * page_size
            hi = min(start + L, lo + page_size)
            pool[phys, : hi - lo] = V[lo:hi]
            logical += 1
        start += L
    return pool, torch.from_numpy(table)


@dataclass
class LayerInputs:
    Q: torch.Tensor
    K: torch.Tensor
    V: torch.Tensor
    W: torch.Tensor


def single_layer(w: Workload, Hr: int | None = None, Hkv: int | None = None):
    """Inputs of one sender layer and one receiver layer (configs with one layer)."""
    rng = np.random.default_rng(w.seed)
    Q, K = sender_qk(w.lengths, w.Hs, w.d, w.dtype, rng)
    V, W = receiver_vw(w.ntok, Hr or w.Hr, Hkv or w.Hkv, w.Hs, w.d, w.dtype, rng)
    return LayerInputs(Q, K, V, W)


def sender_layer(w: Workload, layer: int):
    """Q, K of one sender layer of a multi-layer workload (own stream per layer)."""
    rng = np.random.default_rng(1000 + layer)
    return sender_qk(w.lengths, w.Hs, w.d, w.dtype, rng)


def receiver_layer(w: Workload, receiver: int, layer: int):
    """V, W of one receiver layer of a multi-layer workload (own stream per layer)."""
    rng = np.random.default_rng(2000 + 100 * receiver + layer)
    return receiver_vw(w.ntok, w.Hr, w.Hkv, w.Hs, w.d, w.dtype, rng)


def small_case(lengths, Hs, Hr, Hkv, d, B, tau, dtype="bf16", band_bias=2.0,
               band_width=256, seed=0, sink_gain=SINK_GAIN):
    """A reduced problem with the same generators (for tests that the oracle
    finishes in seconds)."""
    w = Workload("small", list(lengths), Hs, Hr, Hkv, d, B, tau, band_bias,
                 band_width, dtype, seed)
    rng = np.random.default_rng(seed)
    Q, K = sender_qk(w.lengths, Hs, d, dtype, rng, sink_gain=sink_gain)
    V, W = receiver_vw(w.ntok, Hr, Hkv, Hs, d, dtype, rng)
    return w, LayerInputs(Q, K, V, W)
