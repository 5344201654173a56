"""Plain CPU oracle of the MapFlow hot path (fp64, numpy).

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the timed CPU
baseline of the benchmark may import this module; the library never does.  It
shares no code with the CUDA path: the two meet only in the seeded input
generators, which hold none of the method's arithmetic.

What it computes follows the MapFlow article ("Accelerating Cross-Model LLM
Inference via Attention Map Reuse", 163.com):

* section "让复用真正省时", first component: the sender's attention map is
  compressed to a block-sparse map of regular 2-D blocks, keeping blocks by
  cumulative attention probability, with block-level statistics computed
  first and the kept blocks extracted afterwards;
* same section, second component: one sender state serves several receivers;
* same section, third component: the kept blocks are read, the sender heads
  are combined linearly into receiver heads, and the result is multiplied by
  the receiver's own V to accumulate the output (no renormalisation);
* section "从内部表示...": the head map is a learned linear combination
  W[Hr x Hs]; sender and receiver share token positions.

Readings where the article is silent (each is listed in the design notes):
one kept set per (layer, query block) shared by all heads, with the mass
summed over the block's query rows and all sender heads; keep the smallest set
whose cumulative mass reaches tau * total, blocks ordered by mass descending
and ties broken by the lower key-block index; tau >= 1 keeps every causal
block; band bias beta added to the scaled logit when 0 <= i - j < band_width;
contiguous GQA grouping g(r) = floor(r * Hkv / Hr); blocks aligned to each
sequence start, no attention across sequences, partial last blocks.

Round-level selection (the Round Attention page, "方法详解": a watershed
layer's attention decides, per conversation round, which earlier rounds to
keep; the kept rounds then serve the later layers) is the second selection
policy over the same block cache.  Readings: every round starts on a block
boundary of its sequence; a query round always keeps its own tokens and adds
the fewest earlier rounds, heaviest first (ties to the lower round), whose
mass together with its own reaches tau * T, where the mass of key round r for
query round q sums P_h[i, j] over the heads, the rows i of q and the keys j
of r (j <= i), and T sums it over every round up to q; tau >= 1 keeps every
round.  One selection, taken at the watershed layer, gives the kept blocks of
every later layer.

Every function works on one sequence and one query block at a time, so memory
stays O(B * L * Hs) and any single block can be checked at full size.
Every function here is pinned by the tests in tests/test_oracle_pins.py and
tests/test_round_pins.py.
"""
from __future__ import annotations

import math

import numpy as np


def _f64(x) -> np.ndarray:
    """Upcast a torch tensor or array to a float64 numpy array."""
    if hasattr(x, "detach"):
        import torch
        return x.detach().to(torch.float64).cpu().numpy()
    return np.asarray(x, dtype=np.float64)


def scores(Q, K, i0: int, i1: int, band_bias: float, band_width: int) -> np.ndarray:
    """Causal sender logits of query rows [i0, i1) of one sequence.

    s_h[i, j] = q_i . k_j / sqrt(d) + beta * [0 <= i - j < band_width]
    for j <= i, else -inf.  Q, K: [L, Hs, d] float64 (one sequence).
    Returns [Hs, i1 - i0, i1].
    """
    d = Q.shape[2]
    q = np.transpose(Q[i0:i1], (1, 0, 2))            # [Hs, R, d]
    k = np.transpose(K[:i1], (1, 2, 0))              # [Hs, d, i1]
    s = np.matmul(q, k) / math.sqrt(d)               # [Hs, R, i1]
    i = np.arange(i0, i1)[:, None]
    j = np.arange(i1)[None, :]
    delta = i - j
    s = s + band_bias * ((delta >= 0) & (delta < band_width))
    return np.where(delta >= 0, s, -np.inf)


def lse_and_probs(s: np.ndarray):
    """Row-wise log-sum-exp and softmax of causal logits (stable form).

    P_h[i, j] = exp(s - max_j s) / sum_j exp(s - max_j s);
    lse_h[i] = max_j s + log sum_j exp(s - max_j s).
    """
    m = np.max(s, axis=2, keepdims=True)
    e = np.exp(s - m)
    z = np.sum(e, axis=2, keepdims=True)
    return (m + np.log(z))[..., 0], e / z


def block_mass(P: np.ndarray, B: int) -> np.ndarray:
    """Block statistics of one query block's probability strip.

    mass[kb] = sum_h sum_{i in qb} sum_{j in kb} P_h[i, j], kb = 0..ceil(L'/B)-1
    where L' = P.shape[2] is the end of the query block (the causal limit).
    """
    L1 = P.shape[2]
    nkb = (L1 + B - 1) // B
    out = np.zeros(nkb, dtype=np.float64)
    for kb in range(nkb):
        out[kb] = P[:, :, kb * B:min(L1, (kb + 1) * B)].sum()
    return out


def select_blocks(mass: np.ndarray, tau: float) -> np.ndarray:
    """Smallest set of key blocks whose cumulative mass reaches tau * total.

    Order the blocks by mass descending, ties to the lower index; take fp64
    prefix sums c_k in that order, T = c_last; keep the first k* entries with
    k* = min{k : c_k >= tau * T}; tau >= 1 keeps every block.  Returns the
    kept key-block indices in ascending order.
    """
    n = mass.shape[0]
    if tau >= 1.0:
        return np.arange(n)
    order = sorted(range(n), key=lambda kb: (-mass[kb], kb))
    c = 0.0
    csum = []
    for kb in order:
        c += float(mass[kb])
        csum.append(c)
    T = csum[-1]
    kstar = n
    for k in range(n):
        if csum[k] >= tau * T:
            kstar = k + 1
            break
    return np.array(sorted(order[:kstar]), dtype=np.int64)


def cumulative_fractions(mass: np.ndarray):
    """(order, c_k / T) of the selection rule, for near-tau exemption checks."""
    n = mass.shape[0]
    order = sorted(range(n), key=lambda kb: (-mass[kb], kb))
    c = np.cumsum(np.array([mass[kb] for kb in order], dtype=np.float64))
    return np.array(order), c / c[-1]


def mixed_map(P: np.ndarray, kept: np.ndarray, W: np.ndarray, B: int) -> np.ndarray:
    """M_r[i, j] = sum_h W[r, h] P_h[i, j] on kept key blocks, 0 elsewhere."""
    Hs, R, L1 = P.shape
    mask = np.zeros(L1, dtype=bool)
    for kb in kept:
        mask[kb * B:min(L1, (kb + 1) * B)] = True
    Pk = np.where(mask[None, None, :], P, 0.0)
    return np.tensordot(W, Pk, axes=(1, 0))      # sum over h


def mapped_av(M: np.ndarray, V: np.ndarray, Hkv: int) -> np.ndarray:
    """O_r[i, :] = sum_j M_r[i, j] V_{g(r)}[j, :], g(r) = floor(r * Hkv / Hr).

    M: [Hr, R, L1]; V: [L, Hkv, d] (one sequence).  Returns [R, Hr, d].
    """
    Hr, R, L1 = M.shape
    d = V.shape[2]
    O = np.zeros((R, Hr, d), dtype=np.float64)
    for r in range(Hr):
        g = (r * Hkv) // Hr
        O[:, r, :] = M[r] @ V[:L1, g, :]
    return O


def query_block(Qs, Ks, qb: int, B: int, band_bias: float, band_width: int):
    """Logits, lse, probabilities and block masses of query block qb."""
    L = Qs.shape[0]
    i0, i1 = qb * B, min(L, (qb + 1) * B)
    s = scores(Qs, Ks, i0, i1, band_bias, band_width)
    lse, P = lse_and_probs(s)
    return lse, P, block_mass(P, B)


def run_sequence(Qs, Ks, Vs, W, Hkv: int, B: int, tau: float, band_bias: float,
                 band_width: int, qbs=None, want_values: bool = False):
    """The whole path on one sequence (arrays are fp64, one sequence).

    Returns a dict with per-query-block lse [Hs, rows], mass [qb+1], kept key
    blocks, output rows O [rows, Hr, d] and, when asked, the kept probability
    blocks {kb: P [Hs, rows, B]} (zero beyond the causal limit).
    """
    L = Qs.shape[0]
    nqb = (L + B - 1) // B
    out = {}
    for qb in (range(nqb) if qbs is None else qbs):
        lse, P, mass = query_block(Qs, Ks, qb, B, band_bias, band_width)
        kept = select_blocks(mass, tau)
        M = mixed_map(P, kept, W, B)
        rec = {"lse": lse, "mass": mass, "kept": kept, "O": mapped_av(M, Vs, Hkv)}
        if want_values:
            vals = {}
            for kb in kept:
                blk = np.zeros((P.shape[0], P.shape[1], B))
                hi = min(P.shape[2], (kb + 1) * B)
                blk[:, :, :hi - kb * B] = P[:, :, kb * B:hi]
                vals[int(kb)] = blk
            rec["values"] = vals
        out[qb] = rec
    return out


def run_layer(Q, K, V, W, lengths, Hkv: int, B: int, tau: float,
              band_bias: float, band_width: int, want_values: bool = False):
    """The whole path over a packed varlen batch (torch or numpy inputs).

    Q, K: [ntok, Hs, d]; V: [ntok, Hkv, d]; W: [Hr, Hs].
    Returns a list (one dict per sequence, as run_sequence) and the packed
    output O [ntok, Hr, d].
    """
    Q, K, V, W = _f64(Q), _f64(K), _f64(V), _f64(W)
    Hr, d = W.shape[0], V.shape[2]
    O = np.zeros((Q.shape[0], Hr, d))
    res = []
    start = 0
    for L in lengths:
        r = run_sequence(Q[start:start + L], K[start:start + L], V[start:start + L],
                         W, Hkv, B, tau, band_bias, band_width,
                         want_values=want_values)
        for qb, rec in r.items():
            O[start + qb * B:start + qb * B + rec["O"].shape[0]] = rec["O"]
        res.append(r)
        start += L
    return res, O


# ------------------------------------------------ round-level selection


def round_of_token(round_starts, j: int) -> int:
    """Index of the round holding token j (round_starts ascending, [0] = 0)."""
    r = 0
    while r + 1 < len(round_starts) and round_starts[r + 1] <= j:
        r += 1
    return r


def round_mass(Qs, Ks, round_starts, q: int, band_bias: float, band_width: int,
               rows_per_chunk: int = 64) -> np.ndarray:
    """Attention mass of query round q on every round 0..q of one sequence.

    m[r] = sum_h sum_{i in round q} sum_{j in round r, j <= i} P_h[i, j],
    straight from the probabilities of the rows of round q (no block sums),
    taken over the round's rows in chunks to bound memory.
    round_starts: token offsets of the rounds, then the sequence length.
    """
    m = np.zeros(q + 1)
    for c0 in range(round_starts[q], round_starts[q + 1], rows_per_chunk):
        c1 = min(round_starts[q + 1], c0 + rows_per_chunk)
        _, P = lse_and_probs(scores(Qs, Ks, c0, c1, band_bias, band_width))  # [Hs, rows, c1]
        for r in range(q + 1):
            m[r] += P[:, :, round_starts[r]:min(round_starts[r + 1], c1)].sum()
    return m


def select_rounds(m: np.ndarray, tau: float) -> np.ndarray:
    """Kept rounds of the query round q = len(m) - 1, ascending.

    Round q is always kept.  Earlier rounds in order of mass descending, ties
    to the lower index; keep the fewest k of them with m[q] + (sum of the
    first k) >= tau * T, T = sum(m) (fp64 sums in that order); all of them if
    never reached; tau >= 1 keeps every round.
    """
    q = len(m) - 1
    if tau >= 1.0:
        return np.arange(q + 1)
    T = float(np.sum(m))
    order = sorted(range(q), key=lambda r: (-m[r], r))
    c = float(m[q])
    k = 0
    while c < tau * T and k < q:
        c += float(m[order[k]])
        k += 1
    return np.array(sorted(order[:k] + [q]), dtype=np.int64)


def round_kept_blocks(kept_rounds, round_starts, qb: int, B: int) -> np.ndarray:
    """Key blocks kb <= qb that lie in a kept round (rounds start on block
    boundaries, so a block lies in exactly one round)."""
    kept = set(int(r) for r in kept_rounds)
    return np.array([kb for kb in range(qb + 1)
                     if round_of_token(round_starts, kb * B) in kept], dtype=np.int64)


def run_rounds_sequence(Qw, Kw, layers, W, Hkv: int, B: int, tau: float,
                        round_starts, band_bias: float, band_width: int, qbs=None):
    """Round selection on one sequence at the watershed layer (Qw, Kw), then
    every layer of `layers` [(Q, K, V)] through its own probabilities on the
    selected blocks.  Returns {qb: {"rounds": kept rounds of qb's round,
    "kept": kept blocks, "O": [O of each layer]}}.
    """
    L = Qw.shape[0]
    nqb = (L + B - 1) // B
    kept_r = {}
    out = {}
    for qb in (range(nqb) if qbs is None else qbs):
        q = round_of_token(round_starts, qb * B)
        if q not in kept_r:
            kept_r[q] = select_rounds(
                round_mass(Qw, Kw, round_starts, q, band_bias, band_width), tau)
        kept = round_kept_blocks(kept_r[q], round_starts, qb, B)
        Os = []
        for Q, K, V in layers:
            _, P, _ = query_block(Q, K, qb, B, band_bias, band_width)
            Os.append(mapped_av(mixed_map(P, kept, W, B), V, Hkv))
        out[qb] = {"rounds": kept_r[q], "kept": kept, "O": Os}
    return out
