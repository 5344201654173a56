"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test fixes one part of the path (MapFlow article, 163.com, section on the
three system components: block compression by cumulative attention mass,
linear head mixing, multiplication into the receiver's V) by an invariant, a
closed form, brute force, or a library routine (torch's scaled-dot-product
attention, scipy's logsumexp) run in float64 on the CPU.
"""
import itertools
import math
from fractions import Fraction

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

from oracle import mapflow_oracle as orc

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _rand_qk(L, Hs, d, seed, scale=1.5):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((L, Hs, d)) * scale
    K = rng.standard_normal((L, Hs, d)) * scale
    K[:2] += 2.0  # a sink-like skew, so masses are far from uniform
    return Q, K


def _band_mask(L, beta, width):
    i = torch.arange(L)[:, None]
    j = torch.arange(L)[None, :]
    delta = i - j
    m = torch.where(delta >= 0, torch.zeros(L, L, dtype=torch.float64),
                    torch.full((L, L), float("-inf"), dtype=torch.float64))
    return m + beta * ((delta >= 0) & (delta < width)).to(torch.float64)


def _sdpa(q, k, v, mask):
    """torch SDPA, fp64 CPU; q,k: [L, d], v: [L, dv]."""
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None], torch.from_numpy(k)[None, None],
        torch.from_numpy(v)[None, None], attn_mask=mask)[0, 0].numpy()


# ----------------------------------------------------------------- softmax / lse

def test_rows_sum_to_one():
    Q, K = _rand_qk(37, 3, 16, 0)
    s = orc.scores(Q, K, 0, 37, 2.0, 5)
    _, P = orc.lse_and_probs(s)
    np.testing.assert_allclose(P.sum(axis=2), 1.0, rtol=0, atol=1e-13)
    # causal: nothing above the diagonal
    iu = np.triu_indices(37, 1)
    assert np.all(P[:, iu[0], iu[1]] == 0.0)


def test_lse_matches_scipy_logsumexp():
    Q, K = _rand_qk(29, 2, 8, 1)
    s = orc.scores(Q, K, 0, 29, 1.0, 4)
    lse, _ = orc.lse_and_probs(s)
    ref = logsumexp(s, axis=2)
    np.testing.assert_allclose(lse, ref, rtol=1e-13, atol=1e-13)


# ------------------------------------------------- tau = 1: the dense attention

@pytest.mark.parametrize("beta,width", [(0.0, 256), (2.0, 6)])
def test_tau1_identity_map_is_causal_attention(beta, width):
    """Hr = Hs = Hkv, W = I, tau = 1: O_h = softmax(QK^T/sqrt(d) + bias) V_h."""
    L, H, d, B = 45, 3, 16, 8
    Q, K = _rand_qk(L, H, d, 2)
    V = np.random.default_rng(3).standard_normal((L, H, d))
    W = np.eye(H)
    _, O = orc.run_layer(Q, K, V, W, [L], Hkv=H, B=B, tau=1.0,
                         band_bias=beta, band_width=width)
    mask = _band_mask(L, beta, width)
    for h in range(H):
        ref = _sdpa(Q[:, h], K[:, h], V[:, h], mask)
        np.testing.assert_allclose(O[:, h], ref, rtol=1e-11, atol=1e-11)


def test_tau1_mixed_gqa_map():
    """O_r = sum_h W[r,h] softmax_h V_{g(r)}, g from torch's repeat_interleave."""
    L, Hs, Hr, Hkv, d, B = 40, 3, 4, 2, 8, 8
    Q, K = _rand_qk(L, Hs, d, 4)
    rng = np.random.default_rng(5)
    V = rng.standard_normal((L, Hkv, d))
    W = rng.standard_normal((Hr, Hs))
    _, O = orc.run_layer(Q, K, V, W, [L], Hkv=Hkv, B=B, tau=1.0,
                         band_bias=1.5, band_width=7)
    Vr = torch.repeat_interleave(torch.from_numpy(V), Hr // Hkv, dim=1).numpy()
    mask = _band_mask(L, 1.5, 7)
    for r in range(Hr):
        ref = sum(W[r, h] * _sdpa(Q[:, h], K[:, h], Vr[:, r], mask) for h in range(Hs))
        np.testing.assert_allclose(O[:, r], ref, rtol=1e-11, atol=1e-11)


def test_tau_below_one_drops_blocks_without_renormalising():
    """Rows of qb see only kept key blocks, with the full-softmax weights."""
    L, Hs, Hr, Hkv, d, B = 48, 2, 2, 1, 8, 8
    Q, K = _rand_qk(L, Hs, d, 6)
    rng = np.random.default_rng(7)
    V = rng.standard_normal((L, Hkv, d))
    W = rng.standard_normal((Hr, Hs))
    res, O = orc.run_layer(Q, K, V, W, [L], Hkv=Hkv, B=B, tau=0.7,
                           band_bias=0.0, band_width=256)
    mask = _band_mask(L, 0.0, 256)
    dropped_any = False
    for qb, rec in res[0].items():
        keep = np.zeros(L, dtype=bool)
        for kb in rec["kept"]:
            keep[kb * B:(kb + 1) * B] = True
        dropped_any |= len(rec["kept"]) < qb + 1
        Vm = np.where(keep[:, None], V[:, 0], 0.0)
        rows = slice(qb * B, min(L, (qb + 1) * B))
        for r in range(Hr):
            ref = sum(W[r, h] * _sdpa(Q[:, h], K[:, h], Vm, mask) for h in range(Hs))
            np.testing.assert_allclose(O[rows, r], ref[rows], rtol=1e-11, atol=1e-11)
    assert dropped_any


# ------------------------------------------------------- block mass closed forms

def _q0_mass_exact(L, B, Hs, width=None, ebeta=None):
    """Exact block masses for Q = 0 (all logits equal except the band bias).

    Without bias P[i,j] = 1/(i+1).  With bias factor e^beta on the band
    0 <= i-j < width: P[i,j] = w_ij / Z_i, Z_i = sum_j w_ij.
    """
    nqb = (L + B - 1) // B
    out = {}
    for qb in range(nqb):
        m = []
        for kb in range(qb + 1):
            tot = Fraction(0) if ebeta is None else 0.0
            for i in range(qb * B, min(L, (qb + 1) * B)):
                js = range(kb * B, min(i + 1, (kb + 1) * B))
                if ebeta is None:
                    tot += Fraction(len(js), i + 1)
                else:
                    nb = min(i + 1, width)
                    Z = nb * ebeta + (i + 1 - nb)
                    tot += sum((ebeta if i - j < width else 1.0) for j in js) / Z
            m.append(Hs * (float(tot) if ebeta is None else tot))
        out[qb] = np.array(m)
    return out


def test_block_mass_q0_harmonic_closed_form():
    L, Hs, d, B = 30, 2, 4, 4
    Q = np.zeros((L, Hs, d))
    K = np.random.default_rng(8).standard_normal((L, Hs, d))
    exact = _q0_mass_exact(L, B, Hs)
    for qb in range(len(exact)):
        _, _, mass = orc.query_block(Q, K, qb, B, 0.0, 256)
        np.testing.assert_allclose(mass, exact[qb], rtol=1e-14, atol=1e-14)


def test_block_mass_q0_band_closed_form():
    """Pins the band edge: bias on 0 <= i - j < width, not on i - j == width."""
    L, Hs, d, B, beta, width = 26, 1, 4, 4, 2.0, 5
    Q = np.zeros((L, Hs, d))
    K = np.random.default_rng(9).standard_normal((L, Hs, d))
    exact = _q0_mass_exact(L, B, Hs, width=width, ebeta=math.exp(beta))
    for qb in range(len(exact)):
        _, _, mass = orc.query_block(Q, K, qb, B, beta, width)
        np.testing.assert_allclose(mass, exact[qb], rtol=1e-13, atol=1e-14)


def test_block_mass_totals_rows_times_heads():
    L, Hs, d, B = 50, 3, 8, 16
    Q, K = _rand_qk(L, Hs, d, 10)
    for qb in range(4):
        _, _, mass = orc.query_block(Q, K, qb, B, 2.0, 9)
        rows = min(L, (qb + 1) * B) - qb * B
        assert mass.shape == (qb + 1,)
        assert abs(mass.sum() - Hs * rows) < 1e-11


# ------------------------------------------------------------------- selection

def _brute_force(mass, tau):
    n = len(mass)
    T = sum(mass)
    for k in range(1, n + 1):
        best = None
        for sub in itertools.combinations(range(n), k):
            sm = sum(mass[i] for i in sub)
            if sm >= tau * T:
                key = (-sm, sub)
                if best is None or key < best:
                    best = key
        if best is not None:
            return k, best[1]
    return n, tuple(range(n))


@pytest.mark.parametrize("seed", range(12))
def test_selection_matches_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    n = int(rng.integers(1, 10))
    mass = rng.exponential(size=n) ** 2
    tau = float(rng.uniform(0.3, 0.99))
    kept = orc.select_blocks(mass, tau)
    kmin, _ = _brute_force(list(mass), tau)
    assert len(kept) == kmin
    # among minimal sets, the kept one has the largest mass (distinct masses)
    best = max(itertools.combinations(range(n), kmin), key=lambda s: sum(mass[i] for i in s))
    assert tuple(kept) == tuple(sorted(best))


def test_selection_threshold_is_inclusive():
    """c_k equal to tau * T stops the scan (>=, not >)."""
    kept = orc.select_blocks(np.array([1.0, 1.0, 1.0, 1.0]), 0.5)
    assert list(kept) == [0, 1]


def test_selection_ties_go_to_lower_index():
    """Q = 0: every fully past block has the same mass; the lower ones win."""
    L, Hs, d, B = 64, 1, 4, 8
    Q = np.zeros((L, Hs, d))
    K = np.random.default_rng(11).standard_normal((L, Hs, d))
    _, _, mass = orc.query_block(Q, K, 7, B, 0.0, 256)
    # blocks 0..6 are fully past and tie exactly in exact arithmetic
    assert np.ptp(mass[:7]) < 1e-15
    kept = orc.select_blocks(mass, 0.5)
    full = [kb for kb in kept if kb < 7]
    assert full == list(range(len(full)))
    assert 0 < len(full) < 7


def test_tau_one_keeps_every_causal_block():
    Q, K = _rand_qk(40, 2, 8, 12)
    for qb in range(5):
        _, _, mass = orc.query_block(Q, K, qb, 8, 2.0, 9)
        assert list(orc.select_blocks(mass, 1.0)) == list(range(qb + 1))


# ------------------------------------------------------------------ structure

def test_linear_in_w_and_v():
    L, Hs, Hr, Hkv, d, B = 33, 2, 2, 1, 8, 8
    Q, K = _rand_qk(L, Hs, d, 13)
    rng = np.random.default_rng(14)
    V1, V2 = rng.standard_normal((2, L, Hkv, d))
    W1, W2 = rng.standard_normal((2, Hr, Hs))
    run = lambda V, W: orc.run_layer(Q, K, V, W, [L], Hkv, B, 0.8, 2.0, 6)[1]
    np.testing.assert_allclose(run(V1, 2 * W1 - 3 * W2),
                               2 * run(V1, W1) - 3 * run(V1, W2), atol=1e-11)
    np.testing.assert_allclose(run(V1 + V2, W1), run(V1, W1) + run(V2, W1), atol=1e-11)


def test_varlen_packing_equals_per_sequence_runs():
    lens = [19, 8, 27]
    Hs, Hr, Hkv, d, B = 2, 2, 2, 8, 8
    rng = np.random.default_rng(15)
    n = sum(lens)
    Q, K = rng.standard_normal((2, n, Hs, d))
    V = rng.standard_normal((n, Hkv, d))
    W = rng.standard_normal((Hr, Hs))
    _, O = orc.run_layer(Q, K, V, W, lens, Hkv, B, 0.85, 1.0, 5)
    s = 0
    for L in lens:
        _, Os = orc.run_layer(Q[s:s + L], K[s:s + L], V[s:s + L], W, [L], Hkv, B, 0.85, 1.0, 5)
        np.testing.assert_array_equal(O[s:s + L], Os)
        s += L


def test_extracted_blocks_are_the_probabilities():
    L, Hs, d, B = 21, 2, 8, 8
    Q, K = _rand_qk(L, Hs, d, 16)
    V = np.zeros((L, 1, d))
    W = np.ones((1, Hs))
    res = orc.run_sequence(Q, K, V, W, 1, B, 0.9, 2.0, 6, want_values=True)
    for qb, rec in res.items():
        _, P = orc.lse_and_probs(orc.scores(Q, K, qb * B, min(L, (qb + 1) * B), 2.0, 6))
        for kb, blk in rec["values"].items():
            hi = min(P.shape[2], (kb + 1) * B)
            np.testing.assert_array_equal(blk[:, :, :hi - kb * B], P[:, :, kb * B:hi])
            if kb == qb:  # upper triangle of the diagonal block is zero
                for i in range(blk.shape[1]):
                    assert np.all(blk[:, i, i + 1:] == 0.0)


# ------------------------------------------- cumulative fractions (exemptions)

def _check_cumulative_fractions(fn, mass, tau):
    """What the selection rule fixes about (order, c_k / T), independent of the
    oracle: the order is numpy's lexicographic sort by (-mass, index); the
    fractions are the running sums in that order over the plain total; and the
    cut of select_blocks sits where the fraction first reaches tau."""
    order, frac = fn(mass)
    n = len(mass)
    ref_order = np.lexsort((np.arange(n), -mass))          # last key is primary
    assert list(order) == list(ref_order), "order is not (mass desc, index asc)"
    total = math.fsum(mass)
    run = 0.0
    for k, kb in enumerate(ref_order):
        run += mass[kb]
        assert abs(frac[k] - run / total) <= 1e-12, f"fraction {k} is not c_k / T"
    assert abs(frac[-1] - 1.0) <= 1e-12
    kept = orc.select_blocks(mass, tau)
    k = len(kept)
    assert set(kept.tolist()) == set(order[:k].tolist())
    if tau < 1.0:
        assert frac[k - 1] >= tau - 1e-12
        assert k == 1 or frac[k - 2] < tau


def _mass_cases():
    rng = np.random.default_rng(300)
    cases = []
    for _ in range(8):
        n = int(rng.integers(2, 40))
        cases.append((rng.exponential(size=n) ** 2, float(rng.uniform(0.3, 0.99))))
    # exact ties: Q = 0 block masses (blocks fully in the past tie)
    Q = np.zeros((64, 1, 4))
    K = np.random.default_rng(11).standard_normal((64, 1, 4))
    _, _, mass = orc.query_block(Q, K, 7, 8, 0.0, 256)
    cases.append((mass, 0.5))
    cases.append((np.array([3.0, 1.0, 3.0, 2.0, 1.0]), 0.6))
    return cases


def test_cumulative_fractions_order_and_cut():
    for mass, tau in _mass_cases():
        _check_cumulative_fractions(orc.cumulative_fractions, mass, tau)


def _mutant_ascending(mass):
    order = sorted(range(len(mass)), key=lambda kb: (mass[kb], kb))
    c = np.cumsum(np.array([mass[kb] for kb in order]))
    return np.array(order), c / c[-1]


def _mutant_ties_high(mass):
    order = sorted(range(len(mass)), key=lambda kb: (-mass[kb], -kb))
    c = np.cumsum(np.array([mass[kb] for kb in order]))
    return np.array(order), c / c[-1]


def _mutant_shifted(mass):
    order, frac = orc.cumulative_fractions(mass)
    return order, np.concatenate([[0.0], frac[:-1]])       # c_{k-1} in place of c_k


def _mutant_wrong_total(mass):
    order, frac = orc.cumulative_fractions(mass)
    return order, frac * (1.0 - 1.0 / len(mass))           # divided by a larger total


@pytest.mark.parametrize("mutant", [_mutant_ascending, _mutant_ties_high, _mutant_shifted,
                                    _mutant_wrong_total])
def test_cumulative_fraction_pins_catch_planted_mistakes(mutant):
    """Each plausible mistake planted in a copy of the oracle function fails
    the checks above on at least one of the cases."""
    failed = False
    for mass, tau in _mass_cases():
        try:
            _check_cumulative_fractions(mutant, mass, tau)
        except AssertionError:
            failed = True
            break
    assert failed
