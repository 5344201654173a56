"""Pins of the oracle's round-level selection (the Round Attention page,
"方法详解": per conversation round, a watershed layer's attention keeps the
most relevant earlier rounds) against facts that do not come from the oracle:
brute force over subsets, exact fractions for Q = 0, the row-sum invariant,
the block masses (a second route to the same sums), reduction to the block
selection, and torch's scaled-dot-product attention in float64 with the
dropped rounds' V zeroed."""
import itertools
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import mapflow_oracle as orc

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _qk(L, Hs, d, seed):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((L, Hs, d)) * 1.5
    K = rng.standard_normal((L, Hs, d)) * 1.5
    K[:2] += 2.0
    return Q, K


STARTS = [0, 16, 24, 48, 56, 72]   # five rounds of 2, 1, 3, 1, 2 blocks (B = 8), L = 72


def test_round_mass_rows_sum_to_heads_times_rows():
    Q, K = _qk(72, 3, 8, 1)
    for q in range(5):
        m = orc.round_mass(Q, K, STARTS, q, 2.0, 9)
        rows = STARTS[q + 1] - STARTS[q]
        assert m.shape == (q + 1,)
        assert abs(m.sum() - 3 * rows) < 1e-11


def test_round_mass_q0_exact_fractions():
    """Q = 0 without bias: P[i, j] = 1/(i+1) for j <= i."""
    L, Hs = 72, 2
    Q = np.zeros((L, Hs, 4))
    K = np.random.default_rng(2).standard_normal((L, Hs, 4))
    for q in range(5):
        m = orc.round_mass(Q, K, STARTS, q, 0.0, 256)
        for r in range(q + 1):
            exact = Fraction(0)
            for i in range(STARTS[q], STARTS[q + 1]):
                n = len(range(STARTS[r], min(STARTS[r + 1], i + 1)))
                exact += Fraction(n, i + 1)
            assert abs(m[r] - Hs * float(exact)) < 1e-13


def test_round_mass_equals_summed_block_masses():
    """Rounds on block boundaries: the round mass is the sum of the block
    masses of its query blocks over its key blocks."""
    B = 8
    Q, K = _qk(72, 2, 8, 3)
    blk = {qb: orc.query_block(Q, K, qb, B, 2.0, 9)[2] for qb in range(9)}
    for q in range(5):
        m = orc.round_mass(Q, K, STARTS, q, 2.0, 9)
        for r in range(q + 1):
            tot = sum(blk[qb][kb]
                      for qb in range(STARTS[q] // B, STARTS[q + 1] // B)
                      for kb in range(STARTS[r] // B, STARTS[r + 1] // B) if kb <= qb)
            assert abs(m[r] - tot) < 1e-11


def _brute(m, tau):
    """Fewest earlier rounds that, with the own round, reach tau * T."""
    q = len(m) - 1
    T = sum(m)
    for k in range(q + 1):
        best = None
        for sub in itertools.combinations(range(q), k):
            tot = m[q] + sum(m[r] for r in sub)
            if tot >= tau * T and (best is None or tot > best[0]):
                best = (tot, sub)
        if best is not None:
            return sorted(best[1]) + [q]
    return list(range(q + 1))


@pytest.mark.parametrize("seed", range(12))
def test_select_rounds_matches_brute_force(seed):
    rng = np.random.default_rng(400 + seed)
    q = int(rng.integers(0, 8))
    m = rng.exponential(size=q + 1) ** 2
    tau = float(rng.uniform(0.2, 0.99))
    assert list(orc.select_rounds(m, tau)) == _brute(list(m), tau)


def test_select_rounds_own_round_always_ties_low_and_inclusive():
    m = np.array([1.0, 1.0, 1.0, 1.0, 0.5])          # own round is the lightest
    assert list(orc.select_rounds(m, 0.01)) == [4]   # own round alone may suffice
    assert list(orc.select_rounds(m, 0.5)) == [0, 1, 4]   # ties to the lower rounds
    T = m.sum()
    assert list(orc.select_rounds(m, (0.5 + 1.0) / T)) == [0, 4]  # >= stops the scan
    assert list(orc.select_rounds(m, 1.0)) == [0, 1, 2, 3, 4]


def test_single_block_rounds_reduce_to_block_selection():
    """Rounds of one block each and a query block whose own (diagonal) block
    is the heaviest: the round rule is the block rule."""
    B, L = 8, 72
    Q, K = _qk(L, 2, 8, 5)
    starts = list(range(0, L + 1, B))
    checked = 0
    for qb in range(9):
        _, _, mass = orc.query_block(Q, K, qb, B, 3.0, 8)
        if np.argmax(mass) != qb:
            continue
        m = orc.round_mass(Q, K, starts, qb, 3.0, 8)
        for tau in (0.5, 0.8, 0.95):
            assert list(orc.select_rounds(m, tau)) == list(orc.select_blocks(mass, tau))
        checked += 1
    assert checked >= 5


def _sdpa(q, k, v, mask):
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None], torch.from_numpy(k)[None, None],
        torch.from_numpy(v)[None, None], attn_mask=mask)[0, 0].numpy()


def test_dropped_rounds_are_zeroed_v_without_renormalising():
    """The rows of a query round see exactly the kept rounds with full-softmax
    weights: O equals sum_h W[r,h] SDPA with the dropped rounds' V zeroed."""
    B, L, Hs, Hr, Hkv, d = 8, 72, 2, 2, 1, 8
    Q, K = _qk(L, Hs, d, 6)
    rng = np.random.default_rng(7)
    V = rng.standard_normal((L, Hkv, d))
    W = rng.standard_normal((Hr, Hs))
    beta, width = 0.0, 256
    res = orc.run_rounds_sequence(Q, K, [(Q, K, V)], W, Hkv, B, 0.6, STARTS, beta, width)
    i = torch.arange(L)[:, None]
    j = torch.arange(L)[None, :]
    mask = torch.where(i >= j, 0.0, float("-inf")).to(torch.float64)
    dropped_any = False
    for qb, rec in res.items():
        q = orc.round_of_token(STARTS, qb * B)
        keep = np.zeros(L, dtype=bool)
        for r in rec["rounds"]:
            keep[STARTS[r]:STARTS[r + 1]] = True
        dropped_any |= len(rec["rounds"]) < q + 1
        Vm = np.where(keep[:, None], V[:, 0], 0.0)
        rows = slice(qb * B, (qb + 1) * B)
        for r in range(Hr):
            ref = sum(W[r, h] * _sdpa(Q[:, h], K[:, h], Vm, mask) for h in range(Hs))
            np.testing.assert_allclose(rec["O"][0][:, r], ref[rows], rtol=1e-11, atol=1e-11)
    assert dropped_any


def test_later_layers_use_the_watershed_selection():
    """The kept blocks come from the watershed layer only; a later layer's O
    is its own probabilities on those blocks."""
    B, L = 8, 72
    Qw, Kw = _qk(L, 2, 8, 8)
    Q2, K2 = _qk(L, 2, 8, 9)
    V = np.random.default_rng(10).standard_normal((L, 1, 8))
    W = np.ones((1, 2))
    res = orc.run_rounds_sequence(Qw, Kw, [(Q2, K2, V)], W, 1, B, 0.7, STARTS, 1.0, 9)
    for qb, rec in res.items():
        q = orc.round_of_token(STARTS, qb * B)
        m = orc.round_mass(Qw, Kw, STARTS, q, 1.0, 9)
        assert list(rec["rounds"]) == list(orc.select_rounds(m, 0.7))
        _, P, _ = orc.query_block(Q2, K2, qb, B, 1.0, 9)
        ref = orc.mapped_av(orc.mixed_map(P, rec["kept"], W, B), V, 1)
        np.testing.assert_array_equal(rec["O"][0], ref)


def _mutant_no_own(m, tau):
    """The own round competes like any other instead of being kept."""
    return orc.select_blocks(m, tau) if tau < 1 else np.arange(len(m))


def _mutant_ties_high(m, tau):
    q = len(m) - 1
    T = float(np.sum(m))
    order = sorted(range(q), key=lambda r: (-m[r], -r))
    c, k = float(m[q]), 0
    while c < tau * T and k < q:
        c += float(m[order[k]])
        k += 1
    return np.array(sorted(order[:k] + [q]))


def _mutant_strict(m, tau):
    q = len(m) - 1
    T = float(np.sum(m))
    order = sorted(range(q), key=lambda r: (-m[r], r))
    c, k = float(m[q]), 0
    while c <= tau * T and k < q:
        c += float(m[order[k]])
        k += 1
    return np.array(sorted(order[:k] + [q]))


@pytest.mark.parametrize("mutant", [_mutant_no_own, _mutant_ties_high, _mutant_strict])
def test_round_pins_catch_planted_mistakes(mutant):
    m = np.array([1.0, 1.0, 1.0, 1.0, 0.5])
    cases = [(m, 0.01), (m, 0.5), (m, (0.5 + 1.0) / m.sum())]
    rng = np.random.default_rng(500)
    for _ in range(12):
        mm = rng.exponential(size=int(rng.integers(2, 8))) ** 2
        cases.append((mm, float(rng.uniform(0.2, 0.99))))
    bad = any(list(mutant(mm, t)) != _brute(list(mm), t) for mm, t in cases)
    assert bad
