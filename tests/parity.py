"""Helpers that compare the CUDA path (through the C ABI) with the CPU oracle.

Tolerances (from the stated acceptance rule of the hot path):
* kept block sets bit-exact, except query blocks whose oracle cumulative mass
  fraction at the cut lies within 1e-4 of tau ("near tau"), or whose only
  difference swaps blocks across the cut whose oracle masses all lie within
  1e-6 * T of the oracle's mass at the cut ("near swap"); both kinds are
  counted, reported separately at the end of the pytest run, and the exempt
  query block is still checked: its extracted values and its O against the
  oracle evaluated on the GPU's own kept set;
* O: max-abs error <= 2e-2 * max|O| for bf16, <= 1e-4 * max|O| for fp32;
* lse, block masses and extracted probabilities: the float32 arithmetic of
  the kernels on identical (rounded) inputs; bounds are stated per check.
"""
from __future__ import annotations

import numpy as np
import torch

from cross_model_attention_block_b200 import mapflow as mfb
from oracle import mapflow_oracle as orc

NEAR_TAU = 1e-4
NEAR_SWAP = 1e-6


def o_tol(dtype):
    return 1e-4 if dtype == torch.float32 else 2e-2


def run_gpu(ctx, Q, K, V, W, Hkv, tau, page_table=None, page_size=16, Vpool=None):
    """The whole path through the C ABI; returns (lse, mass, cache, O)."""
    lse, mass = mfb.block_stats(ctx, Q, K)
    cache = mfb.select_extract(ctx, Q, K, lse, mass, tau)
    if page_table is None:
        O = mfb.mapped_av(cache, W.shape[0], W, V, Hkv)
    else:
        O = mfb.mapped_av(cache, W.shape[0], W, Vpool, Hkv, page_table=page_table,
                          page_size=page_size)
    mfb.sync_status()
    return lse, mass, cache, O


def kept_sets(cache):
    rp = cache.row_ptr.cpu().numpy()
    ci = cache.col_idx.cpu().numpy()
    return rp, ci


# Exemptions seen during this process, per label: {label: [checked, near_tau, near_swap]}.
REPORT = {}


def record(label, res):
    """Add one comparison's counts to the run's exemption report."""
    r = REPORT.setdefault(label, [0, 0, 0])
    r[0] += res.n
    r[1] += res.near_tau
    r[2] += res.near_swap


def check_selection(oracle_mass, gpu_kept, tau):
    """'' if the kept sets are equal, 'near_tau' or 'near_swap' if the
    difference is exempt; raises otherwise."""
    oracle_kept = orc.select_blocks(oracle_mass, tau)
    if list(oracle_kept) == list(gpu_kept):
        return ""
    order, frac = orc.cumulative_fractions(oracle_mass)
    k = len(oracle_kept)
    near = [abs(frac[k - 1] - tau)]
    if k >= 2:
        near.append(abs(frac[k - 2] - tau))
    if min(near) < NEAR_TAU:
        return "near_tau"
    T = oracle_mass.sum()
    a, b = set(oracle_kept.tolist()), set(int(x) for x in gpu_kept)
    if len(a) == len(b):
        # swaps across the cut: oracle-kept blocks the GPU dropped, and
        # blocks past the cut it kept, all as heavy as the cut block
        m_cut = oracle_mass[order[k - 1]]
        diff = sorted(a ^ b)
        if max(abs(oracle_mass[kb] - m_cut) for kb in diff) < NEAR_SWAP * T:
            return "near_swap"
    raise AssertionError(f"kept sets differ beyond the exemptions: oracle {sorted(a)} "
                         f"gpu {sorted(b)}; cut fractions {near}")


class Result(tuple):
    """(n, exempt, worst) with the exemption kinds by name."""

    def __new__(cls, n, near_tau, near_swap, worst):
        r = super().__new__(cls, (n, near_tau + near_swap, worst))
        r.n, r.near_tau, r.near_swap, r.worst = n, near_tau, near_swap, worst
        return r


def f64(t):
    return t.detach().to(torch.float64).cpu().numpy()


def block_index(cu_blk_s, qb, kb):
    return cu_blk_s + qb * (qb + 1) // 2 + kb


def compare_query_blocks(ctx, Qc, Kc, Vc, Wc, Hkv, tau, gpu, picks, dtype,
                         check_values=True, lse_atol=None, label=None):
    """Compare the GPU result on selected (seq, qb) pairs with the oracle.

    Qc, Kc, Vc, Wc are the CPU copies of the inputs (contiguous V).  The
    extracted values and O are compared on the GPU's kept set, which equals
    the oracle's except on counted exemptions.  Returns a Result
    (n_checked, n_exempt, max_rel_err_O) and, with a label, adds its counts
    to the run's exemption report.
    """
    lse_g, mass_g, cache, O_g = gpu
    B = ctx.B
    cu = ctx.cu_seqlens_host
    lens = np.diff(cu)
    nqb = (lens + B - 1) // B
    cu_qb = np.concatenate([[0], np.cumsum(nqb)])
    cu_blk = np.concatenate([[0], np.cumsum(nqb * (nqb + 1) // 2)])
    rp, ci = kept_sets(cache)
    lse_g = lse_g.cpu().numpy()
    mass_g = mass_g.cpu().numpy()
    W = f64(Wc)
    vals = cache.values_view() if check_values else None
    n_tau = n_swap = 0
    worst = 0.0
    tol = o_tol(dtype)
    if lse_atol is None:
        lse_atol = 2e-5 if dtype == torch.float32 else 1e-4
    for s, qb in picks:
        s0, L = int(cu[s]), int(lens[s])
        i0, i1 = qb * B, min(L, (qb + 1) * B)
        Qs = f64(Qc[s0:s0 + i1])
        Ks = f64(Kc[s0:s0 + i1])
        Vs = f64(Vc[s0:s0 + i1])
        lse_o, P, mass_o = orc.query_block(Qs, Ks, qb, B, ctx.band_bias, ctx.band_width)
        # lse
        np.testing.assert_allclose(lse_g[:, s0 + i0:s0 + i1], lse_o, rtol=0, atol=lse_atol,
                                   err_msg=f"lse seq {s} qb {qb}")
        # block masses (float32 sums of float32 terms)
        b0 = block_index(cu_blk[s], qb, 0)
        T = mass_o.sum()
        np.testing.assert_allclose(mass_g[b0:b0 + qb + 1], mass_o, rtol=0, atol=2e-5 * T,
                                   err_msg=f"mass seq {s} qb {qb}")
        # selection
        g = int(cu_qb[s] + qb)
        kept_g = ci[rp[g]:rp[g + 1]]
        assert np.all(np.diff(kept_g) > 0), "kept blocks not ascending"
        ex = check_selection(mass_o, kept_g, tau)
        n_tau += ex == "near_tau"
        n_swap += ex == "near_swap"
        # extracted probability blocks
        if check_values:
            for e, kb in zip(range(rp[g], rp[g + 1]), kept_g):
                got = stored_to_logical(f64(vals[e]), ctx.Hs, B)  # [Hs, B rows, B keys]
                ref = np.zeros((P.shape[0], B, B))
                hi = min(P.shape[2], (kb + 1) * B)
                ref[:, : i1 - i0, : hi - kb * B] = P[:, :, kb * B:hi]
                if dtype == torch.float32:
                    np.testing.assert_allclose(got, ref, rtol=2e-5, atol=1e-7)
                else:
                    np.testing.assert_allclose(got, ref, rtol=2 ** -8, atol=1e-6)
        # output rows
        M = orc.mixed_map(P, np.array(kept_g), W, B)
        O_o = orc.mapped_av(M, Vs, Hkv)
        O_gpu = f64(O_g[s0 + i0:s0 + i1])
        scale = max(np.abs(O_o).max(), 1e-30)
        err = np.abs(O_gpu - O_o).max() / scale
        worst = max(worst, err)
        assert err <= tol, f"O seq {s} qb {qb}: rel err {err:.3e} > {tol}"
    res = Result(len(picks), n_tau, n_swap, worst)
    if label is not None:
        record(label, res)
    return res


def stored_to_logical(x, Hs, B):
    """One cache entry, stored [B/16 kg][B/8 slice][2 half][Hs][8 chunk][8] ->
    logical [Hs][B rows][B keys] (see the C header)."""
    S16, S8 = B // 16, B // 8
    x = x.reshape(S16, S8, 2, Hs, 8, 8)
    out = np.empty((Hs, B, B), dtype=x.dtype)
    for h in range(Hs):
        perm = np.arange(8) ^ (h & 7)                 # logical chunk -> stored chunk
        ch = x[:, :, :, h][:, :, :, perm]             # [kg, slice, half, chunk, 8]
        ch = ch.reshape(S16, S8, 2, 4, 2, 8)          # chunk = (row % 4, 8-key half)
        out[h] = ch.transpose(1, 2, 3, 0, 4, 5).reshape(B, B)
    return out


def logical_to_stored(y, Hs, B):
    """One cache entry, logical [Hs][B][B] -> stored [B/16][B/8][2][Hs][8][8]."""
    S16, S8 = B // 16, B // 8
    out = np.empty((S16, S8, 2, Hs, 8, 8), dtype=y.dtype)
    for h in range(Hs):
        perm = np.arange(8) ^ (h & 7)
        blk = y[h].reshape(S8, 2, 4, S16, 2, 8).transpose(3, 0, 1, 2, 4, 5)
        blk = blk.reshape(S16, S8, 2, 8, 8)           # [kg, slice, half, chunk, 8]
        out[:, :, :, h][:, :, :, perm] = blk
    return out


def all_picks(ctx):
    cu = ctx.cu_seqlens_host
    B = ctx.B
    return [(s, qb) for s in range(len(cu) - 1)
            for qb in range((int(cu[s + 1] - cu[s]) + B - 1) // B)]
