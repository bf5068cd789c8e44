"""The level-by-level form the backward kernels use is exact (CPU, fp64, no GPU).

The hierarchical mask M_H (Log-Linear Attention, section 2, "Matrici Gerarchiche") couples, at
each level l >= 1, the left and right halves of aligned blocks of 2^l positions, and nothing
else; within a half-block pair the gate factors through the left half's last position m.  The
backward therefore splits into:
  * levels 0..5: causal pairs inside aligned 32-position tiles (done densely);
  * levels >= 6: per block, S = sum_left e^{g_m - g_s} k_s v_s^T and
    U = sum_right lam[t,l] e^{g_t - g_m} q_t do_t^T, applied to the other half;
  * dlog_a from dg_t = q_t . dq_t - k_t . dk_t, summed from the right.
This test rebuilds all five gradients that way in numpy, with code of its own, and compares
them with the oracle's product-by-product differentiation; it also checks that the two parts
partition the causal pairs exactly (every pair in exactly one of them, at its own level).
"""
import numpy as np
import pytest

import oracle as O
from hierarchical_fenwick_state_b200 import inputs as I

TILE, DENSE = 32, 6


def _level(t, s):
    return 0 if t == s else int(t ^ s).bit_length()


def level_form_backward(q, k, v, log_a, lam, do):
    q, k, v, do = (np.asarray(x, np.float64) for x in (q, k, v, do))
    lam = np.asarray(lam, np.float64)
    T, L = lam.shape
    g = np.cumsum(np.asarray(log_a, np.float64))
    dq = np.zeros_like(q); dk = np.zeros_like(k); dv = np.zeros_like(v)
    dlam = np.zeros((T, L))
    # levels 0..5: dense aligned tiles
    for t0 in range(0, T, TILE):
        idx = np.arange(t0, min(T, t0 + TILE))
        A = q[idx] @ k[idx].T
        Bm = do[idx] @ v[idx].T
        E = np.exp(g[idx][:, None] - g[idx][None, :])
        lev = np.array([[_level(i, j) for j in idx] for i in idx])
        causal = idx[None, :] <= idx[:, None]
        M = np.where(causal, np.take_along_axis(lam[idx], np.where(causal, lev, 0), 1) * E, 0.0)
        dq[idx] += (Bm * M) @ k[idx]
        dk[idx] += (Bm * M).T @ q[idx]
        dv[idx] += (A * M).T @ do[idx]
        X = np.where(causal, A * Bm * E, 0.0)
        for lvl in range(min(DENSE, L)):
            dlam[idx, lvl] = np.sum(np.where(lev == lvl, X, 0.0), axis=1)
    # levels >= 6: rank-d interaction of each aligned block's halves
    for lvl in range(DENSE, L):
        half = 1 << (lvl - 1)
        for lo in range(0, T, 2 * half):
            left = np.arange(lo, min(lo + half, T))
            right = np.arange(lo + half, min(lo + 2 * half, T))
            if right.size == 0:
                continue
            m = lo + half - 1
            wl = np.exp(g[m] - g[left])
            wr = lam[right, lvl] * np.exp(g[right] - g[m])
            S = (k[left] * wl[:, None]).T @ v[left]
            U = (q[right] * wr[:, None]).T @ do[right]
            w = (do[right] @ S.T) * np.exp(g[right] - g[m])[:, None]
            dlam[right, lvl] = np.sum(q[right] * w, axis=1)
            dq[right] += lam[right, lvl][:, None] * w
            dk[left] += wl[:, None] * (v[left] @ U.T)
            dv[left] += wl[:, None] * (k[left] @ U)
    dg = np.sum(q * dq, axis=1) - np.sum(k * dk, axis=1)
    dlog_a = np.cumsum(dg[::-1])[::-1]
    return dq, dk, dv, dlog_a, dlam


@pytest.mark.parametrize("T", [1, 31, 32, 33, 64, 100, 257, 700])
def test_level_form_equals_the_oracle(T):
    w = I.Workload("lf", B=1, H=1, T=T, dk=5, dv=4, dtype="f32")
    inp = I.make_inputs(w, T, log_a_mode="slow")
    x = [a[0, :, 0] for a in (inp.q, inp.k, inp.v, inp.log_a, inp.lam)]
    do = np.random.default_rng(T + 1).standard_normal((T, 4))
    got = level_form_backward(*x, do)
    want = O.llattn_backward_seq(*x, do)
    scale = max(np.sqrt(np.mean(want[2] ** 2)), 1e-300)
    for name, a, b in zip(("dq", "dk", "dv", "dlog_a", "dlam"), got, want):
        assert np.max(np.abs(a - b)) <= 1e-10 * max(np.sqrt(np.mean(b ** 2)), scale), name


@pytest.mark.parametrize("T", [33, 200, 1025])
def test_tiles_and_block_halves_partition_the_causal_pairs(T):
    """Every pair s < t lies either in one aligned 32-tile (then its level is <= 5) or in the
    left / right halves of exactly one aligned block at its own level (>= 6)."""
    tt, ss = np.meshgrid(np.arange(T), np.arange(T), indexing="ij")
    lower = ss < tt
    lev = np.frompyfunc(_level, 2, 1)(tt, ss).astype(np.int64)
    same_tile = (tt // TILE) == (ss // TILE)
    assert np.all(lev[lower & same_tile] <= DENSE - 1)
    assert np.all(lev[lower & ~same_tile] >= DENSE)
    # a pair at level l >= 6 has s in the left half and t in the right half of one block
    for t, s in zip(tt[lower & ~same_tile][::97], ss[lower & ~same_tile][::97]):
        lvl = lev[t, s]
        lo = (t >> lvl) << lvl
        assert lo <= s < lo + (1 << (lvl - 1)) <= t < lo + (1 << lvl)
