"""Pins for the Log-Linear Gated DeltaNet oracle (no GPU).

The two forms (explicit products of the gated delta transitions per pair, and one
state per Fenwick level) are checked against each other and against things fixed
outside them:
  * orthonormal keys: every transition leaves the other keys alone, so the output is
    the Log-Linear Mamba-2 oracle's (itself pinned) with v_s scaled by beta_s;
  * lam == 1: plain Gated DeltaNet, one state;
  * the delta rule's overwrite: with beta = 1 and no decay, writing a second value
    under the same unit key replaces the first;
  * one-hot levels summing to lam == 1, linearity in v, causality, beta = 0.
Six mistakes planted in the oracle (on the CPU) are each caught: the new token's write
also taking the transition, a write without beta, a Fenwick level off by one in the brute
force, the gate alpha left out of the transition, the transition product in reverse
order, and the erase term with the wrong sign.
"""
import numpy as np
import pytest

import oracle as O
from hierarchical_fenwick_state_b200 import inputs as I


def _gdn_inputs(T, H=2, dk=4, dv=3, seed=0, B=1, log_a_mode="dist", lam_mode="dist",
                lam_level=-1, beta_mode="dist"):
    w = I.Workload("gdnpin", B=B, H=H, T=T, dk=dk, dv=dv, dtype="f32")
    return I.make_gdn_inputs(w, seed, log_a_mode=log_a_mode, lam_mode=lam_mode,
                             lam_level=lam_level, beta_mode=beta_mode)


@pytest.mark.parametrize("T", [1, 2, 3, 5, 8, 11, 16])
def test_bruteforce_equals_recurrent(T):
    inp = _gdn_inputs(T, seed=T)
    np.testing.assert_allclose(O.gdn_recurrent(inp), O.gdn_bruteforce(inp), rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("beta_mode", ["dist", "ones"])
def test_orthonormal_keys_reduce_to_log_linear_mamba2(beta_mode):
    T, dk = 12, 16
    inp = _gdn_inputs(T, H=2, dk=dk, dv=5, seed=3, beta_mode=beta_mode)
    rng = np.random.default_rng(4)
    for h in range(inp.H):
        Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
        inp.k[0, :, h, :] = Qm[:T].astype(np.float32)      # rows orthonormal
    got = O.gdn_recurrent(inp)
    scaled = I.Inputs(q=inp.q, k=inp.k, v=inp.v * inp.beta[..., None], log_a=inp.log_a,
                      lam=inp.lam, cu_seqlens=None, B=inp.B, H=inp.H, T=inp.T, dk=inp.dk,
                      dv=inp.dv, dtype=inp.dtype)
    np.testing.assert_allclose(got, O.llattn_recurrent(scaled), rtol=1e-5, atol=1e-6)


def test_lam_ones_is_plain_gated_deltanet():
    inp = _gdn_inputs(50, H=3, dk=6, dv=4, seed=5, lam_mode="ones")
    np.testing.assert_allclose(O.gdn_recurrent(inp), O.gated_deltanet(inp), rtol=1e-10, atol=1e-12)


def test_delta_rule_overwrites_a_key():
    # no decay, beta = 1, one unit key written three times: reading it returns the last value
    inp = _gdn_inputs(3, H=1, dk=4, dv=3, seed=6, log_a_mode="zero", lam_mode="ones",
                      beta_mode="ones")
    e = np.array([0.6, 0.0, 0.8, 0.0], np.float32)
    inp.k[0, :, 0, :] = e
    inp.q[0, :, 0, :] = e
    for f in (O.gdn_recurrent, O.gated_deltanet, O.gdn_bruteforce):
        o = f(inp)[0, :, 0]
        np.testing.assert_allclose(o, inp.v[0, :, 0].astype(np.float64), rtol=1e-6, atol=1e-6)


def test_one_hot_levels_sum_to_lam_ones():
    T = 37
    L = I.num_levels(T)
    total = sum(O.gdn_recurrent(_gdn_inputs(T, seed=7, lam_mode="onehot", lam_level=l))
                for l in range(L))
    np.testing.assert_allclose(total, O.gdn_recurrent(_gdn_inputs(T, seed=7, lam_mode="ones")),
                               rtol=1e-10, atol=1e-12)


def test_linear_in_v_and_zero_beta():
    # quarter-integer values, so that v_a + 2 v_b is exact in fp32 storage
    a = _gdn_inputs(29, seed=8)
    a.v = (np.round(a.v * 4.0) / 4.0).astype(np.float32)
    b = _gdn_inputs(29, seed=8)
    b.v = (np.round(np.random.default_rng(9).standard_normal(b.v.shape) * 4.0) / 4.0).astype(np.float32)
    c = _gdn_inputs(29, seed=8)
    c.v = a.v + 2.0 * b.v
    np.testing.assert_allclose(O.gdn_recurrent(c), O.gdn_recurrent(a) + 2.0 * O.gdn_recurrent(b),
                               rtol=1e-9, atol=1e-10)
    z = _gdn_inputs(29, seed=8, beta_mode="zero")
    assert np.all(O.gdn_recurrent(z) == 0.0)


def test_causality():
    a = _gdn_inputs(40, seed=10)
    b = _gdn_inputs(40, seed=10)
    s = 17
    b.k[0, s] += 0.5
    b.v[0, s] -= 1.0
    b.beta[0, s] = 0.3
    da = np.abs(O.gdn_recurrent(a) - O.gdn_recurrent(b))
    assert np.all(da[0, :s] == 0.0)
    assert np.all(da[0, s:].max(axis=(1, 2)) > 0.0)


def test_single_outputs_match_recurrent():
    w = I.Workload("gdnvl", B=3, H=2, T=70, dk=5, dv=4, dtype="f32", varlen=True)
    inp = I.make_gdn_inputs(w, 11, lengths=np.array([70, 1, 33]))
    ref = O.gdn_recurrent(inp).reshape(-1, inp.H, inp.dv)
    samples = [(0, 0), (69, 1), (70, 0), (71, 1), (103, 0), (90, 1), (35, 0)]
    got = O.gdn_sampled(inp, samples)
    np.testing.assert_allclose(got, np.stack([ref[t, h] for t, h in samples]), rtol=1e-10,
                               atol=1e-12)


def test_packed_sequences_are_independent():
    w = I.Workload("gdnvl2", B=3, H=2, T=40, dk=4, dv=3, dtype="f32", varlen=True)
    inp = I.make_gdn_inputs(w, 12, lengths=np.array([40, 0, 23]))
    got = O.gdn_recurrent(inp)
    # the third sequence alone
    sl = slice(40, 63)
    one = I.Inputs(q=inp.q[sl][None], k=inp.k[sl][None], v=inp.v[sl][None],
                   log_a=inp.log_a[sl][None], lam=inp.lam[sl][None], cu_seqlens=None, B=1,
                   H=inp.H, T=23, dk=inp.dk, dv=inp.dv, dtype="f32", beta=inp.beta[sl][None])
    np.testing.assert_allclose(got[sl], O.gdn_recurrent(one)[0], rtol=1e-12, atol=1e-14)
