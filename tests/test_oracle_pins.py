"""Pins for the CPU fp64 oracle (no GPU).

Each test ties the oracle to something other than itself: the textbook Fenwick
(binary indexed tree) prefix decomposition, brute force with explicit gate
products, plain Mamba-2 / SSD, causal linear attention in closed form, one-hot
level structure, causality, linearity and the varlen packing rule.  Together
they are chosen so that a dropped term, a wrong sign, an off-by-one level or
index base, or a transposed operand in any oracle form fails at least one.
"""
import numpy as np
import pytest

import oracle as O
from hierarchical_fenwick_state_b200 import inputs as I


def _rand_inputs(T, H=2, dk=3, dv=4, seed=0, log_a_mode="dist", lam_mode="dist", B=1,
                 lam_level=-1, dtype="f32"):
    w = I.Workload("pin", B=B, H=H, T=T, dk=dk, dv=dv, dtype=dtype)
    return I.make_inputs(w, seed, log_a_mode=log_a_mode, lam_mode=lam_mode, lam_level=lam_level)


def bit_prefix_ranges(t):
    """Textbook Fenwick query over the 1-based prefix of length t: ranges (i - lowbit(i), i].

    Returned as 0-based half-open token ranges [lo, hi) covering [0, t).
    """
    out = []
    i = t
    while i > 0:
        low = i & (-i)
        out.append((i - low, i))
        i -= low
    return out


# ----------------------------------------------------------------------------------------------
# Fenwick level function
# ----------------------------------------------------------------------------------------------
@pytest.mark.parametrize("t", list(range(0, 130)) + [255, 256, 1000, 4095, 8191])
def test_levels_match_fenwick_prefix_decomposition(t):
    """Level l >= 1 of query t is exactly one BIT range of [0, t), of size 2**(l-1)."""
    levels = {}
    for s in range(t + 1):
        levels.setdefault(O.fenwick_level(t, s), []).append(s)
    assert levels[0] == [t]
    ranges = bit_prefix_ranges(t)
    expect = {}
    for lo, hi in ranges:
        size = hi - lo
        assert size & (size - 1) == 0
        expect[1 + size.bit_length() - 1] = list(range(lo, hi))
    got = {l: ss for l, ss in levels.items() if l >= 1}
    assert got == expect
    # one block per set bit of t: popcount(t) + 1 non-empty levels
    assert len(levels) == bin(t).count("1") + 1
    # recent tokens sit in small buckets: level is non-decreasing as s moves back in time
    lv = [O.fenwick_level(t, s) for s in range(t, -1, -1)]
    assert all(a <= b for a, b in zip(lv, lv[1:]))


def test_level_matrix_matches_scalar():
    tt = np.arange(0, 300)
    ss = np.arange(0, 300)
    M = O.fenwick_level_matrix(tt, ss)
    for t in range(0, 300, 7):
        for s in range(0, 300, 5):
            assert M[t, s] == O.fenwick_level(t, s)
    # large positions used by the long workloads
    big = np.array([65535, 65534, 32768, 1])
    Mb = O.fenwick_level_matrix(big, np.array([0, 1, 32767, 65535]))
    for i, t in enumerate(big):
        for j, s in enumerate([0, 1, 32767, 65535]):
            assert Mb[i, j] == O.fenwick_level(int(t), s)


def test_num_levels_of_the_workloads():
    assert [I.WORKLOADS[n].L for n in ("t256_d32_f32", "t2k_d64_bf16", "t8k_d64_bf16",
                                         "t64k_d128_bf16", "varlen8_d64_bf16")] == [9, 12, 14, 17, 15]
    # the largest level that occurs below T is L - 1
    for T in (1, 2, 3, 5, 16, 17, 256, 300):
        L = I.num_levels(T)
        mx = max(O.fenwick_level(t, 0) for t in range(T))
        assert mx == L - 1


# ----------------------------------------------------------------------------------------------
# Worked example written out by hand (T = 4, scalar q,k,v)
# ----------------------------------------------------------------------------------------------
def test_hand_worked_example_t4():
    q = np.array([[0.5], [-1.0], [2.0], [1.5]])
    k = np.array([[1.0], [0.25], [-0.5], [2.0]])
    v = np.array([[3.0], [-2.0], [1.0], [0.5]])
    a = np.array([0.9, 0.8, 0.5, 0.25])
    lam = np.array([[1.0, 2.0, 3.0], [1.5, 2.5, 3.5], [0.5, 0.75, 1.25], [2.0, 4.0, 8.0]])
    la = np.log(a)
    # Fenwick buckets by hand: t=0 {0}; t=1 {1},{0}@1; t=2 {2},{0,1}@2; t=3 {3},{2}@1,{0,1}@2
    o0 = lam[0, 0] * q[0] * k[0] * v[0]
    o1 = lam[1, 0] * q[1] * k[1] * v[1] + lam[1, 1] * a[1] * q[1] * k[0] * v[0]
    o2 = (lam[2, 0] * q[2] * k[2] * v[2] + lam[2, 2] * a[2] * q[2] * k[1] * v[1]
          + lam[2, 2] * a[2] * a[1] * q[2] * k[0] * v[0])
    o3 = (lam[3, 0] * q[3] * k[3] * v[3] + lam[3, 1] * a[3] * q[3] * k[2] * v[2]
          + lam[3, 2] * a[3] * a[2] * q[3] * k[1] * v[1]
          + lam[3, 2] * a[3] * a[2] * a[1] * q[3] * k[0] * v[0])
    expect = np.stack([o0, o1, o2, o3])
    np.testing.assert_allclose(O.llattn_bruteforce_seq(q, k, v, la, lam), expect, rtol=1e-14)
    np.testing.assert_allclose(O.llattn_quadratic_seq(q, k, v, la, lam), expect, rtol=1e-14)
    got = O.llattn_recurrent_seq(q[None], k[None], v[None], la[None], lam[None])[0]
    np.testing.assert_allclose(got, expect, rtol=1e-14)


# ----------------------------------------------------------------------------------------------
# Three forms agree exhaustively on tiny T
# ----------------------------------------------------------------------------------------------
@pytest.mark.parametrize("T", list(range(1, 17)))
@pytest.mark.parametrize("mode", ["dist", "zero", "strong"])
def test_bruteforce_quadratic_recurrent_agree(T, mode):
    inp = _rand_inputs(T, seed=T, log_a_mode=mode)
    bf = O.llattn_bruteforce(inp)
    qd = O.llattn_quadratic(inp, block=5)
    rc = O.llattn_recurrent(inp)
    scale = max(1.0, np.abs(bf).max())
    assert np.abs(bf - qd).max() <= 1e-12 * scale
    assert np.abs(bf - rc).max() <= 1e-12 * scale


def test_quadratic_recurrent_agree_moderate_T():
    inp = _rand_inputs(300, H=2, dk=8, dv=5, seed=3)
    qd = O.llattn_quadratic(inp, block=64)
    rc = O.llattn_recurrent(inp)
    assert O.rel_max_err(rc, qd) < 1e-12


def test_single_output_matches_quadratic():
    inp = _rand_inputs(200, H=3, dk=6, dv=4, seed=5, B=2)
    qd = O.llattn_quadratic(inp)
    samples = [(0, 0), (1, 2), (57, 1), (199, 0), (200, 1), (399, 2), (263, 0)]
    got = O.llattn_sampled(inp, samples)
    ref = qd.reshape(-1, inp.H, inp.dv)
    for i, (tok, h) in enumerate(samples):
        np.testing.assert_allclose(got[i], ref[tok, h], rtol=1e-11, atol=1e-13)


# ----------------------------------------------------------------------------------------------
# Reductions to textbook models
# ----------------------------------------------------------------------------------------------
@pytest.mark.parametrize("c", [1.0, 0.37])
def test_constant_lambda_is_mamba2(c):
    inp = _rand_inputs(130, H=2, dk=5, dv=3, seed=11, lam_mode="ones")
    inp.lam[...] = c
    c = float(np.float32(c))  # the value the fp32 lam array holds
    m2 = O.mamba2_recurrent(inp)
    for f in (O.llattn_recurrent, O.llattn_quadratic):
        np.testing.assert_allclose(f(inp), c * m2, rtol=1e-11, atol=1e-12)


def test_no_decay_unit_lambda_is_causal_linear_attention():
    inp = _rand_inputs(97, H=1, dk=4, dv=6, seed=2, log_a_mode="zero", lam_mode="ones")
    Q = inp.q[0, :, 0].astype(np.float64)
    K = inp.k[0, :, 0].astype(np.float64)
    V = inp.v[0, :, 0].astype(np.float64)
    ref = np.tril(Q @ K.T) @ V
    for f in (O.llattn_recurrent, O.llattn_quadratic, O.mamba2_recurrent):
        np.testing.assert_allclose(f(inp)[0, :, 0], ref, rtol=1e-11, atol=1e-12)


# ----------------------------------------------------------------------------------------------
# One level at a time
# ----------------------------------------------------------------------------------------------
def test_one_hot_levels():
    T = 70
    base = _rand_inputs(T, H=1, dk=4, dv=3, seed=9, log_a_mode="zero")
    L = base.L
    Q = base.q[0, :, 0].astype(np.float64)
    K = base.k[0, :, 0].astype(np.float64)
    V = base.v[0, :, 0].astype(np.float64)
    total = np.zeros((T, 3))
    for l0 in range(L):
        inp = _rand_inputs(T, H=1, dk=4, dv=3, seed=9, log_a_mode="zero", lam_mode="onehot",
                           lam_level=l0)
        got = O.llattn_recurrent(inp)[0, :, 0]
        np.testing.assert_allclose(O.llattn_quadratic(inp)[0, :, 0], got, rtol=1e-11, atol=1e-12)
        for t in range(T):
            if l0 == 0:
                exp = (Q[t] @ K[t]) * V[t]
            else:
                blocks = [(lo, hi) for lo, hi in bit_prefix_ranges(t) if hi - lo == 2 ** (l0 - 1)]
                exp = np.zeros(3)
                for lo, hi in blocks:
                    exp = exp + (Q[t] @ K[lo:hi].T) @ V[lo:hi]
            np.testing.assert_allclose(got[t], exp, rtol=1e-11, atol=1e-12)
        total += got
    ones = _rand_inputs(T, H=1, dk=4, dv=3, seed=9, log_a_mode="zero", lam_mode="ones")
    np.testing.assert_allclose(total, O.llattn_recurrent(ones)[0, :, 0], rtol=1e-11, atol=1e-12)


# ----------------------------------------------------------------------------------------------
# Causality and linearity
# ----------------------------------------------------------------------------------------------
def test_causality():
    inp = _rand_inputs(64, H=2, dk=4, dv=4, seed=4)
    ref = O.llattn_recurrent(inp)
    s = 37
    inp.k[0, s] += 1.0
    inp.v[0, s] -= 2.0
    inp.log_a[0, s] -= 0.3
    got = O.llattn_recurrent(inp)
    assert np.array_equal(got[0, :s], ref[0, :s])
    assert np.abs(got[0, s:] - ref[0, s:]).max() > 1e-3


def test_linearity_in_v():
    a = _rand_inputs(50, seed=1)
    b = _rand_inputs(50, seed=2)
    b.q[...] = a.q
    b.k[...] = a.k
    b.log_a[...] = a.log_a
    b.lam[...] = a.lam
    mix = _rand_inputs(50, seed=1)
    mix.v[...] = (2.0 * a.v.astype(np.float64) - 0.5 * b.v.astype(np.float64)).astype(np.float32)
    lhs = O.llattn_quadratic(mix)
    rhs = 2.0 * O.llattn_quadratic(a) - 0.5 * O.llattn_quadratic(b)
    np.testing.assert_allclose(lhs, rhs, rtol=1e-6, atol=1e-6)


# ----------------------------------------------------------------------------------------------
# Varlen: packed = per-sequence runs concatenated
# ----------------------------------------------------------------------------------------------
def test_varlen_is_per_sequence_concatenation():
    w = I.Workload("vl", B=4, H=2, T=64, dk=4, dv=3, dtype="bf16", varlen=True, len_lo=1, len_hi=64)
    inp = I.make_inputs(w, 3, lengths=np.array([17, 1, 64, 30]))
    got = O.llattn_recurrent(inp)
    assert got.shape == (112, 2, 3)
    for start, n in inp.seq_slices():
        sub = I.Inputs(q=inp.q[start:start + n][None], k=inp.k[start:start + n][None],
                       v=inp.v[start:start + n][None], log_a=inp.log_a[start:start + n][None],
                       lam=inp.lam[start:start + n][None], cu_seqlens=None, B=1, H=2, T=n,
                       dk=4, dv=3, dtype="bf16")
        np.testing.assert_allclose(got[start:start + n], O.llattn_quadratic(sub)[0],
                                   rtol=1e-11, atol=1e-12)


# ----------------------------------------------------------------------------------------------
# Input generator
# ----------------------------------------------------------------------------------------------
def test_bf16_rounding_matches_torch():
    torch = pytest.importorskip("torch")
    x = np.random.default_rng(0).standard_normal(100000).astype(np.float32) * 7.0
    x[:4] = [1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -0.0, 3.0e38]
    ours = I.round_to_bf16(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    assert np.array_equal(ours.view(np.uint32), ref.view(np.uint32))


def test_inputs_are_seeded_and_shaped():
    w = I.shrink(I.WORKLOADS["t2k_d64_bf16"], B=1, H=2, T=128)
    a = I.make_inputs(w, 0)
    b = I.make_inputs(w, 0)
    assert np.array_equal(a.q, b.q) and np.array_equal(a.lam, b.lam)
    assert a.q.shape == (1, 128, 2, 64) and a.lam.shape == (1, 128, 2, 8)
    np.testing.assert_allclose(np.linalg.norm(a.q.astype(np.float64), axis=-1), 1.0, atol=1e-2)
    assert (a.log_a < 0).all() and (a.lam > 0).all()
    assert np.array_equal(I.round_to_bf16(a.v), a.v)


# ----------------------------------------------------------------------------------------------
# Limits with closed forms
# ----------------------------------------------------------------------------------------------
def test_strong_decay_limit_keeps_only_the_token_itself():
    """With every gate a_t ~ 0 (log a = -60), every s < t is weighted by at most e^-60: the
    output reduces to the level-0 term lam[t, 0] (q_t . k_t) v_t."""
    inp = _rand_inputs(40, H=2, dk=5, dv=3, seed=11)
    inp.log_a[...] = -60.0
    q = inp.q.reshape(-1, inp.H, inp.dk).astype(np.float64)
    k = inp.k.reshape(-1, inp.H, inp.dk).astype(np.float64)
    v = inp.v.reshape(-1, inp.H, inp.dv).astype(np.float64)
    lam0 = inp.lam.reshape(-1, inp.H, inp.L)[..., 0].astype(np.float64)
    want = (lam0 * np.einsum("thd,thd->th", q, k))[..., None] * v
    for form in (O.llattn_recurrent, O.llattn_quadratic):
        got = form(inp).reshape(want.shape)
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-20)


def test_two_token_closed_form():
    """T = 2: o_0 = lam[0,0] (q0.k0) v0;  o_1 = lam[1,0] (q1.k1) v1 + lam[1,1] a_1 (q1.k0) v0."""
    inp = _rand_inputs(2, H=1, dk=4, dv=3, seed=12)
    q, k, v = (x.reshape(2, -1).astype(np.float64) for x in (inp.q, inp.k, inp.v))
    lam = inp.lam.reshape(2, inp.L).astype(np.float64)
    a1 = np.exp(np.float64(inp.log_a.reshape(2)[1]))
    o0 = lam[0, 0] * (q[0] @ k[0]) * v[0]
    o1 = lam[1, 0] * (q[1] @ k[1]) * v[1] + lam[1, 1] * a1 * (q[1] @ k[0]) * v[0]
    for form in (O.llattn_bruteforce, O.llattn_quadratic, O.llattn_recurrent):
        got = form(inp).reshape(2, -1)
        np.testing.assert_allclose(got, np.stack([o0, o1]), rtol=1e-13, atol=0)
