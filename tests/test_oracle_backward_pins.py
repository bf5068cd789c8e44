"""Pins for the oracle's backward pass (no GPU).

``llattn_backward_seq`` differentiates the masked form product by product.  It is
tied here to things that share none of its code:
  * central finite differences of the brute-force forward (explicit gate
    products, per-pair level), element by element on tiny inputs, and along
    random directions of the quadratic form on a longer one;
  * dq equals the forward itself with the roles of its inputs swapped
    (queries do, keys v, values k), which follows from the definition;
  * the first token's gate never enters the output, so its gradient is zero;
  * linearity in do, and packed sequences equal per-sequence runs.
A dropped term of the gate gradient, a transposed product, a level read from the
wrong side or a cumulative sum taken the wrong way fails at least one of these.
"""
import numpy as np
import pytest

import oracle as O
from hierarchical_fenwick_state_b200 import inputs as I


def _seq(T, dk=3, dv=4, seed=0, log_a_mode="dist"):
    w = I.Workload("pin", B=1, H=1, T=T, dk=dk, dv=dv, dtype="f32")
    inp = I.make_inputs(w, seed, log_a_mode=log_a_mode)
    x = {"q": inp.q[0, :, 0], "k": inp.k[0, :, 0], "v": inp.v[0, :, 0],
         "log_a": inp.log_a[0, :, 0], "lam": inp.lam[0, :, 0]}
    x = {n: a.astype(np.float64) for n, a in x.items()}
    do = np.random.default_rng(seed + 100).standard_normal((T, dv))
    return x, do


def _loss(fwd, x, do):
    return float(np.sum(do * fwd(x["q"], x["k"], x["v"], x["log_a"], x["lam"])))


def _grads(x, do):
    dq, dk, dv, dla, dlm = O.llattn_backward_seq(x["q"], x["k"], x["v"], x["log_a"], x["lam"], do)
    return {"q": dq, "k": dk, "v": dv, "log_a": dla, "lam": dlm}


@pytest.mark.parametrize("T", [1, 2, 3, 5, 8, 9])
@pytest.mark.parametrize("name", ["q", "k", "v", "log_a", "lam"])
def test_every_element_matches_central_differences(T, name):
    x, do = _seq(T, seed=T)
    g = _grads(x, do)[name]
    eps = 1e-6
    fd = np.zeros_like(x[name])
    for idx in np.ndindex(x[name].shape):
        xp = {n: a.copy() for n, a in x.items()}
        xm = {n: a.copy() for n, a in x.items()}
        xp[name][idx] += eps
        xm[name][idx] -= eps
        fd[idx] = (_loss(O.llattn_bruteforce_seq, xp, do)
                   - _loss(O.llattn_bruteforce_seq, xm, do)) / (2 * eps)
    scale = max(np.abs(fd).max(), 1e-3)
    np.testing.assert_allclose(g, fd, rtol=0, atol=2e-7 * scale)


@pytest.mark.parametrize("name", ["q", "k", "v", "log_a", "lam"])
def test_directional_derivatives_T70(name):
    """Longer sequence (several levels deep), random directions, quadratic-form forward."""
    x, do = _seq(70, dk=5, dv=3, seed=4, log_a_mode="slow")
    g = _grads(x, do)[name]
    rng = np.random.default_rng(5)
    for _ in range(3):
        u = rng.standard_normal(x[name].shape)
        eps = 1e-6
        xp = {n: a.copy() for n, a in x.items()}
        xm = {n: a.copy() for n, a in x.items()}
        xp[name] += eps * u
        xm[name] -= eps * u
        fd = (_loss(O.llattn_quadratic_seq, xp, do) - _loss(O.llattn_quadratic_seq, xm, do)) / (2 * eps)
        an = float(np.sum(g * u))
        assert abs(an - fd) <= 1e-6 * max(abs(fd), 1.0), (an, fd)


def test_dq_is_the_forward_with_roles_swapped():
    """dq_t = sum_{s<=t} lam[t, l(t,s)] exp(g_t - g_s) (do_t . v_s) k_s: the forward on
    queries do, keys v and values k."""
    x, do = _seq(100, dk=4, dv=6, seed=6, log_a_mode="slow")
    g = _grads(x, do)
    want = O.llattn_quadratic_seq(do, x["v"], x["k"], x["log_a"], x["lam"])
    np.testing.assert_allclose(g["q"], want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


def test_first_gate_has_no_gradient():
    """No gate product prod_{r=s+1..t} a_r ever includes position 0."""
    x, do = _seq(50, seed=7)
    g = _grads(x, do)
    assert abs(g["log_a"][0]) <= 1e-12 * np.abs(g["log_a"]).max()


def test_gradients_are_linear_in_do():
    x, do = _seq(30, seed=8)
    do2 = np.random.default_rng(9).standard_normal(do.shape)
    g1, g2, g12 = _grads(x, do), _grads(x, do2), _grads(x, 2.0 * do - 3.0 * do2)
    for n in g1:
        np.testing.assert_allclose(g12[n], 2.0 * g1[n] - 3.0 * g2[n], rtol=1e-10,
                                   atol=1e-12 * max(np.abs(g12[n]).max(), 1.0))


def test_packed_backward_is_per_sequence():
    w = I.Workload("pin", B=3, H=2, T=40, dk=4, dv=4, dtype="f32", varlen=True, len_lo=1,
                   len_hi=40)
    inp = I.make_inputs(w, 10, lengths=np.array([17, 1, 40]))
    do = np.random.default_rng(11).standard_normal(inp.v.shape)
    got = O.llattn_backward(inp, do)
    for start, n in inp.seq_slices():
        for h in range(inp.H):
            sl = slice(start, start + n)
            dq, dk, dv, dla, dlm = O.llattn_backward_seq(
                inp.q[sl, h], inp.k[sl, h], inp.v[sl, h], inp.log_a[sl, h], inp.lam[sl, h],
                do[sl, h])
            np.testing.assert_array_equal(got["q"][sl, h], dq)
            np.testing.assert_array_equal(got["k"][sl, h], dk)
            np.testing.assert_array_equal(got["v"][sl, h], dv)
            np.testing.assert_array_equal(got["log_a"][sl, h], dla)
            np.testing.assert_array_equal(got["lam"][sl, h], dlm)


def test_sampled_rows_equal_the_full_gradients():
    """The per-row / per-column direct sums (used at full size) agree with the full backward,
    on a packed batch with an empty and a one-token sequence."""
    w = I.Workload("pin", B=4, H=2, T=90, dk=6, dv=5, dtype="f32", varlen=True, len_lo=0,
                   len_hi=90)
    inp = I.make_inputs(w, 12, lengths=np.array([33, 0, 1, 90]), log_a_mode="slow")
    do = np.random.default_rng(13).standard_normal(inp.v.shape)
    full = O.llattn_backward(inp, do)
    total = inp.total_tokens
    samples = [(t, h) for t in range(total) for h in range(inp.H)]
    got = O.llattn_backward_sampled(inp, do, samples)
    for name in ("q", "k", "v", "lam"):
        want = np.array([full[name][t, h] for t, h in samples])
        np.testing.assert_allclose(got[name], want, rtol=1e-10, atol=1e-12 * np.abs(want).max())
