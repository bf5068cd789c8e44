"""Pins for the oracle's decoding form (no GPU).

``llattn_decode_step`` walks the binary counter (gate, read out, carry).  It is
tied here to code that shares none of its steps:
  * brute force with explicit gate products and the per-pair level (the
    definition), and the quadratic masked form, over whole sequences decoded
    token by token;
  * ``llattn_level_states``, which builds each level's state from the level
    function l(n, s) directly, after every step (so the carry is checked slot by
    slot), itself checked by reading o_n out of it against brute force;
  * causal linear attention in closed form (no gate, unit weights).
A dropped gate, a carry into the wrong level, an occupancy read off the wrong
bit, or a readout missing level 0 fails at least one of these.
"""
import numpy as np
import pytest

import oracle as O
from hierarchical_fenwick_state_b200 import inputs as I


def _seq(T, dk=3, dv=4, seed=0, log_a_mode="dist", lam_mode="dist"):
    w = I.Workload("pin", B=1, H=1, T=T, dk=dk, dv=dv, dtype="f32")
    inp = I.make_inputs(w, seed, log_a_mode=log_a_mode, lam_mode=lam_mode)
    return inp.q[0, :, 0], inp.k[0, :, 0], inp.v[0, :, 0], inp.log_a[0, :, 0], inp.lam[0, :, 0]


@pytest.mark.parametrize("T", list(range(1, 17)) + [31, 32, 33])
@pytest.mark.parametrize("seed", [0, 1])
def test_decoding_matches_bruteforce(T, seed):
    q, k, v, la, lam = _seq(T, seed=seed)
    got = O.llattn_decode_sequence(q, k, v, la, lam)
    want = O.llattn_bruteforce_seq(q, k, v, la, lam)
    assert O.rel_max_err(got, want) < 1e-12


def test_decoding_matches_quadratic_T300():
    q, k, v, la, lam = _seq(300, dk=8, dv=5, seed=3, log_a_mode="slow")
    got = O.llattn_decode_sequence(q, k, v, la, lam)
    want = O.llattn_quadratic_seq(q, k, v, la, lam)
    assert O.rel_max_err(got, want) < 1e-12


def test_no_gate_unit_weights_is_causal_linear_attention():
    q, k, v, la, lam = _seq(40, seed=4, log_a_mode="zero", lam_mode="ones")
    got = O.llattn_decode_sequence(q, k, v, la, lam)
    scores = np.tril(q.astype(np.float64) @ k.astype(np.float64).T)
    assert O.rel_max_err(got, scores @ v.astype(np.float64)) < 1e-12


@pytest.mark.parametrize("T", [1, 2, 7, 64, 100])
def test_states_after_every_step_are_the_fenwick_buckets(T):
    """After the token at n, every occupied slot equals the bucket built from l(n+1, s)."""
    q, k, v, la, lam = _seq(T, seed=5, log_a_mode="slow")
    nslot = lam.shape[1] - 1
    S = np.zeros((nslot, q.shape[1], v.shape[1]))
    for n in range(T):
        _, S = O.llattn_decode_step(S, n, q[n], k[n], v[n], la[n], lam[n])
        if (n + 1).bit_length() > nslot:
            continue  # the last position of a full counter: no slot for its carry
        want = O.llattn_level_states(k, v, la, n + 1, nslot)
        for lvl in range(1, nslot + 1):
            if ((n + 1) >> (lvl - 1)) & 1:
                np.testing.assert_allclose(S[lvl - 1], want[lvl - 1], rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("n", [0, 1, 2, 3, 5, 6, 7, 8, 11, 12])
def test_level_states_read_out_to_the_definition(n):
    """o_n = lam_0 (q.k_n) v_n + sum over occupied l of lam_l a_n q^T S_l(n) equals brute force."""
    T = 16
    q, k, v, la, lam = _seq(T, seed=6)
    S = O.llattn_level_states(k, v, la, n, lam.shape[1] - 1)
    occupied = [lvl for lvl in range(1, S.shape[0] + 1) if (n >> (lvl - 1)) & 1]
    empty = [lvl for lvl in range(1, S.shape[0] + 1) if lvl not in occupied]
    for lvl in empty:
        assert not S[lvl - 1].any()
    qn, kn, vn = (x[n].astype(np.float64) for x in (q, k, v))
    o = np.float64(lam[n, 0]) * float(np.dot(qn, kn)) * vn
    for lvl in occupied:
        o = o + np.float64(lam[n, lvl]) * np.exp(np.float64(la[n])) * (qn @ S[lvl - 1])
    want = O.llattn_bruteforce_seq(q, k, v, la, lam)[n]
    np.testing.assert_allclose(o, want, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("n", [0, 1, 6, 11, 13, 14])
def test_empty_slots_are_ignored(n):
    """Slots whose bit of n is clear may hold anything: output and occupied states do not move."""
    T = 16
    q, k, v, la, lam = _seq(T, seed=7)
    nslot = lam.shape[1] - 1
    S = O.llattn_level_states(k, v, la, n, nslot)
    junk = S.copy()
    rng = np.random.default_rng(n)
    for lvl in range(1, nslot + 1):
        if not (n >> (lvl - 1)) & 1:
            junk[lvl - 1] = rng.standard_normal(junk[lvl - 1].shape) * 1e3
    o1, S1 = O.llattn_decode_step(S, n, q[n], k[n], v[n], la[n], lam[n])
    o2, S2 = O.llattn_decode_step(junk, n, q[n], k[n], v[n], la[n], lam[n])
    np.testing.assert_array_equal(o1, o2)
    for lvl in range(1, nslot + 1):
        if ((n + 1) >> (lvl - 1)) & 1:
            np.testing.assert_array_equal(S1[lvl - 1], S2[lvl - 1])


def test_last_position_of_a_full_counter_merges_nothing():
    """n = 2**nslot - 1 fills every slot; its carry has no slot, the output is still exact."""
    T = 8
    q, k, v, la, lam = _seq(T, seed=8)
    nslot = lam.shape[1] - 1
    assert nslot == 3
    n = 7
    S = O.llattn_level_states(k, v, la, n, nslot)
    o, S1 = O.llattn_decode_step(S, n, q[n], k[n], v[n], la[n], lam[n])
    np.testing.assert_allclose(o, O.llattn_bruteforce_seq(q, k, v, la, lam)[n], rtol=1e-12)
    a = np.exp(np.float64(la[n]))
    np.testing.assert_allclose(S1, S * a, rtol=1e-15)   # gated, not merged
    with pytest.raises(ValueError):
        O.llattn_decode_step(S1, 8, q[0], k[0], v[0], la[0], lam[0])


def test_batch_rows_keep_their_own_positions():
    """Rows of a batch at different positions decode independently (each its own counter)."""
    T = 16
    B, H = 3, 2
    pos = np.array([5, 0, 12])
    w = I.Workload("pin", B=B, H=H, T=T, dk=3, dv=4, dtype="f32")
    inp = I.make_inputs(w, 9)
    nslot = inp.L - 1
    S = np.zeros((B, H, nslot, 3, 4))
    q = np.zeros((B, H, 3)); k = np.zeros((B, H, 3)); v = np.zeros((B, H, 4))
    la = np.zeros((B, H)); lam = np.zeros((B, H, inp.L))
    for b in range(B):
        n = int(pos[b])
        for h in range(H):
            S[b, h] = O.llattn_level_states(inp.k[b, :, h], inp.v[b, :, h], inp.log_a[b, :, h],
                                            n, nslot)
        q[b], k[b], v[b] = inp.q[b, n], inp.k[b, n], inp.v[b, n]
        la[b], lam[b] = inp.log_a[b, n], inp.lam[b, n]
    o, _ = O.llattn_decode_batch(S, pos, q, k, v, la, lam)
    ref = O.llattn_bruteforce(inp)
    for b in range(B):
        np.testing.assert_allclose(o[b], ref[b, pos[b]], rtol=1e-12, atol=1e-13)
