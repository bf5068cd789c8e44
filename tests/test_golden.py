"""Golden fixtures (tests/golden/) against an independent computation and the oracle.

The fixtures hold outputs for the closed-form inputs of ``inputs.make_patterned``,
written by tests/golden/make_golden.py from the oracle.  Here they are checked
against a computation that shares nothing with the oracle's code: the textbook
Fenwick (binary indexed tree) decomposition of the prefix [0, t) into ranges
(i - lowbit(i), i], each range of 2^m tokens being level m + 1 and the token
itself level 0 ("Log-Linear Attention", gist.science, Italian "Sommario tecnico"
section 2, "Partizionamento Gerarchico (Fenwick Tree)"), with the gate product
over a constant gate taken as a power.  With no decay the sums are done in exact
integer arithmetic, so the stored values must match exactly.
"""
import math
import os

import numpy as np
import pytest

import oracle as O
from hierarchical_fenwick_state_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
FIXTURES = {"patterned_nodecay_T300": 0.0, "patterned_decay8_T300": -0.125}


def load(name):
    rows = []
    with open(os.path.join(GOLDEN, name + ".txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            t, j, o = line.split()
            rows.append((int(t), int(j), float(o)))
    return rows


def bit_ranges(t):
    """[lo, hi) token ranges of the Fenwick decomposition of [0, t)."""
    out, i = [], t
    while i > 0:
        low = i & -i
        out.append((i - low, i))
        i -= low
    return out


def independent_output(inp, t, decay):
    """o[t, head 0, :] from the Fenwick ranges; exact (integer, quarter units) if decay is 0."""
    q = inp.q[0, :, 0].astype(np.int64)
    k = inp.k[0, :, 0].astype(np.int64)
    v = inp.v[0, :, 0].astype(np.int64)
    lam4 = np.rint(inp.lam[0, :, 0] * 4).astype(np.int64)   # lam in quarter units
    assert np.array_equal(lam4 / 4.0, inp.lam[0, :, 0])
    parts = [(0, t, t + 1)]
    for lo, hi in bit_ranges(t):
        parts.append((1 + int(math.log2(hi - lo)), lo, hi))
    if decay == 0.0:
        acc = np.zeros(inp.dv, dtype=np.int64)
        for lvl, lo, hi in parts:
            for s in range(lo, hi):
                acc += lam4[t, lvl] * int(np.dot(q[t], k[s])) * v[s]
        return acc / 4.0
    a = math.exp(decay)
    acc = np.zeros(inp.dv)
    for lvl, lo, hi in parts:
        for s in range(lo, hi):
            acc += (lam4[t, lvl] / 4.0) * a ** (t - s) * float(np.dot(q[t], k[s])) * v[s]
    return acc


@pytest.mark.parametrize("name", list(FIXTURES))
def test_fixture_matches_fenwick_ranges(name):
    decay = FIXTURES[name]
    inp = I.make_patterned(300, log_a=decay, dtype="f32")
    assert float(np.float32(decay)) == decay      # the gate is exact in fp32 too
    rows = load(name)
    by_t = {}
    for t, j, o in rows:
        by_t.setdefault(t, {})[j] = o
    for t, cols in by_t.items():
        want = independent_output(inp, t, decay)
        got = np.array([cols[j] for j in range(inp.dv)])
        if decay == 0.0:
            assert np.array_equal(got, want), f"t={t}"
            assert np.array_equal(got * 4, np.rint(got * 4))   # multiples of 1/4
        else:
            np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-9 * np.abs(want).max())


@pytest.mark.parametrize("name", list(FIXTURES))
def test_oracle_reproduces_fixture(name):
    inp = I.make_patterned(300, log_a=FIXTURES[name], dtype="f32")
    o = O.llattn_recurrent(inp).reshape(300, inp.H, inp.dv)
    rows = load(name)
    got = np.array([o[t, 0, j] for t, j, _ in rows])
    want = np.array([x for _, _, x in rows])
    assert O.rel_max_err(got, want) < 1e-12


def test_patterned_inputs_are_bf16_exact():
    inp = I.make_patterned(300, H=2)
    for x in (inp.q, inp.k, inp.v):
        assert np.array_equal(I.round_to_bf16(x), x)
    assert inp.lam.shape == (1, 300, 2, I.num_levels(300))
