"""Write the golden fixtures of this folder.  Only the CPU oracle computes here.

    python tests/golden/make_golden.py

Each fixture holds sampled outputs o[t, head 0, j] of the log-linear attention
forward (Mamba-2 form) for one of the closed-form inputs of
``inputs.make_patterned``.  The values come from the oracle's brute-force form,
which is the definition written out: "Log-Linear Attention" (gist.science),
Italian "Sommario tecnico" section 2, parts "Partizionamento Gerarchico (Fenwick
Tree)" and "Matrici Gerarchiche", and the Spanish "Resumen tecnico", "Variantes
Propuestas" item 1.  The quadratic and recurrent forms must agree with it before
anything is written.
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle as O  # noqa: E402
from hierarchical_fenwick_state_b200 import inputs as I  # noqa: E402

T = 300
TOKENS = [0, 1, 2, 3, 7, 63, 64, 65, 127, 128, 129, 191, 200, 255, 256, 257, 298, 299]
CASES = {
    # no decay: every output is a multiple of 1/4, computed exactly in fp64
    "patterned_nodecay_T300": 0.0,
    # a_t = exp(-1/8) per step: the gate reaches back ~200 tokens at 1e-11
    "patterned_decay8_T300": -0.125,
}


def write(name, log_a):
    inp = I.make_patterned(T, log_a=log_a, dtype="f32")
    bf = O.llattn_bruteforce(inp)
    qd = O.llattn_quadratic(inp)
    rc = O.llattn_recurrent(inp)
    assert O.rel_max_err(qd, bf) < 1e-12 and O.rel_max_err(rc, bf) < 1e-12
    o = bf.reshape(T, inp.H, inp.dv)
    path = os.path.join(HERE, name + ".txt")
    with open(path, "w") as f:
        f.write(f"# {name}: sampled outputs o[t, 0, j] of the log-linear attention forward\n")
        f.write("# (Mamba-2 form) for inputs.make_patterned(T=%d, H=1, dk=64, dv=64, "
                "log_a=%r).\n" % (T, log_a))
        f.write("# Definition: 'Log-Linear Attention' (gist.science), Italian 'Sommario tecnico'\n")
        f.write("# section 2 (Partizionamento Gerarchico, Matrici Gerarchiche) and Spanish\n")
        f.write("# 'Resumen tecnico', Variantes Propuestas item 1.  Written by make_golden.py\n")
        f.write("# from the fp64 oracle's brute-force form.  Columns: t j o\n")
        for t in TOKENS:
            for j in range(inp.dv):
                f.write(f"{t} {j} {float(o[t, 0, j])!r}\n")
    return path


if __name__ == "__main__":
    for name, la in CASES.items():
        print(write(name, la))
