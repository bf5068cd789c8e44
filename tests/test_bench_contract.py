"""bench.py's JSON line keeps its contract (CPU: the reference arm, which times the oracle)."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                        "--warmup", "1", "--workload", "t2k_d64_bf16"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "impl",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["higher_is_better"] is True and d["data"] == "synthetic"
    assert d["config"]["workload"] == "t2k_d64_bf16"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def _ref_line(*extra):
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                        "--warmup", "0", *extra], cwd=ROOT, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    return json.loads(lines[0])


def test_reference_arm_of_the_decoding_step_and_the_backward():
    d = _ref_line("--workload", "decode_b64_h32_d64_bf16")
    assert d["impl"] == "reference" and d["value"] > 0 and "decode" in d["metric"]
    assert d["config"]["workload"] == "decode_b64_h32_d64_bf16"
    b = _ref_line("--pass", "bwd", "--workload", "t2k_d64_bf16")
    assert b["impl"] == "reference" and b["value"] > 0 and "bwd" in b["metric"]
    assert b["config"]["pass"] == "bwd"


def test_decoding_bytes_counted_by_hand():
    """Two sequences with three level slots: position 5 (0b101: levels 1 and 3 occupied, one
    trailing one bit, so levels 0..1 carry into level 2) and position 7 (the last position a
    full counter holds: three levels read, no carry)."""
    import numpy as np
    sys.path.insert(0, ROOT)
    import bench
    from hierarchical_fenwick_state_b200 import inputs as I
    w = I.DecodeWorkload("t", B=2, H=3, L=4, dk=32, dv=64, dtype="bf16")
    d = I.make_decode_inputs(w, 0, positions=[5, 7])
    state = 4 * 32 * 64
    tok = (2 * 32 + 64) * 2 + 4 + 4 * 4 + 4 * 64
    # n = 5: two levels read, carry written (m = 1 < 3), gates: 2 read, popcount(6) = 2 written
    per5 = (2 + 1) * state + 4 * (2 + 2) + tok
    # n = 7: three levels read, no carry (m = 3), gates: 3 read, popcount(8 & 7) = 0 written
    per7 = 3 * state + 4 * 3 + tok
    assert bench.decode_algorithmic_bytes(d) == (per5 + per7) * 3 + 2 * 4
    assert np.array_equal(d.pos, [5, 7])


def test_backward_flops_counted_by_enumeration():
    """The level-by-level FLOP count equals a direct enumeration of the pairs and blocks."""
    sys.path.insert(0, ROOT)
    import bench
    from hierarchical_fenwick_state_b200 import inputs as I
    w = I.Workload("t", B=1, H=2, T=300, dk=8, dv=8, dtype="f32")
    lengths = [300, 37]
    _, flops, per = bench.bwd_algorithmic(w, lengths)
    d = 8
    want = 0
    for n in lengths:
        for t in range(n):                       # causal pairs inside aligned 32-token tiles
            want += sum(1 for s in range(t + 1) if s // 32 == t // 32) * 10 * d
        for lvl in range(6, w.L):                # blocks with both halves present
            half = 1 << (lvl - 1)
            for lo in range(0, n, 2 * half):
                left = [t for t in range(lo, min(lo + half, n))]
                right = [t for t in range(lo + half, min(lo + 2 * half, n))]
                if right:
                    want += len(left) * 6 * d * d + len(right) * 4 * d * d
    assert flops == want * w.H
    assert per == (2 * 8 + 2 * 8) * 4 + 4 + 4 * w.L + (2 * 8 + 8) * 4 + 4 + 4 * w.L
