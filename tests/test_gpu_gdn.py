"""Log-Linear Gated DeltaNet on the GPU (llattn_gdn_fwd through the C ABI) against the oracle.

The kernel keeps the level states in fp32 and computes in fp32 on the exact input values,
so every case is held to 1e-4 of the output RMS (bf16 inputs included).  Cases: several
levels and ragged lengths, d_k and d_v of 32, 64 and 128, a packed batch with empty and
one-token sequences, one level at a time with no decay (the deep levels), write strength
beta = 1, and sampled outputs at B=2, H=16, T=8192.
"""
import numpy as np
import pytest

import oracle as O
from hierarchical_fenwick_state_b200 import binding
from hierarchical_fenwick_state_b200 import inputs as I

pytestmark = pytest.mark.gpu
TOL = 1e-4
W = I.WORKLOADS


def _run(inp):
    import torch
    dev = torch.device("cuda:0")
    dt = torch.bfloat16 if inp.dtype == "bf16" else torch.float32
    t = {n: torch.from_numpy(getattr(inp, n)).to(dev) for n in ("q", "k", "v", "log_a", "beta", "lam")}
    for n in ("q", "k", "v"):
        t[n] = t[n].to(dt)
    cu = torch.from_numpy(inp.cu_seqlens).to(dev) if inp.cu_seqlens is not None else None
    out = torch.full(inp.v.shape, float("nan"), dtype=torch.float32, device=dev)
    binding.device_status(clear=True)
    binding.gdn_forward(t["q"], t["k"], t["v"], t["log_a"], t["beta"], t["lam"], cu_seqlens=cu,
                        T=inp.T, out=out)
    torch.cuda.synchronize()
    assert binding.device_status(clear=True) == 0
    return out.double().cpu().numpy()


def _check(inp, ref=None):
    ref = O.gdn_recurrent(inp) if ref is None else ref
    got = _run(inp)
    assert np.isfinite(got).all(), "unwritten or non-finite outputs"
    err = O.rel_max_err(got, ref)
    assert err <= TOL, f"rel max err {err:.3e}"


CASES = {
    "t300_d64_bf16": (I.shrink(W["t2k_d64_bf16"], B=2, H=2, T=300), {}),
    "t2k_d64_bf16": (I.shrink(W["t2k_d64_bf16"], B=1, H=2, T=2048), {}),
    "t256_d32_f32": (W["t256_d32_f32"], {}),
    "t700_d128_bf16": (I.shrink(W["t64k_d128_bf16"], H=2, T=700), {}),
    "t2500_d32_f32": (I.Workload("gdn_t2500", B=1, H=2, T=2500, dk=32, dv=32, dtype="f32"), {}),
    "t500_beta1_slow": (I.shrink(W["t2k_d64_bf16"], B=1, H=3, T=500),
                        dict(beta_mode="ones", log_a_mode="slow")),
}


@pytest.mark.parametrize("name", list(CASES))
def test_gdn_matches_oracle(name):
    w, kw = CASES[name]
    _check(I.make_gdn_inputs(w, seed=41, **kw))


@pytest.mark.parametrize("dk,dv", [(32, 128), (128, 32), (64, 32)])
def test_gdn_mixed_head_dims(dk, dv):
    w = I.Workload("gdn_mixed", B=1, H=2, T=260, dk=dk, dv=dv, dtype="bf16")
    _check(I.make_gdn_inputs(w, seed=42))


@pytest.mark.parametrize("T", [1, 2, 33, 129])
def test_gdn_edge_lengths(T):
    _check(I.make_gdn_inputs(I.shrink(W["t2k_d64_bf16"], B=2, H=1, T=T), seed=T))


def test_gdn_packed_sequences():
    w = I.Workload("gdn_vl", B=5, H=2, T=900, dk=64, dv=64, dtype="bf16", varlen=True)
    _check(I.make_gdn_inputs(w, seed=43, lengths=np.array([900, 0, 1, 129, 512])))


@pytest.mark.parametrize("level", [1, 6, 11])
def test_gdn_one_hot_level(level):
    w = I.shrink(W["t2k_d64_bf16"], B=1, H=2, T=2048)
    _check(I.make_gdn_inputs(w, seed=44, log_a_mode="zero", lam_mode="onehot", lam_level=level))


def test_gdn_sampled_at_size():
    w = I.shrink(W["t8k_d64_bf16"], B=2, H=16)
    inp = I.make_gdn_inputs(w, seed=45)
    got = _run(inp).reshape(-1, inp.H, inp.dv)
    assert np.isfinite(got).all()
    rng = np.random.default_rng(46)
    toks = np.concatenate([rng.integers(0, inp.total_tokens, 40), [0, 8191, 8192, 16383]])
    samples = [(int(t), int(h)) for t, h in zip(toks, rng.integers(0, inp.H, len(toks)))]
    ref = O.gdn_sampled(inp, samples)
    err = O.rel_max_err(np.stack([got[t, h] for t, h in samples]), ref)
    assert err <= TOL, f"sampled rel max err {err:.3e}"


def test_gdn_deep_levels_long_sequence():
    """T = 20000 runs the instantiation that holds 17 levels: level 15 (the bucket of the first
    16384 tokens) alone weighs the output, sampled past position 16384."""
    w = I.Workload("gdn_long", B=1, H=2, T=20000, dk=32, dv=32, dtype="bf16")
    inp = I.make_gdn_inputs(w, seed=47, log_a_mode="slow", lam_mode="onehot", lam_level=15)
    got = _run(inp).reshape(-1, inp.H, inp.dv)
    assert np.isfinite(got).all()
    samples = [(t, h) for t in (16384, 16385, 17001, 19999) for h in range(inp.H)]
    ref = O.gdn_sampled(inp, samples)
    assert np.abs(ref).max() > 0.0
    err = O.rel_max_err(np.stack([got[t, h] for t, h in samples]), ref)
    assert err <= TOL, f"sampled rel max err {err:.3e}"
