"""Decoding step on the GPU (llattn_decode_step through the C ABI) against the oracle.

Three kinds of case:
  * whole sequences decoded token by token from a state buffer full of NaN (nothing is
    cleared, positions alone say which slots hold a level), checked against the oracle's
    recurrent form over every output;
  * one step from given level states at deep and edge positions (0, 1, 2^12 - 1, the last
    position a full counter holds, ...), each state split into a stored part and a pending
    gate, checked against the oracle's decoding step for the output and every level that
    stays or becomes occupied;
  * positions outside the range: the row is left untouched and the device status word says so.
The step computes in fp32 on the exact input values, so the bound is 1e-4 of the output RMS
for bf16 inputs too.
"""
import numpy as np
import pytest

import oracle as O
from hierarchical_fenwick_state_b200 import binding
from hierarchical_fenwick_state_b200 import inputs as I

pytestmark = pytest.mark.gpu
TOL = 1e-4
DECODE_POS = 8  # LLATTN_DEV_DECODE_POS


def _dev(x, dtype=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x)).to("cuda:0")
    return t.to(dtype) if dtype is not None else t


def _state_buffer(B, H, L, dk, dv, fill=float("nan")):
    """The caller's state buffer and its two views (levels, gate)."""
    import torch
    n = binding.decode_state_bytes(B, H, L, dk, dv) // 4
    buf = torch.full((n,), fill, dtype=torch.float32, device="cuda:0")
    nlev = B * H * (L - 1) * dk * dv
    return buf, buf[:nlev].view(B, H, L - 1, dk, dv), buf[nlev:].view(B, H, 2, L - 1)


@pytest.mark.parametrize("name,T,dtype", [
    ("t2k_d64_bf16", 300, "bf16"),
    ("t256_d32_f32", 256, "f32"),
    ("t64k_d128_bf16", 130, "bf16"),
])
def test_decoding_whole_sequences_matches_oracle(name, T, dtype):
    import torch
    w = I.shrink(I.WORKLOADS[name], B=3, H=2, T=T)
    inp = I.make_inputs(w, seed=11, log_a_mode="slow")
    ref = O.llattn_recurrent(inp)                     # [B, T, H, dv]
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    q, k, v = (_dev(x, tdt) for x in (inp.q, inp.k, inp.v))
    la, lam = _dev(inp.log_a), _dev(inp.lam)
    B, H, L, dk, dv = inp.B, inp.H, inp.L, inp.dk, inp.dv
    buf, _, _ = _state_buffer(B, H, L, dk, dv)
    pos = torch.zeros(B, dtype=torch.int32, device="cuda:0")
    out = torch.empty((B, H, dv), dtype=torch.float32, device="cuda:0")
    got = torch.empty((B, T, H, dv), dtype=torch.float32, device="cuda:0")
    binding.device_status(clear=True)
    for n in range(T):
        pos.fill_(n)
        binding.decode_step(q[:, n].contiguous(), k[:, n].contiguous(), v[:, n].contiguous(),
                            la[:, n].contiguous(), lam[:, n].contiguous(), pos, buf, out,
                            B, H, L, dk, dv)
        got[:, n] = out
    torch.cuda.synchronize()
    assert binding.device_status(clear=True) == 0
    g = got.double().cpu().numpy()
    assert np.isfinite(g).all()
    err = O.rel_max_err(g, ref)
    assert err <= TOL, f"rel max err {err:.3e}"


def _one_step(d: I.DecodeInputs):
    """Upload a decoding step with its states split into stored part x pending gate; run it;
    return (out, levels, gate) on the host."""
    import torch
    B, H, L, dk, dv = d.B, d.H, d.L, d.dk, d.dv
    tdt = torch.bfloat16 if d.dtype == "bf16" else torch.float32
    buf, lev, gate = _state_buffer(B, H, L, dk, dv)
    occ = np.zeros((B, L - 1), bool)
    for b in range(B):
        occ[b] = [(int(d.pos[b]) >> j) & 1 for j in range(L - 1)]
    stored = d.states * np.exp(-d.pending)[..., None, None]        # fp32, in one pass
    for b in range(B):
        stored[b][:, ~occ[b]] = np.nan                             # empty slots hold NaN
    g = np.full((B, H, 2, L - 1), np.nan, np.float32)
    for b in range(B):
        g[b, :, int(d.pos[b]) & 1] = d.pending[b]
    lev.copy_(_dev(stored))
    gate.copy_(_dev(g))
    out = torch.full((B, H, dv), float("nan"), dtype=torch.float32, device="cuda:0")
    binding.device_status(clear=True)
    binding.decode_step(_dev(d.q, tdt), _dev(d.k, tdt), _dev(d.v, tdt), _dev(d.log_a),
                        _dev(d.lam), _dev(d.pos), buf, out, B, H, L, dk, dv)
    torch.cuda.synchronize()
    status = binding.device_status(clear=True)
    return status, out.double().cpu().numpy(), lev.double().cpu().numpy(), \
        gate.double().cpu().numpy()


def _check_step(d, out, lev, gate, pairs):
    """Output and new level states of the (b, h) pairs against the oracle's decoding step."""
    L = d.L
    o_ref, o_got, s_ref, s_got = [], [], [], []
    for b, h in pairs:
        n = int(d.pos[b])
        o, S1 = O.llattn_decode_step(d.states[b, h], n, d.q[b, h], d.k[b, h], d.v[b, h],
                                     d.log_a[b, h], d.lam[b, h])
        o_ref.append(o)
        o_got.append(out[b, h])
        for j in range(L - 1):
            if ((n + 1) >> j) & 1:
                s_ref.append(S1[j])
                s_got.append(np.exp(gate[b, h, (n + 1) & 1, j]) * lev[b, h, j])
    err = O.rel_max_err(np.array(o_got), np.array(o_ref))
    assert err <= TOL, f"output rel max err {err:.3e}"
    if s_ref:
        err = O.rel_max_err(np.array(s_got), np.array(s_ref))
        assert err <= TOL, f"state rel max err {err:.3e}"


@pytest.mark.parametrize("dtype,dk,dv", [("bf16", 64, 64), ("f32", 32, 128), ("bf16", 128, 32)])
def test_one_step_at_deep_and_edge_positions(dtype, dk, dv):
    L = 14
    positions = [0, 1, 2, 3, 4095, 4096, 5000, 8190, 8191]
    w = I.DecodeWorkload("edge", B=len(positions), H=3, L=L, dk=dk, dv=dv, dtype=dtype)
    d = I.make_decode_inputs(w, seed=dk + dv, positions=positions)
    status, out, lev, gate = _one_step(d)
    assert status == 0
    assert np.isfinite(out).all()
    _check_step(d, out, lev, gate, [(b, h) for b in range(d.B) for h in range(d.H)])


def test_one_step_at_the_benchmark_size_sampled():
    """The launch configuration the benchmark times (64 sequences, H = 32, d = 64, positions
    spread over [0, 8192)); the oracle checks 96 sampled (sequence, head) pairs."""
    d = I.make_decode_inputs(I.DECODE_WORKLOADS["decode_b64_h32_d64_bf16"], seed=5)
    status, out, lev, gate = _one_step(d)
    assert status == 0
    assert np.isfinite(out).all()
    rng = np.random.default_rng(0)
    pairs = list(zip(rng.integers(0, d.B, 96), rng.integers(0, d.H, 96)))
    _check_step(d, out, lev, gate, pairs)


def test_position_out_of_range_leaves_the_row_untouched():
    import torch
    L = 6                                     # positions 0..31
    positions = [32, 5, -1, 31]
    w = I.DecodeWorkload("bad", B=4, H=2, L=L, dk=64, dv=64, dtype="bf16")
    d = I.make_decode_inputs(w, seed=3, positions=positions)
    buf, lev, gate = _state_buffer(d.B, d.H, L, 64, 64, fill=0.25)
    before = buf.clone()
    out = torch.full((d.B, d.H, 64), 7.0, dtype=torch.float32, device="cuda:0")
    binding.device_status(clear=True)
    binding.decode_step(_dev(d.q, torch.bfloat16), _dev(d.k, torch.bfloat16),
                        _dev(d.v, torch.bfloat16), _dev(d.log_a), _dev(d.lam), _dev(d.pos), buf,
                        out, d.B, d.H, L, 64, 64)
    torch.cuda.synchronize()
    assert binding.device_status(clear=True) & DECODE_POS
    o = out.cpu().numpy()
    assert (o[0] == 7.0).all() and (o[2] == 7.0).all()
    assert np.isfinite(o[1]).all() and not (o[1] == 7.0).all()
    lv_b, lv_a = before[:lev.numel()].view(lev.shape), lev
    g_b = before[lev.numel():].view(gate.shape)
    for b in (0, 2):
        assert torch.equal(lv_b[b], lv_a[b]) and torch.equal(g_b[b], gate[b])
    assert binding.device_status(clear=True) == 0
