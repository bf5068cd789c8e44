"""A prompt's hand-off to decoding (llattn_prefill_state through the C ABI) against the oracle.

  * the level states of every (sequence, head) at the position equal to its length, dense and
    packed, against the oracle's level-state definition (the Fenwick buckets of that position,
    gated to just before it), read as exp(gate) * slot in fp64; both gate rows agree, and levels
    without a bucket get gate 0 and keep what their slot held;
  * the continuation: after the prompt's state, decode_step over the next tokens gives the
    oracle's recurrent outputs of prompt + continuation at those positions, from a state buffer
    that started full of NaN;
  * a length the slots cannot hold leaves the state untouched and sets the status bit;
  * full size: the t8k_d64_bf16 shape (32 heads) with lengths 8192, 8191, 5000 and 1, sampled
    heads against the oracle.
The state is summed in fp32 from the exact input values, so the bound is 1e-4 of the slot's RMS
for bf16 inputs too (the same as the decoding step's).
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
    import torch
    n = binding.decode_state_bytes(B, H, L, dk, dv) // 4
    buf = torch.full((n,), fill, dtype=torch.float32, device="cuda:0")
    nlev = B * H * (L - 1) * dk * dv
    return buf, buf[:nlev].view(B, H, L - 1, dk, dv), buf[nlev:].view(B, H, 2, L - 1)


def _tdt(dtype):
    import torch
    return torch.bfloat16 if dtype == "bf16" else torch.float32


def _check_states(inp, levels, gate, L, heads=None):
    """Compare the occupied slots of every sequence (and the given heads) with the oracle.

    The slot is the oracle's level state with the decay after the bucket taken out (log_a set
    to 0 from the bucket's end on: the same definition, nothing pending), and the gate is that
    decay, sum of log_a over the tokens after the bucket, in fp64.  The gate's bound is that of
    fp32 recursive summation, u * (additions per term) * sum |log_a|, with at most
    ceil(m / 256) + 9 additions per term for m terms over 256 threads (a strided per-thread
    sum, then two tree reductions).  Where the whole state is representable, exp(gate) * slot
    is also compared with the oracle's state itself.
    """
    nslot = L - 1
    lv = levels.double().cpu().numpy()
    gt = gate.double().cpu().numpy()
    assert np.array_equal(gt[:, :, 0], gt[:, :, 1]), "both gate rows hold the pending gate"
    for b, (s0, n) in enumerate(inp.seq_slices()):
        for h in (range(inp.H) if heads is None else heads):
            if inp.cu_seqlens is not None:
                k, v, la = inp.k[s0:s0 + n, h], inp.v[s0:s0 + n, h], inp.log_a[s0:s0 + n, h]
            else:
                k, v, la = inp.k[b, :n, h], inp.v[b, :n, h], inp.log_a[b, :n, h]
            ref = O.llattn_level_states(k, v, la, n, nslot)
            for j in range(nslot):
                where = f"seq {b} (n={n}) head {h} level {j + 1}"
                if not (n >> j) & 1:
                    assert gt[b, h, 0, j] == 0.0, where
                    assert np.all(np.isnan(lv[b, h, j])), f"{where}: slot written"
                    continue
                hi = ((n >> (j + 1)) << (j + 1)) + (1 << j)     # end of the bucket
                after = np.asarray(la[hi:n], np.float64)
                la0 = np.array(la, np.float64)
                la0[hi:] = 0.0
                slot = O.llattn_level_states(k, v, la0, n, nslot)[j]
                err = O.rel_max_err(lv[b, h, j], slot)
                assert err <= TOL, f"{where}: slot {err:.3e}"
                g_tol = 2.0 ** -24 * (-(-after.size // 256) + 9) * np.abs(after).sum() + 1e-12
                assert abs(gt[b, h, 0, j] - after.sum()) <= g_tol, where
                if after.sum() > -60.0:
                    err = O.rel_max_err(np.exp(gt[b, h, n & 1, j]) * lv[b, h, j], ref[j])
                    assert err <= TOL, f"{where}: state {err:.3e}"


@pytest.mark.parametrize("T,dk,dv,dtype,mode", [
    (37, 64, 64, "bf16", "dist"),
    (300, 32, 128, "f32", "slow"),
    (1023, 128, 64, "bf16", "dist"),
    (1024, 64, 32, "f32", "slow"),
    (64, 128, 128, "bf16", "zero"),
    (1, 64, 64, "bf16", "dist"),
])
def test_dense_prompt_states_match_oracle(T, dk, dv, dtype, mode):
    import torch
    w = I.Workload("pf", B=3, H=2, T=T, dk=dk, dv=dv, dtype=dtype)
    inp = I.make_inputs(w, seed=T + dk, log_a_mode=mode)
    L = I.num_levels(T + 1)   # slots for position T
    buf, levels, gate = _state_buffer(inp.B, inp.H, L, dk, dv)
    k, v = _dev(inp.k, _tdt(dtype)), _dev(inp.v, _tdt(dtype))
    binding.device_status(clear=True)
    binding.prefill_state(k, v, _dev(inp.log_a), buf, inp.B, inp.H, T, L, dk, dv)
    torch.cuda.synchronize()
    assert binding.device_status(clear=True) == 0
    _check_states(inp, levels, gate, L)


def test_packed_prompt_states_match_oracle():
    import torch
    lengths = np.array([0, 1, 37, 256, 1000, 511])
    w = I.Workload("pfv", B=len(lengths), H=3, T=1024, dk=64, dv=64, dtype="bf16", varlen=True)
    inp = I.make_inputs(w, seed=5, lengths=lengths)
    L = I.num_levels(1025)
    buf, levels, gate = _state_buffer(inp.B, inp.H, L, 64, 64)
    binding.device_status(clear=True)
    binding.prefill_state(_dev(inp.k, torch.bfloat16), _dev(inp.v, torch.bfloat16),
                          _dev(inp.log_a), buf, inp.B, inp.H, 1024, L, 64, 64,
                          cu_seqlens=_dev(inp.cu_seqlens))
    torch.cuda.synchronize()
    assert binding.device_status(clear=True) == 0
    _check_states(inp, levels, gate, L)


@pytest.mark.parametrize("P,K,dk,dv,dtype", [
    (100, 40, 64, 64, "bf16"),
    (255, 3, 32, 128, "f32"),
    (512, 33, 128, 128, "bf16"),
])
def test_decoding_continues_the_prompt(P, K, dk, dv, dtype):
    """Prompt of P tokens through the hand-off, then K decoding steps: the outputs at positions
    P .. P+K-1 are the oracle's for the whole sequence."""
    import torch
    T = P + K
    w = I.Workload("pfc", B=2, H=3, T=T, dk=dk, dv=dv, dtype=dtype)
    inp = I.make_inputs(w, seed=P, log_a_mode="slow")
    ref = O.llattn_recurrent(inp)[:, P:]                # [B, K, H, dv]
    tdt = _tdt(dtype)
    q, k, v = (_dev(x, tdt) for x in (inp.q, inp.k, inp.v))
    la, lam = _dev(inp.log_a), _dev(inp.lam)
    B, H, L = inp.B, inp.H, inp.L
    buf, _, _ = _state_buffer(B, H, L, dk, dv)
    binding.device_status(clear=True)
    binding.prefill_state(k[:, :P].contiguous(), v[:, :P].contiguous(), la[:, :P].contiguous(),
                          buf, B, H, P, L, dk, dv)
    pos = torch.full((B,), P, dtype=torch.int32, device="cuda:0")
    out = torch.empty((B, H, dv), dtype=torch.float32, device="cuda:0")
    got = torch.empty((B, K, H, dv), dtype=torch.float32, device="cuda:0")
    for i in range(K):
        n = P + i
        pos.fill_(n)
        binding.decode_step(q[:, n].contiguous(), k[:, n].contiguous(), v[:, n].contiguous(),
                            la[:, n].contiguous(), lam[:, n].contiguous(), pos, buf, out,
                            B, H, L, dk, dv)
        got[:, i] = out
    torch.cuda.synchronize()
    assert binding.device_status(clear=True) == 0
    g = got.double().cpu().numpy()
    assert np.isfinite(g).all()
    err = O.rel_max_err(g, ref)
    assert err <= TOL, f"rel max err {err:.3e}"


def test_length_beyond_the_slots_leaves_the_state():
    import torch
    lengths = np.array([5, 8, 3])          # L = 4: three slots hold positions below 8
    w = I.Workload("pfx", B=3, H=2, T=8, dk=32, dv=32, dtype="f32", varlen=True)
    inp = I.make_inputs(w, seed=9, lengths=lengths)
    L = 4
    buf, levels, gate = _state_buffer(inp.B, inp.H, L, 32, 32, fill=7.0)
    binding.device_status(clear=True)
    binding.prefill_state(_dev(inp.k), _dev(inp.v), _dev(inp.log_a), buf, inp.B, inp.H, 8, L,
                          32, 32, cu_seqlens=_dev(inp.cu_seqlens))
    torch.cuda.synchronize()
    assert binding.device_status(clear=True) & DECODE_POS
    assert torch.all(levels[1] == 7.0) and torch.all(gate[1] == 7.0)
    assert torch.all(gate[0] != 7.0) and torch.all(gate[2] != 7.0)


def test_full_size_prompts_sampled_heads():
    """The 8192-token, 32-head, d = 64 bf16 shape: one full-counter length (a single bucket of
    all 8192 tokens), one with thirteen buckets, and two others; four heads checked."""
    import torch
    lengths = np.array([8192, 8191, 5000, 1])
    w = I.Workload("pff", B=4, H=32, T=8192, dk=64, dv=64, dtype="bf16", varlen=True)
    inp = I.make_inputs(w, seed=21, lengths=lengths)
    L = I.num_levels(8193)
    buf, levels, gate = _state_buffer(inp.B, inp.H, L, 64, 64)
    binding.device_status(clear=True)
    binding.prefill_state(_dev(inp.k, torch.bfloat16), _dev(inp.v, torch.bfloat16),
                          _dev(inp.log_a), buf, inp.B, inp.H, 8192, L, 64, 64,
                          cu_seqlens=_dev(inp.cu_seqlens))
    torch.cuda.synchronize()
    assert binding.device_status(clear=True) == 0
    _check_states(inp, levels, gate, L, heads=(0, 5, 13, 31))
