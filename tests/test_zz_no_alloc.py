"""llattn_fwd_noalloc against the allocating entry point, through the C ABI.

llattn_fwd_noalloc runs the CUDA-core kernels with their scratch taken from a
fixed 32 MiB array in the library instead of an allocation.  The GPU test makes
two no-allocation calls in a row, the second one smaller, so that any state the
first call left in the shared array would show up, then checks both outputs,
bit for bit, against llattn_fwd_ex on the same path with the library's own
buffer.  It also checks the smaller case against the oracle.  The file is named
so that it is collected last: it has to pass on its own in a fresh process and
after every other test has used the allocating entry points.
"""
import ctypes

import numpy as np
import pytest

import oracle as O
from hierarchical_fenwick_state_b200 import binding
from hierarchical_fenwick_state_b200 import inputs as I

from _llattn_cases import TOL, to_device

W = I.WORKLOADS
LIMIT_STATUS = 9  # LLATTN_ERR_NOALLOC_LIMIT


def _noalloc_raw(in_dtype, B, H, T, dk, dv):
    vp = ctypes.c_void_p
    return binding.lib().llattn_fwd_noalloc(in_dtype, vp(0x1000), vp(0x2000), vp(0x3000),
                                            vp(0x4000), vp(0x5000), vp(0x6000), B, H, T, dk, dv,
                                            None, None)


def test_limit_is_reported_without_cuda():
    w = W["t8k_d64_bf16"]
    need = binding.workspace_bytes(binding.BF16, "simt", 0, w.B, w.H, w.T, w.dk, w.dv, False)
    assert need > binding.NOALLOC_SCRATCH_BYTES
    assert _noalloc_raw(binding.BF16, w.B, w.H, w.T, w.dk, w.dv) == LIMIT_STATUS
    assert b"fixed array" in binding.lib().llattn_status_str(LIMIT_STATUS)
    # shape errors keep their own code
    assert _noalloc_raw(binding.BF16, 1, 1, 64, 48, 64) == 2
    # empty problems are no-ops that touch nothing
    assert _noalloc_raw(binding.BF16, 0, 4, 64, 64, 64) == 0


def test_oracle_sized_workloads_fit():
    for name in ("t256_d32_f32", "t2k_d64_bf16"):
        w = W[name]
        dt = binding.BF16 if w.dtype == "bf16" else binding.F32
        need = binding.workspace_bytes(dt, "simt", 0, w.B, w.H, w.T, w.dk, w.dv, w.varlen)
        assert 0 < need <= binding.NOALLOC_SCRATCH_BYTES, name


@pytest.mark.gpu
def test_noalloc_matches_allocating_entry_point_on_two_calls_in_a_row():
    import torch

    first = I.make_inputs(W["t2k_d64_bf16"], seed=21)  # 31.5 MiB of the 32 MiB array
    second = I.make_inputs(I.shrink(W["varlen8_d64_bf16"], H=2, T=3000, len_lo=1, len_hi=3000),
                           seed=22)
    dev = [to_device(x) for x in (first, second)]
    got = []
    for inp, t in zip((first, second), dev):
        out = torch.full(inp.v.shape, float("nan"), dtype=torch.float32, device="cuda:0")
        B = inp.B if inp.cu_seqlens is None else len(inp.cu_seqlens) - 1
        binding.fwd_noalloc(t["q"], t["k"], t["v"], t["log_a"], t["lam"], out, B, inp.H, inp.T,
                            inp.dk, inp.dv, cu_seqlens=t["cu"])
        got.append(out)
    torch.cuda.synchronize()
    assert binding.device_status(clear=True) == 0

    for inp, t, out in zip((first, second), dev, got):
        ref = binding.forward(t["q"], t["k"], t["v"], t["log_a"], t["lam"], cu_seqlens=t["cu"],
                              T=inp.T, path="simt")
        torch.cuda.synchronize()
        assert torch.isfinite(out).all(), "rows left unwritten"
        assert torch.equal(out, ref), f"max |diff| {(out - ref).abs().max().item():.3e}"
    assert binding.device_status(clear=True) == 0

    want = O.llattn_recurrent(second)
    err = O.rel_max_err(got[1].double().cpu().numpy(), want)
    assert err <= TOL["bf16"], f"rel max err {err:.3e}"
