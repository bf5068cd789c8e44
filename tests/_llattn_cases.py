"""Shared helpers for the GPU parity tests: device upload and one call through the C ABI."""
from __future__ import annotations

import numpy as np

from hierarchical_fenwick_state_b200 import binding
from hierarchical_fenwick_state_b200 import inputs as I

TOL = {"f32": 1e-4, "bf16": 2e-2}  # max |err| / RMS(ref), per input dtype


def to_device(inp: I.Inputs):
    import torch
    dt = torch.bfloat16 if inp.dtype == "bf16" else torch.float32
    dev = torch.device("cuda:0")
    t = {
        "q": torch.from_numpy(inp.q).to(dev).to(dt).contiguous(),
        "k": torch.from_numpy(inp.k).to(dev).to(dt).contiguous(),
        "v": torch.from_numpy(inp.v).to(dev).to(dt).contiguous(),
        "log_a": torch.from_numpy(inp.log_a).to(dev).contiguous(),
        "lam": torch.from_numpy(inp.lam).to(dev).contiguous(),
        "cu": (torch.from_numpy(inp.cu_seqlens).to(dev) if inp.cu_seqlens is not None else None),
    }
    return t


def run(inp: I.Inputs, path: str = "auto", chunk: int = 0, poison: bool = True):
    """Run the forward through llattn_fwd_ex; returns the fp32 output as float64 numpy."""
    import torch
    t = to_device(inp)
    out = torch.empty(inp.v.shape, dtype=torch.float32, device="cuda:0")
    if poison:
        out.fill_(float("nan"))
    binding.forward(t["q"], t["k"], t["v"], t["log_a"], t["lam"], cu_seqlens=t["cu"],
                    T=inp.T, out=out, path=path, chunk=chunk)
    torch.cuda.synchronize()
    assert binding.device_status(clear=True) == 0
    return out.double().cpu().numpy()
