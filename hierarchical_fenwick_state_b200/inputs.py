"""Seeded synthetic inputs for the log-linear attention forward.

This module draws random numbers and lays them out; it holds none of the
method's arithmetic (no decay products, no Fenwick levels, no attention).  It
is the one module shared by the CPU oracle (``oracle/``), the tests, the smoke
check and ``bench.py``, so that both sides see bit-identical inputs.

Workloads follow the value distributions the Log-Linear Attention pages assume
for the Mamba-2 form ("Log-Linear Mamba-2": a scalar selective gate a_t per
token and head, and per-level weights lambda): q and k are standard normal and
L2-normalised per (token, head) row over d_k, v is standard normal,
log a_t = -exp(N(mu, 0.5)) per (b, t, h), lambda = softplus(N(0, 1)) per
(b, t, h, level).  N(mu, sigma) means mean mu and standard deviation sigma.
Draw order is fixed: q, k, v, log_a, lambda, using numpy's ``default_rng``.

bf16 workloads are drawn in fp32 and rounded to bf16 (round to nearest even)
here, on the host, so the oracle computes on exactly the values the device
sees.  log_a and lambda stay fp32 in every workload.

Layouts (token-major, contiguous):
  q, k      [B, T, H, d_k]   (varlen: [total, H, d_k])
  v         [B, T, H, d_v]
  log_a     [B, T, H]
  lam       [B, T, H, L]     L = 1 + ceil(log2 T), level innermost
  cu_seqlens int32 [nseq + 1] for packed variable-length batches.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np


def num_levels(T: int) -> int:
    """Number of Fenwick levels for sequences of at most T tokens: 1 + ceil(log2 T).

    T = 1 gives 1 (only the token itself).  Level 0 is the token itself; level
    l >= 1 is a block of 2**(l-1) earlier tokens, the largest of which, for
    0-based positions below T, is l = ceil(log2 T).
    """
    if T <= 1:
        return 1
    return 1 + (T - 1).bit_length()


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int                 # batch (dense) or number of sequences (varlen)
    H: int
    T: int                 # sequence length (dense) or max length bound (varlen)
    dk: int
    dv: int
    dtype: str             # "bf16" or "f32" for q/k/v (log_a, lam always f32)
    log_a_mu: float = -2.0  # log a = -exp(N(log_a_mu, 0.5))
    varlen: bool = False
    len_lo: int = 0         # varlen: lengths ~ U[len_lo, len_hi] (integers)
    len_hi: int = 0

    @property
    def L(self) -> int:
        return num_levels(self.T)


# The five workloads of the log-linear Mamba-2 forward benchmark matrix.
WORKLOADS = {
    "t256_d32_f32": Workload("t256_d32_f32", B=1, H=2, T=256, dk=32, dv=32, dtype="f32"),
    "t2k_d64_bf16": Workload("t2k_d64_bf16", B=2, H=16, T=2048, dk=64, dv=64, dtype="bf16"),
    "t8k_d64_bf16": Workload("t8k_d64_bf16", B=4, H=32, T=8192, dk=64, dv=64, dtype="bf16"),
    "t64k_d128_bf16": Workload("t64k_d128_bf16", B=1, H=16, T=65536, dk=128, dv=128, dtype="bf16",
                               log_a_mu=-3.0),
    "varlen8_d64_bf16": Workload("varlen8_d64_bf16", B=8, H=16, T=16384, dk=64, dv=64, dtype="bf16",
                                 varlen=True, len_lo=1024, len_hi=16384),
}
HEADLINE = "t8k_d64_bf16"

# Smaller cases of the benchmark workloads for single-kernel profiler captures (inputs still
# larger than L2, a few hundred MB on the device); not part of the benchmark matrix.
PROFILE_WORKLOADS = {
    "t16k_d128_bf16_h8": Workload("t16k_d128_bf16_h8", B=1, H=8, T=16384, dk=128, dv=128,
                                  dtype="bf16", log_a_mu=-3.0),
    "t8k_d64_bf16_b1": Workload("t8k_d64_bf16_b1", B=1, H=32, T=8192, dk=64, dv=64, dtype="bf16"),
}

# Log-Linear Gated DeltaNet forward: the same shapes and distributions (log_a is log alpha),
# plus beta = sigmoid(N(0, 1)) per (token, head) from make_gdn_inputs.
GDN_WORKLOADS = {
    "gdn_t2k_d64_bf16": Workload("gdn_t2k_d64_bf16", B=2, H=16, T=2048, dk=64, dv=64,
                                 dtype="bf16"),
    "gdn_t8k_d64_bf16": Workload("gdn_t8k_d64_bf16", B=4, H=32, T=8192, dk=64, dv=64,
                                 dtype="bf16"),
}


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even); returns fp32 holding bf16 values."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounding = 0x7FFF + ((u >> 16) & 1)
    r = ((u + rounding) >> 16) << 16
    out = r.astype(np.uint32).view(np.float32)
    # NaN/Inf never occur in these draws; keep them untouched if they did.
    bad = ~np.isfinite(x)
    if bad.any():
        out = out.copy()
        out[bad] = x[bad]
    return out


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of fp32 arrays that already hold bf16 values."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def _softplus(x: np.ndarray) -> np.ndarray:
    return np.logaddexp(0.0, x)


def _l2_rows(x: np.ndarray) -> np.ndarray:
    n = np.sqrt(np.sum(x.astype(np.float64) ** 2, axis=-1, keepdims=True))
    return (x / n).astype(np.float32)


@dataclasses.dataclass
class Inputs:
    """Host arrays (fp32 storage; q/k/v hold bf16-exact values for bf16 workloads)."""
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    log_a: np.ndarray
    lam: np.ndarray
    cu_seqlens: Optional[np.ndarray]
    B: int
    H: int
    T: int
    dk: int
    dv: int
    dtype: str
    beta: Optional[np.ndarray] = None   # write strength of the gated delta rule, [..., H]

    @property
    def L(self) -> int:
        return self.lam.shape[-1]

    @property
    def total_tokens(self) -> int:
        if self.cu_seqlens is not None:
            return int(self.cu_seqlens[-1])
        return self.B * self.T

    def seq_slices(self):
        """(token_start, length) per sequence in the flattened [tokens] index space."""
        if self.cu_seqlens is not None:
            c = self.cu_seqlens
            return [(int(c[i]), int(c[i + 1] - c[i])) for i in range(len(c) - 1)]
        return [(b * self.T, self.T) for b in range(self.B)]


def varlen_lengths(w: Workload, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed + 7919)
    return rng.integers(w.len_lo, w.len_hi, size=w.B, endpoint=True).astype(np.int64)


def make_inputs(w: Workload, seed: int = 0, *, log_a_mode: str = "dist",
                lam_mode: str = "dist", lam_level: int = -1,
                lengths: Optional[np.ndarray] = None) -> Inputs:
    """Draw one seeded workload.

    log_a_mode: "dist" (the workload's -exp(N(mu, 0.5))), "zero" (no decay),
      "slow" (-exp(N(-7, 0.5))) or "strong" (-exp(N(1, 0.5)), far beyond fp32 range
      over a chunk, for the overflow guards).
    lam_mode: "dist" (softplus(N(0,1))), "ones", or "onehot" (1 at ``lam_level``,
      0 elsewhere).
    lengths: varlen sequence lengths (default: drawn from the workload's range).
    """
    if w.varlen:
        if lengths is None:
            lengths = varlen_lengths(w, seed)
        lengths = np.asarray(lengths, dtype=np.int64)
        cu = np.zeros(len(lengths) + 1, dtype=np.int32)
        cu[1:] = np.cumsum(lengths)
        lead = (int(cu[-1]),)
        B = len(lengths)
    else:
        cu = None
        lead = (w.B, w.T)
        B = w.B
    H, dk, dv, L = w.H, w.dk, w.dv, w.L
    rng = np.random.default_rng(seed)
    q = _l2_rows(rng.standard_normal(lead + (H, dk), dtype=np.float32))
    k = _l2_rows(rng.standard_normal(lead + (H, dk), dtype=np.float32))
    v = rng.standard_normal(lead + (H, dv), dtype=np.float32)
    z = rng.standard_normal(lead + (H,), dtype=np.float32)
    if log_a_mode == "dist":
        log_a = -np.exp(w.log_a_mu + 0.5 * z)
    elif log_a_mode == "zero":
        log_a = np.zeros_like(z)
    elif log_a_mode == "slow":
        log_a = -np.exp(-7.0 + 0.5 * z)
    elif log_a_mode == "strong":
        log_a = -np.exp(1.0 + 0.5 * z)
    else:
        raise ValueError(log_a_mode)
    zl = rng.standard_normal(lead + (H, L), dtype=np.float32)
    if lam_mode == "dist":
        lam = _softplus(zl)
    elif lam_mode == "ones":
        lam = np.ones_like(zl)
    elif lam_mode == "onehot":
        lam = np.zeros_like(zl)
        lam[..., lam_level] = 1.0
    else:
        raise ValueError(lam_mode)
    if w.dtype == "bf16":
        q, k, v = round_to_bf16(q), round_to_bf16(k), round_to_bf16(v)
    return Inputs(q=np.ascontiguousarray(q, np.float32), k=np.ascontiguousarray(k, np.float32),
                  v=np.ascontiguousarray(v, np.float32),
                  log_a=np.ascontiguousarray(log_a, np.float32),
                  lam=np.ascontiguousarray(lam, np.float32), cu_seqlens=cu,
                  B=B, H=H, T=w.T, dk=dk, dv=dv, dtype=w.dtype)


def _sigmoid(x: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-x))


def make_gdn_inputs(w: Workload, seed: int = 0, *, beta_mode: str = "dist",
                    **kw) -> Inputs:
    """The inputs of ``make_inputs`` (same seed, same draws; log_a is the gate log alpha) plus
    the delta rule's write strength beta per (token, head), from its own seeded stream:
    "dist" sigmoid(N(0, 1)), "ones" (beta = 1) or "zero"."""
    inp = make_inputs(w, seed, **kw)
    lead = inp.log_a.shape
    if beta_mode == "dist":
        z = np.random.default_rng(seed + 104729).standard_normal(lead, dtype=np.float32)
        beta = _sigmoid(z.astype(np.float64)).astype(np.float32)
    elif beta_mode == "ones":
        beta = np.ones(lead, np.float32)
    elif beta_mode == "zero":
        beta = np.zeros(lead, np.float32)
    else:
        raise ValueError(beta_mode)
    inp.beta = np.ascontiguousarray(beta)
    return inp


def make_patterned(T: int, *, H: int = 1, dk: int = 64, dv: int = 64, log_a: float = 0.0,
                   dtype: str = "bf16") -> Inputs:
    """Deterministic small-integer inputs given by closed forms, for the golden fixtures.

    q[t,h,i] = ((3t + 5i + h) mod 7) - 3,   k[t,h,i] = ((5t + 3i + 2h + 1) mod 7) - 3,
    v[t,h,j] = ((2t + 7j + h + 3) mod 5) - 2,
    log_a[t,h] = log_a (one constant),      lam[t,h,l] = 1 + ((t + 3l + h) mod 4) / 4.
    Every value is exact in bf16 and fp32 (log_a too when it is a short binary fraction), so
    the outputs can be known exactly and every dtype sees the same numbers.  One dense
    sequence (B = 1).
    """
    t = np.arange(T)[:, None, None]
    h = np.arange(H)[None, :, None]
    i = np.arange(dk)[None, None, :]
    j = np.arange(dv)[None, None, :]
    L = num_levels(T)
    lv = np.arange(L)[None, None, :]
    q = ((3 * t + 5 * i + h) % 7 - 3).astype(np.float32)[None]
    k = ((5 * t + 3 * i + 2 * h + 1) % 7 - 3).astype(np.float32)[None]
    v = ((2 * t + 7 * j + h + 3) % 5 - 2).astype(np.float32)[None]
    la = np.full((1, T, H), log_a, dtype=np.float32)
    lam = (1.0 + ((t + 3 * lv + h) % 4) / 4.0).astype(np.float32)[None]
    return Inputs(q=np.ascontiguousarray(q), k=np.ascontiguousarray(k),
                  v=np.ascontiguousarray(v), log_a=la, lam=np.ascontiguousarray(lam),
                  cu_seqlens=None, B=1, H=H, T=T, dk=dk, dv=dv, dtype=dtype)


def shrink(w: Workload, *, B: Optional[int] = None, H: Optional[int] = None,
           T: Optional[int] = None, len_lo: Optional[int] = None,
           len_hi: Optional[int] = None, name: Optional[str] = None) -> Workload:
    """Same distributions and head size, smaller extent (for oracle-sized parity cases)."""
    return dataclasses.replace(
        w, name=name or (w.name + "_small"), B=B if B is not None else w.B,
        H=H if H is not None else w.H, T=T if T is not None else w.T,
        len_lo=len_lo if len_lo is not None else w.len_lo,
        len_hi=len_hi if len_hi is not None else w.len_hi)


# ----------------------------------------------------------------------------
# Decoding step inputs: one new token per sequence, level states from earlier tokens
# ----------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    name: str
    B: int        # sequences decoded together (one token each per step)
    H: int
    L: int        # levels; positions stay below 2**(L-1)
    dk: int
    dv: int
    dtype: str    # "bf16" or "f32" for q/k/v
    log_a_mu: float = -2.0


# A serving-style batch: 64 sequences at positions spread over [0, 8192), H = 32, d = 64.
DECODE_WORKLOADS = {
    "decode_b64_h32_d64_bf16": DecodeWorkload("decode_b64_h32_d64_bf16", B=64, H=32, L=14,
                                              dk=64, dv=64, dtype="bf16"),
}


@dataclasses.dataclass
class DecodeInputs:
    """Host arrays for one decoding step (fp32 storage; q/k/v bf16-exact for bf16)."""
    q: np.ndarray          # [B, H, dk]
    k: np.ndarray          # [B, H, dk]
    v: np.ndarray          # [B, H, dv]
    log_a: np.ndarray      # [B, H]
    lam: np.ndarray        # [B, H, L]
    pos: np.ndarray        # int32 [B]
    states: np.ndarray     # [B, H, L-1, dk, dv]  level states before the step (every slot drawn)
    pending: np.ndarray    # [B, H, L-1]  a draw in [-3, 0] per slot, for splitting a state
    B: int
    H: int
    L: int
    dk: int
    dv: int
    dtype: str


def make_decode_inputs(w: DecodeWorkload, seed: int = 0, *, positions=None) -> DecodeInputs:
    """Draw one seeded decoding step.  Token inputs follow the forward's distributions; the
    positions are uniform integers in [0, 2**(L-1)) unless given; the level states are
    N(0, 0.3^2) per element (about the spread of a decayed sum of a few k v^T with unit k and
    standard normal v), drawn for every slot, occupied or not."""
    rng = np.random.default_rng(seed)
    B, H, L, dk, dv = w.B, w.H, w.L, w.dk, w.dv
    q = _l2_rows(rng.standard_normal((B, H, dk), dtype=np.float32))
    k = _l2_rows(rng.standard_normal((B, H, dk), dtype=np.float32))
    v = rng.standard_normal((B, H, dv), dtype=np.float32)
    log_a = -np.exp(w.log_a_mu + 0.5 * rng.standard_normal((B, H), dtype=np.float32))
    lam = _softplus(rng.standard_normal((B, H, L), dtype=np.float32))
    if positions is None:
        pos = rng.integers(0, 1 << (L - 1), size=B)
    else:
        pos = np.asarray(positions)
        assert pos.shape == (B,)
    states = 0.3 * rng.standard_normal((B, H, L - 1, dk, dv), dtype=np.float32)
    pending = -3.0 * rng.random((B, H, L - 1), dtype=np.float32)
    if w.dtype == "bf16":
        q, k, v = round_to_bf16(q), round_to_bf16(k), round_to_bf16(v)
    f = lambda x: np.ascontiguousarray(x, np.float32)  # noqa: E731
    return DecodeInputs(q=f(q), k=f(k), v=f(v), log_a=f(log_a), lam=f(lam),
                        pos=np.ascontiguousarray(pos, np.int32), states=f(states),
                        pending=f(pending), B=B, H=H, L=L, dk=dk, dv=dv, dtype=w.dtype)
