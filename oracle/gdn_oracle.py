"""CPU fp64 oracle for the Log-Linear Gated DeltaNet forward.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference arm may import or run this module.  It
shares no code with the CUDA path and imports nothing from it.

What is computed.  Log-Linear Attention (gist.science summaries, Italian
"Sommario tecnico" section 2, "Generalizzazione"; Spanish "Resumen tecnico",
"Variantes Propuestas" item 2) applies the hierarchical Fenwick structure to the
gated delta rule ("la regla delta con puertas").  The pages print no formula for
it, so this module takes the plainest reading that the rest of the pages fix:

  * the gated delta rule (Gated DeltaNet) keeps one d_k x d_v state with
        S_t = A_t S_{t-1} + beta_t k_t v_t^T,   A_t = alpha_t (I - beta_t k_t k_t^T),
        o_t = S_t^T q_t;
    unrolled, S_t = sum_{s<=t} (A_t A_{t-1} ... A_{s+1}) beta_s k_s v_s^T, so
        o_t = sum_{s<=t} beta_s (q_t^T A_t ... A_{s+1} k_s) v_s;
  * the log-linear version keeps, as for Mamba-2, one such state per Fenwick
    level (section 2, "Forma Ricorrente e Parallelizzata", decoding bullet): every
    occupied level state takes the same transition A_t, the new token's write
    beta_t k_t v_t^T opens level 0, the output weights level l by lam[t, l], and
    levels merge on promotion like a binary counter.  Written out,
        o_t = sum_{s<=t} lam[t, l(t,s)] beta_s (q_t^T A_t A_{t-1} ... A_{s+1} k_s) v_s,
    with l(t, s) the Fenwick level of the Mamba-2 form (0 if s == t, else
    1 + floor(log2(t XOR s))), alpha_t = exp(log_alpha[t]).

With A_t = a_t I (beta_t k_t k_t^T dropped) this is exactly Log-Linear Mamba-2 with
v_s scaled by beta_s; with orthonormal keys it reduces to that as well, since
(I - beta_r k_r k_r^T) k_s = k_s for r != s.  With lam == 1 it is plain Gated
DeltaNet.  Those reductions are the pins (tests/test_oracle_gdn_pins.py).

Forms (each cites the passage it follows):
  * ``gdn_bruteforce_seq`` - the unrolled sum with the explicit product of the
    transition matrices, per pair (tiny T).
  * ``gdn_recurrent_seq``  - one state per Fenwick level, all taking A_t, merged on
    promotion ("Forma Ricorrente"); no level function, no matrix products over pairs.
  * ``gated_deltanet_seq`` - plain Gated DeltaNet (one state), for the lam == 1 pin.
  * ``gdn_single``         - one output o_t by the unrolled sum, for sampled checks.

Parity status: every function here is pinned by tests that do not retype its
formula: brute force = recurrent on T <= 16, the orthonormal-key reduction to the
Mamba-2 oracle, the lam == 1 reduction to plain Gated DeltaNet, the delta rule's
overwrite property, one-hot levels summing to lam == 1, linearity in v and causality.
"""
from __future__ import annotations

import numpy as np

from .llattn_oracle import fenwick_level

F64 = np.float64


def _transition_apply(alpha, beta, k, x):
    """A x = alpha (x - beta k (k^T x)) for a vector or a d_k x n matrix x."""
    return alpha * (x - beta * np.outer(k, k @ x)) if x.ndim == 2 else alpha * (x - beta * k * (k @ x))


# ----------------------------------------------------------------------------
# Brute force: the unrolled sum with explicit transition products (tiny T)
# ----------------------------------------------------------------------------
def gdn_bruteforce_seq(q, k, v, log_alpha, beta, lam):
    """One sequence, one head.  q,k [T,dk]; v [T,dv]; log_alpha, beta [T]; lam [T,L] -> [T,dv].

    For every pair s <= t the matrix P = A_t A_{t-1} ... A_{s+1} (identity at s = t) is
    formed explicitly, A_r = alpha_r (I - beta_r k_r k_r^T), and
    o_t += lam[t, l(t,s)] * beta_s * (q_t^T P k_s) * v_s.
    """
    q = np.asarray(q, F64); k = np.asarray(k, F64); v = np.asarray(v, F64)
    alpha = np.exp(np.asarray(log_alpha, F64))
    beta = np.asarray(beta, F64)
    lam = np.asarray(lam, F64)
    T, dk = q.shape
    eye = np.eye(dk)
    o = np.zeros((T, v.shape[1]), F64)
    for t in range(T):
        for s in range(t + 1):
            P = eye.copy()
            for r in range(t, s, -1):          # P = A_t ... A_{s+1}
                A = alpha[r] * (eye - beta[r] * np.outer(k[r], k[r]))
                P = P @ A
            score = float(q[t] @ P @ k[s])
            o[t] += lam[t, fenwick_level(t, s)] * beta[s] * score * v[s]
    return o


# ----------------------------------------------------------------------------
# Recurrent form: one state per Fenwick level, each taking the gated delta transition
# ----------------------------------------------------------------------------
def gdn_recurrent_seq(q, k, v, log_alpha, beta, lam):
    """Sequences batched along axis 0: q,k [N,T,dk]; v [N,T,dv]; log_alpha, beta [N,T];
    lam [N,T,L] -> o [N,T,dv].

    Level states S_0..S_{L-1} (d_k x d_v).  For t = 0..T-1:
      1. every non-empty S_l (l >= 1) becomes A_t S_l = alpha_t (S_l - beta_t k_t (k_t^T S_l));
      2. S_0 = beta_t k_t v_t^T;
      3. o_t = sum over non-empty l of lam[t, l] * S_l^T q_t;
      4. promotion: with m = number of trailing one bits of t, S_{m+1} = S_0 + ... + S_m and
         levels 0..m become empty; skipped after the last token.
    """
    q = np.asarray(q, F64); k = np.asarray(k, F64); v = np.asarray(v, F64)
    alpha = np.exp(np.asarray(log_alpha, F64))
    beta = np.asarray(beta, F64)
    lam = np.asarray(lam, F64)
    N, T, dk = q.shape
    dv = v.shape[2]
    L = lam.shape[2]
    nlev = max(L, 1 + max(T - 1, 1).bit_length())
    S = np.zeros((N, nlev, dk, dv), F64)
    live = np.zeros(nlev, bool)
    o = np.zeros((N, T, dv), F64)
    for t in range(T):
        idx = np.nonzero(live)[0]
        idx = idx[idx >= 1]
        if idx.size:
            kt = k[:, t]                                            # [N, dk]
            proj = np.einsum("nd,nlde->nle", kt, S[:, idx])         # k^T S_l  [N, l, dv]
            S[:, idx] -= beta[:, t][:, None, None, None] * kt[:, None, :, None] * proj[:, :, None, :]
            S[:, idx] *= alpha[:, t][:, None, None, None]
        S[:, 0] = beta[:, t][:, None, None] * k[:, t, :, None] * v[:, t, None, :]
        live[0] = True
        idx = np.nonzero(live)[0]
        r = np.einsum("nd,nlde->nle", q[:, t], S[:, idx])
        o[:, t] = np.einsum("nl,nle->ne", lam[:, t, idx], r)
        if t == T - 1:
            break
        m = 0
        while (t >> m) & 1:
            m += 1
        S[:, m + 1] = S[:, : m + 1].sum(axis=1)
        S[:, : m + 1] = 0.0
        live[: m + 1] = False
        live[m + 1] = True
    return o


# ----------------------------------------------------------------------------
# Plain Gated DeltaNet (one state), for the lam == 1 reduction
# ----------------------------------------------------------------------------
def gated_deltanet_seq(q, k, v, log_alpha, beta):
    """S_t = alpha_t (S_{t-1} - beta_t k_t (k_t^T S_{t-1})) + beta_t k_t v_t^T, o_t = S_t^T q_t;
    batched like gdn_recurrent_seq."""
    q = np.asarray(q, F64); k = np.asarray(k, F64); v = np.asarray(v, F64)
    alpha = np.exp(np.asarray(log_alpha, F64))
    beta = np.asarray(beta, F64)
    N, T, dk = q.shape
    S = np.zeros((N, dk, v.shape[2]), F64)
    o = np.zeros((N, T, v.shape[2]), F64)
    for t in range(T):
        kt = k[:, t]
        S = S - beta[:, t][:, None, None] * kt[:, :, None] * np.einsum("nd,nde->ne", kt, S)[:, None, :]
        S = alpha[:, t][:, None, None] * S
        S = S + beta[:, t][:, None, None] * kt[:, :, None] * v[:, t, None, :]
        o[:, t] = np.einsum("nd,nde->ne", q[:, t], S)
    return o


# ----------------------------------------------------------------------------
# Single output by the unrolled sum (sampled checks at full size)
# ----------------------------------------------------------------------------
def gdn_single(q_t, k_prefix, v_prefix, log_alpha_prefix, beta_prefix, lam_t):
    """o_t for t = len(prefix) - 1: walk s = t, t-1, ..., 0 carrying u = A_{s+1}^T ... A_t^T q_t
    (A is symmetric, so u^T k_s = q_t^T A_t ... A_{s+1} k_s), O(t d_k) work."""
    k = np.asarray(k_prefix, F64); v = np.asarray(v_prefix, F64)
    alpha = np.exp(np.asarray(log_alpha_prefix, F64))
    beta = np.asarray(beta_prefix, F64)
    lam_t = np.asarray(lam_t, F64)
    t = k.shape[0] - 1
    u = np.asarray(q_t, F64).copy()
    o = np.zeros(v.shape[1], F64)
    for s in range(t, -1, -1):
        o += lam_t[fenwick_level(t, s)] * beta[s] * float(u @ k[s]) * v[s]
        # extend the product by A_s for the next (earlier) key
        u = _transition_apply(alpha[s], beta[s], k[s], u)
    return o


# ----------------------------------------------------------------------------
# Whole-tensor drivers (dense [B,T,H,.] or packed [total,H,.])
# ----------------------------------------------------------------------------
def _per_sequence(inp):
    qf = inp.q.reshape(-1, inp.H, inp.dk)
    kf = inp.k.reshape(-1, inp.H, inp.dk)
    vf = inp.v.reshape(-1, inp.H, inp.dv)
    laf = inp.log_a.reshape(-1, inp.H)
    bf = inp.beta.reshape(-1, inp.H)
    lmf = inp.lam.reshape(-1, inp.H, inp.L)
    for start, n in inp.seq_slices():
        sl = slice(start, start + n)
        yield (sl, qf[sl].transpose(1, 0, 2), kf[sl].transpose(1, 0, 2),
               vf[sl].transpose(1, 0, 2), laf[sl].T, bf[sl].T, lmf[sl].transpose(1, 0, 2))


def gdn_recurrent(inp):
    """Whole input via the recurrent form; fp64 shaped like inp.v.  inp.log_a holds log alpha."""
    out = np.zeros(inp.v.reshape(-1, inp.H, inp.dv).shape, F64)
    for sl, q, k, v, la, b, lm in _per_sequence(inp):
        if q.shape[1] == 0:
            continue
        out[sl] = gdn_recurrent_seq(q, k, v, la, b, lm).transpose(1, 0, 2)
    return out.reshape(inp.v.shape)


def gdn_bruteforce(inp):
    out = np.zeros(inp.v.reshape(-1, inp.H, inp.dv).shape, F64)
    for sl, q, k, v, la, b, lm in _per_sequence(inp):
        for h in range(inp.H):
            out[sl, h] = gdn_bruteforce_seq(q[h], k[h], v[h], la[h], b[h], lm[h])
    return out.reshape(inp.v.shape)


def gated_deltanet(inp):
    out = np.zeros(inp.v.reshape(-1, inp.H, inp.dv).shape, F64)
    for sl, q, k, v, la, b, lm in _per_sequence(inp):
        if q.shape[1] == 0:
            continue
        out[sl] = gated_deltanet_seq(q, k, v, la, b).transpose(1, 0, 2)
    return out.reshape(inp.v.shape)


def gdn_sampled(inp, samples):
    """o at sampled (token_index, head) pairs of the flattened [tokens, H] grid, by gdn_single."""
    qf = inp.q.reshape(-1, inp.H, inp.dk)
    kf = inp.k.reshape(-1, inp.H, inp.dk)
    vf = inp.v.reshape(-1, inp.H, inp.dv)
    laf = inp.log_a.reshape(-1, inp.H)
    bf = inp.beta.reshape(-1, inp.H)
    lmf = inp.lam.reshape(-1, inp.H, inp.L)
    starts = np.array([s for s, _ in inp.seq_slices()], np.int64)
    res = np.zeros((len(samples), inp.dv), F64)
    for i, (tok, h) in enumerate(samples):
        s0 = int(starts[int(np.searchsorted(starts, tok, side="right") - 1)])
        res[i] = gdn_single(qf[tok, h], kf[s0:tok + 1, h], vf[s0:tok + 1, h],
                            laf[s0:tok + 1, h], bf[s0:tok + 1, h], lmf[tok, h])
    return res
