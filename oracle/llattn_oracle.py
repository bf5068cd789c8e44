"""CPU fp64 oracle for the log-linear attention forward (Mamba-2 form).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference arm may import or run this module.  It
shares no code with the CUDA path (hierarchical_fenwick_state_b200/csrc) and
imports nothing from it; the only common module is the seeded input generator,
which holds none of the method's arithmetic.

What is computed.  Log-Linear Attention (gist.science summaries, Italian and
Spanish, "Sommario tecnico" / "Resumen tecnico" section 2) replaces the single
state of a linear-attention / SSM layer by a set of states, one per bucket of a
Fenwick-tree (binary indexed tree) partition of the prefix: recent tokens in
small buckets, distant tokens in large ones (section 2, "Partizionamento
Gerarchico (Fenwick Tree)"), equivalently a hierarchical HODLR mask M_H in
place of the causal mask (section 2, "Matrici Gerarchiche").  At step t the
output is a weighted combination of the level states (section 2, "Forma
Ricorrente e Parallelizzata", decoding bullet), and the Mamba-2 variant keeps
Mamba-2's selective scalar gate (section 2, "Generalizzazione" / Spanish
"Variantes Propuestas" item 1).  Written out, per sequence and head, with
0-based sequence-local positions:

    o_t = sum_{s <= t} lam[t, l(t, s)] * (prod_{r = s+1..t} a_r) * (q_t . k_s) * v_s
    l(t, s) = 0 if s == t else 1 + floor(log2(t XOR s)),   a_r = exp(log_a[r]).

lam[t, l] is a per-(query token, level) weight (level index, not a power).
There is no softmax, no 1/sqrt(d) scale and no normalisation.

Forms (each cites the passage it follows):
  * ``llattn_bruteforce``  - the definition, literally: explicit product of the
    gates, per-pair level.  Tiny T only.
  * ``llattn_quadratic``   - the parallel / masked form O = ((Q K^T) .* M_H) V
    (section 2, "Matrici Gerarchiche"; Spanish "Forma Paralela para
    Entrenamiento").  BLAS for the products.
  * ``llattn_recurrent``   - the recurrent form with one d_k x d_v state per
    Fenwick level, merged on promotion like a binary counter (section 2,
    "Forma Ricorrente e Parallelizzata", decoding; Spanish "Particion
    Jerarquica (Arbol Fenwick)").  No cumulative sums, no level function.
  * ``mamba2_recurrent``   - plain Mamba-2 / SSD (one state), for the
    reduction checks (Spanish "Variantes Propuestas" item 1).
  * ``llattn_single``      - one output o_t by direct summation over s (the
    definition), for sampled checks at full size.
  * ``llattn_decode_step`` - one token of the decoding form: gate the occupied
    level states, read out, carry into the next level (section 2, "Forma
    Ricorrente e Parallelizzata", decoding bullet); occupancy comes from the
    position's bits alone.  ``llattn_level_states`` builds the states before a
    position straight from the level definition, to start or check decoding.
  * ``llattn_backward``    - gradients of sum(do * o) with respect to q, k, v,
    log_a and lam, by differentiating the masked form product by product.

Parity status: every function here is pinned by tests that do not retype its
formula (brute force on tiny inputs, Fenwick prefix decomposition, reduction
to Mamba-2 and to causal linear attention, one-hot levels, causality,
linearity, varlen splitting); see tests/test_oracle_pins.py.
"""
from __future__ import annotations

import numpy as np

F64 = np.float64


# ----------------------------------------------------------------------------
# Fenwick level
# ----------------------------------------------------------------------------
def fenwick_level(t: int, s: int) -> int:
    """l(t, s): 0 for s == t, else 1 + floor(log2(t XOR s)) (0-based positions)."""
    if s == t:
        return 0
    x = int(t) ^ int(s)
    return x.bit_length()  # == 1 + floor(log2 x) for x >= 1


def fenwick_level_matrix(t_idx: np.ndarray, s_idx: np.ndarray) -> np.ndarray:
    """Vectorised l(t, s) for index vectors (rows t, columns s); exact via frexp."""
    x = (np.asarray(t_idx, np.int64)[:, None] ^ np.asarray(s_idx, np.int64)[None, :])
    # frexp(x) = (m, e) with x = m * 2**e, m in [0.5, 1): e == bit_length(x); frexp(0) -> e = 0.
    return np.frexp(x.astype(F64))[1].astype(np.int64)


# ----------------------------------------------------------------------------
# Brute force: the definition written out (tiny T)
# ----------------------------------------------------------------------------
def llattn_bruteforce_seq(q, k, v, log_a, lam):
    """One sequence, one head.  q,k [T,dk]; v [T,dv]; log_a [T]; lam [T,L] -> o [T,dv] (fp64).

    Double loop over (t, s <= t) with the explicit gate product prod_{r=s+1..t} a_r
    (empty product = 1 at s = t) and the per-pair level.
    """
    q = np.asarray(q, F64); k = np.asarray(k, F64); v = np.asarray(v, F64)
    a = np.exp(np.asarray(log_a, F64))
    lam = np.asarray(lam, F64)
    T = q.shape[0]
    o = np.zeros((T, v.shape[1]), F64)
    for t in range(T):
        for s in range(t + 1):
            prod = 1.0
            for r in range(s + 1, t + 1):
                prod *= a[r]
            lvl = fenwick_level(t, s)
            o[t] += lam[t, lvl] * prod * float(np.dot(q[t], k[s])) * v[s]
    return o


# ----------------------------------------------------------------------------
# Quadratic (masked, parallel) form
# ----------------------------------------------------------------------------
def llattn_quadratic_seq(q, k, v, log_a, lam, block: int = 1024):
    """One sequence, one head, O(T^2): O = ((Q K^T) .* M_H) V in row blocks.

    M_H[t, s] = lam[t, l(t, s)] * exp(g_t - g_s) for s <= t (0 above the
    diagonal), g = inclusive cumulative sum of log_a, so exp(g_t - g_s) is the
    gate product over r = s+1..t.
    """
    q = np.asarray(q, F64); k = np.asarray(k, F64); v = np.asarray(v, F64)
    g = np.cumsum(np.asarray(log_a, F64))
    lam = np.asarray(lam, F64)
    T = q.shape[0]
    o = np.zeros((T, v.shape[1]), F64)
    for t0 in range(0, T, block):
        t1 = min(T, t0 + block)
        tt = np.arange(t0, t1)
        ss = np.arange(0, t1)
        A = q[t0:t1] @ k[:t1].T
        lev = fenwick_level_matrix(tt, ss)
        causal = ss[None, :] <= tt[:, None]
        expo = np.where(causal, g[tt][:, None] - g[ss][None, :], -np.inf)
        lam_sel = np.take_along_axis(lam[t0:t1], lev, axis=1)
        M = np.where(causal, lam_sel * np.exp(expo), 0.0)
        o[t0:t1] = (A * M) @ v[:t1]
    return o


# ----------------------------------------------------------------------------
# Recurrent form: one state per Fenwick level, binary-counter promotion
# ----------------------------------------------------------------------------
def llattn_recurrent_seq(q, k, v, log_a, lam):
    """Sequences batched along axis 0: q,k [N,T,dk]; v [N,T,dv]; log_a [N,T]; lam [N,T,L].

    Level states S_0..S_{L-1} (d_k x d_v each).  For t = 0..T-1:
      1. multiply every non-empty S_l (l >= 1) by a_t;
      2. S_0 = k_t v_t^T;
      3. o_t = sum over non-empty l of lam[t, l] * (q_t^T S_l);
      4. promotion: with m = number of trailing one bits of t, S_{m+1} becomes
         S_0 + ... + S_m and levels 0..m become empty (the Fenwick bucket of
         2**m tokens ending at t), skipped after the last token.
    """
    q = np.asarray(q, F64); k = np.asarray(k, F64); v = np.asarray(v, F64)
    a = np.exp(np.asarray(log_a, F64))
    lam = np.asarray(lam, F64)
    N, T, dk = q.shape
    dv = v.shape[2]
    L = lam.shape[2]
    nlev = max(L, 1 + max(T - 1, 1).bit_length())
    S = np.zeros((N, nlev, dk, dv), F64)
    live = np.zeros(nlev, bool)
    o = np.zeros((N, T, dv), F64)
    for t in range(T):
        if live[1:].any():
            idx = np.nonzero(live)[0]
            idx = idx[idx >= 1]
            S[:, idx] *= a[:, t][:, None, None, None]
        S[:, 0] = k[:, t, :, None] * v[:, t, None, :]
        live[0] = True
        idx = np.nonzero(live)[0]
        # readout: sum_l lam[t,l] * q_t^T S_l
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
# Plain Mamba-2 / SSD recurrence (one state), for reduction checks
# ----------------------------------------------------------------------------
def mamba2_recurrent_seq(q, k, v, log_a):
    """S_t = a_t S_{t-1} + k_t v_t^T, o_t = S_t^T q_t; batched like llattn_recurrent_seq."""
    q = np.asarray(q, F64); k = np.asarray(k, F64); v = np.asarray(v, F64)
    a = np.exp(np.asarray(log_a, F64))
    N, T, dk = q.shape
    S = np.zeros((N, dk, v.shape[2]), F64)
    o = np.zeros((N, T, v.shape[2]), F64)
    for t in range(T):
        S = a[:, t][:, None, None] * S + k[:, t, :, None] * v[:, t, None, :]
        o[:, t] = np.einsum("nd,nde->ne", q[:, t], S)
    return o


# ----------------------------------------------------------------------------
# Single output by direct summation (sampled checks at full size)
# ----------------------------------------------------------------------------
def llattn_single(q_t, k_prefix, v_prefix, log_a_prefix, lam_t):
    """o_t for t = len(prefix) - 1 from its prefix: k_prefix [t+1,dk], v_prefix [t+1,dv],
    log_a_prefix [t+1], lam_t [L].  Gate product as exp of a suffix sum of log_a."""
    k_prefix = np.asarray(k_prefix, F64)
    v_prefix = np.asarray(v_prefix, F64)
    la = np.asarray(log_a_prefix, F64)
    t = k_prefix.shape[0] - 1
    # suffix sums: sum_{r=s+1..t} log a_r for every s (0 for s = t)
    suf = np.concatenate([np.cumsum(la[:0:-1])[::-1], [0.0]])
    lev = fenwick_level_matrix(np.array([t]), np.arange(t + 1))[0]
    w = np.asarray(lam_t, F64)[lev] * np.exp(suf)
    scores = k_prefix @ np.asarray(q_t, F64)
    return (w * scores) @ v_prefix


# ----------------------------------------------------------------------------
# Whole-tensor drivers (dense [B,T,H,.] or packed varlen [total,H,.])
# ----------------------------------------------------------------------------
def _per_sequence(inp):
    """Yield (sl, q, k, v, log_a, lam) per sequence with head-major [H, T, .] views."""
    qf = inp.q.reshape(-1, inp.H, inp.dk)
    kf = inp.k.reshape(-1, inp.H, inp.dk)
    vf = inp.v.reshape(-1, inp.H, inp.dv)
    laf = inp.log_a.reshape(-1, inp.H)
    lmf = inp.lam.reshape(-1, inp.H, inp.L)
    for start, n in inp.seq_slices():
        sl = slice(start, start + n)
        yield (sl, qf[sl].transpose(1, 0, 2), kf[sl].transpose(1, 0, 2),
               vf[sl].transpose(1, 0, 2), laf[sl].T, lmf[sl].transpose(1, 0, 2))


def llattn_recurrent(inp):
    """Whole input via the recurrent form; returns fp64 [tokens..., H, dv] like inp.v."""
    out = np.zeros(inp.v.reshape(-1, inp.H, inp.dv).shape, F64)
    for sl, q, k, v, la, lm in _per_sequence(inp):
        if q.shape[1] == 0:
            continue
        out[sl] = llattn_recurrent_seq(q, k, v, la, lm).transpose(1, 0, 2)
    return out.reshape(inp.v.shape)


def llattn_quadratic(inp, block: int = 1024):
    out = np.zeros(inp.v.reshape(-1, inp.H, inp.dv).shape, F64)
    for sl, q, k, v, la, lm in _per_sequence(inp):
        for h in range(inp.H):
            if q.shape[1] == 0:
                continue
            out[sl, h] = llattn_quadratic_seq(q[h], k[h], v[h], la[h], lm[h], block)
    return out.reshape(inp.v.shape)


def llattn_bruteforce(inp):
    out = np.zeros(inp.v.reshape(-1, inp.H, inp.dv).shape, F64)
    for sl, q, k, v, la, lm in _per_sequence(inp):
        for h in range(inp.H):
            out[sl, h] = llattn_bruteforce_seq(q[h], k[h], v[h], la[h], lm[h])
    return out.reshape(inp.v.shape)


def mamba2_recurrent(inp):
    out = np.zeros(inp.v.reshape(-1, inp.H, inp.dv).shape, F64)
    for sl, q, k, v, la, lm in _per_sequence(inp):
        if q.shape[1] == 0:
            continue
        out[sl] = mamba2_recurrent_seq(q, k, v, la).transpose(1, 0, 2)
    return out.reshape(inp.v.shape)


def llattn_sampled(inp, samples):
    """o at sampled (token_index, head) pairs of the flattened [tokens, H] grid -> [n, dv]."""
    qf = inp.q.reshape(-1, inp.H, inp.dk)
    kf = inp.k.reshape(-1, inp.H, inp.dk)
    vf = inp.v.reshape(-1, inp.H, inp.dv)
    laf = inp.log_a.reshape(-1, inp.H)
    lmf = inp.lam.reshape(-1, inp.H, inp.L)
    starts = np.array([s for s, _ in inp.seq_slices()], np.int64)
    res = np.zeros((len(samples), inp.dv), F64)
    for i, (tok, h) in enumerate(samples):
        seq = int(np.searchsorted(starts, tok, side="right") - 1)
        s0 = int(starts[seq])
        res[i] = llattn_single(qf[tok, h], kf[s0:tok + 1, h], vf[s0:tok + 1, h],
                               laf[s0:tok + 1, h], lmf[tok, h])
    return res


def rel_max_err(got, ref) -> float:
    """max |got - ref| / RMS(ref): the parity metric (max abs error relative to output RMS)."""
    ref = np.asarray(ref, F64)
    got = np.asarray(got, F64)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    if ref.size == 0:
        return 0.0
    return float(np.max(np.abs(got - ref)) / max(rms, 1e-300))


# ----------------------------------------------------------------------------
# Decoding form: one token per step over the O(log T) level states
# ----------------------------------------------------------------------------
def llattn_level_states(k, v, log_a, n: int, nslot: int):
    """Level states of one sequence and head just before 0-based position n, from the definition.

    Level l >= 1 holds the earlier tokens s < n with l(n, s) == l (the Fenwick bucket of
    2**(l-1) tokens that exists iff bit l-1 of n is set; Log-Linear Attention, section 2,
    "Partizionamento Gerarchico (Fenwick Tree)"), each as k_s v_s^T times the gate product
    over r = s+1..n-1.  The gate of position n itself belongs to the step that reads the
    states.  k [>= n, dk], v [>= n, dv], log_a [>= n] -> [nslot, dk, dv] for levels 1..nslot
    (zero where the bucket is empty).
    """
    k = np.asarray(k, F64)[:n]
    v = np.asarray(v, F64)[:n]
    la = np.asarray(log_a, F64)[:n]
    S = np.zeros((nslot, k.shape[1] if k.ndim == 2 else 0, v.shape[1] if v.ndim == 2 else 0), F64)
    if n == 0:
        return S
    if n.bit_length() > nslot:
        raise ValueError(f"position {n} needs {n.bit_length()} level slots, have {nslot}")
    lev = fenwick_level_matrix(np.array([n]), np.arange(n))[0]
    # sum_{r=s+1..n-1} log a_r for every s < n (0 for s = n-1)
    suf = np.concatenate([np.cumsum(la[:0:-1])[::-1], [0.0]])
    w = np.exp(suf)
    for lvl in range(1, nslot + 1):
        sel = lev == lvl
        if sel.any():
            S[lvl - 1] = (k[sel] * w[sel, None]).T @ v[sel]
    return S


def llattn_decode_step(S, n: int, q, k, v, log_a, lam):
    """One step of the decoding (recurrent) form for one sequence and head at position n.

    Log-Linear Attention, section 2, "Forma Ricorrente e Parallelizzata", decoding bullet:
    the layer keeps one state per level of the hierarchy and each output is the per-level
    weighted combination of those states; the Mamba-2 variant gates every state with the
    scalar a_n (Spanish page, "Variantes Propuestas" item 1).

    S [nslot, dk, dv]: the states of levels 1..nslot just before position n.  Which levels
    hold a bucket is read off the binary counter n alone: level l is occupied iff bit l-1 of
    n is set; the other slots are ignored, whatever they hold.  q, k [dk]; v [dv]; log_a and
    lam[0 .. bit_length(n)] for this token.  Returns (o [dv], S_next), S_next being the states
    just before position n + 1:
      1. every occupied level is multiplied by a_n = exp(log_a);
      2. the token's own state k v^T is level 0;
      3. o = sum over level 0 and the occupied levels of lam[l] * (q^T S_l);
      4. promotion (binary-counter carry): with m the number of trailing one bits of n,
         levels 0..m add up into level m+1, and levels 1..m are emptied.  When m+1 > nslot,
         position n is the last one the slots can hold and nothing is merged.
    """
    S = np.array(S, F64, copy=True)
    nslot = S.shape[0]
    if n < 0 or n.bit_length() > nslot:
        raise ValueError(f"position {n} out of range for {nslot} level slots")
    q = np.asarray(q, F64); k = np.asarray(k, F64); v = np.asarray(v, F64)
    lam = np.asarray(lam, F64)
    a = float(np.exp(np.float64(log_a)))
    occupied = [lvl for lvl in range(1, nslot + 1) if (n >> (lvl - 1)) & 1]
    for lvl in occupied:
        S[lvl - 1] *= a
    S0 = np.outer(k, v)
    o = lam[0] * (q @ S0)
    for lvl in occupied:
        o = o + lam[lvl] * (q @ S[lvl - 1])
    m = 0
    while (n >> m) & 1:
        m += 1
    if m + 1 <= nslot:
        merged = S0.copy()
        for lvl in range(1, m + 1):
            merged += S[lvl - 1]
            S[lvl - 1] = 0.0
        S[m] = merged
    return o, S


def llattn_decode_sequence(q, k, v, log_a, lam):
    """One sequence and head decoded token by token from empty states: q,k [T,dk], v [T,dv],
    log_a [T], lam [T,L] -> o [T,dv], with L - 1 level slots (levels 1..L-1)."""
    q = np.asarray(q, F64)
    T = q.shape[0]
    lam = np.asarray(lam, F64)
    nslot = lam.shape[1] - 1
    S = np.zeros((nslot, q.shape[1], np.asarray(v).shape[1]), F64)
    o = np.zeros((T, np.asarray(v).shape[1]), F64)
    for n in range(T):
        o[n], S = llattn_decode_step(S, n, q[n], k[n], v[n], log_a[n], lam[n])
    return o


def llattn_decode_batch(S, pos, q, k, v, log_a, lam):
    """Decoding step over a batch: S [B,H,nslot,dk,dv] (states before each row's position),
    pos [B] (tokens each row has absorbed), q,k [B,H,dk], v [B,H,dv], log_a [B,H],
    lam [B,H,L] -> (o [B,H,dv], S_next)."""
    S = np.asarray(S, F64)
    B, H = S.shape[:2]
    o = np.zeros((B, H, np.asarray(v).shape[2]), F64)
    S_next = np.array(S, F64, copy=True)
    for b in range(B):
        for h in range(H):
            o[b, h], S_next[b, h] = llattn_decode_step(S[b, h], int(pos[b]), q[b, h], k[b, h],
                                                       v[b, h], log_a[b, h], lam[b, h])
    return o, S_next


# ----------------------------------------------------------------------------
# Backward: gradients of the masked (parallel) form
# ----------------------------------------------------------------------------
def llattn_backward_seq(q, k, v, log_a, lam, do):
    """Gradients of sum(do * o) for one sequence and head, o = ((Q K^T) .* M_H) V.

    The forward is the parallel form of Log-Linear Attention (section 2, "Matrici
    Gerarchiche"; Spanish "Forma Paralela para Entrenamiento"): A = Q K^T, M[t, s] =
    lam[t, l(t, s)] * exp(g_t - g_s) for s <= t, P = A .* M, O = P V, with g the
    inclusive cumulative sum of log_a.  Differentiating each product in turn:
      dV = P^T dO;   dP = dO V^T;   dQ = (dP .* M) K;   dK = (dP .* M)^T Q;
      dM = dP .* A   (on s <= t);
      dlam[t, l] = sum over s <= t with l(t, s) == l of dM[t, s] * exp(g_t - g_s);
      dE = dM .* M   (the gradient of the exponent g_t - g_s);
      dg_t = sum_s dE[t, s] - sum_t' dE[t', t];
      dlog_a[r] = sum over t >= r of dg_t   (g_t sums log_a over positions <= t).
    Inputs q,k [T,dk]; v, do [T,dv]; log_a [T]; lam [T,L].  Returns fp64
    (dq, dk, dv, dlog_a, dlam).
    """
    q = np.asarray(q, F64); k = np.asarray(k, F64); v = np.asarray(v, F64)
    do = np.asarray(do, F64)
    g = np.cumsum(np.asarray(log_a, F64))
    lam = np.asarray(lam, F64)
    T = q.shape[0]
    L = lam.shape[1]
    tt = np.arange(T)
    lev = fenwick_level_matrix(tt, tt)
    causal = tt[None, :] <= tt[:, None]
    E = np.where(causal, np.exp(np.where(causal, g[:, None] - g[None, :], 0.0)), 0.0)
    lam_sel = np.take_along_axis(lam, np.where(causal, lev, 0), axis=1)
    M = np.where(causal, lam_sel * E, 0.0)
    A = q @ k.T
    P = A * M
    dv = P.T @ do
    dP = do @ v.T
    dA = dP * M
    dq = dA @ k
    dk = dA.T @ q
    dM = np.where(causal, dP * A, 0.0)
    dlam = np.zeros((T, L), F64)
    contrib = dM * E
    for lvl in range(L):
        dlam[:, lvl] = np.sum(np.where(causal & (lev == lvl), contrib, 0.0), axis=1)
    dE = dM * M
    dg = dE.sum(axis=1) - dE.sum(axis=0)
    dlog_a = np.cumsum(dg[::-1])[::-1]
    return dq, dk, dv, dlog_a, dlam


def llattn_backward(inp, do):
    """Whole-input gradients (dense or packed), fp64, laid out like the inputs:
    returns dict q, k, v, log_a, lam.  do has the layout of the output."""
    H = inp.H
    res = {
        "q": np.zeros(inp.q.reshape(-1, H, inp.dk).shape, F64),
        "k": np.zeros(inp.k.reshape(-1, H, inp.dk).shape, F64),
        "v": np.zeros(inp.v.reshape(-1, H, inp.dv).shape, F64),
        "log_a": np.zeros(inp.log_a.reshape(-1, H).shape, F64),
        "lam": np.zeros(inp.lam.reshape(-1, H, inp.L).shape, F64),
    }
    dof = np.asarray(do).reshape(-1, H, inp.dv)
    for sl, q, k, v, la, lm in _per_sequence(inp):
        if q.shape[1] == 0:
            continue
        for h in range(H):
            dq, dk, dv, dla, dlm = llattn_backward_seq(q[h], k[h], v[h], la[h], lm[h], dof[sl, h])
            res["q"][sl, h] = dq
            res["k"][sl, h] = dk
            res["v"][sl, h] = dv
            res["log_a"][sl, h] = dla
            res["lam"][sl, h] = dlm
    return {"q": res["q"].reshape(inp.q.shape), "k": res["k"].reshape(inp.k.shape),
            "v": res["v"].reshape(inp.v.shape), "log_a": res["log_a"].reshape(inp.log_a.shape),
            "lam": res["lam"].reshape(inp.lam.shape)}


def llattn_backward_sampled(inp, do, samples):
    """Gradient rows at sampled (token_index, head) pairs of the flattened [tokens, H] grid,
    each by direct summation over its own row or column of the mask (the definition):
      dq_t  = sum_{s<=t} M[t,s] (do_t . v_s) k_s,     dlam[t, l] = sum_{l(t,s)=l} E[t,s] (q_t . k_s)(do_t . v_s),
      dk_s  = sum_{t>=s} M[t,s] (do_t . v_s) q_t,     dv_s = sum_{t>=s} M[t,s] (q_t . k_s) do_t,
    with E[t, s] the gate product as exp of a sum of log_a and M[t, s] = lam[t, l(t,s)] E[t, s].
    Returns dict q, k, v [n, d] and lam [n, L] (fp64)."""
    qf = np.asarray(inp.q, F64).reshape(-1, inp.H, inp.dk)
    kf = np.asarray(inp.k, F64).reshape(-1, inp.H, inp.dk)
    vf = np.asarray(inp.v, F64).reshape(-1, inp.H, inp.dv)
    laf = np.asarray(inp.log_a, F64).reshape(-1, inp.H)
    lmf = np.asarray(inp.lam, F64).reshape(-1, inp.H, inp.L)
    dof = np.asarray(do, F64).reshape(-1, inp.H, inp.dv)
    starts = np.array([s for s, _ in inp.seq_slices()], np.int64)
    lens = np.array([n for _, n in inp.seq_slices()], np.int64)
    n = len(samples)
    out = {"q": np.zeros((n, inp.dk)), "k": np.zeros((n, inp.dk)), "v": np.zeros((n, inp.dv)),
           "lam": np.zeros((n, inp.L))}
    for i, (tok, h) in enumerate(samples):
        sq = int(np.searchsorted(starts, tok, side="right") - 1)
        s0, ln = int(starts[sq]), int(lens[sq])
        x = tok - s0                                   # sequence-local position
        la = laf[s0:s0 + ln, h]
        # row x: keys s <= x; gate product over r = s+1..x
        ks = np.arange(x + 1)
        pref = np.concatenate([[0.0], np.cumsum(la[1:x + 1])])     # sum of la[1..j]
        E_row = np.exp(pref[x] - pref[ks])
        lev_row = fenwick_level_matrix(np.array([x]), ks)[0]
        a_row = kf[s0 + ks, h] @ qf[tok, h]
        b_row = vf[s0 + ks, h] @ dof[tok, h]
        m_row = lmf[tok, h][lev_row] * E_row
        out["q"][i] = (m_row * b_row) @ kf[s0 + ks, h]
        np.add.at(out["lam"][i], lev_row, E_row * a_row * b_row)
        # column x: queries t >= x; gate product over r = x+1..t
        ts = np.arange(x, ln)
        E_col = np.exp(np.cumsum(np.concatenate([[0.0], la[x + 1:ln]])))
        lev_col = fenwick_level_matrix(ts, np.array([x]))[:, 0]
        m_col = lmf[s0 + ts, h][np.arange(len(ts)), lev_col] * E_col
        a_col = qf[s0 + ts, h] @ kf[tok, h]
        b_col = dof[s0 + ts, h] @ vf[tok, h]
        out["k"][i] = (m_col * b_col) @ qf[s0 + ts, h]
        out["v"][i] = (m_col * a_col) @ dof[s0 + ts, h]
    return out
