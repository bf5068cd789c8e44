"""GPU parity: the CUDA paths (through the C ABI) against the CPU fp64 oracle.

Oracle-sized cases span several chunks and a ragged tail and compare every
output element; full-size cases (the bench's launch configuration) compare
sampled outputs the oracle computes one at a time.  Metric: max |gpu - oracle|
divided by the RMS of the oracle output, <= 1e-4 for fp32 inputs and <= 2e-2 for
bf16 inputs (fp32 accumulation, fp32 output).
"""
import numpy as np
import pytest

import oracle as O
from hierarchical_fenwick_state_b200 import binding
from hierarchical_fenwick_state_b200 import inputs as I

from _llattn_cases import TOL, run

pytestmark = pytest.mark.gpu

W = I.WORKLOADS


def _paths_for(inp):
    paths = ["simt"]
    if inp.dtype == "bf16":
        for path in ("tcgen05", "tcgen05_serial"):
            try:
                binding.workspace_bytes(1, path, 0, inp.B, inp.H, inp.T, inp.dk, inp.dv,
                                        inp.cu_seqlens is not None)
                paths.append(path)
            except binding.LLAttnError:
                pass
    return paths


def _check(inp, ref, path, chunk=0):
    got = run(inp, path=path, chunk=chunk)
    assert np.isfinite(got).all(), "unwritten or non-finite outputs"
    err = O.rel_max_err(got, ref)
    assert err <= TOL[inp.dtype], f"{path} chunk={chunk}: rel max err {err:.3e}"
    return err


# ------------------------------------------------------------------------------------------------
# Element-by-element parity on oracle-sized cases of each workload
# ------------------------------------------------------------------------------------------------
CASES = {
    "t256_d32_f32": W["t256_d32_f32"],
    "t256_d32_f32_ragged": I.shrink(W["t256_d32_f32"], T=250),
    "t2k_d64_bf16": W["t2k_d64_bf16"],
    "t8k_d64_bf16_h2": I.shrink(W["t8k_d64_bf16"], B=1, H=2),
    "t8k_d64_bf16_ragged": I.shrink(W["t8k_d64_bf16"], B=2, H=1, T=8000),
    "t64k_d128_bf16_t8k": I.shrink(W["t64k_d128_bf16"], H=2, T=8192),
    "varlen_small": I.shrink(W["varlen8_d64_bf16"], H=2, T=3000, len_lo=1, len_hi=3000),
    # more than 64 chunks: the seventh chunk level and the two-stage variant of the kernel
    "t12k_d64_bf16_h1": I.shrink(W["t8k_d64_bf16"], B=1, H=1, T=12000),
    "varlen_long": I.shrink(W["varlen8_d64_bf16"], B=3, H=1, T=16384, len_lo=8000, len_hi=16384),
}


@pytest.mark.parametrize("name", list(CASES))
def test_parity_workloads(name):
    inp = I.make_inputs(CASES[name], seed=0)
    ref = O.llattn_recurrent(inp)
    for path in _paths_for(inp):
        _check(inp, ref, path)


# ------------------------------------------------------------------------------------------------
# Stress: decay regimes that reach the deep Fenwick levels, one level at a time
# ------------------------------------------------------------------------------------------------
@pytest.mark.parametrize("mode", ["zero", "slow", "strong"])
@pytest.mark.parametrize("base", ["t2k_d64_bf16", "t256_d32_f32"])
def test_parity_decay_regimes(mode, base):
    w = I.shrink(W[base], B=1, H=2) if base == "t2k_d64_bf16" else W[base]
    inp = I.make_inputs(w, seed=1, log_a_mode=mode)
    ref = O.llattn_recurrent(inp)
    for path in _paths_for(inp):
        _check(inp, ref, path)


@pytest.mark.parametrize("level", [13, 14])
def test_parity_one_hot_deep_level_long(level):
    # level 14 reaches the seventh chunk-level state (blocks of 64 chunks): T > 8192, no decay
    w = I.shrink(W["t8k_d64_bf16"], B=1, H=1, T=16384)
    inp = I.make_inputs(w, seed=4, log_a_mode="zero", lam_mode="onehot", lam_level=level)
    ref = O.llattn_recurrent(inp)
    for path in _paths_for(inp):
        _check(inp, ref, path)


@pytest.mark.parametrize("level", [0, 1, 5, 6, 7, 8, 10, 11])
def test_parity_one_hot_level(level):
    w = I.shrink(W["t2k_d64_bf16"], B=1, H=2)
    inp = I.make_inputs(w, seed=2, log_a_mode="zero", lam_mode="onehot", lam_level=level)
    ref = O.llattn_recurrent(inp)
    for path in _paths_for(inp):
        _check(inp, ref, path)


@pytest.mark.parametrize("chunk", [8, 16, 32, 64])
def test_simt_chunk_invariance(chunk):
    w = I.shrink(W["t2k_d64_bf16"], B=1, H=2, T=1000)
    inp = I.make_inputs(w, seed=3, log_a_mode="slow")
    ref = O.llattn_recurrent(inp)
    _check(inp, ref, "simt", chunk=chunk)


# ------------------------------------------------------------------------------------------------
# Edge cases
# ------------------------------------------------------------------------------------------------
@pytest.mark.parametrize("T", [1, 2, 15, 16, 17, 63, 64, 65, 127, 128, 129, 255, 257])
def test_edge_lengths(T):
    for base in ("t2k_d64_bf16", "t256_d32_f32"):
        w = I.shrink(W[base], B=2, H=1, T=T)
        inp = I.make_inputs(w, seed=T)
        ref = O.llattn_recurrent(inp)
        for path in _paths_for(inp):
            _check(inp, ref, path)


def test_varlen_edge_lengths():
    w = I.Workload("vl_edge", B=7, H=3, T=600, dk=64, dv=64, dtype="bf16", varlen=True)
    inp = I.make_inputs(w, seed=5, lengths=np.array([0, 1, 129, 600, 64, 0, 2]))
    ref = O.llattn_recurrent(inp)
    for path in _paths_for(inp):
        _check(inp, ref, path)


def test_varlen_sequence_longer_than_bound_sets_status():
    import torch
    from _llattn_cases import to_device
    w = I.Workload("vl_bad", B=2, H=1, T=64, dk=64, dv=64, dtype="bf16", varlen=True)
    inp = I.make_inputs(w, seed=6, lengths=np.array([100, 10]))
    t = to_device(inp)
    out = torch.zeros(inp.v.shape, dtype=torch.float32, device="cuda:0")
    binding.forward(t["q"], t["k"], t["v"], t["log_a"], t["lam"], cu_seqlens=t["cu"], T=64,
                    out=out, path="simt")
    torch.cuda.synchronize()
    assert binding.device_status(clear=True) & 1


def test_dims_32_and_128_mixed():
    w = I.Workload("mixed", B=1, H=2, T=300, dk=32, dv=128, dtype="bf16")
    inp = I.make_inputs(w, seed=8)
    ref = O.llattn_recurrent(inp)
    _check(inp, ref, "simt")


# ------------------------------------------------------------------------------------------------
# Full-size workloads in the bench's launch configuration: sampled outputs
# ------------------------------------------------------------------------------------------------
@pytest.mark.parametrize("name", list(W))
def test_full_size_sampled(name):
    w = W[name]
    inp = I.make_inputs(w, seed=0)
    rng = np.random.default_rng(123)
    ntok = inp.total_tokens
    toks = np.concatenate([rng.integers(0, ntok, 120), [0, ntok - 1]])
    # also the last token of every sequence (deepest Fenwick levels)
    toks = np.concatenate([toks, [s + n - 1 for s, n in inp.seq_slices() if n > 0]])
    samples = [(int(t), int(rng.integers(0, inp.H))) for t in toks]
    ref = O.llattn_sampled(inp, samples)
    got = run(inp, path="auto").reshape(-1, inp.H, inp.dv)
    sel = np.stack([got[t, h] for t, h in samples])
    assert np.isfinite(got).all()
    err = O.rel_max_err(sel, ref)
    assert err <= TOL[inp.dtype], f"{name}: sampled rel max err {err:.3e}"


# ------------------------------------------------------------------------------------------------
# Golden fixtures: closed-form integer inputs whose outputs are stored in tests/golden/
# ------------------------------------------------------------------------------------------------
@pytest.mark.parametrize("name,decay", [("patterned_nodecay_T300", 0.0),
                                        ("patterned_decay8_T300", -0.125)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_golden_fixtures(name, decay, dtype):
    from test_golden import load
    inp = I.make_patterned(300, log_a=decay, dtype=dtype)
    rows = load(name)
    want = np.array([o for _, _, o in rows])
    for path in _paths_for(inp):
        got = run(inp, path=path).reshape(300, inp.H, inp.dv)
        sel = np.array([got[t, 0, j] for t, j, _ in rows])
        err = O.rel_max_err(sel, want)
        assert err <= TOL[dtype], f"{path}: rel max err {err:.3e}"


# ------------------------------------------------------------------------------------------------
# Host-buffer entry point (dense batches are pipelined row by row inside the library)
# ------------------------------------------------------------------------------------------------
@pytest.mark.parametrize("name", ["dense_pipelined", "dense_one_row", "varlen", "f32"])
def test_host_entry_point_matches_device_path(name):
    cases = {
        "dense_pipelined": I.shrink(W["t2k_d64_bf16"], B=3, H=2, T=1000),
        "dense_one_row": I.shrink(W["t2k_d64_bf16"], B=1, H=2, T=700),
        "varlen": I.shrink(W["varlen8_d64_bf16"], B=3, H=2, T=2000, len_lo=1, len_hi=2000),
        "f32": I.shrink(W["t256_d32_f32"], B=2, T=250),
    }
    inp = I.make_inputs(cases[name], seed=9)
    bf = inp.dtype == "bf16"
    conv = (lambda x: np.ascontiguousarray(I.bf16_bits(x))) if bf else (lambda x: x)
    out = np.full(inp.v.shape, np.nan, dtype=np.float32)
    cu = np.ascontiguousarray(inp.cu_seqlens) if inp.cu_seqlens is not None else None
    B = inp.B if cu is None else len(cu) - 1
    binding.fwd_host(binding.BF16 if bf else binding.F32, conv(inp.q), conv(inp.k), conv(inp.v),
                     inp.log_a, inp.lam, out, B, inp.H, inp.T, inp.dk, inp.dv, cu_seqlens=cu)
    assert binding.device_status(clear=True) == 0
    dev = run(inp, path="auto").astype(np.float32)
    assert np.array_equal(out, dev), "host entry point differs from the device entry point"
    err = O.rel_max_err(out.astype(np.float64), O.llattn_recurrent(inp))
    assert err <= TOL[inp.dtype], f"rel max err {err:.3e}"


@pytest.mark.parametrize("T", [8192, 8193, 16383])
def test_kernel_boundaries_odd_heads(T):
    # the last length of the six-level kernel, the first of the seven-level one, and a ragged
    # tail at its limit; three heads (odd TMA head stride), two sequences
    w = I.shrink(W["t8k_d64_bf16"], B=2, H=3, T=T)
    inp = I.make_inputs(w, seed=T % 97, log_a_mode="slow")
    ref = O.llattn_recurrent(inp)
    for path in _paths_for(inp):
        _check(inp, ref, path)


# ------------------------------------------------------------------------------------------------
# Range guard of the tensor-core path's fp16 operands, and the status word read per stream
# ------------------------------------------------------------------------------------------------
def test_fp16_range_guard_sets_status_bit():
    """v scaled by 1e5 leaves the fp16 range on the tensor-core path (V, P V and the level
    states are rounded to fp16 there): the output turns non-finite and the kernel sets
    LLATTN_DEV_NONFINITE, read here through the per-stream status call.  The CUDA-core path
    computes in fp32 and matches the oracle on the same inputs."""
    import torch
    w = I.shrink(W["t2k_d64_bf16"], B=1, H=2, T=1000)
    inp = I.make_inputs(w, seed=5)
    inp.v = I.round_to_bf16(inp.v * np.float32(1e5))
    ref = O.llattn_recurrent(inp)
    t = _to_device_for_guard(inp)
    out = torch.empty(inp.v.shape, dtype=torch.float32, device="cuda:0")
    binding.stream_status(clear=True)
    binding.forward(t["q"], t["k"], t["v"], t["log_a"], t["lam"], T=inp.T, out=out,
                    path="tcgen05")
    flags = binding.stream_status(clear=True)
    assert flags & 16, f"LLATTN_DEV_NONFINITE not set (flags {flags})"
    assert not np.isfinite(out.double().cpu().numpy()).all()
    out.fill_(float("nan"))
    binding.forward(t["q"], t["k"], t["v"], t["log_a"], t["lam"], T=inp.T, out=out, path="simt")
    assert binding.stream_status(clear=True) == 0
    got = out.double().cpu().numpy()
    assert O.rel_max_err(got, ref) <= TOL["bf16"]
    # in-range inputs leave the bit clear on the tensor-core path
    inp2 = I.make_inputs(w, seed=5)
    t2 = _to_device_for_guard(inp2)
    binding.forward(t2["q"], t2["k"], t2["v"], t2["log_a"], t2["lam"], T=inp2.T, out=out,
                    path="tcgen05")
    assert binding.stream_status(clear=True) == 0


def _to_device_for_guard(inp):
    from _llattn_cases import to_device
    return to_device(inp)


def test_fwd_bf16_alias_matches_fwd():
    import torch
    w = I.shrink(W["t2k_d64_bf16"], B=1, H=2, T=700)
    inp = I.make_inputs(w, seed=6)
    t = _to_device_for_guard(inp)
    o1 = torch.full(inp.v.shape, float("nan"), dtype=torch.float32, device="cuda:0")
    o2 = torch.full_like(o1, float("nan"))
    args = (t["q"], t["k"], t["v"], t["log_a"], t["lam"])
    binding.fwd(*args, o1, inp.B, inp.H, inp.T, inp.dk, inp.dv)
    binding.fwd_bf16(*args, o2, inp.B, inp.H, inp.T, inp.dk, inp.dv)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)
    assert binding.stream_status(clear=True) == 0



@pytest.mark.parametrize("T", [300, 700])
def test_fwd_f32_entry_both_sides_of_the_short_form(T):
    """llattn_fwd_f32 takes the automatic path: T = 300 runs the one-launch masked form, T = 700
    the chunkwise CUDA-core kernels; both against the oracle at the fp32 bound."""
    import torch
    w = I.Workload("f32_entry", B=2, H=3, T=T, dk=64, dv=32, dtype="f32")
    inp = I.make_inputs(w, seed=T)
    t = _to_device_for_guard(inp)
    out = torch.full(inp.v.shape, float("nan"), dtype=torch.float32, device="cuda:0")
    binding.fwd_f32(t["q"], t["k"], t["v"], t["log_a"], t["lam"], out, inp.B, inp.H, inp.T,
                    inp.dk, inp.dv)
    torch.cuda.synchronize()
    assert binding.stream_status(clear=True) == 0
    err = O.rel_max_err(out.double().cpu().numpy(), O.llattn_recurrent(inp))
    assert err <= TOL["f32"], f"rel max err {err:.3e}"

# ------------------------------------------------------------------------------------------------
# Segments: a CTA walks 2^g chunks, the levels above its segment pre-filled from the block
# states the pre-pass builds (segment totals on the tensor cores, then the counter over segments)
# ------------------------------------------------------------------------------------------------
class _forced_segments:
    def __init__(self, chunks):
        self.chunks = chunks

    def __enter__(self):
        binding.set_segment_chunks(self.chunks)

    def __exit__(self, *exc):
        binding.set_segment_chunks(0)


@pytest.mark.parametrize("chunks", [2, 4, 8, 32])
@pytest.mark.parametrize("mode", ["zero", "slow", "dist"])
def test_segments_forced_lengths(chunks, mode):
    # 63 chunks with a ragged tail: segments of 2..32 chunks, up to five levels pre-filled
    w = I.shrink(W["t8k_d64_bf16"], B=2, H=2, T=8000)
    inp = I.make_inputs(w, seed=31, log_a_mode=mode)
    ref = O.llattn_recurrent(inp)
    with _forced_segments(chunks):
        assert binding.segment_plan(inp.B, inp.H, inp.T, inp.dk, inp.dv) == chunks
        _check(inp, ref, "tcgen05")


@pytest.mark.parametrize("level,chunks", [(8, 2), (9, 2), (10, 4), (12, 4), (13, 8), (14, 4)])
def test_segments_one_hot_levels(level, chunks):
    # one level at a time with no decay, T = 16384: levels 8 + b >= 8 + log2(chunks) come
    # entirely from pre-filled blocks, the lower ones from the walk's own merges
    w = I.shrink(W["t8k_d64_bf16"], B=1, H=1, T=16384)
    inp = I.make_inputs(w, seed=32, log_a_mode="zero", lam_mode="onehot", lam_level=level)
    ref = O.llattn_recurrent(inp)
    with _forced_segments(chunks):
        _check(inp, ref, "tcgen05")


def test_segments_packed_batch():
    w = I.Workload("vl_seg", B=6, H=2, T=5000, dk=64, dv=64, dtype="bf16", varlen=True)
    inp = I.make_inputs(w, seed=33, log_a_mode="slow",
                        lengths=np.array([5000, 1, 0, 129, 4096, 2600]))
    ref = O.llattn_recurrent(inp)
    for chunks in (2, 8):
        with _forced_segments(chunks):
            _check(inp, ref, "tcgen05")
    _check(inp, ref, "tcgen05")   # the automatic plan


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128), (128, 64)])
def test_head_dims_128_on_tensor_cores(dk, dv):
    # d_k = 128: two 64-column passes, the second adding into out; d_v = 128: two value tiles
    w = I.Workload("d128", B=1, H=2, T=3000, dk=dk, dv=dv, dtype="bf16")
    for mode in ("slow", "dist"):
        inp = I.make_inputs(w, seed=34, log_a_mode=mode)
        ref = O.llattn_recurrent(inp)
        _check(inp, ref, "tcgen05")
        with _forced_segments(4):
            _check(inp, ref, "tcgen05")


def test_long_context_d128_deep_levels():
    # the 64K-token, d = 128 workload's own decay at T = 32768 (256 chunks, nine chunk levels),
    # one head, every output against the oracle, automatic segments
    w = I.shrink(W["t64k_d128_bf16"], H=1, T=32768)
    inp = I.make_inputs(w, seed=35)
    ref = O.llattn_recurrent(inp)
    assert binding.segment_plan(inp.B, inp.H, inp.T, inp.dk, inp.dv) > 0
    _check(inp, ref, "tcgen05")


# ------------------------------------------------------------------------------------------------
# Short sequences through the automatic path: the one-launch masked form on CUDA cores
# ------------------------------------------------------------------------------------------------
@pytest.mark.parametrize("T,dk,dv,dtype,mode", [
    (256, 32, 32, "f32", "dist"),
    (1, 32, 32, "f32", "dist"),
    (33, 64, 64, "f32", "slow"),
    (500, 128, 64, "f32", "strong"),
    (512, 64, 32, "f32", "zero"),
    (300, 32, 128, "bf16", "dist"),
    (129, 32, 32, "bf16", "slow"),
])
def test_short_sequences_one_launch(T, dk, dv, dtype, mode):
    """T <= 512 where the tensor cores do not apply (fp32, or d_k = 32): the automatic path
    with the default chunk runs the masked form in one launch; every output element against the
    oracle, the last 16-row block ragged where T is not a multiple of 16.  With 2 x 3 heads the
    row blocks number 6 * ceil(T / 16): T <= 192 splits each block's keys over a cluster of 4
    CTAs, T = 256 and 300 over 2, and T = 500 and 512 run one CTA per block."""
    w = I.Workload("short", B=2, H=3, T=T, dk=dk, dv=dv, dtype=dtype)
    inp = I.make_inputs(w, seed=T + dk + dv, log_a_mode=mode)
    ref = O.llattn_quadratic(inp)
    _check(inp, ref, "auto")


def test_short_sequences_packed_one_launch():
    lengths = np.array([0, 1, 100, 512, 37, 64])
    w = I.Workload("short_vl", B=len(lengths), H=2, T=512, dk=32, dv=32, dtype="f32", varlen=True)
    inp = I.make_inputs(w, seed=71, lengths=lengths)
    _check(inp, O.llattn_quadratic(inp), "auto")


def test_short_sequences_packed_cluster_split():
    """Few row blocks (4 sequences of at most 128 tokens, 2 heads): the keys of a block are
    split over a cluster of 4 CTAs, including blocks with fewer key tiles than CTAs."""
    lengths = np.array([0, 1, 100, 37, 128])
    w = I.Workload("short_vl4", B=len(lengths), H=2, T=128, dk=64, dv=64, dtype="f32", varlen=True)
    inp = I.make_inputs(w, seed=73, lengths=lengths)
    _check(inp, O.llattn_quadratic(inp), "auto")


# ------------------------------------------------------------------------------------------------
# A call captured in a CUDA graph (how the benchmark issues its steps) computes what the direct
# call computes
# ------------------------------------------------------------------------------------------------
@pytest.mark.parametrize("name,B,H,T,dtype,dk,segments", [
    ("segmented", 2, 4, 2048, "bf16", 64, True),    # pre-pass kernels and dependent launches
    ("whole", 4, 32, 700, "bf16", 64, False),       # one CTA per (sequence, head)
    ("short", 2, 4, 300, "f32", 32, None),          # the one-launch masked form
])
def test_graph_replay_matches_direct_call(name, B, H, T, dtype, dk, segments):
    import torch
    w = I.Workload("graph_" + name, B=B, H=H, T=T, dk=dk, dv=dk, dtype=dtype)
    inp = I.make_inputs(w, seed=T + dk)
    t = _to_device_for_guard(inp)
    args = (t["q"], t["k"], t["v"], t["log_a"], t["lam"])
    direct = binding.forward(*args)
    torch.cuda.synchronize()
    if segments is not None:
        cut = binding.segment_plan(inp.B, inp.H, inp.T, inp.dk, inp.dv, False) > 0
        assert cut == segments
    out = torch.full_like(direct, float("nan"))
    ws = torch.empty(max(binding.workspace_bytes(1 if dtype == "bf16" else 0, "auto", 0, inp.B,
                                                 inp.H, inp.T, inp.dk, inp.dv, False), 256),
                     dtype=torch.uint8, device="cuda:0")
    binding.forward(*args, out=out, workspace=ws)          # first call outside the capture
    torch.cuda.synchronize()
    out.fill_(float("nan"))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        binding.forward(*args, out=out, workspace=ws)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert binding.stream_status(clear=True) == 0
    assert torch.equal(out, direct), "a replayed call differs from the direct call"
    err = O.rel_max_err(out.double().cpu().numpy(), O.llattn_recurrent(inp))
    assert err <= TOL[inp.dtype], f"rel max err {err:.3e}"
    del g
