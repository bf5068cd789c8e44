"""The C-ABI library loads, exports every declared symbol, and validates arguments (no GPU).

Only entry points that return before touching CUDA are called here.
"""
import ctypes
import os
import re

import pytest

from hierarchical_fenwick_state_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "llattn.h")


def declared_symbols():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"LLATTN_API\s+[\w\s\*]+?\b(llattn_\w+)\s*\(", src)))


def test_header_declares_the_exports():
    decl = declared_symbols()
    assert "llattn_fwd" in decl and "llattn_fwd_f32" in decl
    assert sorted(binding.EXPORTS) == decl


def test_library_exports_every_declared_symbol():
    lib = binding.lib()
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_num_levels_and_strings():
    lib = binding.lib()
    assert [lib.llattn_num_levels(T) for T in (1, 2, 3, 256, 2048, 8192, 16384, 65536)] == \
        [1, 2, 3, 9, 12, 14, 15, 17]
    assert lib.llattn_abi_version() >= 1
    for s in range(9):
        assert lib.llattn_status_str(s)
    assert lib.llattn_status_str(99) == b"unknown status"


def _call_ex(**kw):
    a = dict(in_dtype=1, path=0, chunk=0, q=0x1000, k=0x2000, v=0x3000, log_a=0x4000,
             lam=0x5000, out=0x6000, B=1, H=1, T=16, dk=64, dv=64, cu=None)
    a.update(kw)
    vp = ctypes.c_void_p
    return binding.lib().llattn_fwd_ex(a["in_dtype"], a["path"], a["chunk"], vp(a["q"]), vp(a["k"]),
                                       vp(a["v"]), vp(a["log_a"]), vp(a["lam"]), vp(a["out"]),
                                       a["B"], a["H"], a["T"], a["dk"], a["dv"],
                                       vp(a["cu"]) if a["cu"] else None, None, 0, None)


@pytest.mark.parametrize("kw,status", [
    (dict(dk=48), 2), (dict(dv=256), 2), (dict(T=-1), 2), (dict(B=-2), 2),
    (dict(in_dtype=7), 4), (dict(path=9), 1), (dict(chunk=24, path=1), 1),
    (dict(chunk=128, path=1), 1), (dict(in_dtype=0, path=2), 4),
    (dict(q=0x1008), 3), (dict(out=0x6004), 3), (dict(lam=0x5002), 3),
    (dict(q=0), 1), (dict(out=0x1000), 1),
    # out overlaps lam's range (lam = 16 tokens * 5 levels * 4 B from 0x5000)
    (dict(out=0x5010), 1),
])
def test_argument_errors_before_launch(kw, status):
    assert _call_ex(**kw) == status


def test_empty_problems_are_no_ops():
    assert _call_ex(B=0) == 0
    assert _call_ex(H=0) == 0
    assert _call_ex(T=0) == 0


def test_workspace_query():
    n = binding.workspace_bytes(1, "simt", 64, 2, 4, 1000, 64, 64, False)
    assert n > 0 and n % 256 == 0
    assert binding.workspace_bytes(1, "simt", 64, 0, 4, 1000, 64, 64, False) == 0
    with pytest.raises(binding.LLAttnError):
        binding.workspace_bytes(1, "simt", 64, 1, 4, 1000, 48, 64, False)


def test_tensor_core_path_limits():
    """The pipelined tensor-core kernel takes d_k, d_v in {64, 128} and T <= 131072 (ten chunk
    levels on chip, long sequences walked in segments); the serial cross-check d = 64 and
    T <= 8192.  Beyond that AUTO falls back to the CUDA-core path (no CUDA call)."""
    ws = binding.workspace_bytes
    for T in (1, 8192, 8193, 16384, 65536, 131072):
        ws(binding.BF16, "tcgen05", 0, 2, 4, T, 64, 64, False)
    for dk, dv in ((128, 128), (64, 128), (128, 64)):
        ws(binding.BF16, "tcgen05", 0, 1, 2, 4096, dk, dv, False)
    ws(binding.BF16, "tcgen05_serial", 0, 2, 4, 8192, 64, 64, False)
    for path, T, d in (("tcgen05", 131073, 64), ("tcgen05_serial", 8193, 64),
                       ("tcgen05_serial", 256, 128), ("tcgen05", 256, 32)):
        with pytest.raises(binding.LLAttnError) as e:
            ws(binding.BF16, path, 0, 2, 4, T, d, d, False)
        assert e.value.status == 8   # LLATTN_ERR_UNSUPPORTED
    with pytest.raises(binding.LLAttnError):   # bf16 inputs only
        ws(binding.F32, "tcgen05", 0, 1, 1, 256, 64, 64, False)
    # AUTO resolves without error for every supported shape (CUDA-core fallback beyond the limit)
    for T in (16384, 16385, 65536, 200000):
        ws(binding.BF16, "auto", 0, 1, 16, T, 64, 64, False)
    ws(binding.BF16, "auto", 0, 1, 16, 65536, 128, 128, False)


def test_segment_plan_and_its_scratch():
    """Shapes with fewer whole-sequence walks than SMs are cut into segments (and then need
    scratch for the segment states); the benchmark's B=4, H=32, T=8192 shape is not."""
    plan = binding.segment_plan
    assert plan(4, 32, 8192, 64, 64) == 0
    assert binding.workspace_bytes(binding.BF16, "tcgen05", 0, 4, 32, 8192, 64, 64, False) == 0
    c = plan(1, 16, 65536, 128, 128)
    assert c >= 2 and c & (c - 1) == 0 and c < 512
    assert binding.workspace_bytes(binding.BF16, "tcgen05", 0, 1, 16, 65536, 128, 128, False) > 0
    assert plan(8, 16, 16384, 64, 64, varlen=True) > 0
    assert plan(1, 4, 100, 64, 64) == 0          # a single chunk is never cut
    assert plan(1, 4, 256, 32, 32) == 0          # no tensor-core path for d = 32
    try:
        binding.set_segment_chunks(4)
        assert plan(4, 32, 8192, 64, 64) == 4
        assert plan(1, 1, 512, 64, 64) == 0      # 4 chunks: one segment holds the sequence
        assert binding.workspace_bytes(binding.BF16, "tcgen05", 0, 4, 32, 8192, 64, 64, False) > 0
    finally:
        binding.set_segment_chunks(0)
    assert plan(4, 32, 8192, 64, 64) == 0
    for bad in (-1, 1, 3, 6):
        with pytest.raises(binding.LLAttnError):
            binding.set_segment_chunks(bad)


def _decode(**kw):
    a = dict(in_dtype=1, q=0x1000, k=0x2000, v=0x3000, log_a=0x4000, lam=0x5000, pos=0x5800,
             state=0x10000, out=0x8000, B=2, H=3, L=14, dk=64, dv=64)
    a.update(kw)
    vp = ctypes.c_void_p
    return binding.lib().llattn_decode_step(a["in_dtype"], vp(a["q"]), vp(a["k"]), vp(a["v"]),
                                            vp(a["log_a"]), vp(a["lam"]), vp(a["pos"]),
                                            vp(a["state"]), vp(a["out"]), a["B"], a["H"], a["L"],
                                            a["dk"], a["dv"], None)


def test_decode_state_bytes():
    for B, H, L, dk, dv in ((1, 1, 1, 32, 32), (64, 32, 14, 64, 64), (3, 5, 17, 128, 32)):
        assert binding.decode_state_bytes(B, H, L, dk, dv) == \
            B * H * (L - 1) * dk * dv * 4 + B * H * 2 * (L - 1) * 4
    for bad in ((1, 1, 0, 64, 64), (1, 1, 33, 64, 64), (1, 1, 14, 48, 64), (-1, 1, 14, 64, 64),
                (65536, 1, 14, 64, 64)):
        with pytest.raises(binding.LLAttnError) as e:
            binding.decode_state_bytes(*bad)
        assert e.value.status == 2


@pytest.mark.parametrize("kw,status", [
    (dict(dk=48), 2), (dict(dv=256), 2), (dict(L=0), 2), (dict(L=33), 2), (dict(B=-1), 2),
    (dict(in_dtype=5), 4),
    (dict(q=0), 1), (dict(pos=0), 1), (dict(state=0), 1),
    (dict(q=0x1008), 3), (dict(state=0x10004), 3), (dict(out=0x8008), 3), (dict(pos=0x5802), 3),
    # out overlaps the state (state starts at 0x10000) or lam (6 rows x 14 levels x 4 B at 0x5000)
    (dict(out=0x10100), 1), (dict(out=0x5010), 1),
])
def test_decode_argument_errors_before_launch(kw, status):
    assert _decode(**kw) == status


def test_decode_empty_batches_are_no_ops():
    assert _decode(B=0) == 0
    assert _decode(H=0) == 0


def _prefill(**kw):
    a = dict(in_dtype=1, k=0x2000, v=0x3000, log_a=0x4000, state=0x100000, B=2, H=3, T=40, L=7,
             dk=64, dv=64, cu=None)
    a.update(kw)
    vp = ctypes.c_void_p
    return binding.lib().llattn_prefill_state(a["in_dtype"], vp(a["k"]), vp(a["v"]),
                                              vp(a["log_a"]), vp(a["state"]), a["B"], a["H"],
                                              a["T"], a["L"], a["dk"], a["dv"],
                                              vp(a["cu"]) if a["cu"] else None, None)


@pytest.mark.parametrize("kw,status", [
    (dict(dk=48), 2), (dict(dv=256), 2), (dict(L=0), 2), (dict(L=33), 2), (dict(B=-1), 2),
    (dict(T=-1), 2), (dict(T=(1 << 24) + 1), 2), (dict(in_dtype=7), 4),
    (dict(k=0), 1), (dict(log_a=0), 1), (dict(state=0), 1),
    (dict(k=0x2008), 3), (dict(v=0x3004), 3), (dict(state=0x100004), 3), (dict(log_a=0x4002), 3),
    (dict(cu=0x5002), 3),
    # the state overlaps v (2 x 40 x 3 rows of 64 bf16 at 0x3000)
    (dict(state=0x3100), 1),
])
def test_prefill_argument_errors_before_launch(kw, status):
    assert _prefill(**kw) == status


def test_prefill_empty_batches_are_no_ops():
    assert _prefill(B=0) == 0
    assert _prefill(H=0) == 0


def _bwd(**kw):
    a = dict(in_dtype=1, q=0x1000, k=0x2000, v=0x3000, log_a=0x4000, lam=0x5000, dout=0x6000,
             dq=0x10000, dk=0x20000, dv=0x30000, dlog_a=0x40000, dlam=0x50000, B=1, H=2, T=16,
             dk_dim=64, dv_dim=64, cu=None)
    a.update(kw)
    vp = ctypes.c_void_p
    return binding.lib().llattn_bwd(a["in_dtype"], vp(a["q"]), vp(a["k"]), vp(a["v"]),
                                    vp(a["log_a"]), vp(a["lam"]), vp(a["dout"]), vp(a["dq"]),
                                    vp(a["dk"]), vp(a["dv"]), vp(a["dlog_a"]), vp(a["dlam"]),
                                    a["B"], a["H"], a["T"], a["dk_dim"], a["dv_dim"],
                                    vp(a["cu"]) if a["cu"] else None, None, 0, None)


def test_bwd_workspace_bytes():
    assert binding.bwd_workspace_bytes(4, 32, 8192, 64, 64) == 4 * 32 * 8192 * 8
    assert binding.bwd_workspace_bytes(1, 3, 5, 32, 32) == 256          # rounded up to 256
    assert binding.bwd_workspace_bytes(0, 3, 5, 32, 32) == 0
    assert binding.bwd_workspace_bytes(1, 2, 700, 128, 128) == (2 * 700 * 8 + 255) // 256 * 256
    for bad in ((1, 1, 16, 64, 32), (1, 1, 16, 48, 48), (1, 1, -1, 64, 64)):
        with pytest.raises(binding.LLAttnError) as e:
            binding.bwd_workspace_bytes(*bad)
        assert e.value.status == 2


@pytest.mark.parametrize("kw,status", [
    (dict(dk_dim=32), 2), (dict(dk_dim=128, dv_dim=64), 2), (dict(dk_dim=48, dv_dim=48), 2), (dict(T=-1), 2),
    (dict(in_dtype=3), 4),
    (dict(dout=0), 1), (dict(dlam=0), 1),
    (dict(dq=0x10008), 3), (dict(dout=0x6008), 3), (dict(dlog_a=0x40002), 3),
    # a gradient overlapping an input (dout: 16 tokens x 2 heads x 64 x 2 B from 0x6000) or
    # another gradient (dq: 16 x 2 x 64 x 4 B = 8 KB from 0x10000)
    (dict(dq=0x6100), 1), (dict(dk=0x10400), 1),
])
def test_bwd_argument_errors_before_launch(kw, status):
    assert _bwd(**kw) == status


def test_bwd_empty_problems_are_no_ops():
    assert _bwd(B=0) == 0 and _bwd(H=0) == 0 and _bwd(T=0) == 0


def _gdn(**kw):
    a = dict(in_dtype=1, q=0x1000, k=0x2000, v=0x3000, log_alpha=0x4000, beta=0x4800,
             lam=0x5000, out=0x6000, B=1, H=1, T=16, dk=64, dv=64, cu=None)
    a.update(kw)
    vp = ctypes.c_void_p
    return binding.lib().llattn_gdn_fwd(a["in_dtype"], vp(a["q"]), vp(a["k"]), vp(a["v"]),
                                        vp(a["log_alpha"]), vp(a["beta"]), vp(a["lam"]),
                                        vp(a["out"]), a["B"], a["H"], a["T"], a["dk"], a["dv"],
                                        vp(a["cu"]) if a["cu"] else None, None)


@pytest.mark.parametrize("kw,status", [
    (dict(dk=48), 2), (dict(dv=256), 2), (dict(T=-1), 2), (dict(T=65537), 2),
    (dict(in_dtype=3), 4), (dict(q=0x1002), 3), (dict(beta=0x4802), 3),
    (dict(beta=0), 1), (dict(out=0x1000), 1), (dict(out=0x4800), 1),
])
def test_gdn_argument_errors_before_launch(kw, status):
    assert _gdn(**kw) == status


def test_gdn_empty_problems_are_no_ops():
    assert _gdn(B=0) == 0 and _gdn(H=0) == 0 and _gdn(T=0) == 0

