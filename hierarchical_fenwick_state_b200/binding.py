"""Thin Python binding of the C ABI in include/llattn.h (argument marshalling only).

Every step of the forward runs in libllattn.so's CUDA kernels; this module
only checks tensors, passes raw device pointers, sizes and the current CUDA
stream, and turns status codes into exceptions.  There is no CPU fallback:
if the library is missing, ``lib()`` raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libllattn.so")

F32, BF16 = 0, 1
PATHS = {"auto": 0, "simt": 1, "tcgen05": 2, "tcgen05_serial": 3}

# Every symbol include/llattn.h declares.
EXPORTS = (
    "llattn_abi_version", "llattn_status_str", "llattn_num_levels", "llattn_fwd",
    "llattn_fwd_f32", "llattn_workspace_bytes", "llattn_fwd_ex", "llattn_device_status",
    "llattn_last_cuda_error", "llattn_fwd_host", "llattn_profile", "llattn_profile_read",
    "llattn_fwd_noalloc", "llattn_decode_state_bytes", "llattn_decode_step",
    "llattn_bwd_workspace_bytes", "llattn_bwd", "llattn_fwd_bf16", "llattn_stream_status",
    "llattn_segment_plan", "llattn_set_segment_chunks", "llattn_gdn_fwd",
    "llattn_prefill_state",
)

NOALLOC_SCRATCH_BYTES = 32 << 20  # LLATTN_NOALLOC_SCRATCH_BYTES

_lib = None


class LLAttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib().llattn_status_str(status).decode()
        if status == 5:
            msg += f" (cudaError {lib().llattn_last_cuda_error()})"
        super().__init__(f"{where}: {msg} [status {status}]")


def lib():
    """Load libllattn.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m hierarchical_fenwick_state_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i, f_p, i_p = ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p
    L.llattn_abi_version.restype = i
    L.llattn_status_str.restype = ctypes.c_char_p
    L.llattn_status_str.argtypes = [i]
    L.llattn_num_levels.restype = i
    L.llattn_num_levels.argtypes = [i]
    L.llattn_fwd.restype = i
    L.llattn_fwd.argtypes = [vp, vp, vp, f_p, f_p, f_p, i, i, i, i, i, i_p, vp]
    L.llattn_fwd_f32.restype = i
    L.llattn_fwd_f32.argtypes = [vp, vp, vp, f_p, f_p, f_p, i, i, i, i, i, i_p, vp]
    L.llattn_workspace_bytes.restype = i
    L.llattn_workspace_bytes.argtypes = [i, i, i, i, i, i, i, i, i, ctypes.POINTER(ctypes.c_size_t)]
    L.llattn_fwd_ex.restype = i
    L.llattn_fwd_ex.argtypes = [i, i, i, vp, vp, vp, f_p, f_p, f_p, i, i, i, i, i, i_p, vp,
                                ctypes.c_size_t, vp]
    L.llattn_device_status.restype = i
    L.llattn_device_status.argtypes = [ctypes.POINTER(ctypes.c_uint), i]
    L.llattn_last_cuda_error.restype = i
    L.llattn_fwd_host.restype = i
    L.llattn_fwd_host.argtypes = [i, vp, vp, vp, f_p, f_p, f_p, i, i, i, i, i, i_p, vp]
    L.llattn_fwd_noalloc.restype = i
    L.llattn_fwd_noalloc.argtypes = [i, vp, vp, vp, f_p, f_p, f_p, i, i, i, i, i, i_p, vp]
    L.llattn_decode_state_bytes.restype = i
    L.llattn_decode_state_bytes.argtypes = [i, i, i, i, i, ctypes.POINTER(ctypes.c_size_t)]
    L.llattn_decode_step.restype = i
    L.llattn_decode_step.argtypes = [i, vp, vp, vp, f_p, f_p, i_p, f_p, f_p, i, i, i, i, i, vp]
    L.llattn_prefill_state.restype = i
    L.llattn_prefill_state.argtypes = [i, vp, vp, f_p, f_p, i, i, i, i, i, i, i_p, vp]
    L.llattn_bwd_workspace_bytes.restype = i
    L.llattn_bwd_workspace_bytes.argtypes = [i, i, i, i, i, ctypes.POINTER(ctypes.c_size_t)]
    L.llattn_bwd.restype = i
    L.llattn_bwd.argtypes = [i, vp, vp, vp, f_p, f_p, vp, f_p, f_p, f_p, f_p, f_p, i, i, i, i, i,
                             i_p, vp, ctypes.c_size_t, vp]
    L.llattn_fwd_bf16.restype = i
    L.llattn_fwd_bf16.argtypes = [vp, vp, vp, f_p, f_p, f_p, i, i, i, i, i, i_p, vp]
    L.llattn_stream_status.restype = i
    L.llattn_stream_status.argtypes = [ctypes.POINTER(ctypes.c_uint), i, vp]
    L.llattn_gdn_fwd.restype = i
    L.llattn_gdn_fwd.argtypes = [i, vp, vp, vp, f_p, f_p, f_p, f_p, i, i, i, i, i, i_p, vp]
    L.llattn_segment_plan.restype = i
    L.llattn_segment_plan.argtypes = [i, i, i, i, i, i, ctypes.POINTER(ctypes.c_int)]
    L.llattn_set_segment_chunks.restype = i
    L.llattn_set_segment_chunks.argtypes = [i]
    L.llattn_profile.restype = i
    L.llattn_profile.argtypes = [i]
    L.llattn_profile_read.restype = i
    L.llattn_profile_read.argtypes = [ctypes.POINTER(ctypes.c_double),
                                      ctypes.POINTER(ctypes.c_longlong),
                                      ctypes.POINTER(ctypes.c_longlong), i]
    _lib = L
    return L


def num_levels(T: int) -> int:
    return int(lib().llattn_num_levels(int(T)))


def _check(st: int, where: str):
    if st != 0:
        raise LLAttnError(st, where)


def workspace_bytes(in_dtype: int, path: str, chunk: int, B: int, H: int, T: int, dk: int,
                    dv: int, varlen: bool) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().llattn_workspace_bytes(in_dtype, PATHS[path], chunk, B, H, T, dk, dv,
                                        int(varlen), ctypes.byref(n)), "llattn_workspace_bytes")
    return int(n.value)


def _stream_handle(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def forward(q, k, v, log_a, lam, *, cu_seqlens=None, T: Optional[int] = None, out=None,
            path: str = "auto", chunk: int = 0, workspace=None, stream=None):
    """o = llattn forward on device tensors (torch).  Returns out (fp32).

    Dense: q,k [B,T,H,dk], v [B,T,H,dv], log_a [B,T,H], lam [B,T,H,L].
    Packed: q,k [total,H,dk] ..., cu_seqlens int32 [B+1] on the device, and T
    the bound on every sequence length.
    """
    import torch
    dtype = q.dtype
    if dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("q/k/v must be bf16 or fp32")
    for t in (q, k, v, log_a, lam):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("inputs must be contiguous CUDA tensors")
    if k.dtype != dtype or v.dtype != dtype:
        raise TypeError("q, k, v must share a dtype")
    if log_a.dtype != torch.float32 or lam.dtype != torch.float32:
        raise TypeError("log_a and lam must be fp32")
    if cu_seqlens is None:
        B, Tq, H, dk = q.shape
        T = Tq
    else:
        if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda:
            raise TypeError("cu_seqlens must be an int32 CUDA tensor")
        B = cu_seqlens.numel() - 1
        _, H, dk = q.shape
        if T is None:
            raise ValueError("varlen needs T (max sequence length bound)")
    dv = v.shape[-1]
    if out is None:
        out = torch.empty(v.shape, dtype=torch.float32, device=v.device)
    ws_ptr, ws_n = None, 0
    if workspace is not None:
        ws_ptr, ws_n = ctypes.c_void_p(workspace.data_ptr()), workspace.numel() * workspace.element_size()
    in_dtype = BF16 if dtype == torch.bfloat16 else F32
    cu_ptr = ctypes.c_void_p(cu_seqlens.data_ptr()) if cu_seqlens is not None else None
    st = lib().llattn_fwd_ex(in_dtype, PATHS[path], int(chunk), ctypes.c_void_p(q.data_ptr()),
                             ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()),
                             ctypes.c_void_p(log_a.data_ptr()), ctypes.c_void_p(lam.data_ptr()),
                             ctypes.c_void_p(out.data_ptr()), int(B), int(H), int(T), int(dk),
                             int(dv), cu_ptr, ws_ptr, ws_n, _stream_handle(stream))
    _check(st, "llattn_fwd_ex")
    return out


def fwd(q, k, v, log_a, lam, out, B, H, T, dk, dv, cu_seqlens=None, stream=None):
    """Direct call of llattn_fwd (bf16 inputs, default path) on raw tensors."""
    st = lib().llattn_fwd(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                          ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(log_a.data_ptr()),
                          ctypes.c_void_p(lam.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                          int(B), int(H), int(T), int(dk), int(dv),
                          ctypes.c_void_p(cu_seqlens.data_ptr()) if cu_seqlens is not None else None,
                          _stream_handle(stream))
    _check(st, "llattn_fwd")
    return out


def fwd_bf16(q, k, v, log_a, lam, out, B, H, T, dk, dv, cu_seqlens=None, stream=None):
    """Direct call of llattn_fwd_bf16 (the same call as llattn_fwd)."""
    st = lib().llattn_fwd_bf16(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                               ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(log_a.data_ptr()),
                               ctypes.c_void_p(lam.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                               int(B), int(H), int(T), int(dk), int(dv),
                               ctypes.c_void_p(cu_seqlens.data_ptr()) if cu_seqlens is not None else None,
                               _stream_handle(stream))
    _check(st, "llattn_fwd_bf16")
    return out


def fwd_f32(q, k, v, log_a, lam, out, B, H, T, dk, dv, cu_seqlens=None, stream=None):
    st = lib().llattn_fwd_f32(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                              ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(log_a.data_ptr()),
                              ctypes.c_void_p(lam.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                              int(B), int(H), int(T), int(dk), int(dv),
                              ctypes.c_void_p(cu_seqlens.data_ptr()) if cu_seqlens is not None else None,
                              _stream_handle(stream))
    _check(st, "llattn_fwd_f32")
    return out


def fwd_host(in_dtype: int, q, k, v, log_a, lam, out, B, H, T, dk, dv, cu_seqlens=None,
             stream=None):
    """llattn_fwd_host on host buffers (numpy arrays or pinned CPU tensors; q/k/v as
    uint16 bf16 bit patterns for in_dtype=BF16).  Copies in, computes, copies out."""
    def ptr(x):
        if x is None:
            return None
        if hasattr(x, "data_ptr"):
            return ctypes.c_void_p(x.data_ptr())
        return ctypes.c_void_p(x.ctypes.data)
    st = lib().llattn_fwd_host(in_dtype, ptr(q), ptr(k), ptr(v), ptr(log_a), ptr(lam), ptr(out),
                               int(B), int(H), int(T), int(dk), int(dv), ptr(cu_seqlens),
                               _stream_handle(stream) if stream is not None else None)
    _check(st, "llattn_fwd_host")
    return out


def fwd_noalloc(q, k, v, log_a, lam, out, B, H, T, dk, dv, cu_seqlens=None, stream=None):
    """Direct call of llattn_fwd_noalloc on raw device tensors (bf16 or fp32 q/k/v):
    the forward with no device allocation, scratch from the library's fixed array."""
    in_dtype = BF16 if str(q.dtype) == "torch.bfloat16" else F32
    st = lib().llattn_fwd_noalloc(in_dtype, ctypes.c_void_p(q.data_ptr()),
                                  ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()),
                                  ctypes.c_void_p(log_a.data_ptr()),
                                  ctypes.c_void_p(lam.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                                  int(B), int(H), int(T), int(dk), int(dv),
                                  ctypes.c_void_p(cu_seqlens.data_ptr()) if cu_seqlens is not None
                                  else None, _stream_handle(stream))
    _check(st, "llattn_fwd_noalloc")
    return out


def decode_state_bytes(B: int, H: int, L: int, dk: int, dv: int) -> int:
    """Bytes of the decoding state buffer (llattn_decode_state_bytes)."""
    n = ctypes.c_size_t(0)
    _check(lib().llattn_decode_state_bytes(int(B), int(H), int(L), int(dk), int(dv),
                                           ctypes.byref(n)), "llattn_decode_state_bytes")
    return int(n.value)


def decode_step(q, k, v, log_a, lam, pos, state, out, B, H, L, dk, dv, stream=None):
    """Direct call of llattn_decode_step on raw device tensors: one new token per sequence.

    q, k [B,H,dk] and v [B,H,dv] (bf16 or fp32), log_a [B,H] and lam [B,H,L] fp32, pos int32
    [B] (tokens each sequence has absorbed; read only), state fp32 of decode_state_bytes()
    bytes (kept between steps), out fp32 [B,H,dv]."""
    in_dtype = BF16 if str(q.dtype) == "torch.bfloat16" else F32
    st = lib().llattn_decode_step(in_dtype, ctypes.c_void_p(q.data_ptr()),
                                  ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()),
                                  ctypes.c_void_p(log_a.data_ptr()),
                                  ctypes.c_void_p(lam.data_ptr()), ctypes.c_void_p(pos.data_ptr()),
                                  ctypes.c_void_p(state.data_ptr()),
                                  ctypes.c_void_p(out.data_ptr()), int(B), int(H), int(L),
                                  int(dk), int(dv), _stream_handle(stream))
    _check(st, "llattn_decode_step")
    return out


def prefill_state(k, v, log_a, state, B, H, T, L, dk, dv, cu_seqlens=None, stream=None):
    """Direct call of llattn_prefill_state: the decoding state of every sequence at the
    position equal to its length (a prompt's hand-off to decode_step).

    k, v dense [B,T,H,d] or packed [total,H,d] (bf16 or fp32) as the forward takes them,
    log_a fp32 [..,H], state fp32 of decode_state_bytes(B,H,L,dk,dv) bytes (written),
    cu_seqlens int32 [B+1] or None."""
    in_dtype = BF16 if str(k.dtype) == "torch.bfloat16" else F32
    st = lib().llattn_prefill_state(in_dtype, ctypes.c_void_p(k.data_ptr()),
                                    ctypes.c_void_p(v.data_ptr()),
                                    ctypes.c_void_p(log_a.data_ptr()),
                                    ctypes.c_void_p(state.data_ptr()), int(B), int(H), int(T),
                                    int(L), int(dk), int(dv),
                                    ctypes.c_void_p(cu_seqlens.data_ptr())
                                    if cu_seqlens is not None else None,
                                    _stream_handle(stream))
    _check(st, "llattn_prefill_state")
    return state


def bwd_workspace_bytes(B: int, H: int, T: int, dk: int, dv: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().llattn_bwd_workspace_bytes(int(B), int(H), int(T), int(dk), int(dv),
                                            ctypes.byref(n)), "llattn_bwd_workspace_bytes")
    return int(n.value)


def backward(q, k, v, log_a, lam, dout, *, cu_seqlens=None, T: Optional[int] = None,
             grads=None, workspace=None, stream=None):
    """Gradients of sum(dout * out) through llattn_bwd, on device tensors (torch).

    Shapes as in forward(); dout like out, in the dtype of q.  Returns a dict of fp32 tensors
    q, k, v, log_a, lam (or fills `grads`, a dict of preallocated ones)."""
    import torch
    in_dtype = BF16 if q.dtype == torch.bfloat16 else F32
    for t in (q, k, v, log_a, lam, dout):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("inputs must be contiguous CUDA tensors")
    if k.dtype != q.dtype or v.dtype != q.dtype or dout.dtype != q.dtype:
        raise TypeError("q, k, v and dout must share a dtype")
    if cu_seqlens is None:
        B, T, H, dk = q.shape
    else:
        B = cu_seqlens.numel() - 1
        _, H, dk = q.shape
        if T is None:
            raise ValueError("varlen needs T (max sequence length bound)")
    dv = v.shape[-1]
    if grads is None:
        grads = {n: torch.empty(x.shape, dtype=torch.float32, device=x.device)
                 for n, x in (("q", q), ("k", k), ("v", v), ("log_a", log_a), ("lam", lam))}
    ws_ptr, ws_n = None, 0
    if workspace is not None:
        ws_ptr, ws_n = ctypes.c_void_p(workspace.data_ptr()), workspace.numel() * workspace.element_size()
    P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = lib().llattn_bwd(in_dtype, P(q), P(k), P(v), P(log_a), P(lam), P(dout), P(grads["q"]),
                          P(grads["k"]), P(grads["v"]), P(grads["log_a"]), P(grads["lam"]),
                          int(B), int(H), int(T), int(dk), int(dv),
                          P(cu_seqlens) if cu_seqlens is not None else None, ws_ptr, ws_n,
                          _stream_handle(stream))
    _check(st, "llattn_bwd")
    return grads


def profile(enable: bool):
    _check(lib().llattn_profile(int(enable)), "llattn_profile")


def profile_read(reset: bool = True):
    """(main-kernel device ms summed, main-kernel launches timed, total kernel launches)."""
    ms, n, tot = ctypes.c_double(0), ctypes.c_longlong(0), ctypes.c_longlong(0)
    _check(lib().llattn_profile_read(ctypes.byref(ms), ctypes.byref(n), ctypes.byref(tot),
                                     int(reset)), "llattn_profile_read")
    return float(ms.value), int(n.value), int(tot.value)


def device_status(clear: bool = True) -> int:
    flags = ctypes.c_uint(0)
    st = lib().llattn_device_status(ctypes.byref(flags), int(clear))
    if st not in (0, 6):
        _check(st, "llattn_device_status")
    return int(flags.value)


def gdn_forward(q, k, v, log_alpha, beta, lam, *, cu_seqlens=None, T: Optional[int] = None,
                out=None, stream=None):
    """Log-Linear Gated DeltaNet forward (llattn_gdn_fwd) on device tensors; returns out (fp32).
    Layouts as ``forward``; log_alpha and beta are [.., H] fp32."""
    import torch
    if q.dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("q/k/v must be bf16 or fp32")
    for t in (q, k, v, log_alpha, beta, lam):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("inputs must be contiguous CUDA tensors")
    H, dk, dv = q.shape[-2], q.shape[-1], v.shape[-1]
    if cu_seqlens is None:
        B, T = q.shape[0], q.shape[1]
    else:
        B = cu_seqlens.numel() - 1
        if T is None:
            raise ValueError("packed inputs need T (the bound on every length)")
    if out is None:
        out = torch.empty(v.shape, dtype=torch.float32, device=v.device)
    in_dtype = BF16 if q.dtype == torch.bfloat16 else F32
    cu_ptr = ctypes.c_void_p(cu_seqlens.data_ptr()) if cu_seqlens is not None else None
    st = lib().llattn_gdn_fwd(in_dtype, ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                              ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(log_alpha.data_ptr()),
                              ctypes.c_void_p(beta.data_ptr()), ctypes.c_void_p(lam.data_ptr()),
                              ctypes.c_void_p(out.data_ptr()), int(B), int(H), int(T), int(dk),
                              int(dv), cu_ptr, _stream_handle(stream))
    _check(st, "llattn_gdn_fwd")
    return out


def segment_plan(B: int, H: int, T: int, dk: int, dv: int, varlen: bool = False) -> int:
    """Chunks per segment of a tensor-core call of this shape (0: whole sequences per CTA)."""
    n = ctypes.c_int(0)
    _check(lib().llattn_segment_plan(B, H, T, dk, dv, int(varlen), ctypes.byref(n)),
           "llattn_segment_plan")
    return int(n.value)


def set_segment_chunks(chunks: int) -> None:
    """Force the tensor-core path's segment length (0: automatic)."""
    _check(lib().llattn_set_segment_chunks(int(chunks)), "llattn_set_segment_chunks")


def stream_status(clear: bool = True, stream=None) -> int:
    """llattn_stream_status: the status word, read in order on one stream (no device sync)."""
    flags = ctypes.c_uint(0)
    st = lib().llattn_stream_status(ctypes.byref(flags), int(clear), _stream_handle(stream))
    if st not in (0, 6):
        _check(st, "llattn_stream_status")
    return int(flags.value)
