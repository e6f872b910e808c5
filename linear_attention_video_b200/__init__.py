"""Python binding of libkda.so: the B200 (sm_100a) forward pass of the
modality-aware short convolution followed by the Kimi Delta Attention scan.

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in ``include/kda.h``.  Tensors are torch
CUDA tensors (torch supplies device memory and streams); the functions take
the same names and arguments as the C entry points and raise ``KdaError``
when an entry point returns a non-zero status.  There is no CPU fallback:
importing this package fails if the compiled library is missing.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkda.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libkda.so not found at {LIB_PATH}; build it with "
                      f"`python linear_attention_video_b200/build.py` (nvcc, sm_100a)")

_lib = ctypes.CDLL(LIB_PATH)

KDA_OK, KDA_ERR_INVALID_ARG, KDA_ERR_UNSUPPORTED, KDA_ERR_MISALIGNED = 0, 1, 2, 3
KDA_ERR_WORKSPACE, KDA_ERR_CUDA, KDA_ERR_TIMEOUT, KDA_ERR_DEVICE_ASSERT, KDA_ERR_RANGE = 4, 5, 6, 7, 8
KDA_DT_BF16, KDA_DT_F32 = 0, 1
KDA_FLAG_VIS_CAUSAL_T = 1
KDA_FLAG_REUSE_RECORDS = 2
KDA_FLAG_QKV_F16 = 4

EXPORTS = ("kda_tokens", "kda_workspace_bytes", "kda_shortconv_fwd", "kda_chunk_fwd", "kda_fwd",
           "kda_chunk_fwd_noalloc", "kda_fwd_host_workspace_bytes", "kda_fwd_host", "kda_bwd_workspace_bytes", "kda_bwd", "kda_read_status", "kda_status_str",
           "kda_last_launch_count")


class kda_problem(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("dk", ctypes.c_int32), ("dv", ctypes.c_int32),
                ("text_len", ctypes.c_int64),
                ("grid_t", ctypes.c_int32), ("grid_h", ctypes.c_int32), ("grid_w", ctypes.c_int32),
                ("text_k", ctypes.c_int32),
                ("vis_kt", ctypes.c_int32), ("vis_kh", ctypes.c_int32), ("vis_kw", ctypes.c_int32),
                ("chunk", ctypes.c_int32), ("flags", ctypes.c_uint32)]


_vp, _sz, _i, _pp = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.POINTER(kda_problem)
_lib.kda_tokens.argtypes = [_pp]
_lib.kda_tokens.restype = ctypes.c_int64
_lib.kda_workspace_bytes.argtypes = [_pp, _i]
_lib.kda_workspace_bytes.restype = _sz
_lib.kda_shortconv_fwd.argtypes = [_pp, _i] + [_vp] * 9
_lib.kda_shortconv_fwd.restype = _i
_lib.kda_chunk_fwd.argtypes = [_pp, _i] + [_vp] * 9 + [_sz, _vp]
_lib.kda_chunk_fwd.restype = _i
_lib.kda_fwd.argtypes = [_pp, _i] + [_vp] * 11 + [_sz, _vp]
_lib.kda_fwd.restype = _i
_lib.kda_chunk_fwd_noalloc.argtypes = [_pp, _i] + [_vp] * 10
_lib.kda_chunk_fwd_noalloc.restype = _i
_lib.kda_fwd_host_workspace_bytes.argtypes = [_pp, _i, ctypes.c_int32]
_lib.kda_fwd_host_workspace_bytes.restype = _sz
_lib.kda_fwd_host.argtypes = [_pp, _i] + [_vp] * 10 + [ctypes.c_int32, _vp, _sz, _vp, _vp, _vp]
_lib.kda_fwd_host.restype = _i
_lib.kda_bwd_workspace_bytes.argtypes = [_pp, _i]
_lib.kda_bwd_workspace_bytes.restype = _sz
_lib.kda_bwd.argtypes = [_pp, _i] + [_vp] * 19 + [_sz, _vp]
_lib.kda_bwd.restype = _i
_lib.kda_read_status.argtypes = [_vp, _vp]
_lib.kda_read_status.restype = _i
_lib.kda_status_str.argtypes = [_i]
_lib.kda_status_str.restype = ctypes.c_char_p
_lib.kda_last_launch_count.argtypes = []
_lib.kda_last_launch_count.restype = _i


class KdaError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {kda_status_str(status)} (status {status})")
        self.status = status


def problem(B, H, d, text_len, grid, text_k=4, vis_k=(3, 3, 3), chunk=64, vis_causal_t=False,
            dv=None, reuse_records=False, qkv_f16=False) -> kda_problem:
    T, Hg, Wg = grid
    flags = ((KDA_FLAG_VIS_CAUSAL_T if vis_causal_t else 0) | (KDA_FLAG_REUSE_RECORDS if reuse_records else 0)
             | (KDA_FLAG_QKV_F16 if qkv_f16 else 0))
    return kda_problem(B, H, d, d if dv is None else dv, text_len, T, Hg, Wg, text_k,
                       vis_k[0], vis_k[1], vis_k[2], chunk, flags)


def _dt(dtype) -> int:
    if dtype == torch.bfloat16:
        return KDA_DT_BF16
    if dtype == torch.float32:
        return KDA_DT_F32
    raise TypeError(f"unsupported dtype {dtype}")


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int, where: str):
    if rc != KDA_OK:
        raise KdaError(rc, where)


def kda_status_str(status: int) -> str:
    return _lib.kda_status_str(status).decode()


def kda_tokens(p: kda_problem) -> int:
    return _lib.kda_tokens(ctypes.byref(p))


def kda_workspace_bytes(p: kda_problem, dtype) -> int:
    return _lib.kda_workspace_bytes(ctypes.byref(p), _dt(dtype) if not isinstance(dtype, int) else dtype)


def kda_last_launch_count() -> int:
    return _lib.kda_last_launch_count()


def alloc_workspace(p: kda_problem, dtype, device="cuda") -> torch.Tensor:
    n = kda_workspace_bytes(p, dtype)
    if n == 0:
        raise KdaError(KDA_ERR_INVALID_ARG, "kda_workspace_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device)


def kda_shortconv_fwd(p, q, k, v, w_text, w_vis, q_out, k_out, v_out, stream=None):
    _check(_lib.kda_shortconv_fwd(ctypes.byref(p), _dt(q.dtype), _ptr(q), _ptr(k), _ptr(v), _ptr(w_text),
                                  _ptr(w_vis), _ptr(q_out), _ptr(k_out), _ptr(v_out), _stream(stream)),
           "kda_shortconv_fwd")


def kda_chunk_fwd(p, q, k, v, log_alpha, beta, o, workspace, initial_state=None, final_state=None,
                  stream=None, workspace_bytes=None):
    nbytes = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    # the problem dtype is o's (q, k, v may be fp16 under KDA_FLAG_QKV_F16)
    _check(_lib.kda_chunk_fwd(ctypes.byref(p), _dt(o.dtype), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha),
                              _ptr(beta), _ptr(initial_state), _ptr(o), _ptr(final_state), _ptr(workspace),
                              nbytes, _stream(stream)),
           "kda_chunk_fwd")


def kda_fwd(p, q, k, v, log_alpha, beta, w_text, w_vis, o, workspace, initial_state=None, final_state=None,
            stream=None, workspace_bytes=None):
    nbytes = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check(_lib.kda_fwd(ctypes.byref(p), _dt(q.dtype), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                        _ptr(w_text), _ptr(w_vis), _ptr(initial_state), _ptr(o), _ptr(final_state),
                        _ptr(workspace), nbytes, _stream(stream)),
           "kda_fwd")


def kda_fwd_host_workspace_bytes(p: kda_problem, dtype, seg_frames: int) -> int:
    return _lib.kda_fwd_host_workspace_bytes(ctypes.byref(p), _dt(dtype), int(seg_frames))


def alloc_fwd_host_workspace(p: kda_problem, dtype, seg_frames: int, device="cuda") -> torch.Tensor:
    n = kda_fwd_host_workspace_bytes(p, dtype, seg_frames)
    if n == 0:
        raise KdaError(KDA_ERR_INVALID_ARG, "kda_fwd_host_workspace_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device)


def kda_fwd_host(p, q, k, v, log_alpha, beta, w_text, w_vis, o, workspace, seg_frames, initial_state=None,
                 final_state=None, stream=None, copy_in_stream=None, copy_out_stream=None, workspace_bytes=None):
    """kda_fwd on host tensors (q, k, v, log_alpha, beta, o on the CPU, pinned for overlap); the weights,
    the states and the workspace are on the device."""
    nbytes = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check(_lib.kda_fwd_host(ctypes.byref(p), _dt(q.dtype), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                             _ptr(w_text), _ptr(w_vis), _ptr(initial_state), _ptr(o), _ptr(final_state),
                             int(seg_frames), _ptr(workspace), nbytes, _stream(stream), _stream(copy_in_stream),
                             _stream(copy_out_stream)),
           "kda_fwd_host")


def kda_chunk_fwd_noalloc(p, q, k, v, log_alpha, beta, o, initial_state=None, final_state=None,
                          device_status=None, stream=None):
    """kda_chunk_fwd without a workspace: scratch is the library's static device
    array (see include/kda.h for its limit and sharing rules)."""
    _check(_lib.kda_chunk_fwd_noalloc(ctypes.byref(p), _dt(o.dtype), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha),
                                      _ptr(beta), _ptr(initial_state), _ptr(o), _ptr(final_state),
                                      _ptr(device_status), _stream(stream)),
           "kda_chunk_fwd_noalloc")


def kda_bwd_workspace_bytes(p: kda_problem, dtype) -> int:
    return _lib.kda_bwd_workspace_bytes(ctypes.byref(p), _dt(dtype))


def alloc_bwd_workspace(p: kda_problem, dtype, device="cuda") -> torch.Tensor:
    n = kda_bwd_workspace_bytes(p, dtype)
    if n == 0:
        raise KdaError(KDA_ERR_INVALID_ARG, "kda_bwd_workspace_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device)


def kda_bwd(p, q, k, v, log_alpha, beta, w_text, w_vis, d_o, dq, dk, dv, d_log_alpha, d_beta, d_w_text, d_w_vis,
            workspace, initial_state=None, d_final_state=None, d_initial_state=None, stream=None,
            workspace_bytes=None):
    nbytes = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check(_lib.kda_bwd(ctypes.byref(p), _dt(q.dtype), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                        _ptr(w_text), _ptr(w_vis), _ptr(initial_state), _ptr(d_o), _ptr(d_final_state), _ptr(dq),
                        _ptr(dk), _ptr(dv), _ptr(d_log_alpha), _ptr(d_beta), _ptr(d_w_text), _ptr(d_w_vis),
                        _ptr(d_initial_state), _ptr(workspace), nbytes, _stream(stream)),
           "kda_bwd")


def kda_read_status(workspace, stream=None) -> int:
    return _lib.kda_read_status(_ptr(workspace), _stream(stream))
