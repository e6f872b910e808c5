"""Python binding of libkda.so: the B200 (sm_100a) forward pass of the
modality-aware short convolution followed by the Kimi Delta Attention scan.

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in ``include/kda.h``.  Tensors are torch
CUDA tensors (torch supplies device memory and streams); the functions take
the same names and arguments as the C entry points and raise ``KdaError``
when an entry point returns a non-zero status.  The C ABI receives bare
addresses and cannot see buffer sizes, so every tensor is first checked
against the problem (element count, dtype, device, contiguity); a mismatch
raises ``KdaError(KDA_ERR_INVALID_ARG)`` before anything is launched.  There
is no CPU fallback: importing this package fails if the compiled library is
missing.
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
           "kda_chunk_fwd_noalloc", "kda_fwd_host_workspace_bytes", "kda_fwd_host", "kda_bwd_workspace_bytes",
           "kda_bwd", "kda_selftest_wait_timeout", "kda_read_status", "kda_status_str", "kda_last_launch_count")


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
_lib.kda_selftest_wait_timeout.argtypes = [_pp, _i] + [_vp] * 7 + [_sz, ctypes.c_int32, ctypes.c_uint32, _vp]
_lib.kda_selftest_wait_timeout.restype = _i
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


# ---------------------------------------------------------------------------
# argument checks: the C ABI takes bare addresses, so sizes are checked here
# ---------------------------------------------------------------------------
def _dims(p: kda_problem):
    n = _lib.kda_tokens(ctypes.byref(p))
    if n < 0 or p.B < 1 or p.H < 1 or p.dk < 1 or p.dv < 1:
        raise KdaError(KDA_ERR_INVALID_ARG, "problem")
    return p.B, n, p.H, p.dk, p.dv


class _Args:
    """Collects the tensor arguments of one call and checks them against the problem."""

    def __init__(self, where: str, device: str = "cuda"):
        self.where, self.device, self.seen = where, device, []

    def fail(self, msg):
        raise KdaError(KDA_ERR_INVALID_ARG, f"{self.where}: {msg}")

    def add(self, name, t, numel, dtypes, device=None, at_least=False):
        if t is None or isinstance(t, int):   # optional argument absent, or a caller-managed raw address
            return self
        if not isinstance(t, torch.Tensor):
            self.fail(f"{name} must be a torch tensor")
        if numel > 0:   # zero-size arguments take any placeholder (the ABI wants a non-NULL address)
            if (t.numel() < numel) if at_least else (t.numel() != numel):
                self.fail(f"{name} has {t.numel()} elements, the problem needs {numel}")
            if t.dtype not in dtypes:
                self.fail(f"{name} has dtype {t.dtype}, expected {' or '.join(map(str, dtypes))}")
        if not t.is_contiguous():
            self.fail(f"{name} must be contiguous")
        self.seen.append((name, t, device or self.device))
        return self

    def check_devices(self):
        cuda = [(n, t) for n, t, dev in self.seen if dev == "cuda"]
        for n, t, dev in self.seen:
            if t.device.type != dev:
                self.fail(f"{n} must be a {dev.upper()} tensor, got {t.device}")
        if cuda:
            idx = {t.device.index for _, t in cuda}
            if len(idx) != 1:
                self.fail("device tensors on different GPUs")
            if idx.pop() != torch.cuda.current_device():
                self.fail("device tensors are not on the current CUDA device")


def _act_dtypes(p: kda_problem, dtype):
    """Element types of the convolved activations: fp16 under KDA_FLAG_QKV_F16, else the problem's."""
    return (torch.float16,) if p.flags & KDA_FLAG_QKV_F16 else (dtype,)


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
    B, N, H, dk, dv = _dims(p)
    dt = q.dtype
    a = _Args("kda_shortconv_fwd")
    for n, t, d in (("q", q, dk), ("k", k, dk), ("v", v, dv)):
        a.add(n, t, B * N * H * d, (dt,))
    for n, t, d in (("q_out", q_out, dk), ("k_out", k_out, dk), ("v_out", v_out, dv)):
        a.add(n, t, B * N * H * d, _act_dtypes(p, dt))
    a.add("w_text", w_text, 3 * H * dk * p.text_k, (torch.float32,))
    a.add("w_vis", w_vis, 3 * H * dk * p.vis_kt * p.vis_kh * p.vis_kw, (torch.float32,))
    a.check_devices()
    _check(_lib.kda_shortconv_fwd(ctypes.byref(p), _dt(q.dtype), _ptr(q), _ptr(k), _ptr(v), _ptr(w_text),
                                  _ptr(w_vis), _ptr(q_out), _ptr(k_out), _ptr(v_out), _stream(stream)),
           "kda_shortconv_fwd")


def _scan_args(where, p, dtype, q, k, v, log_alpha, beta, o, s0, sn, workspace, nbytes, act_dtypes, host=False):
    B, N, H, dk, dv = _dims(p)
    dev = "cpu" if host else "cuda"
    a = _Args(where)
    a.add("q", q, B * N * H * dk, act_dtypes, dev).add("k", k, B * N * H * dk, act_dtypes, dev)
    a.add("v", v, B * N * H * dv, act_dtypes, dev)
    a.add("log_alpha", log_alpha, B * N * H * dk, (torch.float32,), dev)
    a.add("beta", beta, B * N * H, (dtype,), dev).add("o", o, B * N * H * dv, (dtype,), dev)
    a.add("initial_state", s0, B * H * dk * dv, (torch.float32,))
    a.add("final_state", sn, B * H * dk * dv, (torch.float32,))
    if workspace is not None and not isinstance(workspace, int):
        a.add("workspace", workspace, 1, (workspace.dtype,), at_least=True)
        if workspace.numel() * workspace.element_size() < nbytes:
            a.fail(f"workspace holds {workspace.numel() * workspace.element_size()} bytes, fewer than the "
                   f"{nbytes} passed")
    return a


def kda_chunk_fwd(p, q, k, v, log_alpha, beta, o, workspace, initial_state=None, final_state=None,
                  stream=None, workspace_bytes=None):
    nbytes = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    # the problem dtype is o's (q, k, v may be fp16 under KDA_FLAG_QKV_F16)
    _scan_args("kda_chunk_fwd", p, o.dtype, q, k, v, log_alpha, beta, o, initial_state, final_state, workspace,
               nbytes, _act_dtypes(p, o.dtype)).check_devices()
    _check(_lib.kda_chunk_fwd(ctypes.byref(p), _dt(o.dtype), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha),
                              _ptr(beta), _ptr(initial_state), _ptr(o), _ptr(final_state), _ptr(workspace),
                              nbytes, _stream(stream)),
           "kda_chunk_fwd")


def _weight_args(a, p, w_text, w_vis):
    H, dk = p.H, p.dk
    a.add("w_text", w_text, 3 * H * dk * p.text_k, (torch.float32,))
    return a.add("w_vis", w_vis, 3 * H * dk * p.vis_kt * p.vis_kh * p.vis_kw, (torch.float32,))


def kda_fwd(p, q, k, v, log_alpha, beta, w_text, w_vis, o, workspace, initial_state=None, final_state=None,
            stream=None, workspace_bytes=None):
    nbytes = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    a = _scan_args("kda_fwd", p, q.dtype, q, k, v, log_alpha, beta, o, initial_state, final_state, workspace,
                   nbytes, (q.dtype,))
    _weight_args(a, p, w_text, w_vis).check_devices()
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
    a = _scan_args("kda_fwd_host", p, q.dtype, q, k, v, log_alpha, beta, o, initial_state, final_state, workspace,
                   nbytes, (q.dtype,), host=True)
    _weight_args(a, p, w_text, w_vis).check_devices()
    _check(_lib.kda_fwd_host(ctypes.byref(p), _dt(q.dtype), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                             _ptr(w_text), _ptr(w_vis), _ptr(initial_state), _ptr(o), _ptr(final_state),
                             int(seg_frames), _ptr(workspace), nbytes, _stream(stream), _stream(copy_in_stream),
                             _stream(copy_out_stream)),
           "kda_fwd_host")


def kda_chunk_fwd_noalloc(p, q, k, v, log_alpha, beta, o, initial_state=None, final_state=None,
                          device_status=None, stream=None):
    """kda_chunk_fwd without a workspace: scratch is the library's static device
    array (see include/kda.h for its limit and sharing rules)."""
    a = _scan_args("kda_chunk_fwd_noalloc", p, o.dtype, q, k, v, log_alpha, beta, o, initial_state, final_state,
                   None, 0, _act_dtypes(p, o.dtype))
    a.add("device_status", device_status, 1, (torch.int32, torch.uint32), at_least=True).check_devices()
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
    dk_, dv_ = dk, dv
    nbytes = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    a = _scan_args("kda_bwd", p, q.dtype, q, k, v, log_alpha, beta, d_o, initial_state, d_final_state, workspace,
                   nbytes, (q.dtype,))
    _weight_args(a, p, w_text, w_vis)
    B, N, H, dk, dv = _dims(p)
    for n, t, m in (("dq", dq, dk), ("dk", dk_, dk), ("dv", dv_, dv)):
        a.add(n, t, B * N * H * m, (q.dtype,))
    a.add("d_log_alpha", d_log_alpha, B * N * H * dk, (torch.float32,))
    a.add("d_beta", d_beta, B * N * H, (q.dtype,))
    a.add("d_w_text", d_w_text, 3 * H * dk * p.text_k, (torch.float32,))
    a.add("d_w_vis", d_w_vis, 3 * H * dk * p.vis_kt * p.vis_kh * p.vis_kw, (torch.float32,))
    a.add("d_initial_state", d_initial_state, B * H * dk * dv, (torch.float32,)).check_devices()
    _check(_lib.kda_bwd(ctypes.byref(p), _dt(q.dtype), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                        _ptr(w_text), _ptr(w_vis), _ptr(initial_state), _ptr(d_o), _ptr(d_final_state), _ptr(dq),
                        _ptr(dk_), _ptr(dv_), _ptr(d_log_alpha), _ptr(d_beta), _ptr(d_w_text), _ptr(d_w_vis),
                        _ptr(d_initial_state), _ptr(workspace), nbytes, _stream(stream)),
           "kda_bwd")


def kda_selftest_wait_timeout(p, q, k, v, log_alpha, beta, o, workspace, stage, wait_us, stream=None):
    """Runs kda_chunk_fwd's kernels with one load never issued (stage 1: the block-record kernel's,
    stage 2: the state pass's) and every device wait limited to wait_us: the device status then reads
    KDA_ERR_TIMEOUT (see include/kda.h)."""
    nbytes = workspace.numel() * workspace.element_size()
    _scan_args("kda_selftest_wait_timeout", p, o.dtype, q, k, v, log_alpha, beta, o, None, None, workspace, nbytes,
               _act_dtypes(p, o.dtype)).check_devices()
    _check(_lib.kda_selftest_wait_timeout(ctypes.byref(p), _dt(o.dtype), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha),
                                          _ptr(beta), _ptr(o), _ptr(workspace), nbytes, int(stage), int(wait_us),
                                          _stream(stream)),
           "kda_selftest_wait_timeout")


def kda_read_status(workspace, stream=None) -> int:
    if isinstance(workspace, torch.Tensor) and workspace.device.type != "cuda":
        raise KdaError(KDA_ERR_INVALID_ARG, "kda_read_status: workspace must be a CUDA tensor")
    return _lib.kda_read_status(_ptr(workspace), _stream(stream))
