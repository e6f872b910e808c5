"""Seeded synthetic inputs for the KDA + modality-aware short-conv forward pass.

This module is shared by the CPU oracle and the CUDA path and holds none of
the method's arithmetic: only the workload shapes and the value distributions
of the inputs (the Chimera pages' workloads: <=512 umT5 text tokens followed by
the patchified latent grid of a 1024^2 image, a 5 s / 30 s 480x832 video and a
4096^2 image -- "Chimera: Designing and Chinchilla-Scaling Hybrid Visual
Diffusion Transformers", paper.rainbus.top, sections 研究动机 and 实验结果).

Random draws come from a counter-based generator written in C (``synth.c``),
so each tensor is a pure function of (seed, stream, element index).
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libkdasynth.so")
_lock = threading.Lock()
_lib = None

BF16, F32 = 0, 1

# stream ids: one per tensor, fixed forever (changing them changes every input)
STREAM = dict(q=1, k=2, v=3, log_alpha=4, beta=5,
              w_text_q=6, w_text_k=7, w_text_v=8,
              w_vis_q=9, w_vis_k=10, w_vis_v=11, state0=12)


def build(force: bool = False) -> str:
    """Compile libkdasynth.so next to its source (gcc, -O2, pthreads)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-pthread", "-o", _LIB, _SRC, "-lm"])
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            u64, dbl, vp, i32 = ctypes.c_uint64, ctypes.c_double, ctypes.c_void_p, ctypes.c_int
            lib.syn_normal.argtypes = [u64, u64, u64, dbl, dbl, vp, i32, i32]
            lib.syn_unit_rows.argtypes = [u64, u64, u64, u64, vp, i32, i32]
            lib.syn_neg_softplus.argtypes = [u64, u64, u64, dbl, vp, i32, i32]
            lib.syn_sigmoid.argtypes = [u64, u64, u64, dbl, vp, i32, i32]
            for f in (lib.syn_normal, lib.syn_unit_rows, lib.syn_neg_softplus, lib.syn_sigmoid):
                f.restype = i32
            _lib = lib
    return _lib


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and input distribution of one synthetic workload."""
    name: str
    B: int
    H: int
    d: int
    text_len: int
    grid: tuple            # (T, Hg, Wg) of the visual latent grid
    dtype: str             # "bf16" or "f32": dtype of q, k, v, beta and o
    la_scale: float        # log a = -softplus(N(0,1)) * la_scale
    beta_std: float = 1.0  # beta = sigmoid(beta_std * N(0,1))
    text_k: int = 4
    vis_k: tuple = (3, 3, 3)
    chunk: int = 64

    @property
    def N(self) -> int:
        T, Hg, Wg = self.grid
        return self.text_len + T * Hg * Wg

    @property
    def tokens(self) -> int:
        return self.B * self.N


def alpha_scale_for_mean(target_mean: float) -> float:
    """Scale s such that E[exp(-s * softplus(Z))] = target_mean for Z ~ N(0,1).

    Evaluated by quadrature over the normal density and bisection, so the value
    does not depend on any particular sample.
    """
    z = np.linspace(-12.0, 12.0, 200001)
    w = np.exp(-0.5 * z * z)
    w /= w.sum()
    sp = np.logaddexp(0.0, z)

    def mean(s):
        return float((w * np.exp(-s * sp)).sum())

    lo, hi = 0.0, 1.0
    for _ in range(100):
        mid = 0.5 * (lo + hi)
        if mean(mid) > target_mean:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


LONG_MEMORY_SCALE = alpha_scale_for_mean(0.99)

WORKLOADS = [
    Workload("tiny_fp32", 1, 2, 64, 32, (1, 14, 16), "f32", 0.1),
    Workload("image_1024", 1, 16, 128, 512, (1, 64, 64), "bf16", 0.1),
    Workload("video_5s_480x832", 1, 16, 128, 512, (21, 30, 52), "bf16", 0.1),
    Workload("video_30s_480x832", 1, 16, 128, 512, (121, 30, 52), "bf16", LONG_MEMORY_SCALE),
    Workload("image_4096_b2", 2, 16, 128, 512, (1, 256, 256), "bf16", 0.1, beta_std=2.0),
]


def seed_for(index: int) -> int:
    return 20260000 + index


def _nthreads(n):
    return n if n else max(1, min(64, os.cpu_count() or 1))


def _alloc(n, dtype_code):
    return np.empty(n, dtype=np.uint16 if dtype_code == BF16 else np.float32)


def unit_rows(seed, stream, rows, row, dtype_code, nthreads=None):
    out = _alloc(rows * row, dtype_code)
    rc = _load().syn_unit_rows(seed, stream, rows, row, out.ctypes.data, dtype_code, _nthreads(nthreads))
    assert rc == 0
    return out


def normal(seed, stream, n, mean, std, dtype_code, nthreads=None):
    out = _alloc(n, dtype_code)
    rc = _load().syn_normal(seed, stream, n, mean, std, out.ctypes.data, dtype_code, _nthreads(nthreads))
    assert rc == 0
    return out


def neg_softplus(seed, stream, n, scale, nthreads=None):
    out = _alloc(n, F32)
    rc = _load().syn_neg_softplus(seed, stream, n, scale, out.ctypes.data, F32, _nthreads(nthreads))
    assert rc == 0
    return out


def sigmoid(seed, stream, n, std, dtype_code, nthreads=None):
    out = _alloc(n, dtype_code)
    rc = _load().syn_sigmoid(seed, stream, n, std, out.ctypes.data, dtype_code, _nthreads(nthreads))
    assert rc == 0
    return out


def generate(w: Workload, seed: int, nthreads: int | None = None, tokens: int | None = None) -> dict:
    """All inputs of workload ``w``.

    Activations are returned as flat-reshaped numpy arrays: bf16 tensors as
    uint16 bit patterns, fp32 tensors as float32.  Layouts (row-major):
      q, k, log_alpha : [B, N, H, d]      v : [B, N, H, d]      beta : [B, N, H]
      w_text : [3, H*d, text_k]  (q, k, v)   w_vis : [3, H*d, kt*kh*kw]  (q, k, v)
    ``tokens`` (optional) truncates every sequence to its first ``tokens``
    positions; the values are those of the full workload (counter-based draws).
    """
    dt = BF16 if w.dtype == "bf16" else F32
    B, N, H, d = w.B, w.N, w.H, w.d
    n_keep = N if tokens is None else min(N, tokens)
    out = {}

    if n_keep == N:
        out["q"] = unit_rows(seed, STREAM["q"], B * N * H, d, dt, nthreads)
        out["k"] = unit_rows(seed, STREAM["k"], B * N * H, d, dt, nthreads)
        out["v"] = normal(seed, STREAM["v"], B * N * H * d, 0.0, 1.0, dt, nthreads)
        out["log_alpha"] = neg_softplus(seed, STREAM["log_alpha"], B * N * H * d, w.la_scale, nthreads)
        out["beta"] = sigmoid(seed, STREAM["beta"], B * N * H, w.beta_std, dt, nthreads)
    else:
        full = generate(w, seed, nthreads)
        for name in ("q", "k", "v", "log_alpha"):
            out[name] = full[name].reshape(B, N, H, d)[:, :n_keep].reshape(-1).copy()
        out["beta"] = full["beta"].reshape(B, N, H)[:, :n_keep].reshape(-1).copy()
    kv = w.vis_k[0] * w.vis_k[1] * w.vis_k[2]
    wstd = 1.0 / math.sqrt(27.0)
    out["w_text"] = np.stack([normal(seed, STREAM["w_text_" + t], H * d * w.text_k, 0.0, wstd, F32, nthreads)
                              for t in "qkv"]).reshape(3, H * d, w.text_k)
    out["w_vis"] = np.stack([normal(seed, STREAM["w_vis_" + t], H * d * kv, 0.0, wstd, F32, nthreads)
                             for t in "qkv"]).reshape(3, H * d, kv)
    out["dtype"] = w.dtype
    out["shape"] = (B, n_keep, H, d)
    return out


def initial_state(seed: int, B: int, H: int, dk: int, dv: int, std: float = 0.1, nthreads=None) -> np.ndarray:
    """Random fp32 initial state S_0 of shape [B, H, dk, dv]."""
    return normal(seed, STREAM["state0"], B * H * dk * dv, 0.0, std, F32, nthreads).reshape(B, H, dk, dv)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float32."""
    return (bits.astype(np.uint32) << 16).view(np.float32)
