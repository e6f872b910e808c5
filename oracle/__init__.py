"""CPU oracle for the KDA + modality-aware short-convolution forward pass.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares no code
with the CUDA path (``linear_attention_video_b200``) and never imports it.

Two independent formulations live here, both in fp64:

* ``kda_oracle.c`` -- the definition: the depthwise short convolution written
  out tap by tap, and the token-by-token KDA recurrence
  (paper.rainbus.top, section 方法步骤详情, step (5);
  genai-atlas, section "How it works").
* ``kda_oracle.c`` also holds the backward pass: the chain rule written out
  through the recurrence (token by token, in reverse, every state kept) and the
  transpose of the convolution; pinned by finite differences of the forward.
* this module's numpy code -- the chunked (UT/WY) form for any chunk length,
  the dense lower-triangular form, and the update exactly as printed on the
  page (explicit (I - beta k k^T) Diag(alpha) products), used only to
  cross-check the recurrence on small inputs.

Readings of points the pages leave open (the kernels implement the same readings):
  * read-out o_t = S_t^T q_t, no scale on q;
  * kernels: causal 4 taps over text, 3x3x3 over the visual grid, applied as a
    cross-correlation (tap j of the text kernel multiplies x[t-(K-1)+j]);
  * the 3D conv is centred and zero-padded in T, H and W by default; with
    ``vis_causal_t`` its temporal taps cover frames t-kt+1..t instead;
  * no bias, activation or normalisation after the conv;
  * separate depthwise weights for q, k and v;
  * one causal scan over text then visual tokens, no reset in between;
  * batch items are independent and share the text length.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB = os.path.join(_HERE, "libkdaoracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle (plain -O2, IEEE fp64 arithmetic, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-pthread", "-o", _LIB, _SRC, "-lm"])
    return _LIB


class ConvShape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in (
        "B", "N", "text_len", "grid_t", "grid_h", "grid_w", "text_k",
        "vis_kt", "vis_kh", "vis_kw", "vis_causal_t")]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            i64, vp, i32 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
            lib.kdao_shortconv.argtypes = [ctypes.POINTER(ConvShape), i64, i64, i64, vp, vp, vp, vp, i32]
            lib.kdao_shortconv.restype = i32
            lib.kdao_scan.argtypes = [i64, i64, i64, i64, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i32]
            lib.kdao_scan.restype = i32
            lib.kdao_scan_bwd.argtypes = [i64, i64, i64, i64] + [vp] * 14 + [i32]
            lib.kdao_scan_bwd.restype = i32
            lib.kdao_shortconv_bwd.argtypes = [ctypes.POINTER(ConvShape), i64] + [vp] * 7 + [i32]
            lib.kdao_shortconv_bwd.restype = i32
            _lib = lib
    return _lib


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def widen(a: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float32 view of stored inputs: bf16 bit patterns or float32."""
    if dtype == "bf16":
        return (a.astype(np.uint32) << 16).view(np.float32)
    return np.asarray(a, dtype=np.float32)


def conv_shape(B, N, text_len, grid, text_k=4, vis_k=(3, 3, 3), vis_causal_t=False) -> ConvShape:
    T, Hg, Wg = grid
    if N != text_len + T * Hg * Wg:
        raise ValueError("N must equal text_len + T*Hg*Wg")
    return ConvShape(B, N, text_len, T, Hg, Wg, text_k, vis_k[0], vis_k[1], vis_k[2], int(bool(vis_causal_t)))


def shortconv(shape: ConvShape, x: np.ndarray, w_text: np.ndarray, w_vis: np.ndarray,
              c0: int = 0, c1: int | None = None, nthreads: int | None = None) -> np.ndarray:
    """Per-modality depthwise short convolution of x [B, N, C] (float32) in fp64.

    Returns y[:, :, c0:c1] as float64 [B, N, c1-c0].  w_text [C, text_k] and
    w_vis [C, kt*kh*kw] are float32.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    B, N, C = x.shape
    c1 = C if c1 is None else c1
    wt = np.ascontiguousarray(w_text, dtype=np.float32)
    wv = np.ascontiguousarray(w_vis, dtype=np.float32)
    assert wt.shape == (C, shape.text_k) and wv.shape == (C, shape.vis_kt * shape.vis_kh * shape.vis_kw)
    y = np.empty((B, N, c1 - c0), dtype=np.float64)
    rc = _load().kdao_shortconv(ctypes.byref(shape), C, c0, c1, x.ctypes.data, wt.ctypes.data,
                                wv.ctypes.data, y.ctypes.data, nthreads or default_threads())
    if rc:
        raise ValueError(f"kdao_shortconv failed ({rc})")
    return y


def scan(q, k, v, log_alpha, beta, S0=None, j0=0, j1=None, nthreads=None):
    """Token-by-token KDA recurrence for ONE head, fp64.

    q, k, log_alpha : [B, N, dk];  v : [B, N, dv];  beta : [B, N];  S0 : [B, dk, dv] or None.
    Returns (o [B, N, dv], S_N [B, dk, dv]); only columns [j0, j1) are computed
    (the others are zero).
    """
    q, k, v, la, bt = (np.ascontiguousarray(a, dtype=np.float64) for a in (q, k, v, log_alpha, beta))
    B, N, dk = q.shape
    dv = v.shape[-1]
    j1 = dv if j1 is None else j1
    o = np.zeros((B, N, dv), dtype=np.float64)
    SN = np.zeros((B, dk, dv), dtype=np.float64)
    s0p = None
    if S0 is not None:
        S0 = np.ascontiguousarray(S0, dtype=np.float64)
        assert S0.shape == (B, dk, dv)
        s0p = S0.ctypes.data
    rc = _load().kdao_scan(B, N, dk, dv, q.ctypes.data, k.ctypes.data, v.ctypes.data, la.ctypes.data,
                           bt.ctypes.data, s0p, o.ctypes.data, SN.ctypes.data, j0, j1,
                           nthreads or default_threads())
    if rc:
        raise ValueError(f"kdao_scan failed ({rc})")
    return o, SN


def _widened(inp: dict):
    """q, k, v widened once to float32 [B, N, H*d]."""
    B, N, H, d = inp["shape"]
    return [widen(inp[n], inp["dtype"]).reshape(B, N, H * d) for n in ("q", "k", "v")]


def _heads_inputs(inp: dict, h: int, shape: ConvShape, d: int, nthreads=None, v_cols=None, xs=None):
    """Convolved q', k', v' and the gates of head h, all float64."""
    B, N, H, _ = inp["shape"]
    xs = _widened(inp) if xs is None else xs
    out = []
    for idx in range(3):
        c0, c1 = h * d, (h + 1) * d
        if idx == 2 and v_cols is not None:
            c0, c1 = h * d + v_cols[0], h * d + v_cols[1]
        out.append(shortconv(shape, xs[idx], inp["w_text"][idx], inp["w_vis"][idx], c0, c1, nthreads))
    la = inp["log_alpha"].reshape(B, N, H, d)[:, :, h, :].astype(np.float64)
    bt = widen(inp["beta"], inp["dtype"]).reshape(B, N, H)[:, :, h].astype(np.float64)
    return out[0], out[1], out[2], la, bt


def forward(inp: dict, text_len: int, grid, S0=None, heads=None, text_k=4, vis_k=(3, 3, 3),
            vis_causal_t=False, nthreads=None):
    """Conv on q, k, v, then the KDA recurrence, for every (or the listed) head.

    ``inp`` is a dict as produced by ``kda_synth.generate``.  Returns
    (o [B, N, H, d] float64, S_N [B, H, d, d] float64); heads not listed stay 0.
    """
    B, N, H, d = inp["shape"]
    shape = conv_shape(B, N, text_len, grid, text_k, vis_k, vis_causal_t)
    xs = _widened(inp)
    o = np.zeros((B, N, H, d), dtype=np.float64)
    SN = np.zeros((B, H, d, d), dtype=np.float64)
    for h in (range(H) if heads is None else heads):
        qh, kh, vh, la, bt = _heads_inputs(inp, h, shape, d, nthreads, xs=xs)
        s0 = None if S0 is None else np.asarray(S0)[:, h]
        oh, sh = scan(qh, kh, vh, la, bt, s0, nthreads=nthreads)
        o[:, :, h, :] = oh
        SN[:, h] = sh
    return o, SN


def forward_columns(inp: dict, text_len: int, grid, items, S0=None, text_k=4, vis_k=(3, 3, 3),
                    vis_causal_t=False, nthreads=None, workers=1):
    """o[b, :, h, j] for each (h, j) in ``items`` and every batch item b.

    Column j of the state depends only on column j of v, so each sampled
    column is exact at any sequence length.  ``workers`` > 1 evaluates the heads
    concurrently on host threads (the C routines release the interpreter lock);
    the arithmetic is the same.  Returns float64 [len(items), B, N].
    """
    B, N, H, d = inp["shape"]
    shape = conv_shape(B, N, text_len, grid, text_k, vis_k, vis_causal_t)
    xs = _widened(inp)
    res = np.zeros((len(items), B, N), dtype=np.float64)
    by_head = {}
    for i, (h, j) in enumerate(items):
        by_head.setdefault(h, []).append((i, j))

    def one_head(h, lst, nt):
        qh, kh, _, la, bt = _heads_inputs(inp, h, shape, d, nt, v_cols=(0, 1), xs=xs)
        for i, j in lst:
            vj = shortconv(shape, xs[2], inp["w_text"][2], inp["w_vis"][2], h * d + j, h * d + j + 1, nt)
            vfull = np.zeros((B, N, d), dtype=np.float64)
            vfull[:, :, j] = vj[:, :, 0]
            s0 = None if S0 is None else np.asarray(S0)[:, h]
            oh, _ = scan(qh, kh, vfull, la, bt, s0, j0=j, j1=j + 1, nthreads=nt)
            res[i] = oh[:, :, j]

    if workers <= 1:
        for h, lst in by_head.items():
            one_head(h, lst, nthreads)
    else:
        from concurrent.futures import ThreadPoolExecutor
        nt = max(1, (nthreads or default_threads()) // workers)
        with ThreadPoolExecutor(workers) as pool:
            for f in [pool.submit(one_head, h, lst, nt) for h, lst in by_head.items()]:
                f.result()
    return res


# ---------------------------------------------------------------------------
# Backward pass (fp64): the chain rule through the steps above, in kda_oracle.c.
# ---------------------------------------------------------------------------

def scan_bwd(q, k, v, log_alpha, beta, dO, S0=None, dSN=None, nthreads=None):
    """Gradients of one head's recurrence for the loss sum(dO * o) + sum(dSN * S_N).

    Shapes as in ``scan``; dO [B, N, dv], dSN [B, dk, dv] or None.  Returns a dict with
    dq, dk, dla [B, N, dk], dv [B, N, dv], dbeta [B, N] and dS0 [B, dk, dv].  Every state
    is kept: small problems only."""
    q, k, v, la, bt, dO = (np.ascontiguousarray(a, dtype=np.float64) for a in (q, k, v, log_alpha, beta, dO))
    B, N, dk = q.shape
    dv = v.shape[-1]
    out = {"dq": np.zeros((B, N, dk)), "dk": np.zeros((B, N, dk)), "dv": np.zeros((B, N, dv)),
           "dla": np.zeros((B, N, dk)), "dbeta": np.zeros((B, N)), "dS0": np.zeros((B, dk, dv))}
    s0 = None if S0 is None else np.ascontiguousarray(S0, dtype=np.float64)
    dsn = None if dSN is None else np.ascontiguousarray(dSN, dtype=np.float64)
    ptr = lambda a: None if a is None else a.ctypes.data   # noqa: E731
    rc = _load().kdao_scan_bwd(B, N, dk, dv, ptr(q), ptr(k), ptr(v), ptr(la), ptr(bt), ptr(s0), ptr(dO), ptr(dsn),
                               ptr(out["dq"]), ptr(out["dk"]), ptr(out["dv"]), ptr(out["dla"]), ptr(out["dbeta"]),
                               ptr(out["dS0"]), nthreads or default_threads())
    if rc:
        raise ValueError(f"kdao_scan_bwd failed ({rc})")
    return out


def shortconv_bwd(shape: ConvShape, x: np.ndarray, w_text: np.ndarray, w_vis: np.ndarray, dy: np.ndarray,
                  nthreads: int | None = None):
    """Gradients of sum(dy * shortconv(x)) w.r.t. x [B, N, C] and the weights.

    Returns (dx [B, N, C], dw_text [C, text_k], dw_vis [C, kt*kh*kw]), float64."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    B, N, C = x.shape
    wt = np.ascontiguousarray(w_text, dtype=np.float32)
    wv = np.ascontiguousarray(w_vis, dtype=np.float32)
    dy = np.ascontiguousarray(dy, dtype=np.float64)
    dx = np.empty((B, N, C))
    dwt = np.empty(wt.shape)
    dwv = np.empty(wv.shape)
    rc = _load().kdao_shortconv_bwd(ctypes.byref(shape), C, x.ctypes.data, wt.ctypes.data, wv.ctypes.data,
                                    dy.ctypes.data, dx.ctypes.data, dwt.ctypes.data, dwv.ctypes.data,
                                    nthreads or default_threads())
    if rc:
        raise ValueError(f"kdao_shortconv_bwd failed ({rc})")
    return dx, dwt, dwv


def backward(inp: dict, text_len: int, grid, dO, S0=None, dSN=None, text_k=4, vis_k=(3, 3, 3),
             vis_causal_t=False, nthreads=None):
    """Gradients of the whole forward (conv on q, k, v, then the recurrence, every head) for the
    loss sum(dO * o) + sum(dSN * S_N).

    dO [B, N, H, d]; S0, dSN [B, H, d, d] or None.  Returns a dict with dq, dk, dv, dla
    [B, N, H, d], dbeta [B, N, H], dS0 [B, H, d, d] and dw_text, dw_vis [3][C][...] (float64)."""
    B, N, H, d = inp["shape"]
    shape = conv_shape(B, N, text_len, grid, text_k, vis_k, vis_causal_t)
    xs = _widened(inp)
    conv = [shortconv(shape, xs[i], inp["w_text"][i], inp["w_vis"][i], nthreads=nthreads).reshape(B, N, H, d)
            for i in range(3)]
    la = inp["log_alpha"].reshape(B, N, H, d).astype(np.float64)
    bt = widen(inp["beta"], inp["dtype"]).reshape(B, N, H).astype(np.float64)
    dO = np.asarray(dO, dtype=np.float64).reshape(B, N, H, d)
    dconv = [np.zeros((B, N, H, d)) for _ in range(3)]
    g = {"dla": np.zeros((B, N, H, d)), "dbeta": np.zeros((B, N, H)), "dS0": np.zeros((B, H, d, d))}
    for h in range(H):
        r = scan_bwd(conv[0][:, :, h], conv[1][:, :, h], conv[2][:, :, h], la[:, :, h], bt[:, :, h],
                     dO[:, :, h], None if S0 is None else np.asarray(S0)[:, h],
                     None if dSN is None else np.asarray(dSN)[:, h], nthreads)
        for i, n in enumerate(("dq", "dk", "dv")):
            dconv[i][:, :, h] = r[n]
        g["dla"][:, :, h] = r["dla"]
        g["dbeta"][:, :, h] = r["dbeta"]
        g["dS0"][:, h] = r["dS0"]
    g["dw_text"], g["dw_vis"] = [], []
    for i, n in enumerate(("dq", "dk", "dv")):
        dx, dwt, dwv = shortconv_bwd(shape, xs[i], inp["w_text"][i], inp["w_vis"][i],
                                     dconv[i].reshape(B, N, H * d), nthreads)
        g[n] = dx.reshape(B, N, H, d)
        g["dw_text"].append(dwt)
        g["dw_vis"].append(dwv)
    g["dw_text"], g["dw_vis"] = np.stack(g["dw_text"]), np.stack(g["dw_vis"])
    return g


def backward_v_columns(inp: dict, text_len: int, grid, dO, items, S0=None, dSN=None, text_k=4, vis_k=(3, 3, 3),
                       vis_causal_t=False, nthreads=None):
    """dv[b, :, h, j] (the gradient of the raw v) for each (h, j) in ``items``, at any length.

    Column j of the state, and so of its gradient, only involves column j of v, d_o, S0 and
    dSN; the conv is depthwise.  So the gradient of v's channel h*d + j comes from the
    adjoint of a one-column recurrence followed by the transposed conv of that channel.
    Returns float64 [len(items), B, N]."""
    B, N, H, d = inp["shape"]
    shape = conv_shape(B, N, text_len, grid, text_k, vis_k, vis_causal_t)
    xs = _widened(inp)
    dO = np.asarray(dO, dtype=np.float64).reshape(B, N, H, d)
    res = np.zeros((len(items), B, N))
    by_head = {}
    for i, (h, j) in enumerate(items):
        by_head.setdefault(h, []).append((i, j))
    for h, lst in by_head.items():
        qh, kh, _, la, bt = _heads_inputs(inp, h, shape, d, nthreads, v_cols=(0, 1), xs=xs)
        for i, j in lst:
            c = h * d + j
            vj = shortconv(shape, xs[2], inp["w_text"][2], inp["w_vis"][2], c, c + 1, nthreads)
            s0 = None if S0 is None else np.asarray(S0)[:, h, :, j:j + 1]
            dsn = None if dSN is None else np.asarray(dSN)[:, h, :, j:j + 1]
            r = scan_bwd(qh, kh, vj, la, bt, dO[:, :, h, j:j + 1], s0, dsn, nthreads)
            dx, _, _ = shortconv_bwd(shape, xs[2][:, :, c:c + 1], inp["w_text"][2][c:c + 1],
                                     inp["w_vis"][2][c:c + 1], r["dv"], nthreads)
            res[i] = dx[:, :, 0]
    return res


# ---------------------------------------------------------------------------
# Second formulations (numpy, fp64), for cross-checking the recurrence.
# ---------------------------------------------------------------------------

def printed_form_scan(q, k, v, log_alpha, beta, S0=None):
    """The update exactly as printed (paper.rainbus.top, 方法步骤详情 step (5)):
    S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T, then
    o_t = S_t^T q_t.  One head, one batch item: q, k, log_alpha [N, dk]; v [N, dv]."""
    N, dk = q.shape
    dv = v.shape[1]
    S = np.zeros((dk, dv)) if S0 is None else np.array(S0, dtype=np.float64)
    o = np.zeros((N, dv))
    I = np.eye(dk)
    for t in range(N):
        kt = k[t][:, None]
        S = (I - beta[t] * kt @ kt.T) @ np.diag(np.exp(log_alpha[t])) @ S + beta[t] * kt @ v[t][None, :]
        o[t] = S.T @ q[t]
    return o, S


def _chunk_terms(qc, kc, lac, bc):
    """Per-chunk quantities of the chunked form for one head.

    With g_r = sum_{i<=r} log a_i (within the chunk, vector over dk):
      A[r,i] = beta_r sum_c k_rc k_ic exp(g_rc - g_ic)   (i < r)
      P[r,i] = sum_c q_rc k_ic exp(g_rc - g_ic)          (i <= r)
      T = (I + A)^{-1} Diag(beta)
    """
    n = qc.shape[0]
    g = np.cumsum(lac, axis=0)
    diff = g[:, None, :] - g[None, :, :]
    lower = np.tril(np.ones((n, n), dtype=bool))
    diff = np.where(lower[:, :, None], diff, -np.inf)
    E = np.exp(diff)
    A = np.tril(bc[:, None] * np.einsum("rc,ic,ric->ri", kc, kc, E), -1)
    P = np.tril(np.einsum("rc,ic,ric->ri", qc, kc, E))
    T = np.linalg.solve(np.eye(n) + A, np.diag(bc))
    return g, A, P, T


def chunked_scan(q, k, v, log_alpha, beta, S0=None, chunk=64):
    """The chunked (UT/WY) form for one head and one batch item, fp64.

    Per chunk, from the entering state S:
      W = T (K * exp(g)),  U~ = T V,  U = U~ - W S
      O = (Q * exp(g)) S + P U
      S <- Diag(exp(g_last)) S + (K * exp(g_last - g))^T U
    The last chunk may be shorter than ``chunk``.
    """
    N, dk = q.shape
    dv = v.shape[1]
    S = np.zeros((dk, dv)) if S0 is None else np.array(S0, dtype=np.float64)
    o = np.zeros((N, dv))
    for c0 in range(0, N, chunk):
        sl = slice(c0, min(N, c0 + chunk))
        qc, kc, vc, lac, bc = q[sl], k[sl], v[sl], log_alpha[sl], beta[sl]
        g, A, P, T = _chunk_terms(qc, kc, lac, bc)
        W = T @ (kc * np.exp(g))
        U = T @ vc - W @ S
        o[sl] = (qc * np.exp(g)) @ S + P @ U
        S = np.exp(g[-1])[:, None] * S + (kc * np.exp(g[-1][None, :] - g)).T @ U
    return o, S


def _chunk_terms_bwd(q, k, v, la, beta, S0):
    """Forward quantities of one chunk in the chunked (UT/WY) form, every pairwise decay
    exp(g_r - g_i) formed exactly.  Shapes: q, k, la [n, dk], v [n, dv], beta [n], S0 [dk, dv]."""
    n = k.shape[0]
    g = np.cumsum(la, axis=0)
    gl = g[-1]
    E = np.exp(g[:, None, :] - g[None, :, :])                         # [r, i, c]
    strict, incl = np.tril(np.ones((n, n)), -1), np.tril(np.ones((n, n)))
    Ab = np.einsum("rc,ic,ric->ri", k, k, E) * strict                 # A without its beta_r factor
    P = np.einsum("rc,ic,ric->ri", q, k, E) * incl
    X = np.linalg.inv(np.eye(n) + beta[:, None] * Ab)                  # (I + A)^{-1}
    T = X * beta[None, :]
    KG, QG, Kt = k * np.exp(g), q * np.exp(g), k * np.exp(gl - g)
    W = T @ KG
    U = T @ v - W @ S0
    return dict(g=g, gl=gl, E=E, strict=strict, incl=incl, Ab=Ab, P=P, X=X, T=T, KG=KG, QG=QG, Kt=Kt, W=W, U=U)


def chunked_scan_bwd(q, k, v, log_alpha, beta, dO, S0=None, dSN=None, chunk=16):
    """The backward pass in the chunked form, one head and one batch item, fp64: a second
    formulation, cross-checked against the token-by-token adjoint (scan_bwd).

    Per chunk, entering with S0: U = T V - W S0, O = QG S0 + P U,
    S_out = Diag(e^{g_last}) S0 + Kt^T U (the chunked_scan quantities); the chain rule through
    these, then through T = (I + A)^{-1} Diag(beta), A, P and the exponential factors, gives
    the chunk's gradients and dS0, which is the gradient reaching the previous chunk's exit.
    q, k, log_alpha [N, dk]; v, dO [N, dv]; beta [N]; S0, dSN [dk, dv] or None."""
    q, k, v, la, beta, dO = (np.asarray(a, dtype=np.float64) for a in (q, k, v, log_alpha, beta, dO))
    N, dk = q.shape
    dv = v.shape[1]
    S = [np.zeros((dk, dv)) if S0 is None else np.asarray(S0, dtype=np.float64)]
    starts = list(range(0, N, chunk))
    for s in starts:                                                   # entry state of every chunk
        c = _chunk_terms_bwd(q[s:s + chunk], k[s:s + chunk], v[s:s + chunk], la[s:s + chunk], beta[s:s + chunk],
                             S[-1])
        S.append(np.exp(c["gl"])[:, None] * S[-1] + c["Kt"].T @ c["U"])
    out = {"dq": np.zeros((N, dk)), "dk": np.zeros((N, dk)), "dv": np.zeros((N, dv)), "dla": np.zeros((N, dk)),
           "dbeta": np.zeros(N)}
    dS = np.zeros((dk, dv)) if dSN is None else np.asarray(dSN, dtype=np.float64)
    for ci in range(len(starts) - 1, -1, -1):
        s = starts[ci]
        sl = slice(s, s + chunk)
        Kc, Qc, Vc, bc, dOc, S0c = k[sl], q[sl], v[sl], beta[sl], dO[sl], S[ci]
        c = _chunk_terms_bwd(Qc, Kc, Vc, la[sl], bc, S0c)
        g, gl, E, X, T, W, U, P = c["g"], c["gl"], c["E"], c["X"], c["T"], c["W"], c["U"], c["P"]
        dU = P.T @ dOc + c["Kt"] @ dS
        dS0 = np.exp(gl)[:, None] * dS + c["QG"].T @ dOc - W.T @ dU
        dP = (dOc @ U.T) * c["incl"]
        dQG, dKt, dW = dOc @ S0c.T, U @ dS.T, -dU @ S0c.T
        dT = dW @ c["KG"].T + dU @ Vc.T
        dKG = T.T @ dW
        out["dv"][sl] = T.T @ dU
        dA = -(X.T @ (dT * bc[None, :]) @ X.T) * c["strict"]
        out["dbeta"][sl] = np.einsum("ri,ri->i", X, dT) + np.einsum("ri,ri->r", dA, c["Ab"])
        dAb = dA * bc[:, None]
        dq = dQG * np.exp(g) + np.einsum("ri,ic,ric->rc", dP, Kc, E)
        dkk = dKG * np.exp(g) + dKt * np.exp(gl - g)
        dkk += np.einsum("ri,ic,ric->rc", dAb, Kc, E) + np.einsum("ri,rc,ric->ic", dAb, Kc, E)
        dkk += np.einsum("ri,rc,ric->ic", dP, Qc, E)
        dEE = (np.einsum("ri,rc,ic->ric", dAb, Kc, Kc) + np.einsum("ri,rc,ic->ric", dP, Qc, Kc)) * E
        dg = dEE.sum(axis=1) - dEE.sum(axis=0) + dKG * c["KG"] + dQG * c["QG"] - dKt * c["Kt"]
        dg[-1] += (dKt * c["Kt"]).sum(axis=0) + (dS * np.exp(gl)[:, None] * S0c).sum(axis=1)
        out["dla"][sl] = np.cumsum(dg[::-1], axis=0)[::-1]             # g is the running sum of log alpha
        out["dq"][sl], out["dk"][sl] = dq, dkk
        dS = dS0
    out["dS0"] = dS
    return out


def dense_scan(q, k, v, log_alpha, beta):
    """Dense lower-triangular form from a zero state, one head, one batch item.

    Written independently of the chunked form: the decays enter as ratios of
    the running products Gamma_t = prod_{i<=t} alpha_i, and
        (I + A) U = Diag(beta) V,   O = P U
    with A[r,i] = beta_r sum_c k_rc k_ic Gamma_rc / Gamma_ic (i < r) and
    P[r,i] = sum_c q_rc k_ic Gamma_rc / Gamma_ic (i <= r), solved by forward
    substitution.  Only for short sequences with moderate decay (the running
    products must not underflow).
    """
    import scipy.linalg
    N = q.shape[0]
    gam = np.cumprod(np.exp(log_alpha), axis=0)
    A = np.zeros((N, N))
    P = np.zeros((N, N))
    for r in range(N):
        for i in range(r + 1):
            ratio = gam[r] / gam[i]
            P[r, i] = np.sum(q[r] * k[i] * ratio)
            if i < r:
                A[r, i] = beta[r] * np.sum(k[r] * k[i] * ratio)
    U = scipy.linalg.solve_triangular(np.eye(N) + A, beta[:, None] * v, lower=True, unit_diagonal=True)
    return P @ U
