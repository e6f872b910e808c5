"""Backward pass (kda_bwd) vs the oracle's adjoint, through the C ABI (needs a B200).

The oracle's backward is pinned by finite differences (tests/test_oracle_bwd.py).
Each gradient is compared element by element: relative L2 error within the
fp32 bound (1e-5) for fp32 problems; for bf16 problems within the bf16 bounds
(relative L2 5e-3, and max-abs 2e-2 taken relative to the gradient's largest
magnitude, since gradients carry the scale of d_o rather than of o).
"""
import dataclasses
import os

import numpy as np
import pytest
import torch

import kda_synth
import oracle
from tests._util import rel_l2, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kda():
    import linear_attention_video_b200 as kda
    assert torch.cuda.is_available()
    return kda


def run_bwd(kda, w, inp, dO, S0=None, dSN=None, causal=False, status=None):
    B, N, H, d = inp["shape"]
    t = to_device(inp)
    dt = t["q"].dtype
    p = kda.problem(B, H, d, w.text_len, w.grid, vis_causal_t=causal)
    f32 = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()   # noqa: E731
    d_o = torch.from_numpy(np.ascontiguousarray(dO, np.float32)).reshape(B, N, H, d).cuda().to(dt)
    g = {n: torch.empty(B, N, H, d, dtype=dt, device="cuda") for n in ("dq", "dk", "dv")}
    g["dla"] = torch.empty(B, N, H, d, dtype=torch.float32, device="cuda")
    g["dbeta"] = torch.empty(B, N, H, dtype=dt, device="cuda")
    g["dw_text"] = torch.empty(3, H * d, w.text_k, dtype=torch.float32, device="cuda")
    g["dw_vis"] = torch.empty(3, H * d, 27, dtype=torch.float32, device="cuda")
    g["dS0"] = torch.empty(B, H, d, d, dtype=torch.float32, device="cuda")
    ws = kda.alloc_bwd_workspace(p, dt)
    kda.kda_bwd(p, t["q"], t["k"], t["v"], t["log_alpha"], t["beta"], t["w_text"], t["w_vis"], d_o, g["dq"], g["dk"],
                g["dv"], g["dla"], g["dbeta"], g["dw_text"], g["dw_vis"], ws, initial_state=f32(S0),
                d_final_state=f32(dSN), d_initial_state=g["dS0"])
    torch.cuda.synchronize()
    assert kda.kda_read_status(ws) == (kda.KDA_OK if status is None else status)
    # the gradient the oracle sees for d_o is the value actually passed (rounded to dtype)
    return {n: v.float().cpu().numpy() for n, v in g.items()}, d_o.float().cpu().numpy()


def check(got, ref, dtype):
    log = os.environ.get("KDA_PARITY_LOG")
    for n in ("dq", "dk", "dv", "dla", "dbeta", "dw_text", "dw_vis", "dS0"):
        x, r = got[n].reshape(ref[n].shape), ref[n]
        e = rel_l2(x, r)
        if log:   # one line per gradient, for reporting the measured errors
            m = float(np.abs(x - r).max() / max(np.abs(r).max(), 1e-30)) if r.size else 0.0
            with open(log, "a") as f:
                f.write(f"{os.environ.get('PYTEST_CURRENT_TEST', '?').split(' ')[0]}\t{n}\t{dtype}\t{e:.3e}\t{m:.3e}\n")
        if dtype == "f32":
            assert e <= 1e-5, f"{n}: rel_l2={e:.3e}"
        else:
            m = float(np.abs(x - r).max() / max(np.abs(r).max(), 1e-30))
            assert e <= 5e-3 and m <= 2e-2, f"{n}: rel_l2={e:.3e} rel max-abs={m:.3e}"


def _case(kda, w, seed, causal=False, with_state=True, inp=None):
    inp = kda_synth.generate(w, seed) if inp is None else inp
    B, N, H, d = inp["shape"]
    rng = np.random.default_rng(seed)
    dO = rng.standard_normal((B, N, H, d))
    S0 = kda_synth.initial_state(seed + 1, B, H, d, d) if with_state else None
    dSN = rng.standard_normal((B, H, d, d)) * 0.1 if with_state else None
    got, dO_used = run_bwd(kda, w, inp, dO, S0, dSN, causal)
    ref = oracle.backward(inp, w.text_len, w.grid, dO_used, S0=S0, dSN=dSN, vis_causal_t=causal)
    check(got, ref, w.dtype)


def test_bwd_tiny_fp32(kda):
    _case(kda, kda_synth.WORKLOADS[0], 31)


@pytest.mark.parametrize("case", ["causal_t", "text_only", "visual_only", "batch2_ragged"])
def test_bwd_edge_shapes_fp32(kda, case):
    w = kda_synth.WORKLOADS[0]
    if case == "causal_t":
        _case(kda, w, 32, causal=True)
    elif case == "text_only":
        _case(kda, dataclasses.replace(w, text_len=77, grid=(0, 0, 0)), 33)
    elif case == "visual_only":
        _case(kda, dataclasses.replace(w, text_len=0, grid=(3, 5, 7)), 34, with_state=False)
    else:
        _case(kda, dataclasses.replace(w, B=2, text_len=13, grid=(2, 7, 9)), 35)


def test_bwd_bf16_d128(kda):
    """bf16 inputs and gradients, d = 128, several heads: 64 text tokens + a 3 x 8 x 8 grid."""
    w = kda_synth.Workload("bwd_bf16", 1, 4, 128, 64, (3, 8, 8), "bf16", 0.1)
    _case(kda, w, 36)


def test_bwd_rejects_scan_only_flags(kda):
    import ctypes
    w = kda_synth.WORKLOADS[0]
    p = kda.problem(1, w.H, w.d, w.text_len, w.grid, reuse_records=True)
    assert kda.kda_bwd_workspace_bytes(p, torch.float32) == 0
    assert kda._lib.kda_bwd(ctypes.byref(p), 1, *([256] * 19), 1 << 40, None) == kda.KDA_ERR_INVALID_ARG


def test_bwd_bf16_full_size_sampled_v_columns(kda):
    """Full 5 s video: the gradient of v on sampled channels, which the oracle computes exactly at
    any length (one state column at a time; the conv is depthwise)."""
    idx = 2
    w = kda_synth.WORKLOADS[idx]
    inp = kda_synth.generate(w, kda_synth.seed_for(idx))
    B, N, H, d = inp["shape"]
    rng = np.random.default_rng(5)
    dO = rng.standard_normal((B, N, H, d)).astype(np.float32)
    S0 = kda_synth.initial_state(6, B, H, d, d)
    dSN = (rng.standard_normal((B, H, d, d)) * 0.1).astype(np.float32)
    got, dO_used = run_bwd(kda, w, inp, dO, S0, dSN)
    items = [(0, 0), (9, 64), (15, 127)]
    ref = oracle.backward_v_columns(inp, w.text_len, w.grid, dO_used, items, S0=S0, dSN=dSN)
    x = np.stack([got["dv"][:, :, h, j] for h, j in items])
    e = rel_l2(x, ref)
    m = float(np.abs(x - ref).max() / np.abs(ref).max())
    if os.environ.get("KDA_PARITY_LOG"):
        with open(os.environ["KDA_PARITY_LOG"], "a") as f:
            f.write(f"test_bwd_bf16_full_size_sampled_v_columns\tdv columns\tbf16\t{e:.3e}\t{m:.3e}\n")
    assert e <= 5e-3 and m <= 2e-2, f"dv columns: rel_l2={e:.3e} rel max-abs={m:.3e}"


def test_bwd_strong_decay_within_and_beyond_the_range(kda):
    """The backward splits each pairwise decay e^(g_r - g_i) of a 64-token chunk around the
    chunk's middle token in fp32: 37 nats of decay inside a chunk (beyond the forward tensor
    path's fp16 range) is still exact; 70 nats on one side of the middle token is reported
    (KDA_ERR_RANGE), not returned as wrong values."""
    w = kda_synth.WORKLOADS[0]
    inp = kda_synth.generate(w, 37)
    B, N, H, d = inp["shape"]
    la = inp["log_alpha"].reshape(B, N, H, d).copy()
    la[0, 3:40, 1, 5] = -1.0
    _case(kda, w, 37, inp=dict(inp, log_alpha=la.reshape(inp["log_alpha"].shape)))
    la[0, 3:31, 1, 5] = -2.5
    dO = np.random.default_rng(7).standard_normal((B, N, H, d))
    run_bwd(kda, w, dict(inp, log_alpha=la.reshape(inp["log_alpha"].shape)), dO, status=kda.KDA_ERR_RANGE)


def test_bwd_bf16_d64(kda):
    """bf16 with d = 64 (the per-chunk kernels' single-product mode at D = 64), 13 text tokens + 3 x 5 x 7."""
    w = kda_synth.Workload("bwd_bf16_d64", 1, 2, 64, 13, (3, 5, 7), "bf16", 0.1)
    _case(kda, w, 38)


def test_bwd_bf16_long_chain(kda):
    """bf16, d = 128, 33 chunks (the last one ragged) under slow decay (log alpha near -0.02), so the
    chains' fp16 operand roundings compound over many chunks: every gradient against the oracle."""
    w = kda_synth.Workload("bwd_bf16_long", 1, 2, 128, 64, (4, 16, 32), "bf16", 0.02)
    _case(kda, w, 39)


def test_bwd_bf16_strong_decay_inside_a_chunk(kda):
    """bf16, d = 128: 37 nats of decay inside one chunk in one channel (W and Kt of that chunk span
    e^-37 in fp16, below its normal range) still matches the oracle."""
    w = kda_synth.Workload("bwd_bf16", 1, 4, 128, 64, (3, 8, 8), "bf16", 0.1)
    inp = kda_synth.generate(w, 40)
    B, N, H, d = inp["shape"]
    la = inp["log_alpha"].reshape(B, N, H, d).copy()
    la[0, 70:107, 2, 9] = -1.0
    _case(kda, w, 40, inp=dict(inp, log_alpha=la.reshape(inp["log_alpha"].shape)))


@pytest.mark.parametrize("case", ["batch2_ragged", "causal_t", "text_only"])
def test_bwd_bf16_edge_shapes(kda, case):
    """bf16, d = 128 (the fp16 chains, whose launch interleaves batch items and directions in
    blockIdx.z): two batch items with a ragged last chunk, the temporally causal conv, text only."""
    w = kda_synth.Workload("bwd_bf16_edge", 1, 2, 128, 13, (2, 7, 9), "bf16", 0.1)
    if case == "batch2_ragged":
        _case(kda, dataclasses.replace(w, B=2), 41)
    elif case == "causal_t":
        _case(kda, w, 42, causal=True)
    else:
        _case(kda, dataclasses.replace(w, text_len=150, grid=(0, 0, 0)), 43)
