"""Pins for the oracle's backward pass (CPU only).

The pages give no backward pass; the oracle's is the chain rule applied to the
forward steps (the recurrence of paper.rainbus.top, section 方法步骤详情 step
(5), and the per-modality short convolution).  It is pinned against central
finite differences of the (already pinned) forward oracle in fp64: element by
element on tiny inputs, and along random directions for the whole pipeline.
"""
import numpy as np
import pytest

import kda_synth
import oracle

H_FD = 1e-6


def _scan_loss(dO, dSN, q, k, v, la, beta, S0):
    o, S = oracle.scan(q, k, v, la, beta, S0)
    return float((o * dO).sum() + (S * dSN).sum())


def _scan_problem(rng, B=2, N=7, dk=3, dv=2, beta_zero=False):
    q, k = rng.standard_normal((B, N, dk)), rng.standard_normal((B, N, dk))
    la = -np.abs(rng.standard_normal((B, N, dk))) * 0.3
    v = rng.standard_normal((B, N, dv))
    beta = np.zeros((B, N)) if beta_zero else 1 / (1 + np.exp(-rng.standard_normal((B, N))))
    S0 = rng.standard_normal((B, dk, dv))
    return dict(q=q, k=k, v=v, la=la, beta=beta, S0=S0)


@pytest.mark.parametrize("beta_zero", [False, True])
def test_scan_adjoint_matches_finite_differences(beta_zero):
    rng = np.random.default_rng(1)
    args = _scan_problem(rng, beta_zero=beta_zero)
    B, N, dv = args["v"].shape
    dO, dSN = rng.standard_normal((B, N, dv)), rng.standard_normal((B, args["q"].shape[2], dv))
    g = oracle.scan_bwd(args["q"], args["k"], args["v"], args["la"], args["beta"], dO, args["S0"], dSN)
    names = {"q": "dq", "k": "dk", "v": "dv", "la": "dla", "beta": "dbeta", "S0": "dS0"}
    for n, a in args.items():
        fd = np.zeros_like(a)
        for idx in np.ndindex(a.shape):
            p, m = dict(args), dict(args)
            p[n], m[n] = a.copy(), a.copy()
            p[n][idx] += H_FD
            m[n][idx] -= H_FD
            fd[idx] = (_scan_loss(dO, dSN, **p) - _scan_loss(dO, dSN, **m)) / (2 * H_FD)
        assert np.abs(fd - g[names[n]]).max() <= 1e-7 * max(1.0, np.abs(fd).max()), n
    if beta_zero:
        # no writes: v and k never reach the output
        assert not g["dv"].any() and not g["dk"].any()


def _conv_inputs(rng, causal, B=2, C=3, text_len=5, grid=(3, 3, 4)):
    N = text_len + grid[0] * grid[1] * grid[2]
    shape = oracle.conv_shape(B, N, text_len, grid, vis_causal_t=causal)
    x = rng.standard_normal((B, N, C)).astype(np.float32)
    wt = rng.standard_normal((C, 4)).astype(np.float32)
    wv = rng.standard_normal((C, 27)).astype(np.float32)
    return shape, x, wt, wv


@pytest.mark.parametrize("causal", [False, True])
def test_conv_adjoint_is_the_transpose(causal):
    """The conv is linear in x and in the weights, so its adjoint is exact: <dy, conv(x)> equals
    <dx, x> and <dw_text, w_text> + <dw_vis, w_vis>, and each equals the directional derivative."""
    rng = np.random.default_rng(2)
    shape, x, wt, wv = _conv_inputs(rng, causal)
    dy = rng.standard_normal(x.shape)
    y = oracle.shortconv(shape, x, wt, wv)
    dx, dwt, dwv = oracle.shortconv_bwd(shape, x, wt, wv, dy)
    lhs = float((dy * y).sum())
    assert abs(lhs - float((dx * x).sum())) <= 1e-10 * max(1.0, abs(lhs))
    assert abs(lhs - float((dwt * wt).sum() + (dwv * wv).sum())) <= 1e-10 * max(1.0, abs(lhs))
    # element by element against the forward: unit inputs recover single taps
    B, N, C = x.shape
    for (b, n, c) in [(0, 0, 0), (1, 4, 2), (0, 5, 1), (1, N - 1, 0), (0, 5 + 12, 2)]:
        e = np.zeros_like(x)
        e[b, n, c] = 1.0
        col = oracle.shortconv(shape, e, wt, wv)           # every output that reads x[b, n, c]
        assert abs(float((dy * col).sum()) - dx[b, n, c]) <= 1e-12 * max(1.0, abs(dx[b, n, c]))


def _pipeline_loss(inp, w, dO, dSN, S0, causal):
    o, S = oracle.forward(inp, w.text_len, w.grid, S0=S0, vis_causal_t=causal)
    return float((o * dO).sum() + (S * dSN).sum())


@pytest.mark.parametrize("causal", [False, True])
def test_pipeline_adjoint_matches_directional_derivatives(causal):
    w = kda_synth.Workload("bwd_tiny", 1, 2, 8, 4, (3, 3, 4), "f32", 0.1)
    inp = kda_synth.generate(w, 21)
    B, N, H, d = inp["shape"]
    rng = np.random.default_rng(3)
    dO, dSN = rng.standard_normal((B, N, H, d)), rng.standard_normal((B, H, d, d))
    S0 = rng.standard_normal((B, H, d, d)) * 0.1
    g = oracle.backward(inp, w.text_len, w.grid, dO, S0=S0, dSN=dSN, vis_causal_t=causal)
    # the inputs are stored in float32: the perturbed inputs are rounded to float32 and the
    # step actually taken is measured from the rounded values
    for name, gkey, shape in [("q", "dq", (B, N, H, d)), ("k", "dk", (B, N, H, d)), ("v", "dv", (B, N, H, d)),
                              ("log_alpha", "dla", (B, N, H, d)), ("beta", "dbeta", (B, N, H))]:
        r = rng.standard_normal(shape)
        h = 1e-3
        p, m = dict(inp), dict(inp)
        base = np.asarray(inp[name], np.float64).reshape(shape)
        p[name] = (base + h * r).astype(np.float32).reshape(inp[name].shape)
        m[name] = (base - h * r).astype(np.float32).reshape(inp[name].shape)
        step = (np.asarray(p[name], np.float64) - np.asarray(m[name], np.float64)).reshape(shape) / 2
        fd = (_pipeline_loss(p, w, dO, dSN, S0, causal) - _pipeline_loss(m, w, dO, dSN, S0, causal))
        pred = 2 * float((g[gkey] * step).sum())
        assert abs(fd - pred) <= 2e-5 * max(1.0, abs(pred)), (name, fd, pred)
    for name, gkey in [("w_text", "dw_text"), ("w_vis", "dw_vis")]:
        r = rng.standard_normal(inp[name].shape)
        base = np.asarray(inp[name], np.float64)
        p, m = dict(inp), dict(inp)
        p[name] = (base + 1e-3 * r).astype(np.float32)
        m[name] = (base - 1e-3 * r).astype(np.float32)
        step = (np.asarray(p[name], np.float64) - np.asarray(m[name], np.float64)) / 2
        fd = _pipeline_loss(p, w, dO, dSN, S0, causal) - _pipeline_loss(m, w, dO, dSN, S0, causal)
        pred = 2 * float((g[gkey] * step).sum())
        assert abs(fd - pred) <= 2e-5 * max(1.0, abs(pred)), (name, fd, pred)
    r = rng.standard_normal(S0.shape)
    fd = _pipeline_loss(inp, w, dO, dSN, S0 + 1e-6 * r, causal) - _pipeline_loss(inp, w, dO, dSN, S0 - 1e-6 * r, causal)
    assert abs(fd - 2e-6 * float((g["dS0"] * r).sum())) <= 1e-8 * max(1.0, abs(fd))


def test_v_columns_equal_the_full_backward():
    """The one-column route to dv gives the full backward's dv (the column property the GPU
    tests rely on at full length)."""
    w = kda_synth.Workload("bwd_cols", 1, 2, 8, 4, (3, 3, 4), "f32", 0.1)
    inp = kda_synth.generate(w, 23)
    B, N, H, d = inp["shape"]
    rng = np.random.default_rng(4)
    dO, dSN = rng.standard_normal((B, N, H, d)), rng.standard_normal((B, H, d, d))
    S0 = rng.standard_normal((B, H, d, d)) * 0.1
    g = oracle.backward(inp, w.text_len, w.grid, dO, S0=S0, dSN=dSN)
    items = [(0, 0), (1, 5), (1, 7)]
    cols = oracle.backward_v_columns(inp, w.text_len, w.grid, dO, items, S0=S0, dSN=dSN)
    for i, (h, j) in enumerate(items):
        assert np.allclose(cols[i], g["dv"][:, :, h, j], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("chunk", [1, 4, 16, 64])
def test_chunked_backward_equals_the_token_adjoint(chunk):
    """A second formulation of the backward (the chain rule through the chunked UT/WY form)
    agrees with the token-by-token adjoint for any chunk length, ragged last chunk included."""
    rng = np.random.default_rng(6)
    N, dk, dv = 37, 6, 5
    a = _scan_problem(rng, B=1, N=N, dk=dk, dv=dv)
    dO, dSN = rng.standard_normal((1, N, dv)), rng.standard_normal((1, dk, dv))
    ref = oracle.scan_bwd(a["q"], a["k"], a["v"], a["la"], a["beta"], dO, a["S0"], dSN)
    got = oracle.chunked_scan_bwd(a["q"][0], a["k"][0], a["v"][0], a["la"][0], a["beta"][0], dO[0], a["S0"][0],
                                  dSN[0], chunk=chunk)
    for n in ("dq", "dk", "dv", "dla", "dbeta", "dS0"):
        r = ref[n][0]
        assert np.abs(got[n] - r).max() <= 1e-12 * max(1.0, np.abs(r).max()), n
