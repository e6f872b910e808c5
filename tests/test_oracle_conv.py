"""Pins for the oracle's modality-aware short convolution (CPU only).

What the pages fix (Chimera, genai-atlas "How it works"; paper.rainbus.top
核心方法): per-modality depthwise convolution, causal 1D over the text prefix,
3D over the visual tokens reshaped to their (T, H, W) grid, raster order with
text first.  The checks below pin orientation, padding, causality, modality
isolation and the edge counts with values that do not come from the oracle.
"""
import json
import os

import numpy as np
import pytest

import oracle


def _conv(x, wt, wv, L, grid, text_k=4, vis_k=(3, 3, 3), causal_t=False, B=None):
    x = np.asarray(x, dtype=np.float32)
    if x.ndim == 2:
        x = x[None]
    shape = oracle.conv_shape(x.shape[0], x.shape[1], L, grid, text_k, vis_k, causal_t)
    return oracle.shortconv(shape, x, wt, wv, nthreads=2)


def test_text_conv_hand_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "conv_hand.json")))["text"]
    x = np.array(g["x"], dtype=np.float32)[:, None]
    wt = np.array([g["w"]], dtype=np.float32)
    wv = np.zeros((1, 27), dtype=np.float32)
    y = _conv(x, wt, wv, L=len(g["x"]), grid=(0, 1, 1))
    np.testing.assert_allclose(y[0, :, 0], g["y"], rtol=1e-6, atol=1e-7)


def test_vis_conv_hand_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "conv_hand.json")))["vis"]
    x = np.array(g["x_raster"], dtype=np.float32)[:, None]
    wt = np.zeros((1, 4), dtype=np.float32)
    wv = np.ones((1, 27), dtype=np.float32)
    y = _conv(x, wt, wv, L=0, grid=tuple(g["grid"]))
    np.testing.assert_array_equal(y[0, :, 0], np.array(g["y_raster"], dtype=np.float64))


def test_identity_kernels_return_input():
    rng = np.random.default_rng(0)
    L, grid, C = 7, (3, 4, 5), 6
    N = L + 60
    x = rng.standard_normal((2, N, C)).astype(np.float32)
    wt = np.zeros((C, 4), np.float32)
    wt[:, 3] = 1.0          # tap K-1 multiplies x[t]
    wv = np.zeros((C, 27), np.float32)
    wv[:, 13] = 1.0         # centre tap (1,1,1)
    y = _conv(x, wt, wv, L, grid)
    np.testing.assert_array_equal(y, x.astype(np.float64))


def test_impulse_response_is_cross_correlation():
    """An impulse at grid position p produces, at p - (a-1, b-1, e-1), the tap
    w[a, b, e]: the kernel is applied as a cross-correlation, centred."""
    rng = np.random.default_rng(1)
    T, Hg, Wg = 4, 5, 6
    L = 3
    x = np.zeros((L + T * Hg * Wg, 1), np.float32)
    pt, ph, pw = 2, 2, 3
    x[L + (pt * Hg + ph) * Wg + pw] = 1.0
    wv = rng.standard_normal((1, 27)).astype(np.float32)
    wt = rng.standard_normal((1, 4)).astype(np.float32)
    y = _conv(x, wt, wv, L, (T, Hg, Wg))[0, :, 0]
    expect = np.zeros_like(y)
    for a in range(3):
        for b in range(3):
            for e in range(3):
                t, h, w = pt - (a - 1), ph - (b - 1), pw - (e - 1)
                expect[L + (t * Hg + h) * Wg + w] = wv[0, (a * 3 + b) * 3 + e]
    np.testing.assert_array_equal(y, expect)


def test_text_impulse_is_causal_cross_correlation():
    wt = np.array([[1.0, 2.0, 3.0, 4.0]], np.float32)
    x = np.zeros((10, 1), np.float32)
    x[5] = 1.0
    y = _conv(x, wt, np.zeros((1, 27), np.float32), L=10, grid=(0, 1, 1))[0, :, 0]
    expect = np.zeros(10)
    expect[5:9] = [4.0, 3.0, 2.0, 1.0]   # y[t] = sum_j w[j] x[t-3+j]
    np.testing.assert_array_equal(y, expect)


def test_text_causality_and_modality_isolation():
    rng = np.random.default_rng(2)
    L, grid, C = 9, (2, 3, 4), 3
    N = L + 24
    x = rng.standard_normal((1, N, C)).astype(np.float32)
    wt = rng.standard_normal((C, 4)).astype(np.float32)
    wv = rng.standard_normal((C, 27)).astype(np.float32)
    y0 = _conv(x, wt, wv, L, grid)
    # perturb text token 5: text outputs < 5 and every visual output unchanged
    x1 = x.copy()
    x1[0, 5] += 1.0
    y1 = _conv(x1, wt, wv, L, grid)
    np.testing.assert_array_equal(y1[0, :5], y0[0, :5])
    np.testing.assert_array_equal(y1[0, L:], y0[0, L:])
    assert np.all(y1[0, 5:9] != y0[0, 5:9])
    # perturb a visual token: every text output unchanged
    x2 = x.copy()
    x2[0, L + 7] += 1.0
    y2 = _conv(x2, wt, wv, L, grid)
    np.testing.assert_array_equal(y2[0, :L], y0[0, :L])


@pytest.mark.parametrize("causal_t", [False, True])
def test_edge_counts(causal_t):
    """All-ones weights and input: each output counts its in-grid neighbours
    (27 interior, 18 face, 12 edge, 8 corner for the centred kernel)."""
    T, Hg, Wg = 4, 5, 6
    x = np.ones((T * Hg * Wg, 1), np.float32)
    y = _conv(x, np.ones((1, 4), np.float32), np.ones((1, 27), np.float32), 0, (T, Hg, Wg),
              causal_t=causal_t)[0, :, 0].reshape(T, Hg, Wg)

    def cnt(i, n):
        return (i > 0) + 1 + (i < n - 1)
    for t in range(T):
        ct = min(t + 1, 3) if causal_t else cnt(t, T)
        for h in range(Hg):
            for w in range(Wg):
                assert y[t, h, w] == ct * cnt(h, Hg) * cnt(w, Wg)
    if not causal_t:
        assert y[1, 1, 1] == 27 and y[0, 1, 1] == 18 and y[0, 0, 1] == 12 and y[0, 0, 0] == 8


def test_causal_t_reads_no_future_frame():
    rng = np.random.default_rng(3)
    T, Hg, Wg, C = 4, 3, 3, 2
    x = rng.standard_normal((1, T * Hg * Wg, C)).astype(np.float32)
    wt = np.zeros((C, 4), np.float32)
    wv = rng.standard_normal((C, 27)).astype(np.float32)
    y0 = _conv(x, wt, wv, 0, (T, Hg, Wg), causal_t=True)
    x1 = x.copy()
    x1[0, 2 * Hg * Wg:] += 1.0   # change frames 2 and 3
    y1 = _conv(x1, wt, wv, 0, (T, Hg, Wg), causal_t=True)
    np.testing.assert_array_equal(y1[0, :2 * Hg * Wg], y0[0, :2 * Hg * Wg])


def test_single_frame_uses_middle_temporal_slice():
    """T = 1: the centred kernel only meets the grid through its a=1 slice; the
    time-causal one only through a=2."""
    rng = np.random.default_rng(4)
    Hg, Wg, C = 4, 5, 2
    x = rng.standard_normal((1, Hg * Wg, C)).astype(np.float32)
    wv = rng.standard_normal((C, 27)).astype(np.float32)
    wt = np.zeros((C, 4), np.float32)
    for causal, keep in ((False, 1), (True, 2)):
        y = _conv(x, wt, wv, 0, (1, Hg, Wg), causal_t=causal)
        w2 = np.zeros_like(wv)
        w2[:, keep * 9:(keep + 1) * 9] = wv[:, keep * 9:(keep + 1) * 9]
        y2 = _conv(x, wt, w2, 0, (1, Hg, Wg), causal_t=causal)
        np.testing.assert_array_equal(y, y2)


def test_batch_items_independent_and_text_only_and_visual_only():
    rng = np.random.default_rng(5)
    C = 3
    wt = rng.standard_normal((C, 4)).astype(np.float32)
    wv = rng.standard_normal((C, 27)).astype(np.float32)
    for L, grid in ((6, (0, 2, 2)), (0, (2, 3, 2)), (5, (1, 2, 3))):
        N = L + grid[0] * grid[1] * grid[2]
        x = rng.standard_normal((3, N, C)).astype(np.float32)
        y = _conv(x, wt, wv, L, grid)
        for b in range(3):
            yb = _conv(x[b:b + 1], wt, wv, L, grid)
            np.testing.assert_array_equal(y[b:b + 1], yb)


def test_channel_range_matches_full():
    rng = np.random.default_rng(6)
    L, grid, C = 4, (2, 3, 3), 8
    x = rng.standard_normal((1, L + 18, C)).astype(np.float32)
    wt = rng.standard_normal((C, 4)).astype(np.float32)
    wv = rng.standard_normal((C, 27)).astype(np.float32)
    shape = oracle.conv_shape(1, L + 18, L, grid)
    full = oracle.shortconv(shape, x, wt, wv)
    part = oracle.shortconv(shape, x, wt, wv, 3, 6)
    np.testing.assert_array_equal(full[:, :, 3:6], part)


def test_matches_pure_python_loops():
    """A second, loop-by-loop evaluation on a tiny problem (offset form)."""
    rng = np.random.default_rng(7)
    L, (T, Hg, Wg), C = 5, (3, 2, 4), 2
    N = L + T * Hg * Wg
    x = rng.standard_normal((N, C)).astype(np.float32)
    wt = rng.standard_normal((C, 4)).astype(np.float32)
    wv = rng.standard_normal((C, 27)).astype(np.float32)
    y = _conv(x, wt, wv, L, (T, Hg, Wg))[0]
    ref = np.zeros((N, C))
    for c in range(C):
        for t in range(L):
            ref[t, c] = sum(float(wt[c, 3 - s]) * float(x[t - s, c]) for s in range(4) if t - s >= 0)
        for tt in range(T):
            for hh in range(Hg):
                for ww in range(Wg):
                    acc = 0.0
                    for dt in (-1, 0, 1):
                        for dh in (-1, 0, 1):
                            for dw in (-1, 0, 1):
                                t2, h2, w2 = tt + dt, hh + dh, ww + dw
                                if 0 <= t2 < T and 0 <= h2 < Hg and 0 <= w2 < Wg:
                                    acc += float(wv[c, ((dt + 1) * 3 + dh + 1) * 3 + dw + 1]) * \
                                        float(x[L + (t2 * Hg + h2) * Wg + w2, c])
                    ref[L + (tt * Hg + hh) * Wg + ww, c] = acc
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)
