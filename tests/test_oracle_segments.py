"""Segmented forward (the schedule of the host-buffer entry point) equals the whole forward (CPU only).

The host-buffer entry point cuts each batch item's token stream at frame boundaries: each
segment's conv runs over a view reaching the neighbouring frames its taps read (pt frames before,
2 - pt after; the outputs computed for those halo frames, which see zeros past the view, are
dropped), and each segment's scan enters with the state the previous segment left.  The claim
that this reproduces the forward exactly (the conv is local in time and the recurrence is a state
machine) is checked here with the oracle's own conv and scan, in fp64, against oracle.forward.
"""
import dataclasses

import numpy as np
import pytest

import kda_synth
import oracle


def _segmented_forward(inp, w, seg_frames, causal, S0, halo_after=True):
    B, N, H, d = inp["shape"]
    T, Hg, Wg = w.grid
    HW, L = Hg * Wg, w.text_len
    pt = 2 if causal else 1
    xs = oracle._widened(inp)
    o = np.zeros((B, N, H, d))
    SN = np.zeros((B, H, d, d))
    for b in range(B):
        S = None if S0 is None else np.asarray(S0[b])[None]
        starts = list(range(0, T, seg_frames)) if T else [0]
        for f0 in starts:
            f1 = min(T, f0 + seg_frames)
            fv0, fv1 = max(0, f0 - pt), min(T, f1 + (2 - pt if halo_after else 0))   # frames the conv reads
            v_lo = 0 if f0 == 0 else L + fv0 * HW                   # view: text with the first segment
            v_hi = L + fv1 * HW
            lv = L if f0 == 0 else 0
            shape = oracle.conv_shape(1, v_hi - v_lo, lv, (fv1 - fv0, Hg, Wg), vis_causal_t=causal)
            conv = [oracle.shortconv(shape, x[b:b + 1, v_lo:v_hi], inp["w_text"][i], inp["w_vis"][i])
                    for i, x in enumerate(xs)]
            s_lo, s_hi = (0 if f0 == 0 else L + f0 * HW), L + f1 * HW   # the segment's own tokens
            a, z = s_lo - v_lo, s_hi - v_lo
            la = inp["log_alpha"].reshape(B, N, H, d)[b:b + 1, s_lo:s_hi].astype(np.float64)
            bt = oracle.widen(inp["beta"], inp["dtype"]).reshape(B, N, H)[b:b + 1, s_lo:s_hi].astype(np.float64)
            S_next = np.zeros((1, H, d, d))
            for h in range(H):
                c = slice(h * d, (h + 1) * d)
                oh, sh = oracle.scan(conv[0][:, a:z, c], conv[1][:, a:z, c], conv[2][:, a:z, c], la[:, :, h],
                                     bt[:, :, h], None if S is None else S[:, h])
                o[b, s_lo:s_hi, h] = oh[0]
                S_next[:, h] = sh
            S = S_next
        SN[b] = S[0]
    return o, SN


@pytest.mark.parametrize("seg_frames", [1, 2, 4])
@pytest.mark.parametrize("causal", [False, True])
def test_segmented_forward_is_exact(seg_frames, causal):
    w = dataclasses.replace(kda_synth.WORKLOADS[0], B=2, H=1, text_len=9, grid=(5, 4, 6))
    inp = kda_synth.generate(w, 51)
    S0 = kda_synth.initial_state(52, w.B, w.H, w.d, w.d)
    ref, ref_s = oracle.forward(inp, w.text_len, w.grid, S0=S0, vis_causal_t=causal)
    o, s = _segmented_forward(inp, w, seg_frames, causal, S0)
    assert np.abs(o - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())
    assert np.abs(s - ref_s).max() <= 1e-12 * max(1.0, np.abs(ref_s).max())


def test_a_missing_halo_frame_is_caught():
    """Planted mistake: a view that stops at the segment's own last frame (no frame after it) changes
    the centred conv at segment ends, and the comparison above would catch it."""
    w = dataclasses.replace(kda_synth.WORKLOADS[0], B=1, H=1, text_len=9, grid=(4, 4, 6))
    inp = kda_synth.generate(w, 53)
    ref, _ = oracle.forward(inp, w.text_len, w.grid)
    o, _ = _segmented_forward(inp, w, 2, False, None)
    assert np.abs(o - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())
    o, _ = _segmented_forward(inp, w, 2, False, None, halo_after=False)
    assert np.abs(o - ref).max() > 1e-6
