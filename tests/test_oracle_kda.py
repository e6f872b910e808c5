"""Pins for the oracle's KDA recurrence (CPU only).

The update rule is the one printed on paper.rainbus.top (section 方法步骤详情,
step (5)); its qualitative semantics (channel-wise decay, scalar write strength,
causal scan, fixed-size state) are in section 前置知识.  The pages give no
worked numbers, so the recurrence is pinned by a hand-derived example, closed
forms, invariants and independent formulations (chunked, dense, printed form).
"""
import json
import os

import numpy as np
import pytest

import kda_synth
import oracle


def _rand_head(rng, N, dk, dv, la_scale=0.1, beta_std=1.0, unit_keys=True):
    q = rng.standard_normal((N, dk))
    k = rng.standard_normal((N, dk))
    if unit_keys:
        q /= np.linalg.norm(q, axis=1, keepdims=True)
        k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((N, dv))
    la = -np.logaddexp(0, rng.standard_normal((N, dk))) * la_scale
    beta = 1.0 / (1.0 + np.exp(-beta_std * rng.standard_normal(N)))
    return q, k, v, la, beta


def _scan1(q, k, v, la, beta, S0=None):
    o, S = oracle.scan(q[None], k[None], v[None], la[None], beta[None], None if S0 is None else S0[None])
    return o[0], S[0]


def test_hand_derived_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "kda_hand_d2.json")))
    q, k, v = (np.array(g[n], float) for n in ("q", "k", "v"))
    la = np.log(np.array(g["alpha"], float))
    beta = np.array(g["beta"], float)
    o, S = _scan1(q, k, v, la, beta)
    np.testing.assert_allclose(o, g["o"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(S, g["S_final"], rtol=0, atol=1e-14)


def test_matches_printed_update_form():
    rng = np.random.default_rng(10)
    q, k, v, la, beta = _rand_head(rng, 40, 8, 6)
    S0 = rng.standard_normal((8, 6))
    o, S = _scan1(q, k, v, la, beta, S0)
    o2, S2 = oracle.printed_form_scan(q, k, v, la, beta, S0)
    np.testing.assert_allclose(o, o2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S, S2, rtol=1e-12, atol=1e-13)


def test_beta_zero_is_pure_channel_decay():
    """beta = 0: nothing is written, so o_t = S_0^T (exp(g_t) * q_t) with
    g_t = sum_{i<=t} log alpha_i (per channel)."""
    rng = np.random.default_rng(11)
    q, k, v, la, _ = _rand_head(rng, 30, 8, 5)
    S0 = rng.standard_normal((8, 5))
    o, S = _scan1(q, k, v, la, np.zeros(30), S0)
    g = np.cumsum(la, axis=0)
    np.testing.assert_allclose(o, (q * np.exp(g)) @ S0, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(S, np.exp(g[-1])[:, None] * S0, rtol=1e-13, atol=1e-14)


def test_orthonormal_keys_exact_recall():
    """alpha = 1, beta = 1, orthonormal keys k_1..k_m written from a zero state:
    later tokens that only read (beta = 0) with q = k_j return v_j."""
    rng = np.random.default_rng(12)
    d, m = 8, 6
    Qm, _ = np.linalg.qr(rng.standard_normal((d, d)))
    keys = Qm[:, :m].T
    vals = rng.standard_normal((m, 5))
    N = 2 * m
    k = np.vstack([keys, rng.standard_normal((m, d))])
    v = np.vstack([vals, rng.standard_normal((m, 5))])
    q = np.vstack([rng.standard_normal((m, d)), keys])
    beta = np.concatenate([np.ones(m), np.zeros(m)])
    la = np.zeros((N, d))
    o, _ = _scan1(q, k, v, la, beta)
    np.testing.assert_allclose(o[m:], vals, rtol=0, atol=1e-13)


def test_same_key_twice_keeps_second_value():
    """Delta rule overwrites: writing (k, v1) then (k, v2) with alpha = 1, beta = 1
    and |k| = 1 stores v2 under k."""
    rng = np.random.default_rng(13)
    d = 6
    kk = rng.standard_normal(d)
    kk /= np.linalg.norm(kk)
    v1, v2 = rng.standard_normal(4), rng.standard_normal(4)
    k = np.vstack([kk, kk, rng.standard_normal(d)])
    v = np.vstack([v1, v2, rng.standard_normal(4)])
    q = np.vstack([kk, kk, kk])
    beta = np.array([1.0, 1.0, 0.0])
    o, S = _scan1(q, k, v, np.zeros((3, d)), beta)
    np.testing.assert_allclose(o[0], v1, atol=1e-14)
    np.testing.assert_allclose(o[1], v2, atol=1e-14)
    np.testing.assert_allclose(o[2], v2, atol=1e-14)


def test_linear_in_values_and_initial_state():
    rng = np.random.default_rng(14)
    q, k, v1, la, beta = _rand_head(rng, 50, 8, 4)
    v2 = rng.standard_normal(v1.shape)
    s1, s2 = rng.standard_normal((8, 4)), rng.standard_normal((8, 4))
    a, b = 0.7, -1.3
    o1, S1 = _scan1(q, k, v1, la, beta, s1)
    o2, S2 = _scan1(q, k, v2, la, beta, s2)
    o3, S3 = _scan1(q, k, a * v1 + b * v2, la, beta, a * s1 + b * s2)
    np.testing.assert_allclose(o3, a * o1 + b * o2, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S3, a * S1 + b * S2, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("chunk", [1, 16, 32, 64, 128, 200])
def test_chunked_form_equals_recurrence(chunk):
    rng = np.random.default_rng(15)
    N = 200   # 200 = 3*64 + 8: ragged tail for chunk 64, 1 chunk for 200
    q, k, v, la, beta = _rand_head(rng, N, 16, 12)
    S0 = rng.standard_normal((16, 12)) * 0.3
    o, S = _scan1(q, k, v, la, beta, S0)
    oc, Sc = oracle.chunked_scan(q, k, v, la, beta, S0, chunk=chunk)
    np.testing.assert_allclose(oc, o, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(Sc, S, rtol=1e-11, atol=1e-12)


def test_dense_form_equals_recurrence():
    rng = np.random.default_rng(16)
    q, k, v, la, beta = _rand_head(rng, 96, 8, 6, la_scale=0.05)
    o, _ = _scan1(q, k, v, la, beta)
    np.testing.assert_allclose(oracle.dense_scan(q, k, v, la, beta), o, rtol=1e-10, atol=1e-12)


def test_sequence_continuation():
    rng = np.random.default_rng(17)
    q, k, v, la, beta = _rand_head(rng, 150, 8, 8)
    o, S = _scan1(q, k, v, la, beta)
    m = 67
    oa, Sa = _scan1(q[:m], k[:m], v[:m], la[:m], beta[:m])
    ob, Sb = _scan1(q[m:], k[m:], v[m:], la[m:], beta[m:], Sa)
    np.testing.assert_allclose(np.vstack([oa, ob]), o, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(Sb, S, rtol=1e-13, atol=1e-14)


def test_strong_decay_and_edge_values():
    """Extreme but finite gates: log alpha = -60 erases the state; beta in {0, 1}."""
    rng = np.random.default_rng(18)
    q, k, v, la, beta = _rand_head(rng, 64, 8, 4)
    la[20] = -60.0
    beta[::3] = 0.0
    beta[1::3] = 1.0
    o, S = _scan1(q, k, v, la, beta)
    oc, Sc = oracle.chunked_scan(q, k, v, la, beta, chunk=16)
    np.testing.assert_allclose(oc, o, rtol=1e-10, atol=1e-12)
    # after the erase at t=20 the output no longer depends on tokens < 20
    v2 = v.copy()
    v2[:20] += 5.0
    o2, _ = _scan1(q, k, v2, la, beta)
    np.testing.assert_allclose(o2[20:], o[20:], atol=1e-20)


def test_batch_items_independent_and_empty_sequence():
    rng = np.random.default_rng(19)
    heads = [_rand_head(rng, 33, 8, 8) for _ in range(3)]
    q, k, v, la, beta = (np.stack([h[i] for h in heads]) for i in range(5))
    o, S = oracle.scan(q, k, v, la, beta)
    for b in range(3):
        ob, Sb = _scan1(*(x[b] for x in (q, k, v, la, beta)))
        np.testing.assert_array_equal(o[b], ob)
        np.testing.assert_array_equal(S[b], Sb)
    S0 = rng.standard_normal((1, 8, 8))
    o0, S0out = oracle.scan(q[:1, :0], k[:1, :0], v[:1, :0], la[:1, :0], beta[:1, :0], S0)
    assert o0.shape == (1, 0, 8)
    np.testing.assert_array_equal(S0out, S0)


def test_sampled_columns_equal_full_forward():
    import kda_synth
    w = kda_synth.WORKLOADS[0]
    inp = kda_synth.generate(w, kda_synth.seed_for(0))
    o, _ = oracle.forward(inp, w.text_len, w.grid)
    items = [(0, 0), (1, 17), (1, 63)]
    oc = oracle.forward_columns(inp, w.text_len, w.grid, items)
    for i, (h, j) in enumerate(items):
        np.testing.assert_allclose(oc[i], o[:, :, h, j], rtol=1e-13, atol=1e-14)


def test_full_block_against_chunked_form_on_tiny_workload():
    """Conv + scan on the tiny workload: the recurrence agrees with the chunked
    form fed the same convolved inputs."""
    import kda_synth
    w = kda_synth.WORKLOADS[0]
    inp = kda_synth.generate(w, kda_synth.seed_for(0))
    o, SN = oracle.forward(inp, w.text_len, w.grid)
    B, N, H, d = inp["shape"]
    shape = oracle.conv_shape(B, N, w.text_len, w.grid)
    for h in range(H):
        qh, kh, vh, la, bt = oracle._heads_inputs(inp, h, shape, d)
        oc, Sc = oracle.chunked_scan(qh[0], kh[0], vh[0], la[0], bt[0], chunk=64)
        np.testing.assert_allclose(oc, o[0, :, h], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(Sc, SN[0, h], rtol=1e-10, atol=1e-12)


# --- planted mistakes: each plausible slip in a formulation fails a pin -----

def _chunked_with(mistake, q, k, v, la, beta, chunk):
    N, dk = q.shape
    S = np.zeros((dk, v.shape[1]))
    o = np.zeros((N, v.shape[1]))
    for c0 in range(0, N, chunk):
        sl = slice(c0, min(N, c0 + chunk))
        qc, kc, vc, lac, bc = q[sl], k[sl], v[sl], la[sl], beta[sl]
        g, A, P, T = oracle._chunk_terms(qc, kc, lac, bc)
        if mistake == "transpose_T":
            T = T.T
        W = T @ (kc * np.exp(g))
        U = T @ vc + (W @ S if mistake == "sign" else -(W @ S))
        if mistake == "drop_decay":
            o[sl] = qc @ S + P @ U
        else:
            o[sl] = (qc * np.exp(g)) @ S + P @ U
        S = np.exp(g[-1])[:, None] * S + (kc * np.exp(g[-1][None, :] - g)).T @ U
    return o


@pytest.mark.parametrize("mistake", ["transpose_T", "sign", "drop_decay"])
def test_planted_mistakes_are_caught(mistake):
    rng = np.random.default_rng(20)
    q, k, v, la, beta = _rand_head(rng, 96, 8, 6)
    o, _ = _scan1(q, k, v, la, beta)
    bad = _chunked_with(mistake, q, k, v, la, beta, 32)
    assert np.max(np.abs(bad - o)) > 1e-3


def _left_padded_pair(pad=20):
    """A two-item batch whose second item has `pad` fewer text tokens, stored as zero
    tokens (q = k = v = 0, log alpha = 0, beta = 0) at the front of its text span, and
    the same second item as a batch of one with the shorter text."""
    import dataclasses
    w = dataclasses.replace(kda_synth.WORKLOADS[1], B=2, H=2, text_len=60, grid=(2, 5, 7))
    inp = kda_synth.generate(w, 5)
    B, N, H, d = inp["shape"]
    padded = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in inp.items()}
    for name in ("q", "k", "v", "log_alpha"):
        a = padded[name].reshape(B, N, H, d)
        a[1, :pad] = 0
    padded["beta"].reshape(B, N, H)[1, :pad] = 0
    single = dict(inp, shape=(1, N - pad, H, d))
    for name in ("q", "k", "v", "log_alpha"):
        single[name] = np.ascontiguousarray(inp[name].reshape(B, N, H, d)[1, pad:]).reshape(-1)
    single["beta"] = np.ascontiguousarray(inp["beta"].reshape(B, N, H)[1, pad:]).reshape(-1)
    return w, padded, single, pad


def test_left_padded_text_is_exact():
    """Items with fewer text tokens: leading zero tokens leave the state and the causal text
    conv untouched, so the real tokens' outputs equal those of the unpadded item."""
    w, padded, single, pad = _left_padded_pair()
    o_pad, s_pad = oracle.forward(padded, w.text_len, w.grid)
    o_one, s_one = oracle.forward(single, w.text_len - pad, w.grid)
    np.testing.assert_allclose(o_pad[1, pad:], o_one[0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(s_pad[1], s_one[0], rtol=0, atol=1e-12)
