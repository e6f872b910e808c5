"""Pins of the attention-layer oracle (oracle/mixer.py) against closed forms, invariants and brute force
on tiny inputs."""
import itertools
import math

import numpy as np

from oracle import mixer as om


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def test_zero_queries_average_the_values():
    # every score is 0: uniform weights, each output is the mean of its head's values
    rng = np.random.default_rng(0)
    N, H = 7, 3
    q = np.zeros((N, H, 5))
    k, v = _rand(rng, N, H, 5), _rand(rng, N, H, 4)
    o = om.softmax_attention(q, k, v, 0.7)
    assert np.allclose(o, np.broadcast_to(v.mean(axis=0), o.shape), atol=1e-14)


def test_one_dominant_key_selects_its_value():
    rng = np.random.default_rng(1)
    N, H, dk = 6, 2, 4
    k = np.zeros((N, H, dk))
    k[3, :, 0] = 1.0
    q = np.zeros((N, H, dk))
    q[:, :, 0] = 60.0                         # score 60 on token 3, 0 elsewhere
    v = _rand(rng, N, H, 3)
    o = om.softmax_attention(q, k, v, 1.0)
    assert np.allclose(o, np.broadcast_to(v[3], o.shape), atol=5 * math.exp(-60) * np.abs(v).max())


def test_single_token_returns_its_value():
    rng = np.random.default_rng(2)
    q, k, v = _rand(rng, 1, 2, 3), _rand(rng, 1, 2, 3), _rand(rng, 1, 2, 4)
    assert np.allclose(om.softmax_attention(q, k, v, 0.3), v, atol=0)


def test_permutations():
    # keys and values permuted together: same output; queries permuted: outputs permuted alike
    rng = np.random.default_rng(3)
    N, H = 9, 2
    q, k, v = _rand(rng, N, H, 4), _rand(rng, N, H, 4), _rand(rng, N, H, 3)
    o = om.softmax_attention(q, k, v, 0.5)
    perm = rng.permutation(N)
    assert np.allclose(om.softmax_attention(q, k[perm], v[perm], 0.5), o, atol=1e-13)
    assert np.allclose(om.softmax_attention(q[perm], k, v, 0.5), o[perm], atol=1e-13)


def test_brute_force_on_tiny_inputs():
    # the definition evaluated with Python scalars, one (query, head) at a time
    rng = np.random.default_rng(4)
    N, H, dk, dv = 4, 2, 3, 2
    q, k, v = _rand(rng, N, H, dk), _rand(rng, N, H, dk), _rand(rng, N, H, dv)
    scale = 0.9
    o = om.softmax_attention(q, k, v, scale)
    for n, h in itertools.product(range(N), range(H)):
        w = [math.exp(scale * sum(float(q[n, h, c]) * float(k[m, h, c]) for c in range(dk))) for m in range(N)]
        z = sum(w)
        for j in range(dv):
            ref = sum(w[m] * float(v[m, h, j]) for m in range(N)) / z
            assert abs(o[n, h, j] - ref) < 1e-13


def _mla_weights(rng, D, H, dc, dn, dr, dv):
    return {"wdkv": _rand(rng, D, dc) / math.sqrt(D), "wuk": _rand(rng, dc, H * dn) / math.sqrt(dc),
            "wuv": _rand(rng, dc, H * dv) / math.sqrt(dc), "wkr": _rand(rng, D, dr) / math.sqrt(D),
            "wq": _rand(rng, D, H * (dn + dr)) / math.sqrt(D), "wo": _rand(rng, H * dv, D) / math.sqrt(H * dv)}


def test_mla_without_the_shared_key_is_attention_on_latent_keys():
    # k_direct = 0: the shared part adds nothing to any score, so MLA is softmax attention with
    # keys c Wuk and the first d_n query channels, at the scale of the full query width
    rng = np.random.default_rng(5)
    D, H, dc, dn, dr, dv, N = 12, 3, 5, 4, 2, 3, 10
    w = _mla_weights(rng, D, H, dc, dn, dr, dv)
    w["wkr"] = np.zeros_like(w["wkr"])
    x = _rand(rng, N, D)
    c = x @ w["wdkv"]
    q = (x @ w["wq"]).reshape(N, H, dn + dr)[:, :, :dn]
    ref = om.softmax_attention(q, (c @ w["wuk"]).reshape(N, H, dn), (c @ w["wuv"]).reshape(N, H, dv),
                               1.0 / math.sqrt(dn + dr)).reshape(N, -1) @ w["wo"]
    assert np.allclose(om.mla(x, w, H), ref, atol=1e-13)


def test_mla_shared_key_is_the_same_for_every_head():
    # with Wuk = 0 every head scores only against k_direct; heads with equal query parts on it and
    # equal value maps then give equal outputs
    rng = np.random.default_rng(6)
    D, H, dc, dn, dr, dv, N = 12, 4, 5, 3, 2, 3, 8
    w = _mla_weights(rng, D, H, dc, dn, dr, dv)
    w["wuk"] = np.zeros_like(w["wuk"])
    wq = w["wq"].reshape(D, H, dn + dr)
    wq[:, :, dn:] = wq[:, :1, dn:]
    w["wq"] = wq.reshape(D, -1)
    wuv = w["wuv"].reshape(dc, H, dv)
    wuv[:] = wuv[:, :1, :]
    w["wuv"] = wuv.reshape(dc, -1)
    w["wo"] = np.eye(H * dv, D)
    out = om.mla(np.asarray(_rand(rng, N, D)), w, H)[:, :H * dv].reshape(N, H, dv)
    assert np.allclose(out, np.broadcast_to(out[:, :1, :], out.shape), atol=1e-13)


def test_mha_is_linear_in_the_value_map():
    rng = np.random.default_rng(7)
    D, H, N = 8, 2, 6
    w = {n: _rand(rng, D, D) / math.sqrt(D) for n in ("wq", "wk", "wv", "wo")}
    x = _rand(rng, N, D)
    w2 = dict(w, wv=2.5 * w["wv"])
    assert np.allclose(om.mha(x, w2, H), 2.5 * om.mha(x, w, H), atol=1e-13)
