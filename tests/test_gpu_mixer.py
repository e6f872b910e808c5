"""The token-mixer layers of the hybrid-backbone timing (needs a B200): each layer's mixing step on
the GPU against the oracle on the same bf16 inputs (attention for MHA and MLA, the short conv and
KDA scan for the KDA layer), and both four-layer stacks end to end."""
import numpy as np
import pytest
import torch

import oracle
from oracle import mixer as om
from tests._util import assert_parity

pytestmark = pytest.mark.gpu

H, D_HEAD, TEXT, GRID = 4, 128, 64, (2, 16, 16)
N = TEXT + GRID[0] * GRID[1] * GRID[2]


def _x(seed=0):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(1, N, H * D_HEAD, generator=g).to("cuda", torch.bfloat16)


def _f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def test_mha_attention_matches_the_oracle():
    from linear_attention_video_b200 import mixer
    layer = mixer.MHALayer(H, D_HEAD, seed=3)
    x = _x(1)
    q, k, v = ((x @ w).view(1, N, H, D_HEAD) for w in (layer.wq, layer.wk, layer.wv))
    ref = om.softmax_attention(_f64(q[0]), _f64(k[0]), _f64(v[0]), 1.0 / np.sqrt(D_HEAD))
    got = layer.attention(x)[0].float().cpu().numpy()
    assert_parity(got, ref, "bf16", "MHA attention")


def test_mla_attention_matches_the_oracle():
    from linear_attention_video_b200 import mixer
    layer = mixer.MLALayer(H, D_HEAD, seed=4)
    x = _x(2)
    q, k, v = layer.qkv(x)
    # the shared key part is the same in every head
    assert torch.equal(k[..., mixer.D_NOPE:], k[:, :, :1, mixer.D_NOPE:].expand_as(k[..., mixer.D_NOPE:]))
    ref = om.softmax_attention(_f64(q[0]), _f64(k[0]), _f64(v[0]), 1.0 / np.sqrt(mixer.D_NOPE + mixer.D_DIRECT))
    got = layer.attention(x)[0].float().cpu().numpy()
    assert_parity(got, ref, "bf16", "MLA attention")


def test_kda_layer_scan_matches_the_oracle():
    from linear_attention_video_b200 import mixer
    layer = mixer.KDALayer(1, H, D_HEAD, TEXT, GRID, seed=5)
    x = _x(3)
    q, k, v, la, beta = layer.inputs(x)
    o = layer.mix(x)
    inp = {"q": _bits(q), "k": _bits(k), "v": _bits(v), "log_alpha": la.cpu().numpy(), "beta": _bits(beta),
           "w_text": layer.w_text.cpu().numpy(), "w_vis": layer.w_vis.cpu().numpy(),
           "shape": (1, N, H, D_HEAD), "dtype": "bf16"}
    ref, _ = oracle.forward(inp, TEXT, GRID)
    assert_parity(o.float().cpu().numpy(), ref, "bf16", "KDA layer scan")


@pytest.mark.parametrize("kind", ["kda", "mha"])
def test_stacks_run_end_to_end(kind):
    from linear_attention_video_b200 import mixer
    layers = mixer.stack(kind, 1, H, D_HEAD, TEXT, GRID)
    y = mixer.run_stack(layers, _x(4))
    assert y.shape == (1, N, H * D_HEAD) and bool(torch.isfinite(y).all())
