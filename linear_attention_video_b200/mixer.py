"""Token-mixer layers of the hybrid-backbone comparison, with synthetic weights, for timing a
KDA/MLA 3:1 stack against an MHA/MLA 3:1 stack as the token count grows (paper.rainbus.top,
实验结果 and Figure 18; genai-atlas, "Evidence": the hybrid runs 2.14x faster at 255k tokens).

Only the KDA layer's short conv and scan are this library's kernels (``kda_fwd``); the linear
projections are bf16 cuBLAS GEMMs (torch.matmul), the gate activations are torch element-wise ops,
and the softmax attention of the MHA and MLA layers is PyTorch's fused scaled-dot-product attention
(a library kernel, like cuBLAS), bidirectional over all tokens.

Layer readings (the pages give no sizes for the MLA projections):
  * width D = H * d (16 heads of 128: width 2048, the largest trained model's);
  * MLA: latent c = x Wdkv of d_c = 512; per-head keys c Wuk of d_n = 96 and values c Wuv of 128;
    a key part shared by all heads, k_direct = x Wkr of d_r = 32; queries x Wq of d_n + d_r = 128 per
    head; softmax scale 1/sqrt(128);
  * MHA: q, k, v of 128 per head, softmax scale 1/sqrt(128);
  * KDA: q, k, v projections (q and k scaled to a norm of about 1 per head), log alpha =
    -softplus(x Wa - 5) per channel (alpha near 0.99), beta = sigmoid(x Wb) per head, the
    modality-aware short conv and the scan (no scale on q), output projection.
"""
from __future__ import annotations

import math

import torch
import torch.nn.functional as F

from . import alloc_workspace, kda_fwd, problem

D_LATENT, D_NOPE, D_DIRECT = 512, 96, 32
GATE_BIAS = -5.0   # log alpha = -softplus(x Wa - 5): alpha near 0.99, the long-memory regime


def _w(g, shape, fan_in, device, scale=1.0):
    return (torch.randn(*shape, generator=g) * (scale / math.sqrt(fan_in))).to(device=device, dtype=torch.bfloat16)


class MHALayer:
    def __init__(self, H, d, device="cuda", seed=0):
        g = torch.Generator().manual_seed(seed)
        D = H * d
        self.H, self.d = H, d
        self.wq, self.wk, self.wv = (_w(g, (D, D), D, device) for _ in range(3))
        self.wo = _w(g, (D, D), D, device)

    def attention(self, x):
        """Per-head softmax attention output [B, N, H, d] (bf16), before the output projection."""
        B, N, _ = x.shape
        q, k, v = ((x @ w).view(B, N, self.H, self.d).transpose(1, 2) for w in (self.wq, self.wk, self.wv))
        return F.scaled_dot_product_attention(q, k, v).transpose(1, 2)

    def __call__(self, x):
        B, N, _ = x.shape
        return self.attention(x).reshape(B, N, -1) @ self.wo


class MLALayer:
    def __init__(self, H, d, device="cuda", seed=1):
        g = torch.Generator().manual_seed(seed)
        D = H * d
        self.H, self.d = H, d
        self.wdkv = _w(g, (D, D_LATENT), D, device)
        self.wuk = _w(g, (D_LATENT, H * D_NOPE), D_LATENT, device)
        self.wuv = _w(g, (D_LATENT, H * d), D_LATENT, device)
        self.wkr = _w(g, (D, D_DIRECT), D, device)
        self.wq = _w(g, (D, H * (D_NOPE + D_DIRECT)), D, device)
        self.wo = _w(g, (H * d, D), H * d, device)

    def qkv(self, x):
        """Queries, keys (latent part and the shared part) and values, [B, N, H, .] bf16."""
        B, N, _ = x.shape
        c = x @ self.wdkv
        kc = (c @ self.wuk).view(B, N, self.H, D_NOPE)
        v = (c @ self.wuv).view(B, N, self.H, self.d)
        kr = (x @ self.wkr).view(B, N, 1, D_DIRECT).expand(B, N, self.H, D_DIRECT)
        q = (x @ self.wq).view(B, N, self.H, D_NOPE + D_DIRECT)
        return q, torch.cat([kc, kr], dim=3), v

    def attention(self, x):
        q, k, v = self.qkv(x)
        return F.scaled_dot_product_attention(q.transpose(1, 2), k.transpose(1, 2), v.transpose(1, 2)).transpose(1, 2)

    def __call__(self, x):
        B, N, _ = x.shape
        return self.attention(x).reshape(B, N, -1) @ self.wo


class KDALayer:
    """Projections, then the modality-aware short conv and the KDA scan of this library, then the
    output projection.  Sized for one token layout (text_len + T * Hg * Wg tokens)."""

    def __init__(self, B, H, d, text_len, grid, device="cuda", seed=2, vis_causal_t=False, workspace=None):
        g = torch.Generator().manual_seed(seed)
        D = H * d
        self.B, self.H, self.d, self.text_len, self.grid = B, H, d, text_len, tuple(grid)
        # q and k of norm about 1 per head (beta |k'|^2 < 2 keeps the delta-rule update contracting)
        self.wq, self.wk = (_w(g, (D, D), D, device, 1.0 / math.sqrt(d)) for _ in range(2))
        self.wv = _w(g, (D, D), D, device)
        self.wa = _w(g, (D, D), D, device)
        self.wb = _w(g, (D, H), D, device)
        self.wo = _w(g, (D, D), D, device)
        self.w_text = (torch.randn(3, D, 4, generator=g) / 2.0).to(device)
        self.w_vis = (torch.randn(3, D, 27, generator=g) / math.sqrt(27)).to(device)
        self.p = problem(B, H, d, text_len, self.grid, vis_causal_t=vis_causal_t)
        # the workspace (conv outputs, block records) can be shared by layers that run one after another
        self.ws = alloc_workspace(self.p, torch.bfloat16, device) if workspace is None else workspace

    def inputs(self, x):
        """q, k, v (bf16), log alpha (fp32, -softplus) and beta (bf16, sigmoid) of the scan."""
        B, N, _ = x.shape
        q, k, v = ((x @ w).view(B, N, self.H, self.d).contiguous() for w in (self.wq, self.wk, self.wv))
        la = (-F.softplus((x @ self.wa).float() + GATE_BIAS)).view(B, N, self.H, self.d).contiguous()
        beta = torch.sigmoid(x @ self.wb).contiguous()
        return q, k, v, la, beta

    def mix(self, x):
        """The scan output o [B, N, H, d] (bf16), before the output projection."""
        q, k, v, la, beta = self.inputs(x)
        o = torch.empty_like(q)
        kda_fwd(self.p, q, k, v, la, beta, self.w_text, self.w_vis, o, self.ws)
        return o

    def __call__(self, x):
        B, N, _ = x.shape
        return self.mix(x).view(B, N, -1) @ self.wo


def stack(kind: str, B, H, d, text_len, grid, device="cuda"):
    """Four token mixers: 'kda' = KDA, KDA, KDA, MLA; 'mha' = MHA, MHA, MHA, MLA (the pages' 3:1)."""
    if kind == "kda":
        first = KDALayer(B, H, d, text_len, grid, device, seed=10)
        layers = [first] + [KDALayer(B, H, d, text_len, grid, device, seed=10 + i, workspace=first.ws)
                            for i in (1, 2)]
    elif kind == "mha":
        layers = [MHALayer(H, d, device, seed=10 + i) for i in range(3)]
    else:
        raise ValueError(kind)
    return layers + [MLALayer(H, d, device, seed=20)]


def run_stack(layers, x):
    for layer in layers:
        x = x + layer(x)
    return x
