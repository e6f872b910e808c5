"""fp64 CPU reference of the token-mixer layers timed against each other in the hybrid-backbone
comparison (paper.rainbus.top, 实验结果 and Figure 18: a KDA/MLA 3:1 stack against an MHA/MLA 3:1
stack as the token count grows; genai-atlas, "How it works" and "Evidence").

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: only ``tests/`` may import it.  Plain numpy
in fp64; a matmul is the only library step.

Layers (x: [N, D] hidden states of one batch item; weights as in ``linear_attention_video_b200.mixer``):
  * softmax attention, bidirectional over all N tokens, per head (the pages' MLA keeps "full
    bidirectional softmax attention");
  * MHA: q, k, v = x Wq, x Wk, x Wv per head, attention, output projection;
  * MLA (paper.rainbus.top, 前置知识 "Multi-head Latent Attention"): the hidden state is compressed to a
    latent c = x Wdkv, keys and values are decompressed from it per head (c Wuk, c Wuv), and every
    head's key also carries a part shared across heads, k_direct = x Wkr; queries are x Wq with a
    part for each key component; attention over the concatenated key, output projection;
The KDA layer's mixing step (short conv and scan) is ``oracle.forward`` itself.
"""
from __future__ import annotations

import numpy as np


def softmax_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float) -> np.ndarray:
    """o[n, h] = sum_m softmax_m(scale q[n, h] . k[m, h]) v[m, h]; q, k: [N, H, dk], v: [N, H, dv]."""
    q, k, v = (np.asarray(a, dtype=np.float64) for a in (q, k, v))
    N, H, _ = q.shape
    out = np.empty((N, H, v.shape[2]))
    for h in range(H):
        s = scale * (q[:, h, :] @ k[:, h, :].T)          # [N, N] scores
        s -= s.max(axis=1, keepdims=True)                # the softmax is shift invariant
        p = np.exp(s)
        p /= p.sum(axis=1, keepdims=True)
        out[:, h, :] = p @ v[:, h, :]
    return out


def mha(x: np.ndarray, w: dict, H: int) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    N = x.shape[0]
    q = (x @ w["wq"]).reshape(N, H, -1)
    k = (x @ w["wk"]).reshape(N, H, -1)
    v = (x @ w["wv"]).reshape(N, H, -1)
    o = softmax_attention(q, k, v, 1.0 / np.sqrt(q.shape[2]))
    return o.reshape(N, -1) @ w["wo"]


def mla(x: np.ndarray, w: dict, H: int) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    N = x.shape[0]
    c = x @ w["wdkv"]                                     # [N, d_c] latent
    kc = (c @ w["wuk"]).reshape(N, H, -1)                 # per-head keys from the latent
    v = (c @ w["wuv"]).reshape(N, H, -1)
    kr = x @ w["wkr"]                                     # [N, d_r], shared by every head
    q = (x @ w["wq"]).reshape(N, H, -1)                   # [N, H, d_n + d_r]
    k = np.concatenate([kc, np.repeat(kr[:, None, :], H, axis=1)], axis=2)
    o = softmax_attention(q, k, v, 1.0 / np.sqrt(q.shape[2]))
    return o.reshape(N, -1) @ w["wo"]
