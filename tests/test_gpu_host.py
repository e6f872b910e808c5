"""kda_fwd_host (host-resident inputs, segmented with copies overlapping the kernels) vs the oracle,
through the C ABI (needs a B200).

The segments cut each item's token stream at frame boundaries; the scan carries the state across
them and each segment's conv reads its neighbouring frames, so the result is the forward pass
itself: compared element by element with the oracle at the bounds of kda_fwd (fp32 1e-5 relative
L2; bf16 5e-3 relative L2 and 2e-2 max-abs), for one segment per item, several, and a last
segment shorter than the others.
"""
import dataclasses

import numpy as np
import pytest
import torch

import kda_synth
import oracle
from tests._util import assert_parity, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kda():
    import linear_attention_video_b200 as kda
    assert torch.cuda.is_available()
    return kda


def run_host(kda, w, inp, seg_frames, causal=False, S0=None):
    B, N, H, d = inp["shape"]
    p = kda.problem(B, H, d, w.text_len, w.grid, vis_causal_t=causal)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32

    def host(name, shape):   # bf16 arrays hold the raw bf16 bits
        x = torch.from_numpy(np.ascontiguousarray(inp[name]))
        if dt == torch.bfloat16 and name != "log_alpha":
            x = x.view(torch.bfloat16)
        return x.reshape(shape).pin_memory()
    q, k, v = (host(n, (B, N, H, d)) for n in ("q", "k", "v"))
    la = host("log_alpha", (B, N, H, d))
    beta = host("beta", (B, N, H))
    w_text = torch.from_numpy(np.ascontiguousarray(inp["w_text"], np.float32)).cuda()
    w_vis = torch.from_numpy(np.ascontiguousarray(inp["w_vis"], np.float32)).cuda()
    o = torch.empty(B, N, H, d, dtype=dt).pin_memory()
    s0 = None if S0 is None else torch.from_numpy(np.ascontiguousarray(S0, np.float32)).cuda()
    sn = torch.empty(B, H, d, d, dtype=torch.float32, device="cuda")
    ws = kda.alloc_fwd_host_workspace(p, dt, seg_frames)
    main, cin, cout = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    kda.kda_fwd_host(p, q, k, v, la, beta, w_text, w_vis, o, ws, seg_frames, initial_state=s0, final_state=sn,
                     stream=main, copy_in_stream=cin, copy_out_stream=cout)
    main.synchronize()
    assert kda.kda_read_status(ws, stream=main) == kda.KDA_OK
    return o.float().numpy(), sn.cpu().numpy()


@pytest.mark.parametrize("seg_frames", [1, 2, 3])
@pytest.mark.parametrize("causal", [False, True])
def test_host_fp32_segments(kda, seg_frames, causal):
    """fp32 (CUDA-core scan), B = 2 with a ragged text prefix, 5 frames: 5, 3 and 2 segments per item."""
    w = dataclasses.replace(kda_synth.WORKLOADS[0], B=2, text_len=13, grid=(5, 7, 9))
    inp = kda_synth.generate(w, 41)
    S0 = kda_synth.initial_state(42, w.B, w.H, w.d, w.d)
    ref, ref_s = oracle.forward(inp, w.text_len, w.grid, S0=S0, vis_causal_t=causal)
    o, s = run_host(kda, w, inp, seg_frames, causal, S0)
    assert_parity(o, ref, "f32", "o")
    assert rel_l2(s, ref_s) <= 1e-5


@pytest.mark.parametrize("seg_frames", [2, 8])
def test_host_bf16_d128(kda, seg_frames):
    """bf16, d = 128 (tensor-core scan on fp16 conv outputs), 64 text tokens + 5 x 8 x 8 frames."""
    w = kda_synth.Workload("host_bf16", 1, 4, 128, 64, (5, 8, 8), "bf16", 0.1)
    inp = kda_synth.generate(w, 43)
    ref, ref_s = oracle.forward(inp, w.text_len, w.grid)
    o, s = run_host(kda, w, inp, seg_frames)
    assert_parity(o, ref, "bf16", "o")
    assert rel_l2(s, ref_s) <= 5e-3


def test_host_text_only_and_causal_bf16(kda):
    """A text-only problem (no frames: one segment per item) and the temporally causal conv on the
    tensor-core path (halo of two frames before a segment, none after)."""
    w = dataclasses.replace(kda_synth.WORKLOADS[0], B=2, text_len=77, grid=(0, 0, 0))
    inp = kda_synth.generate(w, 44)
    ref, ref_s = oracle.forward(inp, w.text_len, w.grid)
    o, s = run_host(kda, w, inp, 4)
    assert_parity(o, ref, "f32", "o")
    assert rel_l2(s, ref_s) <= 1e-5
    w = kda_synth.Workload("host_bf16_causal", 1, 4, 128, 64, (5, 8, 8), "bf16", 0.1)
    inp = kda_synth.generate(w, 45)
    ref, _ = oracle.forward(inp, w.text_len, w.grid, vis_causal_t=True)
    o, _ = run_host(kda, w, inp, 2, causal=True)
    assert_parity(o, ref, "bf16", "o")
