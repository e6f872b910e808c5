"""Bounded device waits that run out (needs a B200).

Every wait of the tensor-core scan kernels (for a TMA copy, a tensor-core product or another warp)
gives up after a time limit, records KDA_ERR_TIMEOUT in the workspace status word, lets its other
copies land, frees its tensor memory and returns.  kda_selftest_wait_timeout makes one such wait run
out on purpose, by leaving one asynchronous load un-issued in one CTA: nothing faults, traps or hangs.
The test checks that the call returns promptly, that the status reads KDA_ERR_TIMEOUT, and that the
same GPU and stream then compute a normal pass correctly.
"""
import dataclasses
import time

import pytest
import torch

import kda_synth
import oracle
from tests._util import assert_parity, to_device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("stage", [1, 2], ids=["record_kernel", "state_pass"])
def test_bounded_wait_gives_up_and_the_gpu_stays_usable(stage):
    import linear_attention_video_b200 as kda
    w = dataclasses.replace(kda_synth.WORKLOADS[1], H=4, text_len=64, grid=(2, 16, 16))
    inp = kda_synth.generate(w, 17)
    B, N, H, d = inp["shape"]
    t = to_device(inp)
    p = kda.problem(B, H, d, w.text_len, w.grid)
    ws = kda.alloc_workspace(p, torch.bfloat16)
    o = torch.full((B, N, H, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    kda.kda_selftest_wait_timeout(p, t["q"], t["k"], t["v"], t["log_alpha"], t["beta"], o, ws, stage, 20000)
    assert kda.kda_read_status(ws) == kda.KDA_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 5.0          # a 20 ms limit, not the default half second, not a hang
    # the context survived: a normal pass on the same stream and workspace matches the oracle
    o.fill_(float("nan"))
    kda.kda_fwd(p, t["q"], t["k"], t["v"], t["log_alpha"], t["beta"], t["w_text"], t["w_vis"], o, ws)
    assert kda.kda_read_status(ws) == kda.KDA_OK
    assert bool(torch.isfinite(o).all())
    ref, _ = oracle.forward(inp, w.text_len, w.grid, heads=[0, 3])
    got = o.float().cpu().numpy()
    for h in (0, 3):
        assert_parity(got[:, :, h], ref[:, :, h], "bf16", f"head {h} after the timeout")
