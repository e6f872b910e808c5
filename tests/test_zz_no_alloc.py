"""kda_chunk_fwd_noalloc, the entry point for callers that cannot allocate
device memory (allocator callbacks, runtimes that forbid allocation after
start-up, plugins given only their buffers): called through the C ABI, it must
give the same output as kda_chunk_fwd, on two calls in a row that share the
library's static scratch.  Collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

from tests._util import assert_parity

pytestmark = pytest.mark.gpu


def _inputs(B, N, H, d, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, N, H, d, generator=g)
    k = torch.randn(B, N, H, d, generator=g)
    q = q / q.norm(dim=-1, keepdim=True) * 0.5
    k = k / k.norm(dim=-1, keepdim=True) * 0.5
    v = torch.randn(B, N, H, d, generator=g)
    la = -torch.nn.functional.softplus(torch.randn(B, N, H, d, generator=g)) * 0.1
    beta = torch.sigmoid(torch.randn(B, N, H, generator=g))
    dev = lambda x, dt: x.to(dt).contiguous().cuda()
    return (dev(q, torch.bfloat16), dev(k, torch.bfloat16), dev(v, torch.bfloat16), dev(la, torch.float32),
            dev(beta, torch.bfloat16))


def test_noalloc_matches_chunk_fwd_on_two_calls():
    import linear_attention_video_b200 as kda
    lib = kda._lib
    B, N, H, d = 1, 1000, 16, 128            # 8 blocks x 16 heads: 16 MiB of scratch
    p = kda.problem(B, H, d, N, (0, 0, 0))
    ref_o = torch.empty(B, N, H, d, dtype=torch.bfloat16, device="cuda")
    ref_s = torch.empty(B, H, d, d, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    for call, seed in enumerate((11, 12)):
        q, k, v, la, beta = _inputs(B, N, H, d, seed)
        s0 = torch.randn(B, H, d, d, device="cuda") * 0.05
        ws = kda.alloc_workspace(p, torch.bfloat16)
        kda.kda_chunk_fwd(p, q, k, v, la, beta, ref_o, ws, initial_state=s0, final_state=ref_s)
        assert kda.kda_read_status(ws) == kda.KDA_OK
        ref_launches = kda.kda_last_launch_count()
        o = torch.full_like(ref_o, float("nan"))
        sn = torch.full_like(ref_s, float("nan"))
        rc = lib.kda_chunk_fwd_noalloc(ctypes.byref(p), kda.KDA_DT_BF16, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                       la.data_ptr(), beta.data_ptr(), s0.data_ptr(), o.data_ptr(), sn.data_ptr(),
                                       status.data_ptr(), stream)
        assert rc == kda.KDA_OK, kda.kda_status_str(rc)
        torch.cuda.synchronize()
        assert int(status.item()) == kda.KDA_OK
        assert kda.kda_last_launch_count() == ref_launches >= 1   # the same kernels as kda_chunk_fwd
        assert_parity(o.float().cpu().numpy(), ref_o.float().cpu().numpy(), "bf16", f"call {call} o")
        assert_parity(sn.cpu().numpy(), ref_s.cpu().numpy(), "bf16", f"call {call} state")
        # both entry points run the same kernels on the same inputs: the results agree bit for bit
        assert torch.equal(o, ref_o) and torch.equal(sn, ref_s)


def test_noalloc_matches_the_oracle_without_a_status_word():
    """The same entry point with device_status = NULL (conditions then go to a word inside the static
    array), against the oracle's recurrence on the same bf16 values."""
    import linear_attention_video_b200 as kda
    import oracle
    lib = kda._lib
    B, N, H, d = 1, 700, 4, 128
    p = kda.problem(B, H, d, N, (0, 0, 0))
    q, k, v, la, beta = _inputs(B, N, H, d, 13)
    s0 = torch.randn(B, H, d, d, device="cuda") * 0.05
    o = torch.full((B, N, H, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    sn = torch.full((B, H, d, d), float("nan"), device="cuda")
    rc = lib.kda_chunk_fwd_noalloc(ctypes.byref(p), kda.KDA_DT_BF16, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                   la.data_ptr(), beta.data_ptr(), s0.data_ptr(), o.data_ptr(), sn.data_ptr(), None,
                                   torch.cuda.current_stream().cuda_stream)
    assert rc == kda.KDA_OK, kda.kda_status_str(rc)
    torch.cuda.synchronize()
    wide = lambda x: x.float().cpu().numpy().astype(np.float64)   # noqa: E731
    for h in (0, 3):
        ref, ref_s = oracle.scan(wide(q[:, :, h]), wide(k[:, :, h]), wide(v[:, :, h]), wide(la[:, :, h]),
                                 wide(beta[:, :, h]), wide(s0[:, h]))
        assert_parity(o[:, :, h].float().cpu().numpy(), ref, "bf16", f"head {h} o")
        assert_parity(sn[:, h].cpu().numpy(), ref_s, "bf16", f"head {h} state")


def test_noalloc_rejects_problems_beyond_its_scratch():
    import linear_attention_video_b200 as kda
    lib = kda._lib
    p = kda.problem(1, 16, 128, 40000, (0, 0, 0))   # 313 blocks x 16 heads: ~626 MiB of scratch
    rc = lib.kda_chunk_fwd_noalloc(ctypes.byref(p), kda.KDA_DT_BF16, 256, 256, 256, 256, 256, None, 256, None,
                                   None, None)
    assert rc == kda.KDA_ERR_WORKSPACE
