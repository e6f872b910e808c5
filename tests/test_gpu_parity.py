"""CUDA path vs the CPU oracle, through the C ABI (needs a B200).

Small workloads are compared element by element; the full-size video and
4096^2 workloads on sampled value columns, which the oracle computes exactly
at any length (a column of the state only depends on the same column of v).
"""
import numpy as np
import pytest
import torch

import kda_synth
import oracle
from tests._util import assert_parity, rel_l2, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kda():
    import linear_attention_video_b200 as kda
    assert torch.cuda.is_available()
    return kda


_cache = {}


def workload_inputs(i, tokens=None):
    key = (i, tokens)
    if key not in _cache:
        w = kda_synth.WORKLOADS[i]
        _cache[key] = kda_synth.generate(w, kda_synth.seed_for(i), tokens=tokens)
    return _cache[key]


def run_fwd(kda, w, inp, chunk=64, S0=None, want_state=False, vis_causal_t=False, grid=None, text_len=None):
    B, N, H, d = inp["shape"]
    p = kda.problem(B, H, d, w.text_len if text_len is None else text_len, w.grid if grid is None else grid,
                    chunk=chunk, vis_causal_t=vis_causal_t)
    t = to_device(inp)
    dt = t["q"].dtype
    # outputs start as NaN: an element the kernels never write fails the finiteness check
    o = torch.full((B, N, H, d), float("nan"), dtype=dt, device="cuda")
    ws = kda.alloc_workspace(p, dt)
    s0 = None if S0 is None else torch.from_numpy(np.ascontiguousarray(S0, np.float32)).cuda()
    sn = torch.full((B, H, d, d), float("nan"), dtype=torch.float32, device="cuda") if want_state else None
    kda.kda_fwd(p, t["q"], t["k"], t["v"], t["log_alpha"], t["beta"], t["w_text"], t["w_vis"], o, ws,
                initial_state=s0, final_state=sn)
    assert kda.kda_read_status(ws) == kda.KDA_OK
    torch.cuda.synchronize()
    assert bool(torch.isfinite(o).all()), "unwritten or non-finite output elements"
    if want_state:
        assert bool(torch.isfinite(sn).all()), "unwritten or non-finite final state"
    return o.float().cpu().numpy(), (sn.cpu().numpy() if want_state else None)


@pytest.mark.parametrize("chunk", [16, 32, 64])
def test_tiny_fp32_exact_path(kda, chunk):
    w = kda_synth.WORKLOADS[0]
    inp = workload_inputs(0)
    S0 = kda_synth.initial_state(7, 1, w.H, w.d, w.d)
    ref, ref_s = oracle.forward(inp, w.text_len, w.grid, S0=S0)
    o, s = run_fwd(kda, w, inp, chunk=chunk, S0=S0, want_state=True)
    assert_parity(o, ref, "f32", "o")
    assert rel_l2(s, ref_s) <= 1e-5


@pytest.mark.parametrize("i", [1, 2])
def test_bf16_full_parity(kda, i):
    w = kda_synth.WORKLOADS[i]
    inp = workload_inputs(i)
    heads = [0, 7, 15]
    ref, _ = oracle.forward(inp, w.text_len, w.grid, heads=heads)
    o, _ = run_fwd(kda, w, inp)
    for h in heads:
        assert_parity(o[:, :, h], ref[:, :, h], "bf16", f"head {h}")


def sampled_columns(H, d=128):
    """One value column in every 16-column group of every head: each CTA of the serial state pass
    (16 columns per CTA, or 32 when the (item, head) pairs need narrower grids) owns some of them."""
    return [(h, 16 * g + (5 * g + 3 * h) % 16) for h in range(H) for g in range(d // 16)]


@pytest.mark.parametrize("i", [3, 4])
def test_bf16_full_size_sampled_columns(kda, i):
    w = kda_synth.WORKLOADS[i]
    inp = workload_inputs(i)
    items = sampled_columns(w.H, w.d)
    ref = oracle.forward_columns(inp, w.text_len, w.grid, items, workers=8)
    o, _ = run_fwd(kda, w, inp)        # every element is checked finite (NaN-poisoned output)
    got = np.stack([o[:, :, h, j] for h, j in items])
    assert_parity(got, ref, "bf16", f"{len(items)} sampled columns")
    for n, (h, j) in enumerate(items):
        assert_parity(got[n], ref[n], "bf16", f"head {h} col {j}")


def test_shortconv_entry_point(kda):
    w = kda_synth.WORKLOADS[2]
    inp = workload_inputs(2)
    B, N, H, d = inp["shape"]
    p = kda.problem(B, H, d, w.text_len, w.grid)
    t = to_device(inp)
    outs = [torch.empty_like(t["q"]) for _ in range(3)]
    kda.kda_shortconv_fwd(p, t["q"], t["k"], t["v"], t["w_text"], t["w_vis"], *outs)
    torch.cuda.synchronize()
    shape = oracle.conv_shape(B, N, w.text_len, w.grid)
    for idx, name in enumerate("qkv"):
        x = oracle.widen(inp[name], "bf16").reshape(B, N, H * d)
        ref = oracle.shortconv(shape, x, inp["w_text"][idx], inp["w_vis"][idx], 0, 256)
        got = outs[idx].reshape(B, N, H * d)[:, :, :256].float().cpu().numpy()
        # one bf16 rounding of an fp32 sum: within half a bf16 ulp plus fp32 accumulation error
        assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6), name


def test_chunk_entry_point_on_caller_convolved_inputs(kda):
    """kda_chunk_fwd on q', k', v' the caller already convolved (bf16): compared
    with the oracle's recurrence fed exactly those bf16 values."""
    w = kda_synth.WORKLOADS[1]
    inp = workload_inputs(1)
    B, N, H, d = inp["shape"]
    p = kda.problem(B, H, d, w.text_len, w.grid)
    t = to_device(inp)
    conv = [torch.empty_like(t["q"]) for _ in range(3)]
    kda.kda_shortconv_fwd(p, t["q"], t["k"], t["v"], t["w_text"], t["w_vis"], *conv)
    o1 = torch.empty_like(t["q"])
    ws = kda.alloc_workspace(p, t["q"].dtype)
    kda.kda_chunk_fwd(p, conv[0], conv[1], conv[2], t["log_alpha"], t["beta"], o1, ws)
    assert kda.kda_read_status(ws) == kda.KDA_OK
    got = o1.float().cpu().numpy()
    cv = [c.float().cpu().numpy().astype(np.float64) for c in conv]
    la = inp["log_alpha"].reshape(B, N, H, d).astype(np.float64)
    bt = oracle.widen(inp["beta"], "bf16").reshape(B, N, H).astype(np.float64)
    for h in (0, 9):
        ref, _ = oracle.scan(cv[0][:, :, h], cv[1][:, :, h], cv[2][:, :, h], la[:, :, h], bt[:, :, h])
        assert_parity(got[:, :, h], ref, "bf16", f"head {h}")


def test_bf16_tensor_core_state_io(kda):
    """Initial and final state through the tensor-core path (d = 128)."""
    import dataclasses
    w = dataclasses.replace(kda_synth.WORKLOADS[1], text_len=100, grid=(2, 9, 13))
    inp = kda_synth.generate(w, 31)
    B, N, H, d = inp["shape"]
    S0 = kda_synth.initial_state(8, B, H, d, d, std=0.05)
    ref, ref_s = oracle.forward(inp, w.text_len, w.grid, S0=S0, heads=[0, 3])
    o, s = run_fwd(kda, w, inp, S0=S0, want_state=True)
    for h in (0, 3):
        assert_parity(o[:, :, h], ref[:, :, h], "bf16", f"head {h}")
        assert rel_l2(s[:, h], ref_s[:, h]) < 5e-3


@pytest.mark.parametrize("B,H", [(1, 40), (3, 12), (2, 12)])
def test_bf16_tensor_core_many_heads(kda, B, H):
    """Many (batch item, head) pairs: 40 and 36 pairs run the record kernel and then the state-pass
    kernel, with 64 and 32 value columns per CTA; 24 pairs (two batch items) run records and state
    pass in one launch with 24 state CTAs; parity on a few heads."""
    import dataclasses
    w = dataclasses.replace(kda_synth.WORKLOADS[1], B=B, H=H, text_len=70, grid=(2, 11, 13))
    inp = kda_synth.generate(w, 41 + H)
    heads = [0, H // 2, H - 1]
    ref, _ = oracle.forward(inp, w.text_len, w.grid, heads=heads)
    o, _ = run_fwd(kda, w, inp)
    for h in heads:
        assert_parity(o[:, :, h], ref[:, :, h], "bf16", f"head {h}")


def test_bf16_left_padded_text_item(kda):
    """An item with 20 fewer text tokens, padded with zero tokens at the front of its text
    span, gives the unpadded item's outputs at its real tokens (tensor-core path)."""
    import dataclasses
    from tests.test_oracle_kda import _left_padded_pair
    w, padded, single, pad = _left_padded_pair()
    w = dataclasses.replace(w, H=padded["shape"][2])
    ref, _ = oracle.forward(single, w.text_len - pad, w.grid)
    o, _ = run_fwd(kda, w, padded)
    for h in range(w.H):
        assert_parity(o[1, pad:, h], ref[0, :, h], "bf16", f"head {h}")


def test_bf16_causal_t_conv(kda):
    """Temporal-causal 3D conv (taps on frames t-2..t) through the bf16 tensor-core path."""
    import dataclasses
    w = dataclasses.replace(kda_synth.WORKLOADS[1], H=4, text_len=30, grid=(4, 9, 13))
    inp = kda_synth.generate(w, 77)
    ref, _ = oracle.forward(inp, w.text_len, w.grid, vis_causal_t=True)
    o, _ = run_fwd(kda, w, inp, vis_causal_t=True)
    for h in range(w.H):
        assert_parity(o[:, :, h], ref[:, :, h], "bf16", f"head {h}")


def test_bf16_tensor_core_continuation(kda):
    """Two kda_chunk_fwd calls chained through the state equal one call (bf16, d = 128)."""
    w = kda_synth.WORKLOADS[1]
    inp = workload_inputs(1)
    B, N, H, d = inp["shape"]
    t = to_device(inp)
    q, k, v = (t[n] for n in "qkv")

    def call(lo, hi, s0):
        pp = kda.problem(B, H, d, hi - lo, (0, 0, 0))
        o = torch.empty(B, hi - lo, H, d, dtype=q.dtype, device="cuda")
        sn = torch.empty(B, H, d, d, device="cuda")
        ws = kda.alloc_workspace(pp, q.dtype)
        kda.kda_chunk_fwd(pp, *(x[:, lo:hi].contiguous() for x in (q, k, v, t["log_alpha"], t["beta"])), o, ws,
                          initial_state=s0, final_state=sn)
        assert kda.kda_read_status(ws) == kda.KDA_OK
        return o, sn
    o_full, s_full = call(0, N, None)
    m = 1000   # not a multiple of the 128-token block
    o_a, s_a = call(0, m, None)
    o_b, s_b = call(m, N, s_a)
    o_split = torch.cat([o_a, o_b], dim=1).float().cpu().numpy()
    assert rel_l2(o_split, o_full.float().cpu().numpy()) < 2e-3
    assert rel_l2(s_b.cpu().numpy(), s_full.cpu().numpy()) < 2e-3


def strong_gate_inputs(seed=5):
    """The 1024^2 image workload with gates far outside the long-memory regime on a few channels of
    two heads: log alpha drawn uniformly from [-5, 0] on every token, single tokens that forget
    completely (log alpha = -200 and -1e4), and 37 nats of decay inside one 64-token sub-chunk."""
    w = kda_synth.WORKLOADS[1]
    inp = dict(workload_inputs(1))
    B, N, H, d = inp["shape"]
    la = inp["log_alpha"].reshape(B, N, H, d).copy()
    rng = np.random.default_rng(seed)
    la[:, :, 2, :8] = -rng.uniform(0.0, 5.0, (B, N, 8))
    la[:, :, 2, 100:104] = -rng.uniform(0.0, 1.0, (B, N, 4))
    la[:, 700, 2, 50] = -200.0
    la[:, 1000:1003, 2, 51] = -1e4
    la[:, 3:40, 9, 7] = -1.0
    la[:, 2000:2064, 9, 64:80] = -rng.uniform(0.0, 5.0, (B, 64, 16))
    inp["log_alpha"] = la.reshape(inp["log_alpha"].shape).astype(np.float32)
    return w, inp


def test_bf16_strong_gates_parity(kda):
    """Forget gates of any strength go through the bf16 tensor-core path (every decay factor is a
    product of gates <= 1): parity with the oracle on the affected heads and an unaffected one."""
    w, inp = strong_gate_inputs()
    heads = [2, 9, 0]
    ref, _ = oracle.forward(inp, w.text_len, w.grid, heads=heads)
    o, _ = run_fwd(kda, w, inp)
    for h in heads:
        assert_parity(o[:, :, h], ref[:, :, h], "bf16", f"head {h}")


def test_bf16_d64_forward_parity(kda):
    """bf16 storage with d = 64 (the CUDA-core chunked scan): element-by-element parity."""
    import dataclasses
    w = dataclasses.replace(kda_synth.WORKLOADS[1], d=64, H=4, text_len=100, grid=(3, 11, 13))
    inp = kda_synth.generate(w, 64)
    B, N, H, d = inp["shape"]
    S0 = kda_synth.initial_state(10, B, H, d, d, std=0.05)
    ref, ref_s = oracle.forward(inp, w.text_len, w.grid, S0=S0)
    o, s = run_fwd(kda, w, inp, S0=S0, want_state=True)
    assert_parity(o, ref, "bf16", "d = 64")
    assert rel_l2(s, ref_s) < 5e-3


def test_chunk_length_invariance_and_continuation(kda):
    w = kda_synth.WORKLOADS[0]
    inp = workload_inputs(0)
    B, N, H, d = inp["shape"]
    o16, s16 = run_fwd(kda, w, inp, chunk=16, want_state=True)
    o64, s64 = run_fwd(kda, w, inp, chunk=64, want_state=True)
    assert rel_l2(o16, o64) < 1e-5 and rel_l2(s16, s64) < 1e-5
    # split the text prefix: scan tokens [0, m) then [m, N) from the carried state,
    # using the already-convolved sequence through kda_chunk_fwd
    p = kda.problem(B, H, d, w.text_len, w.grid)
    t = to_device(inp)
    conv = [torch.empty_like(t["q"]) for _ in range(3)]
    kda.kda_shortconv_fwd(p, t["q"], t["k"], t["v"], t["w_text"], t["w_vis"], *conv)
    m = 100
    parts = []
    state = None
    for lo, hi in ((0, m), (m, N)):
        pp = kda.problem(B, H, d, hi - lo, (0, 0, 0))
        sl = [c[:, lo:hi].contiguous() for c in conv]
        la, bt = t["log_alpha"][:, lo:hi].contiguous(), t["beta"][:, lo:hi].contiguous()
        o = torch.empty_like(sl[0])
        sn = torch.empty(B, H, d, d, device="cuda")
        ws = kda.alloc_workspace(pp, o.dtype)
        kda.kda_chunk_fwd(pp, sl[0], sl[1], sl[2], la, bt, o, ws, initial_state=state, final_state=sn)
        parts.append(o)
        state = sn
    torch.cuda.synchronize()
    o_split = torch.cat(parts, dim=1).cpu().numpy()
    assert rel_l2(o_split, o64) < 1e-5
    assert rel_l2(state.cpu().numpy(), s64) < 1e-5


@pytest.mark.parametrize("case", ["text_only", "visual_only", "ragged", "batch3", "causal_t", "tiny_grid"])
def test_edge_shapes_fp32(kda, case):
    """Shapes with ragged last chunks, one modality only, several batch items."""
    import dataclasses
    base = kda_synth.WORKLOADS[0]
    shapes = {
        "text_only": dict(text_len=77, grid=(0, 0, 0)),
        "visual_only": dict(text_len=0, grid=(3, 5, 7)),
        "ragged": dict(text_len=5, grid=(2, 3, 11)),
        "batch3": dict(text_len=9, grid=(2, 4, 4), B=3),
        "causal_t": dict(text_len=4, grid=(4, 3, 5)),
        "tiny_grid": dict(text_len=1, grid=(1, 1, 1)),
    }[case]
    w = dataclasses.replace(base, **shapes)
    inp = kda_synth.generate(w, 99)
    causal = case == "causal_t"
    ref, ref_s = oracle.forward(inp, w.text_len, w.grid, vis_causal_t=causal)
    o, s = run_fwd(kda, w, inp, chunk=32, want_state=True, vis_causal_t=causal)
    assert_parity(o, ref, "f32", case)
    assert rel_l2(s, ref_s) <= 1e-5


def test_empty_sequence_copies_state(kda):
    p = kda.problem(2, 2, 64, 0, (0, 0, 0))
    z = torch.empty(2, 0, 2, 64, device="cuda")
    la = torch.empty(2, 0, 2, 64, device="cuda")
    bt = torch.empty(2, 0, 2, device="cuda")
    wt = torch.zeros(3, 128, 4, device="cuda")
    wv = torch.zeros(3, 128, 27, device="cuda")
    s0 = torch.randn(2, 2, 64, 64, device="cuda")
    sn = torch.zeros_like(s0)
    ws = torch.empty(4096, dtype=torch.uint8, device="cuda")
    # zero-sized tensors may have a null data pointer: pass a valid dummy address
    dummy = torch.empty(16, device="cuda")
    args = [x if x.numel() else dummy for x in (z, z, z, la, bt)]
    kda.kda_fwd(p, *args, wt, wv, dummy, ws, initial_state=s0, final_state=sn)
    torch.cuda.synchronize()
    assert torch.equal(sn, s0)


def test_strong_decay_takes_exact_branch(kda):
    """A chunk whose decay exceeds the factorised range (log alpha = -50 on a
    few tokens) still matches the oracle on the fp32 path."""
    import dataclasses
    w = dataclasses.replace(kda_synth.WORKLOADS[0], text_len=40, grid=(1, 8, 8))
    inp = kda_synth.generate(w, 123)
    la = inp["log_alpha"].reshape(1, -1, w.H, w.d)
    la[0, 10, :, :5] = -50.0
    la[0, 70, 1, :] = -90.0
    inp["log_alpha"] = la.reshape(-1).copy()
    ref, _ = oracle.forward(inp, w.text_len, w.grid)
    o, _ = run_fwd(kda, w, inp, chunk=64)
    assert_parity(o, ref, "f32", "strong decay")


@pytest.mark.parametrize("B,H", [(1, 16), (2, 12)])
def test_bf16_record_reuse_reruns_only_the_state_pass(kda, B, H):
    """KDA_FLAG_REUSE_RECORDS: a second kda_chunk_fwd on the same inputs and workspace, from
    another initial state, launches the state pass alone and equals a fresh call bit for bit.  A
    fresh call runs the records and the state pass in one launch; the reused-record call runs the
    separate state-pass kernel, with 16 value columns per CTA for 16 (batch item, head) pairs and
    32 for 24, so both column widths are checked against the single launch."""
    import dataclasses
    w = dataclasses.replace(kda_synth.WORKLOADS[1], B=B, H=H)
    inp = kda_synth.generate(w, 60 + H) if (B, H) != (1, 16) else workload_inputs(1)
    B, N, H, d = inp["shape"]
    t = to_device(inp)
    args = [t[n] for n in ("q", "k", "v", "log_alpha", "beta")]
    s_a, s_b = (torch.from_numpy(kda_synth.initial_state(s, B, H, d, d)).cuda() for s in (3, 4))
    p = kda.problem(B, H, d, w.text_len, w.grid)
    p_reuse = kda.problem(B, H, d, w.text_len, w.grid, reuse_records=True)

    def out():
        return (torch.empty(B, N, H, d, dtype=t["q"].dtype, device="cuda"),
                torch.empty(B, H, d, d, dtype=torch.float32, device="cuda"))
    (o1, n1), (o2, n2), (o3, n3) = out(), out(), out()
    ws1, ws2 = kda.alloc_workspace(p, t["q"].dtype), kda.alloc_workspace(p, t["q"].dtype)
    kda.kda_chunk_fwd(p, *args, o1, ws1, initial_state=s_b, final_state=n1)
    kda.kda_chunk_fwd(p, *args, o2, ws2, initial_state=s_a, final_state=n2)
    kda.kda_chunk_fwd(p_reuse, *args, o3, ws2, initial_state=s_b, final_state=n3)
    assert kda.kda_last_launch_count() == 1
    assert kda.kda_read_status(ws2) == kda.KDA_OK
    assert torch.equal(o3, o1) and torch.equal(n3, n1)
    assert not torch.equal(o2, o1)


@pytest.mark.parametrize("world,causal", [(3, False), (2, True)])
def test_bf16_sequence_sharded_on_thread_ranks(kda, world, causal):
    """The sequence-sharded pass (frames split over ranks, conv halo exchange, per-rank state maps
    composed across ranks) with every rank a thread on this GPU: same result as the unsharded pass,
    and oracle parity on sampled value columns."""
    from linear_attention_video_b200 import seqshard
    w = kda_synth.WORKLOADS[2]
    inp = workload_inputs(2)
    B, N, H, d = inp["shape"]
    t = to_device(inp)
    S0 = kda_synth.initial_state(9, B, H, d, d)
    s0 = torch.from_numpy(S0).cuda()

    def rank_pass(comm):
        seg = seqshard.partition(w.text_len, w.grid, comm.world, causal)[comm.rank]
        x = tuple(t[n][:, seg.t0:seg.t1].contiguous() for n in ("q", "k", "v"))
        be = seqshard.GpuBackend(B, H, d, vis_causal_t=causal)
        return seqshard.seqshard_fwd(be, comm, x, t["log_alpha"][:, seg.t0:seg.t1].contiguous(),
                                     t["beta"][:, seg.t0:seg.t1].contiguous(), t["w_text"], t["w_vis"],
                                     w.text_len, w.grid, s0)
    outs = seqshard.LocalGroup(world, timeout_s=300).run(rank_pass)
    torch.cuda.synchronize()
    o = torch.cat([o_r for o_r, _ in outs], dim=1).float().cpu().numpy()
    s_last = outs[-1][1].cpu().numpy()
    o_full, s_full = run_fwd(kda, w, inp, S0=S0, want_state=True, vis_causal_t=causal)
    assert rel_l2(o, o_full) < 3e-3 and rel_l2(s_last, s_full) < 3e-3
    items = [(0, 0), (7, 77), (15, 127)]
    ref = oracle.forward_columns(inp, w.text_len, w.grid, items, S0=S0, vis_causal_t=causal)
    got = np.stack([o[:, :, h, j] for h, j in items])
    assert_parity(got, ref, "bf16", f"sharded over {world}")


def test_bf16_split_pass_with_fp16_activations_equals_fused(kda):
    """KDA_FLAG_QKV_F16: kda_shortconv_fwd writing fp16 q', k', v' and kda_chunk_fwd reading them
    reproduce kda_fwd (which keeps the same fp16 intermediates) bit for bit."""
    w = kda_synth.WORKLOADS[1]
    inp = workload_inputs(1)
    B, N, H, d = inp["shape"]
    t = to_device(inp)
    p = kda.problem(B, H, d, w.text_len, w.grid, qkv_f16=True)
    conv = [torch.empty(B, N, H, d, dtype=torch.float16, device="cuda") for _ in range(3)]
    kda.kda_shortconv_fwd(p, t["q"], t["k"], t["v"], t["w_text"], t["w_vis"], *conv)
    o_split = torch.empty_like(t["q"])
    ws = kda.alloc_workspace(p, t["q"].dtype)
    kda.kda_chunk_fwd(p, *conv, t["log_alpha"], t["beta"], o_split, ws)
    assert kda.kda_read_status(ws) == kda.KDA_OK
    o_fused, _ = run_fwd(kda, w, inp)
    assert np.array_equal(o_split.float().cpu().numpy(), o_fused)
