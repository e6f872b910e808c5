"""Sequence-sharded forward pass across ranks, on CPU.

The orchestration in ``linear_attention_video_b200.seqshard`` (frame partition,
conv halo exchange, per-rank affine state maps, their all-gather and
composition) runs here with the CPU oracle as its compute backend, over real
``gloo`` process groups (world sizes 2 and 3) and over thread-emulated ranks.
The concatenated per-rank outputs and the last rank's final state must equal
the unsharded oracle forward pass: the scan is the recurrence of
paper.rainbus.top (section 方法步骤详情, step (5)), which is affine in the
entering state, so the composition is exact up to fp64 rounding.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import kda_synth
import oracle
from linear_attention_video_b200 import seqshard

# tiny fp32 workload: 8 text tokens + a 6 x 3 x 4 visual grid (80 tokens), 2 heads of width 16
W = kda_synth.Workload("seq_tiny", 1, 2, 16, 8, (6, 3, 4), "f32", 0.1)
SEED = 11


class OracleBackend:
    """The two compute calls of the sharded pass through the CPU oracle (fp64)."""

    def __init__(self, B, H, d, vis_causal_t=False):
        self.B, self.H, self.d, self.causal = B, H, d, vis_causal_t

    def conv(self, q, k, v, w_text, w_vis, text_len, grid):
        B, N, H, d = q.shape
        shape = oracle.conv_shape(B, N, text_len, grid, vis_causal_t=self.causal)
        out = []
        for i, x in enumerate((q, k, v)):
            y = oracle.shortconv(shape, x.reshape(B, N, H * d).numpy().astype(np.float32),
                                 w_text[i].numpy(), w_vis[i].numpy())
            out.append(torch.from_numpy(y).reshape(B, N, H, d))
        return out

    def scan(self, q, k, v, log_alpha, beta, S0, text_len, grid, reuse):
        B, N, H, d = q.shape
        o = torch.zeros(B, N, H, d, dtype=torch.float64)
        SN = torch.zeros(B, H, d, d, dtype=torch.float64)
        for h in range(H):
            s0 = None if S0 is None else S0[:, h].double().numpy()
            oh, sh = oracle.scan(q[:, :, h].numpy(), k[:, :, h].numpy(), v[:, :, h].numpy(),
                                 log_alpha[:, :, h].numpy(), beta[:, :, h].numpy(), s0)
            o[:, :, h] = torch.from_numpy(oh)
            SN[:, h] = torch.from_numpy(sh)
        return o, SN


def _inputs():
    inp = kda_synth.generate(W, SEED)
    B, N, H, d = inp["shape"]
    t = {n: torch.from_numpy(np.ascontiguousarray(inp[n])).reshape(B, N, H, d) for n in ("q", "k", "v")}
    t["log_alpha"] = torch.from_numpy(inp["log_alpha"]).reshape(B, N, H, d).double()
    t["beta"] = torch.from_numpy(np.ascontiguousarray(inp["beta"])).reshape(B, N, H).double()
    t["w_text"] = torch.from_numpy(np.ascontiguousarray(inp["w_text"]))
    t["w_vis"] = torch.from_numpy(np.ascontiguousarray(inp["w_vis"]))
    S0 = torch.from_numpy(kda_synth.initial_state(SEED + 1, B, H, d, d))
    return inp, t, S0


def _rank_pass(comm, causal):
    """One rank's share: its tokens in, its outputs and exit state out."""
    inp, t, S0 = _inputs()
    seg = seqshard.partition(W.text_len, W.grid, comm.world, causal)[comm.rank]
    x = tuple(t[n][:, seg.t0:seg.t1].contiguous() for n in ("q", "k", "v"))
    be = OracleBackend(W.B, W.H, W.d, causal)
    return seqshard.seqshard_fwd(be, comm, x, t["log_alpha"][:, seg.t0:seg.t1].contiguous(),
                                 t["beta"][:, seg.t0:seg.t1].contiguous(), t["w_text"], t["w_vis"], W.text_len,
                                 W.grid, S0)


def _reference(causal):
    inp, _, S0 = _inputs()
    return oracle.forward(inp, W.text_len, W.grid, S0=S0.numpy(), vis_causal_t=causal)


def _check(outs, causal):
    o_ref, s_ref = _reference(causal)
    o = np.concatenate([np.asarray(o_r) for o_r, _ in outs], axis=1)
    assert o.shape == o_ref.shape
    err = np.abs(o - o_ref).max() / np.abs(o_ref).max()
    assert err < 1e-10, err
    s_err = np.abs(np.asarray(outs[-1][1]) - s_ref).max() / np.abs(s_ref).max()
    assert s_err < 1e-10, s_err


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gloo_worker(rank, world, port, causal, outdir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        o, s = _rank_pass(seqshard.DistComm(), causal)
        np.save(os.path.join(outdir, f"o{rank}.npy"), o.numpy())
        np.save(os.path.join(outdir, f"s{rank}.npy"), s.numpy())
    finally:
        dist.destroy_process_group()


def test_partition_covers_the_sequence_once():
    for world in (1, 2, 3):
        for causal in (False, True):
            segs = seqshard.partition(W.text_len, W.grid, world, causal)
            assert segs[0].t0 == 0 and segs[-1].t1 == W.N and segs[-1].f1 == W.grid[0]
            for a, b in zip(segs, segs[1:]):
                assert a.t1 == b.t0 and a.f1 == b.f0
            lo, hi = seqshard.conv_reach(causal)
            assert [s.halo_lo for s in segs] == [0] + [lo] * (world - 1)
            assert [s.halo_hi for s in segs] == [hi] * (world - 1) + [0]
    with pytest.raises(Exception):
        seqshard.partition(W.text_len, W.grid, 4, True)   # 6 frames cannot give 4 ranks 2 frames each


def test_composed_entry_state_is_the_sequential_map():
    rng = np.random.default_rng(5)
    maps = [(torch.from_numpy(rng.standard_normal((1, 2, 4, 4))), torch.from_numpy(rng.standard_normal((1, 2, 4, 4))))
            for _ in range(3)]
    S0 = torch.from_numpy(rng.standard_normal((1, 2, 4, 4)))
    S = S0.numpy()
    for r in range(3):
        assert np.allclose(seqshard.compose_entry_state(maps, r, S0).numpy(), S, atol=1e-12)
        S = maps[r][0].numpy() @ S + maps[r][1].numpy()


@pytest.mark.parametrize("world,causal", [(2, False), (3, False), (3, True)])
def test_gloo_ranks_match_the_unsharded_pass(world, causal, tmp_path):
    mp.spawn(_gloo_worker, args=(world, _free_port(), causal, str(tmp_path)), nprocs=world, join=True)
    outs = [(np.load(tmp_path / f"o{r}.npy"), np.load(tmp_path / f"s{r}.npy")) for r in range(world)]
    _check(outs, causal)


@pytest.mark.parametrize("world,causal", [(2, True), (3, False)])
def test_thread_ranks_match_the_unsharded_pass(world, causal):
    outs = seqshard.LocalGroup(world, timeout_s=120).run(lambda comm: _rank_pass(comm, causal))
    _check([(o.numpy(), s.numpy()) for o, s in outs], causal)


def test_a_failing_rank_stops_the_others():
    def fn(comm):
        if comm.rank == 1:
            raise RuntimeError("rank 1 fails before the exchange")
        return comm.all_gather(torch.zeros(1))
    with pytest.raises(RuntimeError, match="rank 1 fails"):
        seqshard.LocalGroup(3, timeout_s=30).run(fn)


def _reduce_worker(rank, world, port, outdir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        import bench
        got = bench.reduce_max(1.5 + rank, torch.device("cpu"), world)
        np.save(os.path.join(outdir, f"r{rank}.npy"), np.array([got]))
    finally:
        dist.destroy_process_group()


def test_bench_times_the_slowest_rank(tmp_path):
    """bench.py's multi-rank timing: every rank reports the largest of the ranks' times."""
    mp.spawn(_reduce_worker, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True)
    assert [float(np.load(tmp_path / f"r{r}.npy")[0]) for r in range(2)] == [2.5, 2.5]
