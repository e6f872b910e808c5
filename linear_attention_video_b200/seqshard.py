"""Sequence-sharded forward pass over ranks (one process per GPU).

Each rank owns a contiguous run of the raster-ordered token stream: an even
split of the visual frames, rank 0 also holding the text prefix.  The work
splits as follows (every step runs in the library's kernels; this module only
moves tensors between ranks and composes the per-rank state maps):

1. Conv halo.  The 3D conv of a rank's first and last frames reads frames the
   neighbouring ranks own (one on each side for the centred conv; the two
   before it for the temporally causal one).  They arrive by point-to-point
   send/recv; the rank convolves its frames with that halo (kda_shortconv_fwd)
   and keeps its own frames.
2. State map.  Across a rank's tokens the recurrence
   S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
   (paper.rainbus.top, section 方法步骤详情 step (5)) is affine in the entering
   state: S_out = M_r S_in + B_r.  The rank scans its tokens from S_in = 0
   (giving B_r) and, reusing the block records (KDA_FLAG_REUSE_RECORDS), from
   S_in = I (giving M_r + B_r).
3. Exchange.  All ranks gather every (M_r, B_r) and compose the maps of the
   ranks before them with the initial state: S_in(r) = M_{r-1} S_in(r-1) + B_{r-1}.
4. Output.  The rank scans its tokens once more from S_in(r), again reusing
   the records; the last rank's final state is the sequence's.

Compute goes through a backend with two calls (``conv`` and ``scan``), so the
same orchestration runs on the GPU path (``GpuBackend``) and under test on any
other implementation of the two calls.  Communication goes through a ``comm``
object: ``DistComm`` (torch.distributed, one process per rank) or ``LocalGroup``
(every rank a thread of one process, for one-GPU runs and tests).
"""
from __future__ import annotations

import threading
from dataclasses import dataclass

import torch

from . import (kda_chunk_fwd, kda_shortconv_fwd, kda_last_launch_count, problem, alloc_workspace, KdaError,
               KDA_ERR_INVALID_ARG)


# ---------------------------------------------------------------------------
# partition
# ---------------------------------------------------------------------------
@dataclass(frozen=True)
class Segment:
    """Rank r's share of one sequence: frames [f0, f1) and tokens [t0, t1)."""
    rank: int
    f0: int
    f1: int
    t0: int
    t1: int
    halo_lo: int   # frames before f0 the conv reads (owned by lower ranks)
    halo_hi: int   # frames from f1 on the conv reads (owned by higher ranks)


def conv_reach(vis_causal_t: bool, kt: int = 3) -> tuple[int, int]:
    """Frames the temporal taps reach before and after the output frame."""
    lo = kt - 1 if vis_causal_t else (kt - 1) // 2
    return lo, kt - 1 - lo


def partition(text_len: int, grid, world: int, vis_causal_t: bool = False) -> list[Segment]:
    """Even split of the T frames over `world` ranks (the first T % world ranks get one more).

    Every rank needs at least as many frames as the conv reaches across a boundary, so that a
    halo comes from the direct neighbour only."""
    T, Hg, Wg = grid
    lo, hi = conv_reach(vis_causal_t)
    if world < 1 or T < world * max(1, lo, hi):
        raise KdaError(KDA_ERR_INVALID_ARG, "partition: too few frames for this many ranks")
    base, extra = divmod(T, world)
    segs, f = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        f0, f1 = f, f + n
        t0 = 0 if r == 0 else text_len + f0 * Hg * Wg
        t1 = text_len + f1 * Hg * Wg
        segs.append(Segment(r, f0, f1, t0, t1, lo if r > 0 else 0, hi if r < world - 1 else 0))
        f = f1
    return segs


# ---------------------------------------------------------------------------
# communication
# ---------------------------------------------------------------------------
class DistComm:
    """torch.distributed process group (one process per rank; NCCL on GPUs, gloo on CPU)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def exchange_halo(self, lo_send, hi_send, lo_shape, hi_shape, like):
        """Send lo_send (this rank's first frames) down and hi_send (its last frames) up;
        receive the halo frames below (lo_shape) and above (hi_shape).  Shapes of None skip."""
        d = self.dist
        ops, lo_recv, hi_recv = [], None, None
        if lo_shape is not None:
            lo_recv = torch.empty(lo_shape, dtype=like.dtype, device=like.device)
            ops.append(d.P2POp(d.irecv, lo_recv, self.rank - 1, self.group))
        if hi_shape is not None:
            hi_recv = torch.empty(hi_shape, dtype=like.dtype, device=like.device)
            ops.append(d.P2POp(d.irecv, hi_recv, self.rank + 1, self.group))
        if lo_send is not None:
            ops.append(d.P2POp(d.isend, lo_send.contiguous(), self.rank - 1, self.group))
        if hi_send is not None:
            ops.append(d.P2POp(d.isend, hi_send.contiguous(), self.rank + 1, self.group))
        if ops:
            if d.get_backend(self.group) == "nccl":
                reqs = d.batch_isend_irecv(ops)   # NCCL wants matching sends and receives grouped
            else:
                reqs = [op.op(op.tensor, op.peer, op.group) for op in ops]
            for req in reqs:
                req.wait()
        return lo_recv, hi_recv

    def all_gather(self, t):
        out = [torch.empty_like(t) for _ in range(self.world)]
        self.dist.all_gather(out, t.contiguous(), group=self.group)
        return out


class LocalGroup:
    """All ranks of a group as threads of one process (one-GPU runs and tests): the same
    exchanges as DistComm, through shared slots and a barrier with a time limit."""

    def __init__(self, world: int, timeout_s: float = 600.0):
        self.world = world
        self.barrier = threading.Barrier(world, timeout=timeout_s)
        self.slots = {}
        self.lock = threading.Lock()

    def comm(self, rank: int) -> "LocalComm":
        return LocalComm(self, rank)

    def run(self, fn):
        """fn(comm) on every rank, each in its own thread; returns the results by rank and
        re-raises the first exception (a failing rank breaks the barrier for the others)."""
        results, errors = [None] * self.world, []

        def body(r):
            try:
                results[r] = fn(self.comm(r))
            except BaseException as e:   # noqa: BLE001 - handed to the caller below
                errors.append(e)
                self.barrier.abort()

        threads = [threading.Thread(target=body, args=(r,)) for r in range(self.world)]
        for t in threads:
            t.start()
        for t in threads:
            t.join()
        if errors:
            raise errors[0]
        return results


class LocalComm:
    def __init__(self, group: LocalGroup, rank: int):
        self.group, self.rank, self.world = group, rank, group.world

    def _publish(self, items):
        g = self.group
        with g.lock:
            g.slots.update(items)
        g.barrier.wait()

    def exchange_halo(self, lo_send, hi_send, lo_shape, hi_shape, like):
        self._publish({("down", self.rank): lo_send, ("up", self.rank): hi_send})
        g = self.group
        lo_recv = g.slots[("up", self.rank - 1)].clone() if lo_shape is not None else None
        hi_recv = g.slots[("down", self.rank + 1)].clone() if hi_shape is not None else None
        g.barrier.wait()   # every rank has read before the slots are reused
        return lo_recv, hi_recv

    def all_gather(self, t):
        self._publish({("gather", self.rank): t})
        out = [self.group.slots[("gather", r)].clone() for r in range(self.world)]
        self.group.barrier.wait()
        return out


# ---------------------------------------------------------------------------
# GPU backend: the library's entry points
# ---------------------------------------------------------------------------
class GpuBackend:
    """conv and scan of one rank's segment through libkda (one workspace per segment shape).

    For bf16 problems with d = 128 the convolved q', k', v' travel in fp16 (KDA_FLAG_QKV_F16),
    the intermediate kda_fwd keeps, so the split pass has the fused pass's accuracy."""

    def __init__(self, B, H, d, chunk=64, vis_causal_t=False, stream=None):
        self.B, self.H, self.d, self.chunk, self.causal = B, H, d, chunk, vis_causal_t
        self.stream = stream
        self._ws = {}
        self.launches = 0   # kernels this backend has launched

    def _f16(self, dtype):
        return dtype == torch.bfloat16 and self.d == 128

    def _problem(self, text_len, grid, dtype, reuse=False):
        return problem(self.B, self.H, self.d, text_len, grid, chunk=self.chunk, vis_causal_t=self.causal,
                       reuse_records=reuse, qkv_f16=self._f16(dtype))

    def conv(self, q, k, v, w_text, w_vis, text_len, grid):
        p = self._problem(text_len, grid, q.dtype)
        out_dtype = torch.float16 if self._f16(q.dtype) else q.dtype
        outs = [torch.empty(q.shape, dtype=out_dtype, device=q.device) for _ in range(3)]
        kda_shortconv_fwd(p, q, k, v, w_text, w_vis, *outs, stream=self.stream)
        self.launches += kda_last_launch_count()
        return outs

    def scan(self, q, k, v, log_alpha, beta, S0, text_len, grid, reuse):
        """o, S_N of the segment; `reuse`: the previous scan of the same segment left its records."""
        dtype = beta.dtype   # the problem dtype (q', k', v' may be fp16)
        key = (text_len, tuple(grid), dtype)
        if key not in self._ws:
            self._ws[key] = alloc_workspace(self._problem(text_len, grid, dtype), dtype, q.device)
        ws = self._ws[key]
        o = torch.empty(v.shape, dtype=dtype, device=v.device)
        SN = torch.empty(self.B, self.H, self.d, self.d, dtype=torch.float32, device=q.device)
        kda_chunk_fwd(self._problem(text_len, grid, dtype, reuse), q, k, v, log_alpha, beta, o, ws, S0, SN,
                      stream=self.stream)
        self.launches += kda_last_launch_count()
        return o, SN


# ---------------------------------------------------------------------------
# the algorithm, per rank
# ---------------------------------------------------------------------------
def frames_of(x, seg_text_len, Hg, Wg, f_lo, f_hi, frame0):
    """Frames [f_lo, f_hi) of a segment tensor [B, n, ...] whose visual part starts at frame frame0
    after seg_text_len text tokens."""
    a = seg_text_len + (f_lo - frame0) * Hg * Wg
    b = seg_text_len + (f_hi - frame0) * Hg * Wg
    return x[:, a:b]


def convolve_segment(backend, comm, seg: Segment, x, w_text, w_vis, text_len, grid):
    """Conv of this rank's q, k, v (x: tuple of [B, t1-t0, H, d]) with the halo frames from its
    neighbours; returns the rank's own convolved q', k', v'."""
    T, Hg, Wg = grid
    seg_text = text_len if seg.rank == 0 else 0
    world = comm.world
    lo, hi = conv_reach(backend.causal)
    outs = []
    for xi in x:
        # this rank's first `hi` frames go down (the lower rank's upper halo), its last `lo` up
        lo_send = frames_of(xi, seg_text, Hg, Wg, seg.f0, seg.f0 + hi, seg.f0) if seg.rank > 0 and hi else None
        hi_send = frames_of(xi, seg_text, Hg, Wg, seg.f1 - lo, seg.f1, seg.f0) if seg.rank < world - 1 and lo else None
        fshape = lambda n: (xi.shape[0], n * Hg * Wg) + tuple(xi.shape[2:])
        lo_recv, hi_recv = comm.exchange_halo(lo_send, hi_send, fshape(seg.halo_lo) if seg.halo_lo else None,
                                              fshape(seg.halo_hi) if seg.halo_hi else None, xi)
        parts = ([xi[:, :seg_text]] if seg_text else []) + ([lo_recv] if lo_recv is not None else []) + \
            [xi[:, seg_text:]] + ([hi_recv] if hi_recv is not None else [])
        outs.append(torch.cat(parts, dim=1))
    n_ext = seg.f1 - seg.f0 + seg.halo_lo + seg.halo_hi
    yq, yk, yv = backend.conv(*outs, w_text, w_vis, seg_text, (n_ext, Hg, Wg))
    keep = []
    for y in (yq, yk, yv):
        vis = y[:, seg_text + seg.halo_lo * Hg * Wg: seg_text + (seg.halo_lo + seg.f1 - seg.f0) * Hg * Wg]
        keep.append(torch.cat([y[:, :seg_text], vis], dim=1) if seg_text else vis.contiguous())
    return keep


def segment_map(backend, seg: Segment, qc, kc, vc, log_alpha, beta, text_len, grid):
    """(M_r, B_r) of the rank's tokens: S_out = M_r S_in + B_r, each [B, H, d, d] fp32."""
    T, Hg, Wg = grid
    seg_text = text_len if seg.rank == 0 else 0
    sgrid = (seg.f1 - seg.f0, Hg, Wg)
    B_, H, d = qc.shape[0], qc.shape[2], qc.shape[3]
    _, Br = backend.scan(qc, kc, vc, log_alpha, beta, None, seg_text, sgrid, reuse=False)
    eye = torch.eye(d, dtype=torch.float32, device=qc.device).expand(B_, H, d, d).contiguous()
    _, MB = backend.scan(qc, kc, vc, log_alpha, beta, eye, seg_text, sgrid, reuse=True)
    return MB - Br, Br


def compose_entry_state(maps, rank, S0):
    """S_in of `rank` from the gathered maps [(M_0, B_0), ...] and the sequence's initial state."""
    S = torch.zeros_like(maps[0][1]) if S0 is None else S0.to(maps[0][1].dtype)
    for r in range(rank):
        M, Bm = maps[r]
        S = torch.matmul(M, S) + Bm
    return S


def seqshard_fwd(backend, comm, x, log_alpha, beta, w_text, w_vis, text_len, grid, S0=None):
    """This rank's outputs of the sequence-sharded forward pass.

    x: (q, k, v) of the rank's tokens [B, t1-t0, H, d]; log_alpha, beta: the same tokens.
    Returns (o [B, t1-t0, H, d], S_out [B, H, d, d]); the last rank's S_out is the final state."""
    seg = partition(text_len, grid, comm.world, backend.causal)[comm.rank]
    T, Hg, Wg = grid
    seg_text = text_len if seg.rank == 0 else 0
    sgrid = (seg.f1 - seg.f0, Hg, Wg)
    qc, kc, vc = convolve_segment(backend, comm, seg, x, w_text, w_vis, text_len, grid)
    M, Bm = segment_map(backend, seg, qc, kc, vc, log_alpha, beta, text_len, grid)
    Ms, Bs = comm.all_gather(M), comm.all_gather(Bm)
    S_in = compose_entry_state(list(zip(Ms, Bs)), seg.rank, S0)
    return backend.scan(qc, kc, vc, log_alpha, beta, S_in.contiguous(), seg_text, sgrid, reuse=True)
