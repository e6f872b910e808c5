"""The C-ABI library loads, exports every symbol its header declares, and
rejects bad arguments on the host before touching the GPU (CPU only)."""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")
LIB = os.path.join(ROOT, "linear_attention_video_b200", "libkda.so")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:[A-Za-z_][\w\s\*]*?)\b(kda_\w+)\s*\(", src, flags=re.M)))


@pytest.fixture(scope="module")
def kda():
    if not os.path.exists(LIB):
        import importlib.util
        spec = importlib.util.spec_from_file_location("kda_build", os.path.join(ROOT, "linear_attention_video_b200", "build.py"))
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
        mod.build()
    import linear_attention_video_b200 as kda
    return kda


def test_header_declares_the_boundary():
    fns = declared_functions()
    for name in ("kda_shortconv_fwd", "kda_chunk_fwd", "kda_fwd", "kda_workspace_bytes", "kda_read_status"):
        assert name in fns


def test_library_exports_every_declared_symbol(kda):
    lib = ctypes.CDLL(LIB)
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(kda.EXPORTS) == set(declared_functions())


def _p(kda, **kw):
    args = dict(B=1, H=2, d=64, text_len=32, grid=(1, 14, 16))
    args.update(kw)
    return kda.problem(**args)


def test_sizes_and_workspace(kda):
    p = _p(kda)
    assert kda.kda_tokens(p) == 32 + 224
    ws = kda.kda_workspace_bytes(p, kda.KDA_DT_F32)
    assert ws >= 256 + 3 * 256 * 2 * 64 * 4
    assert kda.kda_workspace_bytes(p, kda.KDA_DT_BF16) < ws
    assert kda.kda_workspace_bytes(_p(kda, d=96), kda.KDA_DT_F32) == 0
    assert kda.kda_tokens(kda.problem(1, 1, 64, 5, (0, 3, 0))) == -1
    assert kda.kda_status_str(kda.KDA_ERR_MISALIGNED).startswith("data pointer")


def _call_fwd(kda, p, dt=0, q=256, k=256, v=256, la=256, beta=256, wt=256, wv=256, s0=None, o=256, sn=None,
              ws=512, ws_bytes=1 << 40):
    lib = kda._lib
    return lib.kda_fwd(ctypes.byref(p), dt, q, k, v, la, beta, wt, wv, s0, o, sn, ws, ws_bytes, None)


def test_host_side_rejections_launch_nothing(kda):
    """Fake (never dereferenced) addresses: validation fails before any CUDA call."""
    p = _p(kda)
    assert _call_fwd(kda, p, q=None) == kda.KDA_ERR_INVALID_ARG
    assert _call_fwd(kda, p, o=0x1008) == kda.KDA_ERR_MISALIGNED
    assert _call_fwd(kda, p, s0=0x1004) == kda.KDA_ERR_MISALIGNED
    assert _call_fwd(kda, p, ws=0x1010) == kda.KDA_ERR_WORKSPACE
    assert _call_fwd(kda, p, ws_bytes=100) == kda.KDA_ERR_WORKSPACE
    assert _call_fwd(kda, p, dt=7) == kda.KDA_ERR_INVALID_ARG
    assert _call_fwd(kda, _p(kda, B=0)) == kda.KDA_ERR_INVALID_ARG
    assert _call_fwd(kda, _p(kda, d=96)) == kda.KDA_ERR_UNSUPPORTED
    assert _call_fwd(kda, _p(kda, dv=128)) == kda.KDA_ERR_UNSUPPORTED
    assert _call_fwd(kda, _p(kda, chunk=48)) == kda.KDA_ERR_UNSUPPORTED
    assert _call_fwd(kda, _p(kda, vis_k=(3, 5, 3))) == kda.KDA_ERR_UNSUPPORTED
    assert _call_fwd(kda, _p(kda, text_k=9)) == kda.KDA_ERR_UNSUPPORTED
    assert _call_fwd(kda, _p(kda, grid=(1, 0, 16))) == kda.KDA_ERR_INVALID_ARG
    # one frame of 4096 x 4096 tokens x 128 channels exceeds the conv's 32-bit frame offsets
    assert _call_fwd(kda, _p(kda, d=128, H=1, grid=(1, 4096, 4096))) == kda.KDA_ERR_UNSUPPORTED
    bad = _p(kda)
    bad.flags = 1 << 5
    assert _call_fwd(kda, bad) == kda.KDA_ERR_INVALID_ARG
    # record reuse is a kda_chunk_fwd option: the conv and fused entry points reject it
    reuse = _p(kda)
    reuse.flags = kda.KDA_FLAG_REUSE_RECORDS
    assert _call_fwd(kda, reuse) == kda.KDA_ERR_INVALID_ARG
    assert kda._lib.kda_shortconv_fwd(ctypes.byref(reuse), 0, 256, 256, 256, 256, 256, 256, 256, 256, None) == \
        kda.KDA_ERR_INVALID_ARG
    assert kda._lib.kda_chunk_fwd_noalloc(ctypes.byref(reuse), 0, 256, 256, 256, 256, 256, None, 256, None, None,
                                          None) == kda.KDA_ERR_INVALID_ARG
    # fp16 activations: bf16 problems with d = 128 only; kda_fwd keeps its own and rejects the flag
    f16 = _p(kda, d=128)
    f16.flags = kda.KDA_FLAG_QKV_F16
    assert _call_fwd(kda, f16) == kda.KDA_ERR_INVALID_ARG
    assert _call_fwd(kda, f16, dt=1) == kda.KDA_ERR_UNSUPPORTED
    f16_64 = _p(kda, d=64)
    f16_64.flags = kda.KDA_FLAG_QKV_F16
    assert _call_fwd(kda, f16_64) == kda.KDA_ERR_UNSUPPORTED
    lib = kda._lib
    assert lib.kda_shortconv_fwd(ctypes.byref(p), 0, 256, 256, 256, 256, 256, 256, 256, 0x1002, None) == \
        kda.KDA_ERR_MISALIGNED
    assert lib.kda_chunk_fwd(ctypes.byref(p), 0, 256, 256, 256, 256, None, None, 256, None, 512, 1 << 40, None) == \
        kda.KDA_ERR_INVALID_ARG
    # host-buffer entry point: host-side checks before any CUDA call (no stream or event is touched)
    host = lambda pp, **kw: lib.kda_fwd_host(ctypes.byref(pp), kw.get("dt", 0), *[kw.get(n, 256) for n in (   # noqa: E731
        "q", "k", "v", "la", "beta", "wt", "wv", "s0", "o", "sn")], kw.get("seg", 4), kw.get("ws", 512),
        kw.get("ws_bytes", 1 << 40), None, None, None)
    assert host(p, seg=0) == kda.KDA_ERR_INVALID_ARG
    assert host(p, q=None) == kda.KDA_ERR_INVALID_ARG
    assert host(p, o=0x1008) == kda.KDA_ERR_MISALIGNED
    assert host(p, ws=0x1010) == kda.KDA_ERR_WORKSPACE
    assert host(p, ws_bytes=1000) == kda.KDA_ERR_WORKSPACE
    assert host(reuse) == kda.KDA_ERR_INVALID_ARG
    assert kda.kda_fwd_host_workspace_bytes(p, torch.bfloat16, 0) == 0
    assert kda.kda_fwd_host_workspace_bytes(p, torch.bfloat16, 4) > kda.kda_workspace_bytes(p, torch.bfloat16)
    # backward entry point: host-side checks before any CUDA call
    lib.kda_bwd.restype = ctypes.c_int
    bwd = lambda pp, **kw: lib.kda_bwd(ctypes.byref(pp), kw.get("dt", 0), *[kw.get(n, 256) for n in (   # noqa: E731
        "q", "k", "v", "la", "beta", "wt", "wv", "s0", "do", "dsn", "dq", "dk", "dv", "dla", "dbeta", "dwt", "dwv",
        "ds0")], kw.get("ws", 512), kw.get("ws_bytes", 1 << 40), None)
    for n in ("q", "do", "dq", "dla", "dwv"):
        assert bwd(p, **{n: None}) == kda.KDA_ERR_INVALID_ARG, n
    assert bwd(p, dv=0x1008) == kda.KDA_ERR_MISALIGNED
    assert bwd(p, ds0=0x1004) == kda.KDA_ERR_MISALIGNED
    assert bwd(p, ws=0x1010) == kda.KDA_ERR_WORKSPACE
    assert bwd(p, ws_bytes=1000) == kda.KDA_ERR_WORKSPACE
    assert bwd(reuse) == kda.KDA_ERR_INVALID_ARG
    assert kda.kda_bwd_workspace_bytes(p, torch.bfloat16) > kda.kda_workspace_bytes(p, torch.bfloat16)
    assert kda.kda_last_launch_count() == 0


def test_chunk_length_rules(kda):
    """chunk: 16, 32 or 64 where the CUDA-core scan runs (fp32; bf16 with d = 64); exactly 64 on the
    bf16 tensor-core path (d = 128), whose blocks are two 64-token sub-chunks; 128 nowhere."""
    for dt, d, chunk, want in [(1, 64, 16, kda.KDA_OK), (1, 128, 32, kda.KDA_OK), (0, 64, 32, kda.KDA_OK),
                               (0, 128, 64, kda.KDA_OK), (0, 128, 32, kda.KDA_ERR_UNSUPPORTED),
                               (0, 128, 16, kda.KDA_ERR_UNSUPPORTED), (0, 128, 128, kda.KDA_ERR_UNSUPPORTED),
                               (1, 64, 128, kda.KDA_ERR_UNSUPPORTED), (0, 64, 128, kda.KDA_ERR_UNSUPPORTED)]:
        p = _p(kda, d=d, chunk=chunk)
        assert (kda.kda_workspace_bytes(p, dt) > 0) == (want == kda.KDA_OK), (dt, d, chunk)
        if want != kda.KDA_OK:
            assert _call_fwd(kda, p, dt=dt) == want, (dt, d, chunk)


def test_selftest_entry_rejects_other_paths(kda):
    """The bounded-wait self-test runs only on the tensor-core path and for stages 1 and 2; host-side
    rejections launch nothing."""
    lib = kda._lib
    call = lambda pp, dt=0, stage=1, wait_us=100: lib.kda_selftest_wait_timeout(   # noqa: E731
        ctypes.byref(pp), dt, 256, 256, 256, 256, 256, 256, 512, 1 << 40, stage, wait_us, None)
    assert call(_p(kda, d=64)) == kda.KDA_ERR_UNSUPPORTED
    assert call(_p(kda, d=128), dt=1) == kda.KDA_ERR_UNSUPPORTED
    assert call(_p(kda, d=128), stage=0) == kda.KDA_ERR_INVALID_ARG
    assert call(_p(kda, d=128), stage=3) == kda.KDA_ERR_INVALID_ARG
    assert call(_p(kda, d=128), wait_us=0) == kda.KDA_ERR_INVALID_ARG
    assert kda.kda_last_launch_count() == 0


def test_binding_checks_tensors_before_the_call(kda):
    """The C ABI sees bare addresses, so the binding checks every tensor against the problem (element
    count, dtype, device, contiguity) and raises KdaError(KDA_ERR_INVALID_ARG) before anything reaches
    the library: a buffer too short for the problem never becomes an out-of-bounds device access.  Host
    tensors stand in everywhere, so the checks run without a GPU."""
    B, H, d, L, grid = 1, 2, 64, 8, (1, 2, 4)
    N = L + 8
    p = kda.problem(B, H, d, L, grid)
    z = lambda *shape, dtype=torch.float32: torch.zeros(*shape, dtype=dtype)   # noqa: E731
    base = dict(q=z(B, N, H, d), k=z(B, N, H, d), v=z(B, N, H, d), log_alpha=z(B, N, H, d), beta=z(B, N, H),
                o=z(B, N, H, d), w_text=z(3, H * d, 4), w_vis=z(3, H * d, 27), s0=z(B, H, d, d), sn=z(B, H, d, d),
                qo=z(B, N, H, d), ko=z(B, N, H, d), vo=z(B, N, H, d), ws=z(4096, dtype=torch.uint8),
                d_o=z(B, N, H, d), dq=z(B, N, H, d), dk=z(B, N, H, d), dv=z(B, N, H, d), dla=z(B, N, H, d),
                dbeta=z(B, N, H), dwt=z(3, H * d, 4), dwv=z(3, H * d, 27), ds0=z(B, H, d, d),
                status=z(1, dtype=torch.int32))
    calls = {
        "kda_fwd": (lambda a: kda.kda_fwd(p, a["q"], a["k"], a["v"], a["log_alpha"], a["beta"], a["w_text"],
                                          a["w_vis"], a["o"], a["ws"], initial_state=a["s0"], final_state=a["sn"]),
                    ("q", "k", "v", "log_alpha", "beta", "w_text", "w_vis", "o", "s0", "sn")),
        "kda_chunk_fwd": (lambda a: kda.kda_chunk_fwd(p, a["q"], a["k"], a["v"], a["log_alpha"], a["beta"], a["o"],
                                                      a["ws"], initial_state=a["s0"], final_state=a["sn"]),
                          ("q", "k", "v", "log_alpha", "beta", "o", "s0", "sn")),
        "kda_shortconv_fwd": (lambda a: kda.kda_shortconv_fwd(p, a["q"], a["k"], a["v"], a["w_text"], a["w_vis"],
                                                              a["qo"], a["ko"], a["vo"]),
                              ("q", "k", "v", "w_text", "w_vis", "qo", "ko", "vo")),
        "kda_chunk_fwd_noalloc": (lambda a: kda.kda_chunk_fwd_noalloc(p, a["q"], a["k"], a["v"], a["log_alpha"],
                                                                      a["beta"], a["o"], a["s0"], a["sn"],
                                                                      a["status"]),
                                  ("q", "k", "v", "log_alpha", "beta", "o", "s0", "sn")),
        "kda_bwd": (lambda a: kda.kda_bwd(p, a["q"], a["k"], a["v"], a["log_alpha"], a["beta"], a["w_text"],
                                          a["w_vis"], a["d_o"], a["dq"], a["dk"], a["dv"], a["dla"], a["dbeta"],
                                          a["dwt"], a["dwv"], a["ws"], initial_state=a["s0"], d_initial_state=a["ds0"]),
                    ("q", "d_o", "dq", "dk", "dv", "dla", "dbeta", "dwt", "dwv", "s0", "ds0")),
    }
    for where, (call, names) in calls.items():
        for n in names:
            bad = dict(base)
            bad[n] = base[n].reshape(-1)[:-1]          # one element short
            with pytest.raises(kda.KdaError) as e:
                call(bad)
            assert e.value.status == kda.KDA_ERR_INVALID_ARG and "elements" in str(e.value), (where, n)
        n = "beta" if "beta" in names else ("dbeta" if "dbeta" in names else "qo")
        bad = dict(base, **{n: base[n].to(torch.bfloat16)})     # wrong dtype for an fp32 problem
        with pytest.raises(kda.KdaError, match="dtype"):
            call(bad)
        bad = dict(base, v=base["v"].transpose(1, 2))            # right size, not contiguous
        if "v" in names:
            with pytest.raises(kda.KdaError, match="contiguous"):
                call(bad)
        with pytest.raises(kda.KdaError, match="CUDA tensor"):  # right sizes, host memory
            call(base)
    # kda_fwd_host takes q, k, v, log_alpha, beta, o on the host and the rest on the device
    host = lambda a: kda.kda_fwd_host(p, a["q"], a["k"], a["v"], a["log_alpha"], a["beta"], a["w_text"],   # noqa: E731
                                      a["w_vis"], a["o"], a["ws"], 2)
    with pytest.raises(kda.KdaError, match="elements"):
        host(dict(base, log_alpha=base["log_alpha"][:, :-1].contiguous()))
    with pytest.raises(kda.KdaError, match="(w_text|workspace) must be a CUDA tensor"):
        host(base)
