"""Helpers shared by the tests: inputs to torch tensors and error metrics."""
import os
import numpy as np
import torch

TOL_BF16_REL_L2 = 5e-3     # relative L2 error bound, bf16 inputs/outputs
TOL_BF16_MAX_ABS = 2e-2    # max-abs error bound, bf16
TOL_F32_REL_L2 = 1e-5      # relative L2 error bound, fp32 debug path


def to_device(inp: dict, device="cuda"):
    """kda_synth arrays -> device tensors in the storage dtypes of the C ABI."""
    B, N, H, d = inp["shape"]
    bf16 = inp["dtype"] == "bf16"

    def act(a, shape):
        t = torch.from_numpy(np.ascontiguousarray(a))
        t = t.view(torch.bfloat16) if bf16 else t
        return t.reshape(shape).to(device)
    out = {name: act(inp[name], (B, N, H, d)) for name in ("q", "k", "v")}
    out["beta"] = act(inp["beta"], (B, N, H))
    out["log_alpha"] = torch.from_numpy(inp["log_alpha"]).reshape(B, N, H, d).to(device)
    out["w_text"] = torch.from_numpy(np.ascontiguousarray(inp["w_text"])).to(device)
    out["w_vis"] = torch.from_numpy(np.ascontiguousarray(inp["w_vis"])).to(device)
    return out


def rel_l2(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / (den if den > 0 else 1.0))


def max_abs(x, ref):
    return float(np.max(np.abs(np.asarray(x, np.float64) - np.asarray(ref, np.float64)))) if np.size(ref) else 0.0


def assert_parity(x, ref, dtype, what=""):
    e, m = rel_l2(x, ref), max_abs(x, ref)
    log = os.environ.get("KDA_PARITY_LOG")
    if log:   # one line per comparison, for reporting the measured errors
        with open(log, "a") as f:
            f.write(f"{os.environ.get('PYTEST_CURRENT_TEST', '?').split(' ')[0]}\t{what}\t{dtype}\t{e:.3e}\t{m:.3e}\n")
    if dtype == "bf16":
        assert e <= TOL_BF16_REL_L2 and m <= TOL_BF16_MAX_ABS, f"{what}: rel_l2={e:.3e} max_abs={m:.3e}"
    else:
        assert e <= TOL_F32_REL_L2, f"{what}: rel_l2={e:.3e} max_abs={m:.3e}"
    return e, m
