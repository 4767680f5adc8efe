"""Shared helpers of the GPU parity tests: tolerances and error measures.

Tolerances (the operator's accuracy bounds):
  * fp32 workload: max |gpu - oracle| <= 1e-5;
  * bf16 V1 with the per-head norm (outputs are O(1)): max abs <= 2e-2 and
    mean abs <= 2e-3;
  * bf16 outputs without the norm (V2, and V1 with the norm off): the same
    two bounds on |gpu - oracle| / max|oracle|.
"""
import json
import os

import numpy as np
import torch

TOL_FP32_MAX = 1e-5
TOL_BF16_MAX = 2e-2
TOL_BF16_MEAN = 2e-3


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().double().numpy()


def errors(got, ref, rel_to_max: bool):
    g = to_np(got) if isinstance(got, torch.Tensor) else np.asarray(got, np.float64)
    r = np.asarray(ref, np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.isfinite(g).all(), "non-finite GPU output"
    d = np.abs(g - r)
    if rel_to_max:
        d = d / np.abs(r).max()
    return float(d.max()), float(d.mean())


def assert_bf16_close(got, ref, rel_to_max: bool, what: str = ""):
    mx, mean = errors(got, ref, rel_to_max)
    assert mx <= TOL_BF16_MAX and mean <= TOL_BF16_MEAN, (
        "%s: max %.3e mean %.3e (rel_to_max=%s)" % (what, mx, mean, rel_to_max))
    return mx, mean


def assert_fp32_close(got, ref, what: str = ""):
    mx, _ = errors(got, ref, False)
    assert mx <= TOL_FP32_MAX, "%s: max %.3e" % (what, mx)
    return mx


def status_word(device="cuda"):
    return torch.zeros(1, dtype=torch.int32, device=device)


def assert_status_ok(st):
    torch.cuda.synchronize()
    assert int(st.item()) == 0, "device status %d" % int(st.item())


def record(name: str, **fields):
    """Append one JSON line about a parity check to the file named by the
    DA_PARITY_REPORT environment variable (nothing if it is unset)."""
    path = os.environ.get("DA_PARITY_REPORT")
    if not path:
        return
    fields["name"] = name
    with open(path, "a") as f:
        f.write(json.dumps(fields) + "\n")
