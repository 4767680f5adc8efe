"""Noise-cancellation measurement through the decode kernel.

Step 4 of the lesson "Atencion Diferencial (V2)" ("medicion de la
cancelacion de ruido") builds a length-1024 query with one signal token
among noise and compares the signal-to-noise ratio of ordinary softmax
attention with that of differential attention; exercise 4 sweeps lambda from
0 (the first softmax alone) to 1 (full subtraction) and exercise 1 varies
the noise amplitude.  This module runs that sweep on the GPU:

  * the inputs come from ``inputs.snr_inputs`` (one configuration per noise
    amplitude and branch-noise correlation, one head per lambda value);
  * one call of the V1 decode kernel computes every configuration and every
    lambda; V is one-hot per group of keys, so the kernel's output rows are
    the differential weights w_j = a1_j - lambda a2_j themselves;
  * the ratio is the weight at the signal position over the RMS weight at
    every other position (the pages fix no formula; this is the reading).

Run ``python -m differential_attention_sm_b200.snr`` for the table.
"""
from __future__ import annotations

import numpy as np
import torch

from . import binding as _b
from . import inputs as _inputs


def weights_from_output(out: torch.Tensor, n_cfg: int, groups: int) -> np.ndarray:
    """Kernel output [C * G, H, dv] -> differential weights [C, H, G * dv]."""
    B, H, dv = out.shape
    if B != n_cfg * groups:
        raise ValueError("output batch %d != %d configurations x %d groups" % (B, n_cfg, groups))
    w = out.float().cpu().view(n_cfg, groups, H, dv).permute(0, 2, 1, 3)
    return w.reshape(n_cfg, H, groups * dv).double().numpy()


def signal_to_noise(w: np.ndarray, pos: int) -> np.ndarray:
    """w[..., pos] / RMS of w over the other positions (last axis)."""
    noise = np.delete(w, pos, axis=-1)
    rms = np.sqrt(np.mean(noise * noise, axis=-1))
    with np.errstate(divide="ignore", invalid="ignore"):
        return w[..., pos] / rms


def run_sweep(x: dict | None = None, *, device: str = "cuda", stream=None) -> dict:
    """Run the sweep on ``device``.  Returns the device inputs' weights
    [C, H, L], the ratios [C, H], the lambda grid and the configurations."""
    if x is None:
        x = _inputs.snr_inputs()
    q = x["q"].to(device)
    kc = x["k_cache"].to(device)
    vc = x["v_cache"].to(device)
    lam = x["lam"].to(device)
    out = _b.diffattn_v1_decode(q, kc, vc, lam, apply_norm=False, stream=stream)
    torch.cuda.synchronize()
    w = weights_from_output(out, len(x["configs"]), x["groups"])
    return {"weights": w, "snr": signal_to_noise(w, x["pos"]),
            "lam": x["lam"].numpy(), "configs": x["configs"], "pos": x["pos"]}


def table(res: dict) -> str:
    lam = res["lam"]
    lines = ["sigma  rho   softmax(lam=0)  best DiffAttn  at lam   gain"]
    for c, (sigma, rho) in enumerate(res["configs"]):
        s = res["snr"][c]
        i = int(np.nanargmax(s))
        lines.append("%5.2f %5.2f %14.2f %14.2f %8.2f %6.1fx" % (
            sigma, rho, s[0], s[i], lam[i], s[i] / s[0]))
    return "\n".join(lines)


if __name__ == "__main__":
    print(table(run_sweep()))
