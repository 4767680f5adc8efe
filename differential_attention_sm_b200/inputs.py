"""Seeded synthetic inputs for differential attention.

This module only draws random numbers and lays them out.  It holds none of
the operator's arithmetic, so both the CUDA path (tests, benchmark) and the
fp64 oracle can take their inputs from it.

Recipe (shared by every test and the benchmark):
  * generator: ``torch.Generator()`` (CPU, MT19937) seeded per workload;
  * draw order: Q, K, V, then the lambda inputs (four [H, d] vectors with
    std 0.1 for V1, or one U(0.2, 0.8) value per query-head pair for V2),
    then planted key positions;
  * values ~ N(0, 1) in float32, rounded to bf16 (round-to-nearest-even)
    for bf16 workloads; the oracle reads the rounded values;
  * decode caches are drawn one batch entry at a time from a generator
    seeded with ``seed * 65536 + b`` (K slice, then V slice), so that a test
    can rebuild any single batch entry without drawing the whole cache.
  * planted signal (long-context V1 workload): for each (batch, head), six
    distinct key positions p < N - 2 are drawn and the branch-1 half of
    K[p] is set to 4 * (Q1[N-2] + Q1[N-1]) / 2 in float32 before rounding.
    This mimics the six-needle retrieval setting of the "Differential
    Transformer" glossary page ("Ventajas comunicadas").
  * noise-cancellation query (``snr_inputs``): one query against 1024 keys,
    following step 4 of the lesson "Atencion Diferencial (V2)" (a signal
    token at a known position, noise everywhere else).  See that function.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

BF16 = torch.bfloat16
FP32 = torch.float32


@dataclass(frozen=True)
class Workload:
    """One synthetic workload (sizes, dtype, seed)."""
    name: str
    kind: str                 # "v1", "v2", "v2_decode", "v1_decode"
    dtype: torch.dtype
    seed: int
    B: int
    N: int = 0                # prefill sequence length
    H: int = 0                # V1 heads
    Hq: int = 0               # V2 query heads
    Hkv: int = 0              # V2 KV heads
    d: int = 0                # per-branch QK width (V1) or head dim (V2)
    dv: int = 0               # V1 value width
    L: int = 0                # decode cache length
    causal: bool = True
    layer: int = 1
    eps: float = 1e-5
    planted: int = 0
    fixed_lambda: float | None = None
    extra: dict = field(default_factory=dict)


# The five workloads: a tiny fp32 V1 oracle check, V1 causal prefill,
# V1 long-context causal prefill with planted needles, V2 causal prefill
# with GQA, and single-token decode (V2, plus V1 for comparison).
WORKLOADS = {
    "tiny_v1_fp32": Workload("tiny_v1_fp32", "v1", FP32, 0, B=1, N=128, H=1, d=8,
                             dv=16, causal=False, layer=1, fixed_lambda=0.8),
    "v1_prefill_bf16": Workload("v1_prefill_bf16", "v1", BF16, 1, B=4, N=4096,
                                H=16, d=64, dv=128, causal=True, layer=12),
    "v1_long_bf16": Workload("v1_long_bf16", "v1", BF16, 2, B=1, N=32768, H=16,
                             d=64, dv=128, causal=True, layer=24, planted=6),
    "v2_prefill_bf16": Workload("v2_prefill_bf16", "v2", BF16, 3, B=2, N=8192,
                                Hq=32, Hkv=8, d=128, causal=True),
    "v2_decode_bf16": Workload("v2_decode_bf16", "v2_decode", BF16, 4, B=64,
                               L=32768, Hq=64, Hkv=8, d=128),
    "v1_decode_bf16": Workload("v1_decode_bf16", "v1_decode", BF16, 4, B=64,
                               L=32768, H=32, d=64, dv=128, layer=12),
    # sliding-window variants (hybrid DIFF + sliding-window models): the V2
    # prefill and decode shapes above with a 1024-key / 4096-entry window
    "v2_prefill_window_bf16": Workload("v2_prefill_window_bf16", "v2", BF16, 3, B=2, N=8192,
                                       Hq=32, Hkv=8, d=128, causal=True,
                                       extra={"window": 1024}),
    "v2_decode_window_bf16": Workload("v2_decode_window_bf16", "v2_decode", BF16, 4, B=64,
                                      L=32768, Hq=64, Hkv=8, d=128, extra={"window": 4096}),
    # noise-cancellation sweep: 3 noise amplitudes x 2 branch-noise correlations,
    # lambda 0, 0.1, ..., 1.0 as 11 heads, run through the V1 decode kernel
    "snr_v1_decode": Workload("snr_v1_decode", "snr", BF16, 5, B=48, L=1024, H=11,
                              d=64, dv=128,
                              extra={"sigmas": (1.0, 2.0, 3.0), "rhos": (1.0, 0.9),
                                     "alpha": 6.0, "pos": 517}),
}


def _gen(seed: int) -> torch.Generator:
    return torch.Generator().manual_seed(int(seed))


def _normal(shape, g: torch.Generator, dtype: torch.dtype) -> torch.Tensor:
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    return x.to(dtype) if dtype != torch.float32 else x


def worked_example():
    """The glossary page's example: seed 0, six tokens, branch width 8,
    values 16 wide.  Returns q1, k1, q2, k2 [6, 8] and v [6, 16] (fp32),
    drawn in the page's order from a generator seeded with 0."""
    g = _gen(0)
    q1, k1, q2, k2 = torch.randn(4, 6, 8, generator=g)
    v = torch.randn(6, 16, generator=g)
    return q1, k1, q2, k2, v


def v1_inputs(B: int, N: int, H: int, d: int, dv: int, seed: int,
              dtype: torch.dtype = BF16, planted: int = 0):
    """V1 prefill inputs.  Returns dict with q, k [B, N, H, 2d], v [B, N, H, dv]
    (dtype), lq1, lk1, lq2, lk2 [H, d] (fp32, std 0.1) and, when planted > 0,
    ``planted_pos`` [B, H, planted] (int64)."""
    g = _gen(seed)
    q = torch.randn(B, N, H, 2 * d, generator=g)
    k = torch.randn(B, N, H, 2 * d, generator=g)
    v = torch.randn(B, N, H, dv, generator=g)
    lvec = [0.1 * torch.randn(H, d, generator=g) for _ in range(4)]
    out = {}
    if planted:
        if N < planted + 2:
            raise ValueError("sequence too short for the planted signal")
        pos = torch.empty(B, H, planted, dtype=torch.int64)
        for b in range(B):
            for h in range(H):
                pos[b, h] = torch.randperm(N - 2, generator=g)[:planted]
        for b in range(B):
            for h in range(H):
                needle = 4.0 * (q[b, N - 2, h, :d] + q[b, N - 1, h, :d]) / 2.0
                k[b, pos[b, h], h, :d] = needle
        out["planted_pos"] = pos
    out.update(q=q.to(dtype), k=k.to(dtype), v=v.to(dtype), lq1=lvec[0],
               lk1=lvec[1], lq2=lvec[2], lk2=lvec[3])
    return out


def v2_inputs(B: int, N: int, Hq: int, Hkv: int, d: int, seed: int,
              dtype: torch.dtype = BF16):
    """V2 prefill inputs: q [B, N, Hq, d], k, v [B, N, Hkv, d] (dtype) and
    lam [Hq/2] ~ U(0.2, 0.8) (fp32)."""
    g = _gen(seed)
    q = _normal((B, N, Hq, d), g, dtype)
    k = _normal((B, N, Hkv, d), g, dtype)
    v = _normal((B, N, Hkv, d), g, dtype)
    lam = 0.2 + 0.6 * torch.rand(Hq // 2, generator=g)
    return {"q": q, "k": k, "v": v, "lam": lam}


def decode_cache_slice(seed: int, b: int, L: int, heads: int, k_width: int,
                       v_width: int, dtype: torch.dtype = BF16):
    """Batch entry b of a decode cache: K [L, heads, k_width] and
    V [L, heads, v_width], from a generator seeded with seed*65536 + b."""
    g = _gen(seed * 65536 + b)
    k = _normal((L, heads, k_width), g, dtype)
    v = _normal((L, heads, v_width), g, dtype)
    return k, v


def v2_decode_inputs(B: int, L: int, Hq: int, Hkv: int, d: int, seed: int,
                     dtype: torch.dtype = BF16, fill_caches: bool = True):
    """V2 decode inputs: q [B, Hq, d], lam [Hq/2] and (if fill_caches) the
    caches k_cache, v_cache [B, L, Hkv, d] built slice by slice."""
    g = _gen(seed)
    q = _normal((B, Hq, d), g, dtype)
    lam = 0.2 + 0.6 * torch.rand(Hq // 2, generator=g)
    out = {"q": q, "lam": lam}
    if fill_caches:
        kc = torch.empty(B, L, Hkv, d, dtype=dtype)
        vc = torch.empty(B, L, Hkv, d, dtype=dtype)
        for b in range(B):
            kc[b], vc[b] = decode_cache_slice(seed, b, L, Hkv, d, d, dtype)
        out.update(k_cache=kc, v_cache=vc)
    return out


def v1_decode_inputs(B: int, L: int, H: int, d: int, dv: int, seed: int,
                     dtype: torch.dtype = BF16, fill_caches: bool = True):
    """V1 decode inputs: q [B, H, 2d], four lambda vectors [H, d] (std 0.1)
    and (if fill_caches) k_cache [B, L, H, 2d], v_cache [B, L, H, dv]."""
    g = _gen(seed)
    q = _normal((B, H, 2 * d), g, dtype)
    lvec = [0.1 * torch.randn(H, d, generator=g) for _ in range(4)]
    out = {"q": q, "lq1": lvec[0], "lk1": lvec[1], "lq2": lvec[2], "lk2": lvec[3]}
    if fill_caches:
        kc = torch.empty(B, L, H, 2 * d, dtype=dtype)
        vc = torch.empty(B, L, H, dv, dtype=dtype)
        for b in range(B):
            kc[b], vc[b] = decode_cache_slice(seed, b, L, H, 2 * d, dv, dtype)
        out.update(k_cache=kc, v_cache=vc)
    return out


def fill_normal_on_device(t: torch.Tensor, seed: int) -> torch.Tensor:
    """Fill a device tensor with N(0, 1) values (rounded to its dtype) from a
    seeded device generator.  Used for the bulk of very large decode caches
    whose contents no oracle row reads; batch entries an oracle does read are
    overwritten with ``decode_cache_slice`` values."""
    g = torch.Generator(device=t.device).manual_seed(int(seed))
    flat = t.view(-1)
    step = 1 << 28
    for lo in range(0, flat.numel(), step):
        hi = min(flat.numel(), lo + step)
        flat[lo:hi] = torch.randn(hi - lo, generator=g, device=t.device,
                                  dtype=torch.float32).to(t.dtype)
    return t


def snr_inputs(seed: int = 5, L: int = 1024, d: int = 64, dv: int = 128,
               sigmas=(1.0, 2.0, 3.0), rhos=(1.0, 0.9), alpha: float = 6.0,
               pos: int = 517, lam_grid=None):
    """Signal-plus-noise query for the noise-cancellation sweep.

    Step 4 of the lesson "Atencion Diferencial (V2)" (section "Paso 4:
    medicion de la cancelacion de ruido") puts a signal token at a known
    position of a length-1024 sequence and fills the rest with noise;
    exercise 4 sweeps lambda from 0 to 1 and exercise 1 varies the noise
    amplitude.  Reading used here (the pages fix no construction):

      * one configuration per (noise amplitude sigma, branch correlation rho);
        u is a seeded random unit vector in R^d and both branches query with
        q1 = q2 = sqrt(d) u, so a key k scores u . k in either branch;
      * noise keys: branch 1 draws n ~ N(0, sigma^2 I); branch 2 uses
        rho n + sqrt(1 - rho^2) n' (n' independent), i.e. the noise both maps
        see is shared to the degree rho;
      * the signal key at ``pos``: branch 1 holds alpha u (score alpha),
        branch 2 an ordinary noise draw (the branches differ on the signal);
      * lambda is swept over ``lam_grid`` (default 0, 0.1, ..., 1.0), one
        value per head, all heads holding the same query and keys.

    To read the per-key differential weights w_j through the decode kernel,
    each configuration is repeated over L / dv batch entries that differ only
    in V: entry g of a configuration has V[j, c] = 1 when j = g * dv + c and
    0 otherwise, so its output row is w restricted to keys [g dv, (g+1) dv).

    Returns q [B, H, 2d], k_cache [B, L, H, 2d], v_cache [B, L, H, dv]
    (bf16), lam [H] (float32), and per configuration the (bf16-rounded)
    query ``q_cfg`` [C, 2d] and keys ``k_cfg`` [C, L, 2d] as float32, with
    ``configs`` [(sigma, rho)], ``groups`` = L / dv and ``pos``.
    """
    if L % dv:
        raise ValueError("L must be a multiple of dv")
    if lam_grid is None:
        lam_grid = [i / 10.0 for i in range(11)]
    H = len(lam_grid)
    configs = [(float(s_), float(r_)) for s_ in sigmas for r_ in rhos]
    C, G = len(configs), L // dv
    g = _gen(seed)
    q_cfg = torch.empty(C, 2 * d)
    k_cfg = torch.empty(C, L, 2 * d)
    for c, (sigma, rho) in enumerate(configs):
        u = torch.randn(d, generator=g)
        u = u / u.norm()
        n1 = sigma * torch.randn(L, d, generator=g)
        n2 = sigma * torch.randn(L, d, generator=g)
        q_cfg[c, :d] = (d ** 0.5) * u
        q_cfg[c, d:] = (d ** 0.5) * u
        k_cfg[c, :, :d] = n1
        k_cfg[c, :, d:] = rho * n1 + (1.0 - rho * rho) ** 0.5 * n2
        k_cfg[c, pos, :d] = alpha * u
    q_cfg = q_cfg.to(BF16).float()
    k_cfg = k_cfg.to(BF16).float()
    B = C * G
    q = q_cfg.repeat_interleave(G, dim=0)[:, None, :].expand(B, H, 2 * d)
    k = k_cfg.repeat_interleave(G, dim=0)[:, :, None, :].expand(B, L, H, 2 * d)
    onehot = torch.zeros(G, L, dv)
    for gi in range(G):
        onehot[gi, gi * dv:(gi + 1) * dv, :] = torch.eye(dv)
    v = onehot.repeat(C, 1, 1)[:, :, None, :].expand(B, L, H, dv)
    return {"q": q.to(BF16).contiguous(), "k_cache": k.to(BF16).contiguous(),
            "v_cache": v.to(BF16).contiguous(),
            "lam": torch.tensor(lam_grid, dtype=FP32), "q_cfg": q_cfg, "k_cfg": k_cfg,
            "configs": configs, "groups": G, "pos": pos}
