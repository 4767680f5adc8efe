"""GPU parity of the prefill path (C ABI via the binding) against the fp64
oracle: the tiny fp32 workload, small ragged bf16 cases on the tensor-core
kernel and the generic kernel, and harder numerics (lambda outside [0, 1],
large logits).  The full-size workloads are in test_gpu_full_size.py."""
import numpy as np
import pytest
import torch

import oracle as O
from differential_attention_sm_b200 import inputs as I
from parity import (assert_bf16_close, assert_fp32_close, assert_status_ok, status_word)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from differential_attention_sm_b200 import binding
    binding.load()
    return binding


def cuda(t):
    return t.cuda().contiguous()


# ---------------------------------------------------------------------------
# tiny fp32 workload: B1 H1 N128 d8 dv16, lambda 0.8 or from params (layer 1)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("lam_mode", ["fixed", "params"])
def test_tiny_v1_fp32(B, causal, lam_mode):
    w = I.WORKLOADS["tiny_v1_fp32"]
    x = I.v1_inputs(w.B, w.N, w.H, w.d, w.dv, w.seed, dtype=torch.float32)
    if lam_mode == "fixed":
        lam_host = np.array([w.fixed_lambda])
        lam_dev = torch.tensor([w.fixed_lambda], dtype=torch.float32, device="cuda")
    else:
        lam_host = O.lambda_from_params(x["lq1"], x["lk1"], x["lq2"], x["lk2"], w.layer)
        lam_dev = B.lambda_from_params(*(cuda(x[n]) for n in ("lq1", "lk1", "lq2", "lk2")),
                                       w.layer)
    st = status_word()
    out = B.diffattn_v1_fwd(cuda(x["q"]), cuda(x["k"]), cuda(x["v"]), lam_dev, causal=causal,
                            dev_status=st)
    assert_status_ok(st)
    ref = O.v1_rows(x["q"], x["k"], x["v"], lam_host, np.arange(w.B * w.N * w.H), causal=causal)
    assert_fp32_close(out.reshape(-1, w.dv), ref, "tiny fp32")


def test_worked_example_on_gpu(B):
    q1, k1, q2, k2, v = I.worked_example()
    q = torch.cat([q1, q2], -1).reshape(1, 6, 1, 16)
    k = torch.cat([k1, k2], -1).reshape(1, 6, 1, 16)
    vv = v.reshape(1, 6, 1, 16)
    lam = torch.tensor([0.8], device="cuda")
    out = B.diffattn_v1_fwd(cuda(q), cuda(k), cuda(vv), lam, causal=False)
    ref = O.v1_rows(q, k, vv, [0.8], np.arange(6), causal=False)
    assert_fp32_close(out.reshape(6, 16), ref, "worked example")


def test_lambda_from_params_matches_oracle(B):
    g = torch.Generator().manual_seed(5)
    vecs = [0.3 * torch.randn(16, 64, generator=g) for _ in range(4)]
    for layer in (1, 12, 24):
        got = B.lambda_from_params(*(cuda(t) for t in vecs), layer).cpu().double().numpy()
        ref = O.lambda_from_params(*vecs, layer)
        assert np.abs(got - ref).max() <= 1e-6 * max(1.0, np.abs(ref).max())


# ---------------------------------------------------------------------------
# V1 bf16, small and ragged (tcgen05 kernel: d_qk 64, d_v 128)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("Bn,N,H,causal", [
    (2, 300, 3, True),    # two full tiles + a ragged tail
    (1, 128, 2, True),    # exactly one tile
    (1, 1, 2, True),      # single token
    (2, 129, 1, True),    # one row past a tile edge
    (1, 200, 2, False),   # non-causal, ragged key tail
    (1, 640, 1, True),    # ten key tiles: every K/V ring stage is reused
])
def test_v1_bf16_small(B, Bn, N, H, causal):
    d, dv, layer = 64, 128, 12
    x = I.v1_inputs(Bn, N, H, d, dv, seed=100 + N, dtype=torch.bfloat16)
    lam_dev = B.lambda_from_params(*(cuda(x[n]) for n in ("lq1", "lk1", "lq2", "lk2")), layer)
    lam_host = O.lambda_from_params(x["lq1"], x["lk1"], x["lq2"], x["lk2"], layer)
    li = O.lambda_init(layer)
    st = status_word()
    out = B.diffattn_v1_fwd(cuda(x["q"]), cuda(x["k"]), cuda(x["v"]), lam_dev, causal=causal,
                            apply_norm=True, norm_eps=1e-5, lambda_init=li, dev_status=st)
    assert_status_ok(st)
    ref = O.v1_rows(x["q"], x["k"], x["v"], lam_host, np.arange(Bn * N * H), causal=causal,
                    apply_norm=True, eps=1e-5, lambda_init_value=li)
    assert_bf16_close(out.reshape(-1, dv), ref, False, "v1 bf16 N=%d" % N)


@pytest.mark.parametrize("offset_bytes", [16, 32])
def test_v1_bf16_output_offset(B, offset_bytes):
    """The output may start at any 16-byte boundary: the V1 kernel writes it by
    TMA tensor stores, whose map takes the caller's base as given.  Rows past
    the ragged end must not be written, nor anything around the output."""
    Bn, N, H, d, dv = 2, 300, 3, 64, 128
    x = I.v1_inputs(Bn, N, H, d, dv, seed=31, dtype=torch.bfloat16)
    lam = torch.tensor([0.4, -0.6, 1.3], dtype=torch.float32)
    n = Bn * N * H * dv
    pad = offset_bytes // 2
    buf = torch.full((n + 2 * pad + 64,), -7.0, dtype=torch.bfloat16, device="cuda")
    out = buf[pad:pad + n].view(Bn, N, H, dv)
    assert out.data_ptr() % 16 == 0
    st = status_word()
    B.diffattn_v1_fwd(cuda(x["q"]), cuda(x["k"]), cuda(x["v"]), cuda(lam), causal=True,
                      apply_norm=True, lambda_init=0.3, out=out, dev_status=st)
    assert_status_ok(st)
    torch.cuda.synchronize()
    assert (buf[:pad] == -7.0).all() and (buf[pad + n:] == -7.0).all(), "write outside the output"
    ref = O.v1_rows(x["q"], x["k"], x["v"], lam.double().numpy(), np.arange(Bn * N * H),
                    causal=True, apply_norm=True, lambda_init_value=0.3)
    assert_bf16_close(out.reshape(-1, dv), ref, False, "v1 bf16 output at +%d bytes" % offset_bytes)


def test_v1_bf16_no_norm_and_gain(B):
    Bn, N, H, d, dv = 1, 257, 2, 64, 128
    x = I.v1_inputs(Bn, N, H, d, dv, seed=7, dtype=torch.bfloat16)
    lam = torch.tensor([0.8, -0.3], dtype=torch.float32)
    out = B.diffattn_v1_fwd(cuda(x["q"]), cuda(x["k"]), cuda(x["v"]), cuda(lam), causal=True)
    ref = O.v1_rows(x["q"], x["k"], x["v"], lam.double().numpy(), np.arange(Bn * N * H),
                    causal=True)
    assert_bf16_close(out.reshape(-1, dv), ref, True, "v1 bf16 no norm")
    g = 0.5 + torch.rand(dv, generator=torch.Generator().manual_seed(3))
    li = O.lambda_init(3)
    out = B.diffattn_v1_fwd(cuda(x["q"]), cuda(x["k"]), cuda(x["v"]), cuda(lam), causal=True,
                            apply_norm=True, norm_weight=cuda(g), lambda_init=li)
    ref = O.v1_rows(x["q"], x["k"], x["v"], lam.double().numpy(), np.arange(Bn * N * H),
                    causal=True, apply_norm=True, norm_weight=g, lambda_init_value=li)
    assert_bf16_close(out.reshape(-1, dv), ref, False, "v1 bf16 gain")


def test_v1_bf16_generic_widths(B):
    """Widths outside the tensor-core kernel run on the CUDA-core kernel."""
    Bn, N, H, d, dv = 1, 150, 2, 32, 64
    x = I.v1_inputs(Bn, N, H, d, dv, seed=8, dtype=torch.bfloat16)
    lam = torch.tensor([0.6, 0.9], dtype=torch.float32)
    out = B.diffattn_v1_fwd(cuda(x["q"]), cuda(x["k"]), cuda(x["v"]), cuda(lam), causal=True,
                            apply_norm=True, lambda_init=0.2)
    ref = O.v1_rows(x["q"], x["k"], x["v"], lam.double().numpy(), np.arange(Bn * N * H),
                    causal=True, apply_norm=True, lambda_init_value=0.2)
    assert_bf16_close(out.reshape(-1, dv), ref, False, "v1 generic")


# ---------------------------------------------------------------------------
# V2 bf16, small and ragged (tcgen05 kernel: head_dim 128)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("Bn,N,Hq,Hkv,causal", [
    (2, 333, 8, 2, True),
    (1, 256, 4, 2, True),    # group of 2: one pair per KV head
    (1, 1, 4, 1, True),
    (1, 190, 8, 1, False),
])
def test_v2_bf16_small(B, Bn, N, Hq, Hkv, causal):
    d = 128
    x = I.v2_inputs(Bn, N, Hq, Hkv, d, seed=200 + N)
    st = status_word()
    out = B.diffattn_v2_prefill(cuda(x["q"]), cuda(x["k"]), cuda(x["v"]), cuda(x["lam"]),
                                causal=causal, dev_status=st)
    assert_status_ok(st)
    ref = O.v2_rows(x["q"], x["k"], x["v"], x["lam"], np.arange(Bn * N * Hq // 2),
                    causal=causal)
    assert_bf16_close(out.reshape(-1, d), ref, True, "v2 bf16 N=%d" % N)


def test_v2_fp32_generic(B):
    Bn, N, Hq, Hkv, d = 1, 70, 4, 2, 16
    x = I.v2_inputs(Bn, N, Hq, Hkv, d, seed=9, dtype=torch.float32)
    out = B.diffattn_v2_prefill(cuda(x["q"]), cuda(x["k"]), cuda(x["v"]), cuda(x["lam"]),
                                causal=True)
    ref = O.v2_rows(x["q"], x["k"], x["v"], x["lam"], np.arange(Bn * N * Hq // 2), causal=True)
    assert_fp32_close(out.reshape(-1, d), ref, "v2 fp32")


# ---------------------------------------------------------------------------
# harder numerics: lambda outside [0, 1], large logits (many lazy rescales)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("lam_values", [(-0.6, 1.4, 0.0), (2.5, -1.2, 0.9)])
def test_v1_bf16_extreme_lambda(B, lam_values):
    Bn, N, H, d, dv = 1, 384, 3, 64, 128
    x = I.v1_inputs(Bn, N, H, d, dv, seed=31, dtype=torch.bfloat16)
    lam = torch.tensor(lam_values, dtype=torch.float32)
    out = B.diffattn_v1_fwd(cuda(x["q"]), cuda(x["k"]), cuda(x["v"]), cuda(lam), causal=True,
                            apply_norm=True, lambda_init=0.3)
    ref = O.v1_rows(x["q"], x["k"], x["v"], lam.double().numpy(), np.arange(Bn * N * H),
                    causal=True, apply_norm=True, lambda_init_value=0.3)
    assert_bf16_close(out.reshape(-1, dv), ref, False, "v1 extreme lambda")


def test_v2_bf16_extreme_lambda(B):
    Bn, N, Hq, Hkv, d = 1, 300, 4, 1, 128
    x = I.v2_inputs(Bn, N, Hq, Hkv, d, seed=32)
    lam = torch.tensor([-0.75, 1.6], dtype=torch.float32)
    out = B.diffattn_v2_prefill(cuda(x["q"]), cuda(x["k"]), cuda(x["v"]), cuda(lam), causal=True)
    ref = O.v2_rows(x["q"], x["k"], x["v"], lam.double().numpy(), np.arange(Bn * N * 2),
                    causal=True)
    assert_bf16_close(out.reshape(-1, d), ref, True, "v2 extreme lambda")


@pytest.mark.parametrize("scale", [3.0, 6.0])
def test_large_logits_rescale_paths(B, scale):
    """Queries scaled up so that row maxima jump by far more than the lazy
    rescale threshold across key tiles (and exponents span a wide range)."""
    Bn, N, H, d, dv = 1, 700, 2, 64, 128
    x = I.v1_inputs(Bn, N, H, d, dv, seed=33, dtype=torch.float32)
    ramp = torch.linspace(0.2, 1.0, N).view(1, N, 1, 1)   # later keys grow: maxima keep rising
    q = (scale * x["q"]).to(torch.bfloat16)
    k = (x["k"] * ramp).to(torch.bfloat16)
    v = x["v"].to(torch.bfloat16)
    lam = torch.tensor([0.7, 0.4], dtype=torch.float32)
    out = B.diffattn_v1_fwd(cuda(q), cuda(k), cuda(v), cuda(lam), causal=True, apply_norm=True,
                            lambda_init=0.2)
    ref = O.v1_rows(q, k, v, lam.double().numpy(), np.arange(Bn * N * H), causal=True,
                    apply_norm=True, lambda_init_value=0.2)
    assert_bf16_close(out.reshape(-1, dv), ref, False, "v1 large logits x%g" % scale)
    x2 = I.v2_inputs(1, N, 4, 2, 128, seed=34, dtype=torch.float32)
    q2 = (scale * x2["q"]).to(torch.bfloat16)
    k2 = (x2["k"] * ramp).to(torch.bfloat16)
    v2 = x2["v"].to(torch.bfloat16)
    out2 = B.diffattn_v2_prefill(cuda(q2), cuda(k2), cuda(v2), cuda(x2["lam"]), causal=True)
    ref2 = O.v2_rows(q2, k2, v2, x2["lam"], np.arange(N * 2), causal=True)
    assert_bf16_close(out2.reshape(-1, 128), ref2, True, "v2 large logits x%g" % scale)
