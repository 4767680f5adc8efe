"""GPU parity of the V2 prefill followed by the output projection (lesson
"Atencion Diferencial (V2)", "V1 vs V2: la diferencia" and step 5): the
oracle's projected rows (``v2_oproj_rows``, fp64) against the GPU's bf16
result, on |gpu - ref| / max|ref|."""
import numpy as np
import pytest
import torch

import oracle as O
from differential_attention_sm_b200 import inputs as I
from parity import assert_bf16_close, assert_status_ok, status_word

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from differential_attention_sm_b200 import binding
    binding.load()
    return binding


def w_o(rows, cols, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(rows, cols, generator=g) / rows ** 0.5).to(torch.bfloat16)


@pytest.mark.parametrize("N,window", [(300, 0), (257, 64)])
def test_oproj_small(B, N, window):
    Bn, Hq, Hkv, d, dm = 2, 8, 2, 128, 192
    x = I.v2_inputs(Bn, N, Hq, Hkv, d, seed=1600 + N)
    W = w_o(Hq // 2 * d, dm, 1601)
    st = status_word()
    out = B.diffattn_v2_prefill_oproj(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(),
                                      x["lam"].cuda(), W.cuda(), window=window, dev_status=st)
    assert_status_ok(st)
    ref = O.v2_oproj_rows(x["q"], x["k"], x["v"], x["lam"], W, np.arange(Bn * N), causal=True,
                          window=window)
    assert_bf16_close(out.reshape(-1, dm), ref, True, "oproj N=%d W=%d" % (N, window))


def test_oproj_full_size(B):
    """V2 prefill workload (B2 Hq32 N8192) projected to d_model 2048:
    one token from every 128-row tile of the projection, all 2048 columns,
    against the oracle; and the whole output against an fp32 product of the
    GPU's own attention output (pinned by the prefill parity tests)."""
    w = I.WORKLOADS["v2_prefill_bf16"]
    dm = 2048
    x = I.v2_inputs(w.B, w.N, w.Hq, w.Hkv, w.d, w.seed)
    W = w_o(w.Hq // 2 * w.d, dm, 1602)
    q, k, v, lam, Wd = (t.cuda() for t in (x["q"], x["k"], x["v"], x["lam"], W))
    st = status_word()
    out = B.diffattn_v2_prefill_oproj(q, k, v, lam, Wd, dev_status=st)
    assert_status_ok(st)
    P = w.Hq // 2
    rng = np.random.default_rng(1603)
    toks = [int(t * 128 + rng.integers(0, 128)) for t in range(w.B * w.N // 128)]
    ref = O.v2_oproj_rows(x["q"], x["k"], x["v"], x["lam"], W, toks, causal=True)
    got = out.reshape(-1, dm)[torch.tensor(toks, device="cuda")]
    assert_bf16_close(got, ref, True, "oproj full size, one token per row tile")
    att = B.diffattn_v2_prefill(q, k, v, lam, causal=True).reshape(w.B * w.N, P * w.d)
    full = (att.float() @ Wd.float()).double().cpu().numpy()
    assert_bf16_close(out.reshape(-1, dm), full, True, "oproj full size, every output")


def test_oproj_ragged_tiles(B):
    """Tails in every dimension of the projection GEMM: 260 rows (M), a
    head width of 72 so that Hq/2 * d = 288 is not a multiple of the 64-wide
    K step (the attention part runs on the CUDA-core kernel), and
    d_model = 136, less than one 256-column tile."""
    Bn, N, Hq, Hkv, d, dm = 2, 130, 8, 2, 72, 136
    x = I.v2_inputs(Bn, N, Hq, Hkv, d, seed=1700)
    W = w_o(Hq // 2 * d, dm, 1701)
    st = status_word()
    out = B.diffattn_v2_prefill_oproj(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(),
                                      x["lam"].cuda(), W.cuda(), dev_status=st)
    assert_status_ok(st)
    ref = O.v2_oproj_rows(x["q"], x["k"], x["v"], x["lam"], W, np.arange(Bn * N), causal=True)
    assert_bf16_close(out.reshape(-1, dm), ref, True, "oproj ragged tiles")
