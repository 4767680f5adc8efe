"""GPU parity of the V2 prefill followed by the output projection (lesson
"Atencion Diferencial (V2)", "V1 vs V2: la diferencia" and step 5): the
oracle's V2 rows (fp64) times O_W in float64, against the GPU's bf16 result,
on |gpu - ref| / max|ref|."""
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
    o = O.v2_rows(x["q"], x["k"], x["v"], x["lam"], np.arange(Bn * N * Hq // 2), causal=True,
                  window=window).reshape(Bn * N, Hq // 2 * d)
    ref = o @ W.double().numpy()
    assert_bf16_close(out.reshape(-1, dm), ref, True, "oproj N=%d W=%d" % (N, window))


def test_oproj_full_size_sampled_rows(B):
    w = I.WORKLOADS["v2_prefill_bf16"]
    dm = 2048
    x = I.v2_inputs(w.B, w.N, w.Hq, w.Hkv, w.d, w.seed)
    W = w_o(w.Hq // 2 * w.d, dm, 1602)
    out = B.diffattn_v2_prefill_oproj(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(),
                                      x["lam"].cuda(), W.cuda())
    P = w.Hq // 2
    tokens = [(0, 0), (0, 4095), (1, 8191), (1, 5000)]
    rows = np.concatenate([np.arange((b * w.N + i) * P, (b * w.N + i + 1) * P) for b, i in tokens])
    o = O.v2_rows(x["q"], x["k"], x["v"], x["lam"], rows, causal=True).reshape(len(tokens), -1)
    ref = o @ W.double().numpy()
    got = torch.stack([out[b, i] for b, i in tokens])
    assert_bf16_close(got, ref, True, "oproj full size")
