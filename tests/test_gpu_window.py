"""GPU parity of the sliding-window variants against the fp64 oracle.

Lesson "Atencion Diferencial (V2)", section "Uselo" (hybrids of differential
and sliding-window attention); reading: query i sees keys (i - W, i] in both
branches, a decode query the last W cache entries.  Covers the tensor-core
prefill (both forms, windows that start inside, at and across 64-key tiles,
W = 1, W >= N), the split-KV decode kernels, the CUDA-core kernel, and decode
== last row of windowed prefill."""
import numpy as np
import pytest
import torch

import oracle as O
from differential_attention_sm_b200 import inputs as I
from parity import assert_bf16_close, assert_fp32_close, assert_status_ok, status_word

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from differential_attention_sm_b200 import binding
    binding.load()
    return binding


def cuda(t):
    return t.cuda().contiguous()


@pytest.mark.parametrize("N,W", [(700, 1), (700, 64), (700, 100), (700, 300), (333, 5000)])
def test_v1_prefill_window(B, N, W):
    Bn, H, d, dv, layer = 1, 3, 64, 128, 12
    x = I.v1_inputs(Bn, N, H, d, dv, seed=500 + W)
    lam_dev = B.lambda_from_params(*(cuda(x[n]) for n in ("lq1", "lk1", "lq2", "lk2")), layer)
    lam = O.lambda_from_params(x["lq1"], x["lk1"], x["lq2"], x["lk2"], layer)
    li = O.lambda_init(layer)
    st = status_word()
    out = B.diffattn_v1_fwd_window(cuda(x["q"]), cuda(x["k"]), cuda(x["v"]), lam_dev, W,
                                   apply_norm=True, lambda_init=li, dev_status=st)
    assert_status_ok(st)
    ref = O.v1_rows(x["q"], x["k"], x["v"], lam, np.arange(Bn * N * H), causal=True,
                    apply_norm=True, lambda_init_value=li, window=W)
    assert_bf16_close(out.reshape(-1, dv), ref, False, "v1 window N=%d W=%d" % (N, W))


@pytest.mark.parametrize("N,W", [(1100, 1), (1100, 127), (1100, 256), (1100, 1000), (200, 64)])
def test_v2_prefill_window(B, N, W):
    Bn, Hq, Hkv, d = 1, 8, 2, 128
    x = I.v2_inputs(Bn, N, Hq, Hkv, d, seed=600 + W)
    st = status_word()
    out = B.diffattn_v2_prefill_window(cuda(x["q"]), cuda(x["k"]), cuda(x["v"]),
                                       cuda(x["lam"]), W, dev_status=st)
    assert_status_ok(st)
    ref = O.v2_rows(x["q"], x["k"], x["v"], x["lam"], np.arange(Bn * N * Hq // 2),
                    causal=True, window=W)
    assert_bf16_close(out.reshape(-1, d), ref, True, "v2 window N=%d W=%d" % (N, W))


def test_window_generic_paths(B):
    # fp32 and widths outside the tensor-core kernels run on the CUDA-core kernel
    Bn, N, H, d, dv, W = 2, 90, 2, 8, 16, 17
    x = I.v1_inputs(Bn, N, H, d, dv, seed=700, dtype=torch.float32)
    lam = torch.tensor([0.8, -0.3])
    out = B.diffattn_v1_fwd_window(cuda(x["q"]), cuda(x["k"]), cuda(x["v"]), cuda(lam), W)
    ref = O.v1_rows(x["q"], x["k"], x["v"], lam.double().numpy(), np.arange(Bn * N * H),
                    causal=True, window=W)
    assert_fp32_close(out.reshape(-1, dv), ref, "v1 fp32 window")
    xd = I.v2_decode_inputs(2, 300, 4, 2, 32, seed=701, dtype=torch.float32)
    lens = [300, 40]
    out = B.diffattn_v2_decode_window(cuda(xd["q"]), cuda(xd["k_cache"]), cuda(xd["v_cache"]),
                                      cuda(xd["lam"]), 50,
                                      cache_lens=cuda(torch.tensor(lens, dtype=torch.int32)))
    ref = O.v2_decode_rows(xd["q"], xd["k_cache"], xd["v_cache"], xd["lam"], np.arange(4),
                           lens=lens, window=50)
    assert_fp32_close(out.reshape(-1, 32), ref, "v2 decode fp32 window")


@pytest.mark.parametrize("W", [1, 64, 700, 5000])
def test_v2_decode_window(B, W):
    Bn, L, Hq, Hkv, d = 3, 3000, 16, 2, 128
    x = I.v2_decode_inputs(Bn, L, Hq, Hkv, d, seed=800 + W)
    lens = [3000, 1, 1500]
    st = status_word()
    out = B.diffattn_v2_decode_window(cuda(x["q"]), cuda(x["k_cache"]), cuda(x["v_cache"]),
                                      cuda(x["lam"]), W,
                                      cache_lens=cuda(torch.tensor(lens, dtype=torch.int32)),
                                      dev_status=st)
    assert_status_ok(st)
    ref = O.v2_decode_rows(x["q"], x["k_cache"], x["v_cache"], x["lam"],
                           np.arange(Bn * Hq // 2), lens=lens, window=W)
    assert_bf16_close(out.reshape(-1, d), ref, True, "v2 decode window W=%d" % W)


@pytest.mark.parametrize("W", [1, 33, 900])
def test_v1_decode_window(B, W):
    Bn, L, H, d, dv, layer = 2, 1000, 3, 64, 128, 12
    x = I.v1_decode_inputs(Bn, L, H, d, dv, seed=900 + W)
    lam_dev = B.lambda_from_params(*(cuda(x[n]) for n in ("lq1", "lk1", "lq2", "lk2")), layer)
    lam = O.lambda_from_params(x["lq1"], x["lk1"], x["lq2"], x["lk2"], layer)
    li = O.lambda_init(layer)
    lens = [1000, 450]
    out = B.diffattn_v1_decode_window(cuda(x["q"]), cuda(x["k_cache"]), cuda(x["v_cache"]),
                                      lam_dev, W,
                                      cache_lens=cuda(torch.tensor(lens, dtype=torch.int32)),
                                      apply_norm=True, lambda_init=li)
    ref = O.v1_decode_rows(x["q"], x["k_cache"], x["v_cache"], lam, np.arange(Bn * H),
                           lens=lens, apply_norm=True, lambda_init_value=li, window=W)
    assert_bf16_close(out.reshape(-1, dv), ref, False, "v1 decode window W=%d" % W)


def test_window_decode_equals_last_row_of_window_prefill(B):
    n, Hq, Hkv, d, W = 777, 8, 2, 128, 200
    x = I.v2_inputs(1, n, Hq, Hkv, d, seed=1001)
    pre = B.diffattn_v2_prefill_window(cuda(x["q"]), cuda(x["k"]), cuda(x["v"]),
                                       cuda(x["lam"]), W)
    dec = B.diffattn_v2_decode_window(cuda(x["q"][:, n - 1]), cuda(x["k"]), cuda(x["v"]),
                                      cuda(x["lam"]), W)
    ref = O.v2_rows(x["q"], x["k"], x["v"], x["lam"],
                    np.arange((n - 1) * Hq // 2, n * Hq // 2), causal=True, window=W)
    assert_bf16_close(pre[0, n - 1], ref, True, "window prefill last row")
    assert_bf16_close(dec[0], ref, True, "window decode")
