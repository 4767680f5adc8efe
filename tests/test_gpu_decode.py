"""GPU parity of single-token decode (V2 split-KV tensor-core kernel, V1
split-KV CUDA-core kernel, and the generic kernel) against the fp64 oracle,
including ragged cache lengths, several GQA group sizes and decode == last
row of prefill.  The full-size workloads are in test_gpu_full_size.py."""
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


@pytest.mark.parametrize("Bn,L,Hq,Hkv,lens", [
    (3, 1000, 16, 2, [1000, 1, 517]),     # group 8 (4 pairs per KV head), ragged lengths
    (2, 777, 8, 2, None),                 # group 4, length not a chunk multiple
    (2, 300, 4, 2, [64, 300]),            # group 2
    (1, 2048, 12, 2, [2047]),             # group 6 (padded heads)
    (4, 64, 16, 2, [64, 63, 1, 2]),       # one chunk
])
def test_v2_decode_small(B, Bn, L, Hq, Hkv, lens):
    d = 128
    x = I.v2_decode_inputs(Bn, L, Hq, Hkv, d, seed=300 + L)
    ln = torch.tensor(lens, dtype=torch.int32) if lens is not None else None
    st = status_word()
    out = B.diffattn_v2_decode(cuda(x["q"]), cuda(x["k_cache"]), cuda(x["v_cache"]),
                               cuda(x["lam"]), cache_lens=None if ln is None else cuda(ln),
                               dev_status=st)
    assert_status_ok(st)
    ref = O.v2_decode_rows(x["q"], x["k_cache"], x["v_cache"], x["lam"],
                           np.arange(Bn * Hq // 2), lens=lens)
    assert_bf16_close(out.reshape(-1, d), ref, True, "v2 decode L=%d" % L)


def test_v2_decode_generic_paths(B):
    # fp32 and a head width outside the fast kernel use the CUDA-core kernel
    Bn, L, Hq, Hkv, d = 2, 90, 8, 2, 32
    x = I.v2_decode_inputs(Bn, L, Hq, Hkv, d, seed=11, dtype=torch.float32)
    lens = [90, 33]
    out = B.diffattn_v2_decode(cuda(x["q"]), cuda(x["k_cache"]), cuda(x["v_cache"]),
                               cuda(x["lam"]), cache_lens=cuda(torch.tensor(lens, dtype=torch.int32)))
    ref = O.v2_decode_rows(x["q"], x["k_cache"], x["v_cache"], x["lam"],
                           np.arange(Bn * Hq // 2), lens=lens)
    assert_fp32_close(out.reshape(-1, d), ref, "v2 decode fp32")
    x = I.v2_decode_inputs(Bn, L, 16, 1, 64, seed=12)   # group 16 > 8: generic bf16
    out = B.diffattn_v2_decode(cuda(x["q"]), cuda(x["k_cache"]), cuda(x["v_cache"]),
                               cuda(x["lam"]))
    ref = O.v2_decode_rows(x["q"], x["k_cache"], x["v_cache"], x["lam"], np.arange(Bn * 8))
    assert_bf16_close(out.reshape(-1, 64), ref, True, "v2 decode generic bf16")


@pytest.mark.parametrize("Bn,L,H,lens", [
    (2, 1000, 3, [1000, 1]),
    (3, 555, 2, None),
    (1, 64, 4, [17]),
])
def test_v1_decode_small(B, Bn, L, H, lens):
    d, dv, layer = 64, 128, 12
    x = I.v1_decode_inputs(Bn, L, H, d, dv, seed=400 + L)
    lam_dev = B.lambda_from_params(*(cuda(x[n]) for n in ("lq1", "lk1", "lq2", "lk2")), layer)
    lam_host = O.lambda_from_params(x["lq1"], x["lk1"], x["lq2"], x["lk2"], layer)
    li = O.lambda_init(layer)
    ln = None if lens is None else cuda(torch.tensor(lens, dtype=torch.int32))
    out = B.diffattn_v1_decode(cuda(x["q"]), cuda(x["k_cache"]), cuda(x["v_cache"]), lam_dev,
                               cache_lens=ln, apply_norm=True, norm_eps=1e-5, lambda_init=li)
    ref = O.v1_decode_rows(x["q"], x["k_cache"], x["v_cache"], lam_host, np.arange(Bn * H),
                           lens=lens, apply_norm=True, eps=1e-5, lambda_init_value=li)
    assert_bf16_close(out.reshape(-1, dv), ref, False, "v1 decode L=%d" % L)
    # without the norm: relative to the largest output
    out = B.diffattn_v1_decode(cuda(x["q"]), cuda(x["k_cache"]), cuda(x["v_cache"]), lam_dev,
                               cache_lens=ln)
    ref = O.v1_decode_rows(x["q"], x["k_cache"], x["v_cache"], lam_host, np.arange(Bn * H),
                           lens=lens)
    assert_bf16_close(out.reshape(-1, dv), ref, True, "v1 decode no norm")


def test_decode_equals_last_prefill_row(B):
    """Decode over a cache of length n gives the last row of causal prefill
    over the same n tokens (GPU against GPU, and both against the oracle)."""
    n, Hq, Hkv, d = 520, 8, 2, 128
    x = I.v2_inputs(1, n, Hq, Hkv, d, seed=13)
    pre = B.diffattn_v2_prefill(cuda(x["q"]), cuda(x["k"]), cuda(x["v"]), cuda(x["lam"]),
                                causal=True)
    dec = B.diffattn_v2_decode(cuda(x["q"][:, n - 1]), cuda(x["k"]), cuda(x["v"]),
                               cuda(x["lam"]))
    ref = O.v2_rows(x["q"], x["k"], x["v"], x["lam"], np.arange((n - 1) * Hq // 2, n * Hq // 2),
                    causal=True)
    assert_bf16_close(pre[0, n - 1], ref, True, "prefill last row")
    assert_bf16_close(dec[0], ref, True, "decode")
    assert_bf16_close(dec[0], pre[0, n - 1].float().cpu().double().numpy(), True, "dec vs pre")


def test_v2_decode_large_logits_and_negative_lambda(B):
    Bn, L, Hq, Hkv, d = 2, 3000, 16, 2, 128
    x = I.v2_decode_inputs(Bn, L, Hq, Hkv, d, seed=35, dtype=torch.float32)
    ramp = torch.linspace(0.1, 1.0, L).view(1, L, 1, 1)
    q = (5.0 * x["q"]).to(torch.bfloat16)
    kc = (x["k_cache"] * ramp).to(torch.bfloat16)
    vc = x["v_cache"].to(torch.bfloat16)
    lam = torch.linspace(-1.0, 1.5, Hq // 2)
    out = B.diffattn_v2_decode(cuda(q), cuda(kc), cuda(vc), cuda(lam))
    ref = O.v2_decode_rows(q, kc, vc, lam.double().numpy(), np.arange(Bn * Hq // 2))
    assert_bf16_close(out.reshape(-1, d), ref, True, "v2 decode large logits")
