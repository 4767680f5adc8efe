"""Randomised shapes against the fp64 oracle: prefill in both forms (batch,
length, heads and GQA grouping, causal or not, sliding windows, lambda
outside [0, 1], V1 with and without the norm) and decode in both forms
(ragged cache lengths, windows).  Every output row of every case is
compared.  The cases come from a fixed seed, so a failure is reproducible;
lengths straddle the 128-row query tiles, the 64-key tiles and the decode
kernels' 64-row chunks."""
import numpy as np
import pytest
import torch

import oracle as O
from differential_attention_sm_b200 import inputs as I
from parity import assert_bf16_close, assert_status_ok, status_word

pytestmark = pytest.mark.gpu

N_CASES = 12


@pytest.fixture(scope="module")
def B():
    from differential_attention_sm_b200 import binding
    binding.load()
    return binding


def cuda(t):
    return t.cuda().contiguous()


def _lengths(rng):
    return int(rng.choice([1, 2, 63, 64, 65, 127, 128, 129, 191, 255, 257, 383, 500, 641]))


@pytest.mark.parametrize("case", range(N_CASES))
def test_random_v1_prefill(B, case):
    rng = np.random.default_rng(7000 + case)
    Bn, N, H = int(rng.integers(1, 4)), _lengths(rng), int(rng.integers(1, 5))
    causal = bool(rng.integers(0, 4) > 0)
    window = int(rng.integers(1, N + 40)) if causal and rng.integers(0, 3) == 0 else 0
    norm = bool(rng.integers(0, 2))
    lam = torch.tensor(rng.uniform(-1.0, 2.0, H), dtype=torch.float32)
    li = float(rng.uniform(0.1, 0.8))
    x = I.v1_inputs(Bn, N, H, 64, 128, seed=7100 + case)
    st = status_word()
    out = B.diffattn_v1_fwd_window(cuda(x["q"]), cuda(x["k"]), cuda(x["v"]), cuda(lam), window,
                                   causal=causal, apply_norm=norm, lambda_init=li,
                                   dev_status=st)
    assert_status_ok(st)
    ref = O.v1_rows(x["q"], x["k"], x["v"], lam.double().numpy(), np.arange(Bn * N * H),
                    causal=causal, window=window, apply_norm=norm, lambda_init_value=li)
    what = "v1 B%d N%d H%d causal=%s window=%d norm=%s" % (Bn, N, H, causal, window, norm)
    assert_bf16_close(out.reshape(-1, 128), ref, not norm, what)


@pytest.mark.parametrize("case", range(N_CASES))
def test_random_v2_prefill(B, case):
    rng = np.random.default_rng(7200 + case)
    Hkv = int(rng.integers(1, 4))
    Hq = Hkv * int(rng.choice([2, 4, 6, 8]))
    Bn, N = int(rng.integers(1, 3)), _lengths(rng)
    causal = bool(rng.integers(0, 4) > 0)
    window = int(rng.integers(1, N + 40)) if causal and rng.integers(0, 3) == 0 else 0
    x = I.v2_inputs(Bn, N, Hq, Hkv, 128, seed=7300 + case)
    lam = torch.tensor(rng.uniform(-1.0, 2.0, Hq // 2), dtype=torch.float32)
    st = status_word()
    out = B.diffattn_v2_prefill_window(cuda(x["q"]), cuda(x["k"]), cuda(x["v"]), cuda(lam),
                                       window, causal=causal, dev_status=st)
    assert_status_ok(st)
    ref = O.v2_rows(x["q"], x["k"], x["v"], lam.double().numpy(), np.arange(Bn * N * Hq // 2),
                    causal=causal, window=window)
    what = "v2 B%d N%d Hq%d Hkv%d causal=%s window=%d" % (Bn, N, Hq, Hkv, causal, window)
    assert_bf16_close(out.reshape(-1, 128), ref, True, what)


@pytest.mark.parametrize("case", range(N_CASES))
def test_random_decode(B, case):
    rng = np.random.default_rng(7400 + case)
    Bn, L = int(rng.integers(1, 5)), int(rng.integers(1, 3000))
    lens = [int(v) for v in rng.integers(1, L + 1, Bn)]
    window = int(rng.integers(1, L + 100)) if rng.integers(0, 3) == 0 else 0
    # V2: group of 2, 4, 6 or 8 query heads per KV head
    Hkv = int(rng.integers(1, 3))
    Hq = Hkv * int(rng.choice([2, 4, 6, 8]))
    x = I.v2_decode_inputs(Bn, L, Hq, Hkv, 128, seed=7500 + case)
    ln = torch.tensor(lens, dtype=torch.int32)
    st = status_word()
    out = B.diffattn_v2_decode_window(cuda(x["q"]), cuda(x["k_cache"]), cuda(x["v_cache"]),
                                      cuda(x["lam"]), window, cache_lens=cuda(ln), dev_status=st)
    assert_status_ok(st)
    ref = O.v2_decode_rows(x["q"], x["k_cache"], x["v_cache"], x["lam"],
                           np.arange(Bn * Hq // 2), lens=lens, window=window)
    assert_bf16_close(out.reshape(-1, 128), ref, True,
                      "v2 decode B%d L%d Hq%d Hkv%d window=%d" % (Bn, L, Hq, Hkv, window))
    # V1 with the norm, same lengths
    H = int(rng.integers(1, 4))
    y = I.v1_decode_inputs(Bn, L, H, 64, 128, seed=7600 + case)
    lam = torch.tensor(rng.uniform(-1.0, 2.0, H), dtype=torch.float32)
    out = B.diffattn_v1_decode_window(cuda(y["q"]), cuda(y["k_cache"]), cuda(y["v_cache"]),
                                      cuda(lam), window, cache_lens=cuda(ln), apply_norm=True,
                                      lambda_init=0.4)
    ref = O.v1_decode_rows(y["q"], y["k_cache"], y["v_cache"], lam.double().numpy(),
                           np.arange(Bn * H), lens=lens, window=window, apply_norm=True,
                           lambda_init_value=0.4)
    assert_bf16_close(out.reshape(-1, 128), ref, False,
                      "v1 decode B%d L%d H%d window=%d" % (Bn, L, H, window))
