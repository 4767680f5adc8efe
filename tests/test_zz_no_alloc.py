"""diffattn_v2_decode_noalloc: the V2 decode entry point for callers that
cannot allocate device memory (its split-KV scratch is a fixed 8 MiB device
array inside the library).  Checked through the C ABI against the fp64
oracle and against the regular diffattn_v2_decode on the same inputs, on two
calls in a row with different sizes, so stale scratch contents from the
first call would show up in the second; and at the array's limit, where the
last partial result sits at its very end.  This file is collected last on
purpose."""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
from differential_attention_sm_b200 import inputs as I
from parity import assert_bf16_close, assert_status_ok, status_word

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from differential_attention_sm_b200 import binding
    return binding.load()


def _call_noalloc(lib, q, kc, vc, lens, lam, out, st):
    return lib.diffattn_v2_decode_noalloc(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(kc.data_ptr()),
        ctypes.c_void_p(vc.data_ptr()),
        None if lens is None else ctypes.c_void_p(lens.data_ptr()),
        kc.shape[1], ctypes.c_void_p(out.data_ptr()), q.shape[0], q.shape[1], kc.shape[2],
        ctypes.c_void_p(lam.data_ptr()), ctypes.c_void_p(st.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_matches_workspace_entry_point_twice(lib):
    from differential_attention_sm_b200 import binding as B
    cases = [  # (batch, cache length, query heads, KV heads, per-batch lengths)
        (3, 1000, 16, 2, [1000, 1, 517]),
        (2, 4100, 8, 2, None),
    ]
    for Bn, L, Hq, Hkv, lens in cases:
        x = I.v2_decode_inputs(Bn, L, Hq, Hkv, 128, seed=900 + L)
        q, kc, vc, lam = (x[n].cuda() for n in ("q", "k_cache", "v_cache", "lam"))
        ln = None if lens is None else torch.tensor(lens, dtype=torch.int32, device="cuda")
        ref = B.diffattn_v2_decode(q, kc, vc, lam, cache_lens=ln)
        out = torch.full((Bn, Hq // 2, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = status_word()
        rc = _call_noalloc(lib, q, kc, vc, ln, lam, out, st)
        assert rc == 0, B.status_string(rc)
        assert_status_ok(st)
        assert_bf16_close(out.reshape(-1, 128),
                          ref.reshape(-1, 128).float().cpu().double().numpy(), True,
                          "noalloc vs workspace decode, L=%d" % L)
        orc = O.v2_decode_rows(x["q"], x["k_cache"], x["v_cache"], x["lam"],
                               np.arange(Bn * Hq // 2), lens=lens)
        assert_bf16_close(out.reshape(-1, 128), orc, True, "noalloc vs oracle, L=%d" % L)


def test_noalloc_at_the_scratch_limit(lib):
    """batch * n_kv_heads = 2016 work units, the most the 8 MiB array holds
    (one split each, 8 heads x 130 floats): the last unit's partials end 2 KB
    short of the array's end.  One more unit is refused."""
    from differential_attention_sm_b200 import binding as B
    Bn, L, Hq, Hkv = 252, 200, 16, 8
    x = I.v2_decode_inputs(Bn, L, Hq, Hkv, 128, seed=950)
    q, kc, vc, lam = (x[n].cuda() for n in ("q", "k_cache", "v_cache", "lam"))
    out = torch.full((Bn, Hq // 2, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    st = status_word()
    rc = _call_noalloc(lib, q, kc, vc, None, lam, out, st)
    assert rc == 0, B.status_string(rc)
    assert_status_ok(st)
    orc = O.v2_decode_rows(x["q"], x["k_cache"], x["v_cache"], x["lam"], np.arange(Bn * Hq // 2))
    assert_bf16_close(out.reshape(-1, 128), orc, True, "noalloc at the limit")
    ref = B.diffattn_v2_decode(q, kc, vc, lam)
    assert_bf16_close(out.reshape(-1, 128), ref.reshape(-1, 128).float().cpu().double().numpy(),
                      True, "noalloc vs workspace decode at the limit")
    p = ctypes.c_void_p(q.data_ptr())
    rc = lib.diffattn_v2_decode_noalloc(p, p, p, None, L, p, 2017, 2, 1,
                                        ctypes.c_void_p(lam.data_ptr()), None, None)
    assert rc == B.DA_ERR_UNSUPPORTED


def test_noalloc_rejects_sizes_beyond_its_scratch(lib):
    from differential_attention_sm_b200 import binding as B
    q = torch.zeros(16, dtype=torch.bfloat16, device="cuda")   # never read: rejected first
    lam = torch.zeros(4, dtype=torch.float32, device="cuda")
    p = ctypes.c_void_p(q.data_ptr())
    # 4096 batch entries x 8 KV heads: partials for even one split exceed 8 MiB
    rc = lib.diffattn_v2_decode_noalloc(p, p, p, None, 64, p, 4096, 64, 8,
                                        ctypes.c_void_p(lam.data_ptr()), None, None)
    assert rc == B.DA_ERR_UNSUPPORTED
    # group of 16 query heads per KV head: not handled by the split-KV kernel
    rc = lib.diffattn_v2_decode_noalloc(p, p, p, None, 64, p, 1, 16, 1,
                                        ctypes.c_void_p(lam.data_ptr()), None, None)
    assert rc == B.DA_ERR_UNSUPPORTED
