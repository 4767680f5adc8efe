"""Failure detection on the GPU without a fault: the pipelines' bounded wait
is run to its timeout on a barrier that nothing arrives on; the kernel
reports DA_ERR_DEVICE_TIMEOUT in the status word and returns, and the same
context then runs a prefill that matches the oracle."""
import numpy as np
import pytest
import torch

import oracle as O
from differential_attention_sm_b200 import inputs as I
from parity import assert_bf16_close, assert_status_ok, status_word

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_stays_usable():
    from differential_attention_sm_b200 import binding as B
    B.load()
    st = status_word()
    waited = torch.zeros(1, dtype=torch.int64, device="cuda")
    B.diffattn_selftest_wait_timeout(20000, st, waited)   # 20 ms limit
    torch.cuda.synchronize()
    assert int(st.item()) == B.DA_ERR_DEVICE_TIMEOUT
    ns = int(waited.item())
    assert 20e6 <= ns < 2e9, ns
    # the context is still usable: a prefill right after matches the oracle
    x = I.v2_inputs(1, 200, 8, 2, 128, seed=1700)
    st2 = status_word()
    out = B.diffattn_v2_prefill(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(), x["lam"].cuda(),
                                dev_status=st2)
    assert_status_ok(st2)
    ref = O.v2_rows(x["q"], x["k"], x["v"], x["lam"], np.arange(200 * 4), causal=True)
    assert_bf16_close(out.reshape(-1, 128), ref, True, "prefill after a timeout")
