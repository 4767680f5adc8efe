"""GPU parity of the noise-cancellation sweep (lesson "Atencion Diferencial
(V2)", step 4 and exercises 1 and 4): the differential weights that the V1
decode kernel produces for the signal-plus-noise query, and the
signal-to-noise ratios computed from them, against the fp64 oracle."""
import numpy as np
import pytest

import oracle as O
from differential_attention_sm_b200 import inputs as I
from parity import TOL_BF16_MAX as BF16_MAX_ABS, TOL_BF16_MEAN as BF16_MEAN_ABS

pytestmark = pytest.mark.gpu


def test_snr_sweep_matches_oracle():
    from differential_attention_sm_b200 import binding, snr
    binding.load()
    x = I.snr_inputs()
    res = snr.run_sweep(x)
    lam = x["lam"].double().numpy()
    pos = x["pos"]
    for c, cfg in enumerate(x["configs"]):
        ref = O.v1_query_weights(x["q_cfg"][c], x["k_cfg"][c], lam)
        got = res["weights"][c]
        scale = np.abs(ref).max()
        err = np.abs(got - ref)
        assert err.max() <= BF16_MAX_ABS * scale, (cfg, err.max() / scale)
        assert err.mean() <= BF16_MEAN_ABS * scale, (cfg, err.mean() / scale)
        r_ref = O.snr(ref, pos)
        r_got = res["snr"][c]
        # away from the exact-cancellation point, where the ratio diverges
        ok = np.isfinite(r_ref) & (np.abs(r_ref) < 2000.0)
        assert np.abs(r_got[ok] / r_ref[ok] - 1.0).max() < 0.02, (cfg, r_got, r_ref)
        # the lambda that maximises the ratio, where the oracle's choice is clear
        top = np.sort(r_ref)[::-1]
        if top[0] > 1.05 * top[1]:
            assert np.argmax(r_got) == np.argmax(r_ref), (cfg, r_got, r_ref)
