"""Pins of the fp64 oracle against facts the pages and the mathematics fix.

None of these tests re-types the oracle's formula: each checks the oracle
against a value the pages print, a closed form, an invariant, or an
independent library routine (torch's scaled_dot_product_attention and
rms_norm in float64).  Together they fail on a dropped term, a flipped sign,
a wrong scale, a swapped branch half, a wrong head/KV mapping or a wrong
mask.

Sources: "Differential Transformer" (Ultralytics glossary), section
"Cómo funciona la atención diferencial" [G]; "Atención Diferencial (V2)"
(ai-engineering.academy), sections "La idea diferencial", "V1 vs V2: la
diferencia", "Implementación" and "Ejercicios" [L].
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle as O
from differential_attention_sm_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def sdpa(q, k, v, causal=False, enable_gqa=False):
    """torch float64 SDPA on [B, N, H, D] tensors (scale 1/sqrt(D_q))."""
    qt, kt, vt = (x.double().permute(0, 2, 1, 3) for x in (q, k, v))
    o = F.scaled_dot_product_attention(qt, kt, vt, is_causal=causal,
                                       enable_gqa=enable_gqa)
    return o.permute(0, 2, 1, 3)


def all_rows_v1(B, N, H):
    return np.arange(B * N * H)


def rand(*shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g)


# --------------------------------------------------------------------------
# [G] worked example: seed 0, n=6, d=8, lambda 0.8 -> "0.20; 13 of 36"
# --------------------------------------------------------------------------
def test_worked_example_matches_printed_line():
    gold = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    q1, k1, q2, k2, v = I.worked_example()
    n = gold["n"]
    q = torch.cat([q1, q2], -1).reshape(1, n, 1, 2 * gold["d"])
    k = torch.cat([k1, k2], -1).reshape(1, n, 1, 2 * gold["d"])
    vv = v.reshape(1, n, 1, gold["dv"])
    out, w = O.v1_rows(q, k, vv, [gold["lambda"]], np.arange(n), causal=False,
                       return_weights=True)
    sums = w.sum(axis=1)
    assert all("%.2f" % s == gold["printed_row_sum"] for s in sums)
    assert int((w < 0).sum()) == gold["negative_weights"]
    assert w.size == gold["total_weights"]
    # the output is the weights applied to V (the page's `diff @ v`)
    assert np.allclose(out, w @ v.double().numpy(), rtol=0, atol=1e-13)


# --------------------------------------------------------------------------
# [G]: every row of the difference map sums to 1 - lambda, for any lambda
# --------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("lam", [0.8, -0.35, 1.7, 0.0])
def test_row_sums_equal_one_minus_lambda(causal, lam):
    B, N, H, d, dv = 2, 19, 3, 5, 7
    q, k, v = rand(B, N, H, 2 * d, seed=1), rand(B, N, H, 2 * d, seed=2), rand(B, N, H, dv, seed=3)
    lams = [lam, lam * 0.5 - 0.1, lam + 0.3]
    _, w = O.v1_rows(q, k, v, lams, all_rows_v1(B, N, H), causal=causal,
                     return_weights=True)
    h = np.arange(B * N * H) % H
    i = (np.arange(B * N * H) // H) % N
    expect = 1.0 - np.asarray(lams)[h]
    assert np.abs(w.sum(axis=1) - expect).max() < 1e-12
    if causal:  # keys after the query carry no weight
        for r in range(w.shape[0]):
            assert np.all(w[r, i[r] + 1:] == 0.0)
    # some weights are negative whenever lambda > 0 (softmax maps never are)
    if lam > 0.5:
        assert (w < 0).any()


# --------------------------------------------------------------------------
# [L] exercise 4: lambda = 0 is plain softmax attention of branch 1
# --------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [False, True])
def test_lambda_zero_is_softmax_attention(causal):
    B, N, H, d, dv = 2, 23, 3, 6, 10
    q, k, v = rand(B, N, H, 2 * d, seed=4), rand(B, N, H, 2 * d, seed=5), rand(B, N, H, dv, seed=6)
    out = O.v1_rows(q, k, v, [0.0] * H, all_rows_v1(B, N, H), causal=causal)
    ref = sdpa(q[..., :d], k[..., :d], v, causal)
    assert np.abs(out - ref.reshape(-1, dv).numpy()).max() < 1e-12


# --------------------------------------------------------------------------
# [G]: each map is ordinary softmax attention -> A1 V - lambda A2 V
# --------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [False, True])
def test_v1_is_difference_of_two_attentions(causal):
    B, N, H, d, dv = 2, 29, 4, 8, 16
    q, k, v = rand(B, N, H, 2 * d, seed=7), rand(B, N, H, 2 * d, seed=8), rand(B, N, H, dv, seed=9)
    lams = torch.tensor([0.8, -0.2, 1.3, 0.45], dtype=torch.float64)
    out = O.v1_rows(q, k, v, lams, all_rows_v1(B, N, H), causal=causal)
    a1 = sdpa(q[..., :d], k[..., :d], v, causal)
    a2 = sdpa(q[..., d:], k[..., d:], v, causal)
    ref = a1 - lams.view(1, 1, H, 1) * a2
    assert np.abs(out - ref.reshape(-1, dv).numpy()).max() < 1e-12


def test_identical_branches_scale_softmax_attention():
    B, N, H, d, dv = 1, 31, 2, 8, 16
    half_q, half_k = rand(B, N, H, d, seed=10), rand(B, N, H, d, seed=11)
    q, k = torch.cat([half_q, half_q], -1), torch.cat([half_k, half_k], -1)
    v = rand(B, N, H, dv, seed=12)
    lam = [0.8, 0.3]
    out = O.v1_rows(q, k, v, lam, all_rows_v1(B, N, H), causal=True)
    ref = sdpa(half_q, half_k, v, True) * (1 - torch.tensor(lam, dtype=torch.float64)).view(1, 1, H, 1)
    assert np.abs(out - ref.reshape(-1, dv).numpy()).max() < 1e-12


def test_causal_first_row_closed_form():
    B, N, H, d, dv = 2, 9, 2, 4, 8
    q, k, v = rand(B, N, H, 2 * d, seed=13), rand(B, N, H, 2 * d, seed=14), rand(B, N, H, dv, seed=15)
    lam = [0.8, -0.6]
    rows = np.array([(b * N + 0) * H + h for b in range(B) for h in range(H)])
    out = O.v1_rows(q, k, v, lam, rows, causal=True)
    for t, r in enumerate(rows):
        b, h = r // (N * H), r % H
        assert np.allclose(out[t], (1 - lam[h]) * v[b, 0, h].double().numpy(), rtol=0, atol=1e-15)
    # with the per-head norm the row becomes RMSNorm((1-lam) V0) (1 - lambda_init)
    li = O.lambda_init(5)
    outn = O.v1_rows(q, k, v, lam, rows, causal=True, apply_norm=True, eps=1e-5,
                     lambda_init_value=li)
    for t, r in enumerate(rows):
        b, h = r // (N * H), r % H
        pre = (1 - lam[h]) * v[b, 0, h].double()
        ref = F.rms_norm(pre, (dv,), eps=1e-5) * (1 - li)
        assert np.allclose(outn[t], ref.numpy(), rtol=0, atol=1e-14)


# --------------------------------------------------------------------------
# [G] per-head normalisation then (1 - lambda_init): library rms_norm pin
# --------------------------------------------------------------------------
def test_head_norm_matches_library_rms_norm():
    B, N, H, d, dv = 1, 17, 3, 8, 16
    q, k, v = rand(B, N, H, 2 * d, seed=16), rand(B, N, H, 2 * d, seed=17), rand(B, N, H, dv, seed=18)
    g = 0.5 + rand(dv, seed=19).abs()
    lam = [0.7, 0.2, -0.1]
    li = O.lambda_init(12)
    rows = all_rows_v1(B, N, H)
    pre = O.v1_rows(q, k, v, lam, rows, causal=True)
    post = O.v1_rows(q, k, v, lam, rows, causal=True, apply_norm=True,
                     norm_weight=g, eps=1e-5, lambda_init_value=li)
    ref = F.rms_norm(torch.from_numpy(pre), (dv,), weight=g.double(), eps=1e-5) * (1 - li)
    assert np.abs(post - ref.numpy()).max() < 1e-13
    # with unit gain every row's RMS is (1 - lambda_init) up to eps
    post1 = O.v1_rows(q, k, v, lam, rows, causal=True, apply_norm=True, eps=0.0,
                      lambda_init_value=li)
    rms = np.sqrt((post1 ** 2).mean(axis=1))
    assert np.abs(rms - (1 - li)).max() < 1e-13


# --------------------------------------------------------------------------
# lambda_init schedule and lambda re-parameterisation ([G], [L])
# --------------------------------------------------------------------------
def test_lambda_init_schedule():
    assert O.lambda_init(1) == pytest.approx(0.2, abs=1e-15)   # exp(0) = 1
    assert math.isnan(O.lambda_init(0))
    vals = [O.lambda_init(l) for l in range(1, 40)]
    assert all(b > a for a, b in zip(vals, vals[1:]))          # deeper -> closer to 0.8
    assert O.lambda_init(2000) == pytest.approx(0.8, abs=1e-15)
    # the gap to 0.8 shrinks by the same factor exp(-0.3) every layer
    ratios = [(0.8 - b) / (0.8 - a) for a, b in zip(vals, vals[1:])]
    assert max(ratios) - min(ratios) < 1e-9
    assert ratios[0] == pytest.approx(math.exp(-0.3), rel=1e-12)


def test_lambda_from_params_special_cases():
    H, dim = 3, 4
    z = np.zeros((H, dim), np.float32)
    for layer in (1, 12, 24):
        assert np.allclose(O.lambda_from_params(z, z, z, z, layer),
                           O.lambda_init(layer), rtol=0, atol=1e-15)
    # head 1: lq1 . lk1 = 1 exactly, the second dot 0 -> e - 1 + lambda_init
    # head 2: the second dot is 2 -> 1 - e^2 + lambda_init (negative lambda)
    lq1, lk1, lq2, lk2 = (np.zeros((H, dim), np.float32) for _ in range(4))
    lq1[1, :2] = [0.5, 0.25]
    lk1[1, :2] = [1.0, 2.0]
    lq2[2, 3] = 4.0
    lk2[2, 3] = 0.5
    lam = O.lambda_from_params(lq1, lk1, lq2, lk2, 12)
    li = O.lambda_init(12)
    assert lam[0] == pytest.approx(li, abs=1e-15)
    assert lam[1] == pytest.approx(math.e - 1 + li, abs=1e-14)
    assert lam[2] == pytest.approx(1 - math.e ** 2 + li, abs=1e-13)
    assert lam[2] < 0


# --------------------------------------------------------------------------
# V2: paired query heads sharing GQA KV heads ([L] "V1 vs V2", exercise 5)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [True, False])
def test_v2_is_difference_of_paired_gqa_attentions(causal):
    B, N, Hq, Hkv, d = 2, 21, 8, 2, 16
    q, k, v = rand(B, N, Hq, d, seed=20), rand(B, N, Hkv, d, seed=21), rand(B, N, Hkv, d, seed=22)
    lam = 0.2 + 0.6 * torch.rand(Hq // 2, generator=torch.Generator().manual_seed(23))
    rows = np.arange(B * N * (Hq // 2))
    out = O.v2_rows(q, k, v, lam, rows, causal=causal)
    per_head = sdpa(q, k, v, causal, enable_gqa=True)   # head h reads kv h // (Hq/Hkv)
    ref = per_head[:, :, 0::2] - lam.double().view(1, 1, -1, 1) * per_head[:, :, 1::2]
    assert np.abs(out - ref.reshape(-1, d).numpy()).max() < 1e-12


def test_v2_equals_v1_relaid_out():
    """[L] step 2: V1 and V2 share the maths, only the bookkeeping differs."""
    B, N, Hq, Hkv, d = 1, 13, 4, 1, 8
    q, k, v = rand(B, N, Hq, d, seed=24), rand(B, N, Hkv, d, seed=25), rand(B, N, Hkv, d, seed=26)
    lam = [0.8, 0.25]
    out2 = O.v2_rows(q, k, v, lam, np.arange(B * N * 2), causal=True)
    # as V1: head p has Q = [q_{2p} | q_{2p+1}], K = [k_g | k_g], V = v_g
    q1 = torch.stack([torch.cat([q[:, :, 2 * p], q[:, :, 2 * p + 1]], -1) for p in range(2)], 2)
    k1 = torch.stack([torch.cat([k[:, :, 0], k[:, :, 0]], -1) for _ in range(2)], 2)
    v1 = torch.stack([v[:, :, 0] for _ in range(2)], 2)
    out1 = O.v1_rows(q1, k1, v1, lam, np.arange(B * N * 2), causal=True)
    assert np.abs(out1 - out2).max() < 1e-14


def test_v2_gqa_cache_size_matches_baseline():
    """[L] exercise 5: with 32 query heads and 8 KV heads the V2 cache is the
    size of a baseline GQA cache (no doubling)."""
    w = I.WORKLOADS["v2_decode_bf16"]
    x = I.v2_decode_inputs(2, 8, w.Hq, w.Hkv, w.d, seed=0)
    assert x["k_cache"].shape == (2, 8, w.Hkv, w.d)
    assert x["k_cache"].numel() * 2 == 2 * 8 * w.Hkv * w.d * 2
    assert x["q"].shape[1] == 2 * (w.Hq // 2)


# --------------------------------------------------------------------------
# decode: one query against the first len_b cache entries
# --------------------------------------------------------------------------
def test_v2_decode_matches_library_and_prefill_last_row():
    B, L, Hq, Hkv, d = 3, 40, 8, 2, 16
    x = I.v2_decode_inputs(B, L, Hq, Hkv, d, seed=27, dtype=torch.float32)
    lens = [40, 1, 17]
    rows = np.arange(B * Hq // 2)
    out = O.v2_decode_rows(x["q"], x["k_cache"], x["v_cache"], x["lam"], rows, lens=lens)
    for b in range(B):
        n = lens[b]
        qq = x["q"][b].reshape(1, 1, Hq, d)
        kk = x["k_cache"][b, :n].reshape(1, n, Hkv, d)
        vv = x["v_cache"][b, :n].reshape(1, n, Hkv, d)
        per_head = sdpa(qq, kk, vv, False, enable_gqa=True)[0, 0]
        ref = per_head[0::2] - x["lam"].double().view(-1, 1) * per_head[1::2]
        got = out[b * Hq // 2:(b + 1) * Hq // 2]
        assert np.abs(got - ref.numpy()).max() < 1e-12
        # same as the last row of causal prefill over the cached sequence
        qseq = torch.zeros(1, n, Hq, d)
        qseq[0, n - 1] = x["q"][b]
        pre = O.v2_rows(qseq, kk, vv, x["lam"], np.arange((n - 1) * Hq // 2, n * Hq // 2),
                        causal=True)
        assert np.abs(pre - got).max() < 1e-14


def test_v1_decode_matches_library_with_norm():
    B, L, H, d, dv = 2, 33, 3, 8, 16
    x = I.v1_decode_inputs(B, L, H, d, dv, seed=28, dtype=torch.float32)
    lam = O.lambda_from_params(x["lq1"], x["lk1"], x["lq2"], x["lk2"], 12)
    li = O.lambda_init(12)
    lens = [33, 5]
    out = O.v1_decode_rows(x["q"], x["k_cache"], x["v_cache"], lam, np.arange(B * H),
                           lens=lens, apply_norm=True, eps=1e-5, lambda_init_value=li)
    for b in range(B):
        n = lens[b]
        qq = x["q"][b].reshape(1, 1, H, 2 * d)
        kk = x["k_cache"][b, :n].reshape(1, n, H, 2 * d)
        vv = x["v_cache"][b, :n].reshape(1, n, H, dv)
        a1 = sdpa(qq[..., :d], kk[..., :d], vv)[0, 0]
        a2 = sdpa(qq[..., d:], kk[..., d:], vv)[0, 0]
        pre = a1 - torch.from_numpy(lam).view(H, 1) * a2
        ref = F.rms_norm(pre, (dv,), eps=1e-5) * (1 - li)
        assert np.abs(out[b * H:(b + 1) * H] - ref.numpy()).max() < 1e-13


# --------------------------------------------------------------------------
# planted signal of the long-context workload: branch 1 finds the needles
# --------------------------------------------------------------------------
def test_planted_signal_is_found_by_branch_one():
    B, N, H, d, dv = 1, 2048, 2, 64, 128
    x = I.v1_inputs(B, N, H, d, dv, seed=2, dtype=torch.bfloat16, planted=6)
    rows = np.array([(N - 2) * H + h for h in range(H)] + [(N - 1) * H + h for h in range(H)])
    _, w = O.v1_rows(x["q"], x["k"], x["v"], [0.0] * H, rows, causal=True,
                     return_weights=True)   # lambda = 0: w is branch 1's map
    for t, r in enumerate(rows):
        h = r % H
        pos = x["planted_pos"][0, h].numpy()
        assert w[t, pos].sum() > 0.8


def test_oracle_rejects_out_of_range_rows():
    q = torch.zeros(1, 4, 1, 4)
    with pytest.raises(ValueError):
        O.v1_rows(q, q, torch.zeros(1, 4, 1, 2), [0.5], np.array([4]), causal=True)


def test_large_logits_stay_finite_and_exact():
    """[L] step 1 subtracts the row maximum before exponentiating, so logits
    in the hundreds (far beyond exp's float64 range once summed) still give
    the library's softmax attention."""
    B, N, H, d, dv = 1, 11, 2, 8, 8
    q = 60.0 * rand(B, N, H, 2 * d, seed=40)
    k = 60.0 * rand(B, N, H, 2 * d, seed=41)
    v = rand(B, N, H, dv, seed=42)
    lam = [0.8, -0.4]
    out = O.v1_rows(q, k, v, lam, all_rows_v1(B, N, H), causal=False)
    assert np.isfinite(out).all()
    a1 = sdpa(q[..., :d], k[..., :d], v)
    a2 = sdpa(q[..., d:], k[..., d:], v)
    ref = a1 - torch.tensor(lam, dtype=torch.float64).view(1, 1, H, 1) * a2
    assert np.abs(out - ref.reshape(-1, dv).numpy()).max() < 1e-9


# --------------------------------------------------------------------------
# [L] step 4 / exercises 1 and 4: noise cancellation on a signal-plus-noise
# query.  The ratio is the signal weight over the RMS of the other weights.
# --------------------------------------------------------------------------
def test_snr_statistic_on_hand_built_rows():
    w = np.full(101, 0.01)
    w[1::2] = -0.01
    w[40] = 0.5
    assert O.snr(w, 40) == pytest.approx(50.0, rel=1e-14)
    w2 = np.zeros(7)
    w2[3] = 0.25
    assert O.snr(w2, 3) == math.inf
    w3 = np.array([3.0, 1.0, 1.0, 1.0, 4.0])   # noise rms = sqrt((9+1+1+16)/4) at pos 1
    assert O.snr(w3, 1) == pytest.approx(1.0 / math.sqrt(27.0 / 4.0), rel=1e-14)


def _snr_scores(x, c):
    """fp64 scores of the sweep query against its keys, per branch."""
    q = x["q_cfg"][c].double()
    k = x["k_cfg"][c].double()
    d = q.numel() // 2
    return (k[:, :d] @ q[:d]) / math.sqrt(d), (k[:, d:] @ q[d:]) / math.sqrt(d)


def test_snr_sweep_lambda_zero_is_softmax_and_rows_sum_to_one_minus_lambda():
    x = I.snr_inputs()
    lam = x["lam"].double().numpy()
    for c in range(len(x["configs"])):
        w = O.v1_query_weights(x["q_cfg"][c], x["k_cfg"][c], lam)
        s1, _ = _snr_scores(x, c)
        assert np.abs(w[0] - torch.softmax(s1, 0).numpy()).max() < 1e-15
        assert np.abs(w.sum(1) - (1.0 - lam)).max() < 1e-12


def test_snr_shared_noise_cancels_exactly_at_partition_ratio():
    """With q1 = q2 and the same noise keys in both branches, every noise
    weight is e^{s_j} (1/Z1 - lambda/Z2): all of them vanish together at
    lambda* = Z2 / Z1, where only the signal weight is left."""
    x = I.snr_inputs(sigmas=(1.5,), rhos=(1.0,))
    s1, s2 = _snr_scores(x, 0)
    pos = x["pos"]
    mask = torch.ones_like(s1, dtype=torch.bool)
    mask[pos] = False
    assert torch.equal(s1[mask], s2[mask])
    lam_star = float(torch.exp(torch.logsumexp(s2, 0) - torch.logsumexp(s1, 0)))
    w = O.v1_query_weights(x["q_cfg"][0], x["k_cfg"][0], [lam_star, 0.5])
    noise = np.delete(w[0], pos)
    assert np.abs(noise).max() < 1e-15 * np.abs(w[0]).max() + 1e-300
    sig = float(torch.softmax(s1, 0)[pos] - lam_star * torch.softmax(s2, 0)[pos])
    assert w[0, pos] == pytest.approx(sig, rel=1e-12)
    assert O.snr(w[1:], pos)[0] < O.snr(w[:1], pos)[0]


def test_snr_identical_branches_do_not_depend_on_lambda():
    """K2 = K1 everywhere (the signal included): w = (1 - lambda) softmax, so
    the ratio is the same for every lambda < 1."""
    x = I.snr_inputs(sigmas=(1.0,), rhos=(1.0,))
    k = x["k_cfg"][0].clone()
    d = k.shape[1] // 2
    k[:, d:] = k[:, :d]
    lam = np.array([0.0, 0.3, 0.6, 0.9])
    r = O.snr(O.v1_query_weights(x["q_cfg"][0], k, lam), x["pos"])
    assert np.abs(r / r[0] - 1.0).max() < 1e-12


# --------------------------------------------------------------------------
# [L] "Úselo": differential attention combined with sliding-window attention.
# Reading: query i sees keys j with i - W < j <= i, in both branches.
# --------------------------------------------------------------------------
def _band_mask(N, W):
    i = torch.arange(N)[:, None]
    j = torch.arange(N)[None, :]
    return (j <= i) & (j > i - W)


@pytest.mark.parametrize("W", [1, 5, 16, 40])
def test_window_is_difference_of_band_masked_attentions(W):
    B, N, H, d, dv = 2, 37, 3, 8, 16
    q, k, v = rand(B, N, H, 2 * d, seed=70), rand(B, N, H, 2 * d, seed=71), rand(B, N, H, dv, seed=72)
    lams = torch.tensor([0.8, -0.3, 1.2], dtype=torch.float64)
    out = O.v1_rows(q, k, v, lams, all_rows_v1(B, N, H), causal=True, window=W)
    m = _band_mask(N, W)

    def att(qh, kh):
        qt, kt, vt = (x.double().permute(0, 2, 1, 3) for x in (qh, kh, v))
        return F.scaled_dot_product_attention(qt, kt, vt, attn_mask=m).permute(0, 2, 1, 3)

    ref = att(q[..., :d], k[..., :d]) - lams.view(1, 1, H, 1) * att(q[..., d:], k[..., d:])
    assert np.abs(out - ref.reshape(-1, dv).numpy()).max() < 1e-12


def test_window_one_keeps_only_the_diagonal_and_wide_window_is_causal():
    B, N, H, d, dv = 1, 19, 2, 8, 16
    q, k, v = rand(B, N, H, 2 * d, seed=73), rand(B, N, H, 2 * d, seed=74), rand(B, N, H, dv, seed=75)
    lam = [0.6, 1.4]
    out = O.v1_rows(q, k, v, lam, all_rows_v1(B, N, H), causal=True, window=1)
    ref = (1.0 - torch.tensor(lam, dtype=torch.float64)).view(1, 1, H, 1) * v.double()
    assert np.abs(out - ref.reshape(-1, dv).numpy()).max() < 1e-15
    full = O.v1_rows(q, k, v, lam, all_rows_v1(B, N, H), causal=True)
    wide = O.v1_rows(q, k, v, lam, all_rows_v1(B, N, H), causal=True, window=N)
    assert np.array_equal(full, wide)


def test_window_row_equals_last_row_of_the_sliced_sequence():
    """Row i under window W is causal attention over tokens i-W+1..i alone."""
    B, N, Hq, Hkv, d, W = 1, 41, 4, 2, 16, 9
    x = I.v2_inputs(B, N, Hq, Hkv, d, seed=76, dtype=torch.float32)
    P = Hq // 2
    out = O.v2_rows(x["q"], x["k"], x["v"], x["lam"], np.arange(B * N * P), causal=True,
                    window=W).reshape(N, P, d)
    for i in (0, 5, W - 1, W, 23, N - 1):
        a = max(0, i - W + 1)
        sl = O.v2_rows(x["q"][:, a:i + 1], x["k"][:, a:i + 1], x["v"][:, a:i + 1], x["lam"],
                       np.arange((i - a) * P, (i - a + 1) * P), causal=True).reshape(P, d)
        assert np.abs(out[i] - sl).max() < 1e-13


def test_window_decode_equals_decode_over_the_last_entries():
    Bn, L, Hq, Hkv, d, W = 2, 70, 8, 2, 16, 13
    x = I.v2_decode_inputs(Bn, L, Hq, Hkv, d, seed=77, dtype=torch.float32)
    lens = [70, 31]
    rows = np.arange(Bn * Hq // 2)
    out = O.v2_decode_rows(x["q"], x["k_cache"], x["v_cache"], x["lam"], rows, lens=lens,
                           window=W).reshape(Bn, Hq // 2, d)
    for b, n in enumerate(lens):
        kc = x["k_cache"][b:b + 1, n - W:n]
        vc = x["v_cache"][b:b + 1, n - W:n]
        ref = O.v2_decode_rows(x["q"][b:b + 1], kc, vc, x["lam"], np.arange(Hq // 2))
        assert np.abs(out[b] - ref).max() < 1e-13
    # V1 decode: the window applies before the norm
    x1 = I.v1_decode_inputs(Bn, L, 3, 8, 16, seed=78)
    lam1 = np.array([0.7, 0.2, -0.4])
    o1 = O.v1_decode_rows(x1["q"], x1["k_cache"], x1["v_cache"], lam1, np.arange(Bn * 3),
                          lens=lens, apply_norm=True, lambda_init_value=0.5,
                          window=W).reshape(Bn, 3, 16)
    for b, n in enumerate(lens):
        r1 = O.v1_decode_rows(x1["q"][b:b + 1], x1["k_cache"][b:b + 1, n - W:n],
                              x1["v_cache"][b:b + 1, n - W:n], lam1, np.arange(3),
                              apply_norm=True, lambda_init_value=0.5)
        assert np.abs(o1[b] - r1).max() < 1e-13


# --------------------------------------------------------------------------
# Backward pass: gradients of the forward defined by [G] / [L], pinned to
# float64 torch autograd of an SDPA-based statement of the same forward and
# to central finite differences of the oracle's own (pinned) forward.
# --------------------------------------------------------------------------
def _torch_v1_forward(q, k, v, lam, g, causal, window, apply_norm, lam_init, eps=1e-5):
    d = q.shape[-1] // 2
    N = q.shape[1]
    mask = None
    if causal:
        mask = _band_mask(N, window if window > 0 else N)

    def att(qh, kh):
        qt, kt, vt = (x.permute(0, 2, 1, 3) for x in (qh, kh, v))
        return F.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask).permute(0, 2, 1, 3)

    o = att(q[..., :d], k[..., :d]) - lam.view(1, 1, -1, 1) * att(q[..., d:], k[..., d:])
    if apply_norm:
        o = F.rms_norm(o, (o.shape[-1],), weight=g, eps=eps) * (1.0 - lam_init)
    return o


@pytest.mark.parametrize("causal,window,apply_norm", [(True, 0, True), (False, 0, False),
                                                       (True, 6, True), (True, 0, False)])
def test_v1_backward_matches_float64_autograd(causal, window, apply_norm):
    B, N, H, d, dv = 2, 17, 3, 8, 16
    q, k, v = rand(B, N, H, 2 * d, seed=80), rand(B, N, H, 2 * d, seed=81), rand(B, N, H, dv, seed=82)
    dout = rand(B, N, H, dv, seed=83)
    lam = torch.tensor([0.8, -0.25, 1.3], dtype=torch.float64)
    g = (1.0 + 0.3 * rand(dv, seed=84)).double()
    li = 0.55
    res = O.v1_bwd(q, k, v, dout, lam, causal=causal, window=window, apply_norm=apply_norm,
                   norm_weight=g.float() if apply_norm else None, lambda_init_value=li)
    qt, kt, vt = (x.double().requires_grad_(True) for x in (q, k, v))
    lt = lam.clone().requires_grad_(True)
    gt = g.clone().requires_grad_(True)
    y = _torch_v1_forward(qt, kt, vt, lt, gt, causal, window, apply_norm, li)
    (y * dout.double()).sum().backward()
    for name, ref in (("dq", qt.grad), ("dk", kt.grad), ("dv", vt.grad), ("dlambda", lt.grad)):
        assert np.abs(res[name] - ref.numpy()).max() < 1e-11, name
    if apply_norm:
        assert np.abs(res["dnorm_weight"] - gt.grad.numpy()).max() < 1e-11


@pytest.mark.parametrize("causal,window", [(True, 0), (False, 0), (True, 9)])
def test_v2_backward_matches_float64_autograd(causal, window):
    B, N, Hq, Hkv, d = 1, 19, 8, 2, 8
    x = I.v2_inputs(B, N, Hq, Hkv, d, seed=85, dtype=torch.float32)
    dout = rand(B, N, Hq // 2, d, seed=86)
    res = O.v2_bwd(x["q"], x["k"], x["v"], dout, x["lam"], causal=causal, window=window)
    qt, kt, vt = (x[n].double().requires_grad_(True) for n in ("q", "k", "v"))
    lt = x["lam"].double().clone().requires_grad_(True)
    mask = _band_mask(N, window if window > 0 else N) if causal else None

    def att(qh):
        return F.scaled_dot_product_attention(qh.permute(0, 2, 1, 3), kt.permute(0, 2, 1, 3),
                                              vt.permute(0, 2, 1, 3), attn_mask=mask,
                                              enable_gqa=True).permute(0, 2, 1, 3)

    y = att(qt[:, :, 0::2]) - lt.view(1, 1, -1, 1) * att(qt[:, :, 1::2])
    (y * dout.double()).sum().backward()
    for name, ref in (("dq", qt.grad), ("dk", kt.grad), ("dv", vt.grad), ("dlambda", lt.grad)):
        assert np.abs(res[name] - ref.numpy()).max() < 1e-11, name


def test_v1_backward_matches_finite_differences_of_the_oracle():
    B, N, H, d, dv = 1, 6, 2, 3, 4
    q, k, v = rand(B, N, H, 2 * d, seed=87).double(), rand(B, N, H, 2 * d, seed=88).double(), rand(B, N, H, dv, seed=89).double()
    dout = rand(B, N, H, dv, seed=90).double()
    lam = np.array([0.7, -0.4])
    li, eps_n = 0.3, 1e-5
    rows = all_rows_v1(B, N, H)

    def loss(qq, kk, vv, ll):
        o = O.v1_rows(qq.float(), kk.float(), vv.float(), ll, rows, causal=True,
                      apply_norm=True, lambda_init_value=li, eps=eps_n)
        return float((o * dout.reshape(-1, dv).numpy()).sum())

    # float32 inputs: step sizes well above float32 resolution, tolerance to match
    res = O.v1_bwd(q, k, v, dout, lam, causal=True, apply_norm=True, lambda_init_value=li)
    h = 1e-2
    for name, t in (("dq", q), ("dk", k), ("dv", v)):
        for idx in [(0, 0, 0, 0), (0, 3, 1, 2), (0, 5, 1, t.shape[-1] - 1)]:
            tp, tm = t.clone(), t.clone()
            tp[idx] += h
            tm[idx] -= h
            args_p = {"dq": (tp, k, v), "dk": (q, tp, v), "dv": (q, k, tp)}[name]
            args_m = {"dq": (tm, k, v), "dk": (q, tm, v), "dv": (q, k, tm)}[name]
            fd = (loss(*args_p, lam) - loss(*args_m, lam)) / (2 * h)
            assert res[name][idx] == pytest.approx(fd, rel=2e-3, abs=2e-4), (name, idx)
    for hh in range(H):
        lp, lm = lam.copy(), lam.copy()
        lp[hh] += 1e-4
        lm[hh] -= 1e-4
        fd = (loss(q, k, v, lp) - loss(q, k, v, lm)) / 2e-4
        assert res["dlambda"][hh] == pytest.approx(fd, rel=1e-6, abs=1e-9)


def test_lambda_params_backward_matches_autograd():
    H, dim = 3, 5
    vecs = [0.3 * rand(H, dim, seed=91 + i) for i in range(4)]
    dl = np.array([0.5, -1.25, 2.0])
    res = O.lambda_params_bwd(*vecs, dl)
    ts = [x.double().requires_grad_(True) for x in vecs]
    lam = torch.exp((ts[0] * ts[1]).sum(1)) - torch.exp((ts[2] * ts[3]).sum(1)) + 0.2
    (lam * torch.tensor(dl)).sum().backward()
    for name, t in zip(("dlq1", "dlk1", "dlq2", "dlk2"), ts):
        assert np.abs(res[name] - t.grad.numpy()).max() < 1e-14, name


def test_oproj_is_the_flattened_pairs_times_o_w():
    """Output projection ([L] "V1 vs V2", step 5).  With O_W the identity the
    result is each token's pair rows laid end to end in pair order; with a
    0/1 matrix that picks feature sel[j] into column j, column j holds that
    feature (a transposed O_W or another flattening order fails both)."""
    Bn, N, Hq, Hkv, d = 2, 9, 6, 1, 4
    x = I.v2_inputs(Bn, N, Hq, Hkv, d, seed=41, dtype=torch.float32)
    P = Hq // 2
    toks = np.array([0, 5, 9, 17])
    rows = O.v2_rows(x["q"], x["k"], x["v"], x["lam"], np.arange(Bn * N * P), causal=True)
    per_tok = rows.reshape(Bn * N, P * d)
    ident = np.eye(P * d, dtype=np.float32)
    got = O.v2_oproj_rows(x["q"], x["k"], x["v"], x["lam"], ident, toks, causal=True)
    np.testing.assert_allclose(got, per_tok[toks], rtol=0, atol=1e-15)
    sel = np.random.default_rng(42).integers(0, P * d, 7)   # 7 output columns
    pick = np.zeros((P * d, sel.size), dtype=np.float32)
    pick[sel, np.arange(sel.size)] = 1.0
    got = O.v2_oproj_rows(x["q"], x["k"], x["v"], x["lam"], pick, toks, causal=True)
    for j, f in enumerate(sel):
        p_, c_ = divmod(int(f), d)   # feature f = pair p_, channel c_
        want = rows.reshape(Bn * N, P, d)[toks, p_, c_]
        np.testing.assert_allclose(got[:, j], want, rtol=0, atol=1e-15)
