"""GPU parity of the backward pass against the fp64 oracle backward (itself
pinned to float64 autograd and finite differences): dq, dk, dv, dlambda and,
for V1 with the norm, the norm gain's gradient; both forms, causal,
non-causal and sliding-window masks, ragged lengths, GQA, the lambda
re-parameterisation, and one full-size V1 head (batch 4, 16 heads, 4096)."""
import numpy as np
import pytest
import torch

import oracle as O
from differential_attention_sm_b200 import inputs as I
from parity import assert_status_ok, status_word

pytestmark = pytest.mark.gpu

# bf16 operands (maps and dS rounded to bf16, fp32 accumulation): the same
# relative bounds as the bf16 forward outputs, on |gpu - ref| / max|ref|.
TOL_MAX, TOL_MEAN = 2e-2, 2e-3


@pytest.fixture(scope="module")
def B():
    from differential_attention_sm_b200 import binding
    binding.load()
    return binding


def cuda(t):
    return t.cuda().contiguous()


def close(got, ref, what):
    g = got.detach().double().cpu().numpy() if isinstance(got, torch.Tensor) else np.asarray(got)
    r = np.asarray(ref, np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.isfinite(g).all(), what
    scale = np.abs(r).max()
    err = np.abs(g - r) / scale
    assert err.max() <= TOL_MAX, (what, err.max(), err.mean())
    # dlambda and the gain gradient are a handful of values, each a reduction
    # over N x dv products of bf16-rounded operands with cancellation: the
    # mean bound applies to the element-wise gradients only
    if r.size > 256:
        assert err.mean() <= TOL_MEAN, (what, err.max(), err.mean())


@pytest.mark.parametrize("N,causal,window,norm", [(300, True, 0, True), (256, False, 0, False),
                                                  (333, True, 70, True), (129, True, 0, False)])
def test_v1_backward(B, N, causal, window, norm):
    Bn, H, d, dv, layer = 2, 3, 64, 128, 12
    x = I.v1_inputs(Bn, N, H, d, dv, seed=1100 + N)
    dout = I.v1_inputs(Bn, N, H, d, dv, seed=1200 + N)["v"]
    lam_dev = B.lambda_from_params(*(cuda(x[n]) for n in ("lq1", "lk1", "lq2", "lk2")), layer)
    lam = O.lambda_from_params(x["lq1"], x["lk1"], x["lq2"], x["lk2"], layer)
    li = O.lambda_init(layer)
    g = (1.0 + 0.2 * torch.randn(dv, generator=torch.Generator().manual_seed(5))).float()
    st = status_word()
    res = B.diffattn_v1_bwd(cuda(x["q"]), cuda(x["k"]), cuda(x["v"]), cuda(dout), lam_dev,
                            causal=causal, window=window, apply_norm=norm,
                            norm_weight=cuda(g) if norm else None, lambda_init=li,
                            dev_status=st)
    assert_status_ok(st)
    ref = O.v1_bwd(x["q"], x["k"], x["v"], dout, lam, causal=causal, window=window,
                   apply_norm=norm, norm_weight=g if norm else None, lambda_init_value=li)
    for name in ("dq", "dk", "dv", "dlambda"):
        close(res[name], ref[name], "v1 %s N=%d" % (name, N))
    if norm:
        close(res["dnorm_weight"], ref["dnorm_weight"], "v1 dnorm_weight")
    # lambda re-parameterisation: same dlambda into both sides
    dl = res["dlambda"]
    gp = B.lambda_from_params_bwd(*(cuda(x[n]) for n in ("lq1", "lk1", "lq2", "lk2")), dl)
    rp = O.lambda_params_bwd(x["lq1"], x["lk1"], x["lq2"], x["lk2"], dl.double().cpu().numpy())
    for n in ("dlq1", "dlk1", "dlq2", "dlk2"):
        assert np.abs(gp[n].double().cpu().numpy() - rp[n]).max() <= 1e-5 * max(1.0, np.abs(rp[n]).max())


@pytest.mark.parametrize("N,Hq,Hkv,causal,window", [(520, 8, 2, True, 0), (300, 8, 4, False, 0),
                                                     (400, 16, 2, True, 100)])
def test_v2_backward(B, N, Hq, Hkv, causal, window):
    Bn, d = 1, 128
    x = I.v2_inputs(Bn, N, Hq, Hkv, d, seed=1300 + N)
    dout = I.v2_inputs(Bn, N, Hq, Hkv, d, seed=1400 + N)["q"][:, :, : Hq // 2].contiguous()
    st = status_word()
    res = B.diffattn_v2_bwd(cuda(x["q"]), cuda(x["k"]), cuda(x["v"]), cuda(dout),
                            cuda(x["lam"]), causal=causal, window=window, dev_status=st)
    assert_status_ok(st)
    ref = O.v2_bwd(x["q"], x["k"], x["v"], dout, x["lam"], causal=causal, window=window)
    for name in ("dq", "dk", "dv", "dlambda"):
        close(res[name], ref[name], "v2 %s N=%d" % (name, N))


def test_backward_other_widths_materialised_path(B):
    """Widths outside the tensor-core forward run the materialising path."""
    Bn, N, H, d, dv = 2, 200, 2, 32, 64
    x = I.v1_inputs(Bn, N, H, d, dv, seed=1500)
    dout = I.v1_inputs(Bn, N, H, d, dv, seed=1501)["v"]
    lam = torch.tensor([0.7, -0.2])
    res = B.diffattn_v1_bwd(cuda(x["q"]), cuda(x["k"]), cuda(x["v"]), cuda(dout), cuda(lam),
                            causal=True, apply_norm=True, lambda_init=0.3)
    ref = O.v1_bwd(x["q"], x["k"], x["v"], dout, lam.double().numpy(), causal=True,
                   apply_norm=True, lambda_init_value=0.3)
    for name in ("dq", "dk", "dv", "dlambda", "dnorm_weight"):
        close(res[name], ref[name], "v1 d32 %s" % name)
    x = I.v2_inputs(1, 150, 8, 2, 64, seed=1502)
    dout = I.v2_inputs(1, 150, 8, 2, 64, seed=1503)["q"][:, :, :4].contiguous()
    res = B.diffattn_v2_bwd(cuda(x["q"]), cuda(x["k"]), cuda(x["v"]), cuda(dout),
                            cuda(x["lam"]), causal=True, window=40)
    ref = O.v2_bwd(x["q"], x["k"], x["v"], dout, x["lam"], causal=True, window=40)
    for name in ("dq", "dk", "dv", "dlambda"):
        close(res[name], ref[name], "v2 d64 %s" % name)


def test_v1_backward_full_size_one_head(B):
    """The benchmark's V1 shape (batch 4, 16 heads, 4096, causal, norm): the
    gradients of one (batch, head) unit depend on that unit alone, so the
    oracle runs on its slice."""
    w = I.WORKLOADS["v1_prefill_bf16"]
    x = I.v1_inputs(w.B, w.N, w.H, w.d, w.dv, w.seed)
    dout = I.v1_inputs(w.B, w.N, w.H, w.d, w.dv, w.seed + 77)["v"]
    lam_dev = B.lambda_from_params(*(cuda(x[n]) for n in ("lq1", "lk1", "lq2", "lk2")), w.layer)
    lam = O.lambda_from_params(x["lq1"], x["lk1"], x["lq2"], x["lk2"], w.layer)
    li = O.lambda_init(w.layer)
    res = B.diffattn_v1_bwd(cuda(x["q"]), cuda(x["k"]), cuda(x["v"]), cuda(dout), lam_dev,
                            causal=True, apply_norm=True, norm_eps=w.eps, lambda_init=li)
    b, h = 2, 11
    sl = lambda t: t[b:b + 1, :, h:h + 1].contiguous()
    ref = O.v1_bwd(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(dout), lam[h:h + 1], causal=True,
                   apply_norm=True, eps=w.eps, lambda_init_value=li)
    for name in ("dq", "dk", "dv"):
        close(res[name][b:b + 1, :, h:h + 1], ref[name], "v1 full %s" % name)


def test_v2_backward_full_size_one_pair(B):
    """The V2 prefill shape (batch 2, 32 query heads on 8 KV heads, 8192,
    causal): dQ of one head pair depends on that pair alone, so the oracle
    runs on its slice (both pairs of the group stay in the slice, since dK
    and dV sum over them)."""
    w = I.WORKLOADS["v2_prefill_bf16"]
    x = I.v2_inputs(w.B, w.N, w.Hq, w.Hkv, w.d, w.seed)
    dout = I.v2_inputs(w.B, w.N, w.Hq, w.Hkv, w.d, w.seed + 77)["q"][:, :, : w.Hq // 2].contiguous()
    st = status_word()
    res = B.diffattn_v2_bwd(cuda(x["q"]), cuda(x["k"]), cuda(x["v"]), cuda(dout), cuda(x["lam"]),
                            causal=True, dev_status=st)
    assert_status_ok(st)
    # batch 1, KV head 5: query heads 20..23 (pairs 10, 11); a 2048-token prefix
    # keeps the oracle in seconds (causal: rows < n depend on keys < n only)
    b, g, n = 1, 5, 2048
    qs = x["q"][b:b + 1, :n, 4 * g:4 * g + 4].contiguous()
    ks = x["k"][b:b + 1, :n, g:g + 1].contiguous()
    vs = x["v"][b:b + 1, :n, g:g + 1].contiguous()
    ds = dout[b:b + 1, :n, 2 * g:2 * g + 2].contiguous()
    ref = O.v2_bwd(qs, ks, vs, ds, x["lam"][2 * g:2 * g + 2], causal=True)
    close(res["dq"][b:b + 1, :n, 4 * g:4 * g + 4], ref["dq"], "v2 full dq")


# ---------------------------------------------------------------------------
# training forward with saves, and the backward from the saves
# ---------------------------------------------------------------------------
def same_up_to_rounding(a, b, what):
    """The training forward is a separate instantiation of the forward kernel
    (it also writes the saves), compiled on its own, so its bf16 output may
    differ from the plain forward's by a rounding step: within one bf16 unit
    in the last place of the largest output, everywhere."""
    d = (a.float() - b.float()).abs().max().item()
    assert d <= b.float().abs().max().item() * 2.0 ** -7, (what, d)
@pytest.mark.parametrize("N,causal,window,norm", [(300, True, 0, True), (200, False, 0, False),
                                                  (333, True, 70, True)])
def test_v1_train_forward_and_saved_backward(B, N, causal, window, norm):
    """The training forward's output matches the plain forward's (up to a
    bf16 rounding step) and the oracle's; the backward from its saves equals
    the self-contained backward (and the oracle backward).  dq, dk, dv come from the same kernels on the
    same saves, so they are compared bit for bit; dlambda and the gain
    gradient are block reductions with atomic adds, so within rounding."""
    Bn, H, d, dv, layer = 2, 3, 64, 128, 12
    x = I.v1_inputs(Bn, N, H, d, dv, seed=1400 + N)
    dout = cuda(I.v1_inputs(Bn, N, H, d, dv, seed=1500 + N)["v"])
    q, k, v = cuda(x["q"]), cuda(x["k"]), cuda(x["v"])
    lam_dev = B.lambda_from_params(*(cuda(x[n]) for n in ("lq1", "lk1", "lq2", "lk2")), layer)
    lam = O.lambda_from_params(x["lq1"], x["lk1"], x["lq2"], x["lk2"], layer)
    li = O.lambda_init(layer)
    g = (1.0 + 0.2 * torch.randn(dv, generator=torch.Generator().manual_seed(6))).float()
    kw = dict(causal=causal, window=window, apply_norm=norm,
              norm_weight=cuda(g) if norm else None, lambda_init=li)
    st = status_word()
    out, saves = B.diffattn_v1_fwd_train(q, k, v, lam_dev, dev_status=st, **kw)
    assert_status_ok(st)
    plain = B.diffattn_v1_fwd_window(q, k, v, lam_dev, window,
                                     **{n: a for n, a in kw.items() if n != "window"})
    same_up_to_rounding(out, plain, "v1 training forward vs forward")
    ref_o = O.v1_rows(x["q"], x["k"], x["v"], lam, np.arange(Bn * N * H), causal=causal,
                      window=window, apply_norm=norm, norm_weight=g if norm else None,
                      lambda_init_value=li)
    close(out.reshape(-1, dv), ref_o, "v1 training forward")
    res = B.diffattn_v1_bwd_saved(q, k, v, dout, lam_dev, saves, dev_status=st, **kw)
    assert_status_ok(st)
    full = B.diffattn_v1_bwd(q, k, v, dout, lam_dev, **kw)
    for name in ("dq", "dk", "dv"):
        assert torch.equal(res[name], full[name]), name
    ref = O.v1_bwd(x["q"], x["k"], x["v"], dout.cpu(), lam, causal=causal, window=window,
                   apply_norm=norm, norm_weight=g if norm else None, lambda_init_value=li)
    for name in ("dq", "dk", "dv", "dlambda") + (("dnorm_weight",) if norm else ()):
        close(res[name], ref[name], "v1 saved %s N=%d" % (name, N))


@pytest.mark.parametrize("N,Hq,Hkv,causal,window", [(520, 8, 2, True, 0), (300, 8, 4, False, 0),
                                                     (400, 16, 2, True, 100)])
def test_v2_train_forward_and_saved_backward(B, N, Hq, Hkv, causal, window):
    Bn, d = 1, 128
    x = I.v2_inputs(Bn, N, Hq, Hkv, d, seed=1600 + N)
    dout = torch.randn(Bn, N, Hq // 2, d, generator=torch.Generator().manual_seed(N)).to(
        torch.bfloat16)
    q, k, v, lam = (cuda(x[n]) for n in ("q", "k", "v", "lam"))
    st = status_word()
    out, saves = B.diffattn_v2_prefill_train(q, k, v, lam, causal=causal, window=window,
                                             dev_status=st)
    assert_status_ok(st)
    plain = B.diffattn_v2_prefill_window(q, k, v, lam, window, causal=causal)
    same_up_to_rounding(out, plain, "v2 training forward vs forward")
    ref_o = O.v2_rows(x["q"], x["k"], x["v"], x["lam"], np.arange(Bn * N * Hq // 2),
                      causal=causal, window=window)
    close(out.reshape(-1, d), ref_o, "v2 training forward")
    res = B.diffattn_v2_bwd_saved(q, k, v, cuda(dout), lam, saves, causal=causal, window=window,
                                  dev_status=st)
    assert_status_ok(st)
    full = B.diffattn_v2_bwd(q, k, v, cuda(dout), lam, causal=causal, window=window)
    for name in ("dq", "dk", "dv"):
        assert torch.equal(res[name], full[name]), name
    ref = O.v2_bwd(x["q"], x["k"], x["v"], dout, x["lam"], causal=causal, window=window)
    for name in ("dq", "dk", "dv", "dlambda"):
        close(res[name], ref[name], "v2 saved %s N=%d" % (name, N))
