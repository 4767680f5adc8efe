"""Out-of-bounds writes: every output (and every workspace) is a view into a
larger buffer whose guard regions before and after it hold a sentinel bit
pattern; after the call the guards must be bit-for-bit unchanged.  Covers
the prefill (both forms, ragged lengths, windows), decode (both forms,
ragged cache lengths, the workspace-free entry point), the output
projection and the backward pass; the results themselves are checked
against the oracle elsewhere, here only that they are finite."""
import numpy as np
import pytest
import torch

from differential_attention_sm_b200 import inputs as I
from parity import assert_status_ok, status_word

pytestmark = pytest.mark.gpu

GUARD_BYTES = 64 * 1024   # each side; a multiple of 16 so the view stays aligned
SENTINEL = {torch.bfloat16: (torch.int16, 0x7FA5), torch.float32: (torch.int32, 0x7FC0DEAD),
            torch.uint8: (torch.uint8, 0xA5)}


@pytest.fixture(scope="module")
def B():
    from differential_attention_sm_b200 import binding
    binding.load()
    return binding


class Guarded:
    """A device tensor of `shape` inside a buffer with sentinel guards."""

    def __init__(self, shape, dtype):
        esz = torch.empty(0, dtype=dtype).element_size()
        self.g = GUARD_BYTES // esz
        n = int(np.prod(shape)) if len(shape) else 1
        self.buf = torch.empty(n + 2 * self.g, dtype=dtype, device="cuda")
        itype, pat = SENTINEL[dtype]
        if itype.is_signed and pat >= 2 ** (8 * esz - 1):
            pat -= 2 ** (8 * esz)
        self.buf.view(itype).fill_(pat)
        self.before = self.buf[:self.g].clone()
        self.after = self.buf[self.g + n:].clone()
        self.t = self.buf[self.g:self.g + n].view(shape)

    def check(self, what):
        torch.cuda.synchronize()
        n = self.t.numel()
        assert torch.equal(self.buf[:self.g].view(torch.uint8), self.before.view(torch.uint8)), (
            "%s: write before the output" % what)
        assert torch.equal(self.buf[self.g + n:].view(torch.uint8),
                           self.after.view(torch.uint8)), "%s: write past the output" % what
        if self.t.dtype != torch.uint8:
            assert torch.isfinite(self.t.float()).all(), "%s: non-finite output" % what


def ws(nbytes):
    return Guarded((max(int(nbytes), 16),), torch.uint8)


@pytest.mark.parametrize("Bn,N,H,window", [(2, 300, 3, 0), (1, 129, 2, 0), (1, 1, 1, 0),
                                           (2, 777, 2, 200)])
def test_v1_prefill_guards(B, Bn, N, H, window):
    x = I.v1_inputs(Bn, N, H, 64, 128, seed=2000 + N)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    lam = torch.linspace(0.3, 0.7, H, device="cuda")
    o = Guarded((Bn, N, H, 128), torch.bfloat16)
    st = status_word()
    B.diffattn_v1_fwd_window(q, k, v, lam, window, causal=True, apply_norm=True,
                             lambda_init=0.4, out=o.t, dev_status=st)
    assert_status_ok(st)
    o.check("v1 prefill N=%d" % N)
    # fp32 and other widths: the CUDA-core kernel
    x = I.v1_inputs(Bn, N, H, 8, 16, seed=2100 + N, dtype=torch.float32)
    o = Guarded((Bn, N, H, 16), torch.float32)
    B.diffattn_v1_fwd_window(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(), lam, window,
                             causal=True, out=o.t)
    o.check("v1 generic N=%d" % N)


@pytest.mark.parametrize("Bn,N,Hq,Hkv,window", [(2, 333, 8, 2, 0), (1, 190, 4, 1, 0),
                                                (1, 1000, 8, 2, 300)])
def test_v2_prefill_guards(B, Bn, N, Hq, Hkv, window):
    x = I.v2_inputs(Bn, N, Hq, Hkv, 128, seed=2200 + N)
    q, k, v, lam = (x[n].cuda() for n in ("q", "k", "v", "lam"))
    o = Guarded((Bn, N, Hq // 2, 128), torch.bfloat16)
    st = status_word()
    B.diffattn_v2_prefill_window(q, k, v, lam, window, causal=True, out=o.t, dev_status=st)
    assert_status_ok(st)
    o.check("v2 prefill N=%d" % N)


@pytest.mark.parametrize("Bn,L,Hq,Hkv,lens,window", [
    (3, 1000, 16, 2, [1000, 1, 517], 0),
    (2, 777, 12, 2, None, 0),
    (2, 3000, 8, 2, [3000, 2999], 1000),
])
def test_v2_decode_guards(B, Bn, L, Hq, Hkv, lens, window):
    x = I.v2_decode_inputs(Bn, L, Hq, Hkv, 128, seed=2300 + L)
    q, kc, vc, lam = (x[n].cuda() for n in ("q", "k_cache", "v_cache", "lam"))
    ln = None if lens is None else torch.tensor(lens, dtype=torch.int32, device="cuda")
    span = min(window, L) if window else L
    w = ws(B.diffattn_v2_decode_workspace_size(Bn, Hq, Hkv, 128, span))
    o = Guarded((Bn, Hq // 2, 128), torch.bfloat16)
    st = status_word()
    B.diffattn_v2_decode_window(q, kc, vc, lam, window, cache_lens=ln, workspace=w.t, out=o.t,
                                dev_status=st)
    assert_status_ok(st)
    o.check("v2 decode L=%d" % L)
    w.check("v2 decode workspace L=%d" % L)
    if window == 0 and Hq // Hkv in (2, 4, 6, 8):
        o = Guarded((Bn, Hq // 2, 128), torch.bfloat16)
        B.diffattn_v2_decode_noalloc(q, kc, vc, lam, cache_lens=ln, out=o.t, dev_status=st)
        assert_status_ok(st)
        o.check("v2 decode noalloc L=%d" % L)


@pytest.mark.parametrize("Bn,L,H,lens,window", [(2, 1000, 3, [1000, 1], 0),
                                                 (3, 555, 2, None, 100)])
def test_v1_decode_guards(B, Bn, L, H, lens, window):
    x = I.v1_decode_inputs(Bn, L, H, 64, 128, seed=2400 + L)
    q, kc, vc = (x[n].cuda() for n in ("q", "k_cache", "v_cache"))
    lam = torch.linspace(0.2, 0.8, H, device="cuda")
    ln = None if lens is None else torch.tensor(lens, dtype=torch.int32, device="cuda")
    span = min(window, L) if window else L
    w = ws(B.diffattn_v1_decode_workspace_size(Bn, H, 64, 128, span))
    o = Guarded((Bn, H, 128), torch.bfloat16)
    B.diffattn_v1_decode_window(q, kc, vc, lam, window, cache_lens=ln, apply_norm=True,
                                lambda_init=0.3, workspace=w.t, out=o.t)
    o.check("v1 decode L=%d" % L)
    w.check("v1 decode workspace L=%d" % L)


def test_oproj_guards(B):
    Bn, N, Hq, Hkv, dm = 2, 300, 8, 2, 192
    x = I.v2_inputs(Bn, N, Hq, Hkv, 128, seed=2500)
    W = (torch.randn(Hq // 2 * 128, dm, generator=torch.Generator().manual_seed(1)) /
         (Hq // 2 * 128) ** 0.5).to(torch.bfloat16).cuda()
    w = ws(B.diffattn_v2_prefill_oproj_workspace_size(Bn, N, Hq, 128))
    o = Guarded((Bn, N, dm), torch.bfloat16)
    st = status_word()
    B.diffattn_v2_prefill_oproj(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(), x["lam"].cuda(), W,
                                workspace=w.t, out=o.t, dev_status=st)
    assert_status_ok(st)
    o.check("oproj out")
    w.check("oproj workspace")


@pytest.mark.parametrize("form,N", [("v1", 200), ("v1", 333), ("v2", 257)])
def test_backward_guards(B, form, N):
    if form == "v1":
        Bn, H = 1, 2
        x = I.v1_inputs(Bn, N, H, 64, 128, seed=2600 + N)
        q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
        dout = I.v1_inputs(Bn, N, H, 64, 128, seed=2700 + N)["v"].cuda()
        lam = torch.tensor([0.6, -0.3], device="cuda")
        g = {"dq": Guarded(q.shape, torch.float32), "dk": Guarded(k.shape, torch.float32),
             "dv": Guarded(v.shape, torch.float32), "dlambda": Guarded((H,), torch.float32),
             "dnorm_weight": Guarded((128,), torch.float32)}
        w = ws(B.diffattn_v1_bwd_workspace_size(Bn, N, H, 64, 128))
        st = status_word()
        B.diffattn_v1_bwd(q, k, v, dout, lam, causal=True, apply_norm=True, lambda_init=0.4,
                          workspace=w.t, out={n: t.t for n, t in g.items()}, dev_status=st)
    else:
        Bn, Hq, Hkv = 1, 8, 2
        x = I.v2_inputs(Bn, N, Hq, Hkv, 128, seed=2800 + N)
        q, k, v, lam = (x[n].cuda() for n in ("q", "k", "v", "lam"))
        dout = torch.randn(Bn, N, Hq // 2, 128, generator=torch.Generator().manual_seed(N)).to(
            torch.bfloat16).cuda()
        g = {"dq": Guarded(q.shape, torch.float32), "dk": Guarded(k.shape, torch.float32),
             "dv": Guarded(v.shape, torch.float32), "dlambda": Guarded((Hq // 2,), torch.float32)}
        w = ws(B.diffattn_v2_bwd_workspace_size(Bn, N, Hq, Hkv, 128))
        st = status_word()
        B.diffattn_v2_bwd(q, k, v, dout, lam, causal=True, workspace=w.t,
                          out={n: t.t for n, t in g.items()}, dev_status=st)
    assert_status_ok(st)
    for name, t in g.items():
        t.check("%s backward %s" % (form, name))
    w.check("%s backward workspace" % form)
