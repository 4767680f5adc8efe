"""GPU parity at the full sizes of the five workloads, in the launch
configuration the benchmark times, against the fp64 oracle:

  * V1 causal prefill (batch 4, 16 heads, 4096 tokens) and V2 causal prefill
    (batch 2, 32 query heads, 8 KV heads, 8192 tokens): every output row;
  * V1 long-context prefill (16 heads, 32768 tokens, planted signal): one
    random row and the last row of every (batch, head, 128-row query tile),
    and the two rows the signal was planted for in every head, so that each
    tile the scheduler hands out is checked;
  * V2 decode (batch 64, cache 32768, 64 query heads, 8 KV heads) and V1
    decode (batch 64, cache 32768, 32 heads): every batch entry, each
    entry's cache slice copied to the host in turn.

Each test records the error it reached and the oracle's time and thread
count (``parity.record``; written when DA_PARITY_REPORT names a file)."""
import time

import numpy as np
import pytest
import torch

import oracle as O
from differential_attention_sm_b200 import inputs as I
from parity import assert_bf16_close, assert_status_ok, errors, record, status_word

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from differential_attention_sm_b200 import binding
    binding.load()
    return binding


def cuda(t):
    return t.cuda().contiguous()


def timed_oracle(fn, *a, **kw):
    t0 = time.perf_counter()
    r = fn(*a, **kw)
    return r, time.perf_counter() - t0


def tile_rows(Bn, N, H, seed):
    """Rows (b*N + i)*H + h: for every (b, h, 128-row tile) its last row and
    one random row inside it."""
    rng = np.random.default_rng(seed)
    n_t = (N + 127) // 128
    rows = []
    for b in range(Bn):
        for h in range(H):
            for t in range(n_t):
                lo, hi = 128 * t, min(N, 128 * t + 128)
                for i in (hi - 1, int(rng.integers(lo, hi))):
                    rows.append((b * N + i) * H + h)
    return np.unique(np.array(rows, dtype=np.int64))


def test_v1_prefill_every_row(B):
    w = I.WORKLOADS["v1_prefill_bf16"]
    x = I.v1_inputs(w.B, w.N, w.H, w.d, w.dv, w.seed)
    lam_dev = B.lambda_from_params(*(cuda(x[n]) for n in ("lq1", "lk1", "lq2", "lk2")), w.layer)
    lam_host = O.lambda_from_params(x["lq1"], x["lk1"], x["lq2"], x["lk2"], w.layer)
    li = O.lambda_init(w.layer)
    st = status_word()
    out = B.diffattn_v1_fwd(cuda(x["q"]), cuda(x["k"]), cuda(x["v"]), lam_dev, causal=True,
                            apply_norm=True, norm_eps=w.eps, lambda_init=li, dev_status=st)
    assert_status_ok(st)
    rows = np.arange(w.B * w.N * w.H)
    ref, secs = timed_oracle(O.v1_rows, x["q"], x["k"], x["v"], lam_host, rows, causal=True,
                             apply_norm=True, eps=w.eps, lambda_init_value=li)
    mx, mean = assert_bf16_close(out.reshape(-1, w.dv), ref, False, w.name)
    record(w.name, max_err=mx, mean_err=mean, form="abs", rows=int(rows.size),
           rows_total=int(rows.size), oracle_s=secs, oracle_threads=O.n_threads())


def test_v2_prefill_every_row(B):
    w = I.WORKLOADS["v2_prefill_bf16"]
    x = I.v2_inputs(w.B, w.N, w.Hq, w.Hkv, w.d, w.seed)
    st = status_word()
    out = B.diffattn_v2_prefill(cuda(x["q"]), cuda(x["k"]), cuda(x["v"]), cuda(x["lam"]),
                                causal=True, dev_status=st)
    assert_status_ok(st)
    rows = np.arange(w.B * w.N * (w.Hq // 2))
    ref, secs = timed_oracle(O.v2_rows, x["q"], x["k"], x["v"], x["lam"], rows, causal=True)
    mx, mean = assert_bf16_close(out.reshape(-1, w.d), ref, True, w.name)
    record(w.name, max_err=mx, mean_err=mean, form="rel_to_max", rows=int(rows.size),
           rows_total=int(rows.size), oracle_s=secs, oracle_threads=O.n_threads())


def test_v1_long_every_query_tile(B):
    w = I.WORKLOADS["v1_long_bf16"]
    x = I.v1_inputs(w.B, w.N, w.H, w.d, w.dv, w.seed, planted=w.planted)
    lam_dev = B.lambda_from_params(*(cuda(x[n]) for n in ("lq1", "lk1", "lq2", "lk2")), w.layer)
    lam_host = O.lambda_from_params(x["lq1"], x["lk1"], x["lq2"], x["lk2"], w.layer)
    li = O.lambda_init(w.layer)
    st = status_word()
    out = B.diffattn_v1_fwd(cuda(x["q"]), cuda(x["k"]), cuda(x["v"]), lam_dev, causal=True,
                            apply_norm=True, norm_eps=w.eps, lambda_init=li, dev_status=st)
    assert_status_ok(st)
    planted = [(b * w.N + i) * w.H + h for b in range(w.B) for i in (w.N - 2, w.N - 1)
               for h in range(w.H)]
    rows = np.unique(np.concatenate([tile_rows(w.B, w.N, w.H, w.seed), np.array(planted)]))
    # every (batch, head, tile) is represented
    tiles = {((r // w.H) // w.N, r % w.H, ((r // w.H) % w.N) // 128) for r in rows.tolist()}
    assert len(tiles) == w.B * w.H * ((w.N + 127) // 128)
    ref, secs = timed_oracle(O.v1_rows, x["q"], x["k"], x["v"], lam_host, rows, causal=True,
                             apply_norm=True, eps=w.eps, lambda_init_value=li)
    got = out.reshape(-1, w.dv)[torch.from_numpy(rows).cuda()]
    mx, mean = assert_bf16_close(got, ref, False, w.name)
    record(w.name, max_err=mx, mean_err=mean, form="abs", rows=int(rows.size),
           rows_total=w.B * w.N * w.H, oracle_s=secs, oracle_threads=O.n_threads(),
           note="one random row and the last row of every (batch, head, 128-row tile), "
                "plus rows N-2 and N-1 of every head")


def _entry_by_entry(name, out, kc, vc, one_entry_ref, rel_to_max):
    """Compares every batch entry of a decode output with the oracle, copying
    that entry's cache slices to the host in turn."""
    worst, means, secs = 0.0, [], 0.0
    for b in range(out.shape[0]):
        k, v = kc[b].cpu(), vc[b].cpu()
        t0 = time.perf_counter()
        ref = one_entry_ref(b, k, v)
        secs += time.perf_counter() - t0
        mx, mean = assert_bf16_close(out[b], ref, rel_to_max, "%s b=%d" % (name, b))
        worst = max(worst, mx)
        means.append(mean)
    return worst, float(np.mean(means)), secs


def test_v2_decode_every_batch_entry(B):
    w = I.WORKLOADS["v2_decode_bf16"]
    x = I.v2_decode_inputs(w.B, w.L, w.Hq, w.Hkv, w.d, w.seed, fill_caches=False)
    kc = I.fill_normal_on_device(torch.empty(w.B, w.L, w.Hkv, w.d, dtype=torch.bfloat16,
                                             device="cuda"), w.seed * 2 + 1)
    vc = I.fill_normal_on_device(torch.empty_like(kc), w.seed * 2 + 2)
    st = status_word()
    out = B.diffattn_v2_decode(cuda(x["q"]), kc, vc, cuda(x["lam"]), dev_status=st)
    assert_status_ok(st)
    P = w.Hq // 2

    def ref(b, k, v):
        return O.v2_decode_rows(x["q"][b:b + 1], k[None], v[None], x["lam"], np.arange(P))

    mx, mean, secs = _entry_by_entry(w.name, out, kc, vc, ref, True)
    record(w.name, max_err=mx, mean_err=mean, form="rel_to_max (per batch entry)",
           rows=w.B * P, rows_total=w.B * P, oracle_s=secs, oracle_threads=O.n_threads(),
           note="caches filled from a seeded device generator")
    del kc, vc
    torch.cuda.empty_cache()


def test_v1_decode_every_batch_entry(B):
    w = I.WORKLOADS["v1_decode_bf16"]
    x = I.v1_decode_inputs(w.B, w.L, w.H, w.d, w.dv, w.seed, fill_caches=False)
    kc = I.fill_normal_on_device(torch.empty(w.B, w.L, w.H, 2 * w.d, dtype=torch.bfloat16,
                                             device="cuda"), w.seed * 2 + 3)
    vc = I.fill_normal_on_device(torch.empty(w.B, w.L, w.H, w.dv, dtype=torch.bfloat16,
                                             device="cuda"), w.seed * 2 + 4)
    lam_dev = B.lambda_from_params(*(cuda(x[n]) for n in ("lq1", "lk1", "lq2", "lk2")), w.layer)
    lam_host = O.lambda_from_params(x["lq1"], x["lk1"], x["lq2"], x["lk2"], w.layer)
    li = O.lambda_init(w.layer)
    out = B.diffattn_v1_decode(cuda(x["q"]), kc, vc, lam_dev, apply_norm=True, norm_eps=w.eps,
                               lambda_init=li)
    torch.cuda.synchronize()

    def ref(b, k, v):
        return O.v1_decode_rows(x["q"][b:b + 1], k[None], v[None], lam_host, np.arange(w.H),
                                apply_norm=True, eps=w.eps, lambda_init_value=li)

    mx, mean, secs = _entry_by_entry(w.name, out, kc, vc, ref, False)
    record(w.name, max_err=mx, mean_err=mean, form="abs", rows=w.B * w.H,
           rows_total=w.B * w.H, oracle_s=secs, oracle_threads=O.n_threads(),
           note="caches filled from a seeded device generator")
    del kc, vc
    torch.cuda.empty_cache()


@pytest.mark.parametrize("causal", [False, True])
def test_tiny_fp32_margin(B, causal):
    """The fp32 workload in full, with its error recorded next to the 1e-5
    bound (the CUDA-core kernel is built without fast-math)."""
    w = I.WORKLOADS["tiny_v1_fp32"]
    x = I.v1_inputs(w.B, w.N, w.H, w.d, w.dv, w.seed, dtype=torch.float32)
    lam_dev = torch.tensor([w.fixed_lambda], dtype=torch.float32, device="cuda")
    out = B.diffattn_v1_fwd(cuda(x["q"]), cuda(x["k"]), cuda(x["v"]), lam_dev, causal=causal)
    rows = np.arange(w.B * w.N * w.H)
    ref, secs = timed_oracle(O.v1_rows, x["q"], x["k"], x["v"], [w.fixed_lambda], rows,
                             causal=causal)
    mx, mean = errors(out.reshape(-1, w.dv), ref, False)
    assert mx <= 1e-5
    record("%s_%s" % (w.name, "causal" if causal else "noncausal"), max_err=mx, mean_err=mean,
           form="abs", rows=int(rows.size), rows_total=int(rows.size), oracle_s=secs,
           oracle_threads=O.n_threads(), bound=1e-5, margin=1e-5 / max(mx, 1e-30))
