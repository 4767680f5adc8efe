"""The seeded input recipe that the CUDA path and the oracle share: draw
order, bf16 rounding, per-entry decode caches, the planted signal and the
workload table (no GPU)."""
import torch

from differential_attention_sm_b200 import inputs as I


def _redraw_v1(B, N, H, d, dv, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, N, H, 2 * d, generator=g)
    k = torch.randn(B, N, H, 2 * d, generator=g)
    v = torch.randn(B, N, H, dv, generator=g)
    lvec = [0.1 * torch.randn(H, d, generator=g) for _ in range(4)]
    return q, k, v, lvec, g


def test_v1_draw_order_and_rounding():
    B, N, H, d, dv, seed = 2, 17, 3, 8, 16, 11
    x = I.v1_inputs(B, N, H, d, dv, seed)
    q, k, v, lvec, _ = _redraw_v1(B, N, H, d, dv, seed)
    for name, ref in (("q", q), ("k", k), ("v", v)):
        assert x[name].dtype == torch.bfloat16
        assert torch.equal(x[name], ref.to(torch.bfloat16)), name
    for name, ref in zip(("lq1", "lk1", "lq2", "lk2"), lvec):
        assert x[name].dtype == torch.float32
        assert torch.equal(x[name], ref), name
    # the same seed gives the same draws, another seed different ones
    assert torch.equal(I.v1_inputs(B, N, H, d, dv, seed)["k"], x["k"])
    assert not torch.equal(I.v1_inputs(B, N, H, d, dv, seed + 1)["k"], x["k"])


def test_v2_draw_order_and_lambda_range():
    B, N, Hq, Hkv, d, seed = 2, 9, 8, 2, 16, 12
    x = I.v2_inputs(B, N, Hq, Hkv, d, seed)
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, N, Hq, d, generator=g)
    k = torch.randn(B, N, Hkv, d, generator=g)
    v = torch.randn(B, N, Hkv, d, generator=g)
    lam = 0.2 + 0.6 * torch.rand(Hq // 2, generator=g)
    for name, ref in (("q", q), ("k", k), ("v", v)):
        assert torch.equal(x[name], ref.to(torch.bfloat16)), name
    assert torch.equal(x["lam"], lam)
    assert x["lam"].shape == (Hq // 2,)
    assert bool(((x["lam"] >= 0.2) & (x["lam"] <= 0.8)).all())


def test_decode_cache_entries_rebuild_one_at_a_time():
    B, L, Hq, Hkv, d, seed = 3, 40, 8, 2, 16, 7
    x = I.v2_decode_inputs(B, L, Hq, Hkv, d, seed)
    for b in range(B):
        kb, vb = I.decode_cache_slice(seed, b, L, Hkv, d, d)
        assert torch.equal(x["k_cache"][b], kb) and torch.equal(x["v_cache"][b], vb)
        g = torch.Generator().manual_seed(seed * 65536 + b)
        assert torch.equal(kb, torch.randn(L, Hkv, d, generator=g).to(torch.bfloat16))
        assert torch.equal(vb, torch.randn(L, Hkv, d, generator=g).to(torch.bfloat16))
    # distinct entries differ; the query and lambda come from the workload seed
    assert not torch.equal(x["k_cache"][0], x["k_cache"][1])
    y = I.v2_decode_inputs(B, L, Hq, Hkv, d, seed, fill_caches=False)
    assert torch.equal(y["q"], x["q"]) and torch.equal(y["lam"], x["lam"])
    z = I.v1_decode_inputs(2, L, 3, 8, 16, seed)
    kb, vb = I.decode_cache_slice(seed, 1, L, 3, 16, 16)
    assert torch.equal(z["k_cache"][1], kb) and torch.equal(z["v_cache"][1], vb)


def test_planted_signal_positions_and_keys():
    B, N, H, d, dv, seed, planted = 2, 64, 3, 8, 16, 13, 6
    x = I.v1_inputs(B, N, H, d, dv, seed, planted=planted)
    q, k, _, _, g = _redraw_v1(B, N, H, d, dv, seed)
    pos = x["planted_pos"]
    assert pos.shape == (B, H, planted)
    for b in range(B):
        for h in range(H):
            ref = torch.randperm(N - 2, generator=g)[:planted]
            assert torch.equal(pos[b, h], ref)
            p = pos[b, h].tolist()
            assert len(set(p)) == planted and max(p) < N - 2 and min(p) >= 0
            needle = (4.0 * (q[b, N - 2, h, :d] + q[b, N - 1, h, :d]) / 2.0).to(torch.bfloat16)
            for j in range(N):
                if j in p:   # branch-1 half replaced, branch-2 half untouched
                    assert torch.equal(x["k"][b, j, h, :d], needle)
                else:
                    assert torch.equal(x["k"][b, j, h, :d], k[b, j, h, :d].to(torch.bfloat16))
                assert torch.equal(x["k"][b, j, h, d:], k[b, j, h, d:].to(torch.bfloat16))


def test_workload_table():
    W = I.WORKLOADS
    assert (W["tiny_v1_fp32"].seed, W["v1_prefill_bf16"].seed, W["v1_long_bf16"].seed,
            W["v2_prefill_bf16"].seed, W["v2_decode_bf16"].seed) == (0, 1, 2, 3, 4)
    w = W["v1_prefill_bf16"]
    assert (w.B, w.N, w.H, w.d, w.dv, w.layer, w.causal) == (4, 4096, 16, 64, 128, 12, True)
    w = W["v1_long_bf16"]
    assert (w.B, w.N, w.H, w.layer, w.planted) == (1, 32768, 16, 24, 6)
    w = W["v2_prefill_bf16"]
    assert (w.B, w.N, w.Hq, w.Hkv, w.d) == (2, 8192, 32, 8, 128)
    w = W["v2_decode_bf16"]
    assert (w.B, w.L, w.Hq, w.Hkv, w.d) == (64, 32768, 64, 8, 128)
    w = W["tiny_v1_fp32"]
    assert w.dtype == torch.float32 and (w.N, w.d, w.dv, w.fixed_lambda) == (128, 8, 16, 0.8)
