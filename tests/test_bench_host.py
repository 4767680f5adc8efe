"""Host-side pieces of bench.py, on the CPU: the algorithmic work formulas
against brute-force counts, and the bounded oracle samplers that give each
secondary workload its CPU baseline."""
import numpy as np
import torch

import bench
import oracle as O
from differential_attention_sm_b200 import inputs as I


def test_pair_counts_match_brute_force():
    for N, W in ((1, 1), (7, 3), (130, 128), (300, 1000)):
        mask = np.tril(np.ones((N, N), bool))
        assert bench.prefill_pairs(2, N, 3) == 2 * 3 * mask.sum()
        band = mask & (np.arange(N)[:, None] - np.arange(N)[None, :] < W)
        assert bench.window_pairs(2, N, 3, W) == 2 * 3 * band.sum()
    assert bench.v1_flops_per_pair(64, 128) == 768
    assert bench.v2_flops_per_pair(128) == 1024
    assert bench.v1_bwd_flops_per_pair(64, 128) == 1792


def test_decode_bytes():
    # K and V of every cached entry once, plus q and the output, in bf16
    assert bench.v2_decode_bytes(64, 32768, 8, 128, 64) == (
        64 * 32768 * 8 * 128 * 2 * 2 + 64 * 64 * 128 * 2 + 64 * 32 * 128 * 2)
    assert bench.v1_decode_bytes(64, 32768, 32, 64, 128) == (
        64 * 32768 * 32 * 256 * 2 + 64 * 32 * 128 * 2 + 64 * 32 * 128 * 2)


def test_oracle_samplers_run_and_count_work():
    x = I.v2_inputs(1, 64, 4, 2, 16, seed=1, dtype=torch.float32)
    P = 2
    run = bench._rows_sampler(
        lambda r: O.v2_rows(x["q"], x["k"], x["v"], x["lam"], r, causal=True),
        64 * P, lambda r: ((r // P) % 64 + 1) * bench.v2_flops_per_pair(16), 3)
    res = bench.oracle_rate(run, 0.05, 1e9, "rows")
    assert res["value"] > 0 and res["kind"] == "oracle" and res["cores"] >= 1
    d = I.v2_decode_inputs(3, 50, 4, 2, 16, seed=2, dtype=torch.float32)
    runs = bench._decode_sampler(
        lambda b, k, v: O.v2_decode_rows(d["q"][b:b + 1], k[None], v[None], d["lam"],
                                         np.arange(P)),
        (d["k_cache"], d["v_cache"]), 3, bench.v2_decode_bytes(1, 50, 2, 16, 4), 4)
    assert runs(2) == 2 * bench.v2_decode_bytes(1, 50, 2, 16, 4)


def test_kernel_hash_ignores_comments_only():
    """The hash that keys the recorded DRAM traffic changes with the code and
    not with comments or blank lines."""
    code = "int a = 1;  // one\n/* block\n comment */\nint b = a + 2;\n\n"
    same = "// header\nint a = 1;\n\nint b = a + 2;  /* two */\n"
    other = "int a = 1;\nint b = a + 3;\n"
    strip = bench.code_without_comments
    assert strip(code) == strip(same) == "int a = 1;\nint b = a + 2;"
    assert strip(other) != strip(code)
    assert len(bench.kernel_source_hash()) == 16
