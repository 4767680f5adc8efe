"""The C-ABI library builds, loads without a GPU, exports every symbol the
public header declares, and rejects bad arguments on the host before any
CUDA call (so these run on a machine with no device)."""
import ctypes
import math
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "diffattn.h")


@pytest.fixture(scope="module")
def lib():
    from differential_attention_sm_b200 import build as B
    B.build()
    from differential_attention_sm_b200 import binding
    return binding.load()


def declared_symbols():
    text = open(HEADER).read()
    return set(re.findall(r"DA_API\s+[\w\s\*]+?\b(\w+)\s*\(", text))


def test_header_declares_the_entry_points():
    syms = declared_symbols()
    for name in ("diffattn_v1_fwd", "diffattn_v2_prefill", "diffattn_v2_decode",
                 "lambda_from_params"):
        assert name in syms


def test_library_exports_every_declared_symbol(lib):
    from differential_attention_sm_b200 import binding
    syms = declared_symbols()
    assert syms == set(binding.EXPORTS)
    for name in syms:
        assert hasattr(lib, name), name


def test_lambda_init_and_status_strings(lib):
    from differential_attention_sm_b200 import binding as b
    assert b.diffattn_lambda_init(1) == pytest.approx(0.2, abs=1e-15)
    assert math.isnan(b.diffattn_lambda_init(0))
    import oracle
    for l in (1, 2, 12, 24, 100):
        assert b.diffattn_lambda_init(l) == pytest.approx(oracle.lambda_init(l), abs=1e-15)
    assert b.status_string(b.DA_OK) == "DA_OK"
    assert b.status_string(b.DA_ERR_DEVICE_TIMEOUT) == "DA_ERR_DEVICE_TIMEOUT"
    assert b.status_string(b.DA_ERR_SCHEDULE) == "DA_ERR_SCHEDULE"
    assert b.status_string(12345) == "DA_ERR_UNKNOWN"


# Fake device addresses: validation must reject before dereferencing anything.
A = 0x10000   # 16-byte aligned
U = 0x10008   # misaligned


def test_v1_fwd_host_validation(lib):
    from differential_attention_sm_b200 import binding as b
    f = lib.diffattn_v1_fwd
    ok = (A, A, A, A, b.DA_BF16, 1, 128, 1, 64, 128, A, 1, 1, None, 1e-5, 0.2, None, None)
    bad = list(ok); bad[0] = None
    assert f(*bad) == b.DA_ERR_INVALID_ARG
    bad = list(ok); bad[4] = 7
    assert f(*bad) == b.DA_ERR_INVALID_ARG
    bad = list(ok); bad[6] = 0
    assert f(*bad) == b.DA_ERR_INVALID_ARG
    bad = list(ok); bad[8] = 129
    assert f(*bad) == b.DA_ERR_UNSUPPORTED
    bad = list(ok); bad[1] = U
    assert f(*bad) == b.DA_ERR_ALIGNMENT
    bad = list(ok); bad[14] = -1.0
    assert f(*bad) == b.DA_ERR_INVALID_ARG


def test_v2_prefill_host_validation(lib):
    from differential_attention_sm_b200 import binding as b
    f = lib.diffattn_v2_prefill
    ok = [A, A, A, A, b.DA_BF16, 2, 256, 32, 8, 128, A, 1, None, None]
    bad = list(ok); bad[7] = 31          # odd query heads
    assert f(*bad) == b.DA_ERR_INVALID_ARG
    bad = list(ok); bad[7], bad[8] = 8, 8  # group 1: a pair would span two KV heads
    assert f(*bad) == b.DA_ERR_INVALID_ARG
    bad = list(ok); bad[3] = U
    assert f(*bad) == b.DA_ERR_ALIGNMENT
    bad = list(ok); bad[10] = None
    assert f(*bad) == b.DA_ERR_INVALID_ARG


def test_decode_workspace_and_validation(lib):
    from differential_attention_sm_b200 import binding as b
    ws = b.diffattn_v2_decode_workspace_size(64, 64, 8, 128, 32768)
    assert ws > 0 and ws % 16 == 0
    assert b.diffattn_v2_decode_workspace_size(64, 64, 8, 64, 32768) == 0   # generic path
    assert b.diffattn_v2_decode_workspace_size(0, 64, 8, 128, 32768) == 0
    assert b.diffattn_v1_decode_workspace_size(64, 32, 64, 128, 32768) > 0
    f = lib.diffattn_v2_decode
    args = [A, A, A, None, 32768, A, b.DA_BF16, 64, 64, 8, 128, A, A, ws - 16, None, None]
    assert f(*args) == b.DA_ERR_WORKSPACE
    args[12] = None
    args[13] = ws
    assert f(*args) == b.DA_ERR_WORKSPACE
    args[12] = U
    assert f(*args) == b.DA_ERR_ALIGNMENT
    args[12] = A
    args[4] = 0
    assert f(*args) == b.DA_ERR_INVALID_ARG
    g = lib.diffattn_v1_decode
    wsv1 = b.diffattn_v1_decode_workspace_size(2, 4, 64, 128, 1000)
    args = [A, A, A, None, 1000, A, b.DA_BF16, 2, 4, 64, 128, A, 1, None, 1e-5, 0.2, A,
            wsv1 - 1, None, None]
    assert g(*args) == b.DA_ERR_WORKSPACE
    args[1] = U
    assert g(*args) == b.DA_ERR_ALIGNMENT


def test_noalloc_host_validation(lib):
    """diffattn_v2_decode_noalloc refuses bad arguments, and sizes whose
    partial results do not fit its fixed 8 MiB scratch, before touching the
    device."""
    from differential_attention_sm_b200 import binding as b
    f = lib.diffattn_v2_decode_noalloc
    #        q  k  v  lens  L    out batch Hq Hkv lam status stream
    args = [A, A, A, None, 200, A, 252, 16, 8, A, None, None]
    bad = list(args)
    bad[0] = None
    assert f(*bad) == b.DA_ERR_INVALID_ARG
    bad = list(args)
    bad[8] = 16                                   # a group of one query head
    assert f(*bad) == b.DA_ERR_INVALID_ARG
    bad = list(args)
    bad[7], bad[8] = 32, 2                        # a group of 16
    assert f(*bad) == b.DA_ERR_UNSUPPORTED
    bad = list(args)
    bad[5] = U
    assert f(*bad) == b.DA_ERR_ALIGNMENT
    # 2017 units (batch x KV heads), one more than the scratch holds
    assert f(A, A, A, None, 200, A, 2017, 2, 1, A, None, None) == b.DA_ERR_UNSUPPORTED
    assert f(A, A, A, None, 64, A, 4096, 64, 8, A, None, None) == b.DA_ERR_UNSUPPORTED


def test_lambda_from_params_validation(lib):
    from differential_attention_sm_b200 import binding as b
    f = lib.lambda_from_params
    assert f(A, A, A, A, 4, 64, 0, A, None) == b.DA_ERR_INVALID_ARG
    assert f(A, None, A, A, 4, 64, 1, A, None) == b.DA_ERR_INVALID_ARG
    assert f(A, A, A, A, 0, 64, 1, A, None) == b.DA_ERR_INVALID_ARG


def test_product_path_has_no_oracle_dependency():
    """The library and its binding never load the oracle."""
    pkg = os.path.join(ROOT, "differential_attention_sm_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, fn), encoding="utf-8").read()
                assert "import oracle" not in text and "from oracle" not in text, fn
                assert "diffattn_oracle" not in text, fn


def test_window_variants_host_validation(lib):
    from differential_attention_sm_b200 import binding as b
    f = lib.diffattn_v1_fwd_window
    ok = [A, A, A, A, b.DA_BF16, 1, 128, 1, 64, 128, A, 1, 16, 1, None, 1e-5, 0.2, None, None]
    bad = list(ok); bad[12] = -1                 # negative window
    assert f(*bad) == b.DA_ERR_INVALID_ARG
    bad = list(ok); bad[11] = 0                  # a window needs causal masking
    assert f(*bad) == b.DA_ERR_INVALID_ARG
    bad = list(ok); bad[1] = U
    assert f(*bad) == b.DA_ERR_ALIGNMENT
    g = lib.diffattn_v2_prefill_window
    ok = [A, A, A, A, b.DA_BF16, 2, 256, 32, 8, 128, A, 1, 64, None, None]
    bad = list(ok); bad[12] = -5
    assert g(*bad) == b.DA_ERR_INVALID_ARG
    bad = list(ok); bad[11] = 0
    assert g(*bad) == b.DA_ERR_INVALID_ARG
    # windowed decode plans over min(window, max_len) entries
    ws_w = b.diffattn_v2_decode_workspace_size(64, 64, 8, 128, 4096)
    h = lib.diffattn_v2_decode_window
    args = [A, A, A, None, 32768, 4096, A, b.DA_BF16, 64, 64, 8, 128, A, A, ws_w - 16,
            None, None]
    assert h(*args) == b.DA_ERR_WORKSPACE
    args[5] = -1
    assert h(*args) == b.DA_ERR_INVALID_ARG
    k = lib.diffattn_v1_decode_window
    ws1 = b.diffattn_v1_decode_workspace_size(2, 4, 64, 128, 100)
    args = [A, A, A, None, 1000, 100, A, b.DA_BF16, 2, 4, 64, 128, A, 1, None, 1e-5, 0.2, A,
            ws1 - 1, None, None]
    assert k(*args) == b.DA_ERR_WORKSPACE
    args[5] = -2
    assert k(*args) == b.DA_ERR_INVALID_ARG


def test_backward_host_validation(lib):
    from differential_attention_sm_b200 import binding as b
    ws = b.diffattn_v1_bwd_workspace_size(4, 4096, 16, 64, 128)   # fused path
    assert ws >= 4 * 4096 * 16 * 128 * 2 * 5                       # no N x N buffers
    assert ws < 4 * 10 * 4096 * 4096                               # vs 10 N^2 per entry
    assert b.diffattn_v1_bwd_workspace_size(4, 4096, 16, 32, 64) >= 4 * 10 * 4096 * 4096
    assert b.diffattn_v1_bwd_workspace_size(0, 4096, 16, 64, 128) == 0
    f = lib.diffattn_v1_bwd
    ok = [A, A, A, A, A, b.DA_BF16, 4, 4096, 16, 64, 128, 1, 0, 1, None, 1e-5, 0.2, A, A, A, A,
          None, A, ws, None, None]
    bad = list(ok); bad[22] = None
    assert f(*bad) == b.DA_ERR_WORKSPACE
    bad = list(ok); bad[23] = ws - 1
    assert f(*bad) == b.DA_ERR_WORKSPACE
    bad = list(ok); bad[5] = b.DA_FP32
    assert f(*bad) == b.DA_ERR_UNSUPPORTED
    bad = list(ok); bad[12] = 5; bad[11] = 0          # window without causal
    assert f(*bad) == b.DA_ERR_INVALID_ARG
    bad = list(ok); bad[17] = None
    assert f(*bad) == b.DA_ERR_INVALID_ARG
    bad = list(ok); bad[0] = U
    assert f(*bad) == b.DA_ERR_ALIGNMENT
    g = lib.diffattn_v2_bwd
    ws2 = b.diffattn_v2_bwd_workspace_size(2, 8192, 32, 8, 128)
    ok = [A, A, A, A, A, b.DA_BF16, 2, 8192, 32, 8, 128, 1, 0, A, A, A, A, A, ws2, None, None]
    bad = list(ok); bad[8] = 6                         # group 32/6 not an integer
    assert g(*bad) == b.DA_ERR_INVALID_ARG
    bad = list(ok); bad[10] = 256
    assert g(*bad) == b.DA_ERR_UNSUPPORTED
    assert lib.lambda_from_params_bwd(A, A, A, A, A, 0, 4, A, A, A, A, None) == b.DA_ERR_INVALID_ARG


def test_oproj_host_validation(lib):
    from differential_attention_sm_b200 import binding as b
    ws = b.diffattn_v2_prefill_oproj_workspace_size(2, 8192, 32, 128)
    assert ws >= 2 * 8192 * 16 * 128 * 2
    f = lib.diffattn_v2_prefill_oproj
    ok = [A, A, A, A, A, A, b.DA_BF16, 2, 8192, 32, 8, 128, 2048, 1, 0, A, ws, None, None]
    bad = list(ok); bad[15] = None
    assert f(*bad) == b.DA_ERR_WORKSPACE
    bad = list(ok); bad[16] = ws - 1
    assert f(*bad) == b.DA_ERR_WORKSPACE
    bad = list(ok); bad[4] = None
    assert f(*bad) == b.DA_ERR_INVALID_ARG
    bad = list(ok); bad[12] = 0
    assert f(*bad) == b.DA_ERR_INVALID_ARG
    bad = list(ok); bad[6] = b.DA_FP32
    assert f(*bad) == b.DA_ERR_UNSUPPORTED
    bad = list(ok); bad[5] = U
    assert f(*bad) == b.DA_ERR_ALIGNMENT
    bad = list(ok); bad[12] = 2044   # row pitch of the output not a multiple of 16 bytes
    assert f(*bad) == b.DA_ERR_UNSUPPORTED
    bad = list(ok); bad[11] = 100; bad[9] = 2   # Hq/2 * head_dim = 100
    assert f(*bad) == b.DA_ERR_UNSUPPORTED


def test_saved_state_host_validation(lib):
    from differential_attention_sm_b200 import binding as b
    sz = b.load().diffattn_v1_fwd_train_saves_size(2, 300, 3)
    assert sz >= 2 * 3 * 2 * 320 * 4 + 2 * 300 * 3 * 256 * 4   # fp32 log-sum-exp and outputs
    assert b.load().diffattn_v1_fwd_train_saves_size(0, 300, 3) == 0
    f = lib.diffattn_v1_fwd_train
    ok = [A, A, A, A, b.DA_BF16, 2, 300, 3, 64, 128, A, 1, 0, 1, None, 1e-5, 0.2, A, sz, None,
          None]
    bad = list(ok); bad[18] = sz - 1
    assert f(*bad) == b.DA_ERR_WORKSPACE
    bad = list(ok); bad[8] = 32                     # not the tensor-core widths
    assert f(*bad) == b.DA_ERR_UNSUPPORTED
    bad = list(ok); bad[17] = U
    assert f(*bad) == b.DA_ERR_ALIGNMENT
    bad = list(ok); bad[12] = 5; bad[11] = 0        # window without causal
    assert f(*bad) == b.DA_ERR_INVALID_ARG
    ws = b.load().diffattn_v1_bwd_saved_workspace_size(2, 300, 3)
    g = lib.diffattn_v1_bwd_saved
    ok = [A, A, A, A, A, b.DA_BF16, 2, 300, 3, 64, 128, 1, 0, 1, None, 1e-5, 0.2, A, sz, A, A, A,
          A, A, A, ws, None, None]
    bad = list(ok); bad[25] = ws - 1
    assert g(*bad) == b.DA_ERR_WORKSPACE
    bad = list(ok); bad[19] = None
    assert g(*bad) == b.DA_ERR_INVALID_ARG
    bad = list(ok); bad[5] = b.DA_FP32
    assert g(*bad) == b.DA_ERR_UNSUPPORTED
    sz2 = b.load().diffattn_v2_prefill_train_saves_size(1, 300, 8)
    h = lib.diffattn_v2_prefill_train
    ok = [A, A, A, A, b.DA_BF16, 1, 300, 8, 2, 128, A, 1, 0, A, sz2, None, None]
    bad = list(ok); bad[9] = 64
    assert h(*bad) == b.DA_ERR_UNSUPPORTED
    bad = list(ok); bad[8] = 3                      # 8 query heads over 3 KV heads
    assert h(*bad) == b.DA_ERR_INVALID_ARG
    ws2 = b.load().diffattn_v2_bwd_saved_workspace_size(1, 300, 8)
    k = lib.diffattn_v2_bwd_saved
    ok = [A, A, A, A, A, b.DA_BF16, 1, 300, 8, 2, 128, 1, 0, A, sz2, A, A, A, A, A, ws2, None,
          None]
    bad = list(ok); bad[14] = sz2 - 1
    assert k(*bad) == b.DA_ERR_WORKSPACE


def test_selftest_host_validation(lib):
    from differential_attention_sm_b200 import binding as b
    f = lib.diffattn_selftest_wait_timeout
    assert f(1000, None, None, None) == b.DA_ERR_INVALID_ARG
    assert f(0, A, None, None) == b.DA_ERR_INVALID_ARG
    assert f(2000000, A, None, None) == b.DA_ERR_INVALID_ARG
    # the tile-counter hook checks its slot before enqueuing anything
    g = lib.diffattn_selftest_hold_tile_counter
    assert g(-1, 0, 0, None) == b.DA_ERR_INVALID_ARG
    assert g(64, 0, 0, None) == b.DA_ERR_INVALID_ARG
    k = lib.diffattn_selftest_keep_tile_counter
    assert k(64, 1, 10, None) == b.DA_ERR_INVALID_ARG
    assert k(0, 1, 0, None) == b.DA_ERR_INVALID_ARG
    assert k(0, 1, 10001, None) == b.DA_ERR_INVALID_ARG
