"""Thin ctypes binding over libdiffattn.so (``include/diffattn.h``).

Every function here has the name of the C entry point it wraps and only
marshals arguments: torch tensors (device memory allocated by PyTorch) are
passed as raw pointers together with their sizes, on the current CUDA
stream.  All arithmetic happens in the library's CUDA kernels.  There is no
fallback: if the library is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdiffattn.so")

DA_OK = 0
DA_ERR_INVALID_ARG = -1
DA_ERR_UNSUPPORTED = -2
DA_ERR_ALIGNMENT = -3
DA_ERR_WORKSPACE = -4
DA_ERR_CUDA = -5
DA_ERR_DEVICE_TIMEOUT = -6
DA_ERR_SCHEDULE = -7
DA_BF16 = 0
DA_FP32 = 1

# Every symbol include/diffattn.h declares.
EXPORTS = (
    "diffattn_status_string",
    "diffattn_lambda_init",
    "lambda_from_params",
    "diffattn_v1_fwd",
    "diffattn_v2_prefill",
    "diffattn_v2_decode_workspace_size",
    "diffattn_v2_decode",
    "diffattn_v2_decode_noalloc",
    "diffattn_v1_decode_workspace_size",
    "diffattn_v1_decode",
    "diffattn_v1_fwd_window",
    "diffattn_v2_prefill_window",
    "diffattn_v2_decode_window",
    "diffattn_v1_decode_window",
    "diffattn_v1_bwd_workspace_size",
    "diffattn_v1_bwd",
    "diffattn_v2_bwd_workspace_size",
    "diffattn_v2_bwd",
    "lambda_from_params_bwd",
    "diffattn_v1_fwd_train_saves_size",
    "diffattn_v1_fwd_train",
    "diffattn_v1_bwd_saved_workspace_size",
    "diffattn_v1_bwd_saved",
    "diffattn_v2_prefill_train_saves_size",
    "diffattn_v2_prefill_train",
    "diffattn_v2_bwd_saved_workspace_size",
    "diffattn_v2_bwd_saved",
    "diffattn_v2_prefill_oproj_workspace_size",
    "diffattn_v2_prefill_oproj",
    "diffattn_reset_tile_counters",
    "diffattn_selftest_hold_tile_counter",
    "diffattn_selftest_keep_tile_counter",
    "diffattn_selftest_wait_timeout",
)


class DiffAttnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__("%s failed: %s (%d)" % (fn, status_string(status), status))


_lib = None
_vp = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float
_sz = ctypes.c_size_t


def load(path: str | None = None) -> ctypes.CDLL:
    """Load the library (once).  Raises if it is missing: there is no
    CPU or library fallback for the operator."""
    global _lib
    if _lib is not None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise ImportError("libdiffattn.so not built (run __graft_entry__.build() or "
                          "python -m differential_attention_sm_b200.build)")
    lib = ctypes.CDLL(p)
    lib.diffattn_status_string.restype = ctypes.c_char_p
    lib.diffattn_status_string.argtypes = [_i]
    lib.diffattn_lambda_init.restype = ctypes.c_double
    lib.diffattn_lambda_init.argtypes = [_i]
    lib.lambda_from_params.restype = _i
    lib.lambda_from_params.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _vp, _vp]
    lib.diffattn_v1_fwd.restype = _i
    lib.diffattn_v1_fwd.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _i, _i,
                                    _vp, _f, _f, _vp, _vp]
    lib.diffattn_v2_prefill.restype = _i
    lib.diffattn_v2_prefill.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _i,
                                        _vp, _vp]
    lib.diffattn_v2_decode_workspace_size.restype = _sz
    lib.diffattn_v2_decode_workspace_size.argtypes = [_i, _i, _i, _i, _i]
    lib.diffattn_v2_decode.restype = _i
    lib.diffattn_v2_decode.argtypes = [_vp, _vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _vp,
                                       _vp, _sz, _vp, _vp]
    lib.diffattn_v2_decode_noalloc.restype = _i
    lib.diffattn_v2_decode_noalloc.argtypes = [_vp, _vp, _vp, _vp, _i, _vp, _i, _i, _i, _vp,
                                               _vp, _vp]
    lib.diffattn_v1_decode_workspace_size.restype = _sz
    lib.diffattn_v1_decode_workspace_size.argtypes = [_i, _i, _i, _i, _i]
    lib.diffattn_v1_decode.restype = _i
    lib.diffattn_v1_decode.argtypes = [_vp, _vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _vp,
                                       _i, _vp, _f, _f, _vp, _sz, _vp, _vp]
    lib.diffattn_v1_fwd_window.restype = _i
    lib.diffattn_v1_fwd_window.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _i,
                                           _i, _i, _vp, _f, _f, _vp, _vp]
    lib.diffattn_v2_prefill_window.restype = _i
    lib.diffattn_v2_prefill_window.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp,
                                               _i, _i, _vp, _vp]
    lib.diffattn_v2_decode_window.restype = _i
    lib.diffattn_v2_decode_window.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _vp, _i, _i, _i, _i,
                                              _i, _vp, _vp, _sz, _vp, _vp]
    lib.diffattn_v1_decode_window.restype = _i
    lib.diffattn_v1_decode_window.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _vp, _i, _i, _i, _i,
                                              _i, _vp, _i, _vp, _f, _f, _vp, _sz, _vp, _vp]
    lib.diffattn_v1_bwd_workspace_size.restype = _sz
    lib.diffattn_v1_bwd_workspace_size.argtypes = [_i, _i, _i, _i, _i]
    lib.diffattn_v1_bwd.restype = _i
    lib.diffattn_v1_bwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i,
                                    _i, _vp, _f, _f, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp,
                                    _vp]
    lib.diffattn_v2_bwd_workspace_size.restype = _sz
    lib.diffattn_v2_bwd_workspace_size.argtypes = [_i, _i, _i, _i, _i]
    lib.diffattn_v2_bwd.restype = _i
    lib.diffattn_v2_bwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i,
                                    _vp, _vp, _vp, _vp, _vp, _sz, _vp, _vp]
    lib.lambda_from_params_bwd.restype = _i
    lib.lambda_from_params_bwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _vp, _vp, _vp, _vp,
                                           _vp]
    for name in ("diffattn_v1_fwd_train_saves_size", "diffattn_v1_bwd_saved_workspace_size",
                 "diffattn_v2_prefill_train_saves_size", "diffattn_v2_bwd_saved_workspace_size"):
        getattr(lib, name).restype = _sz
        getattr(lib, name).argtypes = [_i, _i, _i]
    lib.diffattn_v1_fwd_train.restype = _i
    lib.diffattn_v1_fwd_train.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _i,
                                          _i, _i, _vp, _f, _f, _vp, _sz, _vp, _vp]
    lib.diffattn_v1_bwd_saved.restype = _i
    lib.diffattn_v1_bwd_saved.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i,
                                          _i, _i, _vp, _f, _f, _vp, _sz, _vp, _vp, _vp, _vp,
                                          _vp, _vp, _sz, _vp, _vp]
    lib.diffattn_v2_prefill_train.restype = _i
    lib.diffattn_v2_prefill_train.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp,
                                              _i, _i, _vp, _sz, _vp, _vp]
    lib.diffattn_v2_bwd_saved.restype = _i
    lib.diffattn_v2_bwd_saved.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i,
                                          _i, _vp, _sz, _vp, _vp, _vp, _vp, _vp, _sz, _vp, _vp]
    lib.diffattn_v2_prefill_oproj_workspace_size.restype = _sz
    lib.diffattn_v2_prefill_oproj_workspace_size.argtypes = [_i, _i, _i, _i]
    lib.diffattn_v2_prefill_oproj.restype = _i
    lib.diffattn_v2_prefill_oproj.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i,
                                              _i, _i, _i, _i, _vp, _sz, _vp, _vp]
    lib.diffattn_reset_tile_counters.restype = _i
    lib.diffattn_reset_tile_counters.argtypes = [_vp]
    lib.diffattn_selftest_hold_tile_counter.restype = _i
    lib.diffattn_selftest_hold_tile_counter.argtypes = [_i, ctypes.c_uint, ctypes.c_uint, _vp]
    lib.diffattn_selftest_keep_tile_counter.restype = _i
    lib.diffattn_selftest_keep_tile_counter.argtypes = [_i, ctypes.c_uint, ctypes.c_uint, _vp]
    lib.diffattn_selftest_wait_timeout.restype = _i
    lib.diffattn_selftest_wait_timeout.argtypes = [ctypes.c_uint, _vp, _vp, _vp]
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().diffattn_status_string(int(status)).decode()


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return DA_BF16
    if t.dtype == torch.float32:
        return DA_FP32
    raise TypeError("unsupported dtype %s" % t.dtype)


def _check(fn: str, status: int) -> None:
    if status != DA_OK:
        raise DiffAttnError(fn, status)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not isinstance(t, int):
            if not t.is_cuda or not t.is_contiguous():
                raise ValueError("tensors must be contiguous CUDA tensors")


def diffattn_lambda_init(layer: int) -> float:
    return float(load().diffattn_lambda_init(int(layer)))


def lambda_from_params(lq1, lk1, lq2, lk2, layer: int, out=None, stream=None):
    """lambda [H] (fp32, device) from four [H, dim] fp32 device vectors."""
    _need_cuda(lq1, lk1, lq2, lk2)
    H, dim = lq1.shape
    if out is None:
        out = torch.empty(H, dtype=torch.float32, device=lq1.device)
    _check("lambda_from_params", load().lambda_from_params(
        _ptr(lq1), _ptr(lk1), _ptr(lq2), _ptr(lk2), H, dim, int(layer), _ptr(out),
        _stream(stream)))
    return out


def diffattn_v1_fwd(q, k, v, lam, *, causal=True, apply_norm=False, norm_weight=None,
                    norm_eps=1e-5, lambda_init=0.0, out=None, dev_status=None, stream=None):
    """V1 prefill.  q, k [B, N, H, 2d]; v [B, N, H, dv]; lam [H] fp32."""
    _need_cuda(q, k, v, lam, norm_weight, dev_status)
    B, N, H, d2 = q.shape
    dv = v.shape[-1]
    if out is None:
        out = torch.empty(B, N, H, dv, dtype=q.dtype, device=q.device)
    _check("diffattn_v1_fwd", load().diffattn_v1_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _dtype_code(q), B, N, H, d2 // 2, dv,
        _ptr(lam), int(bool(causal)), int(bool(apply_norm)), _ptr(norm_weight),
        float(norm_eps), float(lambda_init), _ptr(dev_status), _stream(stream)))
    return out


def diffattn_v2_prefill(q, k, v, lam, *, causal=True, out=None, dev_status=None, stream=None):
    """V2 prefill.  q [B, N, Hq, d]; k, v [B, N, Hkv, d]; lam [Hq/2] fp32."""
    _need_cuda(q, k, v, lam, dev_status)
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    if out is None:
        out = torch.empty(B, N, Hq // 2, d, dtype=q.dtype, device=q.device)
    _check("diffattn_v2_prefill", load().diffattn_v2_prefill(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _dtype_code(q), B, N, Hq, Hkv, d, _ptr(lam),
        int(bool(causal)), _ptr(dev_status), _stream(stream)))
    return out


def diffattn_v2_decode_workspace_size(batch, n_q_heads, n_kv_heads, head_dim, max_len) -> int:
    return int(load().diffattn_v2_decode_workspace_size(batch, n_q_heads, n_kv_heads, head_dim,
                                                        max_len))


def diffattn_v2_decode(q, k_cache, v_cache, lam, *, cache_lens=None, workspace=None, out=None,
                       dev_status=None, stream=None):
    """V2 decode.  q [B, Hq, d]; caches [B, L, Hkv, d]; lam [Hq/2] fp32;
    cache_lens int32 [B] or None; workspace a uint8 device tensor or None
    (allocated here from the size query)."""
    _need_cuda(q, k_cache, v_cache, lam, cache_lens, dev_status)
    B, Hq, d = q.shape
    L, Hkv = k_cache.shape[1], k_cache.shape[2]
    ws_need = diffattn_v2_decode_workspace_size(B, Hq, Hkv, d, L)
    if workspace is None and ws_need:
        workspace = torch.empty(ws_need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if out is None:
        out = torch.empty(B, Hq // 2, d, dtype=q.dtype, device=q.device)
    _check("diffattn_v2_decode", load().diffattn_v2_decode(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(cache_lens), L, _ptr(out), _dtype_code(q),
        B, Hq, Hkv, d, _ptr(lam), _ptr(workspace), ws_bytes, _ptr(dev_status),
        _stream(stream)))
    return out


def diffattn_v2_decode_noalloc(q, k_cache, v_cache, lam, *, cache_lens=None, out=None,
                               dev_status=None, stream=None):
    """V2 decode without a workspace (bf16, head_dim 128): for callers that
    cannot allocate device memory.  The split-KV partials live in the
    library's fixed 8 MiB device array; calls that overlap on the GPU race
    on it.  Note that this wrapper still allocates `out` through PyTorch when
    it is not given."""
    _need_cuda(q, k_cache, v_cache, lam, cache_lens, dev_status)
    B, Hq, d = q.shape
    L, Hkv = k_cache.shape[1], k_cache.shape[2]
    if out is None:
        out = torch.empty(B, Hq // 2, d, dtype=q.dtype, device=q.device)
    _check("diffattn_v2_decode_noalloc", load().diffattn_v2_decode_noalloc(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(cache_lens), L, _ptr(out), B, Hq, Hkv,
        _ptr(lam), _ptr(dev_status), _stream(stream)))
    return out


def diffattn_v1_decode_workspace_size(batch, n_heads, d_qk, d_v, max_len) -> int:
    return int(load().diffattn_v1_decode_workspace_size(batch, n_heads, d_qk, d_v, max_len))


def diffattn_v1_decode(q, k_cache, v_cache, lam, *, cache_lens=None, apply_norm=False,
                       norm_weight=None, norm_eps=1e-5, lambda_init=0.0, workspace=None,
                       out=None, dev_status=None, stream=None):
    """V1 decode.  q [B, H, 2d]; k_cache [B, L, H, 2d]; v_cache [B, L, H, dv]."""
    _need_cuda(q, k_cache, v_cache, lam, cache_lens, norm_weight, dev_status)
    B, H, d2 = q.shape
    L, dv = k_cache.shape[1], v_cache.shape[-1]
    ws_need = diffattn_v1_decode_workspace_size(B, H, d2 // 2, dv, L)
    if workspace is None and ws_need:
        workspace = torch.empty(ws_need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if out is None:
        out = torch.empty(B, H, dv, dtype=q.dtype, device=q.device)
    _check("diffattn_v1_decode", load().diffattn_v1_decode(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(cache_lens), L, _ptr(out), _dtype_code(q),
        B, H, d2 // 2, dv, _ptr(lam), int(bool(apply_norm)), _ptr(norm_weight),
        float(norm_eps), float(lambda_init), _ptr(workspace), ws_bytes, _ptr(dev_status),
        _stream(stream)))
    return out


# ---- sliding-window variants: query i sees keys (i - window, i]; a decode
# query the last `window` cache entries (window 0 = no window) -------------
def diffattn_v1_fwd_window(q, k, v, lam, window, *, causal=True, apply_norm=False,
                           norm_weight=None, norm_eps=1e-5, lambda_init=0.0, out=None,
                           dev_status=None, stream=None):
    """V1 prefill with a sliding window.  Shapes as diffattn_v1_fwd."""
    _need_cuda(q, k, v, lam, norm_weight, dev_status)
    B, N, H, d2 = q.shape
    dv = v.shape[-1]
    if out is None:
        out = torch.empty(B, N, H, dv, dtype=q.dtype, device=q.device)
    _check("diffattn_v1_fwd_window", load().diffattn_v1_fwd_window(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _dtype_code(q), B, N, H, d2 // 2, dv,
        _ptr(lam), int(bool(causal)), int(window), int(bool(apply_norm)), _ptr(norm_weight),
        float(norm_eps), float(lambda_init), _ptr(dev_status), _stream(stream)))
    return out


def diffattn_v2_prefill_window(q, k, v, lam, window, *, causal=True, out=None, dev_status=None,
                               stream=None):
    """V2 prefill with a sliding window.  Shapes as diffattn_v2_prefill."""
    _need_cuda(q, k, v, lam, dev_status)
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    if out is None:
        out = torch.empty(B, N, Hq // 2, d, dtype=q.dtype, device=q.device)
    _check("diffattn_v2_prefill_window", load().diffattn_v2_prefill_window(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _dtype_code(q), B, N, Hq, Hkv, d, _ptr(lam),
        int(bool(causal)), int(window), _ptr(dev_status), _stream(stream)))
    return out


def _span(L, window):
    return min(int(window), L) if window and window > 0 else L


def diffattn_v2_decode_window(q, k_cache, v_cache, lam, window, *, cache_lens=None,
                              workspace=None, out=None, dev_status=None, stream=None):
    """V2 decode over the last `window` cache entries.  Shapes as
    diffattn_v2_decode; the workspace is sized for min(window, L) entries."""
    _need_cuda(q, k_cache, v_cache, lam, cache_lens, dev_status)
    B, Hq, d = q.shape
    L, Hkv = k_cache.shape[1], k_cache.shape[2]
    ws_need = diffattn_v2_decode_workspace_size(B, Hq, Hkv, d, _span(L, window))
    if workspace is None and ws_need:
        workspace = torch.empty(ws_need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if out is None:
        out = torch.empty(B, Hq // 2, d, dtype=q.dtype, device=q.device)
    _check("diffattn_v2_decode_window", load().diffattn_v2_decode_window(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(cache_lens), L, int(window), _ptr(out),
        _dtype_code(q), B, Hq, Hkv, d, _ptr(lam), _ptr(workspace), ws_bytes, _ptr(dev_status),
        _stream(stream)))
    return out


def diffattn_v1_decode_window(q, k_cache, v_cache, lam, window, *, cache_lens=None,
                              apply_norm=False, norm_weight=None, norm_eps=1e-5,
                              lambda_init=0.0, workspace=None, out=None, dev_status=None,
                              stream=None):
    """V1 decode over the last `window` cache entries.  Shapes as
    diffattn_v1_decode; the workspace is sized for min(window, L) entries."""
    _need_cuda(q, k_cache, v_cache, lam, cache_lens, norm_weight, dev_status)
    B, H, d2 = q.shape
    L, dv = k_cache.shape[1], v_cache.shape[-1]
    ws_need = diffattn_v1_decode_workspace_size(B, H, d2 // 2, dv, _span(L, window))
    if workspace is None and ws_need:
        workspace = torch.empty(ws_need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if out is None:
        out = torch.empty(B, H, dv, dtype=q.dtype, device=q.device)
    _check("diffattn_v1_decode_window", load().diffattn_v1_decode_window(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(cache_lens), L, int(window), _ptr(out),
        _dtype_code(q), B, H, d2 // 2, dv, _ptr(lam), int(bool(apply_norm)),
        _ptr(norm_weight), float(norm_eps), float(lambda_init), _ptr(workspace), ws_bytes,
        _ptr(dev_status), _stream(stream)))
    return out


# ---- backward ---------------------------------------------------------------
def diffattn_v1_bwd_workspace_size(batch, seqlen, n_heads, d_qk, d_v) -> int:
    return int(load().diffattn_v1_bwd_workspace_size(batch, seqlen, n_heads, d_qk, d_v))


def diffattn_v1_bwd(q, k, v, dout, lam, *, causal=True, window=0, apply_norm=False,
                    norm_weight=None, norm_eps=1e-5, lambda_init=0.0, workspace=None,
                    out=None, dev_status=None, stream=None):
    """V1 gradients.  Returns dict of fp32 device tensors dq, dk (like q),
    dv (like v), dlambda [H] and, with the norm, dnorm_weight [dv]; `out`
    may supply any of them (caller-owned, written in place)."""
    _need_cuda(q, k, v, dout, lam, norm_weight)
    B, N, H, d2 = q.shape
    dvw = v.shape[-1]
    if workspace is None:
        workspace = torch.empty(diffattn_v1_bwd_workspace_size(B, N, H, d2 // 2, dvw),
                                dtype=torch.uint8, device=q.device)
    f32 = dict(dtype=torch.float32, device=q.device)
    res = {"dq": torch.empty(q.shape, **f32), "dk": torch.empty(k.shape, **f32),
           "dv": torch.empty(v.shape, **f32), "dlambda": torch.empty(H, **f32),
           "dnorm_weight": torch.empty(dvw, **f32) if apply_norm else None}
    res.update(out or {})
    _check("diffattn_v1_bwd", load().diffattn_v1_bwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(lam), _dtype_code(q), B, N, H, d2 // 2,
        dvw, int(bool(causal)), int(window), int(bool(apply_norm)), _ptr(norm_weight),
        float(norm_eps), float(lambda_init), _ptr(res["dq"]), _ptr(res["dk"]), _ptr(res["dv"]),
        _ptr(res["dlambda"]), _ptr(res["dnorm_weight"]), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(dev_status), _stream(stream)))
    return res


def diffattn_v2_bwd_workspace_size(batch, seqlen, n_q_heads, n_kv_heads, head_dim) -> int:
    return int(load().diffattn_v2_bwd_workspace_size(batch, seqlen, n_q_heads, n_kv_heads,
                                                     head_dim))


def diffattn_v2_bwd(q, k, v, dout, lam, *, causal=True, window=0, workspace=None,
                    out=None, dev_status=None, stream=None):
    """V2 gradients.  Returns dict of fp32 device tensors dq (like q), dk,
    dv (like k) and dlambda [Hq/2]; `out` may supply any of them."""
    _need_cuda(q, k, v, dout, lam)
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    if workspace is None:
        workspace = torch.empty(diffattn_v2_bwd_workspace_size(B, N, Hq, Hkv, d),
                                dtype=torch.uint8, device=q.device)
    f32 = dict(dtype=torch.float32, device=q.device)
    res = {"dq": torch.empty(q.shape, **f32), "dk": torch.empty(k.shape, **f32),
           "dv": torch.empty(v.shape, **f32), "dlambda": torch.empty(Hq // 2, **f32)}
    res.update(out or {})
    _check("diffattn_v2_bwd", load().diffattn_v2_bwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(lam), _dtype_code(q), B, N, Hq, Hkv, d,
        int(bool(causal)), int(window), _ptr(res["dq"]), _ptr(res["dk"]), _ptr(res["dv"]),
        _ptr(res["dlambda"]), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _ptr(dev_status), _stream(stream)))
    return res


# ---- training forward with saves, and the backward from the saves ----------
def _nbytes(t):
    return t.numel() * t.element_size()


def diffattn_v1_fwd_train(q, k, v, lam, *, causal=True, window=0, apply_norm=False,
                          norm_weight=None, norm_eps=1e-5, lambda_init=0.0, out=None,
                          saves=None, dev_status=None, stream=None):
    """V1 forward that also writes the saves the backward reads.  Returns
    (out, saves); saves is a uint8 device tensor (allocated here if None)."""
    _need_cuda(q, k, v, lam, norm_weight, dev_status)
    B, N, H, d2 = q.shape
    dvw = v.shape[-1]
    if saves is None:
        saves = torch.empty(int(load().diffattn_v1_fwd_train_saves_size(B, N, H)),
                            dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty(B, N, H, dvw, dtype=q.dtype, device=q.device)
    _check("diffattn_v1_fwd_train", load().diffattn_v1_fwd_train(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _dtype_code(q), B, N, H, d2 // 2, dvw, _ptr(lam),
        int(bool(causal)), int(window), int(bool(apply_norm)), _ptr(norm_weight),
        float(norm_eps), float(lambda_init), _ptr(saves), _nbytes(saves), _ptr(dev_status),
        _stream(stream)))
    return out, saves


def diffattn_v1_bwd_saved(q, k, v, dout, lam, saves, *, causal=True, window=0,
                          apply_norm=False, norm_weight=None, norm_eps=1e-5, lambda_init=0.0,
                          workspace=None, out=None, dev_status=None, stream=None):
    """V1 gradients from the saves of diffattn_v1_fwd_train (same dict as
    diffattn_v1_bwd)."""
    _need_cuda(q, k, v, dout, lam, saves, norm_weight)
    B, N, H, d2 = q.shape
    dvw = v.shape[-1]
    if workspace is None:
        workspace = torch.empty(int(load().diffattn_v1_bwd_saved_workspace_size(B, N, H)),
                                dtype=torch.uint8, device=q.device)
    f32 = dict(dtype=torch.float32, device=q.device)
    res = {"dq": torch.empty(q.shape, **f32), "dk": torch.empty(k.shape, **f32),
           "dv": torch.empty(v.shape, **f32), "dlambda": torch.empty(H, **f32),
           "dnorm_weight": torch.empty(dvw, **f32) if apply_norm else None}
    res.update(out or {})
    _check("diffattn_v1_bwd_saved", load().diffattn_v1_bwd_saved(
        _ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(lam), _dtype_code(q), B, N, H, d2 // 2,
        dvw, int(bool(causal)), int(window), int(bool(apply_norm)), _ptr(norm_weight),
        float(norm_eps), float(lambda_init), _ptr(saves), _nbytes(saves), _ptr(res["dq"]),
        _ptr(res["dk"]), _ptr(res["dv"]), _ptr(res["dlambda"]), _ptr(res["dnorm_weight"]),
        _ptr(workspace), _nbytes(workspace), _ptr(dev_status), _stream(stream)))
    return res


def diffattn_v2_prefill_train(q, k, v, lam, *, causal=True, window=0, out=None, saves=None,
                              dev_status=None, stream=None):
    """V2 prefill that also writes the saves the backward reads.  Returns
    (out, saves)."""
    _need_cuda(q, k, v, lam, dev_status)
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    if saves is None:
        saves = torch.empty(int(load().diffattn_v2_prefill_train_saves_size(B, N, Hq)),
                            dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty(B, N, Hq // 2, d, dtype=q.dtype, device=q.device)
    _check("diffattn_v2_prefill_train", load().diffattn_v2_prefill_train(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _dtype_code(q), B, N, Hq, Hkv, d, _ptr(lam),
        int(bool(causal)), int(window), _ptr(saves), _nbytes(saves), _ptr(dev_status),
        _stream(stream)))
    return out, saves


def diffattn_v2_bwd_saved(q, k, v, dout, lam, saves, *, causal=True, window=0, workspace=None,
                          out=None, dev_status=None, stream=None):
    """V2 gradients from the saves of diffattn_v2_prefill_train (same dict
    as diffattn_v2_bwd)."""
    _need_cuda(q, k, v, dout, lam, saves)
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    if workspace is None:
        workspace = torch.empty(int(load().diffattn_v2_bwd_saved_workspace_size(B, N, Hq)),
                                dtype=torch.uint8, device=q.device)
    f32 = dict(dtype=torch.float32, device=q.device)
    res = {"dq": torch.empty(q.shape, **f32), "dk": torch.empty(k.shape, **f32),
           "dv": torch.empty(v.shape, **f32), "dlambda": torch.empty(Hq // 2, **f32)}
    res.update(out or {})
    _check("diffattn_v2_bwd_saved", load().diffattn_v2_bwd_saved(
        _ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(lam), _dtype_code(q), B, N, Hq, Hkv, d,
        int(bool(causal)), int(window), _ptr(saves), _nbytes(saves), _ptr(res["dq"]),
        _ptr(res["dk"]), _ptr(res["dv"]), _ptr(res["dlambda"]), _ptr(workspace),
        _nbytes(workspace), _ptr(dev_status), _stream(stream)))
    return res


def lambda_from_params_bwd(lq1, lk1, lq2, lk2, dlambda, stream=None):
    """Gradients of the four lambda vectors: dict of fp32 [H, dim] tensors."""
    _need_cuda(lq1, lk1, lq2, lk2, dlambda)
    H, dim = lq1.shape
    outs = {n: torch.empty(H, dim, dtype=torch.float32, device=lq1.device)
            for n in ("dlq1", "dlk1", "dlq2", "dlk2")}
    _check("lambda_from_params_bwd", load().lambda_from_params_bwd(
        _ptr(lq1), _ptr(lk1), _ptr(lq2), _ptr(lk2), _ptr(dlambda), H, dim,
        *(_ptr(outs[n]) for n in ("dlq1", "dlk1", "dlq2", "dlk2")), _stream(stream)))
    return outs


# ---- V2 prefill + output projection ------------------------------------------
def diffattn_v2_prefill_oproj_workspace_size(batch, seqlen, n_q_heads, head_dim) -> int:
    return int(load().diffattn_v2_prefill_oproj_workspace_size(batch, seqlen, n_q_heads,
                                                                head_dim))


def diffattn_v2_prefill_oproj(q, k, v, lam, w_o, *, causal=True, window=0, workspace=None,
                              out=None, dev_status=None, stream=None):
    """V2 prefill followed by out = o . w_o.  q [B, N, Hq, d]; k, v
    [B, N, Hkv, d]; w_o [Hq/2 * d, d_model] bf16.  Returns [B, N, d_model]."""
    _need_cuda(q, k, v, lam, w_o, dev_status)
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    d_model = w_o.shape[1]
    if workspace is None:
        workspace = torch.empty(diffattn_v2_prefill_oproj_workspace_size(B, N, Hq, d),
                                dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty(B, N, d_model, dtype=q.dtype, device=q.device)
    _check("diffattn_v2_prefill_oproj", load().diffattn_v2_prefill_oproj(
        _ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(w_o), _ptr(out), _dtype_code(q), B, N, Hq,
        Hkv, d, d_model, int(bool(causal)), int(window), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(dev_status), _stream(stream)))
    return out


def diffattn_selftest_wait_timeout(timeout_us, dev_status, waited_ns=None, stream=None):
    """Run the bounded-wait path to its timeout (see the header); the status
    word then holds DA_ERR_DEVICE_TIMEOUT."""
    _need_cuda(dev_status, waited_ns)
    _check("diffattn_selftest_wait_timeout", load().diffattn_selftest_wait_timeout(
        int(timeout_us), _ptr(dev_status), _ptr(waited_ns), _stream(stream)))


def diffattn_reset_tile_counters(stream=None):
    """Free every tile counter of the tensor-core prefill on the current
    device (see the header)."""
    _check("diffattn_reset_tile_counters",
           load().diffattn_reset_tile_counters(_stream(stream)))


def diffattn_selftest_hold_tile_counter(slot, tag, count, stream=None):
    """Test hook: set tile counter `slot` to (tag, count) and make the next
    tensor-core prefill launch take it (see the header)."""
    _check("diffattn_selftest_hold_tile_counter", load().diffattn_selftest_hold_tile_counter(
        int(slot), int(tag), int(count), _stream(stream)))


def diffattn_selftest_keep_tile_counter(slot, tag, duration_ms, stream=None):
    """Test hook: keep tile counter `slot` held by `tag`, as a launch in
    flight would, for `duration_ms` (see the header)."""
    _check("diffattn_selftest_keep_tile_counter", load().diffattn_selftest_keep_tile_counter(
        int(slot), int(tag), int(duration_ms), _stream(stream)))
