"""ctypes front-end of the fp64 C oracle (``diffattn_oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
CPU-baseline leg of the benchmark, never by the product path.

The C code takes float32 arrays (bf16 inputs are widened to float32 first,
which is exact) and computes every requested output row in double precision.
This module only marshals arrays and spreads independent rows over host
threads; all arithmetic happens in the C file.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "diffattn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None
_lock = threading.Lock()

_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)
_i32p = ctypes.POINTER(ctypes.c_int)


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain IEEE double: no fast-math, no FMA
    contraction).  Returns the shared-library path."""
    stale = (not os.path.exists(_LIB_PATH)) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + ".%d.tmp" % os.getpid()
        subprocess.check_call([
            "gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fno-fast-math",
            "-ffp-contract=off", "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        lib.oracle_lambda_init.restype = ctypes.c_double
        lib.oracle_lambda_init.argtypes = [ctypes.c_int]
        lib.oracle_lambda_from_params.restype = ctypes.c_int
        lib.oracle_lambda_from_params.argtypes = [
            _f32p, _f32p, _f32p, _f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, _f64p]
        lib.oracle_v1_rows.restype = ctypes.c_int
        lib.oracle_v1_rows.argtypes = [
            _f32p, _f32p, _f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, _f64p, ctypes.c_int, ctypes.c_int, ctypes.c_int, _f32p,
            ctypes.c_double, ctypes.c_double, _i64p, ctypes.c_int64, _f64p, _f64p]
        lib.oracle_v2_rows.restype = ctypes.c_int
        lib.oracle_v2_rows.argtypes = [
            _f32p, _f32p, _f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, _f64p, ctypes.c_int, ctypes.c_int, _i64p, ctypes.c_int64,
            _f64p, _f64p]
        lib.oracle_v2_decode_rows.restype = ctypes.c_int
        lib.oracle_v2_decode_rows.argtypes = [
            _f32p, _f32p, _f32p, _i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, _f64p, _i64p, ctypes.c_int64, _f64p]
        lib.oracle_v1_bwd.restype = ctypes.c_int
        lib.oracle_v1_bwd.argtypes = [
            _f32p, _f32p, _f32p, _f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, _f64p, ctypes.c_int, ctypes.c_int, ctypes.c_int, _f32p,
            ctypes.c_double, ctypes.c_double, _f64p, _f64p, _f64p, _f64p, _f64p]
        lib.oracle_v2_bwd.restype = ctypes.c_int
        lib.oracle_v2_bwd.argtypes = [
            _f32p, _f32p, _f32p, _f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, _f64p, ctypes.c_int, ctypes.c_int, _f64p, _f64p, _f64p, _f64p]
        lib.oracle_lambda_params_bwd.restype = ctypes.c_int
        lib.oracle_lambda_params_bwd.argtypes = [
            _f32p, _f32p, _f32p, _f32p, ctypes.c_int, ctypes.c_int, _f64p, _f64p, _f64p,
            _f64p, _f64p]
        lib.oracle_snr.restype = ctypes.c_int
        lib.oracle_snr.argtypes = [_f64p, ctypes.c_int64, ctypes.c_int64, _f64p]
        lib.oracle_v1_decode_rows.restype = ctypes.c_int
        lib.oracle_v1_decode_rows.argtypes = [
            _f32p, _f32p, _f32p, _i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, _f64p, ctypes.c_int, _f32p, ctypes.c_double,
            ctypes.c_double, _i64p, ctypes.c_int64, _f64p]
        _lib = lib
        return lib


def n_threads() -> int:
    """Host threads the oracle spreads rows over (the process's CPU set)."""
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return max(1, os.cpu_count() or 1)


def _f32(a) -> np.ndarray:
    """float32, C-contiguous view of a numpy array or a CPU torch tensor."""
    if hasattr(a, "detach"):  # torch tensor, possibly bf16
        import torch
        a = a.detach().to("cpu", torch.float32).contiguous().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _ptr(a, t):
    return a.ctypes.data_as(t) if a is not None else None


def _run_rows(call, rows: np.ndarray, width: int, weights_width: int | None,
              threads: int | None):
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1))
    out = np.zeros((rows.size, width), dtype=np.float64)
    w = (np.zeros((rows.size, weights_width), dtype=np.float64)
         if weights_width else None)
    nt = max(1, min(threads or n_threads(), rows.size))
    chunks = np.array_split(np.arange(rows.size), nt)

    def work(idx):
        if idx.size == 0:
            return 0
        lo, hi = int(idx[0]), int(idx[-1]) + 1
        r = rows[lo:hi]
        o = out[lo:hi]
        ww = w[lo:hi] if w is not None else None
        return call(r, o, ww)

    if nt == 1:
        rcs = [work(chunks[0])]
    else:
        with ThreadPoolExecutor(max_workers=nt) as ex:
            rcs = list(ex.map(work, chunks))
    if any(rc != 0 for rc in rcs):
        raise ValueError("oracle rejected its arguments (status %s)" % rcs)
    return (out, w) if weights_width else out


def lambda_init(layer: int) -> float:
    """lambda_init(l) = 0.8 - 0.6 exp(-0.3 (l - 1)), NaN for l < 1."""
    return float(_load().oracle_lambda_init(int(layer)))


def lambda_from_params(lq1, lk1, lq2, lk2, layer: int) -> np.ndarray:
    """Per-head lambda from the four [H, dim] vectors (double result)."""
    a, b, c, d = (_f32(x) for x in (lq1, lk1, lq2, lk2))
    H, dim = a.shape
    out = np.zeros(H, dtype=np.float64)
    rc = _load().oracle_lambda_from_params(
        _ptr(a, _f32p), _ptr(b, _f32p), _ptr(c, _f32p), _ptr(d, _f32p),
        H, dim, int(layer), _ptr(out, _f64p))
    if rc != 0:
        raise ValueError("oracle_lambda_from_params status %d" % rc)
    return out


def v1_rows(q, k, v, lam, rows, *, causal: bool, apply_norm: bool = False,
            norm_weight=None, eps: float = 1e-5, lambda_init_value: float = 0.0,
            return_weights: bool = False, window: int = 0, threads: int | None = None):
    """V1 rows r = (b*N + i)*H + h of out [B, N, H, dv] (double).
    q, k: [B, N, H, 2d]; v: [B, N, H, dv]; lam: [H].  window > 0 keeps only
    the last ``window`` visible keys of each row (sliding window)."""
    qf, kf, vf = _f32(q), _f32(k), _f32(v)
    B, N, H, d2 = qf.shape
    dv = vf.shape[-1]
    lamd = np.ascontiguousarray(np.asarray(lam, dtype=np.float64).reshape(-1))
    g = _f32(norm_weight) if norm_weight is not None else None
    lib = _load()

    def call(r, o, w):
        return lib.oracle_v1_rows(
            _ptr(qf, _f32p), _ptr(kf, _f32p), _ptr(vf, _f32p), B, N, H, d2 // 2, dv,
            _ptr(lamd, _f64p), int(causal), int(window), int(apply_norm), _ptr(g, _f32p),
            float(eps), float(lambda_init_value), _ptr(r, _i64p), r.size,
            _ptr(o, _f64p), _ptr(w, _f64p))

    return _run_rows(call, rows, dv, N if return_weights else None, threads)


def v2_rows(q, k, v, lam, rows, *, causal: bool, return_weights: bool = False,
            window: int = 0, threads: int | None = None):
    """V2 rows r = (b*N + i)*(Hq/2) + p of out [B, N, Hq/2, d] (double).
    q: [B, N, Hq, d]; k, v: [B, N, Hkv, d]; lam: [Hq/2]."""
    qf, kf, vf = _f32(q), _f32(k), _f32(v)
    B, N, Hq, d = qf.shape
    Hkv = kf.shape[2]
    lamd = np.ascontiguousarray(np.asarray(lam, dtype=np.float64).reshape(-1))
    lib = _load()

    def call(r, o, w):
        return lib.oracle_v2_rows(
            _ptr(qf, _f32p), _ptr(kf, _f32p), _ptr(vf, _f32p), B, N, Hq, Hkv, d,
            _ptr(lamd, _f64p), int(causal), int(window), _ptr(r, _i64p), r.size,
            _ptr(o, _f64p), _ptr(w, _f64p))

    return _run_rows(call, rows, d, N if return_weights else None, threads)


def v2_oproj_rows(q, k, v, lam, w_o, tokens, *, causal: bool, window: int = 0,
                  threads: int | None = None):
    """Output projection of the V2 prefill (lesson "Atencion Diferencial
    (V2)", "V1 vs V2: la diferencia" and step 5 of "Implementacion": the
    paired heads, Hq/2 of width d, go through O_W).  For each token
    t = b*N + i of ``tokens``: its Hq/2 pair rows from ``v2_rows``, laid end
    to end in pair order ([Hq/2 * d]), times w_o [Hq/2 * d, d_model], in
    float64 (numpy matrix product).  Returns [len(tokens), d_model]."""
    qf = _f32(q)
    P = qf.shape[2] // 2
    d = qf.shape[3]
    t = np.asarray(tokens, dtype=np.int64).reshape(-1)
    rows = (t[:, None] * P + np.arange(P)[None, :]).reshape(-1)
    o = v2_rows(qf, k, v, lam, rows, causal=causal, window=window, threads=threads)
    w = np.asarray(_f32(w_o), dtype=np.float64)
    if w.shape[0] != P * d:
        raise ValueError("w_o must have Hq/2 * head_dim rows")
    return o.reshape(t.size, P * d) @ w


def v2_decode_rows(q, k_cache, v_cache, lam, rows, *, lens=None, window: int = 0,
                   threads: int | None = None):
    """V2 decode rows r = b*(Hq/2) + p of out [B, Hq/2, d] (double).
    q: [B, Hq, d]; caches: [B, max_len, Hkv, d]; lens: [B] or None."""
    qf, kf, vf = _f32(q), _f32(k_cache), _f32(v_cache)
    B, Hq, d = qf.shape
    max_len, Hkv = kf.shape[1], kf.shape[2]
    lamd = np.ascontiguousarray(np.asarray(lam, dtype=np.float64).reshape(-1))
    ln = (np.ascontiguousarray(np.asarray(lens, dtype=np.int32).reshape(-1))
          if lens is not None else None)
    lib = _load()

    def call(r, o, w):
        return lib.oracle_v2_decode_rows(
            _ptr(qf, _f32p), _ptr(kf, _f32p), _ptr(vf, _f32p), _ptr(ln, _i32p),
            max_len, int(window), B, Hq, Hkv, d, _ptr(lamd, _f64p), _ptr(r, _i64p), r.size,
            _ptr(o, _f64p))

    return _run_rows(call, rows, d, None, threads)


def v1_decode_rows(q, k_cache, v_cache, lam, rows, *, lens=None,
                   apply_norm: bool = False, norm_weight=None, eps: float = 1e-5,
                   lambda_init_value: float = 0.0, window: int = 0,
                   threads: int | None = None):
    """V1 decode rows r = b*H + h of out [B, H, dv] (double).
    q: [B, H, 2d]; k_cache: [B, max_len, H, 2d]; v_cache: [B, max_len, H, dv]."""
    qf, kf, vf = _f32(q), _f32(k_cache), _f32(v_cache)
    B, H, d2 = qf.shape
    max_len, dv = kf.shape[1], vf.shape[-1]
    lamd = np.ascontiguousarray(np.asarray(lam, dtype=np.float64).reshape(-1))
    ln = (np.ascontiguousarray(np.asarray(lens, dtype=np.int32).reshape(-1))
          if lens is not None else None)
    g = _f32(norm_weight) if norm_weight is not None else None
    lib = _load()

    def call(r, o, w):
        return lib.oracle_v1_decode_rows(
            _ptr(qf, _f32p), _ptr(kf, _f32p), _ptr(vf, _f32p), _ptr(ln, _i32p),
            max_len, int(window), B, H, d2 // 2, dv, _ptr(lamd, _f64p), int(apply_norm),
            _ptr(g, _f32p), float(eps), float(lambda_init_value), _ptr(r, _i64p),
            r.size, _ptr(o, _f64p))

    return _run_rows(call, rows, dv, None, threads)


def v1_query_weights(q_row, keys, lam):
    """Differential weights w_j = a1_j - lam_h * a2_j of ONE V1 query row
    against L keys, for every lambda in ``lam``: returns [len(lam), L]
    (double).  q_row: [2d]; keys: [L, 2d].  Computed by the oracle's V1
    row routine (non-causal, query placed at row 0 of an L-row block)."""
    q_row = np.asarray(q_row, dtype=np.float32).reshape(-1)
    keys = np.asarray(keys, dtype=np.float32)
    L, d2 = keys.shape
    H = int(np.asarray(lam).size)
    q = np.zeros((1, L, H, d2), dtype=np.float32)
    q[0, 0, :, :] = q_row
    k = np.ascontiguousarray(np.broadcast_to(keys[None, :, None, :], (1, L, H, d2)))
    v = np.zeros((1, L, H, 1), dtype=np.float32)
    _, w = v1_rows(q, k, v, lam, np.arange(H), causal=False, return_weights=True)
    return w


def snr(weights, pos: int):
    """Signal-to-noise ratio of each weight row (last axis): the weight at
    ``pos`` over the RMS weight elsewhere (``oracle_snr``)."""
    w = np.ascontiguousarray(np.asarray(weights, dtype=np.float64))
    flat = w.reshape(-1, w.shape[-1])
    out = np.empty(flat.shape[0])
    lib = _load()
    one = np.zeros(1)
    for i in range(flat.shape[0]):
        row = np.ascontiguousarray(flat[i])
        rc = lib.oracle_snr(_ptr(row, _f64p), row.size, int(pos), _ptr(one, _f64p))
        if rc != 0:
            raise ValueError("oracle_snr status %d" % rc)
        out[i] = one[0]
    return out.reshape(w.shape[:-1])


def v1_bwd(q, k, v, dout, lam, *, causal: bool, window: int = 0, apply_norm: bool = False,
           norm_weight=None, eps: float = 1e-5, lambda_init_value: float = 0.0):
    """Gradients of sum(out * dout) for the V1 forward: dict with dq, dk
    [B, N, H, 2d], dv [B, N, H, dv], dlambda [H] and, with the norm,
    dnorm_weight [dv] (all double)."""
    qf, kf, vf, gf = _f32(q), _f32(k), _f32(v), _f32(dout)
    B, N, H, d2 = qf.shape
    dv = vf.shape[-1]
    lamd = np.ascontiguousarray(np.asarray(lam, dtype=np.float64).reshape(-1))
    g = _f32(norm_weight) if norm_weight is not None else None
    res = {"dq": np.empty(qf.shape), "dk": np.empty(kf.shape), "dv": np.empty(vf.shape),
           "dlambda": np.empty(H), "dnorm_weight": np.empty(dv) if apply_norm else None}
    rc = _load().oracle_v1_bwd(
        _ptr(qf, _f32p), _ptr(kf, _f32p), _ptr(vf, _f32p), _ptr(gf, _f32p), B, N, H, d2 // 2,
        dv, _ptr(lamd, _f64p), int(causal), int(window), int(apply_norm), _ptr(g, _f32p),
        float(eps), float(lambda_init_value), _ptr(res["dq"], _f64p), _ptr(res["dk"], _f64p),
        _ptr(res["dv"], _f64p), _ptr(res["dlambda"], _f64p), _ptr(res["dnorm_weight"], _f64p))
    if rc != 0:
        raise ValueError("oracle_v1_bwd status %d" % rc)
    return res


def v2_bwd(q, k, v, dout, lam, *, causal: bool, window: int = 0):
    """Gradients of sum(out * dout) for the V2 forward: dict with dq
    [B, N, Hq, d], dk, dv [B, N, Hkv, d], dlambda [Hq/2] (double)."""
    qf, kf, vf, gf = _f32(q), _f32(k), _f32(v), _f32(dout)
    B, N, Hq, d = qf.shape
    Hkv = kf.shape[2]
    lamd = np.ascontiguousarray(np.asarray(lam, dtype=np.float64).reshape(-1))
    res = {"dq": np.empty(qf.shape), "dk": np.empty(kf.shape), "dv": np.empty(vf.shape),
           "dlambda": np.empty(Hq // 2)}
    rc = _load().oracle_v2_bwd(
        _ptr(qf, _f32p), _ptr(kf, _f32p), _ptr(vf, _f32p), _ptr(gf, _f32p), B, N, Hq, Hkv, d,
        _ptr(lamd, _f64p), int(causal), int(window), _ptr(res["dq"], _f64p),
        _ptr(res["dk"], _f64p), _ptr(res["dv"], _f64p), _ptr(res["dlambda"], _f64p))
    if rc != 0:
        raise ValueError("oracle_v2_bwd status %d" % rc)
    return res


def lambda_params_bwd(lq1, lk1, lq2, lk2, dlambda):
    """Gradients of the four [H, dim] lambda vectors (double) given
    d(loss)/d(lambda) [H]."""
    a, b, c, d = (_f32(x) for x in (lq1, lk1, lq2, lk2))
    H, dim = a.shape
    dl = np.ascontiguousarray(np.asarray(dlambda, dtype=np.float64).reshape(-1))
    outs = [np.empty((H, dim)) for _ in range(4)]
    rc = _load().oracle_lambda_params_bwd(
        _ptr(a, _f32p), _ptr(b, _f32p), _ptr(c, _f32p), _ptr(d, _f32p), H, dim,
        _ptr(dl, _f64p), *(_ptr(o, _f64p) for o in outs))
    if rc != 0:
        raise ValueError("oracle_lambda_params_bwd status %d" % rc)
    return dict(zip(("dlq1", "dlk1", "dlq2", "dlk2"), outs))
