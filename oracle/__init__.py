"""Oracle for attention-level speculation decode attention (fp64, CPU).

TEST INFRASTRUCTURE ONLY.  Only tests/, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA product
path never imports it, and it shares no code with the kernels.

The arithmetic lives in ``alspec_oracle.c`` (plain C, double precision,
two-pass softmax).  This module only marshals numpy arrays into it.

What it computes (Attention-Level Speculation, atlas.scime.ai summary,
"Approach"; ICML 2025 poster page, abstract): for each decode query, the
exact softmax attention over all cached tokens and the attention-sink
approximation over the first S plus the last W tokens, then the per-token
relative L2 error of the approximation and the commit (r <= lambda) or
discard flag.
"""
import ctypes
import os

import numpy as np

from . import build as _build

F32, BF16, F64 = 0, 1, 2

_SIGS = {
    "alspec_oracle_head": ("i", "i", "i", "p", "p", "p", "i", "i", "p", "p", "p", "p"),
    "alspec_oracle_rel_l2": ("p", "p", "l"),
    "alspec_oracle_commit": ("d", "d"),
    "alspec_oracle_decode": ("i", "i", "i", "i", "i", "i", "p", "p", "p", "p", "i",
                             "i", "d", "p", "p", "p", "p", "i"),
    "alspec_oracle_oproj": ("i", "i", "i", "p", "p", "i", "p"),
    "alspec_oracle_oproj_gated": ("i", "i", "i", "p", "p", "p", "p", "i", "p"),
}
_RES = {"alspec_oracle_head": "i", "alspec_oracle_rel_l2": "d",
        "alspec_oracle_commit": "i", "alspec_oracle_decode": "i",
        "alspec_oracle_oproj": "i", "alspec_oracle_oproj_gated": "i"}
_CT = {"i": ctypes.c_int, "p": ctypes.c_void_p, "l": ctypes.c_long, "d": ctypes.c_double}

_libs = {}


def _load(path=None):
    """The oracle library at ``path`` (default: the built oracle/liboracle.so)."""
    path = path or _build.build()
    if path not in _libs:
        lib = ctypes.CDLL(path)
        for name, args in _SIGS.items():
            fn = getattr(lib, name)
            fn.argtypes = [_CT[a] for a in args]
            fn.restype = _CT[_RES[name]]
        _libs[path] = lib
    return _libs[path]


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.float64:
        return F64
    if a.dtype == np.uint16:  # bfloat16 bit patterns
        return BF16
    raise TypeError(f"oracle reads float32, float64 or bfloat16 bits (uint16), got {a.dtype}")


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def head(q, k, v, n_sink, window, weights=False, lib=None):
    """Both attention outputs for one query row over one KV head.

    q: [d]; k, v: [L, d] (same element type; bfloat16 as uint16 bits).
    Returns (o_spec, o_exact) as float64 [d] arrays, plus (w_spec, w_exact)
    float64 [L] softmax weights when ``weights`` is true.
    """
    q = np.ascontiguousarray(q)
    k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v)
    code = _dtype_code(q)
    assert _dtype_code(k) == code and _dtype_code(v) == code
    L, d = k.shape
    o_spec = np.zeros(d, np.float64)
    o_exact = np.zeros(d, np.float64)
    w_spec = np.zeros(L, np.float64) if weights else None
    w_exact = np.zeros(L, np.float64) if weights else None
    rc = _load(lib).alspec_oracle_head(
        d, L, code, _ptr(q), _ptr(k), _ptr(v), int(n_sink), int(window),
        _ptr(o_spec), _ptr(o_exact),
        _ptr(w_spec) if weights else None, _ptr(w_exact) if weights else None)
    if rc != 0:
        raise ValueError(f"alspec_oracle_head failed with status {rc}")
    if weights:
        return o_spec, o_exact, w_spec, w_exact
    return o_spec, o_exact


def rel_l2(o_spec, o_exact, lib=None) -> float:
    """sqrt(sum (O_exact - O_spec)^2 / sum O_exact^2) over all values given."""
    a = np.ascontiguousarray(o_spec, dtype=np.float64).ravel()
    b = np.ascontiguousarray(o_exact, dtype=np.float64).ravel()
    assert a.size == b.size
    return float(_load(lib).alspec_oracle_rel_l2(_ptr(a), _ptr(b), a.size))


def commit(r: float, lam: float, lib=None) -> int:
    """1 when r <= lambda, else 0 (NaN never commits)."""
    return int(_load(lib).alspec_oracle_commit(float(r), float(lam)))


def decode(q, k, v, seq_lens, n_sink, window, lam, n_threads=0, lib=None):
    """The whole decode step.

    q: [B, Hq, d]; k, v: [B, Hkv, Lmax, d]; seq_lens: [B] int32.
    Returns dict(out_spec, out_exact [B, Hq, d] float64, rel_l2 [B] float64,
    commit [B] uint8, threads=int).  ``lib`` selects another build of the
    oracle source (the tests use this to check that mutated builds fail).
    """
    q = np.ascontiguousarray(q)
    k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v)
    seq = np.ascontiguousarray(seq_lens, dtype=np.int32)
    code = _dtype_code(q)
    assert _dtype_code(k) == code and _dtype_code(v) == code
    B, Hq, d = q.shape
    Bk, Hkv, Lmax, dk = k.shape
    assert Bk == B and dk == d and v.shape == k.shape and seq.shape == (B,)
    out_spec = np.zeros((B, Hq, d), np.float64)
    out_exact = np.zeros((B, Hq, d), np.float64)
    rel = np.zeros(B, np.float64)
    flag = np.zeros(B, np.uint8)
    used = _load(lib).alspec_oracle_decode(
        B, Hq, Hkv, d, Lmax, code, _ptr(q), _ptr(k), _ptr(v), _ptr(seq),
        int(n_sink), int(window), float(lam), _ptr(out_spec), _ptr(out_exact),
        _ptr(rel), _ptr(flag), int(n_threads))
    if used < 0:
        raise ValueError(f"alspec_oracle_decode failed with status {-used}")
    return dict(out_spec=out_spec, out_exact=out_exact, rel_l2=rel, commit=flag,
                threads=used)


def oproj(x, w, lib=None):
    """y[b, j] = sum_i x[b, i] * w[j, i] in fp64 (the projection after attention).

    x: [B, K] (any float array, widened to fp64); w: [N, K] float32, float64
    or bfloat16 bits (uint16)."""
    x = np.ascontiguousarray(np.asarray(x, np.float64).reshape(-1, np.shape(w)[-1]))
    w = np.ascontiguousarray(w)
    B, K = x.shape
    N = w.shape[0]
    y = np.zeros((B, N), np.float64)
    rc = _load(lib).alspec_oracle_oproj(B, K, N, _ptr(x), _ptr(w), _dtype_code(w), _ptr(y))
    if rc != 0:
        raise ValueError(f"oracle oproj rejected its arguments ({rc})")
    return y


def oproj_gated(o_spec, o_exact, commit, w, lib=None):
    """y[b] = oproj(commit[b] ? o_spec[b] : o_exact[b]) (commit or discard)."""
    w = np.ascontiguousarray(w)
    K = w.shape[1]
    os_ = np.ascontiguousarray(np.asarray(o_spec, np.float64).reshape(-1, K))
    oe = np.ascontiguousarray(np.asarray(o_exact, np.float64).reshape(-1, K))
    c = np.ascontiguousarray(np.asarray(commit, np.uint8).reshape(-1))
    B, N = os_.shape[0], w.shape[0]
    y = np.zeros((B, N), np.float64)
    rc = _load(lib).alspec_oracle_oproj_gated(B, K, N, _ptr(os_), _ptr(oe), _ptr(c), _ptr(w),
                                              _dtype_code(w), _ptr(y))
    if rc != 0:
        raise ValueError(f"oracle oproj_gated rejected its arguments ({rc})")
    return y
