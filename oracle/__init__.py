"""fp64 CPU oracle for the generalized-causal GQA attention with 2D RoPE.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / reference leg of ``bench.py``.  The product path
(``joint_text_image_b200``) never imports it.  The arithmetic lives in
``oracle.c`` (plain C, fp64); this module only marshals numpy arrays.

Every function cites its passage in ``oracle.c``.  Parity pins live in
``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (plain gcc, IEEE fp64, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-std=c11",
                               "-D_GNU_SOURCE", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        D = ctypes.c_double
        G = [P, P, P, P, P]  # flat geometry: n_img, text_before, img_h, img_w, suffix
        lib.oracle_mask.argtypes = [I, I, *G, P]
        lib.oracle_positions.argtypes = [I, I, *G, P, P]
        lib.oracle_rope_tables.argtypes = [I, I, I, *G, D, P, P]
        lib.oracle_rope_apply.argtypes = [I, I, I, I, *G, D, I, P, P]
        lib.oracle_attn_fwd.argtypes = [I, I, I, I, I, *G, P, P, P, D, D, I, P, I, P, P, P, D, P, P, I]
        lib.oracle_attn_bwd.argtypes = [I, I, I, I, I, *G, P, P, P, P, D, D, I, P, I, P, P, P, D,
                                        P, P, P, P, P, I]
        _lib = lib
    return _lib


def _geom(samples):
    """Flat geometry (oracle.c, ogeom) from samples given either as
    (prefix, img_h, img_w, suffix) -- one image, or text only when h = w = 0 --
    or as (images, suffix) with images a list of (text_before, img_h, img_w):
    returns the int32 arrays n_img, text_before, img_h, img_w, suffix."""
    n_img, tb, hh, ww, suf = [], [], [], [], []
    for smp in samples:
        if len(smp) == 2:
            images, suffix = smp
        else:
            p, h, w, sfx = smp
            if min(p, h, w, sfx) < 0 or (h == 0) != (w == 0):
                images, suffix = [(-1, 0, 0)], -1  # bad geometry: refused by the C side
            elif h == 0:
                images, suffix = [], p + sfx
            else:
                images, suffix = [(p, h, w)], sfx
        n_img.append(len(images))
        for (t, h, w) in images:
            tb.append(t)
            hh.append(h)
            ww.append(w)
        suf.append(suffix)
    arr = lambda x: np.ascontiguousarray(np.asarray(x if x else [0], dtype=np.int32))
    return [arr(n_img), arr(tb), arr(hh), arr(ww), arr(suf)]


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def mask(samples, S: int) -> np.ndarray:
    """uint8 [B, S, S] indexed [b, query, key] from the literal rule."""
    g = _geom(samples)
    out = np.zeros((len(samples), S, S), dtype=np.uint8)
    if _load().oracle_mask(len(samples), S, *map(_p, g), _p(out)) != 0:
        raise ValueError("bad sample geometry")
    return out


def positions(samples, S: int):
    """(x, y) int64 [B, S] 2D RoPE positions."""
    g = _geom(samples)
    B = len(samples)
    x = np.zeros((B, S), dtype=np.int64)
    y = np.zeros((B, S), dtype=np.int64)
    if _load().oracle_positions(B, S, *map(_p, g), _p(x), _p(y)) != 0:
        raise ValueError("bad sample geometry")
    return x, y


def rope_tables(samples, S: int, D: int, base: float = 10000.0):
    """(cos, sin) fp64 [B, S, D]."""
    g = _geom(samples)
    B = len(samples)
    c = np.zeros((B, S, D))
    s = np.zeros((B, S, D))
    if _load().oracle_rope_tables(B, S, D, *map(_p, g), float(base), _p(c), _p(s)) != 0:
        raise ValueError("bad arguments")
    return c, s


def rope_apply(samples, x: np.ndarray, base: float = 10000.0, inverse: bool = False):
    """R x (or R^T x) for x fp64 [B, S, H, D]."""
    g = _geom(samples)
    x = np.ascontiguousarray(x, dtype=np.float64)
    B, S, H, D = x.shape
    y = np.zeros_like(x)
    if _load().oracle_rope_apply(B, S, H, D, *map(_p, g), float(base), int(inverse), _p(x), _p(y)) != 0:
        raise ValueError("bad arguments")
    return y


def _norm_args(qk_norm, D):
    """qk_norm = (wq [D], wk [D], eps) or None -> (wq, wk, eps) for the C call."""
    if qk_norm is None:
        return None, None, 0.0
    wq, wk, eps = qk_norm
    wq = np.ascontiguousarray(wq, dtype=np.float64).reshape(D)
    wk = np.ascontiguousarray(wk, dtype=np.float64).reshape(D)
    return wq, wk, float(eps)


def attn_fwd(samples, q, k, v, scale=None, base=10000.0, rotate=True, rows=None,
             groups=None, nthreads=0, qk_norm=None):
    """Forward: returns (o [B,S,Hq,D], lse [B,Hq,S], threads_used).

    q [B,S,Hq,D], k/v [B,S,Hkv,D] as fp64 (exact copies of the bf16 inputs).
    rows: optional int list of query rows; groups: optional bool [B, Hkv].
    qk_norm: optional (wq [D], wk [D], eps): per-head RMSNorm of the rotated
    q and k rows (oracle.c, rms_norm)."""
    g = _geom(samples)
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int32)
    gs = None if groups is None else np.ascontiguousarray(groups, dtype=np.uint8).reshape(-1)
    wq, wk, eps = _norm_args(qk_norm, D)
    o = np.zeros((B, S, Hq, D))
    lse = np.zeros((B, Hq, S))
    used = _load().oracle_attn_fwd(B, S, Hq, Hkv, D, *map(_p, g), _p(q), _p(k), _p(v),
                                   float(scale), float(base), int(rotate), _p(r),
                                   0 if r is None else len(r), _p(gs), _p(wq), _p(wk), eps,
                                   _p(o), _p(lse), int(nthreads))
    if used < 0:
        raise ValueError("bad arguments")
    return o, lse, used


def attn_bwd(samples, q, k, v, dout, scale=None, base=10000.0, rotate=True, groups=None,
             nthreads=0, rows=None):
    """Backward: returns (dq [B,S,Hq,D], dk, dv [B,S,Hkv,D], threads_used).

    rows: optional query-row subset (dq of those rows; dk, dv summed over them)."""
    dq, dk, dv, _, _, used = _attn_bwd(samples, q, k, v, dout, scale, base, rotate, groups,
                                       nthreads, rows, None)
    return dq, dk, dv, used


def attn_bwd_qknorm(samples, q, k, v, dout, qk_norm, scale=None, base=10000.0, rotate=True,
                    groups=None, nthreads=0, rows=None):
    """Backward with the per-head QK RMSNorm qk_norm = (wq, wk, eps): returns
    (dq, dk, dv, dwq [D], dwk [D], threads_used) (oracle.c, rms_norm_vjp)."""
    return _attn_bwd(samples, q, k, v, dout, scale, base, rotate, groups, nthreads, rows, qk_norm)


def _attn_bwd(samples, q, k, v, dout, scale, base, rotate, groups, nthreads, rows, qk_norm):
    g = _geom(samples)
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    dout = np.ascontiguousarray(dout, dtype=np.float64)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    gs = None if groups is None else np.ascontiguousarray(groups, dtype=np.uint8).reshape(-1)
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int32)
    wq, wk, eps = _norm_args(qk_norm, D)
    dq = np.zeros((B, S, Hq, D))
    dk = np.zeros((B, S, Hkv, D))
    dv = np.zeros((B, S, Hkv, D))
    dwq = np.zeros(D) if qk_norm is not None else None
    dwk = np.zeros(D) if qk_norm is not None else None
    used = _load().oracle_attn_bwd(B, S, Hq, Hkv, D, *map(_p, g), _p(q), _p(k), _p(v), _p(dout),
                                   float(scale), float(base), int(rotate), _p(r),
                                   0 if r is None else len(r), _p(gs), _p(wq), _p(wk), eps,
                                   _p(dq), _p(dk), _p(dv), _p(dwq), _p(dwk), int(nthreads))
    if used < 0:
        raise ValueError("bad arguments")
    return dq, dk, dv, dwq, dwk, used
