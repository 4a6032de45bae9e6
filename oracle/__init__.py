"""Plain double-precision CPU oracle for the fused Gaussian kernel reductions.

TEST INFRASTRUCTURE ONLY: the test-suite, the smoke check and the benchmark's
CPU-baseline leg may import this package; the product library never does.
It shares no code with the CUDA path.  The arithmetic lives in
``gauss_oracle.c``; this module only loads it and marshals numpy arrays.

Functions, each the plain definition ("Kernel matrix reduction", Implementation
sketch, eq. 1 and eq. 2; "Fast Gauss Sums via Flash Attention", Algorithm 1,
step 2):

* ``gauss_sum(x, y, w, tau, rows=None)``  -> [B, R, C]
* ``gauss_lse(x, y, w, tau, rows=None)``  -> [B, R, C]
* ``gauss_sum_bwd(x, y, w, g, tau, rows=None, wrows=None)`` -> (grad_x, grad_w)
* ``gauss_sum_vjp_y_tau(x, y, w, g, tau, yrows=None)`` -> (grad_y, grad_tau)
* ``gauss_lse_bwd(x, y, w, g, tau)`` -> (grad_x, grad_y, grad_w, grad_tau)
* ``knn(x, y, K, rows=None, f32=False)`` -> (sq_dist [B, R, K], index [B, R, K])
* ``diffusion_scales(x, tau, alpha)`` -> (q, d, s) and ``diffusion_apply(x, s, v, tau)``

Inputs are float64 arrays x [B,M,D], y [B,N,D], w [B,N,C], g [B,M,C] (2-D
arrays are read as B = 1).  Values must already be the quantised values the
device sees (fp16/bf16/fp32 widened to double).
"""
import ctypes
import os

import numpy as np

from .build import LIB, build_oracle

_lib = None
_i64 = ctypes.c_int64
_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int64)


def _load(path=None):
    global _lib
    if path is not None:
        lib = ctypes.CDLL(path)
    else:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build_oracle())
    for name in ("oracle_gauss_sum", "oracle_gauss_lse"):
        f = getattr(lib, name)
        f.restype = ctypes.c_int
        f.argtypes = [_dp, _dp, _dp, _dp, _i64, _i64, _i64, _i64, _i64,
                      ctypes.c_double, _ip, _i64]
    f = lib.oracle_gauss_sum_bwd
    f.restype = ctypes.c_int
    f.argtypes = [_dp, _dp, _dp, _dp, _dp, _dp, _i64, _i64, _i64, _i64, _i64,
                  ctypes.c_double, _ip, _i64, _ip, _i64]
    f = lib.oracle_gauss_sum_vjp_y_tau
    f.restype = ctypes.c_int
    f.argtypes = [_dp, _dp, _dp, _dp, _dp, _dp, _i64, _i64, _i64, _i64, _i64, ctypes.c_double,
                  _ip, _i64]
    f = lib.oracle_gauss_lse_bwd
    f.restype = ctypes.c_int
    f.argtypes = [_dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _i64, _i64, _i64, _i64, _i64,
                  ctypes.c_double]
    _fp = ctypes.POINTER(ctypes.c_float)
    f = lib.oracle_knn
    f.restype = ctypes.c_int
    f.argtypes = [_dp, _dp, _dp, _ip, _i64, _i64, _i64, _i64, _i64, _ip, _i64]
    f = lib.oracle_knn_f32
    f.restype = ctypes.c_int
    f.argtypes = [_fp, _fp, _fp, _ip, _i64, _i64, _i64, _i64, _i64, _ip, _i64]
    f = lib.oracle_diffusion_scales
    f.restype = ctypes.c_int
    f.argtypes = [_dp, _dp, _dp, _dp, _i64, _i64, _i64, ctypes.c_double, ctypes.c_double]
    f = lib.oracle_diffusion_apply
    f.restype = ctypes.c_int
    f.argtypes = [_dp, _dp, _dp, _dp, _i64, _i64, _i64, _i64, ctypes.c_double]
    lib.oracle_num_threads.restype = ctypes.c_int
    if path is None:
        _lib = lib
    return lib


def num_threads():
    """Threads the oracle's OpenMP loops use."""
    return int(_load().oracle_num_threads())


def _as3(a, name):
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float64))
    if a.ndim == 2:
        a = a[None]
    if a.ndim != 3:
        raise ValueError(f"{name}: expected a 2-D or 3-D array, got shape {a.shape}")
    return a


def _ptr(a):
    return a.ctypes.data_as(_dp) if a is not None else None


def _rows(rows):
    if rows is None:
        return None, 0, None
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    return r, int(r.size), r.ctypes.data_as(_ip)


def _check(x, y, w):
    B, M, D = x.shape
    if y.shape[0] != B or y.shape[2] != D or w.shape[0] != B or w.shape[1] != y.shape[1]:
        raise ValueError(f"shape mismatch x{x.shape} y{y.shape} w{w.shape}")
    return B, M, y.shape[1], D, w.shape[2]


def _reduce(fn_name, x, y, w, tau, rows, lib):
    x, y, w = _as3(x, "x"), _as3(y, "y"), _as3(w, "w")
    B, M, N, D, C = _check(x, y, w)
    r, nr, rp = _rows(rows)
    R = nr if r is not None else M
    out = np.empty((B, R, C), dtype=np.float64)
    rc = getattr(lib or _load(), fn_name)(_ptr(x), _ptr(y), _ptr(w), _ptr(out), B, M, N, D, C,
                                          float(tau), rp, nr)
    if rc != 0:
        raise ValueError(f"{fn_name} rejected its arguments (code {rc})")
    return out


def gauss_sum(x, y, w, tau, rows=None, lib=None):
    """out[b,i,c] = sum_j exp(-tau/2 |x_i - y_j|^2) w[b,j,c]."""
    return _reduce("oracle_gauss_sum", x, y, w, tau, rows, lib)


def gauss_lse(x, y, w, tau, rows=None, lib=None):
    """out[b,i,c] = log sum_j w[b,j,c] exp(-tau/2 |x_i - y_j|^2), max-shifted."""
    return _reduce("oracle_gauss_lse", x, y, w, tau, rows, lib)


def gauss_sum_bwd(x, y, w, g, tau, rows=None, wrows=None, want_x=True, want_w=True, lib=None):
    """Gradients of sum(g * gauss_sum(x, y, w)) with respect to x and w."""
    x, y, w, g = _as3(x, "x"), _as3(y, "y"), _as3(w, "w"), _as3(g, "g")
    B, M, N, D, C = _check(x, y, w)
    if g.shape != (B, M, C):
        raise ValueError(f"g must be {(B, M, C)}, got {g.shape}")
    r, nr, rp = _rows(rows)
    rw, nrw, rwp = _rows(wrows)
    R = nr if r is not None else M
    Rw = nrw if rw is not None else N
    gx = np.empty((B, R, D), dtype=np.float64) if want_x else None
    gw = np.empty((B, Rw, C), dtype=np.float64) if want_w else None
    rc = (lib or _load()).oracle_gauss_sum_bwd(_ptr(x), _ptr(y), _ptr(w), _ptr(g), _ptr(gx),
                                              _ptr(gw), B, M, N, D, C, float(tau), rp, nr,
                                              rwp, nrw)
    if rc != 0:
        raise ValueError(f"oracle_gauss_sum_bwd rejected its arguments (code {rc})")
    return gx, gw


def gauss_sum_vjp_y_tau(x, y, w, g, tau, yrows=None, want_y=True, want_tau=True, lib=None):
    """Gradients of sum(g * gauss_sum(x, y, w)) with respect to y and tau."""
    x, y, w, g = _as3(x, "x"), _as3(y, "y"), _as3(w, "w"), _as3(g, "g")
    B, M, N, D, C = _check(x, y, w)
    if g.shape != (B, M, C):
        raise ValueError(f"g must be {(B, M, C)}, got {g.shape}")
    r, nr, rp = _rows(yrows)
    R = nr if r is not None else N
    gy = np.empty((B, R, D), dtype=np.float64) if want_y else None
    gt = np.zeros(1, dtype=np.float64) if want_tau else None
    rc = (lib or _load()).oracle_gauss_sum_vjp_y_tau(_ptr(x), _ptr(y), _ptr(w), _ptr(g), _ptr(gy),
                                                    _ptr(gt), B, M, N, D, C, float(tau), rp, nr)
    if rc != 0:
        raise ValueError(f"oracle_gauss_sum_vjp_y_tau rejected its arguments (code {rc})")
    return gy, (float(gt[0]) if want_tau else None)


def gauss_lse_bwd(x, y, w, g, tau, lib=None):
    """Gradients of sum(g * gauss_lse(x, y, w)) w.r.t. x, y, w and tau (small sizes)."""
    x, y, w, g = _as3(x, "x"), _as3(y, "y"), _as3(w, "w"), _as3(g, "g")
    B, M, N, D, C = _check(x, y, w)
    if g.shape != (B, M, C):
        raise ValueError(f"g must be {(B, M, C)}, got {g.shape}")
    gx = np.empty((B, M, D)); gy = np.empty((B, N, D)); gw = np.empty((B, N, C))
    gt = np.zeros(1)
    rc = (lib or _load()).oracle_gauss_lse_bwd(_ptr(x), _ptr(y), _ptr(w), _ptr(g), _ptr(gx), _ptr(gy),
                                              _ptr(gw), _ptr(gt), B, M, N, D, C, float(tau))
    if rc != 0:
        raise ValueError(f"oracle_gauss_lse_bwd rejected its arguments (code {rc})")
    return gx, gy, gw, float(gt[0])


def knn(x, y, K, rows=None, lib=None, f32=False):
    """K smallest squared distances |x_i - y_j|^2 per row (ascending, ties by lower j)
    and their indices; f32=True decides in float (fixed order of operations)."""
    if f32:
        x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
        y = np.ascontiguousarray(np.asarray(y, dtype=np.float32))
        if x.ndim == 2:
            x, y = x[None], y[None]
    else:
        x, y = _as3(x, "x"), _as3(y, "y")
    B, M, D = x.shape
    N = y.shape[1]
    if y.shape[0] != B or y.shape[2] != D:
        raise ValueError(f"shape mismatch x{x.shape} y{y.shape}")
    r, nr, rp = _rows(rows)
    R = nr if r is not None else M
    od = np.empty((B, R, K), dtype=np.float32 if f32 else np.float64)
    oi = np.empty((B, R, K), dtype=np.int64)
    L = lib or _load()
    if f32:
        fp = ctypes.POINTER(ctypes.c_float)
        rc = L.oracle_knn_f32(x.ctypes.data_as(fp), y.ctypes.data_as(fp), od.ctypes.data_as(fp),
                              oi.ctypes.data_as(_ip), B, M, N, D, int(K), rp, nr)
    else:
        rc = L.oracle_knn(_ptr(x), _ptr(y), _ptr(od), oi.ctypes.data_as(_ip), B, M, N, D, int(K), rp, nr)
    if rc != 0:
        raise ValueError(f"oracle knn rejected its arguments (code {rc})")
    return od, oi


def diffusion_scales(x, tau, alpha, lib=None):
    """(q, d, s) of the alpha-normalised diffusion operator over the point set x."""
    x = _as3(x, "x")
    B, N, D = x.shape
    q, d, s = (np.empty((B, N)) for _ in range(3))
    rc = (lib or _load()).oracle_diffusion_scales(_ptr(x), _ptr(q), _ptr(d), _ptr(s), B, N, D,
                                                 float(tau), float(alpha))
    if rc != 0:
        raise ValueError(f"oracle_diffusion_scales rejected its arguments (code {rc})")
    return q, d, s


def diffusion_apply(x, s, v, tau, lib=None):
    """diag(s) K diag(s) v over the point set x."""
    x, v = _as3(x, "x"), _as3(v, "v")
    B, N, D = x.shape
    C = v.shape[2]
    s = np.ascontiguousarray(np.asarray(s, dtype=np.float64).reshape(B, N))
    out = np.empty((B, N, C))
    rc = (lib or _load()).oracle_diffusion_apply(_ptr(x), _ptr(s), _ptr(v), _ptr(out), B, N, D, C,
                                                float(tau))
    if rc != 0:
        raise ValueError(f"oracle_diffusion_apply rejected its arguments (code {rc})")
    return out


__all__ = ["diffusion_scales", "diffusion_apply", "knn", "gauss_sum_vjp_y_tau", "gauss_lse_bwd", "gauss_sum", "gauss_lse", "gauss_sum_bwd", "num_threads", "build_oracle", "LIB"]
