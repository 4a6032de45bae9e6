"""Python binding of the B200 fused Gaussian kernel reduction library.

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``libgauss_b200.so`` (declared in ``include/gauss.h``); PyTorch
provides device memory and the current stream.  There is no CPU fallback: if
the shared library is missing, importing this package raises.

    gauss_sum_fwd(x, y, w, tau)           -> out [B, M, C] float32
    gauss_lse_fwd(x, y, w, tau)           -> out [B, M, C] float32
    gauss_sum_bwd(x, y, w, g, tau)        -> (grad_x [B, M, D], grad_w [B, N, C])

x [B, M, D], y [B, N, D], w [B, N, C] share one dtype (float32, float16 or
bfloat16) and must be contiguous CUDA tensors; 2-D inputs are read as B = 1.
"""
import ctypes
import os

import torch

from . import build as _build

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = _build.LIB

GS_F32, GS_F16, GS_BF16 = 0, 1, 2
GS_OP_SUM, GS_OP_LSE, GS_OP_SUM_BWD, GS_OP_LSE_BWD, GS_OP_KNN, GS_OP_DIFFUSION = 0, 1, 2, 3, 4, 5
GS_OP_SUM_FWD_BWD, GS_OP_DIFFUSION_BLOCK = 6, 7
STATUS = {0: "GS_OK", 1: "GS_ERR_INVALID_ARG", 2: "GS_ERR_UNSUPPORTED", 3: "GS_ERR_ALIGNMENT",
          4: "GS_ERR_WORKSPACE", 5: "GS_ERR_TIMEOUT", 6: "GS_ERR_CUDA"}
_DT = {torch.float32: GS_F32, torch.float16: GS_F16, torch.bfloat16: GS_BF16}

# Every symbol include/gauss.h declares, with its ctypes signature.
_i64, _f, _vp, _sz = ctypes.c_int64, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t
SIGNATURES = {
    "gs_workspace_bytes": (_sz, [ctypes.c_int, _i64, _i64, _i64, _i64, _i64, ctypes.c_int]),
    "gauss_sum_fwd": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _f,
                                     ctypes.c_int, _vp, _sz, _vp]),
    "gauss_lse_fwd": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _f,
                                     ctypes.c_int, _vp, _sz, _vp]),
    "gauss_sum_bwd": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64,
                                     _f, ctypes.c_int, _vp, _sz, _vp]),
    "gauss_sum_vjp": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64,
                                     _i64, _f, ctypes.c_int, _vp, _sz, _vp]),
    "gauss_sum_fwd_saved": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64,
                                           _f, ctypes.c_int, _vp, _sz, _vp]),
    "gauss_sum_bwd_saved": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64,
                                           _i64, _i64, _f, ctypes.c_int, _vp, _sz, _vp]),
    "gauss_lse_bwd": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64,
                                     _i64, _i64, _f, ctypes.c_int, _vp, _sz, _vp]),
    "gauss_knn": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, ctypes.c_int, _vp,
                                 _sz, _vp]),
    "gauss_diffusion_scales": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _f, _f,
                                              ctypes.c_int, _vp, _sz, _vp]),
    "gauss_diffusion_apply": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _f,
                                             ctypes.c_int, _vp, _sz, _vp]),
    "gs_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "gs_last_device_error": (ctypes.c_int, [_vp]),
    "gs_version": (ctypes.c_int, []),
    "gauss_sum_fwd_bwd": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64,
                                         _i64, _f, ctypes.c_int, _vp, _sz, _vp]),
    "gauss_diffusion_block": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _f,
                                             ctypes.c_int, _vp, _sz, _vp]),
    "gs_test_exp2_poly": (ctypes.c_int, [_vp, _vp, _i64, ctypes.c_int, _vp]),
    "gs_test_set_waits": (ctypes.c_int, [ctypes.c_uint64, ctypes.c_int]),
    "gs_test_read_error_word": (ctypes.c_int, [_vp, _vp]),
    "gs_test_ex2_probe": (ctypes.c_int, [_vp, _vp, ctypes.c_int, ctypes.c_int, _vp]),
    "gs_test_mma_probe": (ctypes.c_int, [_vp, _vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, _vp]),
    "gauss_sum_fwd_noalloc": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _f,
                                             ctypes.c_int, _vp]),
}


class GaussError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn}: {STATUS.get(status, status)} ({_lib.gs_status_string(status).decode()})")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python pairwise_reductions_b200/build.py` (needs nvcc)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


_lib = _load()


def library():
    """The loaded ctypes handle of libgauss_b200.so."""
    return _lib


def status_string(code):
    return _lib.gs_status_string(int(code)).decode()


def workspace_bytes(op, B, M, N, D, C, dtype):
    """Bytes of workspace a call needs (see gs_workspace_bytes)."""
    v = _lib.gs_workspace_bytes(int(op), B, M, N, D, C, _DT[dtype] if isinstance(dtype, torch.dtype) else int(dtype))
    if v == ctypes.c_size_t(-1).value:
        raise ValueError("gs_workspace_bytes rejected the arguments")
    return int(v)


def _as3(t, name):
    if t.dim() == 2:
        t = t.unsqueeze(0)
    if t.dim() != 3:
        raise ValueError(f"{name}: expected a 2-D or 3-D tensor, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None and t.numel() > 0 else ctypes.c_void_p(0)


def _workspace(nbytes, device, ws):
    if nbytes == 0:
        return None
    if ws is not None and ws.numel() >= nbytes:
        return ws
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def _check(fn, st):
    if st != 0:
        raise GaussError(fn, st)


def _dims(x, y, w):
    B, M, D = x.shape
    if y.shape[0] != B or y.shape[2] != D or w.shape[0] != B or w.shape[1] != y.shape[1]:
        raise ValueError(f"shape mismatch x{tuple(x.shape)} y{tuple(y.shape)} w{tuple(w.shape)}")
    if not (x.dtype == y.dtype == w.dtype) or x.dtype not in _DT:
        raise ValueError("x, y, w must share one dtype among float32, float16, bfloat16")
    return B, M, y.shape[1], D, w.shape[2]


def _reduce(name, op, x, y, w, tau, out, workspace, stream):
    x, y, w = _as3(x, "x"), _as3(y, "y"), _as3(w, "w")
    B, M, N, D, C = _dims(x, y, w)
    if out is None:
        out = torch.empty((B, M, C), dtype=torch.float32, device=x.device)
    nbytes = workspace_bytes(op, B, M, N, D, C, x.dtype)
    ws = _workspace(nbytes, x.device, workspace)
    st = getattr(_lib, name)(_ptr(x), _ptr(y), _ptr(w), _ptr(out), B, M, N, D, C, float(tau),
                             _DT[x.dtype], _ptr(ws), nbytes if ws is not None else 0,
                             _stream(stream))
    _check(name, st)
    return out


def gauss_sum_fwd(x, y, w, tau, out=None, workspace=None, stream=None):
    """out[b,i,c] = sum_j exp(-tau/2 |x_i - y_j|^2) w[b,j,c]   (float32 result)."""
    return _reduce("gauss_sum_fwd", GS_OP_SUM, x, y, w, tau, out, workspace, stream)


def gauss_sum_fwd_noalloc(x, y, w, tau, out=None, stream=None):
    """gauss_sum_fwd without a workspace: for callers that cannot allocate device
    memory; the library's fixed 32 MiB scratch array is used instead (see
    include/gauss.h for its limits: calls that overlap on the GPU race on it)."""
    x, y, w = _as3(x, "x"), _as3(y, "y"), _as3(w, "w")
    B, M, N, D, C = _dims(x, y, w)
    if out is None:
        out = torch.empty((B, M, C), dtype=torch.float32, device=x.device)
    st = _lib.gauss_sum_fwd_noalloc(_ptr(x), _ptr(y), _ptr(w), _ptr(out), B, M, N, D, C,
                                    float(tau), _DT[x.dtype], _stream(stream))
    _check("gauss_sum_fwd_noalloc", st)
    return out


def gauss_lse_fwd(x, y, w, tau, out=None, workspace=None, stream=None):
    """out[b,i,c] = log sum_j w[b,j,c] exp(-tau/2 |x_i - y_j|^2)   (w > 0)."""
    return _reduce("gauss_lse_fwd", GS_OP_LSE, x, y, w, tau, out, workspace, stream)


def gauss_sum_bwd(x, y, w, g, tau, want_x=True, want_w=True, workspace=None, stream=None):
    """Gradients of sum(g * gauss_sum_fwd(x, y, w)) with respect to x and w."""
    x, y, w, g = _as3(x, "x"), _as3(y, "y"), _as3(w, "w"), _as3(g, "g")
    B, M, N, D, C = _dims(x, y, w)
    if g.shape != (B, M, C) or g.dtype != torch.float32:
        raise ValueError(f"g must be float32 of shape {(B, M, C)}")
    gx = torch.empty((B, M, D), dtype=torch.float32, device=x.device) if want_x else None
    gw = torch.empty((B, N, C), dtype=torch.float32, device=x.device) if want_w else None
    nbytes = workspace_bytes(GS_OP_SUM_BWD, B, M, N, D, C, x.dtype)
    ws = _workspace(nbytes, x.device, workspace)
    st = _lib.gauss_sum_bwd(_ptr(x), _ptr(y), _ptr(w), _ptr(g), _ptr(gx) if want_x else None,
                            _ptr(gw) if want_w else None, B, M, N, D, C, float(tau), _DT[x.dtype],
                            _ptr(ws), nbytes if ws is not None else 0, _stream(stream))
    _check("gauss_sum_bwd", st)
    return gx, gw


def gauss_sum_fwd_saved(x, y, w, tau, out=None, saved=None, workspace=None, stream=None):
    """The forward sum plus the sums its x-gradient needs (one fused pass):
    returns (out [B, M, C], saved [B, M, C (1 + D)]) for gauss_sum_bwd_saved."""
    x, y, w = _as3(x, "x"), _as3(y, "y"), _as3(w, "w")
    B, M, N, D, C = _dims(x, y, w)
    if out is None:
        out = torch.empty((B, M, C), dtype=torch.float32, device=x.device)
    if saved is None:
        saved = torch.empty((B, M, C * (1 + D)), dtype=torch.float32, device=x.device)
    nbytes = workspace_bytes(GS_OP_SUM_BWD, B, M, N, D, C, x.dtype)
    ws = _workspace(nbytes, x.device, workspace)
    st = _lib.gauss_sum_fwd_saved(_ptr(x), _ptr(y), _ptr(w), _ptr(out), _ptr(saved), B, M, N, D, C,
                                  float(tau), _DT[x.dtype], _ptr(ws),
                                  nbytes if ws is not None else 0, _stream(stream))
    _check("gauss_sum_fwd_saved", st)
    return out, saved


def gauss_sum_bwd_saved(x, y, w, g, saved, tau, want_x=True, want_w=True, workspace=None,
                        stream=None):
    """gauss_sum_bwd from the sums gauss_sum_fwd_saved kept: (grad_x, grad_w)."""
    x, y, w, g = _as3(x, "x"), _as3(y, "y"), _as3(w, "w"), _as3(g, "g")
    B, M, N, D, C = _dims(x, y, w)
    if g.shape != (B, M, C) or g.dtype != torch.float32:
        raise ValueError(f"g must be float32 of shape {(B, M, C)}")
    if saved.shape != (B, M, C * (1 + D)) or saved.dtype != torch.float32:
        raise ValueError(f"saved must be float32 of shape {(B, M, C * (1 + D))}")
    gx = torch.empty((B, M, D), dtype=torch.float32, device=x.device) if want_x else None
    gw = torch.empty((B, N, C), dtype=torch.float32, device=x.device) if want_w else None
    nbytes = workspace_bytes(GS_OP_SUM_BWD, B, M, N, D, C, x.dtype)
    ws = _workspace(nbytes, x.device, workspace)
    st = _lib.gauss_sum_bwd_saved(_ptr(x), _ptr(y), _ptr(w), _ptr(g), _ptr(saved),
                                  _ptr(gx) if want_x else None, _ptr(gw) if want_w else None,
                                  B, M, N, D, C, float(tau), _DT[x.dtype], _ptr(ws),
                                  nbytes if ws is not None else 0, _stream(stream))
    _check("gauss_sum_bwd_saved", st)
    return gx, gw


def gauss_sum_fwd_bwd(x, y, w, g, tau, want_x=True, want_w=True, out=None, grad_x=None,
                      grad_w=None, workspace=None, stream=None):
    """Forward sum and the gradients of sum(g * out) in one call, for an upstream
    gradient g known in advance: returns (out, grad_x, grad_w) (None where not
    wanted).  fp16 / bf16 with C = 1 and D <= 47 evaluates each kernel value once."""
    x, y, w, g = _as3(x, "x"), _as3(y, "y"), _as3(w, "w"), _as3(g, "g")
    B, M, N, D, C = _dims(x, y, w)
    if g.shape != (B, M, C) or g.dtype != torch.float32:
        raise ValueError(f"g must be float32 of shape {(B, M, C)}")
    if out is None:
        out = torch.empty((B, M, C), dtype=torch.float32, device=x.device)
    if want_x and grad_x is None:
        grad_x = torch.empty((B, M, D), dtype=torch.float32, device=x.device)
    if want_w and grad_w is None:
        grad_w = torch.empty((B, N, C), dtype=torch.float32, device=x.device)
    gx = grad_x if want_x else None
    gw = grad_w if want_w else None
    nbytes = workspace_bytes(GS_OP_SUM_FWD_BWD, B, M, N, D, C, x.dtype)
    ws = _workspace(nbytes, x.device, workspace)
    st = _lib.gauss_sum_fwd_bwd(_ptr(x), _ptr(y), _ptr(w), _ptr(g), _ptr(out),
                                _ptr(gx) if want_x else None, _ptr(gw) if want_w else None,
                                B, M, N, D, C, float(tau), _DT[x.dtype], _ptr(ws),
                                nbytes if ws is not None else 0, _stream(stream))
    _check("gauss_sum_fwd_bwd", st)
    return out, gx, gw


def gauss_sum_vjp(x, y, w, g, tau, want=("x", "y", "w", "tau"), workspace=None, stream=None):
    """Every first-order gradient of sum(g * gauss_sum_fwd(x, y, w, tau)):
    returns a dict with the requested keys among x, y, w, tau."""
    x, y, w, g = _as3(x, "x"), _as3(y, "y"), _as3(w, "w"), _as3(g, "g")
    B, M, N, D, C = _dims(x, y, w)
    if g.shape != (B, M, C) or g.dtype != torch.float32:
        raise ValueError(f"g must be float32 of shape {(B, M, C)}")
    dev = x.device
    out = {"x": torch.empty((B, M, D), dtype=torch.float32, device=dev) if "x" in want else None,
           "y": torch.empty((B, N, D), dtype=torch.float32, device=dev) if "y" in want else None,
           "w": torch.empty((B, N, C), dtype=torch.float32, device=dev) if "w" in want else None,
           "tau": torch.empty((1,), dtype=torch.float32, device=dev) if "tau" in want else None}
    nbytes = workspace_bytes(GS_OP_SUM_BWD, B, M, N, D, C, x.dtype)
    ws = _workspace(nbytes, dev, workspace)
    p = lambda t: _ptr(t) if t is not None else None
    st = _lib.gauss_sum_vjp(_ptr(x), _ptr(y), _ptr(w), _ptr(g), p(out["x"]), p(out["y"]),
                            p(out["w"]), p(out["tau"]), B, M, N, D, C, float(tau), _DT[x.dtype],
                            _ptr(ws), nbytes if ws is not None else 0, _stream(stream))
    _check("gauss_sum_vjp", st)
    return {k: v for k, v in out.items() if v is not None}


def gauss_lse_bwd(x, y, w, lse, g, tau, want=("x", "y", "w", "tau"), workspace=None, stream=None):
    """Every first-order gradient of sum(g * lse) with lse = gauss_lse_fwd(x, y, w, tau);
    returns a dict with the requested keys among x, y, w, tau."""
    x, y, w, lse, g = (_as3(t, n) for t, n in ((x, "x"), (y, "y"), (w, "w"), (lse, "lse"), (g, "g")))
    B, M, N, D, C = _dims(x, y, w)
    for t, n in ((lse, "lse"), (g, "g")):
        if t.shape != (B, M, C) or t.dtype != torch.float32:
            raise ValueError(f"{n} must be float32 of shape {(B, M, C)}")
    dev = x.device
    out = {"x": torch.empty((B, M, D), dtype=torch.float32, device=dev) if "x" in want else None,
           "y": torch.empty((B, N, D), dtype=torch.float32, device=dev) if "y" in want else None,
           "w": torch.empty((B, N, C), dtype=torch.float32, device=dev) if "w" in want else None,
           "tau": torch.empty((1,), dtype=torch.float32, device=dev) if "tau" in want else None}
    nbytes = workspace_bytes(GS_OP_LSE_BWD, B, M, N, D, C, x.dtype)
    ws = _workspace(nbytes, dev, workspace)
    p = lambda t: _ptr(t) if t is not None else None
    st = _lib.gauss_lse_bwd(_ptr(x), _ptr(y), _ptr(w), _ptr(lse), _ptr(g), p(out["x"]), p(out["y"]),
                            p(out["w"]), p(out["tau"]), B, M, N, D, C, float(tau), _DT[x.dtype],
                            _ptr(ws), nbytes if ws is not None else 0, _stream(stream))
    _check("gauss_lse_bwd", st)
    return {k: v for k, v in out.items() if v is not None}


def gauss_knn(x, y, K, workspace=None, stream=None):
    """K smallest squared distances per row (ascending, ties by the lower index)
    and their int64 indices, decided in fp32 (fp16 / bf16 inputs exactly widened)."""
    x, y = _as3(x, "x"), _as3(y, "y")
    B, M, D = x.shape
    N = y.shape[1]
    if y.shape[0] != B or y.shape[2] != D or x.dtype != y.dtype or x.dtype not in _DT:
        raise ValueError(f"shape/dtype mismatch x{tuple(x.shape)} y{tuple(y.shape)}")
    od = torch.empty((B, M, K), dtype=torch.float32, device=x.device)
    oi = torch.empty((B, M, K), dtype=torch.int64, device=x.device)
    nbytes = workspace_bytes(GS_OP_KNN, B, M, N, D, K, x.dtype)
    ws = _workspace(nbytes, x.device, workspace)
    st = _lib.gauss_knn(_ptr(x), _ptr(y), _ptr(od), _ptr(oi), B, M, N, D, int(K), _DT[x.dtype],
                        _ptr(ws), nbytes if ws is not None else 0, _stream(stream))
    _check("gauss_knn", st)
    return od, oi


def gauss_diffusion_block(x_rows, x_cols, v, tau, out=None, workspace=None, stream=None):
    """K(x_rows, x_cols) v with float32 values v [B, N, C] whatever the points' dtype."""
    xr, xc, v = _as3(x_rows, "x_rows"), _as3(x_cols, "x_cols"), _as3(v, "v")
    B, M, D = xr.shape
    N, C = xc.shape[1], v.shape[2]
    if (xc.shape[0] != B or xc.shape[2] != D or xc.dtype != xr.dtype or v.shape[:2] != (B, N)
            or v.dtype != torch.float32):
        raise ValueError(f"shape/dtype mismatch x_rows{tuple(xr.shape)} x_cols{tuple(xc.shape)} "
                         f"v{tuple(v.shape)}")
    if out is None:
        out = torch.empty((B, M, C), dtype=torch.float32, device=xr.device)
    nbytes = workspace_bytes(GS_OP_DIFFUSION_BLOCK, B, M, N, D, C, xr.dtype)
    ws = _workspace(nbytes, xr.device, workspace)
    st = _lib.gauss_diffusion_block(_ptr(xr), _ptr(xc), _ptr(v), _ptr(out), B, M, N, D, C, float(tau),
                                    _DT[xr.dtype], _ptr(ws), nbytes if ws is not None else 0,
                                    _stream(stream))
    _check("gauss_diffusion_block", st)
    return out


def gauss_diffusion_scales(x, tau, alpha, workspace=None, stream=None):
    """(q, d, s) of the alpha-normalised diffusion operator over the point set x."""
    x = _as3(x, "x")
    B, N, D = x.shape
    q, d, s = (torch.empty((B, N), dtype=torch.float32, device=x.device) for _ in range(3))
    nbytes = workspace_bytes(GS_OP_DIFFUSION, B, N, N, D, 1, x.dtype)
    ws = _workspace(nbytes, x.device, workspace)
    st = _lib.gauss_diffusion_scales(_ptr(x), _ptr(q), _ptr(d), _ptr(s), B, N, D, float(tau),
                                     float(alpha), _DT[x.dtype], _ptr(ws),
                                     nbytes if ws is not None else 0, _stream(stream))
    _check("gauss_diffusion_scales", st)
    return q, d, s


def gauss_diffusion_apply(x, s, v, tau, out=None, workspace=None, stream=None):
    """diag(s) K diag(s) v over the point set x (float32 s, v)."""
    x, v = _as3(x, "x"), _as3(v, "v")
    B, N, D = x.shape
    C = v.shape[2]
    if out is None:
        out = torch.empty((B, N, C), dtype=torch.float32, device=x.device)
    nbytes = workspace_bytes(GS_OP_DIFFUSION, B, N, N, D, C, x.dtype)
    ws = _workspace(nbytes, x.device, workspace)
    st = _lib.gauss_diffusion_apply(_ptr(x), _ptr(s.contiguous()), _ptr(v), _ptr(out), B, N, D, C,
                                    float(tau), _DT[x.dtype], _ptr(ws),
                                    nbytes if ws is not None else 0, _stream(stream))
    _check("gauss_diffusion_apply", st)
    return out


def test_exp2_poly(x, degree, stream=None):
    """Device evaluation of the FMA-pipe 2^x (test hook, see include/gauss_testing.h)."""
    if x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous float32 CUDA tensor")
    out = torch.empty_like(x)
    _check("gs_test_exp2_poly", _lib.gs_test_exp2_poly(_ptr(x), _ptr(out), x.numel(), int(degree),
                                                       _stream(stream)))
    return out


def test_set_waits(limit_ns, stall):
    """Wait limit and stall mode of the tensor-core kernels (test hook, see
    include/gauss_testing.h); restore with test_set_waits(2_000_000_000, 0)."""
    _check("gs_test_set_waits", _lib.gs_test_set_waits(int(limit_ns), int(stall)))


def test_read_error_word(stream=None):
    """Synchronise, then read and clear the raw device error word (test hook,
    see include/gauss_testing.h): bit 0 a wait ran out, bit 1 mismatched boxes,
    bit 2 a drain wait ran out."""
    word = ctypes.c_int(0)
    _check("gs_test_read_error_word", _lib.gs_test_read_error_word(ctypes.byref(word),
                                                                   _stream(stream)))
    return word.value


def test_ex2_probe(blocks, iters, stream=None):
    """SM cycles of each CTA of the MUFU ex2 rate probe (test hook, see
    include/gauss_testing.h): CTA b evaluated 1024 * 8 * iters exponentials."""
    dev = torch.device("cuda", torch.cuda.current_device())
    cycles = torch.zeros(int(blocks), dtype=torch.int64, device=dev)
    sink = torch.empty(int(blocks) * 1024, dtype=torch.float32, device=dev)
    _check("gs_test_ex2_probe", _lib.gs_test_ex2_probe(_ptr(cycles), _ptr(sink), int(blocks),
                                                       int(iters), _stream(stream)))
    return cycles


def test_mma_probe(blocks, n_mma, n_cols, stream=None):
    """SM cycles of each CTA of the tcgen05.mma issue probe (test hook, see
    include/gauss_testing.h), and the status word (0: every wait completed)."""
    dev = torch.device("cuda", torch.cuda.current_device())
    cycles = torch.zeros(int(blocks), dtype=torch.int64, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    _check("gs_test_mma_probe", _lib.gs_test_mma_probe(_ptr(cycles), _ptr(status), int(blocks),
                                                       int(n_mma), int(n_cols), _stream(stream)))
    return cycles, status


def last_device_error(stream=None):
    """Synchronise and read/clear the device error word (0 = none)."""
    return int(_lib.gs_last_device_error(_stream(stream)))


__all__ = ["gauss_sum_fwd", "gauss_sum_fwd_noalloc", "gauss_lse_fwd", "gauss_sum_bwd",
           "gauss_sum_fwd_saved", "gauss_sum_bwd_saved", "gauss_sum_fwd_bwd", "gauss_sum_vjp", "gauss_lse_bwd", "gauss_knn", "gauss_diffusion_block", "gauss_diffusion_scales", "gauss_diffusion_apply", "workspace_bytes",
           "last_device_error", "library", "status_string", "GaussError", "SIGNATURES",
           "LIB_PATH"]
