"""torch.autograd wrappers: gradients through the fused reductions.

"Kernel matrix reduction" (Variants) and the LazyTensor API of "KeOps: a
symbolic tensor that never materialises the matrix it represents" take
gradients of a kernel reduction with torch.autograd.grad; these functions give
the same for this library's Gaussian sum and log-sum-exp.  They only marshal:
the forward and the backward are the library's entry points.

    a = gauss_sum(x, y, w, tau)      # [B, M, C] float32, differentiable in x, y, w, tau
    l = gauss_lse(x, y, w, tau)      # log-sum-exp, w > 0

`tau` may be a float or a 0-d / 1-element tensor (differentiable if it
requires grad).  When only x and w need gradients, the sum's forward keeps the
sums its x-gradient needs (gauss_sum_fwd_saved), so forward + backward cost two
passes; otherwise the backward is gauss_sum_vjp.  Gradients are returned in the
dtype of the input they belong to.

`kernels` replaces the six library calls (a dict with the keys of
`_default_kernels`, same signatures); the default is the CUDA library.
"""
import torch


def _default_kernels():
    from . import (gauss_lse_bwd, gauss_lse_fwd, gauss_sum_bwd_saved, gauss_sum_fwd,
                   gauss_sum_fwd_saved, gauss_sum_vjp)
    return {"sum_fwd": gauss_sum_fwd, "sum_fwd_saved": gauss_sum_fwd_saved,
            "sum_bwd_saved": gauss_sum_bwd_saved, "sum_vjp": gauss_sum_vjp,
            "lse_fwd": gauss_lse_fwd, "lse_bwd": gauss_lse_bwd}


def _tau_value(tau):
    if not torch.is_tensor(tau):
        return float(tau)
    if tau.numel() != 1:
        raise ValueError(f"tau must hold one value, got shape {tuple(tau.shape)}")
    return float(tau.detach().reshape(-1)[0].item())


def _cast(g, like):
    return None if g is None else g.to(like.dtype).reshape(like.shape)


def _tau_grad(r, ctx):
    return r["tau"].reshape(ctx.tau_shape) if "tau" in r else None


def _setup(ctx, x, y, w, tau, tau_t, kernels):
    ctx.tau = tau
    ctx.k = kernels or _default_kernels()
    ctx.tau_shape = tau_t.shape if tau_t is not None else ()
    ctx.squeeze = x.dim() == 2
    return x.contiguous(), y.contiguous(), w.contiguous()


def _out(ctx, out):
    return out.squeeze(0) if ctx.squeeze else out


class _GaussSum(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, y, w, tau, tau_t, kernels):
        need_x, need_y, need_w = ctx.needs_input_grad[0:3]
        need_tau = tau_t is not None and ctx.needs_input_grad[4]
        x, y, w = _setup(ctx, x, y, w, tau, tau_t, kernels)
        ctx.saved_mode = (need_x or need_w) and not need_y and not need_tau
        if ctx.saved_mode:
            out, saved = ctx.k["sum_fwd_saved"](x, y, w, tau)
            ctx.save_for_backward(x, y, w, saved)
        else:
            out = ctx.k["sum_fwd"](x, y, w, tau)
            ctx.save_for_backward(x, y, w)
        return _out(ctx, out)

    @staticmethod
    def backward(ctx, g):
        g = g.contiguous()   # (the output's dtype: float32 from the library)
        need_x, need_y, need_w = ctx.needs_input_grad[0:3]
        need_tau = ctx.needs_input_grad[4]
        if ctx.saved_mode:
            x, y, w, saved = ctx.saved_tensors
            gx, gw = ctx.k["sum_bwd_saved"](x, y, w, g, saved, ctx.tau, want_x=need_x, want_w=need_w)
            return _cast(gx, x), None, _cast(gw, w), None, None, None
        x, y, w = ctx.saved_tensors
        want = tuple(k for k, n in (("x", need_x), ("y", need_y), ("w", need_w), ("tau", need_tau))
                     if n)
        if not want:
            return None, None, None, None, None, None
        r = ctx.k["sum_vjp"](x, y, w, g, ctx.tau, want=want)
        return (_cast(r.get("x"), x), _cast(r.get("y"), y), _cast(r.get("w"), w), None,
                _tau_grad(r, ctx), None)


class _GaussLse(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, y, w, tau, tau_t, kernels):
        x, y, w = _setup(ctx, x, y, w, tau, tau_t, kernels)
        out = ctx.k["lse_fwd"](x, y, w, tau)
        ctx.save_for_backward(x, y, w, out)
        return _out(ctx, out)

    @staticmethod
    def backward(ctx, g):
        x, y, w, lse = ctx.saved_tensors
        need = dict(zip(("x", "y", "w"), ctx.needs_input_grad[0:3]))
        need["tau"] = ctx.needs_input_grad[4]
        want = tuple(k for k, n in need.items() if n)
        if not want:
            return None, None, None, None, None, None
        g = g.contiguous().to(lse.dtype).reshape(lse.shape)
        r = ctx.k["lse_bwd"](x, y, w, lse, g, ctx.tau, want=want)
        return (_cast(r.get("x"), x), _cast(r.get("y"), y), _cast(r.get("w"), w), None,
                _tau_grad(r, ctx), None)


def gauss_sum(x, y, w, tau, kernels=None):
    """sum_j exp(-tau/2 |x_i - y_j|^2) w_j, differentiable in x, y, w and tau."""
    tau_t = tau if torch.is_tensor(tau) else None
    return _GaussSum.apply(x, y, w, _tau_value(tau), tau_t, kernels)


def gauss_lse(x, y, w, tau, kernels=None):
    """log sum_j w_j exp(-tau/2 |x_i - y_j|^2) (w > 0), differentiable in x, y, w and tau."""
    tau_t = tau if torch.is_tensor(tau) else None
    return _GaussLse.apply(x, y, w, _tau_value(tau), tau_t, kernels)


__all__ = ["gauss_sum", "gauss_lse"]
