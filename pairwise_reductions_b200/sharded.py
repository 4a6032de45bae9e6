"""One Gauss-sum problem sharded over the ranks of a process group.

The rows of a Gauss sum are independent once every source is known, so a
problem splits by rows with a single exchange of the sources: rank r holds the
query rows x_r and a shard (y_r, w_r) of the sources; one all-gather gives every
rank the whole (y, w), and rank r computes its rows.  "FlashDiffusion" (§3,
multi-GPU runs) shards its kernel application over the row axis the same way.
The gradient adds one more exchange: dL/dx of the local rows needs (y, w) as
above, while dL/dw and dL/dy of the local sources need every row and its
upstream gradient, i.e. an all-gather of (x, g).

The log-sum-exp backward shards the same way: dL/dx of the local rows (and
their share of dL/dtau) against the gathered (y, w); dL/dy and dL/dw of the
local sources against the gathered (x, g, lse) -- the backward takes the
forward's lse of every row as an input, so a pass over a subset of the sources
still normalises by the full sum --; the dL/dtau shares are summed over the
ranks.

The diffusion operator of "FlashDiffusion" (§2.2: q = K 1, d = q^-alpha
(K q^-alpha), s = q^-alpha d^-1/2, then diag(s) K diag(s) V) shards by rows of
its one point set: every rank needs every point (one all-gather of x), then
the q^-alpha of every point for its rows of d (a second all-gather), and for
the operator the s V of every point (a third).  Each rank's rows of q, d, s and
of the operator's output are its own; the pair work is
`gauss_diffusion_block` (rows of this rank, columns of every rank, float32
values), the per-point arithmetic between the passes is elementwise.

The exchanges are `torch.distributed` collectives on the group's backend (NCCL
over NVLink for CUDA tensors); the pair work runs in this library's kernels
(`gauss_sum_fwd`, `gauss_lse_fwd`, `gauss_sum_bwd`, `gauss_sum_vjp`,
`gauss_lse_bwd`).  Shards
may differ in size; they are concatenated in rank order.  Every rank makes the
same calls with the same `want`, so the collectives match.

`kernels` replaces the compute calls (same signatures); the default is the
CUDA library.  `row_counts` / `src_counts` (every rank's number of rows /
sources, from `shard_counts`) spare each gather the exchange of the counts and
its host synchronisation; without them the counts are exchanged every call.
"""
import torch
import torch.distributed as dist


def _default_kernels():
    from . import (gauss_diffusion_block, gauss_lse_bwd, gauss_lse_fwd, gauss_sum_bwd,
                   gauss_sum_fwd, gauss_sum_vjp)
    return {"sum": gauss_sum_fwd, "lse": gauss_lse_fwd, "bwd": gauss_sum_bwd,
            "lse_bwd": gauss_lse_bwd, "vjp": gauss_sum_vjp, "block": gauss_diffusion_block}


def shard_counts(n_local, device, group=None):
    """Every rank's n_local, in rank order (one small all-gather and a host sync)."""
    world = dist.get_world_size(group)
    n = torch.tensor([n_local], dtype=torch.int64, device=device)
    counts = [torch.zeros_like(n) for _ in range(world)]
    dist.all_gather(counts, n, group=group)
    return [int(c.item()) for c in counts]


def all_gather_rows(t, group=None, counts=None):
    """Concatenate every rank's t [B, n_r, ...] along dim 1, in rank order.

    Shards may have different n_r (`counts`, exchanged here when not given):
    every shard is padded to the largest, gathered, and trimmed.
    """
    world = dist.get_world_size(group)
    if counts is None:
        counts = shard_counts(t.shape[1], t.device, group)
    if len(counts) != world or counts[dist.get_rank(group)] != t.shape[1]:
        raise ValueError("counts do not match the group or this rank's shard")
    nmax = max(counts)
    pad = t
    if t.shape[1] < nmax:
        shape = list(t.shape)
        shape[1] = nmax - t.shape[1]
        pad = torch.cat([t, t.new_zeros(shape)], dim=1)
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad.contiguous(), group=group)
    return torch.cat([p[:, :c] for p, c in zip(parts, counts)], dim=1).contiguous()


def sharded_sum_fwd(x, y, w, tau, group=None, kernels=None, src_counts=None):
    """Rows x of this rank against the sources of every rank: [B, M_r, C] float32."""
    k = kernels or _default_kernels()
    if src_counts is None:
        src_counts = shard_counts(y.shape[1], y.device, group)
    return k["sum"](x, all_gather_rows(y, group, src_counts), all_gather_rows(w, group, src_counts),
                    tau)


def sharded_lse_fwd(x, y, w, tau, group=None, kernels=None, src_counts=None):
    """Log-sum-exp of this rank's rows against the sources of every rank."""
    k = kernels or _default_kernels()
    if src_counts is None:
        src_counts = shard_counts(y.shape[1], y.device, group)
    return k["lse"](x, all_gather_rows(y, group, src_counts), all_gather_rows(w, group, src_counts),
                    tau)


def sharded_sum_bwd(x, y, w, g, tau, group=None, kernels=None, row_counts=None, src_counts=None):
    """(dL/dx for this rank's rows, dL/dw for this rank's sources) of L = <g, sum>.

    dL/dx_i sums over every source (all-gathered y, w); dL/dw_j sums over every
    row (all-gathered x, g).
    """
    k = kernels or _default_kernels()
    if src_counts is None:
        src_counts = shard_counts(y.shape[1], y.device, group)
    if row_counts is None:
        row_counts = shard_counts(x.shape[1], x.device, group)
    gx, _ = k["bwd"](x, all_gather_rows(y, group, src_counts), all_gather_rows(w, group, src_counts),
                     g, tau, want_x=True, want_w=False)
    _, gw = k["bwd"](all_gather_rows(x, group, row_counts), y, w,
                     all_gather_rows(g, group, row_counts), tau, want_x=False, want_w=True)
    return gx, gw


def sharded_sum_vjp(x, y, w, g, tau, group=None, kernels=None, row_counts=None, src_counts=None,
                    want=("x", "y", "w", "tau")):
    """Every first-order gradient of L = <g, sum> over the whole problem: a dict with
    the requested keys -- x for this rank's rows (and its share of tau) against the
    gathered (y, w); y and w for this rank's sources against the gathered (x, g);
    tau summed over the ranks."""
    k = kernels or _default_kernels()
    out = {}
    row_side = tuple(n for n in ("x", "tau") if n in want)
    src_side = tuple(n for n in ("y", "w") if n in want)
    if row_side:
        if src_counts is None:
            src_counts = shard_counts(y.shape[1], y.device, group)
        out.update(k["vjp"](x, all_gather_rows(y, group, src_counts),
                            all_gather_rows(w, group, src_counts), g, tau, want=row_side))
    if src_side:
        if row_counts is None:
            row_counts = shard_counts(x.shape[1], x.device, group)
        out.update(k["vjp"](all_gather_rows(x, group, row_counts), y, w,
                            all_gather_rows(g, group, row_counts), tau, want=src_side))
    if "tau" in out:
        t = out["tau"].clone()
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
        out["tau"] = t
    return out


def sharded_lse_bwd(x, y, w, lse, g, tau, group=None, kernels=None, row_counts=None,
                    src_counts=None, want=("x", "y", "w", "tau")):
    """Gradients of L = <g, lse> with lse = the log-sum-exp over every rank's sources:
    a dict with the requested keys -- x for this rank's rows, y and w for this rank's
    sources, tau (summed over the ranks).  lse and g are this rank's rows."""
    k = kernels or _default_kernels()
    out = {}
    row_side = tuple(n for n in ("x", "tau") if n in want)
    src_side = tuple(n for n in ("y", "w") if n in want)
    if row_side:
        if src_counts is None:
            src_counts = shard_counts(y.shape[1], y.device, group)
        r = k["lse_bwd"](x, all_gather_rows(y, group, src_counts), all_gather_rows(w, group, src_counts),
                         lse, g, tau, want=row_side)
        out.update(r)
    if src_side:
        if row_counts is None:
            row_counts = shard_counts(x.shape[1], x.device, group)
        r = k["lse_bwd"](all_gather_rows(x, group, row_counts), y, w,
                         all_gather_rows(lse, group, row_counts), all_gather_rows(g, group, row_counts),
                         tau, want=src_side)
        out.update(r)
    if "tau" in out:
        t = out["tau"].clone()
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
        out["tau"] = t
    return out


def sharded_diffusion_scales(x, tau, alpha, group=None, kernels=None, counts=None):
    """(q, d, s) of the alpha-normalised diffusion operator for this rank's points
    x [B, N_r, D] of a point set sharded by rows: each [B, N_r] float32 (float64
    when the compute is), over the kernel of every rank's points."""
    k = kernels or _default_kernels()
    if counts is None:
        counts = shard_counts(x.shape[1], x.device, group)
    xa = all_gather_rows(x, group, counts)
    B = x.shape[0]
    dt = torch.float64 if x.dtype == torch.float64 else torch.float32
    ones = torch.ones((B, xa.shape[1], 1), dtype=dt, device=x.device)
    q = k["block"](x, xa, ones, tau)[..., 0]
    qa = q.pow(-alpha)
    u = k["block"](x, xa, all_gather_rows(qa[..., None].contiguous(), group, counts), tau)[..., 0]
    d = qa * u
    s = qa * d.rsqrt()
    return q, d, s


def sharded_diffusion_apply(x, s, v, tau, group=None, kernels=None, counts=None):
    """This rank's rows of diag(s) K diag(s) V over the whole point set: x [B, N_r, D],
    s [B, N_r] and v [B, N_r, C] are this rank's points, scales and rows of V."""
    k = kernels or _default_kernels()
    if counts is None:
        counts = shard_counts(x.shape[1], x.device, group)
    xa = all_gather_rows(x, group, counts)
    sv = all_gather_rows((s[..., None] * v).contiguous(), group, counts)
    return s[..., None] * k["block"](x, xa, sv, tau)


__all__ = ["shard_counts", "all_gather_rows", "sharded_sum_fwd", "sharded_lse_fwd",
           "sharded_sum_bwd", "sharded_sum_vjp", "sharded_lse_bwd", "sharded_diffusion_scales",
           "sharded_diffusion_apply"]
