"""One Gauss-sum problem sharded over the ranks of a process group.

The rows of a Gauss sum are independent once every source is known, so a
problem splits by rows with a single exchange of the sources: rank r holds the
query rows x_r and a shard (y_r, w_r) of the sources; one all-gather gives every
rank the whole (y, w), and rank r computes its rows.  "FlashDiffusion" (§3,
multi-GPU runs) shards its kernel application over the row axis the same way.
The gradient adds one more exchange: dL/dx of the local rows needs (y, w) as
above, while dL/dw and dL/dy of the local sources need every row and its
upstream gradient, i.e. an all-gather of (x, g).

The exchanges are `torch.distributed` collectives on the group's backend (NCCL
over NVLink for CUDA tensors); the pair work runs in this library's kernels
(`gauss_sum_fwd`, `gauss_lse_fwd`, `gauss_sum_bwd`).  Shards may differ in
size; they are concatenated in rank order.

`kernels` replaces the three compute calls (same signatures); the default is
the CUDA library.
"""
import torch
import torch.distributed as dist


def _default_kernels():
    from . import gauss_lse_fwd, gauss_sum_bwd, gauss_sum_fwd
    return {"sum": gauss_sum_fwd, "lse": gauss_lse_fwd, "bwd": gauss_sum_bwd}


def all_gather_rows(t, group=None):
    """Concatenate every rank's t [B, n_r, ...] along dim 1, in rank order.

    Shards may have different n_r: the counts are exchanged first, every shard
    is padded to the largest, gathered, and trimmed.
    """
    world = dist.get_world_size(group)
    n = torch.tensor([t.shape[1]], dtype=torch.int64, device=t.device)
    counts = [torch.zeros_like(n) for _ in range(world)]
    dist.all_gather(counts, n, group=group)
    counts = [int(c.item()) for c in counts]
    nmax = max(counts)
    pad = t
    if t.shape[1] < nmax:
        shape = list(t.shape)
        shape[1] = nmax - t.shape[1]
        pad = torch.cat([t, t.new_zeros(shape)], dim=1)
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad.contiguous(), group=group)
    return torch.cat([p[:, :c] for p, c in zip(parts, counts)], dim=1).contiguous()


def sharded_sum_fwd(x, y, w, tau, group=None, kernels=None):
    """Rows x of this rank against the sources of every rank: [B, M_r, C] float32."""
    k = kernels or _default_kernels()
    return k["sum"](x, all_gather_rows(y, group), all_gather_rows(w, group), tau)


def sharded_lse_fwd(x, y, w, tau, group=None, kernels=None):
    """Log-sum-exp of this rank's rows against the sources of every rank."""
    k = kernels or _default_kernels()
    return k["lse"](x, all_gather_rows(y, group), all_gather_rows(w, group), tau)


def sharded_sum_bwd(x, y, w, g, tau, group=None, kernels=None):
    """(dL/dx for this rank's rows, dL/dw for this rank's sources) of L = <g, sum>.

    dL/dx_i sums over every source (all-gathered y, w); dL/dw_j sums over every
    row (all-gathered x, g).
    """
    k = kernels or _default_kernels()
    gx, _ = k["bwd"](x, all_gather_rows(y, group), all_gather_rows(w, group), g, tau,
                     want_x=True, want_w=False)
    _, gw = k["bwd"](all_gather_rows(x, group), y, w, all_gather_rows(g, group), tau,
                     want_x=False, want_w=True)
    return gx, gw


__all__ = ["all_gather_rows", "sharded_sum_fwd", "sharded_lse_fwd", "sharded_sum_bwd"]
