"""One problem sharded over ranks (pairwise_reductions_b200.sharded).

CPU part: two gloo ranks, each holding a different-sized shard of the rows and
of the sources; the pair work is done by the oracle (injected as the compute
calls), so what is tested is the exchange -- counts, padding, rank order, and
which tensors each gradient gathers -- against the oracle on the whole problem.
GPU part: a one-rank NCCL group runs the same functions on the CUDA library.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TAU = 0.7
# rows and sources of each rank (different sizes, so padding is exercised)
ROWS = (37, 21)
SRCS = (15, 40)


ALPHA = 0.5


def _diffusion_v():
    g = torch.Generator().manual_seed(78)
    return torch.randn(2, sum(SRCS), 3, generator=g, dtype=torch.float64)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _full_problem():
    g = torch.Generator().manual_seed(77)
    B, D, C = 2, 3, 2
    M, N = sum(ROWS), sum(SRCS)
    x = torch.randn(B, M, D, generator=g, dtype=torch.float64)
    y = torch.randn(B, N, D, generator=g, dtype=torch.float64)
    w = torch.rand(B, N, C, generator=g, dtype=torch.float64) + 0.5
    gr = torch.randn(B, M, C, generator=g, dtype=torch.float64)
    return x, y, w, gr


def _oracle_kernels():
    import oracle
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    n = lambda a: a.numpy()

    def bwd(x, y, w, g, tau, want_x=True, want_w=True):
        gx, gw = oracle.gauss_sum_bwd(n(x), n(y), n(w), n(g), tau)
        return (t(gx) if want_x else None), (t(gw) if want_w else None)

    def vjp(x, y, w, g, tau, want=("x", "y", "w", "tau")):
        gx, gw = oracle.gauss_sum_bwd(n(x), n(y), n(w), n(g), tau)
        gy, gt = oracle.gauss_sum_vjp_y_tau(n(x), n(y), n(w), n(g), tau)
        full = {"x": t(gx), "y": t(gy), "w": t(gw), "tau": torch.tensor([gt], dtype=torch.float64)}
        return {kk: full[kk] for kk in want}
    return {"sum": lambda x, y, w, tau: t(oracle.gauss_sum(n(x), n(y), n(w), tau)),
            "lse": lambda x, y, w, tau: t(oracle.gauss_lse(n(x), n(y), n(w), tau)),
            "bwd": bwd, "lse_bwd": _lse_bwd_given_lse, "vjp": vjp,
            "block": lambda xr, xc, v, tau: t(oracle.gauss_sum(n(xr), n(xc), n(v), tau))}


def _lse_bwd_given_lse(x, y, w, lse, g, tau, want=("x", "y", "w", "tau")):
    """Gradients of <g, lse> for the given sources, normalised by the given lse
    (dense float64 from the definition: p_ijc = w_jc K_ij exp(-lse_ic))."""
    d2 = ((x[:, :, None, :] - y[:, None, :, :]) ** 2).sum(-1)            # [B, M, N]
    K = torch.exp(-0.5 * tau * d2)
    p = w[:, None, :, :] * K[..., None] * torch.exp(-lse)[:, :, None, :]  # [B, M, N, C]
    gp = (g[:, :, None, :] * p).sum(-1)                                  # sum_c g_ic p_ijc
    out = {}
    if "x" in want:
        out["x"] = -tau * (x * gp.sum(2)[..., None] - gp @ y)
    if "y" in want:
        out["y"] = tau * (gp.transpose(1, 2) @ x - y * gp.sum(1)[..., None])
    if "w" in want:
        out["w"] = ((g * torch.exp(-lse))[:, :, None, :] * K[..., None]).sum(1)
    if "tau" in want:
        out["tau"] = (-0.5 * gp * d2).sum().reshape(1)
    return out


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from pairwise_reductions_b200 import sharded
    dist.init_process_group("gloo", rank=rank, world_size=world)
    x, y, w, g = _full_problem()
    r0, s0 = sum(ROWS[:rank]), sum(SRCS[:rank])
    xs, gs_ = x[:, r0:r0 + ROWS[rank]].contiguous(), g[:, r0:r0 + ROWS[rank]].contiguous()
    ys, ws = y[:, s0:s0 + SRCS[rank]].contiguous(), w[:, s0:s0 + SRCS[rank]].contiguous()
    k = _oracle_kernels()
    out = {
        "gather_y": sharded.all_gather_rows(ys),
        "sum": sharded.sharded_sum_fwd(xs, ys, ws, TAU, kernels=k),
        "lse": sharded.sharded_lse_fwd(xs, ys, ws, TAU, kernels=k),
    }
    out["gx"], out["gw"] = sharded.sharded_sum_bwd(xs, ys, ws, gs_, TAU, kernels=k)
    lg = sharded.sharded_lse_bwd(xs, ys, ws, out["lse"], gs_, TAU, kernels=k)
    vg = sharded.sharded_sum_vjp(xs, ys, ws, gs_, TAU, kernels=k)
    out.update({"vjp_g" + kk: v for kk, v in vg.items()})
    out.update({"lse_g" + kk: v for kk, v in lg.items()})
    # the diffusion operator over the point set y, sharded by its rows (the sources)
    dv = _diffusion_v()
    vs = dv[:, s0:s0 + SRCS[rank]].contiguous()
    out["dq"], out["dd"], out["ds"] = sharded.sharded_diffusion_scales(ys, TAU, ALPHA, kernels=k)
    out["dapply"] = sharded.sharded_diffusion_apply(ys, out["ds"], vs, TAU, kernels=k)
    q.put((rank, {kk: v.numpy() for kk, v in out.items()}))
    dist.destroy_process_group()


def test_sharded_problem_matches_the_whole_problem_gloo():
    sys.path.insert(0, ROOT)
    import oracle
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    x, y, w, g = (t.numpy() for t in _full_problem())
    s = oracle.gauss_sum(x, y, w, TAU)
    lse = oracle.gauss_lse(x, y, w, TAU)
    gx, gw = oracle.gauss_sum_bwd(x, y, w, g, TAU)
    lgx, lgy, lgw, lgt = oracle.gauss_lse_bwd(x, y, w, g, TAU)
    vgy, vgt = oracle.gauss_sum_vjp_y_tau(x, y, w, g, TAU)
    dq, dd, ds = oracle.diffusion_scales(y, TAU, ALPHA)
    dap = oracle.diffusion_apply(y, ds, _diffusion_v().numpy(), TAU)
    for rank in range(world):
        r0, s0 = sum(ROWS[:rank]), sum(SRCS[:rank])
        rows, srcs = slice(r0, r0 + ROWS[rank]), slice(s0, s0 + SRCS[rank])
        o = got[rank]
        np.testing.assert_array_equal(o["gather_y"], y)            # rank order, trimmed padding
        np.testing.assert_allclose(o["sum"], s[:, rows], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(o["lse"], lse[:, rows], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(o["gx"], gx[:, rows], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(o["gw"], gw[:, srcs], rtol=1e-12, atol=1e-12)
        # log-sum-exp backward: x of the local rows, y and w of the local sources,
        # tau summed over the ranks
        np.testing.assert_allclose(o["lse_gx"], lgx[:, rows], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(o["lse_gy"], lgy[:, srcs], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(o["lse_gw"], lgw[:, srcs], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(o["lse_gtau"], [lgt], rtol=1e-10)
        # every gradient of the sum: tau summed over the ranks
        np.testing.assert_allclose(o["vjp_gx"], gx[:, rows], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(o["vjp_gy"], vgy[:, srcs], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(o["vjp_gw"], gw[:, srcs], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(o["vjp_gtau"], [vgt], rtol=1e-12)
        # diffusion operator: this rank's rows of q, d, s and of diag(s) K diag(s) V
        np.testing.assert_allclose(o["dq"], dq[:, srcs], rtol=1e-12)
        np.testing.assert_allclose(o["dd"], dd[:, srcs], rtol=1e-12)
        np.testing.assert_allclose(o["ds"], ds[:, srcs], rtol=1e-12)
        np.testing.assert_allclose(o["dapply"], dap[:, srcs], rtol=1e-11, atol=1e-14)


def _gpu_worker(port, q):
    os.environ.update(RANK="0", WORLD_SIZE="1", MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import pairwise_reductions_b200 as m
    from pairwise_reductions_b200 import sharded
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    x, y, w, g = (t.float().cuda() for t in _full_problem())
    a = sharded.sharded_sum_fwd(x, y, w, TAU)
    b = m.gauss_sum_fwd(x, y, w, TAU)
    gx, gw = sharded.sharded_sum_bwd(x, y, w, g, TAU)
    rx, rw = m.gauss_sum_bwd(x, y, w, g, TAU)
    lse = m.gauss_lse_fwd(x, y, w, TAU)
    lg = sharded.sharded_lse_bwd(x, y, w, lse, g, TAU)
    rl = m.gauss_lse_bwd(x, y, w, lse, g, TAU)
    # diffusion operator of the point set y: one rank against the single-GPU entry points
    dq, dd, ds = sharded.sharded_diffusion_scales(y, TAU, 0.5)
    rq, rd, rs = m.gauss_diffusion_scales(y, TAU, 0.5)
    v = torch.rand(y.shape[0], y.shape[1], 2, device="cuda")
    da = sharded.sharded_diffusion_apply(y, ds, v, TAU)
    ra = m.gauss_diffusion_apply(y, rs, v, TAU)
    torch.cuda.synchronize()
    lse_ok = all(torch.allclose(lg[k], rl[k], rtol=1e-6, atol=1e-7) for k in ("x", "y", "w", "tau"))
    diff_ok = (torch.equal(dq, rq) and all(torch.allclose(p_, r_, rtol=1e-6)
                                           for p_, r_ in ((dd, rd), (ds, rs), (da, ra))))
    q.put(bool(torch.equal(a, b) and torch.equal(gx, rx) and torch.equal(gw, rw) and lse_ok
               and diff_ok))
    dist.destroy_process_group()


@pytest.mark.gpu
def test_sharded_single_rank_nccl_runs_the_cuda_library():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_gpu_worker, args=(_free_port(), q))
    p.start()
    ok = q.get(timeout=300)
    p.join(60)
    assert p.exitcode == 0 and ok


def test_bench_shards_cover_the_problem_once():
    """bench.py --sharded: the ranks' contiguous slices tile the rows and the sources."""
    sys.path.insert(0, ROOT)
    import bench
    x, y, w, g = _full_problem()
    inp = {"x": x, "y": y, "w": w, "g": g, "tau": TAU}
    for world in (1, 2, 3, 5):
        parts = [bench.shard_of(inp, r, world) for r in range(world)]
        for k, dim_src in (("x", x), ("y", y), ("w", w), ("g", g)):
            assert torch.equal(torch.cat([p[k] for p in parts], dim=1), dim_src)
