"""The multi-rank path on CPU: world size 2 over gloo (127.0.0.1).  Each rank runs the fp64
oracle on its token shard; the shards reassemble to the single-process result (tokens are
independent), and the timing reduction takes the max over ranks.  For the backward, each
rank's parameter gradients over its shard, summed across ranks by allreduce_param_grads,
equal the gradients over all tokens."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from mhc_hyper_connections_b200 import dist as mdist


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import torch.distributed as dist

    import oracle
    from mhc_hyper_connections_b200 import workloads as wl
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = wl.make_inputs(T=37, n=4, d=16, dtype="bf16", seed=3)
        a, b = mdist.token_shard(w.T, rank, world)
        sub = w.tokens(np.arange(a, b))
        s = w.scalars()
        x_in, H = oracle.mhc_pre(sub.values(sub.X), sub.phi, sub.b_pre, sub.b_post, sub.b_res,
                                 s["alpha_pre"], s["alpha_post"], s["alpha_res"], eps=s["eps"],
                                 t_max=s["t_max"])
        y = oracle.mhc_post(sub.values(sub.X), sub.values(sub.F_out), H)
        np.savez(os.path.join(out_dir, f"r{rank}.npz"), x_in=x_in, H=H, y=y, a=a, b=b)
        m = mdist.max_over_ranks(10.0 + 5.0 * rank)
        np.save(os.path.join(out_dir, f"m{rank}.npy"), np.array([m]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_token_shard_partition():
    for T in (0, 1, 5, 16384, 16385):
        for world in (1, 2, 3, 8):
            spans = [mdist.token_shard(T, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == T
            assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        mdist.token_shard(10, 2, 2)


def test_job_throughput():
    assert mdist.job_throughput(16384, 10, 5.0, 4) == pytest.approx(4 * 16384 * 10 / 0.005)
    assert mdist.max_over_ranks(3.5) == 3.5          # no process group: identity


def test_two_gloo_ranks_reassemble_and_reduce(tmp_path):
    import oracle
    from mhc_hyper_connections_b200 import workloads as wl
    oracle.build()
    world, port = 2, _free_port()
    mp.start_processes(_worker, args=(world, port, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    parts = [np.load(tmp_path / f"r{r}.npz") for r in range(world)]
    w = wl.make_inputs(T=37, n=4, d=16, dtype="bf16", seed=3)
    s = w.scalars()
    x_in, H = oracle.mhc_pre(w.values(w.X), w.phi, w.b_pre, w.b_post, w.b_res, s["alpha_pre"],
                             s["alpha_post"], s["alpha_res"], eps=s["eps"], t_max=s["t_max"])
    y = oracle.mhc_post(w.values(w.X), w.values(w.F_out), H)
    np.testing.assert_array_equal(np.concatenate([p["x_in"] for p in parts]), x_in)
    np.testing.assert_array_equal(np.concatenate([p["H"] for p in parts]), H)
    np.testing.assert_array_equal(np.concatenate([p["y"] for p in parts]), y)
    for r in range(world):
        assert float(np.load(tmp_path / f"m{r}.npy")[0]) == 15.0


def _bwd_worker(rank, world, port, out_dir):
    import torch
    import torch.distributed as dist

    import oracle
    from mhc_hyper_connections_b200 import workloads as wl
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, dY, dx = _bwd_problem()
        a, b = mdist.token_shard(w.T, rank, world)
        sub = w.tokens(np.arange(a, b))
        s = w.scalars()
        g = oracle.mhc_backward(sub.values(sub.X), sub.values(sub.F_out), sub.phi, sub.b_pre,
                                sub.b_post, sub.b_res, s["alpha_pre"], s["alpha_post"],
                                s["alpha_res"], dY[a:b], dx[a:b], eps=s["eps"], t_max=s["t_max"])
        tg = {k: torch.from_numpy(g[k]) for k in mdist.PARAM_GRADS}
        mdist.allreduce_param_grads(tg)
        np.savez(os.path.join(out_dir, f"g{rank}.npz"), dX=g["dX"], dF_out=g["dF_out"],
                 **{k: v.numpy() for k, v in tg.items()})
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _bwd_problem():
    from mhc_hyper_connections_b200 import workloads as wl
    w = wl.make_inputs(T=37, n=3, d=16, dtype="bf16", seed=8, alpha=0.4)
    rng = np.random.default_rng(9)
    return w, rng.normal(size=(w.T, w.n, w.d)), rng.normal(size=(w.T, w.d))


def test_two_gloo_ranks_sum_the_parameter_gradients(tmp_path):
    import oracle
    oracle.build()
    world, port = 2, _free_port()
    mp.start_processes(_bwd_worker, args=(world, port, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    parts = [np.load(tmp_path / f"g{r}.npz") for r in range(world)]
    w, dY, dx = _bwd_problem()
    s = w.scalars()
    ref = oracle.mhc_backward(w.values(w.X), w.values(w.F_out), w.phi, w.b_pre, w.b_post, w.b_res,
                              s["alpha_pre"], s["alpha_post"], s["alpha_res"], dY, dx,
                              eps=s["eps"], t_max=s["t_max"])
    np.testing.assert_array_equal(np.concatenate([p["dX"] for p in parts]), ref["dX"])
    np.testing.assert_array_equal(np.concatenate([p["dF_out"] for p in parts]), ref["dF_out"])
    for k in mdist.PARAM_GRADS:
        for p in parts:                     # every rank holds the whole job's gradient
            np.testing.assert_allclose(p[k].reshape(ref[k].shape), ref[k], rtol=1e-12, atol=1e-14)
    assert mdist.allreduce_param_grads({}) is None    # no process group here: a no-op
