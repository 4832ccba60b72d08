"""The data-parallel (N > 1) path on CPU with gloo, world size 2: every rank computes the dq of
its own token shard; summing over ranks (the bench's reduction) must give the dq of the whole
batch, and the step time taken is the slowest rank's."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O

WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer(seed=3, m=32, n=48, b=8, T=20):
    rng = np.random.default_rng(seed)
    d = dict(X=rng.standard_normal((T, m)), dY=rng.standard_normal((T, n)),
             W0=rng.standard_normal((m, n)),
             q_r=rng.standard_normal((m // b, b * (b - 1) // 2)) * 0.1,
             q_p=rng.standard_normal((n // b, b * (b - 1) // 2)) * 0.1,
             perm_r=rng.permutation(m), perm_p=rng.permutation(n), b=b)
    d["W0m"] = O.merge_permutations(d["W0"], d["perm_r"], d["perm_p"])
    return d


def _dq(d, rows):
    G_r, G_p = O.cnp(d["q_r"], d["b"]), O.cnp(d["q_p"], d["b"])
    g = O.linear_bwd(d["X"][rows], d["dY"][rows], d["W0m"], d["perm_r"], d["perm_p"], G_r, G_p,
                     d["q_r"], d["q_p"], d["b"])
    return np.concatenate([g["dq_r"].ravel(), g["dq_p"].ravel()])


def _worker(rank, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    try:
        import bench
        d = _layer()
        shard = np.array_split(np.arange(d["X"].shape[0]), WORLD)[rank]
        flat = torch.from_numpy(_dq(d, shard))
        bench.sum_over_ranks_(flat)
        slowest = bench.max_over_ranks(10.0 + rank)
        if rank == 0:
            out.put((flat.numpy(), slowest))
    finally:
        dist.destroy_process_group()


def test_data_parallel_dq_reduction_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    summed, slowest = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    d = _layer()
    full = _dq(d, np.arange(d["X"].shape[0]))
    np.testing.assert_allclose(summed, full, rtol=1e-11, atol=1e-12)
    assert slowest == 11.0


SHAPES = [(32, 48, 8), (16, 32, 8), (48, 16, 16)]   # three linears (m, n, b)


def _worker_async(rank, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    try:
        import bench
        red = bench.DqReducer()
        flats = []
        for li, (m, n, b) in enumerate(SHAPES):
            d = _layer(seed=10 + li, m=m, n=n, b=b)
            shard = np.array_split(np.arange(d["X"].shape[0]), WORLD)[rank]
            flat = torch.from_numpy(_dq(d, shard))
            flats.append(flat)
            red.add(flat)            # issued while the next linear is still to be computed
        red.finish()
        if rank == 0:
            out.put([f.numpy() for f in flats])
    finally:
        dist.destroy_process_group()


def test_per_linear_async_dq_reduction_two_ranks():
    """The bench's per-linear reduction: each linear's dq all-reduce is issued right after that
    linear's backward, asynchronously, with the next linear's work in between; after finish()
    every linear holds the dq of the whole batch, so the collectives were matched linear by
    linear across the ranks."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_async, args=(r, port, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    got = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for li, (m, n, b) in enumerate(SHAPES):
        d = _layer(seed=10 + li, m=m, n=n, b=b)
        full = _dq(d, np.arange(d["X"].shape[0]))
        np.testing.assert_allclose(got[li], full, rtol=1e-11, atol=1e-12)


def test_single_process_helpers_are_identity():
    import bench
    flat = torch.arange(4.0)
    assert torch.equal(bench.sum_over_ranks_(flat.clone()), flat)
    assert bench.max_over_ranks(3.5) == 3.5
    red = bench.DqReducer()
    red.add(flat)
    red.finish()
    assert not red.works
