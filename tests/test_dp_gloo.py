"""Host-side multi-process checks (world size 2, gloo on CPU): the
data-parallel gradient exchange and the bench's max-over-ranks timing."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from transformer_layer_pre_b200.dp import FlatGrads, allreduce_mean
        import bench
        g = FlatGrads(64, 256, "cpu")
        for i, n in enumerate(g.views):
            g[n].fill_(float(rank * 100 + i))
        allreduce_mean(g)
        ok_mean = all(torch.all(g[n] == float(50 + i)) for i, n in enumerate(g.views))
        # views stay aligned and disjoint
        ptrs = sorted((g[n].data_ptr(), g[n].numel()) for n in g.views)
        aligned = all(p % 16 == 0 for p, _ in ptrs)
        disjoint = all(p1 + 4 * n1 <= p2 for (p1, n1), (p2, _) in zip(ptrs, ptrs[1:]))
        # per-layer buckets submitted one by one (the stack's overlapped exchange)
        from transformer_layer_pre_b200.dp import GradExchanger
        layers = [FlatGrads(32, 64, "cpu") for _ in range(3)]
        ex = GradExchanger()
        for l in reversed(range(3)):
            layers[l].flat.fill_(float(rank * 10 + l))
            ex.submit(layers[l])
        ex.finish()
        ok_layers = all(torch.all(layers[l].flat == float(5 + l)) for l in range(3))
        mx = bench.reduce_max(1.0 + rank)
        bench.barrier()
        q.put((rank, bool(ok_mean) and bool(ok_layers), aligned, disjoint, mx))
    finally:
        dist.destroy_process_group()


def test_gradient_allreduce_and_max_timing_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ok_mean, aligned, disjoint, mx in res:
        assert ok_mean and aligned and disjoint
        assert mx == 2.0


def test_flat_grads_single_process_is_noop():
    from transformer_layer_pre_b200.dp import FlatGrads, allreduce_mean
    g = FlatGrads(32, 128, "cpu")
    g["w1"].fill_(3.0)
    allreduce_mean(g)
    assert torch.all(g["w1"] == 3.0)
    assert g["w1"].shape == (128, 32) and g["bqkv"].shape == (96,)
