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


def _oracle_shard_worker(rank: int, world: int, port: int, q):
    """Rank r runs the float64 oracle on its shard of a batch (sequences
    r::world, their global indices fixing their dropout bits), exchanges the
    gradients with allreduce_mean and reports them."""
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    sys.path.insert(0, os.path.join(root, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import numpy as np
        import oracle
        from parity import oracle_config
        from transformer_layer_pre_b200.dp import FlatGrads, allreduce_mean
        from transformer_layer_pre_b200.synthetic import make_inputs, to_f64
        inp = make_inputs(SHARDED)
        idx = np.arange(rank, SHARDED.batch, world)
        cfg = oracle_config(SHARDED, len(idx))
        wt = {n: to_f64(inp.weights[0][n]) for n in oracle.WEIGHT_NAMES}
        r = oracle.layer_forward_backward(cfg, to_f64(inp.x)[idx], to_f64(inp.mask)[idx], wt, to_f64(inp.dy)[idx],
                                          seq_index=idx)
        g = FlatGrads(SHARDED.hidden, SHARDED.ffn, "cpu")
        g.flat = g.flat.double()   # the exchange itself in float64 for this check
        g.views = {n: g.flat[v.storage_offset():v.storage_offset() + v.numel()].view(v.shape)
                   for n, v in g.views.items()}
        for n in oracle.WEIGHT_NAMES:
            g[n].copy_(torch.from_numpy(r["grads"][n]))
        allreduce_mean(g)
        q.put((rank, {n: g[n].numpy().copy() for n in oracle.WEIGHT_NAMES}, idx, r["dx"]))
    finally:
        dist.destroy_process_group()


def _sharded_workload():
    from transformer_layer_pre_b200.synthetic import Workload
    return Workload("dp-shard-f32", 4, 16, 64, 4, 256, "f32", 0.1, 0.1, lengths=(9, 16))


SHARDED = _sharded_workload()


def test_data_parallel_mean_equals_full_batch_gradient_two_ranks():
    """Two gloo ranks, each the oracle on half the sequences; after the
    exchange (the mean over ranks of per-rank gradients, each a sum over
    its rank's tokens) world x the mean equals the full-batch oracle's
    gradient (a sum over all tokens), and each rank's dx equals the full
    batch's dx of its sequences.  Convention: a layer's parameter gradient
    is a sum over the tokens it saw; the data-parallel exchange averages
    over ranks, i.e. it yields the gradient of the mean of the per-rank
    losses."""
    import numpy as np
    import oracle
    from parity import oracle_config
    from transformer_layer_pre_b200.synthetic import make_inputs, to_f64
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_oracle_shard_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=300) for _ in procs], key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    inp = make_inputs(SHARDED)
    full = oracle.layer_forward_backward(oracle_config(SHARDED, SHARDED.batch), to_f64(inp.x), to_f64(inp.mask),
                                         {n: to_f64(inp.weights[0][n]) for n in oracle.WEIGHT_NAMES},
                                         to_f64(inp.dy))
    for rank, grads, idx, dx in res:
        for n in oracle.WEIGHT_NAMES:
            ref = full["grads"][n]
            assert np.abs(2.0 * grads[n] - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max()), (rank, n)
        ref = full["dx"][idx]
        assert np.abs(dx - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max()), rank
    assert np.array_equal(res[0][1]["w1"], res[1][1]["w1"])


def test_flat_grads_single_process_is_noop():
    from transformer_layer_pre_b200.dp import FlatGrads, allreduce_mean
    g = FlatGrads(32, 128, "cpu")
    g["w1"].fill_(3.0)
    allreduce_mean(g)
    assert torch.all(g["w1"] == 3.0)
    assert g["w1"].shape == (128, 32) and g["bqkv"].shape == (96,)
