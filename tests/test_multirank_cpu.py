"""The N>1 bench path on CPU: two gloo ranks agree on the max-over-ranks
timing and barrier the way bench.py does on NCCL (replicas: no data-path
collective)."""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    w, r, lr = bench.dist_setup()
    assert (w, r, lr) == (world, rank, rank)
    bench.barrier(world)
    got = bench.max_over_ranks(10.0 + rank, world)
    q.put((rank, got))
    dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(90)
    assert all(p.exitcode == 0 for p in procs)
    res = dict(q.get(timeout=5) for _ in range(2))
    assert res == {0: 11.0, 1: 11.0}


def test_single_rank_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.copies_for(21_233_664 + 2_621_440, 126 * 2**20) >= 16


# ---------------------------------------------------------------- row-sharded decode
# The host logic of bit_lifted_gemm_b200.sharded on 2 gloo ranks: row partition,
# padding to a common shard height, all-gather in rank order and reassembly. Each
# rank's shard output comes from the float64 oracle here (test infrastructure), so
# the check needs no GPU; the GPU test runs the same class on the library's kernels.

def test_row_partition_properties():
    from bit_lifted_gemm_b200.sharded import row_range, shard_height
    for out in (1, 7, 16, 13824, 28673):
        for world in (1, 2, 3, 8):
            if out < world:
                continue
            spans = [row_range(out, world, g) for g in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == out
            assert all(spans[g][1] == spans[g + 1][0] for g in range(world - 1))
            sizes = [r1 - r0 for r0, r1 in spans]
            assert max(sizes) - min(sizes) <= 1 and max(sizes) == shard_height(out, world)
    with pytest.raises(ValueError):
        row_range(2, 3, 0)


def _shard_worker(rank, world, port, q):
    import datetime

    import numpy as np
    import torch
    import torch.distributed as dist

    import oracle
    from bit_lifted_gemm_b200.sharded import assemble, row_range, shard_height
    from datagen import CONFIGS, make_layer
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    L = make_layer(CONFIGS["tiny"], 3)
    out = 509  # ragged: shards of 170, 170, 169 rows (world 3) or 255, 254 (world 2)
    packed, s = L.packed[:out], L.s[:out]
    u = oracle.lift(oracle.whiten(oracle.to_f64(L.a), None), oracle.to_f64(L.M), L.cfg.K)
    r0, r1 = row_range(out, world, rank)
    h = shard_height(out, world)
    local = np.zeros((3, h))
    local[:, : r1 - r0] = oracle.contract(packed[r0:r1], s[r0:r1], u)
    pieces = [torch.empty((3, h), dtype=torch.float64) for _ in range(world)]
    dist.all_gather(pieces, torch.from_numpy(local), group=None)
    o = assemble(pieces, out, world).numpy()
    q.put((rank, bool(np.array_equal(o, oracle.contract(packed, s, u)))))
    dist.destroy_process_group()


@pytest.mark.timeout(120)
@pytest.mark.parametrize("world", [2, 3])
def test_sharded_decode_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(90)
    assert all(p.exitcode == 0 for p in procs)
    res = dict(q.get(timeout=5) for _ in range(world))
    assert all(res[r] for r in range(world))
