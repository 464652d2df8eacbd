"""The N > 1 path on CPU: sharding plan, per-problem seeds and the timing
reduction, run as two gloo ranks.

On the GPU each rank runs the forward kernel on its own problem; here each
rank runs the oracle on its shard instead (the oracle is the per-problem
computation the kernel is checked against), so what is tested is everything
the multi-GPU run adds: which problems a rank owns, which inputs it draws,
that the union over ranks is the whole batch with each problem once, and the
max-over-ranks time the whole-job throughput divides by.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from block_sparse_long_bsa_b200 import inputs, sharding
from oracle import attention as A
from oracle import layouts as L

N, B, D, HEADS, KV = 192, 64, 32, 2, 1
GLOBAL_BATCH = 5


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem(element):
    qs, ks, vs = inputs.qkv_bits(HEADS, KV, N, D, sharding.element_seeds(element))
    q, k, v = (inputs.bf16_bits_to_f64(x) for x in (qs, ks, vs))
    sets = L.kept_sets(L.DYADIC, N, B, 1, window=1, global_first=1, dyadic_kmin=2)
    return A.forward_sparse(q, k, v, sets, B, 1.0 / np.sqrt(D))


def _rank_main(rank, world, port, out_dir):
    import torch
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        mine = sharding.shard(GLOBAL_BATCH, world, rank)
        results = {e: _problem(e) for e in mine.elements}
        # Each rank reports a different time; all must see the slowest.
        t_max = sharding.max_over_ranks(10.0 + rank, world)
        gathered = [None] * world
        dist.all_gather_object(gathered, {"elements": list(mine.elements), "t_max": t_max,
                                          "results": results})
        if rank == 0:
            np.save(os.path.join(out_dir, "gathered.npy"), np.array(gathered, dtype=object),
                    allow_pickle=True)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_shard_is_a_partition():
    for world in range(1, 9):
        for batch in range(0, 20):
            parts = [sharding.shard(batch, world, r) for r in range(world)]
            flat = [e for p in parts for e in p.elements]
            assert flat == list(range(batch))
            sizes = [len(p) for p in parts]
            assert max(sizes) - min(sizes) <= 1
            assert sizes == sorted(sizes, reverse=True)


def test_shard_rejects_bad_arguments():
    with pytest.raises(ValueError):
        sharding.shard(4, 0, 0)
    with pytest.raises(ValueError):
        sharding.shard(4, 2, 2)
    with pytest.raises(ValueError):
        sharding.shard(-1, 2, 0)
    with pytest.raises(ValueError):
        sharding.element_seeds(-1)


def test_seeds_distinct_and_rank0_matches_single_run():
    assert sharding.element_seeds(0) == (inputs.Q_SEED, inputs.K_SEED, inputs.V_SEED)
    seen = set()
    for e in range(64):
        for s in sharding.element_seeds(e):
            assert s not in seen
            seen.add(s)


def test_aggregate_rate():
    assert sharding.aggregate_rate(3.0, 4, 2.0) == 6.0
    assert sharding.aggregate_rate([1.0, 2.0, 3.0], 3, 3.0) == 2.0
    assert sharding.max_over_ranks(7.5, 1) == 7.5
    with pytest.raises(ValueError):
        sharding.aggregate_rate([1.0], 2, 1.0)
    with pytest.raises(ValueError):
        sharding.aggregate_rate(1.0, 1, 0.0)


def test_two_gloo_ranks_cover_the_batch(tmp_path):
    world = 2
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]

    gathered = np.load(tmp_path / "gathered.npy", allow_pickle=True)
    assert [g["t_max"] for g in gathered] == [11.0, 11.0]
    owned = [e for g in gathered for e in g["elements"]]
    assert owned == list(range(GLOBAL_BATCH))
    merged = {}
    for g in gathered:
        merged.update(g["results"])
    # The sharded run reproduces a single-process run of the whole batch, and
    # the problems really are different draws.
    for e in range(GLOBAL_BATCH):
        o_ref, lse_ref = _problem(e)
        o, lse = merged[e]
        assert np.array_equal(o, o_ref) and np.array_equal(lse, lse_ref)
    assert not np.array_equal(merged[0][0], merged[1][0])
