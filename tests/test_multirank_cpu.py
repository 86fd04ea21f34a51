"""The N > 1 plumbing of bench.py on CPU with the gloo backend (world size 2).

The path shards tokens across ranks with no data-path collective; the only
cross-rank steps are the barrier and the reduction of timings (max over
ranks) and units (sum over ranks).  These run here unchanged on gloo.
"""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    # rank r pretends its kernels took (10 + r) ms and (2 + 3r) ms
    times, units = bench.reduce_job([10.0 + rank, 2.0 + 3 * rank], 4608 * (rank + 1))
    dist.barrier()
    out[rank] = (times, units, bench.rank_seed(rank))
    dist.destroy_process_group()


def test_reduce_job_max_time_sum_units_two_ranks():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        times, units, seed = res[rank]
        assert times == [11.0, 5.0]          # max over ranks, element-wise
        assert units == 4608 * 3             # sum over ranks
    assert res[0][2] != res[1][2]            # each rank quantises its own shard


def test_reduce_job_single_process_is_identity():
    import bench
    times, units = bench.reduce_job([1.5, 2.5], 7)
    assert times == [1.5, 2.5] and units == 7


def _shard_worker(rank, world, port, out):
    import numpy as np
    import torch
    import torch.distributed as dist
    from oracle.lloydmax import lloydmax_table
    from oracle.quant import quantize_act
    from oracle.rng import rpbh_draw
    from oracle.rpbh import rpbh_matrix
    import synth
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    d, T = 256, 40
    # the rotation and codebook are drawn from the shared seed on every rank
    Pi = rpbh_matrix(*rpbh_draw(d, 11))
    _, bounds = lloydmax_table(d, 3)
    X = synth.rng(5, 0).standard_normal((T, d))
    lo, hi = rank * T // world, (rank + 1) * T // world
    q = quantize_act(X[lo:hi], Pi, bounds)
    codes = torch.from_numpy(np.ascontiguousarray(q["codes"]))
    parts = [torch.empty_like(codes) for _ in range(world)]
    dist.all_gather(parts, codes)
    out[rank] = torch.cat(parts).numpy().tolist()
    dist.destroy_process_group()


def test_token_shards_concatenate_to_the_unsharded_result():
    """Rows are independent: quantising each rank's contiguous token shard
    with the shared rotation and concatenating gives the codes of the whole
    batch, so sharding tokens needs no data-path collective."""
    import numpy as np
    from oracle.lloydmax import lloydmax_table
    from oracle.quant import quantize_act
    from oracle.rng import rpbh_draw
    from oracle.rpbh import rpbh_matrix
    import synth
    world, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_shard_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    d, T = 256, 40
    Pi = rpbh_matrix(*rpbh_draw(d, 11))
    _, bounds = lloydmax_table(d, 3)
    whole = quantize_act(synth.rng(5, 0).standard_normal((T, d)), Pi, bounds)["codes"]
    for rank in range(world):
        assert np.array_equal(np.asarray(res[rank]), whole)
