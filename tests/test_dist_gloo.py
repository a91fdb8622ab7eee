"""Multi-rank host logic on CPU with the gloo backend (world size 2).

The decode step shards by sequence with no data-path collective: each rank
decodes its own sequences; results gathered from the ranks must equal the
single-process result, and the step time is the max over ranks."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from head_partitioned_sparse_b200 import shard


def test_shard_sequences_partitions_the_batch():
    for n in (1, 2, 3, 7, 16):
        for world in (1, 2, 3, 4, 8):
            parts = [shard.shard_sequences(n, world, r) for r in range(world)]
            assert np.array_equal(np.concatenate(parts), np.arange(n))
            sizes = [len(p) for p in parts]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard.shard_sequences(4, 2, 2)
    assert len({shard.rank_seed(0, r) for r in range(8)}) == 8


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist

    import oracle as O
    from head_partitioned_sparse_b200 import synth

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    try:
        import datetime
        dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
        assert shard.dist_env()[0] == rank and shard.dist_env()[2] == world
        inp = synth.make_inputs("tiny", 3, overrides={"B": 3, "L": 700, "window": 32}, seq_lens=[700, 450, 90])
        mine = shard.shard_sequences(inp.B, world, rank)
        idx = O.index_cache_for(inp, heads=[0])
        out, _ = O.decode_inputs(inp, idx_cache=idx, slices=[(int(b), g) for b in mine for g in range(inp.Hkv)])
        blocks = shard.gather_rows(out[mine].astype(np.float64), inp.B)
        t = shard.reduce_max(float(rank + 1))
        if rank == 0:
            full, _ = O.decode_inputs(inp, idx_cache=idx)
            got = np.concatenate(blocks)
            q.put(("ok", float(np.abs(got - full).max()), t))
        dist.barrier()
        dist.destroy_process_group()
    except Exception as e:  # report to the parent instead of hanging it
        q.put(("err", repr(e), None))
        raise


def test_two_rank_decode_gathers_to_the_single_process_result():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()
    assert not alive, "a rank did not finish"
    status, err, t = q.get(timeout=5)
    assert status == "ok", err
    assert err == 0.0
    assert t == 2.0
    assert all(p.exitcode == 0 for p in procs)
