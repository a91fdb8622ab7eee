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


# ------------------------------------------------------------------ context-parallel exchange
# The phases of a context-parallel step run in a host model (cp_host_model) that reads
# and writes the exchange buffers in libspa's layout; the orchestration and the
# all-gathers are the package's own.  Rank r holds positions [r C, (r + 1) C).
CP_CASE = dict(name="tiny", seed=5, overrides={"B": 3, "L": 9000, "window": 64, "p": 0.9}, seq_lens=[9000, 4700, 90])
CP_C = 4500


def _cp_inputs():
    import oracle as O
    from head_partitioned_sparse_b200 import synth
    inp = synth.make_inputs(CP_CASE["name"], CP_CASE["seed"], overrides=CP_CASE["overrides"],
                            seq_lens=CP_CASE["seq_lens"])
    idx = O.index_cache_for(inp, heads=[g for g in range(inp.Hkv) if inp.head_mask[g]])
    return inp, idx


def _cp_check(inp, idx, out, rows, p=None):
    """Union of the ranks' rows = the oracle's sets (band 1e-5 around p); output = the
    oracle on those rows."""
    import oracle as O
    p = inp.p if p is None else p
    _, res = O.decode_inputs(inp, idx_cache=idx, p=p)
    listed = {}
    for b in range(inp.B):
        sw = O.sink_window(int(inp.seq_lens[b]), inp.n_sink, inp.window)
        for g in range(inp.Hkv):
            got = rows[(b, g)]
            assert np.all(np.diff(got) > 0)
            if not inp.head_mask[g]:
                assert np.array_equal(got, sw)
                continue
            assert np.isin(sw, got).all()
            listed[(b, g)] = np.setdiff1d(got, sw)
            diff = np.setxor1d(listed[(b, g)], res[(b, g)].listed)
            assert np.all(np.abs(res[(b, g)].topp.c_before[diff] - p) <= 1e-5)
    ref, _ = O.decode_inputs(inp, idx_cache=idx, p=p, attend_sets=listed)
    return float(np.abs(out - ref).max())


@pytest.mark.parametrize("R,p", [(1, None), (2, None), (3, None), (5, None), (3, 0.5), (4, 0.99), (2, 1.0)])
def test_cp_phases_emulated_in_one_process_match_the_oracle(R, p):
    import torch
    import cp_host_model as M
    from head_partitioned_sparse_b200 import context_parallel as cp
    inp, idx = _cp_inputs()
    pp = inp.p if p is None else float(np.float32(p))
    C = -(-int(inp.seq_lens.max()) // R)
    bufs = {n: torch.zeros(sz, dtype=torch.uint8) for n, sz in
            zip(cp.BUFFERS, M.exchange_sizes(inp.B, inp.Hq, inp.Hkv, C, R, inp.head_mask))}
    ranks = [M.HostRank(inp, idx, r, R, C, bufs, p=pp, n_sink=inp.n_sink, window=inp.window) for r in range(R)]
    cp.run_step(range(R), lambda ph, r: ranks[r].phase(ph), lambda name: None)
    out = M.combine(ranks[0].out_all, ranks[0].lse_all)
    rows = {k: np.concatenate([rk.rows[k] for rk in ranks]) for k in ranks[0].rows}
    assert _cp_check(inp, idx, out, rows, p=pp) <= 1e-5


@pytest.mark.parametrize("retrieval", [[1, 3], [0, 1, 2, 3], [2], []])
def test_cp_exchange_rows_are_the_retrieval_slices_only(retrieval):
    """The statistics and histograms hold one row per retrieval slice (streaming heads
    never select): sizes scale with the retrieval heads, and the phases still reach the
    oracle's sets with retrieval heads anywhere in the head order, all of them, or none
    (nothing exchanged but the outputs)."""
    import torch
    import cp_host_model as M
    import oracle as O
    from head_partitioned_sparse_b200 import context_parallel as cp
    from head_partitioned_sparse_b200 import synth
    inp = synth.make_inputs("tiny", 6, overrides={"B": 2, "Hq": 16, "Hkv": 4, "retrieval": retrieval, "L": 6000,
                                                   "window": 64, "p": 0.9}, seq_lens=[6000, 2500])
    idx = O.index_cache_for(inp, heads=retrieval)
    R, C = 3, 2000
    sizes = M.exchange_sizes(inp.B, inp.Hq, inp.Hkv, C, R, inp.head_mask)
    every = M.exchange_sizes(inp.B, inp.Hq, inp.Hkv, C, R, [1] * inp.Hkv)
    assert all(sizes[i] * inp.Hkv == every[i] * len(retrieval) for i in range(4))
    assert sizes[4:] == every[4:]
    bufs = {n: torch.zeros(sz, dtype=torch.uint8) for n, sz in zip(cp.BUFFERS, sizes)}
    ranks = [M.HostRank(inp, idx, r, R, C, bufs, p=inp.p, n_sink=inp.n_sink, window=inp.window) for r in range(R)]
    cp.run_step(range(R), lambda ph, r: ranks[r].phase(ph), lambda name: None)
    out = M.combine(ranks[0].out_all, ranks[0].lse_all)
    rows = {k: np.concatenate([rk.rows[k] for rk in ranks]) for k in ranks[0].rows}
    assert _cp_check(inp, idx, out, rows) <= 1e-5


def _cp_worker(rank, world, port, q):
    import datetime

    import torch
    import torch.distributed as dist

    import cp_host_model as M
    from head_partitioned_sparse_b200 import context_parallel as cp

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
        inp, idx = _cp_inputs()
        bufs = {n: torch.zeros(sz, dtype=torch.uint8) for n, sz in
                zip(cp.BUFFERS, M.exchange_sizes(inp.B, inp.Hq, inp.Hkv, CP_C, world, inp.head_mask))}
        me = M.HostRank(inp, idx, rank, world, CP_C, bufs, p=inp.p, n_sink=inp.n_sink, window=inp.window)
        cp.run_step([rank], lambda ph, r: me.phase(ph), lambda name: cp.exchange_buffer(bufs, name, world, rank))
        out = M.combine(me.out_all, me.lse_all)
        # every rank holds the same combined output; rows are gathered to rank 0
        gathered = [None] * world
        dist.all_gather_object(gathered, {k: v.tolist() for k, v in me.rows.items()})
        outs = [None] * world
        dist.all_gather_object(outs, out.tolist())
        if rank == 0:
            rows = {k: np.concatenate([np.asarray(gathered[r][k], np.int64) for r in range(world)])
                    for k in gathered[0]}
            err = _cp_check(inp, idx, out, rows)
            same = all(np.array_equal(np.asarray(o), out) for o in outs)
            # the same phases emulated in one process give the same bits
            ebufs = {n: torch.zeros(sz, dtype=torch.uint8) for n, sz in
                     zip(cp.BUFFERS, M.exchange_sizes(inp.B, inp.Hq, inp.Hkv, CP_C, world, inp.head_mask))}
            er = [M.HostRank(inp, idx, r, world, CP_C, ebufs, p=inp.p, n_sink=inp.n_sink, window=inp.window)
                  for r in range(world)]
            cp.run_step(range(world), lambda ph, r: er[r].phase(ph), lambda name: None)
            emu = M.combine(er[0].out_all, er[0].lse_all)
            hist_same = all(torch.equal(bufs[n], ebufs[n]) for n in cp.BUFFERS)
            q.put(("ok", err, same and np.array_equal(emu, out) and hist_same))
        dist.barrier()
        dist.destroy_process_group()
    except Exception as e:  # report to the parent instead of hanging it
        q.put(("err", repr(e), None))
        raise


def test_cp_two_rank_gloo_exchange_matches_oracle_and_emulation():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_cp_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()
    assert not alive, "a rank did not finish"
    status, err, same = q.get(timeout=5)
    assert status == "ok", err
    assert err <= 1e-5
    assert same, "the gloo run and the one-process emulation differ"
    assert all(p.exitcode == 0 for p in procs)


def _sum_worker(rank, world, port, q):
    import datetime

    import torch
    import torch.distributed as dist

    from head_partitioned_sparse_b200 import context_parallel as cp

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
        words = np.array(_SUM_WORDS[rank], np.uint64)
        bufs = {"hist1": torch.from_numpy(words.view(np.uint8).copy()),
                "hist3": torch.zeros(world * 16, dtype=torch.uint8)}
        bufs["hist3"][rank * 16:(rank + 1) * 16] = rank + 1
        cp.exchange_buffer(bufs, "hist1", world, rank)
        cp.exchange_buffer(bufs, "hist3", world, rank)
        q.put((rank, bufs["hist1"].numpy().view(np.uint64).tolist(), bufs["hist3"].tolist()))
        dist.barrier()
        dist.destroy_process_group()
    except Exception as e:  # report to the parent instead of hanging it
        q.put((rank, "err", repr(e)))
        raise


# uint64 words at and above 2^63, whose sums wrap modulo 2^64
_SUM_WORDS = [[2 ** 63, 2 ** 64 - 1, 5, 2 ** 62], [2 ** 63 + 3, 2, 2 ** 64 - 5, 2 ** 62 + 2 ** 61]]


def test_cp_summed_buffers_all_reduce_as_unsigned_64_bit_words():
    """The summed histograms go through an int64 all-reduce: every rank must end with the
    unsigned sum modulo 2^64 of every rank's words (two's complement addition), and a
    gathered buffer with every rank's slot."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_sum_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()
    assert not alive, "a rank did not finish"
    want = [(a + b) % 2 ** 64 for a, b in zip(*_SUM_WORDS)]
    got = sorted(q.get(timeout=5) for _ in range(2))
    for rank, words, gathered in got:
        assert words != "err", gathered
        assert words == want
        assert gathered == [1] * 16 + [2] * 16
    assert all(p.exitcode == 0 for p in procs)


def test_cp_phases_ties_across_ranks_go_to_the_lowest_positions():
    """Identical index rows (pi = 1/L everywhere): the kept ties are the lowest positions
    of the whole context, so rank 0 keeps all of its rows, rank 1 a prefix, rank 2 none."""
    import torch
    import cp_host_model as M
    import oracle as O
    from head_partitioned_sparse_b200 import context_parallel as cp
    from head_partitioned_sparse_b200 import synth
    inp = synth.make_inputs("tiny", 8, overrides={"L": 1000, "window": 8, "p": float(np.float32(0.7005))})
    idx = O.index_cache_for(inp, heads=[0])
    idx[0, 0, :1000] = idx[0, 0, 500]
    R, C = 3, 400
    bufs = {n: torch.zeros(sz, dtype=torch.uint8) for n, sz in
            zip(cp.BUFFERS, M.exchange_sizes(inp.B, inp.Hq, inp.Hkv, C, R, inp.head_mask))}
    ranks = [M.HostRank(inp, idx, r, R, C, bufs, p=inp.p, n_sink=inp.n_sink, window=8) for r in range(R)]
    cp.run_step(range(R), lambda ph, r: ranks[r].phase(ph), lambda name: None)
    sw = O.sink_window(1000, inp.n_sink, 8)
    kept = np.setdiff1d(np.concatenate([rk.rows[(0, 0)] for rk in ranks]), sw)
    assert np.array_equal(kept, np.setdiff1d(np.arange(701), sw))
    assert len(ranks[2].rows[(0, 0)]) == len(np.intersect1d(sw, np.arange(800, 1000)))


def _decoder_worker(rank, world, port, q):
    """ContextParallelDecoder.step itself over gloo, with the library calls routed to the
    host model of the phases (the buffers, the phase order and the all-gathers are the
    decoder's own)."""
    import datetime

    import torch
    import torch.distributed as dist

    import cp_host_model as M
    from head_partitioned_sparse_b200 import binding as spa
    from head_partitioned_sparse_b200 import context_parallel as cp

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
        inp, idx = _cp_inputs()
        model = {}
        calls = []
        spa.spa_cp_exchange_sizes = lambda h, B, R, mask: M.exchange_sizes(B, inp.Hq, inp.Hkv, CP_C, R, mask)
        spa.spa_cp_phase = lambda h, phase, args, stream=None: (calls.append(phase), model["m"].phase(phase))
        spa.spa_cp_combine = lambda h, out_all, lse_all, R, B, out, stream=None: out.copy_(
            torch.from_numpy(M.combine(model["m"].out_all, model["m"].lse_all)))
        dec = cp.ContextParallelDecoder(0, B=inp.B, capacity=CP_C, device="cpu", head_mask=inp.head_mask)
        model["m"] = M.HostRank(inp, idx, rank, world, CP_C, dec.bufs, p=inp.p, n_sink=inp.n_sink,
                                window=inp.window)
        z = torch.zeros(16, dtype=torch.uint8)
        out = torch.full((inp.B, inp.Hq, 128), float("nan"), dtype=torch.float32)
        dec.step(q_pre=z, k_cache=z, v_cache=z, idx_cache=z, head_mask=inp.head_mask,
                 seq_lens=torch.from_numpy(inp.seq_lens.astype(np.int64)), p=inp.p, n_sink=inp.n_sink,
                 window=inp.window, out=out)
        rows = [None] * world
        dist.all_gather_object(rows, {k: v.tolist() for k, v in model["m"].rows.items()})
        if rank == 0:
            got = {k: np.concatenate([np.asarray(rows[r][k], np.int64) for r in range(world)]) for k in rows[0]}
            err = _cp_check(inp, idx, out.numpy().astype(np.float64), got)
            q.put(("ok", err, calls == [0, 1, 2, 3, 4]))
        dist.barrier()
        dist.destroy_process_group()
    except Exception as e:  # report to the parent instead of hanging it
        q.put(("err", repr(e), None))
        raise


def test_context_parallel_decoder_step_over_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_decoder_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()
    assert not alive, "a rank did not finish"
    status, err, order_ok = q.get(timeout=5)
    assert status == "ok", err
    assert err <= 1e-5
    assert order_ok, "the phases must run once each, in order"
    assert all(p.exitcode == 0 for p in procs)


def test_emulated_step_rejects_exchange_buffers_sized_for_another_mask(monkeypatch):
    """Buffers reused from a step with fewer retrieval heads are too small for this one:
    the driver refuses before any phase is launched."""
    import torch
    import cp_host_model as M
    from head_partitioned_sparse_b200 import binding as spa
    from head_partitioned_sparse_b200 import context_parallel as cp
    B, Hq, Hkv, C, R = 2, 16, 4, 2000, 3
    calls = []
    monkeypatch.setattr(spa, "spa_cp_exchange_sizes", lambda h, b, r, mask: M.exchange_sizes(b, Hq, Hkv, C, r, mask))
    monkeypatch.setattr(spa, "spa_cp_phase", lambda *a, **k: calls.append(a))
    monkeypatch.setattr(spa, "make_cp_args", lambda **k: None)
    small = {n: torch.zeros(sz, dtype=torch.uint8) for n, sz in
             zip(cp.BUFFERS, M.exchange_sizes(B, Hq, Hkv, C, R, [1, 0, 0, 0]))}
    z = torch.zeros(16, dtype=torch.uint8)
    shards = [{"k": z, "v": z, "idx": z}] * R
    kw = dict(q_pre=z, seq_lens=z, Bsz=B, p=0.9, n_sink=4, window=64, capacity=C, out=z, combine=False)
    with pytest.raises(ValueError, match="hist1"):
        cp.emulated_step([0] * R, shards, head_mask=[1, 0, 1, 0], bufs=small, **kw)
    assert calls == []
    cp.emulated_step([0] * R, shards, head_mask=[0, 0, 1, 0], bufs=small, **kw)   # same size: accepted
    assert len(calls) == 5 * R


def test_cp_host_model_masses_are_exact_fixed_point():
    """mass_q(bits(x)) = x * 2^63 exactly for float32 x >= 2^-40, else 0 (the quantised
    mass the histograms sum); cut_desc finds the first bin, from the top, where the
    running mass reaches the target."""
    from fractions import Fraction

    import cp_host_model as M
    rng = np.random.default_rng(3)
    xs = np.concatenate([rng.random(2000, dtype=np.float32) ** 8, np.float32([1.0, 2.0 ** -40, 2.0 ** -41, 0.0])])
    got = M.mass_q(xs.view(np.uint32))
    for x, q in zip(xs.tolist(), got.tolist()):
        want = int(Fraction(x) * 2 ** 63) if x >= 2.0 ** -40 else 0
        assert q == want
    h = np.array([5, 0, 3, 2], np.uint64)          # bins 0..3; from the top: 2, 3, 0, 5
    assert M.cut_desc(h, 0, 1) == (3, 0)
    assert M.cut_desc(h, 0, 3) == (2, 2)
    assert M.cut_desc(h, 0, 5) == (2, 2)
    assert M.cut_desc(h, 0, 6) == (0, 5)
    assert M.cut_desc(h, 4, 10) == (0, 9)
    assert M.cut_desc(h, 0, 11)[0] == -1
