"""Context-parallel decode: one decode step over sequences whose positions are split
across ranks (host orchestration of the ``spa_cp_*`` phases of libspa).

Rank r holds positions [r C, (r + 1) C) of every sequence in its own caches (C = its
handle's ``max_ctx``; every rank's handle has the same configuration).  A step is the
five phases of ``spa_cp_phase``, each followed by the exchange of the buffer it wrote,
then ``spa_cp_combine``:

    phase          exchanged after it
    SPA_CP_STATS   stats     all-gather: per-head (max, sum of exp) of the local scores
    SPA_CP_MASS    hist1     all-reduce: round-1 mass histogram of the probabilities
    SPA_CP_ROUND2  hist2     all-reduce: round-2 histogram inside the round-1 cut bin
    SPA_CP_ROUND3  hist3     all-gather: round-3 histogram with counts (ties go rank by rank)
    SPA_CP_ATTEND  out_all, lse_all   all-gather: the rank's output and log2-sum-exp

The histograms hold integer masses, so the all-reduced sums are exact.  The statistics
and histograms have rows for the retrieval slices only (streaming heads never select),
so the buffers are sized for one head mask.

Two drivers share that sequence (``run_step``):
  * ``ContextParallelDecoder``: one process per GPU; the exchange is
    ``torch.distributed.all_gather`` or ``all_reduce`` (NCCL on GPUs, gloo for the
    CPU tests);
  * ``emulated_step``: several handles on one GPU, run phase by phase, every rank in
    turn; the ranks share the exchange buffers, so nothing has to move.  No kernel
    waits on another, so this is a plain sequence of launches.

Everything computed runs in libspa's kernels; this module only allocates buffers,
orders the calls and moves the exchanged bytes.
"""
from __future__ import annotations

from typing import Callable, Iterable, List, Sequence, Tuple

from . import binding as spa

BUFFERS = ("stats", "hist1", "hist2", "hist3", "out_all", "lse_all")
# (phase, buffers gathered after it), in order
EXCHANGES: Tuple[Tuple[int, Tuple[str, ...]], ...] = (
    (spa.SPA_CP_STATS, ("stats",)),
    (spa.SPA_CP_MASS, ("hist1",)),
    (spa.SPA_CP_ROUND2, ("hist2",)),
    (spa.SPA_CP_ROUND3, ("hist3",)),
    (spa.SPA_CP_ATTEND, ("out_all", "lse_all")),
)


def run_step(ranks: Iterable[int], run_phase: Callable[[int, int], None], exchange: Callable[[str], None]) -> None:
    """The phase sequence of one step: every phase on each driven rank, then the
    exchange of the buffers that phase wrote.  ``ranks`` is every rank when one process
    emulates them all, else this process's rank."""
    ranks = list(ranks)
    for phase, bufs in EXCHANGES:
        for r in ranks:
            run_phase(phase, r)
        for name in bufs:
            exchange(name)


def rank_span(rank: int, capacity: int) -> Tuple[int, int]:
    """Global positions [pos0, pos0 + capacity) held by ``rank`` in the contiguous split."""
    return rank * capacity, (rank + 1) * capacity


# buffers summed over the ranks (all-reduce); the others have a slot per rank (all-gather)
SUMMED = ("hist1", "hist2")


def allreduce_sum(buf, group=None) -> None:
    """All-reduce (sum) of a buffer of uint64 words, done as int64: two's complement
    addition is unsigned addition modulo 2^64, so the bits are the unsigned sum."""
    import torch
    import torch.distributed as dist
    if buf.numel() == 0:   # no retrieval head: nothing to exchange (the same on every rank)
        return
    dist.all_reduce(buf.view(torch.int64), op=dist.ReduceOp.SUM, group=group)


def exchange_buffer(bufs, name: str, n_ranks: int, rank: int, group=None) -> None:
    """The exchange of buffer ``name`` after the phase that wrote it."""
    if name in SUMMED:
        allreduce_sum(bufs[name], group)
    else:
        allgather_slot(bufs[name], n_ranks, rank, group)


def allgather_slot(buf, n_ranks: int, rank: int, group=None) -> None:
    """All-gather of a [n_ranks][...] buffer whose slot ``rank`` this rank wrote."""
    import torch.distributed as dist
    if buf.numel() == 0:   # no retrieval head: nothing to exchange (the same on every rank)
        return
    v = buf.view(n_ranks, -1)
    mine = v[rank].clone()
    dist.all_gather(list(v.unbind(0)), mine, group=group)


def alloc_exchange(sizes: Sequence[int], device):
    """Exchange buffers (byte tensors) of the sizes spa_cp_exchange_sizes reports.  The
    float outputs are viewed with their element type by the callers."""
    import torch
    return {name: torch.zeros(int(n), dtype=torch.uint8, device=device) for name, n in zip(BUFFERS, sizes)}


def _mask_list(mask):
    return [1 if int(v) else 0 for v in (mask.tolist() if hasattr(mask, "tolist") else mask)]


def _views(bufs):
    import torch
    return bufs["out_all"].view(torch.float32), bufs["lse_all"].view(torch.float32)


class ContextParallelDecoder:
    """One rank of a context-parallel decode step (one process per GPU).

    handle    -- this rank's libspa handle (max_ctx = C, the rank's share of positions)
    B         -- batch of the steps
    head_mask -- [Hkv] retrieval heads of every step (the exchange buffers hold their
                 slices only)
    group     -- torch.distributed process group (default: the world)
    """

    def __init__(self, handle, *, B: int, capacity: int, device, head_mask, group=None):
        import torch.distributed as dist
        self.h = handle
        self.B = B
        self.C = capacity
        self.group = group
        self.rank = dist.get_rank(group)
        self.n_ranks = dist.get_world_size(group)
        self.head_mask = _mask_list(head_mask)
        self.bufs = alloc_exchange(spa.spa_cp_exchange_sizes(handle, B, self.n_ranks, self.head_mask), device)

    def step(self, *, q_pre, k_cache, v_cache, idx_cache, head_mask, seq_lens, p: float, n_sink: int, window: int,
             out, max_seq_len: int = 0, sel_count=None, list_out=None) -> None:
        """Writes the step's output for every query head into ``out`` [B][Hq][128] (on
        every rank).  k/v/idx caches are this rank's shards; seq_lens are global;
        head_mask must be the one the decoder was built with."""
        if _mask_list(head_mask) != self.head_mask:
            raise ValueError("head_mask differs from the one the exchange buffers were sized for")
        out_all, lse_all = _views(self.bufs)
        pos0, _ = rank_span(self.rank, self.C)
        args = spa.make_cp_args(q_pre=q_pre, k_cache=k_cache, v_cache=v_cache, idx_cache=idx_cache,
                              head_mask=head_mask, seq_lens=seq_lens, B=self.B, p=p, n_sink=n_sink, window=window,
                              n_ranks=self.n_ranks, rank=self.rank, pos0=pos0,
                              max_seq_len=max_seq_len or self.n_ranks * self.C,
                              stats=self.bufs["stats"], hist1=self.bufs["hist1"], hist2=self.bufs["hist2"],
                              hist3=self.bufs["hist3"], out_all=out_all, lse_all=lse_all,
                              sel_count_opt=sel_count, list_opt=list_out)
        run_step([self.rank], lambda phase, r: spa.spa_cp_phase(self.h, phase, args),
                 lambda name: exchange_buffer(self.bufs, name, self.n_ranks, self.rank, self.group))
        spa.spa_cp_combine(self.h, out_all, lse_all, self.n_ranks, self.B, out)


def emulated_step(handles: Sequence, shards: Sequence[dict], *, q_pre, head_mask, seq_lens, Bsz: int, p: float,
                  n_sink: int, window: int, capacity: int, out, bufs=None, max_seq_len: int = 0,
                  sel_counts: Sequence = None, lists: Sequence = None, stream=None, ranks: Sequence[int] = None,
                  combine: bool = True, exchange: Callable[[str], None] = None) -> dict:
    """All ranks of a context-parallel step on one GPU: handles[r] and shards[r] (dict of
    ``k``, ``v``, ``idx`` device tensors) are rank r's.  Returns the exchange buffers
    (reusable for the next call through ``bufs``, with the same ``head_mask``).
    ``ranks`` restricts the phases to some ranks (to time one rank's share: the other
    slots of ``bufs`` must then hold an earlier step's exchanged data, and ``exchange``,
    called with each buffer's name after the phase that wrote it, must put the sums
    over all ranks into the summed buffers); ``combine=False`` skips the final merge."""
    R = len(handles)
    need = spa.spa_cp_exchange_sizes(handles[0], Bsz, R, head_mask)
    if bufs is None:
        bufs = alloc_exchange(need, q_pre.device)
    else:   # reused buffers: the kernels index them by this step's batch and head mask
        short = [name for name, n in zip(BUFFERS, need) if bufs[name].numel() < int(n)]
        if short:
            raise ValueError(f"exchange buffers {short} are smaller than this step's batch and head mask need")
    out_all, lse_all = _views(bufs)
    args: List[spa.spa_cp_args] = []
    for r in range(R):
        pos0, _ = rank_span(r, capacity)
        args.append(spa.make_cp_args(
            q_pre=q_pre, k_cache=shards[r]["k"], v_cache=shards[r]["v"], idx_cache=shards[r]["idx"],
            head_mask=head_mask, seq_lens=seq_lens, B=Bsz, p=p, n_sink=n_sink, window=window, n_ranks=R, rank=r,
            pos0=pos0, max_seq_len=max_seq_len or R * capacity, stats=bufs["stats"], hist1=bufs["hist1"],
            hist2=bufs["hist2"], hist3=bufs["hist3"], out_all=out_all, lse_all=lse_all,
            sel_count_opt=None if sel_counts is None else sel_counts[r],
            list_opt=None if lists is None else lists[r]))
    run_step(range(R) if ranks is None else ranks, lambda phase, r: spa.spa_cp_phase(handles[r], phase, args[r], stream),
             exchange or (lambda name: None))
    if combine:
        spa.spa_cp_combine(handles[0], out_all, lse_all, R, Bsz, out, stream)
    return bufs
