"""Context-parallel decode (the positions of every sequence split over ranks), with the
ranks emulated on one GPU: one handle and one cache shard per rank, the phases run rank
after rank and the exchange buffers shared (no kernel waits on another).

The union of the ranks' attended rows must be the oracle's set (top-p set, sinks and
window of the whole context; tokens within the selection band of p may differ), and
the combined output must match the oracle evaluated on those rows.
"""
import numpy as np
import pytest
import torch

import oracle as O
from head_partitioned_sparse_b200 import binding as B
from head_partitioned_sparse_b200 import context_parallel as cp
from head_partitioned_sparse_b200 import synth
from spa_testutil import OUT_ATOL, DevInputs, Handle, check_selection, dev_storage, gpu_decode, oracle_idx

pytestmark = pytest.mark.gpu


def _ret(inp):
    return [g for g in range(inp.Hkv) if inp.head_mask[g]]


def _shard(a: np.ndarray, r: int, C: int) -> np.ndarray:
    """Rows [r C, (r + 1) C) of a [B][Hkv][Lmax][d] cache, zero past its end."""
    out = np.zeros(a.shape[:2] + (C,) + a.shape[3:], a.dtype)
    lo, hi = r * C, min((r + 1) * C, a.shape[2])
    if hi > lo:
        out[:, :, :hi - lo] = a[:, :, lo:hi]
    return out


def run_cp(inp, idx, R, C=None, p=None, n_sink=None, window=None):
    """Emulated context-parallel step; returns (out, {(b, g): global rows attended})."""
    L_need = int(inp.seq_lens.max())
    C = C or max(64, -(-L_need // R))
    assert R * C >= L_need
    pp = inp.p if p is None else p
    ns = inp.n_sink if n_sink is None else n_sink
    w = inp.window if window is None else window
    handles = [Handle(inp, max_ctx=C) for _ in range(R)]
    try:
        shards = [{"k": dev_storage(_shard(inp.k_cache, r, C), inp.dtype),
                   "v": dev_storage(_shard(inp.v_cache, r, C), inp.dtype),
                   "idx": dev_storage(_shard(idx, r, C), "bf16")} for r in range(R)]
        q = dev_storage(inp.q_pre, inp.dtype)
        lens = torch.from_numpy(inp.seq_lens.astype(np.int64)).cuda()
        lists = [torch.full((inp.B, inp.Hkv, C), -1, dtype=torch.int32, device="cuda") for _ in range(R)]
        cnts = [torch.full((inp.B * inp.Hkv,), -1, dtype=torch.int32, device="cuda") for _ in range(R)]
        out = torch.full((inp.B, inp.Hq, 128), float("nan"), dtype=torch.float32, device="cuda")
        cp.emulated_step([h.h for h in handles], shards, q_pre=q, head_mask=inp.head_mask, seq_lens=lens,
                         Bsz=inp.B, p=pp, n_sink=ns, window=w, capacity=C, out=out, sel_counts=cnts, lists=lists)
        torch.cuda.synchronize()
        for h in handles:
            B.spa_device_status(h.h)
    finally:
        for h in handles:
            h.close()
    rows = {}
    for b in range(inp.B):
        for g in range(inp.Hkv):
            parts = []
            for r in range(R):
                n = int(cnts[r][b * inp.Hkv + g])
                assert 0 <= n <= C
                loc = lists[r][b, g, :n].cpu().numpy().astype(np.int64)
                assert np.all(np.diff(loc) > 0), "a rank's rows must be strictly ascending"
                parts.append(loc + r * C)
            rows[(b, g)] = np.concatenate(parts)
    return out.cpu().numpy().astype(np.float64), rows


def check_cp(inp, idx, out, rows, p, n_sink, window):
    _, res = O.decode_inputs(inp, idx_cache=idx, p=p, n_sink=n_sink, window=window)
    listed = {}
    for b in range(inp.B):
        L = int(inp.seq_lens[b])
        sw = O.sink_window(L, n_sink, window)
        for g in range(inp.Hkv):
            got = rows[(b, g)]
            assert len(got) == 0 or (got.min() >= 0 and got.max() < L)
            if inp.head_mask[g]:
                assert np.isin(sw, got).all(), "every sink and window position is attended"
                listed[(b, g)] = np.setdiff1d(got, sw)
                check_selection(listed[(b, g)], res[(b, g)], p, n_sink, window)
            else:
                assert np.array_equal(got, sw)
    ref_on_sets, _ = O.decode_inputs(inp, idx_cache=idx, p=p, n_sink=n_sink, window=window, attend_sets=listed)
    assert np.isfinite(out).all()
    err = np.abs(out - ref_on_sets).max()
    assert err <= OUT_ATOL, err
    return listed, res


CASES = {
    "bf16_g4_ragged": ("tiny", 1, {"dtype": "bf16", "B": 3, "L": 3 * 4096 + 123, "window": 300},
                       [3 * 4096 + 123, 7000, 4097]),
    "g8_two_retrieval": ("tiny", 2, {"dtype": "bf16", "Hq": 16, "Hkv": 2, "L": 9000, "retrieval": [0, 1],
                                     "n_planted": 16, "p": 0.95}, None),
    "g1": ("tiny", 3, {"dtype": "bf16", "Hq": 4, "Hkv": 4, "L": 5000, "retrieval": [0, 2], "p": 0.8}, None),
    "g2": ("tiny", 4, {"dtype": "bf16", "Hq": 8, "Hkv": 4, "L": 6000, "retrieval": [1, 2, 3]}, None),
    "broad_halves": ("ctx128k", 0, {"L": 20000, "window": 512, "n_planted_broad": 600}, None),
}
_CACHE = {}


def _prepare(case):
    if case not in _CACHE:
        name, seed, ov, lens = CASES[case]
        inp = synth.make_inputs(name, seed, overrides=ov, seq_lens=lens)
        _CACHE[case] = (inp, oracle_idx(inp, heads=_ret(inp)))
    return _CACHE[case]


@pytest.mark.parametrize("case", list(CASES))
@pytest.mark.parametrize("R", [1, 2, 3, 4])
def test_context_parallel_matches_oracle(case, R):
    inp, idx = _prepare(case)
    out, rows = run_cp(inp, idx, R)
    check_cp(inp, idx, out, rows, inp.p, inp.n_sink, inp.window)


@pytest.mark.parametrize("p", [0.5, 0.99, 1.0])
def test_context_parallel_p_values_and_single_gpu_agreement(p):
    inp, idx = _prepare("bf16_g4_ragged")
    pp = float(np.float32(p))
    out, rows = run_cp(inp, idx, 3, p=pp)
    check_cp(inp, idx, out, rows, pp, inp.n_sink, inp.window)
    with Handle(inp) as h:
        single, _ = gpu_decode(h, inp, DevInputs(inp, idx), p=pp)
    assert np.abs(out - single).max() <= OUT_ATOL


@pytest.mark.parametrize("C", [64, 1000, 4096, 4160])
def test_rank_capacity_edges(C):
    """Shards of one 64-row block, a ragged capacity, exactly one chunk, one chunk plus
    a block; many ranks hold nothing of the shorter sequences."""
    inp, idx = _prepare("g1")
    R = -(-int(inp.seq_lens.max()) // C)
    if R > 80:
        pytest.skip("too many emulated ranks")
    out, rows = run_cp(inp, idx, R, C=C)
    check_cp(inp, idx, out, rows, inp.p, inp.n_sink, inp.window)


def test_ties_across_ranks_keep_lowest_positions():
    """Every token identical (pi = 1/L): the kept ties are positions 0..700 whichever
    rank holds them (rank 0 all of its rows, rank 1 a prefix, rank 2 none)."""
    inp = synth.make_inputs("tiny", 8, overrides={"L": 1000, "dtype": "bf16", "window": 8})
    idx = oracle_idx(inp, heads=[0])
    idx[0, 0, :1000] = idx[0, 0, 500]
    p = float(np.float32(0.7005))
    out, rows = run_cp(inp, idx, 3, C=400, p=p, window=8)
    sw = O.sink_window(1000, inp.n_sink, 8)
    assert np.array_equal(np.setdiff1d(rows[(0, 0)], sw), np.setdiff1d(np.arange(701), sw))
    check_cp(inp, idx, out, rows, p, inp.n_sink, 8)


def test_partial_tie_group_across_ranks_is_cut_by_position():
    inp = synth.make_inputs("tiny", 9, overrides={"L": 6000, "dtype": "bf16", "window": 8})
    idx = oracle_idx(inp, heads=[0])
    rng = np.random.default_rng(0)
    hot = np.sort(rng.choice(np.arange(4, 5990), 50, replace=False))
    idx[0, 0, :6000] = synth.f32_to_bf16_bits(np.full(16, 0.0, np.float32))
    qi = np.einsum("grd,gd->gr", inp.P_q[0:4].astype(np.float64), inp.storage_to_f32(inp.q_pre[0, 0:4]))
    idx[0, 0, hot] = synth.f32_to_bf16_bits((2.0 * qi.mean(0) / np.linalg.norm(qi.mean(0)) * 6).astype(np.float32))
    for p in (0.05, 0.3, 0.6):
        pp = float(np.float32(p))
        out, rows = run_cp(inp, idx, 4, C=1500, p=pp, window=8)
        listed, _ = check_cp(inp, idx, out, rows, pp, inp.n_sink, 8)
        kept_hot = np.intersect1d(listed[(0, 0)], hot)
        if 0 < len(kept_hot) < len(hot):
            assert np.array_equal(kept_hot, hot[:len(kept_hot)])


def test_context_parallel_is_deterministic():
    inp, idx = _prepare("g2")
    a, ra = run_cp(inp, idx, 3)
    b, rb = run_cp(inp, idx, 3)
    assert np.array_equal(a, b)
    assert all(np.array_equal(ra[k], rb[k]) for k in ra)


def test_exchange_rows_are_the_retrieval_slices_only():
    """The statistics and histograms are sized for the retrieval slices of the head mask
    (the layout of the CPU host model of the phases); a mask without retrieval heads
    exchanges none of them (NULL buffers are accepted) and still decodes."""
    import cp_host_model as M
    inp, _ = _prepare("g1")
    with Handle(inp, max_ctx=2048) as h:
        for mask in ([1, 0, 1, 0], [0, 0, 0, 1], [1, 1, 1, 1], [0, 0, 0, 0]):
            got = B.spa_cp_exchange_sizes(h.h, inp.B, 3, mask)
            assert got == M.exchange_sizes(inp.B, inp.Hq, inp.Hkv, 2048, 3, mask)
    inp0 = synth.make_inputs("tiny", 3, overrides={"dtype": "bf16", "Hq": 4, "Hkv": 4, "L": 5000, "retrieval": []})
    idx0 = oracle_idx(inp0, heads=[])
    for R in (1, 3):
        out, rows = run_cp(inp0, idx0, R)
        check_cp(inp0, idx0, out, rows, inp0.p, inp0.n_sink, inp0.window)


def test_context_parallel_argument_errors():
    inp, idx = _prepare("g1")
    with Handle(inp, max_ctx=2048) as h:
        z = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
        good = dict(q_pre=z, k_cache=z, v_cache=z, idx_cache=z, head_mask=inp.head_mask, seq_lens=z, B=inp.B,
                    p=0.9, n_sink=4, window=64, n_ranks=3, rank=1, pos0=2048, max_seq_len=0, stats=z, hist1=z,
                    hist2=z, hist3=z, out_all=z, lse_all=z)
        for bad in ({"rank": 3}, {"n_ranks": 0}, {"p": 0.0}, {"p": 1.5}, {"B": 0}, {"pos0": -1},
                    {"n_sink": 0, "window": 0}, {"stats": None}):
            with pytest.raises(B.SpaError) as e:
                B.spa_cp_phase(h.h, B.SPA_CP_STATS, B.make_cp_args(**{**good, **bad}))
            assert e.value.status == B.SPA_ERR_INVALID_ARG
        with pytest.raises(B.SpaError) as e:
            B.spa_cp_phase(h.h, 7, B.make_cp_args(**good))
        assert e.value.status == B.SPA_ERR_INVALID_ARG
        before = B.spa_launch_count(h.h)
        assert before == 0
