"""CUDA path vs the float64 oracle, element by element, through the C ABI.

Sizes span several selection chunks (4096 tokens) and attention tiles (64 rows)
with ragged tails.  Index caches fed to selection/decode come from the oracle,
so no expected value or input here is produced by the CUDA path.
"""
import numpy as np
import pytest
import torch

import oracle as O
from head_partitioned_sparse_b200 import binding as B
from head_partitioned_sparse_b200 import synth
from index_band import check_index_codes
from spa_testutil import (OUT_ATOL, DevInputs, Handle, check_selection, dev_storage, gpu_decode, gpu_select,
                          oracle_idx)

pytestmark = pytest.mark.gpu


def _ret(inp):
    return [g for g in range(inp.Hkv) if inp.head_mask[g]]


# ------------------------------------------------------------------ index append
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_index_append_prefill_parity(dtype):
    inp = synth.make_inputs("tiny", 5, overrides={"L": 3000, "dtype": dtype, "B": 2})
    to64 = (lambda a: O.bf16_bits_to_f64(a)) if dtype == "bf16" else (lambda a: np.asarray(a, np.float64))
    with Handle(inp) as h:
        k = dev_storage(inp.k_pre, dtype)
        idx = torch.zeros((inp.B, inp.Hkv, inp.Lmax, 16), dtype=torch.int16, device="cuda")
        start = torch.zeros(inp.B, dtype=torch.int64, device="cuda")
        B.spa_index_append(h.h, k, start, inp.B, inp.Lmax, idx)
        B.spa_device_status(h.h)
    got = idx.cpu().numpy().view(np.uint16)
    # the float64 definition, bit-exact except next to a bf16 rounding midpoint
    n_off = sum(check_index_codes(got[:, g], to64(inp.k_pre[:, g]), inp.P_k[g]) for g in range(inp.Hkv))
    print(f"index codes one step from the definition (next to a midpoint): {n_off} of {got.size}")
    assert n_off <= 1e-3 * got.size


def test_index_append_decode_rows_at_offsets():
    inp = synth.make_inputs("tiny", 6, overrides={"L": 512, "dtype": "bf16", "B": 3})
    with Handle(inp) as h:
        idx = torch.zeros((3, inp.Hkv, 512, 16), dtype=torch.int16, device="cuda")
        starts = [511, 0, 77]
        T = 1
        k_new = np.stack([inp.k_pre[b, :, starts[b]:starts[b] + T] for b in range(3)])   # [B][Hkv][T][128]
        B.spa_index_append(h.h, dev_storage(k_new, "bf16"), torch.tensor(starts, device="cuda"), 3, T, idx)
        B.spa_device_status(h.h)
        got = idx.cpu().numpy().view(np.uint16)
        k64 = O.bf16_bits_to_f64(inp.k_pre)
        for b in range(3):
            for g in range(inp.Hkv):
                check_index_codes(got[b, g, starts[b]], k64[b, g, starts[b]], inp.P_k[g])
            mask = np.ones(512, bool)
            mask[starts[b]] = False
            assert not got[b][:, mask].any()       # nothing else written
        # an out-of-range start position is skipped and reported
        B.spa_index_append(h.h, dev_storage(k_new, "bf16"), torch.tensor([512, 0, 0], device="cuda"), 3, T, idx)
        with pytest.raises(B.SpaError) as e:
            B.spa_device_status(h.h)
        assert e.value.status == B.SPA_ERR_DEVICE_RANGE
        B.spa_device_status(h.h)   # cleared


# ------------------------------------------------------------------ selection + decode
CASES = {
    "tiny": ("tiny", 0, {}, None),
    "bf16_g4_ragged": ("tiny", 1, {"dtype": "bf16", "B": 3, "L": 3 * 4096 + 123, "window": 300},
                       [3 * 4096 + 123, 7000, 4097]),
    "g8_two_retrieval": ("tiny", 2, {"dtype": "bf16", "Hq": 16, "Hkv": 2, "L": 9000, "retrieval": [0, 1],
                                     "n_planted": 16, "p": 0.95}, None),
    "g1": ("tiny", 3, {"dtype": "bf16", "Hq": 4, "Hkv": 4, "L": 5000, "retrieval": [0, 2], "p": 0.8}, None),
    "g2": ("tiny", 4, {"dtype": "bf16", "Hq": 8, "Hkv": 4, "L": 6000, "retrieval": [1, 2, 3]}, None),
    "broad_halves": ("ctx128k", 0, {"L": 20000, "window": 512, "n_planted_broad": 600}, None),
    "choice": ("batch16_64k", 0, {"B": 4, "L": 10000, "window": 256}, None),
}


def _prepare(case):
    name, seed, ov, lens = CASES[case]
    inp = synth.make_inputs(name, seed, overrides=ov, seq_lens=lens)
    idx = oracle_idx(inp, heads=_ret(inp))
    return inp, idx


@pytest.fixture(scope="module")
def prepared():
    cache = {}

    def get(case):
        if case not in cache:
            cache[case] = _prepare(case)
        return cache[case]
    return get


@pytest.mark.parametrize("case", list(CASES))
@pytest.mark.parametrize("p", [None, 0.5, 0.99, 1.0])
def test_select_and_decode_parity(prepared, case, p):
    inp, idx = prepared(case)
    pp = inp.p if p is None else float(np.float32(p))
    with Handle(inp) as h:
        dev = DevInputs(inp, idx)
        lists, cnt = gpu_select(h, inp, dev, p=pp)
        out, cnt2 = gpu_decode(h, inp, dev, p=pp)
        B.spa_device_status(h.h)
    assert np.array_equal(cnt, cnt2)
    ref, res = O.decode_inputs(inp, idx_cache=idx, p=pp)
    ref_on_gpu_sets, _ = O.decode_inputs(inp, idx_cache=idx, p=pp,
                                         attend_sets={k: v for k, v in lists.items() if inp.head_mask[k[1]]})
    for b in range(inp.B):
        for g in range(inp.Hkv):
            if inp.head_mask[g]:
                nd = check_selection(lists[(b, g)], res[(b, g)], pp, inp.n_sink, inp.window)
                if pp >= 1.0:
                    assert len(lists[(b, g)]) == len(res[(b, g)].listed)
            else:
                assert cnt[b, g] == 0
    assert np.isfinite(out).all()
    err = np.abs(out - ref_on_gpu_sets).max()
    assert err <= OUT_ATOL, err
    same = all(np.array_equal(lists[k], res[k].listed) for k in lists if inp.head_mask[k[1]])
    if same:
        assert np.abs(out - ref).max() <= OUT_ATOL


def test_batch_split_over_several_selection_launches():
    # more retrieval slices (320) than co-resident selection CTAs: the batch runs as
    # several prologue + selection launches over whole sequences; ragged lengths catch a
    # launch reading another launch's sequences
    n_b = 320
    lens = [64 + (37 * b) % 449 for b in range(n_b)]
    inp = synth.make_inputs("tiny", 11, overrides={"B": n_b, "L": 512, "dtype": "bf16", "window": 32},
                            seq_lens=lens)
    idx = oracle_idx(inp, heads=_ret(inp))
    pp = float(np.float32(inp.p))
    with Handle(inp) as h:
        dev = DevInputs(inp, idx)
        lists, cnt = gpu_select(h, inp, dev, p=pp)
        out, cnt2 = gpu_decode(h, inp, dev, p=pp)
        B.spa_device_status(h.h)
    assert np.array_equal(cnt, cnt2)
    ref_on_gpu_sets, res = O.decode_inputs(inp, idx_cache=idx, p=pp,
                                           attend_sets={k: v for k, v in lists.items() if inp.head_mask[k[1]]})
    for b in range(inp.B):
        for g in range(inp.Hkv):
            if inp.head_mask[g]:
                check_selection(lists[(b, g)], res[(b, g)], pp, inp.n_sink, inp.window)
            else:
                assert cnt[b, g] == 0
    assert np.isfinite(out).all()
    assert np.abs(out - ref_on_gpu_sets).max() <= OUT_ATOL


@pytest.mark.parametrize("L", [1, 2, 17, 4095, 4096, 4097])
@pytest.mark.parametrize("n_sink,window", [(4, 0), (0, 1), (4, 256), (0, 10 ** 6), (4, 64)])
def test_edge_lengths_and_windows(L, n_sink, window):
    inp = synth.make_inputs("tiny", 7, overrides={"L": max(L, 8), "dtype": "bf16", "window": 16},
                            seq_lens=[L])
    idx = oracle_idx(inp, heads=[0])
    with Handle(inp) as h:
        dev = DevInputs(inp, idx)
        lists, _ = gpu_select(h, inp, dev, n_sink=n_sink, window=window)
        out, _ = gpu_decode(h, inp, dev, n_sink=n_sink, window=window)
        B.spa_device_status(h.h)
    ref, res = O.decode_inputs(inp, idx_cache=idx, n_sink=n_sink, window=window,
                               attend_sets={(0, 0): lists[(0, 0)]})
    check_selection(lists[(0, 0)], O.decode_inputs(inp, idx_cache=idx, n_sink=n_sink, window=window)[1][(0, 0)],
                    inp.p, n_sink, window)
    assert np.abs(out - ref).max() <= OUT_ATOL


def test_uniform_index_ties_keep_lowest_positions():
    inp = synth.make_inputs("tiny", 8, overrides={"L": 1000, "dtype": "bf16", "window": 8})
    idx = oracle_idx(inp, heads=[0])
    idx[0, 0, :1000] = idx[0, 0, 500]          # every token identical: pi = 1/L
    p = float(np.float32(0.7005))               # keeps ceil(700.5) = 701 tokens: positions 0..700
    with Handle(inp) as h:
        dev = DevInputs(inp, idx)
        lists, _ = gpu_select(h, inp, dev, p=p)
        out, _ = gpu_decode(h, inp, dev, p=p)
    want = np.setdiff1d(np.arange(701), O.sink_window(1000, inp.n_sink, 8))
    assert np.array_equal(lists[(0, 0)], want)
    _, res = O.decode_inputs(inp, idx_cache=idx, p=p, window=8)
    assert np.array_equal(res[(0, 0)].listed, want)
    ref, _ = O.decode_inputs(inp, idx_cache=idx, p=p, window=8)
    assert np.abs(out - ref).max() <= OUT_ATOL


def test_partial_tie_group_is_cut_by_position():
    inp = synth.make_inputs("tiny", 9, overrides={"L": 6000, "dtype": "bf16", "window": 8})
    idx = oracle_idx(inp, heads=[0])
    rng = np.random.default_rng(0)
    hot = np.sort(rng.choice(np.arange(4, 5990), 50, replace=False))
    row = synth.f32_to_bf16_bits(np.full(16, 0.0, np.float32))
    idx[0, 0, :6000] = row                                   # cold tokens: logit 0
    qi = np.einsum("grd,gd->gr", inp.P_q[0:4].astype(np.float64), inp.storage_to_f32(inp.q_pre[0, 0:4]))
    hot_row = synth.f32_to_bf16_bits((2.0 * qi.mean(0) / np.linalg.norm(qi.mean(0)) * 6).astype(np.float32))
    idx[0, 0, hot] = hot_row                                 # 50 identical hot tokens
    with Handle(inp) as h:
        dev = DevInputs(inp, idx)
        for p in (0.05, 0.3, 0.6):
            pp = float(np.float32(p))
            lists, _ = gpu_select(h, inp, dev, p=pp)
            _, res = O.decode_inputs(inp, idx_cache=idx, p=pp, window=8)
            check_selection(lists[(0, 0)], res[(0, 0)], pp, inp.n_sink, 8)
            kept_hot = np.intersect1d(lists[(0, 0)], hot)
            if 0 < len(kept_hot) < len(hot):
                assert np.array_equal(kept_hot, hot[:len(kept_hot)])   # lowest positions first


@pytest.mark.parametrize("split_rows", [64, 128, 576, 8192])
def test_split_count_does_not_change_the_output(prepared, split_rows):
    inp, idx = prepared("bf16_g4_ragged")
    with Handle(inp, split_rows=split_rows) as h:
        out, _ = gpu_decode(h, inp, DevInputs(inp, idx))
    with Handle(inp, split_rows=64) as h:
        out64, _ = gpu_decode(h, inp, DevInputs(inp, idx))
    ref, _ = O.decode_inputs(inp, idx_cache=idx)
    assert np.abs(out - ref).max() <= OUT_ATOL
    assert np.abs(out - out64).max() <= 1e-4


def test_decode_is_deterministic(prepared):
    inp, idx = prepared("broad_halves")
    with Handle(inp) as h:
        dev = DevInputs(inp, idx)
        a = gpu_decode(h, inp, dev)
        la, _ = gpu_select(h, inp, dev)
        b = gpu_decode(h, inp, dev)
        lb, _ = gpu_select(h, inp, dev)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    assert all(np.array_equal(la[k], lb[k]) for k in la)


def test_reads_stay_inside_each_sequence():
    # rows at positions >= seq_len are NaN: any read past the context would show up
    inp = synth.make_inputs("tiny", 10, overrides={"dtype": "bf16", "B": 3, "L": 9000, "window": 100},
                            seq_lens=[9000, 4100, 33], poison_tail=True)
    idx = oracle_idx(inp, heads=[0])
    idx[1, :, 4100:] = 0x7FC0
    idx[2, :, 33:] = 0x7FC0
    with Handle(inp) as h:
        dev = DevInputs(inp, idx)
        lists, _ = gpu_select(h, inp, dev)
        out, _ = gpu_decode(h, inp, dev)
    assert np.isfinite(out).all()
    _, res = O.decode_inputs(inp, idx_cache=idx)
    for b in range(3):
        check_selection(lists[(b, 0)], res[(b, 0)], inp.p, inp.n_sink, inp.window)
    ref, _ = O.decode_inputs(inp, idx_cache=idx, attend_sets={(b, 0): lists[(b, 0)] for b in range(3)})
    assert np.abs(out - ref).max() <= OUT_ATOL


@pytest.mark.parametrize("retrieval", [[], [0, 1, 2, 3]])
def test_all_streaming_and_all_retrieval(retrieval):
    inp = synth.make_inputs("tiny", 4, overrides={"dtype": "bf16", "Hq": 8, "Hkv": 4, "L": 6000,
                                                  "retrieval": retrieval})
    idx = oracle_idx(inp)
    with Handle(inp) as h:
        dev = DevInputs(inp, idx)
        lists, _ = gpu_select(h, inp, dev)
        n0 = B.spa_launch_count(h.h)
        out, cnt = gpu_decode(h, inp, dev)
        launches = B.spa_launch_count(h.h) - n0
    assert launches == (2 if inp.dtype == "bf16" else 3)   # selection, attention (+ combine for float32 caches)
    _, res = O.decode_inputs(inp, idx_cache=idx)
    for g in retrieval:
        check_selection(lists[(0, g)], res[(0, g)], inp.p, inp.n_sink, inp.window)
    ref, _ = O.decode_inputs(inp, idx_cache=idx, attend_sets={(0, g): lists[(0, g)] for g in retrieval})
    assert np.abs(out - ref).max() <= OUT_ATOL
    if not retrieval:
        assert not cnt.any()


def test_host_argument_errors_launch_nothing():
    inp = synth.make_inputs("tiny", 11, overrides={"L": 256, "dtype": "bf16", "window": 16})
    idx = oracle_idx(inp, heads=[0])
    with Handle(inp) as h:
        dev = DevInputs(inp, idx)
        out = torch.zeros((1, 8, 128), dtype=torch.float32, device="cuda")
        n0 = B.spa_launch_count(h.h)
        bad = [
            dict(p=0.0), dict(p=1.5), dict(p=float("nan")), dict(n_sink=0, window=0), dict(n_sink=-1),
            dict(Bn=2), dict(max_seq_len=257), dict(q_off=2), dict(out_off=4),
        ]
        for kw in bad:
            args = dict(p=0.9, n_sink=4, window=16, Bn=1, max_seq_len=0, q_off=0, out_off=0)
            args.update(kw)
            with pytest.raises(B.SpaError) as e:
                B.spa_decode(h.h, dev.q_pre.data_ptr() + args["q_off"], dev.k_cache, dev.v_cache, dev.idx,
                             inp.head_mask, dev.seq_lens, args["Bn"], args["max_seq_len"], args["p"],
                             args["n_sink"], args["window"], out.data_ptr() + args["out_off"])
            assert e.value.status == B.SPA_ERR_INVALID_ARG, kw
        assert B.spa_launch_count(h.h) == n0
        # a device-resident length beyond max_seq_len is clamped and reported
        bad_lens = torch.tensor([300], dtype=torch.int64, device="cuda")
        B.spa_decode(h.h, dev.q_pre, dev.k_cache, dev.v_cache, dev.idx, inp.head_mask, bad_lens, 1, 0, 0.9, 4, 16,
                     out)
        with pytest.raises(B.SpaError) as e:
            B.spa_device_status(h.h)
        assert e.value.status == B.SPA_ERR_DEVICE_RANGE
        B.spa_device_status(h.h)


def test_untied_projectors():
    inp = synth.make_inputs("tiny", 12, overrides={"dtype": "bf16", "L": 5000}, tied=False)
    idx = oracle_idx(inp, heads=[0])
    with Handle(inp) as h:
        dev = DevInputs(inp, idx)
        lists, _ = gpu_select(h, inp, dev)
        out, _ = gpu_decode(h, inp, dev)
    ref, res = O.decode_inputs(inp, idx_cache=idx, attend_sets={(0, 0): lists[(0, 0)]})
    check_selection(lists[(0, 0)], O.decode_inputs(inp, idx_cache=idx)[1][(0, 0)], inp.p, inp.n_sink, inp.window)
    assert np.abs(out - ref).max() <= OUT_ATOL
