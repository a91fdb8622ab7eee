"""Top-k selector variant: CUDA path vs the float64 oracle through the C ABI.

The oracle's top_k keeps the first k tokens of the (probability desc, position asc)
order.  The GPU ranks float32 probabilities, so tokens whose oracle probability lies
within a relative 1e-4 of the k-th probability may swap places across the cut; every
other token must agree.  Exact ties (all-zero index rows) must resolve to the lowest
positions bit for bit.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from head_partitioned_sparse_b200 import binding as B
from head_partitioned_sparse_b200 import synth
from spa_testutil import OUT_ATOL, DevInputs, Handle, oracle_idx

pytestmark = pytest.mark.gpu

CUT_RTOL = 1e-4


def _ret(inp):
    return [g for g in range(inp.Hkv) if inp.head_mask[g]]


def gpu_select_topk(h, inp, dev, k, max_seq_len=0):
    sel = torch.full((inp.B, inp.Hkv, inp.Lmax), -1, dtype=torch.int32, device="cuda")
    cnt = torch.full((inp.B * inp.Hkv,), -1, dtype=torch.int32, device="cuda")
    B.spa_select_topk(h.h, dev.q_pre, dev.idx, inp.head_mask, dev.seq_lens, inp.B, max_seq_len, k,
                      inp.n_sink, inp.window, sel, cnt)
    torch.cuda.synchronize()
    sel, cnt = sel.cpu().numpy(), cnt.cpu().numpy()
    lists = {(b, g): sel[b, g, :cnt[b * inp.Hkv + g]].astype(np.int64) for b in range(inp.B) for g in range(inp.Hkv)}
    return lists, cnt.reshape(inp.B, inp.Hkv)


def gpu_decode_topk(h, inp, dev, k):
    out = torch.full((inp.B, inp.Hq, 128), float("nan"), dtype=torch.float32, device="cuda")
    cnt = torch.full((inp.B * inp.Hkv,), -1, dtype=torch.int32, device="cuda")
    B.spa_decode_topk(h.h, dev.q_pre, dev.k_cache, dev.v_cache, dev.idx, inp.head_mask, dev.seq_lens, inp.B, 0, k,
                      inp.n_sink, inp.window, out, cnt)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64), cnt.cpu().numpy().reshape(inp.B, inp.Hkv)


def check_topk(gpu_list, sr, k, n_sink, window):
    """GPU list == oracle list except tokens within CUT_RTOL of the k-th probability."""
    assert np.all(np.diff(gpu_list) > 0), "list must be strictly ascending"
    assert len(gpu_list) == 0 or (gpu_list.min() >= 0 and gpu_list.max() < sr.L)
    assert len(np.intersect1d(gpu_list, O.sink_window(sr.L, n_sink, window))) == 0
    diff = np.setxor1d(gpu_list, sr.listed)
    if len(diff):
        assert k < sr.L, "k >= L must keep everything"
        cut = sr.pi[sr.topp.order[k - 1]]
        off = np.abs(sr.pi[diff] - cut)
        bad = diff[off > CUT_RTOL * cut]
        assert len(bad) == 0, f"{len(bad)} tokens differ away from the cut: {bad[:8]}"
    return len(diff)


CASES = {
    "bf16_g4_ragged": ("tiny", 1, {"dtype": "bf16", "B": 3, "L": 3 * 4096 + 123, "window": 300},
                       [3 * 4096 + 123, 7000, 4097]),
    "g8": ("tiny", 2, {"dtype": "bf16", "Hq": 16, "Hkv": 2, "L": 9000, "retrieval": [0, 1], "n_planted": 16}, None),
    "f32": ("tiny", 0, {}, None),
    "broad": ("ctx128k", 0, {"L": 20000, "window": 512, "n_planted_broad": 600}, None),
}


@pytest.mark.parametrize("case", list(CASES))
@pytest.mark.parametrize("k", [1, 37, 1000, 5000, 10 ** 7])
def test_topk_select_and_decode_parity(case, k):
    name, seed, ov, lens = CASES[case]
    inp = synth.make_inputs(name, seed, overrides=ov, seq_lens=lens)
    idx = oracle_idx(inp, heads=_ret(inp))
    with Handle(inp) as h:
        dev = DevInputs(inp, idx)
        lists, cnt = gpu_select_topk(h, inp, dev, k)
        out, cnt2 = gpu_decode_topk(h, inp, dev, k)
        B.spa_device_status(h.h)
    assert np.array_equal(cnt, cnt2)
    _, res = O.decode_inputs(inp, idx_cache=idx, k=k)
    sets = {kk: v for kk, v in lists.items() if inp.head_mask[kk[1]]}
    ref_gpu, _ = O.decode_inputs(inp, idx_cache=idx, k=k, attend_sets=sets)
    for b in range(inp.B):
        for g in range(inp.Hkv):
            if inp.head_mask[g]:
                check_topk(lists[(b, g)], res[(b, g)], k, inp.n_sink, inp.window)
            else:
                assert cnt[b, g] == 0
    assert np.isfinite(out).all()
    assert np.abs(out - ref_gpu).max() <= OUT_ATOL


def test_topk_ties_keep_lowest_positions():
    # all-zero index rows: every probability is 1/L exactly, the order is the position order
    inp = synth.make_inputs("tiny", 3, overrides={"dtype": "bf16", "L": 8192, "window": 100})
    idx = np.zeros(inp.k_pre.shape[:3] + (16,), np.uint16)
    with Handle(inp) as h:
        dev = DevInputs(inp, idx)
        for k in (1, 4, 5, 777, 8091, 8092, 8193):
            lists, _ = gpu_select_topk(h, inp, dev, k)
            want = np.setdiff1d(np.arange(min(k, 8192)), O.sink_window(8192, inp.n_sink, 100))
            for g in _ret(inp):
                assert np.array_equal(lists[(0, g)], want), k


def test_topk_full_size_ctx128k():
    inp = synth.make_inputs("ctx128k", 0, draw_streaming_kpre=False)
    to64 = lambda a: O.bf16_bits_to_f64(a)
    sample = [(0, 0), (3, 2)]
    idx = np.zeros(inp.k_pre.shape[:3] + (16,), np.uint16)
    for (b, g) in sample:
        idx[b, g] = O.index_rows(to64(inp.k_pre[b, g]), inp.P_k[g])
    k = 4096
    with Handle(inp) as h:
        dev = DevInputs(inp, idx)
        lists, cnt = gpu_select_topk(h, inp, dev, k)
    _, res = O.decode_inputs(inp, slices=sample, idx_cache=idx, k=k)
    for s in sample:
        check_topk(lists[s], res[s], k, inp.n_sink, inp.window)
    L = int(inp.seq_lens[0])
    want = np.setdiff1d(np.arange(k), O.sink_window(L, inp.n_sink, inp.window))
    for b in range(inp.B):
        for g in _ret(inp):
            if (b, g) not in sample:
                assert np.array_equal(lists[(b, g)], want)


def test_topk_rejects_a_zero_budget():
    inp = synth.make_inputs("tiny", 0)
    idx = oracle_idx(inp, heads=_ret(inp))
    with Handle(inp) as h:
        dev = DevInputs(inp, idx)
        n0 = B.spa_launch_count(h.h)
        with pytest.raises(B.SpaError) as e:
            gpu_select_topk(h, inp, dev, 0)
        assert e.value.status == B.SPA_ERR_INVALID_ARG
        assert B.spa_launch_count(h.h) == n0
