"""Block-granular top-p variant: CUDA path vs the float64 oracle through the C ABI.

The oracle's block_top_p ranks 64-token blocks by their summed probability and
keeps whole blocks while the mass before them is below p.  The GPU sums float32
probabilities, so a block whose oracle running mass lies within SEL_BAND of p may
fall on either side of the cut; every other block must agree, and every listed
token's block must be listed whole (sinks and window aside).
"""
import numpy as np
import pytest
import torch

import oracle as O
from head_partitioned_sparse_b200 import binding as B
from head_partitioned_sparse_b200 import synth
from spa_testutil import OUT_ATOL, DevInputs, Handle, check_selection, oracle_idx

pytestmark = pytest.mark.gpu

BLOCK = O.BLOCK


def _ret(inp):
    return [g for g in range(inp.Hkv) if inp.head_mask[g]]


def gpu_select_blocks(h, inp, dev, p, max_seq_len=0, n_sink=None, window=None):
    sel = torch.full((inp.B, inp.Hkv, inp.Lmax), -1, dtype=torch.int32, device="cuda")
    cnt = torch.full((inp.B * inp.Hkv,), -1, dtype=torch.int32, device="cuda")
    B.spa_select_blocks(h.h, dev.q_pre, dev.idx, inp.head_mask, dev.seq_lens, inp.B, max_seq_len, p,
                        inp.n_sink if n_sink is None else n_sink, inp.window if window is None else window, sel, cnt)
    torch.cuda.synchronize()
    sel, cnt = sel.cpu().numpy(), cnt.cpu().numpy()
    lists = {(b, g): sel[b, g, :cnt[b * inp.Hkv + g]].astype(np.int64) for b in range(inp.B) for g in range(inp.Hkv)}
    return lists, cnt.reshape(inp.B, inp.Hkv)


def gpu_decode_blocks(h, inp, dev, p):
    out = torch.full((inp.B, inp.Hq, 128), float("nan"), dtype=torch.float32, device="cuda")
    cnt = torch.full((inp.B * inp.Hkv,), -1, dtype=torch.int32, device="cuda")
    B.spa_decode_blocks(h.h, dev.q_pre, dev.k_cache, dev.v_cache, dev.idx, inp.head_mask, dev.seq_lens, inp.B, 0, p,
                        inp.n_sink, inp.window, out, cnt)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64), cnt.cpu().numpy().reshape(inp.B, inp.Hkv)


def check_whole_blocks(gpu_list, L, n_sink, window):
    """Every block that holds a listed token is listed whole (minus sinks and window)."""
    base = set(O.sink_window(L, n_sink, window).tolist())
    got = set(gpu_list.tolist())
    for blk in np.unique(gpu_list // BLOCK):
        want = {j for j in range(blk * BLOCK, min(L, (blk + 1) * BLOCK)) if j not in base}
        assert want <= got, f"block {blk} listed in part"


CASES = {
    "bf16_g4_ragged": ("tiny", 1, {"dtype": "bf16", "B": 3, "L": 3 * 4096 + 123, "window": 300},
                       [3 * 4096 + 123, 7000, 4097]),
    "g8": ("tiny", 2, {"dtype": "bf16", "Hq": 16, "Hkv": 2, "L": 9000, "retrieval": [0, 1], "n_planted": 16}, None),
    "f32": ("tiny", 0, {}, None),
    "broad": ("ctx128k", 0, {"L": 20000, "window": 512, "n_planted_broad": 600}, None),
    "short": ("tiny", 4, {"dtype": "bf16", "B": 4, "L": 200, "window": 8, "n_sink": 2}, [200, 1, 63, 65]),
}


@pytest.mark.parametrize("case", list(CASES))
@pytest.mark.parametrize("p", [0.5, 0.9, 0.99, 1.0])
def test_blocks_select_and_decode_parity(case, p):
    name, seed, ov, lens = CASES[case]
    inp = synth.make_inputs(name, seed, overrides=ov, seq_lens=lens)
    idx = oracle_idx(inp, heads=_ret(inp))
    with Handle(inp) as h:
        dev = DevInputs(inp, idx)
        lists, cnt = gpu_select_blocks(h, inp, dev, p)
        out, cnt2 = gpu_decode_blocks(h, inp, dev, p)
        B.spa_device_status(h.h)
    assert np.array_equal(cnt, cnt2)
    _, res = O.decode_inputs(inp, idx_cache=idx, p=p, blocks=True)
    sets = {kk: v for kk, v in lists.items() if inp.head_mask[kk[1]]}
    ref_gpu, _ = O.decode_inputs(inp, idx_cache=idx, p=p, blocks=True, attend_sets=sets)
    for b in range(inp.B):
        L = int(inp.seq_lens[b])
        for g in range(inp.Hkv):
            if inp.head_mask[g]:
                check_selection(lists[(b, g)], res[(b, g)], p, inp.n_sink, inp.window)
                check_whole_blocks(lists[(b, g)], L, inp.n_sink, inp.window)
            else:
                assert cnt[b, g] == 0
    assert np.isfinite(out).all()
    assert np.abs(out - ref_gpu).max() <= OUT_ATOL


@pytest.mark.parametrize("L", [8192, 8192 + 100, 64, 1])
def test_blocks_ties_keep_lowest_blocks(L):
    # all-zero index rows: full blocks have equal mass, ties go to the lowest blocks
    inp = synth.make_inputs("tiny", 3, overrides={"dtype": "bf16", "L": max(L, 64), "window": 10, "n_sink": 0},
                            seq_lens=[L])
    idx = np.zeros(inp.k_pre.shape[:3] + (16,), np.uint16)
    with Handle(inp) as h:
        dev = DevInputs(inp, idx)
        for p in (0.25, 0.5, 0.75):
            lists, _ = gpu_select_blocks(h, inp, dev, p)
            pi = np.full(L, 1.0 / L)
            want = np.setdiff1d(O.block_top_p(pi, p).kept, O.sink_window(L, 0, 10))
            for g in _ret(inp):
                assert np.array_equal(lists[(0, g)], want), (L, p)


def test_blocks_full_size_ctx128k():
    inp = synth.make_inputs("ctx128k", 0, draw_streaming_kpre=False)
    to64 = lambda a: O.bf16_bits_to_f64(a)
    sample = [(0, 0), (3, 2)]
    idx = np.zeros(inp.k_pre.shape[:3] + (16,), np.uint16)
    for (b, g) in sample:
        idx[b, g] = O.index_rows(to64(inp.k_pre[b, g]), inp.P_k[g])
    with Handle(inp) as h:
        dev = DevInputs(inp, idx)
        lists, cnt = gpu_select_blocks(h, inp, dev, inp.p)
    _, res = O.decode_inputs(inp, slices=sample, idx_cache=idx, p=inp.p, blocks=True)
    for (b, g) in sample:
        L = int(inp.seq_lens[b])
        check_selection(lists[(b, g)], res[(b, g)], inp.p, inp.n_sink, inp.window)
        check_whole_blocks(lists[(b, g)], L, inp.n_sink, inp.window)
    # the other slices have all-zero index rows: equal block masses, lowest blocks first
    L = int(inp.seq_lens[0])
    want = np.setdiff1d(O.block_top_p(np.full(L, 1.0 / L), inp.p).kept, O.sink_window(L, inp.n_sink, inp.window))
    for b in range(inp.B):
        for g in _ret(inp):
            if (b, g) not in sample:
                assert np.array_equal(lists[(b, g)], want)


def test_blocks_rejects_a_bad_p():
    inp = synth.make_inputs("tiny", 0)
    idx = oracle_idx(inp, heads=_ret(inp))
    with Handle(inp) as h:
        dev = DevInputs(inp, idx)
        n0 = B.spa_launch_count(h.h)
        for p in (0.0, 1.5, float("nan")):
            with pytest.raises(B.SpaError) as e:
                gpu_select_blocks(h, inp, dev, p)
            assert e.value.status == B.SPA_ERR_INVALID_ARG
        assert B.spa_launch_count(h.h) == n0
