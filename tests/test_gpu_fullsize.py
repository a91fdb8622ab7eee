"""Full-size workloads, in the launch configuration bench.py times (default split
size, full selection grid, whole batches): the CUDA path runs every slice, and the
float64 oracle checks sampled (sequence, KV head) slices one by one.

Index rows of the sampled retrieval slices come from the oracle; the other
retrieval slices get all-zero index rows, which makes every probability equal (1/L
exactly), so their kept lists are known in closed form: the lowest positions, up to
ceil(p * L) tokens, minus sinks and window.  That checks the tie rule at full size.
"""
import math

import numpy as np
import pytest

import oracle as O
from head_partitioned_sparse_b200 import synth
from spa_testutil import OUT_ATOL, DevInputs, Handle, check_selection, gpu_decode, gpu_select

pytestmark = pytest.mark.gpu


def _to64(inp):
    return (lambda a: O.bf16_bits_to_f64(a)) if inp.dtype == "bf16" else (lambda a: np.asarray(a, np.float64))


def _uniform_list(L, p, n_sink, window):
    """Kept positions outside sinks/window when every probability is 1/L (L a power of 2)."""
    n_keep = L if p >= 1.0 else math.ceil(float(np.float32(p)) * L)
    keep = np.arange(n_keep, dtype=np.int64)
    return np.setdiff1d(keep, O.sink_window(L, n_sink, window))


def _check(name, seed, sample, ps):
    inp = synth.make_inputs(name, seed, draw_streaming_kpre=False)
    assert all(int(L) & (int(L) - 1) == 0 for L in inp.seq_lens)   # closed form needs L = 2^k
    to64 = _to64(inp)
    idx = np.zeros(inp.k_pre.shape[:3] + (16,), np.uint16)
    for (b, g) in sample:
        if inp.head_mask[g]:
            idx[b, g] = O.index_rows(to64(inp.k_pre[b, g]), inp.P_k[g])
    with Handle(inp) as h:
        dev = DevInputs(inp, idx)
        for p in ps:
            pp = float(np.float32(p))
            lists, cnt = gpu_select(h, inp, dev, p=pp)
            out, cnt2 = gpu_decode(h, inp, dev, p=pp)
            assert np.array_equal(cnt, cnt2)
            assert np.isfinite(out).all()
            ref, res = O.decode_inputs(inp, slices=sample, idx_cache=idx, p=pp)
            gpu_sets = {k: lists[k] for k in sample if inp.head_mask[k[1]]}
            ref_gpu, _ = O.decode_inputs(inp, slices=sample, idx_cache=idx, p=pp, attend_sets=gpu_sets)
            G = inp.Hq // inp.Hkv
            for (b, g) in sample:
                heads = slice(g * G, (g + 1) * G)
                if inp.head_mask[g]:
                    check_selection(lists[(b, g)], res[(b, g)], pp, inp.n_sink, inp.window)
                else:
                    assert cnt[b, g] == 0
                err = np.abs(out[b, heads] - ref_gpu[b, heads]).max()
                assert err <= OUT_ATOL, ((b, g), p, err)
            for b in range(inp.B):
                for g in range(inp.Hkv):
                    if inp.head_mask[g] and (b, g) not in sample:
                        want = _uniform_list(int(inp.seq_lens[b]), pp, inp.n_sink, inp.window)
                        assert np.array_equal(lists[(b, g)], want), ((b, g), p)
                    elif not inp.head_mask[g]:
                        assert cnt[b, g] == 0


def test_fullsize_ctx128k_p_sweep():
    # b = 0 concentrated, b = 3 broad (retrieval KV heads 0, 2, 4, 6), plus a streaming slice
    _check("ctx128k", 0, [(0, 0), (3, 2), (1, 1)], [0.8, 0.9, 0.95, 0.99])


def test_fullsize_llama3_8b_32k():
    _check("llama3_8b_32k", 0, [(0, g) for g in range(8)], [0.95])


def test_fullsize_batch16_64k():
    _check("batch16_64k", 0, [(0, 0), (5, 4), (10, 0), (15, 4), (7, 1)], [0.9])


def test_fullsize_ctx1m():
    _check("ctx1m", 0, [(0, 0), (0, 4), (0, 1)], [0.95])
