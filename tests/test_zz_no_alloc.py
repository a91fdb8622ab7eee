"""spa_select_noalloc: the selection for callers that cannot call cudaMalloc.

Such callers (a host framework that has reserved the GPU's memory for its own
pool, or a decode loop that cannot afford an allocation's implicit device
synchronisation) get an entry point with no handle whose scratch is a static
device array.  Its result must equal spa_select's, exactly (selection is
integer work), on consecutive calls that reuse the same static scratch, and
must agree with the float64 oracle under the selection band.

The calls go from the largest footprint to smaller ones, so a later call lays
its buffers over bytes an earlier call left non-zero: the synchronisation and
per-slice state sit at fixed offsets and are cleared before every launch.

This file is collected last so that, if it fails, a run that stops at the first
failure has already run every other test.
"""
import numpy as np
import pytest
import torch

import oracle as O
from head_partitioned_sparse_b200 import binding as B
from head_partitioned_sparse_b200 import synth
from spa_testutil import DevInputs, Handle, check_selection, gpu_select, kv_dtype_code

pytestmark = pytest.mark.gpu


def _noalloc_select(inp, dev, P_q, p):
    sel = torch.full((inp.B, inp.Hkv, inp.Lmax), -1, dtype=torch.int32, device="cuda")
    cnt = torch.full((inp.B * inp.Hkv,), -1, dtype=torch.int32, device="cuda")
    B.spa_select_noalloc(P_q, inp.Hq, inp.Hkv, kv_dtype_code(inp.dtype), inp.idx_scale, inp.Lmax, dev.q_pre,
                         dev.idx, inp.head_mask, dev.seq_lens, inp.B, 0, p, inp.n_sink, inp.window, sel, cnt)
    torch.cuda.synchronize()
    sel, cnt = sel.cpu().numpy(), cnt.cpu().numpy()
    return {(b, g): sel[b, g, :cnt[b * inp.Hkv + g]].astype(np.int64)
            for b in range(inp.B) for g in range(inp.Hkv)}, cnt.reshape(inp.B, inp.Hkv)


def _cases():
    return [
        # largest footprint first: 2 heads x 2^18 tokens = the 2^19-token limit
        (synth.make_inputs("tiny", 23, overrides={"dtype": "bf16", "L": 1 << 18}), 0.9),
        (synth.make_inputs("tiny", 21, overrides={"dtype": "bf16", "B": 3, "L": 2 * 4096 + 99, "window": 200},
                           seq_lens=[2 * 4096 + 99, 5000, 700]), 0.9),
        (synth.make_inputs("tiny", 22, overrides={"dtype": "bf16", "Hq": 16, "Hkv": 2, "L": 20000,
                                                  "retrieval": [0, 1], "n_planted": 16}), 0.5),
    ]


def test_noalloc_select_matches_spa_select_and_the_oracle_on_calls_in_a_row():
    for rep in range(2):                       # every case twice, on the same static scratch
        for inp, p in _cases():
            pp = float(np.float32(p))
            ret = [g for g in range(inp.Hkv) if inp.head_mask[g]]
            idx = O.index_cache_for(inp, heads=ret)
            with Handle(inp) as h:
                dev = DevInputs(inp, idx)
                want, want_cnt = gpu_select(h, inp, dev, p=pp)
                got, got_cnt = _noalloc_select(inp, dev, h.P_q, pp)
            assert np.array_equal(got_cnt, want_cnt), (rep, inp.L)
            for k in want:
                assert np.array_equal(got[k], want[k]), (rep, k)
            assert got_cnt[:, np.asarray(inp.head_mask) == 1].min() > 0
            if rep == 0:                       # against the float64 oracle, once per case
                _, res = O.decode_inputs(inp, idx_cache=idx, p=pp,
                                         slices=[(b, g) for b in range(inp.B) for g in ret])
                for (b, g), sr in res.items():
                    check_selection(got[(b, g)], sr, pp, inp.n_sink, inp.window)


def test_noalloc_select_rejects_requests_beyond_its_static_scratch():
    inp = synth.make_inputs("tiny", 23, overrides={"dtype": "bf16", "L": 1 << 18})   # 2 heads x 2^18 = 2^19: fits
    idx = O.index_cache_for(inp, heads=[0])
    dev = DevInputs(inp, idx)
    P_q = torch.from_numpy(inp.P_q).cuda()
    sel = torch.zeros((1, 2, 1 << 18), dtype=torch.int32, device="cuda")
    cnt = torch.zeros(2, dtype=torch.int32, device="cuda")
    with pytest.raises(B.SpaError) as e:   # a batch of 2 would need 2^20 tokens of scratch
        B.spa_select_noalloc(P_q, 8, 2, B.SPA_BF16, 0.25, 1 << 18, dev.q_pre, dev.idx, inp.head_mask,
                             torch.tensor([1 << 18, 5], device="cuda"), 2, 0, 0.9, 4, 256, sel, cnt)
    assert e.value.status == B.SPA_ERR_WORKSPACE
    # the largest request that fits runs and agrees with the handle-based path
    got, got_cnt = _noalloc_select(inp, dev, P_q, inp.p)
    with Handle(inp) as h:
        want, want_cnt = gpu_select(h, inp, dev)
    assert np.array_equal(got_cnt, want_cnt) and np.array_equal(got[(0, 0)], want[(0, 0)])
