"""Failure detection without a GPU fault: a bounded device-side wait runs out.

With the test hook on, the selection kernel's first CTA leaves before the first grid
barrier, so every other CTA waits there for an arrival that never comes until its
bounded wait gives up.  The kernel still completes, spa_device_status reports
SPA_ERR_DEVICE_TIMEOUT, and the next call on the same handle is correct again.
"""
import time

import numpy as np
import pytest

import oracle as O
from head_partitioned_sparse_b200 import binding as B
from head_partitioned_sparse_b200 import synth
from spa_testutil import DevInputs, Handle, check_selection, gpu_decode, gpu_select, oracle_idx, OUT_ATOL

pytestmark = pytest.mark.gpu


def test_missing_barrier_arrival_times_out_and_the_handle_recovers():
    inp = synth.make_inputs("tiny", 0, overrides={"dtype": "bf16", "L": 8192, "window": 256})
    ret = [g for g in range(inp.Hkv) if inp.head_mask[g]]
    idx = oracle_idx(inp, heads=ret)
    with Handle(inp) as h:
        dev = DevInputs(inp, idx)
        B.spa_debug_drop_publish(h.h, True)
        t0 = time.time()
        gpu_select(h, inp, dev)           # returns once the waits have given up
        waited = time.time() - t0
        with pytest.raises(B.SpaError) as e:
            B.spa_device_status(h.h)
        assert e.value.status == B.SPA_ERR_DEVICE_TIMEOUT
        assert 0.5 < waited < 60.0, waited
        B.spa_device_status(h.h)          # reported once, then cleared
        # recovery: the same handle selects and decodes correctly again
        B.spa_debug_drop_publish(h.h, False)
        lists, cnt = gpu_select(h, inp, dev)
        out, cnt2 = gpu_decode(h, inp, dev)
        B.spa_device_status(h.h)
    assert np.array_equal(cnt, cnt2)
    _, res = O.decode_inputs(inp, idx_cache=idx)
    for g in ret:
        check_selection(lists[(0, g)], res[(0, g)], inp.p, inp.n_sink, inp.window)
    sets = {(0, g): lists[(0, g)] for g in ret}
    ref, _ = O.decode_inputs(inp, idx_cache=idx, attend_sets=sets)
    assert np.abs(out - ref).max() <= OUT_ATOL
