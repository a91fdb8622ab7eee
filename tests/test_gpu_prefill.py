"""Prefill chunk attention on the GPU vs the float64 oracle.

Tolerance: every checked output element is within a bound derived per element from
the two roundings the kernel makes (everything else is float32): the rotated query is
rounded to bf16 (unit roundoff 2^-8), which moves each
score s_j by at most e_j = 2^-8 sum_d |q_d k_jd| / sqrt(128), so each softmax weight by a
factor within exp(+-2 E), E = max_j e_j; and each weight is rounded to bf16 (2^-8)
before P V.  Hence
  |out_d - oracle_d| <= (2.02 E + 2^-8 + 1e-5) * sum_j p_j |v_jd| + 1e-6,
with 1e-5 covering the float32 scores, exp2 and accumulation.
"""
import numpy as np
import pytest
import torch

import oracle as O
from oracle import prefill_oracle as PF
from head_partitioned_sparse_b200 import binding as B
from head_partitioned_sparse_b200 import synth
from spa_testutil import Handle, dev_storage

pytestmark = pytest.mark.gpu


def run_prefill(h, inp, q, start, T, n_sink=None, window=None):
    out = torch.full((inp.B, inp.Hq, T, 128), float("nan"), dtype=torch.float32, device="cuda")
    B.spa_prefill(h.h, dev_storage(q, "bf16"), dev_storage(inp.k_cache, "bf16"), dev_storage(inp.v_cache, "bf16"),
                  inp.head_mask, torch.tensor(start, dtype=torch.int64, device="cuda"), inp.B, T,
                  inp.n_sink if n_sink is None else n_sink, inp.window if window is None else window, out)
    torch.cuda.synchronize()
    B.spa_device_status(h.h)
    return out.cpu().numpy().astype(np.float64)


def check_rows(inp, q, start, got, rows, n_sink, window):
    f = O.bf16_bits_to_f64
    want = PF.prefill(q, inp.k_cache, inp.v_cache, inp.head_mask, start, n_sink, window, inp.rope_theta,
                      to_f64=f, rows=rows)
    worst = 0.0
    for (b, h, i) in rows:
        keys, p = PF.prefill_weights(q, inp.k_cache, inp.head_mask, start, n_sink, window, inp.rope_theta,
                                     b, h, i, to_f64=f)
        g = h // inp.G
        qr = O.rope(f(q[b, h, i]), int(start[b]) + i, inp.rope_theta)
        K, V = f(inp.k_cache[b, g, keys]), f(inp.v_cache[b, g, keys])
        E = 2.0 ** -8 * np.max(np.abs(K) @ np.abs(qr)) / np.sqrt(128.0)
        bound = (2.02 * E + 2.0 ** -8 + 1e-5) * (p @ np.abs(V)) + 1e-6
        err = np.abs(got[b, h, i] - want[b, h, i])
        assert np.all(err <= bound), (b, h, i, float(err.max()), float(bound[np.argmax(err - bound)]))
        worst = max(worst, float((err / bound).max()))
    return worst


CASES = {
    # name: (overrides, seq starts, chunk T)
    "g4_chunk": ({"dtype": "bf16", "B": 2, "L": 700, "window": 100, "n_sink": 4}, [400, 137], 300),
    "g4_full": ({"dtype": "bf16", "B": 1, "L": 600, "window": 64, "n_sink": 2}, [0], 600),
    "g8": ({"dtype": "bf16", "Hq": 32, "Hkv": 4, "L": 520, "retrieval": [1, 2], "window": 33, "n_sink": 5}, [100], 420),
    "g1": ({"dtype": "bf16", "Hq": 4, "Hkv": 4, "L": 400, "retrieval": [0, 3], "window": 70, "n_sink": 1}, [3], 397),
    "g2_small": ({"dtype": "bf16", "Hq": 4, "Hkv": 2, "L": 90, "window": 7, "n_sink": 3}, [0], 90),
}


@pytest.mark.parametrize("case", list(CASES))
def test_prefill_matches_the_oracle(case):
    ov, start, T = CASES[case]
    inp = synth.make_inputs("tiny", 21, overrides=ov)
    q = synth.prefill_queries(inp, 21, T)
    start = np.array(start, np.int64)
    with Handle(inp) as h:
        got = run_prefill(h, inp, q, start, T)
    assert np.isfinite(got).all()
    rows = [(b, hh, i) for b in range(inp.B) for hh in range(inp.Hq) for i in range(T)]
    rng = np.random.default_rng(1)
    if len(rows) > 1500:
        keep = rng.choice(len(rows), 1500, replace=False)
        rows = [rows[k] for k in sorted(keep)] + [(0, 0, T - 1), (inp.B - 1, inp.Hq - 1, 0)]
    check_rows(inp, q, start, got, rows, inp.n_sink, inp.window)


def test_prefill_long_chunk_sampled_rows():
    inp = synth.make_inputs("tiny", 22, overrides={"dtype": "bf16", "L": 9000, "window": 512, "n_sink": 4})
    T = 9000
    q = synth.prefill_queries(inp, 22, T)
    start = np.array([0], np.int64)
    with Handle(inp) as h:
        got = run_prefill(h, inp, q, start, T)
    assert np.isfinite(got).all()
    rng = np.random.default_rng(2)
    rows = [(0, int(hh), int(i)) for hh, i in zip(rng.integers(0, inp.Hq, 120), rng.integers(0, T, 120))]
    rows += [(0, 0, T - 1), (0, 7, T - 1), (0, 3, 0), (0, 5, 511), (0, 5, 512), (0, 5, 513)]
    check_rows(inp, q, start, got, rows, inp.n_sink, inp.window)


def test_prefill_last_row_equals_dense_decode_step():
    # the chunk's last query is a decode query of length L; with p = 1 the decode path
    # attends the same keys (all of them on retrieval heads, sinks + window elsewhere)
    from spa_testutil import DevInputs, gpu_decode
    inp = synth.make_inputs("tiny", 23, overrides={"dtype": "bf16", "L": 3000, "window": 200})
    T = 64
    q = synth.prefill_queries(inp, 23, T)
    inp.q_pre = np.ascontiguousarray(q[:, :, T - 1])
    idx = O.index_cache_for(inp, heads=[0])
    with Handle(inp) as h:
        got = run_prefill(h, inp, q, np.array([3000 - T], np.int64), T)
        dev = DevInputs(inp, idx)
        dec, _ = gpu_decode(h, inp, dev, p=1.0)
    # both against the oracle: decode within its 2e-3, prefill within its derived bound,
    # and the oracle's decode row is the oracle's prefill row
    want, _ = O.decode_inputs(inp, idx_cache=idx, p=1.0)
    assert np.abs(dec - want).max() <= 2e-3
    start = np.array([3000 - T], np.int64)
    rows = [(0, hh, T - 1) for hh in range(inp.Hq)]
    pre = PF.prefill(q, inp.k_cache, inp.v_cache, inp.head_mask, start, inp.n_sink, inp.window, inp.rope_theta,
                     to_f64=O.bf16_bits_to_f64, rows=rows)
    np.testing.assert_allclose(pre[0, :, T - 1], want[0], atol=1e-12)
    check_rows(inp, q, start, got, rows, inp.n_sink, inp.window)


def test_prefill_rejects_bad_arguments_and_reports_out_of_range_chunks():
    inp = synth.make_inputs("tiny", 0, overrides={"dtype": "bf16", "L": 256})
    q = synth.prefill_queries(inp, 0, 16)
    with Handle(inp) as h:
        with pytest.raises(B.SpaError) as e:
            run_prefill(h, inp, q, np.array([0]), 16, n_sink=0, window=0)
        assert e.value.status == B.SPA_ERR_INVALID_ARG
        with pytest.raises(B.SpaError) as e:
            run_prefill(h, inp, q, np.array([250]), 16)      # 250 + 16 > Lmax
        assert e.value.status == B.SPA_ERR_DEVICE_RANGE
    f32 = synth.make_inputs("tiny", 0, overrides={"L": 256})
    with Handle(f32) as h:
        out = torch.empty((1, f32.Hq, 16, 128), dtype=torch.float32, device="cuda")
        k = torch.zeros((1, f32.Hkv, 256, 128), dtype=torch.float32, device="cuda")
        with pytest.raises(B.SpaError) as e:
            B.spa_prefill(h.h, k, k, k, f32.head_mask, torch.zeros(1, dtype=torch.int64, device="cuda"), 1, 16, 4, 8, out)
        assert e.value.status == B.SPA_ERR_INVALID_ARG
