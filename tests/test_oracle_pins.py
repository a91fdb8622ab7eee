"""Pins for the float64 oracle: checks against things other than the oracle itself.

Each test ties one oracle function to a hand-worked case, a closed form, an
invariant, brute force, or an independent library routine (torch), so that a
dropped term, a wrong sign or index, or a transposed operand fails here.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
from index_band import check_index_codes, f32_accumulation_bound, f32_sequential_codes
from head_partitioned_sparse_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield [c.strip() for c in line.split("|")]


# ---------------------------------------------------------------- bf16 rounding
def test_bf16_rounding_matches_torch_on_fp32_values():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(10.0) ** rng.integers(-30, 30, 20000).astype(np.float32),
        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, -3.0e38, 1e-40, -1e-40, 1.17e-38], np.float32),
    ])
    # exact midpoints between neighbouring bf16 values, both parities of the last kept bit
    u = rng.integers(0x00800000, 0x7F000000, 5000, dtype=np.uint64).astype(np.uint32)
    mid = ((u & np.uint32(0xFFFF0000)) | np.uint32(0x8000)).view(np.float32)
    x = np.concatenate([x, mid, -mid])
    ours = O.f64_to_bf16_bits(x.astype(np.float64))
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_bf16_rounding_from_f64_is_single_rounding():
    # 1 + 2^-8 + 2^-40 is just above the midpoint between 1 and 1+2^-7: must round up.
    # Rounding through fp32 first would land exactly on the midpoint and round to even (down).
    v = 1.0 + 2.0 ** -8 + 2.0 ** -40
    assert O.bf16_bits_to_f64(O.f64_to_bf16_bits(np.array([v])))[0] == 1.0 + 2.0 ** -7
    assert O.bf16_bits_to_f64(O.f64_to_bf16_bits(np.array([1.0 + 2.0 ** -8])))[0] == 1.0  # tie -> even


def test_bf16_decode_roundtrip():
    bits = np.arange(0, 0x7F80, 7, dtype=np.uint16)
    assert np.array_equal(O.f64_to_bf16_bits(O.bf16_bits_to_f64(bits)), bits)
    ref = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.bf16_bits_to_f64(bits), ref)


# ---------------------------------------------------------------- RoPE
def test_rope_golden_anchors():
    n = 0
    for row in _rows("rope_cases.txt"):
        if len(row) == 4:
            theta, pos, dim, outs = float(row[0]), int(row[1]), int(row[2]), row[3]
            x = np.zeros(128)
            x[dim] = 1.0
            y = O.rope(x, pos, theta)
            want = np.zeros(128)
            for kv in outs.split():
                k, v = kv.split(":")
                want[int(k)] = float(v)
            np.testing.assert_allclose(y, want, atol=1e-12, rtol=0)
        else:
            theta, i, val = float(row[0]), int(row[1]), float(row[2])
            assert O.rope_inv_freq(128, theta)[i] == pytest.approx(val, rel=1e-14)
        n += 1
    assert n >= 8


def test_rope_is_a_complex_rotation():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((5, 128))
    pos = np.array([0, 1, 17, 4095, 1048575])
    y = O.rope(x, pos, 500000.0)
    # independent construction: z_i = x_i + i x_{i+64}, rotated by exp(i * pos * w_i), w_i geometric
    w = np.exp(-np.arange(64) / 64.0 * math.log(500000.0))
    z = (x[:, :64] + 1j * x[:, 64:]) * np.exp(1j * pos[:, None] * w[None, :])
    np.testing.assert_allclose(y[:, :64], z.real, atol=1e-9)
    np.testing.assert_allclose(y[:, 64:], z.imag, atol=1e-9)


def test_rope_invariants():
    rng = np.random.default_rng(3)
    q, k = rng.standard_normal(128), rng.standard_normal(128)
    np.testing.assert_allclose(O.rope(q, 0, 5e5), q, atol=0)
    assert np.linalg.norm(O.rope(q, 12345, 5e5)) == pytest.approx(np.linalg.norm(q), rel=1e-13)
    a = O.rope(q, 100, 5e5) @ O.rope(k, 40, 5e5)
    b = O.rope(q, 1100, 5e5) @ O.rope(k, 1040, 5e5)
    assert a == pytest.approx(b, rel=1e-9, abs=1e-9)


# ---------------------------------------------------------------- index projection
def test_index_rows_unit_projector_selects_components():
    rng = np.random.default_rng(4)
    perm = rng.permutation(128)[:16]
    P = np.zeros((16, 128))
    P[np.arange(16), perm] = 1.0
    k_bits = synth.f32_to_bf16_bits(rng.standard_normal((33, 128)).astype(np.float32))
    k = O.bf16_bits_to_f64(k_bits)
    got = O.index_rows(k, P)
    assert np.array_equal(got, k_bits[:, perm])          # row r picks component perm[r]
    got2 = O.index_rows(k, 2.0 * P)
    assert np.array_equal(O.bf16_bits_to_f64(got2), 2.0 * k[:, perm])


def test_index_rows_rounds_sum_at_midpoint_to_even():
    P = np.zeros((16, 128))
    P[0, 0] = 1.0
    P[0, 1] = 1.0
    k = np.zeros((2, 128))
    k[0, :2] = [1.0, 2.0 ** -8]          # 1 + 2^-8: midpoint of 1 and 1+2^-7 -> 1 (even)
    k[1, :2] = [1.0 + 2.0 ** -7, 2.0 ** -8]  # midpoint of 1+2^-7 and 1+2^-6 -> 1+2^-6 (even)
    got = O.bf16_bits_to_f64(O.index_rows(k, P))[:, 0]
    assert got[0] == 1.0 and got[1] == 1.0 + 2.0 ** -6


# ---------------------------------------------------------------- index probabilities
def test_index_probs_against_torch_softmax_and_group_mean():
    rng = np.random.default_rng(5)
    G, L = 4, 300
    q = rng.standard_normal((G, 128))
    P = rng.standard_normal((G, 16, 128)) / math.sqrt(128)
    idx = rng.standard_normal((L, 16))
    pi, a = O.index_probs(q, P, idx, 0.25)
    tq, tP, ti = (torch.from_numpy(t) for t in (q, P, idx))
    q_idx = torch.stack([tP[h] @ tq[h] for h in range(G)])           # [G][16]
    ref_a = torch.softmax(0.25 * (ti @ q_idx.T).T, dim=-1)           # [G][L]
    np.testing.assert_allclose(a, ref_a.numpy(), rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(pi, ref_a.mean(0).numpy(), rtol=1e-12, atol=1e-15)
    assert pi.sum() == pytest.approx(1.0, abs=1e-12)


def test_index_probs_projector_acts_on_query_side():
    # With a unit projector, q_idx is a subset of q's components; scores are exact.
    q = np.zeros((1, 128))
    q[0, 7] = 2.0
    P = np.zeros((1, 16, 128))
    P[0, 3, 7] = 1.0                     # index dim 3 <- query dim 7
    idx = np.zeros((3, 16))
    idx[1, 3] = 1.0                      # token 1 matches: score 2 -> logit 0.5
    pi, _ = O.index_probs(q, P, idx, 0.25)
    e = math.exp(0.5)
    np.testing.assert_allclose(pi, [1 / (2 + e), e / (2 + e), 1 / (2 + e)], rtol=1e-14)


# ---------------------------------------------------------------- top-p
def test_top_p_golden_cases():
    n = 0
    for p, masses, kept in _rows("top_p_cases.txt"):
        pi = np.array([float(m) for m in masses.split()])
        want = [int(k) for k in kept.split()]
        assert list(O.top_p(pi, float(p)).kept) == want, (p, masses)
        n += 1
    assert n >= 15


def test_top_p_matches_brute_force_subset_search():
    rng = np.random.default_rng(6)
    for trial in range(300):
        L = int(rng.integers(1, 11))
        pi = rng.random(L) ** 3
        if trial % 5 == 0 and L > 2:   # inject exact ties
            pi[rng.integers(0, L)] = pi[rng.integers(0, L)]
        pi /= pi.sum()
        p = float(rng.choice([0.3, 0.5, 0.8, 0.9, 0.95, 0.99]))
        tp = O.top_p(pi, p)
        # brute force: smallest cardinality whose best subset reaches p
        best = None
        for r in range(1, L + 1):
            cands = [c for c in itertools.combinations(range(L), r) if pi[list(c)].sum() >= p]
            if cands:
                top = max(pi[list(c)].sum() for c in cands)
                best = (r, top)
                break
        if best is None:       # rounding kept the total below p: everything is kept
            assert len(tp.kept) == L
            continue
        assert len(tp.kept) == best[0]
        assert pi[tp.kept].sum() == pytest.approx(best[1], abs=1e-12)


def test_top_p_minimality_and_tie_order():
    rng = np.random.default_rng(7)
    for _ in range(50):
        L = int(rng.integers(50, 400))
        pi = rng.lognormal(0, 2, L)
        pi /= pi.sum()
        for p in (0.5, 0.9, 0.99):
            kept = O.top_p(pi, p).kept
            mass = pi[kept].sum()
            assert mass >= p - 1e-12
            assert mass - pi[kept].min() < p
            # every kept token outranks every dropped one
            dropped = np.setdiff1d(np.arange(L), kept)
            if len(dropped):
                assert pi[kept].min() >= pi[dropped].max()
    pi = np.array([0.2, 0.1, 0.2, 0.1, 0.2, 0.2])
    assert list(O.top_p(pi, 0.5).kept) == [0, 2, 4]   # three tied 0.2s, lowest positions


def test_top_p_p_one_keeps_all():
    pi = np.array([0.7, 0.3, 0.0, 0.0])
    assert list(O.top_p(pi, 1.0).kept) == [0, 1, 2, 3]


# ---------------------------------------------------------------- sink/window
# ---------------------------------------------------------------- top-k
def test_top_k_golden_cases():
    n = 0
    for k, masses, kept in _rows("top_k_cases.txt"):
        pi = np.array([float(m) for m in masses.split()])
        want = [int(x) for x in kept.split()]
        assert list(O.top_k(pi, int(k)).kept) == want, (k, masses)
        n += 1
    assert n >= 13


def test_top_k_is_the_heaviest_k_subset_with_lowest_positions_on_ties():
    rng = np.random.default_rng(16)
    for trial in range(300):
        L = int(rng.integers(1, 10))
        pi = np.round(rng.random(L) * 8) / 8      # coarse values: many exact ties
        k = int(rng.integers(1, L + 2))
        got = list(O.top_k(pi, k).kept)
        if k >= L:
            assert got == list(range(L))
            continue
        # brute force over every k-subset: the largest mass, then the smallest
        # ascending position tuple among subsets of that mass
        best = None
        for c in itertools.combinations(range(L), k):
            key = (-pi[list(c)].sum(), c)
            if best is None or key < best:
                best = key
        assert got == list(best[1]), (pi, k)


def test_top_k_with_the_top_p_count_is_the_top_p_set():
    rng = np.random.default_rng(17)
    for _ in range(100):
        L = int(rng.integers(20, 300))
        pi = rng.lognormal(0, 2, L)
        pi /= pi.sum()
        for p in (0.5, 0.9, 0.99):
            tp = O.top_p(pi, p).kept
            assert np.array_equal(O.top_k(pi, len(tp)).kept, tp)


def test_decode_top_k_covering_context_equals_dense_for_retrieval_heads():
    inp = synth.make_inputs("tiny", 0, overrides={"L": 300, "window": 16})
    dense, _ = O.decode_inputs(inp, p=1.0)
    out, res = O.decode_inputs(inp, k=300)
    r = [g for g in range(inp.Hkv) if inp.head_mask[g]]
    for g in r:
        assert len(res[(0, g)].listed) == 300 - len(O.sink_window(300, inp.n_sink, 16))
    np.testing.assert_allclose(out, dense, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- block-granular top-p
def test_block_top_p_golden_cases():
    n = 0
    for p, blk, masses, kept in _rows("block_top_p_cases.txt"):
        pi = np.array([float(m) for m in masses.split()])
        want = [int(x) for x in kept.split()]
        assert list(O.block_top_p(pi, float(p), int(blk)).kept) == want, (p, blk, masses)
        n += 1
    assert n >= 12


def test_block_top_p_with_unit_blocks_is_top_p():
    rng = np.random.default_rng(18)
    for _ in range(100):
        L = int(rng.integers(1, 200))
        pi = rng.lognormal(0, 2, L)
        pi /= pi.sum()
        for p in (0.3, 0.9, 0.99, 1.0):
            assert np.array_equal(O.block_top_p(pi, p, 1).kept, O.top_p(pi, p).kept)


def test_block_top_p_matches_brute_force_over_blocks():
    rng = np.random.default_rng(19)
    for trial in range(200):
        blk = int(rng.integers(2, 6))
        L = int(rng.integers(1, 8 * blk))
        pi = rng.random(L) ** 3
        pi /= pi.sum()
        p = float(rng.choice([0.3, 0.6, 0.9, 0.99]))
        got = O.block_top_p(pi, p, blk).kept
        nb = (L + blk - 1) // blk
        mass = [pi[b * blk:(b + 1) * blk].sum() for b in range(nb)]
        best = None   # fewest blocks reaching p, then the largest mass
        for r in range(1, nb + 1):
            ok = [c for c in itertools.combinations(range(nb), r) if sum(mass[b] for b in c) >= p]
            if ok:
                best = (r, max(sum(mass[b] for b in c) for c in ok))
                break
        if best is None:          # rounding left the total below p: everything is kept
            assert len(got) == L
            continue
        kept_blocks = sorted({int(j) // blk for j in got})
        assert len(kept_blocks) == best[0]
        assert sum(mass[b] for b in kept_blocks) == pytest.approx(best[1], abs=1e-12)
        # whole blocks only
        for b in kept_blocks:
            assert all(j in set(got.tolist()) for j in range(b * blk, min((b + 1) * blk, L)))


def test_decode_blocks_p1_equals_dense_for_retrieval_heads():
    inp = synth.make_inputs("tiny", 0, overrides={"L": 300, "window": 16})
    dense, _ = O.decode_inputs(inp, p=1.0)
    out, _ = O.decode_inputs(inp, p=1.0, blocks=True)
    np.testing.assert_allclose(out, dense, rtol=0, atol=1e-12)


def test_sink_window_golden():
    for L, ns, w, pos in _rows("sink_window_cases.txt"):
        assert list(O.sink_window(int(L), int(ns), int(w))) == [int(x) for x in pos.split()]


# ---------------------------------------------------------------- attention
def test_attend_matches_torch_sdpa():
    rng = np.random.default_rng(8)
    q, K, V = rng.standard_normal((4, 128)), rng.standard_normal((77, 128)), rng.standard_normal((77, 128))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None], torch.from_numpy(K)[None, None], torch.from_numpy(V)[None, None])
    np.testing.assert_allclose(O.attend(q, K, V), ref[0, 0].numpy(), rtol=1e-12, atol=1e-12)


def _dense_ref(inp, b, g):
    """Full causal-decode attention over all L tokens via torch (independent of the oracle)."""
    L = int(inp.seq_lens[b])
    G = inp.G
    f = (lambda a: O.bf16_bits_to_f64(a)) if inp.dtype == "bf16" else (lambda a: np.asarray(a, np.float64))
    q = f(inp.q_pre[b, g * G:(g + 1) * G])
    # RoPE written independently as a complex rotation
    w = np.exp(-np.arange(64) / 64.0 * math.log(inp.rope_theta))
    z = (q[:, :64] + 1j * q[:, 64:]) * np.exp(1j * (L - 1) * w)
    qr = np.concatenate([z.real, z.imag], axis=1)
    K, V = f(inp.k_cache[b, g, :L]), f(inp.v_cache[b, g, :L])
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(qr)[None, None], torch.from_numpy(K)[None, None], torch.from_numpy(V)[None, None])[0, 0].numpy()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decode_p1_equals_dense_for_retrieval_heads(dtype):
    inp = synth.make_inputs("tiny", 0, overrides={"L": 600, "window": 64, "dtype": dtype, "B": 2},
                            seq_lens=[600, 333])
    out, res = O.decode_inputs(inp, p=1.0)
    for b in range(inp.B):
        ref = _dense_ref(inp, b, 0)
        np.testing.assert_allclose(out[b, 0:4], ref, atol=1e-10)
        assert len(res[(b, 0)].attended) == inp.seq_lens[b]


def test_decode_window_covering_context_equals_dense_for_all_heads():
    inp = synth.make_inputs("tiny", 1, overrides={"L": 500, "window": 64})
    out, _ = O.decode_inputs(inp, window=10 ** 6, p=0.5)
    for g in range(inp.Hkv):
        np.testing.assert_allclose(out[0, g * 4:(g + 1) * 4], _dense_ref(inp, 0, g), atol=1e-10)


def test_decode_streaming_head_sees_only_sinks_and_window():
    inp = synth.make_inputs("tiny", 2, overrides={"L": 700, "window": 32})
    out, res = O.decode_inputs(inp)
    sr = res[(0, 1)]
    assert list(sr.attended) == list(range(4)) + list(range(700 - 32, 700))
    # changing streaming-head keys outside sinks/window changes nothing
    inp.k_cache[0, 1, 100:600] = inp.k_cache[0, 1, 100:600][::-1]
    out2, _ = O.decode_inputs(inp)
    np.testing.assert_array_equal(out[0, 4:8], out2[0, 4:8])


def test_retrieval_output_invariant_to_permuting_kv_order():
    inp = synth.make_inputs("tiny", 3, overrides={"L": 1024, "window": 64})
    idx = O.index_cache_for(inp)
    out, res = O.decode_inputs(inp, idx_cache=idx)
    lo, hi = inp.n_sink, 1024 - inp.window
    rng = np.random.default_rng(9)
    perm = np.arange(1024)
    perm[lo:hi] = lo + rng.permutation(hi - lo)       # new position j holds old row perm[j]
    for arr in (inp.k_cache, inp.v_cache, inp.k_pre):
        arr[0, 0] = arr[0, 0][perm]
    idx2 = idx.copy()
    idx2[0, 0] = idx[0, 0][perm]
    out2, res2 = O.decode_inputs(inp, idx_cache=idx2)
    np.testing.assert_allclose(out2[0, 0:4], out[0, 0:4], atol=1e-12)
    inv = np.argsort(perm)
    assert sorted(perm[res2[(0, 0)].listed]) == sorted(res[(0, 0)].listed)
    assert len(inv) == 1024


def test_index_append_matches_projection_of_each_head():
    inp = synth.make_inputs("tiny", 4, overrides={"L": 64})
    k = np.asarray(inp.k_pre, np.float64)
    bits = O.index_append(k, inp.P_k)
    assert bits.shape == (1, 2, 64, 16)
    # head 1 uses P_k[1], not P_k[0]
    v1 = O.bf16_bits_to_f64(bits[0, 1])
    np.testing.assert_allclose(v1, k[0, 1] @ inp.P_k[1].astype(np.float64).T, rtol=2 ** -8, atol=1e-30)
    assert not np.allclose(v1, k[0, 1] @ inp.P_k[0].astype(np.float64).T, rtol=1e-2)


def test_planted_keys_are_recalled_in_tiny_workload():
    inp = synth.make_inputs("tiny", 0)
    _, res = O.decode_inputs(inp)
    sr = res[(0, 0)]
    planted = inp.planted[(0, 0)]
    assert len(planted) == 4
    assert set(planted) <= set(sr.topp.kept)
    assert len(sr.topp.kept) < 0.05 * inp.seq_lens[0]   # concentrated: a small selected set


# ---------------------------------------------------------------- float32 accumulation band
def test_band_admits_float32_sum_that_straddles_a_midpoint():
    # fp32 inputs: 1 + 2^-8 then four 2^-30 terms.  In float32 each 2^-30 is lost
    # (spacing at 1 is 2^-23), the sum stays on the bf16 midpoint and rounds to even
    # (1.0); the exact value lies above the midpoint and rounds up to 1 + 2^-7.
    P = np.zeros((16, 128), np.float32)
    P[0, :5] = 1.0
    k = np.zeros((1, 128), np.float64)
    k[0, :5] = [1.0 + 2.0 ** -8] + [2.0 ** -30] * 4
    f32 = f32_sequential_codes(k, P)
    assert O.bf16_bits_to_f64(f32)[0, 0] == 1.0
    assert O.bf16_bits_to_f64(O.index_rows(k, P))[0, 0] == 1.0 + 2.0 ** -7
    assert check_index_codes(f32, k, P) == 1          # admitted, and counted as differing


def test_band_float32_model_matches_torch_float32_loop_and_is_admitted():
    rng = np.random.default_rng(12)
    k = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(rng.standard_normal((2000, 128)).astype(np.float32)))
    P = (rng.standard_normal((16, 128)) / math.sqrt(128)).astype(np.float32)
    got = f32_sequential_codes(k.astype(np.float64), P)
    # independent float32 sequential sum with torch (no fused multiply-add on CPU tensors)
    tk, tP = torch.from_numpy(k), torch.from_numpy(P)
    acc = torch.zeros((2000, 16), dtype=torch.float32)
    for d in range(128):
        acc = acc + tk[:, d:d + 1] * tP[None, :, d]
    ref = acc.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)
    n_off = check_index_codes(got, k.astype(np.float64), P)
    assert n_off < 0.01 * got.size                    # rare: only next to a midpoint
    assert check_index_codes(O.index_rows(k.astype(np.float64), P), k.astype(np.float64), P) == 0


def test_band_rejects_a_code_one_step_off_away_from_a_midpoint():
    rng = np.random.default_rng(13)
    k = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(rng.standard_normal((64, 128)).astype(np.float32)))
    P = (rng.standard_normal((16, 128)) / math.sqrt(128)).astype(np.float32)
    k64 = k.astype(np.float64)
    bits = O.index_rows(k64, P).copy()
    exact = k64 @ P.astype(np.float64).T
    beta = f32_accumulation_bound(k64, P)
    far = O.f64_to_bf16_bits(exact - beta) == O.f64_to_bf16_bits(exact + beta)
    i, r = np.argwhere(far)[0]
    bits[i, r] = bits[i, r] + 1                       # next bf16 magnitude
    with pytest.raises(AssertionError):
        check_index_codes(bits, k64, P)
