"""Compact KV layout: streaming heads keep only sinks and a ring-buffered window.

The layout rule (a storage layout, no arithmetic): retrieval head of rank r keeps every
position in [b][r][Lmax]; streaming head of rank r keeps position t at ring row t
(t < n_sink) or n_sink + (t - n_sink) mod window.  The expected caches below are built
from that rule in NumPy; decode on the compact caches must equal decode on the full
caches bit for bit (same rows, same order) and the oracle within the usual tolerance.
"""
import numpy as np
import pytest
import torch

import oracle as O
from head_partitioned_sparse_b200 import binding as B
from head_partitioned_sparse_b200 import synth
from index_band import check_index_codes
from spa_testutil import OUT_ATOL, DevInputs, Handle, check_selection, dev_storage, gpu_decode, gpu_select, oracle_idx

pytestmark = pytest.mark.gpu


def ring_row(t, n_sink, window):
    return t if t < n_sink or window <= 0 else n_sink + (t - n_sink) % window


def ranks(mask):
    r, nr, ns = [], 0, 0
    for m in mask:
        r.append(nr if m else ns)
        nr, ns = (nr + 1, ns) if m else (nr, ns + 1)
    return r, nr, ns


class Compact:
    """Device buffers of the compact layout for a synth.Inputs bundle."""

    def __init__(self, inp, n_sink, window, fill=0.0):
        self.rank, self.n_ret, self.n_str = ranks(inp.head_mask)
        self.ring = n_sink + window
        tdt = torch.bfloat16 if inp.dtype == "bf16" else torch.float32
        mk = lambda *shape: torch.full(shape, fill, dtype=tdt, device="cuda")
        self.k_ret = mk(inp.B, max(self.n_ret, 1), inp.Lmax, 128)
        self.v_ret = mk(inp.B, max(self.n_ret, 1), inp.Lmax, 128)
        self.k_ring = mk(inp.B, max(self.n_str, 1), max(self.ring, 1), 128)
        self.v_ring = mk(inp.B, max(self.n_str, 1), max(self.ring, 1), 128)
        self.idx_ret = torch.zeros((inp.B, max(self.n_ret, 1), inp.Lmax, 16), dtype=torch.int16, device="cuda")


def append_sequence(h, inp, dev, cp, b, t0, t1, n_sink, window):
    """Append positions [t0, t1) of sequence b (one call, B = 1, pointers at slot b)."""
    k = dev.k_cache[b:b + 1, :, t0:t1].contiguous()
    v = dev.v_cache[b:b + 1, :, t0:t1].contiguous()
    start = torch.tensor([t0], dtype=torch.int64, device="cuda")
    B.spa_kv_append_compact(h.h, k, v, start, 1, t1 - t0, inp.head_mask, n_sink, window,
                            cp.k_ret[b], cp.v_ret[b], cp.k_ring[b], cp.v_ring[b])


def expected_rows(inp, b, g, L, n_sink, window):
    """(cache row, position) pairs a head must hold after positions [0, L) were appended."""
    if inp.head_mask[g]:
        return [(t, t) for t in range(L)]
    keep = sorted(set(range(min(n_sink, L))) | set(range(max(n_sink, L - window), L)))
    return [(ring_row(t, n_sink, window), t) for t in keep]


def check_layout(inp, cp, lens, n_sink, window):
    kr, vr = cp.k_ret.float().cpu().numpy(), cp.v_ret.float().cpu().numpy()
    ks, vs = cp.k_ring.float().cpu().numpy(), cp.v_ring.float().cpu().numpy()
    to32 = (lambda a: O.bf16_bits_to_f64(a).astype(np.float32)) if inp.dtype == "bf16" else (lambda a: a)
    K, V = to32(inp.k_cache), to32(inp.v_cache)
    for b in range(inp.B):
        for g in range(inp.Hkv):
            rows = expected_rows(inp, b, g, int(lens[b]), n_sink, window)
            r = cp.rank[g]
            kk, vv = (kr[b, r], vr[b, r]) if inp.head_mask[g] else (ks[b, r], vs[b, r])
            idx_r = np.array([x for x, _ in rows], np.int64)
            idx_t = np.array([t for _, t in rows], np.int64)
            assert np.array_equal(kk[idx_r], K[b, g, idx_t]), (b, g)
            assert np.array_equal(vv[idx_r], V[b, g, idx_t]), (b, g)


def ret_idx(idx, ret, cp):
    if not ret:
        return cp.idx_ret
    return torch.from_numpy(np.ascontiguousarray(idx[:, ret]).view(np.int16)).cuda()


CASES = {
    "bf16_g4_ragged": ("tiny", 1, {"dtype": "bf16", "B": 3, "L": 3 * 4096 + 123, "window": 300},
                       [3 * 4096 + 123, 7000, 4097]),
    "g8_mixed": ("tiny", 2, {"dtype": "bf16", "Hq": 32, "Hkv": 4, "L": 9000, "retrieval": [1, 2], "window": 77,
                             "n_sink": 5}, None),
    "f32": ("tiny", 0, {"window": 100}, None),
}


@pytest.mark.parametrize("case", list(CASES))
def test_compact_layout_and_decode_match_full(case):
    name, seed, ov, lens = CASES[case]
    inp = synth.make_inputs(name, seed, overrides=ov, seq_lens=lens)
    ret = [g for g in range(inp.Hkv) if inp.head_mask[g]]
    idx = oracle_idx(inp, heads=ret)
    with Handle(inp) as h:
        dev = DevInputs(inp, idx)
        cp = Compact(inp, inp.n_sink, inp.window, fill=float("nan"))
        # ragged prefill: one call per sequence, in uneven chunks
        for b in range(inp.B):
            L = int(inp.seq_lens[b])
            cuts = sorted({0, L, min(L, 1), min(L, 1000), min(L, 1000 + inp.window // 2), min(L, L - 1)})
            for t0, t1 in zip(cuts[:-1], cuts[1:]):
                if t1 > t0:
                    append_sequence(h, inp, dev, cp, b, t0, t1, inp.n_sink, inp.window)
        # the retrieval heads' index rows through the compact index append
        kp = dev_storage(inp.k_pre, inp.dtype)
        B.spa_index_append_compact(h.h, kp, torch.zeros(inp.B, dtype=torch.int64, device="cuda"), inp.B, inp.Lmax,
                                   inp.head_mask, cp.idx_ret)
        B.spa_device_status(h.h)
        check_layout(inp, cp, inp.seq_lens, inp.n_sink, inp.window)
        got_idx = cp.idx_ret.cpu().numpy().view(np.uint16)
        to64 = (lambda a: O.bf16_bits_to_f64(a)) if inp.dtype == "bf16" else (lambda a: np.asarray(a, np.float64))
        for r, g in enumerate(ret):   # the float64 definition, up to float32 accumulation next to a midpoint
            check_index_codes(got_idx[:, r, :inp.Lmax], to64(inp.k_pre[:, g]), inp.P_k[g])
        # selection and decode: compact == full, bit for bit
        lists_full, cnt_full = gpu_select(h, inp, dev)
        out_full, _ = gpu_decode(h, inp, dev)
        sel = torch.full((inp.B, inp.Hkv, inp.Lmax), -1, dtype=torch.int32, device="cuda")
        cnt = torch.full((inp.B * inp.Hkv,), -1, dtype=torch.int32, device="cuda")
        # the oracle's index rows of the retrieval heads, at their rank
        idx_c = ret_idx(idx, ret, cp)
        B.spa_select_compact(h.h, dev.q_pre, idx_c, inp.head_mask, dev.seq_lens, inp.B, 0, inp.p, inp.n_sink,
                             inp.window, sel, cnt)
        out = torch.full((inp.B, inp.Hq, 128), float("nan"), dtype=torch.float32, device="cuda")
        cnt2 = torch.full((inp.B * inp.Hkv,), -1, dtype=torch.int32, device="cuda")
        B.spa_decode_compact(h.h, dev.q_pre, cp.k_ret, cp.v_ret, cp.k_ring, cp.v_ring, idx_c, inp.head_mask,
                             dev.seq_lens, inp.B, 0, inp.p, inp.n_sink, inp.window, out, cnt2)
        torch.cuda.synchronize()
        B.spa_device_status(h.h)
    cnt = cnt.cpu().numpy().reshape(inp.B, inp.Hkv)
    assert np.array_equal(cnt, cnt_full)
    assert np.array_equal(cnt2.cpu().numpy().reshape(inp.B, inp.Hkv), cnt_full)
    sel = sel.cpu().numpy()
    for (b, g), lst in lists_full.items():
        assert np.array_equal(sel[b, g, :cnt[b, g]], lst)
    out = out.cpu().numpy().astype(np.float64)
    assert np.array_equal(out, out_full), "compact decode must equal full decode bit for bit"
    # and the oracle, on the GPU's sets
    sets = {kk: v for kk, v in lists_full.items() if inp.head_mask[kk[1]]}
    ref, res = O.decode_inputs(inp, idx_cache=idx, attend_sets=sets)
    assert np.abs(out - ref).max() <= OUT_ATOL
    _, own = O.decode_inputs(inp, idx_cache=idx)
    for (b, g), lst in sets.items():
        check_selection(lst, own[(b, g)], inp.p, inp.n_sink, inp.window)


@pytest.mark.parametrize("mask", [[0, 0], [1, 1]])
def test_compact_all_streaming_or_all_retrieval(mask):
    inp = synth.make_inputs("tiny", 5, overrides={"dtype": "bf16", "L": 5000, "window": 64, "retrieval": [],
                                                  "B": 2}, seq_lens=[5000, 333])
    inp.head_mask[:] = np.array(mask, np.uint8)
    ret = [g for g in range(inp.Hkv) if mask[g]]
    idx = oracle_idx(inp, heads=ret) if ret else np.zeros(inp.k_pre.shape[:3] + (16,), np.uint16)
    with Handle(inp) as h:
        dev = DevInputs(inp, idx)
        cp = Compact(inp, inp.n_sink, inp.window)
        for b in range(inp.B):
            append_sequence(h, inp, dev, cp, b, 0, int(inp.seq_lens[b]), inp.n_sink, inp.window)
        check_layout(inp, cp, inp.seq_lens, inp.n_sink, inp.window)
        out_full, cnt_full = gpu_decode(h, inp, dev)
        idx_c = ret_idx(idx, ret, cp)
        out = torch.full((inp.B, inp.Hq, 128), float("nan"), dtype=torch.float32, device="cuda")
        B.spa_decode_compact(h.h, dev.q_pre, cp.k_ret if ret else None, cp.v_ret if ret else None,
                             cp.k_ring if len(ret) < inp.Hkv else None, cp.v_ring if len(ret) < inp.Hkv else None,
                             idx_c, inp.head_mask, dev.seq_lens, inp.B, 0, inp.p, inp.n_sink, inp.window, out)
        torch.cuda.synchronize()
        B.spa_device_status(h.h)
    assert np.array_equal(out.cpu().numpy().astype(np.float64), out_full)


def test_compact_decode_steps_wrap_the_ring():
    # a prefill, then single-token appends past several ring wraps; after each append
    # the ring holds exactly the sinks and the last `window` positions
    n_sink, window = 3, 50
    inp = synth.make_inputs("tiny", 7, overrides={"dtype": "bf16", "L": 700, "window": window, "n_sink": n_sink})
    with Handle(inp) as h:
        dev = DevInputs(inp, np.zeros(inp.k_pre.shape[:3] + (16,), np.uint16))
        cp = Compact(inp, n_sink, window, fill=float("nan"))
        append_sequence(h, inp, dev, cp, 0, 0, 400, n_sink, window)
        for t in range(400, 700):
            append_sequence(h, inp, dev, cp, 0, t, t + 1, n_sink, window)
            if t % 37 == 0 or t == 699:
                B.spa_device_status(h.h)
                check_layout(inp, cp, [t + 1], n_sink, window)


def test_compact_append_rejects_out_of_range_positions():
    inp = synth.make_inputs("tiny", 0, overrides={"dtype": "bf16", "L": 256, "window": 16})
    with Handle(inp) as h:
        dev = DevInputs(inp, np.zeros(inp.k_pre.shape[:3] + (16,), np.uint16))
        cp = Compact(inp, inp.n_sink, inp.window)
        k = dev.k_cache[:, :, :8].contiguous()
        start = torch.tensor([252], dtype=torch.int64, device="cuda")   # 252 + 8 > Lmax = 256
        B.spa_kv_append_compact(h.h, k, k, start, 1, 8, inp.head_mask, inp.n_sink, inp.window,
                                cp.k_ret, cp.v_ret, cp.k_ring, cp.v_ring)
        with pytest.raises(B.SpaError) as e:
            B.spa_device_status(h.h)
        assert e.value.status == B.SPA_ERR_DEVICE_RANGE
        with pytest.raises(B.SpaError) as e:
            B.spa_kv_append_compact(h.h, k, k, start, 1, 8, inp.head_mask, -1, inp.window,
                                    cp.k_ret, cp.v_ret, cp.k_ring, cp.v_ring)
        assert e.value.status == B.SPA_ERR_INVALID_ARG


@pytest.mark.parametrize("selector", ["top_k", "blocks"])
def test_compact_layout_with_other_selectors_matches_full(selector):
    inp = synth.make_inputs("tiny", 9, overrides={"dtype": "bf16", "B": 2, "L": 6000, "window": 200},
                            seq_lens=[6000, 4321])
    ret = [g for g in range(inp.Hkv) if inp.head_mask[g]]
    idx = oracle_idx(inp, heads=ret)
    k_budget = 700
    sel_code = B.SPA_SELECT_TOP_K if selector == "top_k" else B.SPA_SELECT_BLOCKS
    with Handle(inp) as h:
        dev = DevInputs(inp, idx)
        cp = Compact(inp, inp.n_sink, inp.window, fill=float("nan"))
        for b in range(inp.B):
            append_sequence(h, inp, dev, cp, b, 0, int(inp.seq_lens[b]), inp.n_sink, inp.window)
        idx_c = ret_idx(idx, ret, cp)
        out_full = torch.full((inp.B, inp.Hq, 128), float("nan"), dtype=torch.float32, device="cuda")
        cnt_full = torch.full((inp.B * inp.Hkv,), -1, dtype=torch.int32, device="cuda")
        if selector == "top_k":
            B.spa_decode_topk(h.h, dev.q_pre, dev.k_cache, dev.v_cache, dev.idx, inp.head_mask, dev.seq_lens, inp.B,
                              0, k_budget, inp.n_sink, inp.window, out_full, cnt_full)
        else:
            B.spa_decode_blocks(h.h, dev.q_pre, dev.k_cache, dev.v_cache, dev.idx, inp.head_mask, dev.seq_lens,
                                inp.B, 0, inp.p, inp.n_sink, inp.window, out_full, cnt_full)
        out = torch.full_like(out_full, float("nan"))
        cnt = torch.full_like(cnt_full, -1)
        B.spa_decode_compact_sel(h.h, dev.q_pre, cp.k_ret, cp.v_ret, cp.k_ring, cp.v_ring, idx_c, inp.head_mask,
                                 dev.seq_lens, inp.B, 0, sel_code, inp.p, k_budget, inp.n_sink, inp.window, out, cnt)
        sel = torch.full((inp.B, inp.Hkv, inp.Lmax), -1, dtype=torch.int32, device="cuda")
        cnt_s = torch.full_like(cnt_full, -1)
        B.spa_select_compact_sel(h.h, dev.q_pre, idx_c, inp.head_mask, dev.seq_lens, inp.B, 0, sel_code, inp.p,
                                 k_budget, inp.n_sink, inp.window, sel, cnt_s)
        torch.cuda.synchronize()
        B.spa_device_status(h.h)
        with pytest.raises(B.SpaError) as e:   # a bad selector is refused before any launch
            B.spa_select_compact_sel(h.h, dev.q_pre, idx_c, inp.head_mask, dev.seq_lens, inp.B, 0, 7, inp.p,
                                     k_budget, inp.n_sink, inp.window, sel, cnt_s)
        assert e.value.status == B.SPA_ERR_INVALID_ARG
    assert np.array_equal(cnt.cpu().numpy(), cnt_full.cpu().numpy())
    assert np.array_equal(cnt_s.cpu().numpy(), cnt_full.cpu().numpy())
    assert np.array_equal(out.cpu().numpy(), out_full.cpu().numpy()), "compact must equal full bit for bit"
