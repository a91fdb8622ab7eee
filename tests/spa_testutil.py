"""Helpers shared by the GPU tests: upload seeded inputs, run the library through
its C ABI, and compare with the float64 oracle under the stated tolerances."""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
from head_partitioned_sparse_b200 import binding as B
from head_partitioned_sparse_b200 import synth

# Tolerances (stated for this method's decode step):
#  - selected sets: identical except tokens whose oracle running mass before them
#    lies within SEL_BAND of p;
#  - attention outputs: max-abs OUT_ATOL (bf16 inputs, fp32 accumulation).
SEL_BAND = 1e-5
OUT_ATOL = 2e-3


def dev_storage(a: np.ndarray, dtype: str) -> torch.Tensor:
    """Upload a storage array (uint16 bf16 bits or float32) to the GPU."""
    if dtype == "bf16" or a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def kv_dtype_code(dtype: str) -> int:
    return B.SPA_BF16 if dtype == "bf16" else B.SPA_F32


class Handle:
    """spa_create / spa_destroy around a synth.Inputs bundle."""

    def __init__(self, inp: synth.Inputs, split_rows: int = 0, max_batch: int = None, max_ctx: int = None):
        self.P_q = torch.from_numpy(inp.P_q).cuda()
        self.P_k = torch.from_numpy(inp.P_k).cuda()
        cfg = B.make_config(max_batch=max_batch or inp.B, n_q_heads=inp.Hq, n_kv_heads=inp.Hkv,
                            max_ctx=max_ctx or inp.Lmax, kv_dtype=kv_dtype_code(inp.dtype),
                            P_q=self.P_q, P_k=self.P_k, rope_theta=inp.rope_theta,
                            idx_scale=inp.idx_scale, split_rows=split_rows)
        self.h = B.spa_create(cfg)

    def close(self):
        if self.h:
            B.spa_destroy(self.h)
            self.h = None

    def __enter__(self):
        return self

    def __exit__(self, *a):
        self.close()


class DevInputs:
    """Device copies of one step's inputs; idx_cache comes from the oracle (bf16 bits)."""

    def __init__(self, inp: synth.Inputs, idx_bits: np.ndarray):
        self.q_pre = dev_storage(inp.q_pre, inp.dtype)
        self.k_cache = dev_storage(inp.k_cache, inp.dtype)
        self.v_cache = dev_storage(inp.v_cache, inp.dtype)
        self.idx = dev_storage(idx_bits, "bf16")
        self.seq_lens = torch.from_numpy(inp.seq_lens.astype(np.int64)).cuda()


def gpu_select(h: Handle, inp, dev: DevInputs, p=None, n_sink=None, window=None, max_seq_len=0):
    sel = torch.full((inp.B, inp.Hkv, inp.Lmax), -1, dtype=torch.int32, device="cuda")
    cnt = torch.full((inp.B * inp.Hkv,), -1, dtype=torch.int32, device="cuda")
    B.spa_select(h.h, dev.q_pre, dev.idx, inp.head_mask, dev.seq_lens, inp.B, max_seq_len,
                 inp.p if p is None else p, inp.n_sink if n_sink is None else n_sink,
                 inp.window if window is None else window, sel, cnt)
    torch.cuda.synchronize()
    sel, cnt = sel.cpu().numpy(), cnt.cpu().numpy()
    lists = {}
    for b in range(inp.B):
        for g in range(inp.Hkv):
            lists[(b, g)] = sel[b, g, :cnt[b * inp.Hkv + g]].astype(np.int64)
    return lists, cnt.reshape(inp.B, inp.Hkv)


def gpu_decode(h: Handle, inp, dev: DevInputs, p=None, n_sink=None, window=None, max_seq_len=0):
    out = torch.full((inp.B, inp.Hq, 128), float("nan"), dtype=torch.float32, device="cuda")
    cnt = torch.full((inp.B * inp.Hkv,), -1, dtype=torch.int32, device="cuda")
    B.spa_decode(h.h, dev.q_pre, dev.k_cache, dev.v_cache, dev.idx, inp.head_mask, dev.seq_lens, inp.B,
                 max_seq_len, inp.p if p is None else p, inp.n_sink if n_sink is None else n_sink,
                 inp.window if window is None else window, out, cnt)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64), cnt.cpu().numpy().reshape(inp.B, inp.Hkv)


def check_selection(gpu_list: np.ndarray, sr, p: float, n_sink: int, window: int, band: float = SEL_BAND) -> int:
    """GPU list == oracle list except tokens whose oracle running mass is within band of p.
    Returns the number of tokens that differ (all inside the band)."""
    assert np.all(np.diff(gpu_list) > 0), "list must be strictly ascending"
    want = sr.listed
    diff = np.setxor1d(gpu_list, want)
    if len(diff):
        assert p < 1.0, f"p = 1 must keep everything; {len(diff)} tokens differ"
        off = np.abs(sr.topp.c_before[diff] - p)
        bad = diff[off > band]
        assert len(bad) == 0, (f"{len(bad)} tokens differ outside the {band} band around p={p}: "
                               f"positions {bad[:8]}, |C_before - p| = {off[off > band][:8]}")
    # nothing outside [0, L) or inside sinks/window
    assert len(gpu_list) == 0 or (gpu_list.min() >= 0 and gpu_list.max() < sr.L)
    assert len(np.intersect1d(gpu_list, O.sink_window(sr.L, n_sink, window))) == 0
    return len(diff)


def oracle_idx(inp, heads=None) -> np.ndarray:
    return O.index_cache_for(inp, heads=heads)
