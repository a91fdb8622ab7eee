"""Seeded synthetic inputs for one decode step of head-partitioned sparse attention.

This module is the only code shared by the CUDA path's tests/bench and the
float64 oracle's tests.  It draws random numbers and lays them out; it holds none
of the method's arithmetic (no RoPE, no projection, no softmax, no selection).

Workload shapes follow the decode setting of "Full Attention Strikes Back"
(RTPurbo summary), Methodology §1-§3: a long KV cache, a few retrieval KV heads
that score every cached token in a 16-dim index space, and streaming heads that
only see sinks plus a recent window.  The pages measure on model datasets
(RULER, LongBench, ...) that are not available; these seeded Gaussian inputs
with planted keys stand in for them.

Conventions
-----------
* Every tensor is drawn from its own NumPy ``PCG64`` stream keyed by
  ``SeedSequence([seed, tensor_id, b, g])``, so a draw never depends on thread
  scheduling or on which other tensors were requested.
* ``N(0, x)`` means variance ``x``.
* bf16 tensors are returned as their raw ``uint16`` bit patterns, rounded
  to nearest-even from the float32 draw; f32 tensors are returned as float32.
* Planted keys live in the pre-RoPE key space (``k_pre``), the space the index
  cache is built from.  Planted key ``i`` of retrieval KV head ``g`` copies the
  (stored) pre-RoPE query of head ``g*G + (i mod G)`` times ``scale`` and adds
  ``N(0, 0.5)`` noise.
* ``k_cache`` (the post-RoPE key cache that attention reads) is drawn directly
  as i.i.d. ``N(0, 1)``: a rotation of an ``N(0, I)`` vector is again
  ``N(0, I)``, so this has the law of rotated Gaussian keys without doing any
  rotation here.
"""
from __future__ import annotations

import concurrent.futures as _fut
import dataclasses
import os
from typing import Dict, List, Optional, Sequence

import numpy as np

HEAD_DIM = 128
IDX_DIM = 16

# tensor ids for SeedSequence keys
_T_P, _T_PQ, _T_Q, _T_KPRE, _T_KCACHE, _T_V, _T_NPLANT, _T_POS, _T_NOISE = range(9)


# Named workloads (sizes as stated in the decode experiments these pages describe;
# the planted-key recipe is the synthetic stand-in for real retrieval traffic).
CONFIGS: Dict[str, dict] = {
    # batch 1, GQA 4, 4K context, float32 storage, KV head 0 retrieval.
    "tiny": dict(B=1, Hq=8, Hkv=2, L=4096, dtype="f32", retrieval=[0],
                 planted="fixed", n_planted=4, scale=3.0,
                 n_sink=4, window=256, p=0.9),
    # one Llama-3-8B attention layer, 32K context.
    "llama3_8b_32k": dict(B=1, Hq=32, Hkv=8, L=32768, dtype="bf16", retrieval=[0, 4],
                          planted="fixed", n_planted=16, scale=3.0,
                          n_sink=4, window=1024, p=0.95),
    # batch-16 decode at 64K, per-sequence planted count from {1, 8, 64, 512}.
    "batch16_64k": dict(B=16, Hq=32, Hkv=8, L=65536, dtype="bf16", retrieval=[0, 4],
                        planted="choice", planted_choices=[1, 8, 64, 512], scale=3.0,
                        n_sink=4, window=2048, p=0.9),
    # batch-4 decode at 128K: sequences 0,1 concentrated, 2,3 broad.
    "ctx128k": dict(B=4, Hq=32, Hkv=8, L=131072, dtype="bf16", retrieval=[0, 2, 4, 6],
                    planted="halves", n_planted_conc=8, scale_conc=4.0,
                    n_planted_broad=4096, scale_broad=1.0,
                    n_sink=4, window=4096, p=0.9, p_sweep=[0.8, 0.9, 0.95, 0.99]),
    # one 1M-token sequence, GQA 8, 32 planted keys evenly spaced.
    "ctx1m": dict(B=1, Hq=64, Hkv=8, L=1048576, dtype="bf16", retrieval=[0, 4],
                  planted="even", n_planted=32, scale=3.0,
                  n_sink=4, window=8192, p=0.95),
}

ROPE_THETA = 500000.0
IDX_SCALE = 0.25  # 1/sqrt(16)


def _rng(seed: int, tensor_id: int, b: int = 0, g: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tensor_id, b, g])))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest-even) and return the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclasses.dataclass
class Inputs:
    """One decode step's inputs.  Storage arrays are uint16 (bf16 bits) or float32."""
    name: str
    dtype: str                 # "bf16" or "f32"
    B: int
    Hq: int
    Hkv: int
    Lmax: int                  # cache capacity (rows per (b, kv head))
    seq_lens: np.ndarray       # int64 [B], context length incl. the current token
    head_mask: np.ndarray      # uint8 [Hkv], 1 = retrieval head
    P_k: np.ndarray            # float32 [Hkv][16][128]
    P_q: np.ndarray            # float32 [Hq][16][128]
    q_pre: np.ndarray          # [B][Hq][128] pre-RoPE query
    k_pre: np.ndarray          # [B][Hkv][Lmax][128] pre-RoPE keys (index side)
    k_cache: np.ndarray        # [B][Hkv][Lmax][128] post-RoPE keys (attention side)
    v_cache: np.ndarray        # [B][Hkv][Lmax][128]
    planted: Dict[tuple, np.ndarray]  # (b, g) -> planted positions
    p: float
    n_sink: int
    window: int
    rope_theta: float = ROPE_THETA
    idx_scale: float = IDX_SCALE

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def storage_to_f32(self, a: np.ndarray) -> np.ndarray:
        return bf16_bits_to_f32(a) if self.dtype == "bf16" else np.asarray(a, dtype=np.float32)


def _store(x32: np.ndarray, dtype: str) -> np.ndarray:
    return f32_to_bf16_bits(x32) if dtype == "bf16" else x32.astype(np.float32, copy=False)


def _planted_plan(cfg: dict, B: int, seq_lens: np.ndarray, n_sink: int, window: int,
                  seed: int, retrieval: Sequence[int]):
    """(b, g) -> (positions, scale).  Positions are distinct, in [n_sink, L_b - window)."""
    plan = {}
    kind = cfg["planted"]
    for b in range(B):
        L = int(seq_lens[b])
        lo, hi = n_sink, L - window
        if kind == "fixed":
            n, scale = cfg["n_planted"], cfg["scale"]
        elif kind == "choice":
            n = int(_rng(seed, _T_NPLANT, b).choice(cfg["planted_choices"]))
            scale = cfg["scale"]
        elif kind == "halves":
            conc = b < B // 2
            n = cfg["n_planted_conc"] if conc else cfg["n_planted_broad"]
            scale = cfg["scale_conc"] if conc else cfg["scale_broad"]
        elif kind == "even":
            n, scale = cfg["n_planted"], cfg["scale"]
        else:
            raise ValueError(kind)
        for g in retrieval:
            if hi <= lo:
                plan[(b, g)] = (np.zeros(0, np.int64), scale)
                continue
            m = min(n, hi - lo)
            if kind == "even":
                pos = np.unique(np.linspace(lo, hi - 1, m).round().astype(np.int64))
            else:
                pos = np.sort(_rng(seed, _T_POS, b, g).choice(hi - lo, size=m, replace=False)).astype(np.int64) + lo
            plan[(b, g)] = (pos, scale)
    return plan


def make_inputs(name: str = "tiny", seed: int = 0, *,
                overrides: Optional[dict] = None,
                seq_lens: Optional[Sequence[int]] = None,
                tied: bool = True,
                draw_streaming_kpre: bool = True,
                poison_tail: bool = False,
                threads: Optional[int] = None) -> Inputs:
    """Draw one decode step's inputs for a named workload.

    overrides          -- replace config fields (e.g. ``{"L": 512, "B": 2}``).
    seq_lens           -- per-sequence context lengths (ragged batches); the cache
                          capacity stays ``L``.
    tied               -- P_q[h] = P_k[g(h)] (one projector per KV group).  With
                          ``False`` the query projectors are independent draws.
    draw_streaming_kpre-- draw pre-RoPE keys for streaming heads too (their index
                          rows are never read by a decode step); zeros otherwise.
    poison_tail        -- fill cache rows at positions >= seq_lens[b] with NaN so
                          any read past the context shows up in the output.
    """
    cfg = dict(CONFIGS[name])
    if overrides:
        cfg.update(overrides)
    B, Hq, Hkv, L, dtype = cfg["B"], cfg["Hq"], cfg["Hkv"], cfg["L"], cfg["dtype"]
    G = Hq // Hkv
    retrieval = [g for g in cfg["retrieval"] if g < Hkv]
    n_sink, window = cfg["n_sink"], cfg["window"]
    lens = np.full(B, L, np.int64) if seq_lens is None else np.asarray(seq_lens, np.int64)
    assert lens.shape == (B,) and lens.min() >= 1 and lens.max() <= L
    head_mask = np.zeros(Hkv, np.uint8)
    head_mask[retrieval] = 1

    std_p = np.float32(1.0 / np.sqrt(HEAD_DIM))
    P_k = np.stack([_rng(seed, _T_P, 0, g).standard_normal((IDX_DIM, HEAD_DIM), dtype=np.float32) * std_p
                    for g in range(Hkv)])
    if tied:
        P_q = np.repeat(P_k, G, axis=0).copy()
    else:
        P_q = np.stack([_rng(seed, _T_PQ, 0, h).standard_normal((IDX_DIM, HEAD_DIM), dtype=np.float32) * std_p
                        for h in range(Hq)])

    q32 = np.stack([_rng(seed, _T_Q, b).standard_normal((Hq, HEAD_DIM), dtype=np.float32) for b in range(B)])
    q_pre = _store(q32, dtype)
    q_stored = bf16_bits_to_f32(q_pre) if dtype == "bf16" else q_pre

    st_dtype = np.uint16 if dtype == "bf16" else np.float32
    shape = (B, Hkv, L, HEAD_DIM)
    k_pre = np.empty(shape, st_dtype)
    k_cache = np.empty(shape, st_dtype)
    v_cache = np.empty(shape, st_dtype)
    plan = _planted_plan(cfg, B, lens, n_sink, window, seed, retrieval)
    noise_std = np.float32(np.sqrt(0.5))

    def fill(b: int, g: int) -> None:
        for tid, dst in ((_T_KCACHE, k_cache), (_T_V, v_cache)):
            dst[b, g] = _store(_rng(seed, tid, b, g).standard_normal((L, HEAD_DIM), dtype=np.float32), dtype)
        if g in retrieval or draw_streaming_kpre:
            kp = _rng(seed, _T_KPRE, b, g).standard_normal((L, HEAD_DIM), dtype=np.float32)
            if (b, g) in plan:
                pos, scale = plan[(b, g)]
                if len(pos):
                    src = q_stored[b, g * G + (np.arange(len(pos)) % G)]
                    noise = _rng(seed, _T_NOISE, b, g).standard_normal((len(pos), HEAD_DIM), dtype=np.float32)
                    kp[pos] = np.float32(scale) * src + noise_std * noise
            k_pre[b, g] = _store(kp, dtype)
        else:
            k_pre[b, g] = 0
        if poison_tail and lens[b] < L:
            nan = np.uint16(0x7FC0) if dtype == "bf16" else np.float32(np.nan)
            for arr in (k_pre, k_cache, v_cache):
                arr[b, g, lens[b]:] = nan

    jobs = [(b, g) for b in range(B) for g in range(Hkv)]
    nthreads = threads or min(len(jobs), max(1, len(os.sched_getaffinity(0))))
    if nthreads > 1 and len(jobs) > 1:
        with _fut.ThreadPoolExecutor(nthreads) as ex:
            list(ex.map(lambda bg: fill(*bg), jobs))
    else:
        for bg in jobs:
            fill(*bg)

    return Inputs(name=name, dtype=dtype, B=B, Hq=Hq, Hkv=Hkv, Lmax=L, seq_lens=lens,
                  head_mask=head_mask, P_k=P_k, P_q=P_q, q_pre=q_pre, k_pre=k_pre,
                  k_cache=k_cache, v_cache=v_cache,
                  planted={k: v[0] for k, v in plan.items()},
                  p=float(np.float32(cfg["p"])), n_sink=n_sink, window=window)


_T_WQ, _T_WK, _T_WBASIS = 100, 101, 102
_T_QCHUNK = 103


def prefill_queries(inp: "Inputs", seed: int, T: int) -> np.ndarray:
    """Seeded pre-RoPE queries of a prefill chunk: [B][Hq][T][128] N(0, 1) entries, in the
    bundle's storage dtype (bf16 bits or float32), one stream per (sequence, head)."""
    q = np.empty((inp.B, inp.Hq, T, HEAD_DIM), np.float32)
    for b in range(inp.B):
        for h in range(inp.Hq):
            q[b, h] = _rng(seed, _T_QCHUNK, b, h).standard_normal((T, HEAD_DIM), dtype=np.float32)
    return _store(q, inp.dtype)


def make_head_weights(seed: int = 0, Hq: int = 32, Hkv: int = 8, d_model: int = 4096,
                      retrieval=(0, 4), rank: int = 8, noise: float = 0.05):
    """Seeded synthetic query/key projections for head labelling by effective rank.

    Returns (W_Q [Hq][128][d_model], W_K [Hkv][128][d_model]) as float32.  Streaming-like
    KV heads (and their query heads) get i.i.d. N(0, 1/d_model) entries: a diffuse
    query-key spectrum.  For a retrieval-like KV head g listed in ``retrieval``, the key
    head and its G query heads share one rank-``rank`` row space drawn for the group:
    W = sqrt(d_model / 128) C_W B_g + noise * N(0, 1/d_model), with B_g [rank][d_model]
    of N(0, 1/d_model) entries and a per-matrix C_W [128][rank] of N(0, 1/rank)
    entries, so a few query-key directions dominate (a concentrated spectrum).
    """
    G = Hq // Hkv
    WQ = np.empty((Hq, HEAD_DIM, d_model), np.float32)
    WK = np.empty((Hkv, HEAD_DIM, d_model), np.float32)
    sd = np.float32(1.0 / np.sqrt(d_model))
    for g in range(Hkv):
        concentrated = g in retrieval
        if concentrated:
            basis = _rng(seed, _T_WBASIS, 0, g).standard_normal((rank, d_model), dtype=np.float32) * sd
        for m in range(G + 1):   # m < G: query head g G + m; m = G: the key head
            tid = _T_WQ if m < G else _T_WK
            r = _rng(seed, tid, m, g)
            w = r.standard_normal((HEAD_DIM, d_model), dtype=np.float32) * sd
            if concentrated:
                coef = r.standard_normal((HEAD_DIM, rank), dtype=np.float32) / np.float32(np.sqrt(rank))
                w = coef @ basis * np.float32(np.sqrt(d_model / HEAD_DIM)) + np.float32(noise) * w
            if m < G:
                WQ[g * G + m] = w
            else:
                WK[g] = w
    return WQ, WK


def list_configs() -> List[str]:
    return list(CONFIGS)
