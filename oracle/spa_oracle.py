"""Float64 CPU oracle for one decode step of head-partitioned sparse attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The product path (the
CUDA library and its Python binding) never calls it, and it shares no code,
header, table or constant generator with the CUDA sources.

It is written to be read against the pages, step by step, in float64, with no
blocking, fusion or reordering beyond what the method states.  Library
primitives (a matrix product, a stable sort, a running sum) serve as steps.

Sources (page title, section):
  [FASB] "Full Attention Strikes Back" (RTPurbo summary), Methodology
         §1 head specialisation: local heads use a sliding window with attention
            sinks; retrieval heads keep the full cache and switch to dynamic sparse
            selection during decoding;
         §2 low-dimensional token indexing: a 16-dim projector applied to query and
            key features before RoPE is injected; relevance is estimated there;
         §3 dynamic top-p: attention mass in the low-dim space is accumulated until
            the cumulative threshold p is reached (contrasted there with a fixed
            top-k budget, built here as the selector variant ``top_k``);
         §5 hardware-aware kernels (histogram thresholding, sparse decode).
  [HGA]  "Hierarchical Global Attention" summary, Central mechanism §4: exact
         token attention, plain softmax over the bounded selected set.
  [AoH]  "Autonomy of Heads" summary, Deployment strategy: GQA head scores are
         aggregated to the group by their mean; streaming heads keep a sink cache
         and a recent window.

Readings taken where the pages are silent:
  * index softmax temperature = idx_scale (1/sqrt(16) by default);
  * per query head probabilities, averaged over the GQA group (the group mean
    of [AoH]); one selected set per (sequence, KV head);
  * tokens are ordered by (probability desc, position asc); token j is kept
    iff the running mass *before* it is < p ("until p is reached"), so the
    kept set is the shortest prefix whose mass is >= p; p >= 1 keeps all;
  * the top-k variant keeps the first k tokens of that same order (all L when
    k >= L), over all L tokens like top-p, sinks and window attended anyway;
  * the block-granular variant scores blocks of 64 consecutive positions by
    their mass (the sum of their tokens' probabilities), orders blocks by (mass
    desc, block index asc), keeps a block iff the running mass before it is < p,
    and keeps every token of a kept block ([HGA] routes chunks, not tokens);
  * sinks = positions [0, n_sink), window = the last ``window`` positions
    (the current token included); both are always attended, the union
    de-duplicated;
  * RoPE: rotate-half pairing (i, i + d/2), inv_freq_i = theta^(-2i/d), angle
    = position * inv_freq_i, query at position L-1, no frequency rescaling;
  * index cache rows are bf16: the exact product rounded once to nearest-even.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Tuple

import numpy as np

HEAD_DIM = 128
IDX_DIM = 16


# --------------------------------------------------------------------------
# bf16 storage <-> float64
# --------------------------------------------------------------------------
def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns (a bf16 is the top half of an fp32)."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16, ties to even; return bit patterns.

    bf16 keeps 8 significant bits.  For |x| in [2^e, 2^(e+1)) the spacing is
    2^(e-7); below the smallest normal (2^-126) the spacing stays 2^-133.
    Rounding is done once, from the float64 value (no detour through fp32).
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.float64)
    finite = np.isfinite(x)
    ax = np.abs(np.where(finite, x, 0.0))
    _, e = np.frexp(ax)                       # ax = m * 2^e, m in [0.5, 1)
    e = e.astype(np.int64) - 1                # ax in [2^e, 2^(e+1))
    e = np.maximum(e, -126)
    spacing = np.ldexp(1.0, (e - 7).astype(np.int32))
    q = np.rint(ax / spacing)                 # exact scaling; rint = ties-to-even
    mag = q * spacing
    mag = np.where(mag >= 2.0 ** 128, np.inf, mag)  # beyond bf16 max -> inf
    out = np.where(finite, np.copysign(mag, x), x)
    f32 = out.astype(np.float32)              # exact: every bf16 value is an fp32 value
    return (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


# --------------------------------------------------------------------------
# RoPE  ([FASB] §2: the index is built before RoPE; attention keys are post-RoPE)
# --------------------------------------------------------------------------
def rope_inv_freq(head_dim: int, theta: float) -> np.ndarray:
    i = np.arange(head_dim // 2, dtype=np.float64)
    return np.power(np.float64(theta), -2.0 * i / head_dim)


def rope(x: np.ndarray, pos, theta: float) -> np.ndarray:
    """Rotate-half RoPE of x[..., d] at integer position(s) ``pos`` (float64)."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    h = d // 2
    ang = np.asarray(pos, dtype=np.float64)[..., None] * rope_inv_freq(d, theta)
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :h], x[..., h:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


# --------------------------------------------------------------------------
# Index cache  ([FASB] §2)
# --------------------------------------------------------------------------
def index_rows(k_pre_rows: np.ndarray, P_k_g: np.ndarray) -> np.ndarray:
    """bf16 bits of P_k[g] . k for each pre-RoPE key row; [n, 128] -> [n, 16].

    The definition: the exact (float64) product of the projector and the key,
    rounded once to the nearest bf16, ties to even.
    """
    return f64_to_bf16_bits(np.asarray(k_pre_rows, np.float64) @ np.asarray(P_k_g, np.float64).T)


def index_append(k_pre: np.ndarray, P_k: np.ndarray) -> np.ndarray:
    """[B][Hkv][T][128] pre-RoPE keys (float64 values) -> [B][Hkv][T][16] bf16 bits."""
    B, Hkv = k_pre.shape[:2]
    out = np.empty(k_pre.shape[:3] + (IDX_DIM,), np.uint16)
    for b in range(B):
        for g in range(Hkv):
            out[b, g] = index_rows(k_pre[b, g], P_k[g])
    return out


# --------------------------------------------------------------------------
# Index probabilities and dynamic top-p  ([FASB] §2, §3; [AoH] GQA mean)
# --------------------------------------------------------------------------
def softmax(z: np.ndarray, axis: int = -1) -> np.ndarray:
    z = np.asarray(z, np.float64)
    z = z - z.max(axis=axis, keepdims=True)
    w = np.exp(z)
    return w / w.sum(axis=axis, keepdims=True)


def index_probs(q_pre_group: np.ndarray, P_q_group: np.ndarray, idx_rows_f64: np.ndarray,
                idx_scale: float) -> Tuple[np.ndarray, np.ndarray]:
    """Group index distribution over the cached tokens.

    q_pre_group [G][128]: pre-RoPE queries of the group's heads.
    P_q_group   [G][16][128]: their query projectors.
    idx_rows_f64 [L][16]: the cached index rows (values of the bf16 cache).
    Returns (pi [L], a [G][L]) with a[h] = softmax_j(idx_scale * <P_q[h] q_h, idx_j>)
    and pi = mean_h a[h].
    """
    q_idx = np.einsum("grd,gd->gr", np.asarray(P_q_group, np.float64), np.asarray(q_pre_group, np.float64))
    scores = q_idx @ np.asarray(idx_rows_f64, np.float64).T          # [G][L]
    a = softmax(np.float64(idx_scale) * scores, axis=-1)
    return a.mean(axis=0), a


@dataclasses.dataclass
class TopP:
    kept: np.ndarray        # positions in the top-p set, ascending
    order: np.ndarray       # all positions in (pi desc, pos asc) order
    c_before: np.ndarray    # [L] running mass before each position (position-indexed)


def top_p(pi: np.ndarray, p: float) -> TopP:
    """Shortest prefix of (pi desc, position asc) whose mass reaches p.

    Token j is kept iff the float64 running sum of the tokens ahead of it is < p.
    If p >= 1 every token is kept.
    """
    pi = np.asarray(pi, np.float64)
    L = pi.shape[0]
    pos = np.arange(L)
    order = np.lexsort((pos, -pi))            # primary: -pi ascending; secondary: position
    run = np.cumsum(pi[order])                # sequential running sum in that order
    before_sorted = np.concatenate([[0.0], run[:-1]])
    c_before = np.empty(L, np.float64)
    c_before[order] = before_sorted
    if p >= 1.0:
        kept = pos.copy()
    else:
        kept = np.sort(order[before_sorted < p])
    return TopP(kept=kept, order=order, c_before=c_before)


def top_k(pi: np.ndarray, k: int) -> TopP:
    """The first k tokens of the (pi desc, position asc) order (all L when k >= L).

    A fixed budget in place of the mass threshold of ``top_p``; ``c_before`` is
    still the running mass before each position in that order.
    """
    pi = np.asarray(pi, np.float64)
    L = pi.shape[0]
    pos = np.arange(L)
    order = np.lexsort((pos, -pi))
    run = np.cumsum(pi[order])
    before_sorted = np.concatenate([[0.0], run[:-1]])
    c_before = np.empty(L, np.float64)
    c_before[order] = before_sorted
    kept = pos.copy() if k >= L else np.sort(order[:max(int(k), 0)])
    return TopP(kept=kept, order=order, c_before=c_before)


BLOCK = 64


def block_top_p(pi: np.ndarray, p: float, block: int = BLOCK) -> TopP:
    """Top-p over blocks of ``block`` consecutive positions, whole blocks kept.

    Block b covers positions [b block, min((b + 1) block, L)); its mass is the sum
    of its tokens' probabilities.  Blocks are ordered by (mass desc, block index
    asc) and a block is kept iff the running mass before it is < p (p >= 1 keeps
    all).  ``c_before`` gives, for every position, the running mass before its
    block; ``order`` lists the blocks in that order.
    """
    pi = np.asarray(pi, np.float64)
    L = pi.shape[0]
    nb = (L + block - 1) // block
    bmass = np.array([pi[b * block:(b + 1) * block].sum() for b in range(nb)])
    bidx = np.arange(nb)
    order = np.lexsort((bidx, -bmass))
    run = np.cumsum(bmass[order])
    before_sorted = np.concatenate([[0.0], run[:-1]])
    b_before = np.empty(nb, np.float64)
    b_before[order] = before_sorted
    kept_blocks = bidx if p >= 1.0 else np.sort(order[before_sorted < p])
    kept = np.concatenate([np.arange(b * block, min((b + 1) * block, L)) for b in kept_blocks]) \
        if len(kept_blocks) else np.zeros(0, np.int64)
    c_before = np.repeat(b_before, block)[:L]
    return TopP(kept=kept.astype(np.int64), order=order, c_before=c_before)


def sink_window(L: int, n_sink: int, window: int) -> np.ndarray:
    """Positions always attended: [0, n_sink) union [L - window, L), clipped to [0, L)."""
    s = set(range(min(max(n_sink, 0), L)))
    s.update(range(max(0, L - max(window, 0)), L))
    return np.array(sorted(s), dtype=np.int64)


# --------------------------------------------------------------------------
# Exact attention over a token set  ([HGA] §4, [FASB] §1)
# --------------------------------------------------------------------------
def attend(q_rot: np.ndarray, K: np.ndarray, V: np.ndarray) -> np.ndarray:
    """softmax(q . k / sqrt(d)) . v for each query row; q_rot [G][d], K,V [n][d]."""
    q_rot = np.asarray(q_rot, np.float64)
    d = q_rot.shape[-1]
    s = (q_rot @ np.asarray(K, np.float64).T) / np.sqrt(np.float64(d))
    return softmax(s, axis=-1) @ np.asarray(V, np.float64)


# --------------------------------------------------------------------------
# One decode step
# --------------------------------------------------------------------------
@dataclasses.dataclass
class SliceResult:
    b: int
    g: int
    retrieval: bool
    L: int
    attended: np.ndarray              # all attended positions, ascending
    listed: np.ndarray                # top-p positions outside sinks/window (retrieval), ascending
    topp: Optional[TopP] = None
    pi: Optional[np.ndarray] = None


def decode(q_pre, k_cache, v_cache, idx_cache, head_mask, seq_lens, p, n_sink, window,
           P_q, rope_theta, idx_scale, *, to_f64=None, slices=None,
           attend_sets: Optional[Dict[Tuple[int, int], np.ndarray]] = None, k: Optional[int] = None,
           blocks: bool = False):
    """One decode step for every (b, kv head) in ``slices`` (default: all).

    Retrieval heads select by top-p (``p``), by top-k when ``k`` is given, or by
    block-granular top-p when ``blocks`` is set.

    Array arguments hold storage values; ``to_f64`` maps a storage array to its
    exact float64 values (bf16 bits -> values, or identity for float32).
    idx_cache always holds bf16 bits.  ``attend_sets`` (optional) replaces the
    selected top-p list of a retrieval slice, to evaluate attention on a set
    chosen elsewhere.
    Returns (out [B][Hq][128] float64, NaN for heads not computed; {(b,g): SliceResult}).
    """
    if to_f64 is None:
        to_f64 = lambda a: np.asarray(a, np.float64)
    B, Hq = q_pre.shape[:2]
    Hkv = k_cache.shape[1]
    G = Hq // Hkv
    out = np.full((B, Hq, HEAD_DIM), np.nan)
    res: Dict[Tuple[int, int], SliceResult] = {}
    todo = slices if slices is not None else [(b, g) for b in range(B) for g in range(Hkv)]
    for (b, g) in todo:
        L = int(seq_lens[b])
        t = L - 1
        heads = list(range(g * G, (g + 1) * G))
        qp = to_f64(q_pre[b, heads])                                  # [G][128]
        base = sink_window(L, n_sink, window)
        retrieval = bool(head_mask[g])
        sr = SliceResult(b=b, g=g, retrieval=retrieval, L=L, attended=base,
                         listed=np.zeros(0, np.int64))
        if retrieval:
            idx = bf16_bits_to_f64(idx_cache[b, g, :L])
            pi, _ = index_probs(qp, np.asarray(P_q, np.float64)[heads], idx, idx_scale)
            tp = block_top_p(pi, p) if blocks else (top_p(pi, p) if k is None else top_k(pi, k))
            sr.topp, sr.pi = tp, pi
            listed = np.setdiff1d(tp.kept, base)
            if attend_sets is not None and (b, g) in attend_sets:
                listed = np.asarray(attend_sets[(b, g)], np.int64)
            sr.listed = listed
            sr.attended = np.union1d(base, listed)
        q_rot = rope(qp, t, rope_theta)
        K = to_f64(k_cache[b, g, sr.attended])
        V = to_f64(v_cache[b, g, sr.attended])
        out[b, heads] = attend(q_rot, K, V)
        res[(b, g)] = sr
    return out, res


def decode_inputs(inp, *, slices=None, attend_sets=None, p=None, n_sink=None, window=None,
                  idx_cache=None, k=None, blocks=False):
    """``decode`` on a ``synth.Inputs`` bundle (index cache built by ``index_append``)."""
    to_f64 = (lambda a: bf16_bits_to_f64(a)) if inp.dtype == "bf16" else (lambda a: np.asarray(a, np.float64))
    if idx_cache is None:
        idx_cache = index_cache_for(inp)
    return decode(inp.q_pre, inp.k_cache, inp.v_cache, idx_cache, inp.head_mask, inp.seq_lens,
                  inp.p if p is None else p,
                  inp.n_sink if n_sink is None else n_sink,
                  inp.window if window is None else window,
                  inp.P_q, inp.rope_theta, inp.idx_scale, to_f64=to_f64, slices=slices,
                  attend_sets=attend_sets, k=k, blocks=blocks)


def index_cache_for(inp, heads: Optional[List[int]] = None) -> np.ndarray:
    """bf16 index cache of a ``synth.Inputs`` bundle; rows of other heads stay 0."""
    to_f64 = (lambda a: bf16_bits_to_f64(a)) if inp.dtype == "bf16" else (lambda a: np.asarray(a, np.float64))
    out = np.zeros(inp.k_pre.shape[:3] + (IDX_DIM,), np.uint16)
    hs = range(inp.Hkv) if heads is None else heads
    for b in range(inp.B):
        for g in hs:
            out[b, g] = index_rows(to_f64(inp.k_pre[b, g]), inp.P_k[g])
    return out
