"""Float64 CPU oracle for a prefill chunk of head-partitioned attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/`` and ``bench.py``'s reference legs may
import this module; it shares no code with the CUDA sources.

Sources (page title, section):
  "Full Attention Strikes Back" (RTPurbo summary), Methodology §1: retrieval heads
  keep the full context (dense attention in prefill; the sparse selection is a
  decode-time step); local heads attend a sliding window with attention sinks.
  "Autonomy of Heads" summary, Deployment strategy: streaming heads keep a sink
  cache and a recent window from the first token on, prefill included.

Readings taken where the pages are silent:
  * a chunk holds the T queries at absolute positions start[b] .. start[b] + T - 1;
    the caches already hold every position up to the chunk's last (keys post-RoPE);
  * a query at position t attends causally: a retrieval head keys [0, t]; a
    streaming head the sinks [0, n_sink) and the window [t - window + 1, t], the
    set a decode step at length t + 1 attends;
  * the query is rotated to its own position t (the decode step's RoPE), the score
    scale is 1/sqrt(128), and the output is float64.
"""
from __future__ import annotations

import numpy as np

from .spa_oracle import attend, rope, sink_window


def prefill_keys(t: int, retrieval: bool, n_sink: int, window: int) -> np.ndarray:
    """Positions the query at absolute position t attends, ascending."""
    if retrieval:
        return np.arange(t + 1, dtype=np.int64)
    return sink_window(t + 1, n_sink, window)


def prefill(q_chunk, k_cache, v_cache, head_mask, start, n_sink, window, rope_theta, *, to_f64=None,
            rows=None):
    """Attention outputs of a prefill chunk.

    q_chunk [B][Hq][T][128] and the caches [B][Hkv][Lmax][128] hold storage values;
    ``to_f64`` maps storage to exact float64 (identity by default).  ``rows`` (optional)
    limits the work to a list of (b, h, i) query rows.  Returns out [B][Hq][T][128]
    float64, NaN where not computed.
    """
    if to_f64 is None:
        to_f64 = lambda a: np.asarray(a, np.float64)
    B, Hq, T = q_chunk.shape[:3]
    Hkv = k_cache.shape[1]
    G = Hq // Hkv
    out = np.full((B, Hq, T, q_chunk.shape[3]), np.nan)
    if rows is None:
        rows = [(b, h, i) for b in range(B) for h in range(Hq) for i in range(T)]
    for (b, h, i) in rows:
        t = int(start[b]) + i
        g = h // G
        keys = prefill_keys(t, bool(head_mask[g]), n_sink, window)
        q = rope(to_f64(q_chunk[b, h, i]), t, rope_theta)
        out[b, h, i] = attend(q[None], to_f64(k_cache[b, g, keys]), to_f64(v_cache[b, g, keys]))[0]
    return out


def prefill_weights(q_chunk, k_cache, head_mask, start, n_sink, window, rope_theta, b, h, i, *, to_f64=None):
    """(attended positions, softmax weights) of one query row (for error bounds)."""
    if to_f64 is None:
        to_f64 = lambda a: np.asarray(a, np.float64)
    Hq, Hkv = q_chunk.shape[1], k_cache.shape[1]
    g = h // (Hq // Hkv)
    t = int(start[b]) + i
    keys = prefill_keys(t, bool(head_mask[g]), n_sink, window)
    q = rope(to_f64(q_chunk[b, h, i]), t, rope_theta)
    s = to_f64(k_cache[b, g, keys]) @ q / np.sqrt(np.float64(q.shape[0]))
    w = np.exp(s - s.max())
    return keys, w / w.sum()
