"""Pins of the prefill oracle: causal SDPA for retrieval heads, a masked SDPA for
streaming heads (torch, RoPE written as a complex rotation), and agreement with the
decode oracle at the chunk's last position."""
import math

import numpy as np
import pytest
import torch

import oracle as O
from oracle import prefill_oracle as PF
from head_partitioned_sparse_b200 import synth


def _rot(q, pos, theta):
    w = np.exp(-np.arange(64) / 64.0 * math.log(theta))
    z = (q[..., :64] + 1j * q[..., 64:]) * np.exp(1j * np.asarray(pos)[:, None] * w)
    return np.concatenate([z.real, z.imag], axis=-1)


def _inputs(dtype="f32", L=300, T=40, seed=0):
    inp = synth.make_inputs("tiny", seed, overrides={"L": L, "window": 24, "n_sink": 3, "dtype": dtype})
    q = synth.prefill_queries(inp, seed, T)
    f = (lambda a: O.bf16_bits_to_f64(a)) if dtype == "bf16" else (lambda a: np.asarray(a, np.float64))
    return inp, q, f


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_retrieval_heads_are_causal_sdpa(dtype):
    inp, q, f = _inputs(dtype)
    T, L = q.shape[2], inp.Lmax
    start = np.array([L - T])
    out = PF.prefill(q, inp.k_cache, inp.v_cache, inp.head_mask, start, inp.n_sink, inp.window, inp.rope_theta,
                     to_f64=f)
    pos = L - T + np.arange(T)
    for h in range(inp.G):   # KV head 0 is a retrieval head
        qr = _rot(f(q[0, h]), pos, inp.rope_theta)
        K, V = f(inp.k_cache[0, 0, :L]), f(inp.v_cache[0, 0, :L])
        mask = np.arange(L)[None, :] <= pos[:, None]
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(qr)[None, None], torch.from_numpy(K)[None, None], torch.from_numpy(V)[None, None],
            attn_mask=torch.from_numpy(mask)[None, None])[0, 0].numpy()
        np.testing.assert_allclose(out[0, h], ref, atol=1e-10)


def test_streaming_heads_are_banded_sdpa_with_sinks():
    inp, q, f = _inputs("f32", L=200, T=60)
    start = np.array([200 - 60])
    out = PF.prefill(q, inp.k_cache, inp.v_cache, inp.head_mask, start, inp.n_sink, inp.window, inp.rope_theta,
                     to_f64=f)
    pos = 140 + np.arange(60)
    j = np.arange(200)[None, :]
    mask = ((j < inp.n_sink) | ((j > pos[:, None] - inp.window) & (j <= pos[:, None]))) & (j <= pos[:, None])
    for h in range(inp.G, 2 * inp.G):   # KV head 1 streams
        qr = _rot(f(q[0, h]), pos, inp.rope_theta)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(qr)[None, None], torch.from_numpy(f(inp.k_cache[0, 1]))[None, None],
            torch.from_numpy(f(inp.v_cache[0, 1]))[None, None], attn_mask=torch.from_numpy(mask)[None, None])
        np.testing.assert_allclose(out[0, h], ref[0, 0].numpy(), atol=1e-10)


def test_last_row_of_a_chunk_is_a_decode_step():
    # the chunk's last query at position L - 1 is the decode query of length L
    inp, q, f = _inputs("bf16", L=400, T=16, seed=4)
    T = q.shape[2]
    start = np.array([400 - T])
    out = PF.prefill(q, inp.k_cache, inp.v_cache, inp.head_mask, start, inp.n_sink, inp.window, inp.rope_theta,
                     to_f64=f, rows=[(0, h, T - 1) for h in range(inp.Hq)])
    inp.q_pre = np.ascontiguousarray(q[:, :, T - 1])
    dec, _ = O.decode_inputs(inp, p=1.0)
    np.testing.assert_allclose(out[0, :, T - 1], dec[0], atol=1e-12)


def test_sink_window_covering_everything_makes_streaming_dense():
    inp, q, f = _inputs("f32", L=120, T=30, seed=5)
    start = np.array([90])
    a = PF.prefill(q, inp.k_cache, inp.v_cache, inp.head_mask, start, 0, 10 ** 6, inp.rope_theta, to_f64=f)
    dense_mask = np.ones_like(inp.head_mask)
    b = PF.prefill(q, inp.k_cache, inp.v_cache, dense_mask, start, 0, 10 ** 6, inp.rope_theta, to_f64=f)
    np.testing.assert_allclose(a, b, atol=0)
    keys, w = PF.prefill_weights(q, inp.k_cache, inp.head_mask, start, 3, 8, inp.rope_theta, 0, 5, 29, to_f64=f)
    assert list(keys) == [0, 1, 2] + list(range(119 - 7, 120)) and w.sum() == pytest.approx(1.0, abs=1e-14)
