"""Acceptance band for index codes computed with float32 accumulation.

The index code is defined as the exact product P_k[g] . k rounded once to bf16
("Full Attention Strikes Back", Methodology §2: a 16-dim projection of the
pre-RoPE keys; the cache is bf16).  A device that accumulates the 128 products
in float32, in any order, with or without fused multiply-add, reaches a sum
within gamma_128 * sum |P k| of the exact value (u = 2^-24; Higham, Accuracy
and Stability of Numerical Algorithms, eq. 3.5).  Its code equals the defined
code unless that interval holds a bf16 rounding midpoint; there it may be any
code the interval rounds to: the neighbour across the midpoint when the bound is
below one bf16 step, several steps when the products cancel and the exact value
is small next to the bound.

Test infrastructure: numpy only, no GPU.
"""
from __future__ import annotations

import numpy as np

import oracle as O

U32 = 2.0 ** -24


def _ordinal(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> integers in the order of their values (+0 and -0 both 0)."""
    b = np.asarray(bits, np.uint16).astype(np.int64)
    mag = b & 0x7FFF
    return np.where(b & 0x8000, -mag, mag)


def f32_accumulation_bound(k_f64: np.ndarray, P: np.ndarray) -> np.ndarray:
    """gamma_n * sum_d |k_d| |P_rd| for n = 128 float32 roundings, slightly widened."""
    n = k_f64.shape[-1]
    gamma = n * U32 / (1.0 - n * U32)
    return gamma * 1.01 * np.einsum("...d,rd->...r", np.abs(k_f64), np.abs(np.asarray(P, np.float64)))


def check_index_codes(got_bits: np.ndarray, k_f64: np.ndarray, P: np.ndarray) -> int:
    """Every code is the defined one, or - only where the exact value lies within the
    float32 accumulation bound of a bf16 midpoint - another code that interval rounds
    to.  Returns the number of codes that differ from the definition.

    got_bits [..., 16] bf16 bits; k_f64 [..., 128] exact key values; P [16, 128]."""
    exact = np.einsum("...d,rd->...r", np.asarray(k_f64, np.float64), np.asarray(P, np.float64))
    want = O.f64_to_bf16_bits(exact)
    beta = f32_accumulation_bound(k_f64, P)
    lo = _ordinal(O.f64_to_bf16_bits(exact - beta))
    hi = _ordinal(O.f64_to_bf16_bits(exact + beta))
    g, w = _ordinal(got_bits), _ordinal(want)
    near_midpoint = lo != hi
    ok = (g == w) | (near_midpoint & (g >= lo) & (g <= hi))
    assert np.all(ok), (f"{int((~ok).sum())} index codes outside the band; first at "
                        f"{np.argwhere(~ok)[:4].tolist()}")
    return int((g != w).sum())


def f32_sequential_codes(k_f64: np.ndarray, P: np.ndarray) -> np.ndarray:
    """A model of one float32 evaluation order (products rounded to float32, running
    sum in ascending d), used only to show the band admits such codes."""
    k = np.asarray(k_f64, np.float32)
    Pf = np.asarray(P, np.float32)
    acc = np.zeros(k.shape[:-1] + (Pf.shape[0],), np.float32)
    for d in range(k.shape[-1]):
        acc = acc + k[..., d:d + 1] * Pf[:, d]
    return O.f64_to_bf16_bits(acc.astype(np.float64))
