"""Float64 CPU oracle for data-free head labelling by effective rank.

TEST INFRASTRUCTURE ONLY.  Only ``tests/`` and ``bench.py``'s reference legs may
import this module; it shares no code with the CUDA sources.

Source: "Autonomy of Heads" (AoH) summary, Methodology:
  §1 the kernel operator of head h is M_h = W_K^{h T} W_Q^h (d_model x d_model),
     the query-key matching directions of its frozen weights;
  §2 its effective rank is exp(-sum_k s_k log s_k) over the normalised singular
     values s_k = sigma_k / sum_j sigma_j: low = concentrated spectrum (retrieval),
     high = diffuse spectrum (streaming);
  §3 the nonzero singular values of M_h come from the d_head x d_head proxy
     C_h = (W_Q^h W_Q^{h T})(W_K^h W_K^{h T}) (Sylvester's determinant theorem):
     sigma_k^2 are the eigenvalues of C_h.  The oracle takes the singular values of
     M_h by definition (through a QR factorisation, no squaring) and keeps the proxy
     route beside it, pinned to agree where the spectrum is well conditioned;
  §4 heads are ranked by effective rank, the k lowest are retrieval heads, the
     rest streaming; under GQA head scores are aggregated to the group by their
     mean.

Readings taken where the summary is silent:
  * W_Q^h and W_K^g are the d_head x d_model row blocks of the query and key
    projections (q = W_Q^h x); a query head uses the key head of its GQA group;
  * log is the natural logarithm (exp and log of the same base: the effective
    rank does not depend on it); zero singular values contribute 0;
  * the group score is the mean of the G query heads' effective ranks; ties in
    the ranking go to the lower KV head index.
"""
from __future__ import annotations

import numpy as np


def effective_rank(sigma: np.ndarray) -> float:
    """exp of the Shannon entropy of the normalised singular values (AoH §2)."""
    s = np.asarray(sigma, np.float64)
    s = s[s > 0]
    if s.size == 0:
        return 0.0
    p = s / s.sum()
    return float(np.exp(-np.sum(p * np.log(p))))


def proxy_matrix(Wq: np.ndarray, Wk: np.ndarray) -> np.ndarray:
    """C_h = (W_Q W_Q^T)(W_K W_K^T), d_head x d_head (AoH §3)."""
    Wq = np.asarray(Wq, np.float64)
    Wk = np.asarray(Wk, np.float64)
    return (Wq @ Wq.T) @ (Wk @ Wk.T)


def proxy_singular_values(Wq: np.ndarray, Wk: np.ndarray) -> np.ndarray:
    """sqrt of the eigenvalues of C_h, descending: the summary's route (AoH §3).  C_h is
    a product of two positive semi-definite matrices, so its eigenvalues are real and
    >= 0 (rounding residue below 0 is clamped).  Squaring costs accuracy near zero: a
    zero singular value comes back as about sqrt(eps) * sigma_max."""
    lam = np.linalg.eigvals(proxy_matrix(Wq, Wk)).real
    return np.sort(np.sqrt(np.clip(lam, 0.0, None)))[::-1]


def singular_values(Wq: np.ndarray, Wk: np.ndarray) -> np.ndarray:
    """The d_head largest singular values of M_h = W_K^T W_Q, descending (AoH §1), without
    forming M_h or squaring: with the thin QR factorisation W_K^T = Q_K R_K (Q_K has
    orthonormal columns), M_h = Q_K (R_K W_Q) has the singular values of the
    d_head x d_model matrix R_K W_Q.  Library QR and SVD serve as the steps."""
    Wq = np.asarray(Wq, np.float64)
    Wk = np.asarray(Wk, np.float64)
    _, R = np.linalg.qr(Wk.T)
    return np.linalg.svd(R @ Wq, compute_uv=False)


def head_effective_ranks(W_Q: np.ndarray, W_K: np.ndarray) -> np.ndarray:
    """Effective rank of every query head.  W_Q [Hq][d_head][d_model],
    W_K [Hkv][d_head][d_model]; query head h uses key head h // (Hq // Hkv)."""
    Hq, Hkv = W_Q.shape[0], W_K.shape[0]
    G = Hq // Hkv
    return np.array([effective_rank(singular_values(W_Q[h], W_K[h // G])) for h in range(Hq)])


def group_effective_ranks(er_q: np.ndarray, Hkv: int) -> np.ndarray:
    """Mean of the G query heads' effective ranks per KV head (AoH §4, GQA)."""
    return np.asarray(er_q, np.float64).reshape(Hkv, -1).mean(axis=1)


def retrieval_mask(er_kv: np.ndarray, k: int) -> np.ndarray:
    """The k KV heads of lowest effective rank are retrieval heads (1), the rest
    streaming (0); equal scores go to the lower head index."""
    er_kv = np.asarray(er_kv, np.float64)
    order = np.lexsort((np.arange(er_kv.size), er_kv))
    mask = np.zeros(er_kv.size, np.uint8)
    mask[order[:max(0, min(k, er_kv.size))]] = 1
    return mask
