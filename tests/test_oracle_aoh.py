"""Pins of the effective-rank head labelling oracle ("Autonomy of Heads" summary,
Methodology §1-§4) against closed forms, hand-worked values and a brute-force SVD."""
import os

import numpy as np
import pytest

from oracle import aoh_oracle as A
from head_partitioned_sparse_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "aoh_effective_rank_cases.txt")


def _cases():
    for line in open(GOLDEN):
        line = line.split("#")[0].strip()
        if line:
            sv, er = line.split("|")
            yield np.array([float(x) for x in sv.split()]), float(er)


def test_effective_rank_golden_values():
    n = 0
    for sv, er in _cases():
        assert A.effective_rank(sv) == pytest.approx(er, rel=1e-14, abs=0)
        n += 1
    assert n >= 6


def test_hand_worked_weights():
    # W_Q = [[1,0,0],[0,2,0]], W_K = [[1,0,0],[0,1,0]]: M = W_K^T W_Q = diag(1, 2, 0)
    Wq = np.array([[1.0, 0, 0], [0, 2.0, 0]])
    Wk = np.array([[1.0, 0, 0], [0, 1.0, 0]])
    assert np.allclose(A.singular_values(Wq, Wk), [2.0, 1.0], rtol=0, atol=1e-14)
    assert A.effective_rank(A.singular_values(Wq, Wk)) == pytest.approx(1.8898815748423097, rel=1e-14)


@pytest.mark.parametrize("d_head,d_model", [(8, 20), (16, 16), (5, 40)])
def test_proxy_spectrum_equals_svd_of_the_kernel_operator(d_head, d_model):
    # the oracle's singular values and the summary's proxy route (Sylvester: the nonzero
    # singular values of M = W_K^T W_Q are the square roots of the eigenvalues of
    # C = (W_Q W_Q^T)(W_K W_K^T)) against a brute-force SVD of the d_model x d_model M
    rng = np.random.default_rng(d_head * 100 + d_model)
    for _ in range(5):
        Wq = rng.standard_normal((d_head, d_model))
        Wk = rng.standard_normal((d_head, d_model)) * rng.uniform(0.1, 3.0, (d_head, 1))
        direct = np.linalg.svd(Wk.T @ Wq, compute_uv=False)[:d_head]
        np.testing.assert_allclose(A.singular_values(Wq, Wk), direct, rtol=1e-10, atol=1e-12 * direct[0])
        np.testing.assert_allclose(A.proxy_singular_values(Wq, Wk), direct, rtol=1e-7, atol=1e-7 * direct[0])
        assert A.effective_rank(A.singular_values(Wq, Wk)) == pytest.approx(A.effective_rank(direct), rel=1e-12)
        assert A.effective_rank(A.proxy_singular_values(Wq, Wk)) == pytest.approx(A.effective_rank(direct), rel=1e-8)


def test_closed_forms():
    rng = np.random.default_rng(3)
    Q, _ = np.linalg.qr(rng.standard_normal((64, 64)))
    # orthonormal rows (scaled): C = c^4 I, every singular value equal, ER = d_head
    Wq, Wk = 3.0 * Q[:16], 0.5 * Q[:16]
    assert A.effective_rank(A.singular_values(Wq, Wk)) == pytest.approx(16.0, rel=1e-12)
    # rank one: ER = 1
    u, v = rng.standard_normal((16, 1)), rng.standard_normal((1, 64))
    assert A.effective_rank(A.singular_values(u @ v, Q[:16])) == pytest.approx(1.0, rel=1e-9)
    # rank r with equal singular values: ER = r
    r = 5
    Wq = np.zeros((16, 64))
    Wq[:r] = Q[:r]
    assert A.effective_rank(A.singular_values(Wq, Q[:16])) == pytest.approx(float(r), rel=1e-9)


def test_invariances():
    rng = np.random.default_rng(4)
    Wq, Wk = rng.standard_normal((12, 48)), rng.standard_normal((12, 48))
    er = A.effective_rank(A.singular_values(Wq, Wk))
    R, _ = np.linalg.qr(rng.standard_normal((48, 48)))      # rotation of the model space
    U, _ = np.linalg.qr(rng.standard_normal((12, 12)))      # the same rotation of q and k
    assert A.effective_rank(A.singular_values(Wq @ R, Wk @ R)) == pytest.approx(er, rel=1e-10)
    assert A.effective_rank(A.singular_values(U @ Wq, U @ Wk)) == pytest.approx(er, rel=1e-10)
    assert A.effective_rank(A.singular_values(7.0 * Wq, 0.2 * Wk)) == pytest.approx(er, rel=1e-10)
    # swapping the roles of W_Q and W_K transposes M: same singular values
    assert A.effective_rank(A.singular_values(Wk, Wq)) == pytest.approx(er, rel=1e-10)


def test_group_mean_and_mask():
    er_q = np.array([1.0, 3.0, 10.0, 12.0, 2.0, 2.0, 7.0, 9.0])
    er_kv = A.group_effective_ranks(er_q, 4)
    assert np.array_equal(er_kv, [2.0, 11.0, 2.0, 8.0])
    assert np.array_equal(A.retrieval_mask(er_kv, 1), [1, 0, 0, 0])        # tie -> lower index
    assert np.array_equal(A.retrieval_mask(er_kv, 2), [1, 0, 1, 0])
    assert np.array_equal(A.retrieval_mask(er_kv, 3), [1, 0, 1, 1])
    assert np.array_equal(A.retrieval_mask(er_kv, 0), [0, 0, 0, 0])
    assert np.array_equal(A.retrieval_mask(er_kv, 9), [1, 1, 1, 1])


def test_synthetic_weights_label_the_planted_heads():
    WQ, WK = synth.make_head_weights(0, Hq=8, Hkv=4, d_model=512, retrieval=(1, 2))
    er_kv = A.group_effective_ranks(A.head_effective_ranks(WQ, WK), 4)
    assert np.array_equal(A.retrieval_mask(er_kv, 2), [0, 1, 1, 0])
    assert er_kv[[1, 2]].max() < 0.5 * er_kv[[0, 3]].min()
