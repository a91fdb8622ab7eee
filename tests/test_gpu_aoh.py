"""Effective-rank head labels on the GPU vs the float64 oracle ("Autonomy of Heads"
summary, Methodology §1-§4).

Tolerances follow from the route the library takes (eigenvalues of the squared
operator in float64): full-rank heads agree to ~1e-9 relative (ER_RTOL), and a zero
singular value returns as about sqrt(128 eps) sigma_max, which bounds the ER error of a
rank-deficient head by 128 * 1.7e-7 * |ln 1.7e-7| ~ 4e-4 relative (ER_RTOL_DEFICIENT).
"""
import time

import numpy as np
import pytest
import torch

from oracle import aoh_oracle as A
from head_partitioned_sparse_b200 import binding as B
from head_partitioned_sparse_b200 import synth

pytestmark = pytest.mark.gpu

ER_RTOL = 1e-8
ER_RTOL_DEFICIENT = 5e-4


def gpu_ranks(WQ, WK, n_ret):
    Hq, Hkv, d_model = WQ.shape[0], WK.shape[0], WQ.shape[2]
    wq = torch.from_numpy(np.ascontiguousarray(WQ, np.float32)).cuda()
    wk = torch.from_numpy(np.ascontiguousarray(WK, np.float32)).cuda()
    nbytes = B.spa_head_ranks_workspace_size(Hq, Hkv)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    er_q = torch.full((Hq,), float("nan"), dtype=torch.float64, device="cuda")
    er_kv = torch.full((Hkv,), float("nan"), dtype=torch.float64, device="cuda")
    mask = torch.full((Hkv,), 7, dtype=torch.uint8, device="cuda")
    sig = torch.full((Hq, 128), float("nan"), dtype=torch.float64, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    B.spa_head_effective_ranks(wq, wk, Hq, Hkv, d_model, n_ret, ws, nbytes, er_q, er_kv, mask, sig)
    torch.cuda.synchronize()
    ms = (time.perf_counter() - t0) * 1e3
    return er_q.cpu().numpy(), er_kv.cpu().numpy(), mask.cpu().numpy(), sig.cpu().numpy(), ms


@pytest.mark.parametrize("Hq,Hkv,d_model,ret", [(8, 4, 512, (1, 2)), (32, 8, 4096, (0, 4)), (16, 16, 300, (3,)),
                                                (64, 8, 1024, (5, 6, 7))])
def test_effective_ranks_match_the_oracle(Hq, Hkv, d_model, ret):
    WQ, WK = synth.make_head_weights(11, Hq=Hq, Hkv=Hkv, d_model=d_model, retrieval=ret)
    er_q, er_kv, mask, sig, ms = gpu_ranks(WQ, WK, len(ret))
    want_q = A.head_effective_ranks(WQ, WK)
    np.testing.assert_allclose(er_q, want_q, rtol=ER_RTOL, atol=0)
    want_kv = A.group_effective_ranks(want_q, Hkv)
    np.testing.assert_allclose(er_kv, want_kv, rtol=ER_RTOL, atol=0)
    assert np.array_equal(mask, A.retrieval_mask(want_kv, len(ret)))
    assert np.array_equal(np.flatnonzero(mask), sorted(ret))
    G = Hq // Hkv
    for h in range(Hq):
        s = A.singular_values(WQ[h], WK[h // G])
        np.testing.assert_allclose(sig[h], s, rtol=0, atol=1e-7 * s[0])
        assert np.all(np.diff(sig[h]) <= 0)
    print(f"head ranks {Hq}/{Hkv} heads, d_model {d_model}: {ms:.2f} ms")


def test_closed_form_and_rank_deficient_heads():
    rng = np.random.default_rng(5)
    d_model = 256
    Q, _ = np.linalg.qr(rng.standard_normal((d_model, d_model)))
    WQ = np.empty((4, 128, d_model), np.float32)
    WK = np.empty((2, 128, d_model), np.float32)
    # KV head 0: orthonormal rows for q and k -> every singular value equal -> ER = 128
    WK[0] = Q[:128]
    WQ[0] = 2.0 * Q[:128]
    WQ[1] = 0.5 * Q[:128]
    # KV head 1: rank-deficient keys (rank 16) and a rank-1 query head
    WK[1] = rng.standard_normal((128, 16)) @ rng.standard_normal((16, d_model)) / 16.0
    WQ[2] = rng.standard_normal((128, 1)) @ rng.standard_normal((1, d_model))
    WQ[3] = rng.standard_normal((128, d_model)) / 16.0
    er_q, er_kv, mask, _, _ = gpu_ranks(WQ, WK, 1)
    want = A.head_effective_ranks(WQ.astype(np.float64), WK.astype(np.float64))
    np.testing.assert_allclose(er_q[:2], [128.0, 128.0], rtol=1e-9)
    np.testing.assert_allclose(er_q[:2], want[:2], rtol=ER_RTOL)
    np.testing.assert_allclose(er_q[2:], want[2:], rtol=ER_RTOL_DEFICIENT)
    assert np.array_equal(mask, [0, 1])


def test_head_ranks_reject_bad_arguments():
    WQ, WK = synth.make_head_weights(0, Hq=4, Hkv=2, d_model=64, retrieval=(0,))
    with pytest.raises(B.SpaError) as e:
        B.spa_head_ranks_workspace_size(6, 4)
    assert e.value.status == B.SPA_ERR_INVALID_ARG
    wq, wk = torch.from_numpy(WQ).cuda(), torch.from_numpy(WK).cuda()
    nbytes = B.spa_head_ranks_workspace_size(4, 2)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    out = torch.empty(8, dtype=torch.float64, device="cuda")
    m = torch.empty(2, dtype=torch.uint8, device="cuda")
    for args in [(4, 2, 64, 3, ws, nbytes), (4, 2, 0, 1, ws, nbytes), (4, 2, 64, 1, ws, nbytes - 8)]:
        with pytest.raises(B.SpaError) as e:
            B.spa_head_effective_ranks(wq, wk, *args, out, out, m)
        assert e.value.status == B.SPA_ERR_INVALID_ARG
