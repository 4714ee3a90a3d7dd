"""The two nearest centroids (fk_assign_top2) against the oracle: both labels
bit-exact on every row (the GPU re-decides near-ties of either pass in fp64),
distances within fp32 rounding, on the tensor-core and CUDA-core paths."""
import numpy as np
import pytest
import torch

import distance_argmin_flashassign_b200 as fk
import oracle
import workloads
from tests.parity import TORCH_DT, f64, record

pytestmark = pytest.mark.gpu
DEV = "cuda:0"

CASES = [(5000, 128, 300, "f16"), (4097, 128, 1024, "bf16"), (3000, 64, 33, "f16"), (2000, 32, 100, "f32"),
         (1500, 256, 257, "bf16"), (600, 100, 40, "f16"), (1000, 16, 2, "f32")]


def _check(X, C, dtype, case):
    Xd, Cd = X.to(DEV), C.to(DEV)
    l1, l2, d1, d2 = fk.fk_assign_top2(Xd, Cd, want_dist=True)
    C64 = oracle.round_to(dtype, f64(C.float()))
    o1, o2, e1, e2 = oracle.top2(f64(X), C64)
    g1, g2 = l1.cpu().numpy(), l2.cpu().numpy()
    mism1, mism2 = int((g1 != o1).sum()), int((g2 != o2).sum())
    record(case, N=X.shape[0], mismatch=mism1, mismatch_second=mism2)
    assert mism1 == 0 and mism2 == 0, f"{case}: {mism1} first and {mism2} second labels differ"
    scale = float(np.abs(e2).max()) + 1.0
    assert np.abs(d1.cpu().numpy() - e1).max() <= 1e-5 * scale
    assert np.abs(d2.cpu().numpy() - e2).max() <= 1e-5 * scale


@pytest.mark.parametrize("N,D,K,dtype", CASES, ids=lambda v: str(v))
def test_top2_matches_oracle(N, D, K, dtype):
    s = workloads.spec("embed_f16", N=N, D=D, K=K, n_centers=max(8, K // 4), dtype=dtype)
    w = workloads.make(s, seed=N + K)
    _check(w.X, w.C0.to(TORCH_DT[dtype]), dtype, f"top2 {dtype} N={N} D={D} K={K}")


def test_top2_duplicated_centroids():
    """Every centroid twice: the second label is the first one's duplicate
    (equal distance, next index) unless an earlier index ties -- decided
    exactly through the fp64 re-decision of both passes."""
    s = workloads.spec("embed_f16", N=3000, K=64, n_centers=16)
    w = workloads.make(s, seed=9)
    C = torch.cat([w.C0[:32], w.C0[:32]]).to(torch.float16)
    _check(w.X, C, "f16", "top2 duplicated centroids")


def test_top2_single_centroid():
    X = torch.randn(100, 8, device=DEV)
    C = torch.randn(1, 8, device=DEV)
    l1, l2, d1, d2 = fk.fk_assign_top2(X, C, want_dist=True)
    assert torch.all(l1 == 0) and torch.all(l2 == -1) and torch.all(torch.isinf(d2))


def test_top2_rejects_aliased_outputs():
    X = torch.randn(10, 8, device=DEV)
    C = torch.randn(3, 8, device=DEV)
    lab = torch.empty(10, dtype=torch.int32, device=DEV)
    with pytest.raises(fk.FKError):
        fk.fk_assign_top2(X, C, label1=lab, label2=lab)
