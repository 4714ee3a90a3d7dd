"""The single-pass Lloyd iteration (fk_lloyd_fused) against the oracle.

Every step starts from the oracle's centroids of that step (inputs flow from
the oracle to the GPU only): labels must be the oracle's exactly, counts
exactly, centroids within the flat 1e-4 rel-L2 gate of the oracle's means
from the oracle's labels.  Multi-iteration calls (one cooperative launch for
all iterations) are checked against the oracle's own trajectory and against
fk_lloyd, and the summation order is checked to be fixed."""
import numpy as np
import pytest
import torch

import distance_argmin_flashassign_b200 as fk
import oracle
import workloads
from tests.parity import check_centroids, check_labels, f64

pytestmark = pytest.mark.gpu
DEV = "cuda:0"

# (workload recipe, N, D, K, dtype): the tiny configuration at full size,
# tails in N (not whole 512-row passes), D (not a multiple of 4, more than
# one 32-dimension chunk, wide rows) and K (not whole 32-centroid tiles),
# fp16/bf16 inputs, a problem smaller than one pass, K = 1.
CASES = [
    ("tiny_f32", 32768, 32, 128, "f32"),
    ("tiny_f32", 20001, 30, 100, "f32"),
    ("tiny_f32", 9000, 100, 57, "f16"),
    ("tiny_f32", 7777, 64, 200, "bf16"),
    ("tiny_f32", 300, 16, 40, "f32"),
    ("tiny_f32", 5000, 512, 16, "f16"),
    ("tiny_f32", 4000, 24, 1, "f32"),
]


def _data(cfg, N, D, K, dtype, seed=0):
    s = workloads.spec(cfg, N=N, D=D, K=K, n_centers=max(K, 2), dtype=dtype)
    return s, workloads.make(s, seed=seed)


@pytest.mark.parametrize("cfg,N,D,K,dtype", CASES, ids=lambda v: str(v))
def test_fused_step_by_step(cfg, N, D, K, dtype):
    s, w = _data(cfg, N, D, K, dtype)
    X64 = f64(w.X)
    Xd = w.X.to(DEV)
    C = f64(w.C0)
    for t in range(3):
        C_next, lab, mind, _, counts = oracle.lloyd_step(X64, C, s.dtype)
        Cg = torch.from_numpy(C.astype(np.float32)).to(DEV)
        Cg, labels, gmind, gcounts = fk.fk_lloyd(Xd, Cg, 1, want_mindist=True, fused=True)
        check_labels(X64, oracle.round_to(s.dtype, C), labels, s.dtype, gpu_mindist=gmind,
                     case=f"fused {dtype} N={N} D={D} K={K} step {t}")
        assert np.array_equal(gcounts.cpu().numpy(), counts), "counts differ from the oracle's"
        check_centroids(Cg, C_next)
        C = C_next


def test_fused_trajectory_and_two_pass_agree():
    """All five configured iterations of the tiny workload in one call: the
    oracle's trajectory, and fk_lloyd's (same labels; centroids to fp32
    rounding of a different summation order)."""
    s = workloads.spec("tiny_f32")
    w = workloads.make(s, seed=0)
    Xd = w.X.to(DEV)
    Cf, lf, mf, cf = fk.fk_lloyd(Xd, w.C0.clone().to(DEV), s.iters, want_mindist=True, fused=True)
    Ct, lt, mt, ct = fk.fk_lloyd(Xd, w.C0.clone().to(DEV), s.iters, want_mindist=True)
    out = oracle.lloyd(f64(w.X), f64(w.C0), s.iters, s.dtype)
    check_centroids(Cf, out["C"])
    assert torch.equal(lf, lt)
    assert torch.equal(cf, ct)
    assert float((Cf - Ct).norm() / Ct.norm()) < 1e-6


def test_fused_is_deterministic():
    s, w = _data("tiny_f32", 20001, 30, 100, "f32", seed=3)
    Xd = w.X.to(DEV)
    a = fk.fk_lloyd(Xd, w.C0.clone().to(DEV), 4, fused=True)
    b = fk.fk_lloyd(Xd, w.C0.clone().to(DEV), 4, fused=True)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1]) and torch.equal(a[3], b[3])


def test_fused_empty_cluster_keeps_centroid():
    """A centroid far from every point stays where it is; its count is 0."""
    s, w = _data("tiny_f32", 3000, 8, 10, "f32", seed=4)
    C = w.C0.clone()
    C[7] = 1e4
    Cg, labels, _, counts = fk.fk_lloyd(w.X.to(DEV), C.clone().to(DEV), 1, fused=True)
    assert int(counts[7]) == 0
    assert torch.equal(Cg[7].cpu(), C[7])


def test_fused_rejects_large_shapes():
    X = torch.zeros(100, 128, device=DEV)
    C = torch.zeros(1024, 128, device=DEV)
    with pytest.raises(fk.FKError):
        fk.fk_lloyd(X, C, 1, fused=True)
