"""Parity at the full sizes of the configured workloads, one Lloyd step at a
time, in bench.py's launch configuration (fk_prepare_centroids,
fk_prepare_points once, fk_assign_prepared and fk_update on inputs resident in
HBM; the out-of-core case runs fk_lloyd_ooc from pinned host memory).

* Embedding (2^20 x 128, K = 1024, 20 iterations) and batched (32 problems of
  32,768 x 128, K = 256, 10 iterations): the oracle runs its own trajectory
  over every row (its screened assignment, which gives the plain oracle's
  labels exactly), and every GPU step starts from the oracle's centroids of
  that step.  Labels of all rows, counts and the next centroids are compared.
* Zipf (2^23 x 128, K = 65,536): one oracle step over every row needs about
  1.4e14 fp64 flops, so at this size the GPU's own trajectory is checked
  step by step for what holds at any size -- the labels of a seeded sample of
  rows are the nearest of the centroids that step used (oracle, exact), the
  counts are the label histogram, sampled clusters (the largest among them)
  are the oracle's means of their members, and every empty cluster keeps its
  centroid.  The oracle's own trajectory is compared over every row on the
  same recipe at 2^19 rows and K = 4,096.
"""
import numpy as np
import pytest
import torch

import distance_argmin_flashassign_b200 as fk
import oracle
import workloads
from tests.parity import CENTROID_REL_L2, check_centroids, check_labels, f64, record, rel_l2

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
DEV = "cuda:0"
SAMPLE_ROWS = 4096
SAMPLE_CLUSTERS = 16


class BenchStep:
    """One Lloyd step as bench.py times it, on inputs resident in HBM."""

    def __init__(self, X):
        self.X = X
        self.xnorm = fk.fk_prepare_points(X)

    def __call__(self, C):
        """C: fp32 master centroids on the device.  Returns (rounded
        centroids, labels, new centroids, counts)."""
        X = self.X
        C_dt, bias = fk.fk_prepare_centroids(C, X.dtype)
        labels = torch.empty(X.shape[:-1], dtype=torch.int32, device=X.device)
        fk.fk_assign_prepared(X, C_dt, bias, labels, xnorm=self.xnorm)
        C_new = C.clone()
        counts = torch.empty(C.shape[:-1], dtype=torch.int32, device=X.device)
        fk.fk_update(X, labels, C_new, counts)
        fk.fk_sync()
        return C_dt, labels, C_new, counts


def _oracle_trajectory_check(name, X, C0, dtype, iters, problem_ids=None):
    """Every step: GPU from the oracle's C_t against the oracle's step."""
    step = BenchStep(X)
    batched = X.dim() == 3
    probs = list(range(X.shape[0])) if batched else [None]
    X64 = [f64(X[b]) if batched else f64(X) for b in probs]
    C = [f64(C0[b]) if batched else f64(C0) for b in probs]
    for t in range(iters):
        Cg = torch.from_numpy(np.stack(C) if batched else C[0]).float().to(DEV)
        _, labels, C_new, counts = step(Cg)
        for i, b in enumerate(probs):
            C_next, lab, mind, second, cnt = oracle.lloyd_step(X64[i], C[i], dtype, screened=True)
            gl = labels[b] if batched else labels
            st = check_labels(X64[i], oracle.round_to(dtype, C[i]), gl, dtype, oracle_out=(lab, mind, second),
                              case=f"full size {name} step {t}" + (f" problem {b}" if batched else ""))
            gc = (counts[b] if batched else counts).cpu().numpy()
            assert np.array_equal(gc, cnt), "counts differ from the oracle's"
            st["centroid_rel_l2"] = check_centroids(C_new[b] if batched else C_new, C_next)
            C[i] = C_next


def test_full_size_embedding_trajectory():
    s = workloads.spec("embed_f16")
    w = workloads.make(s, device=DEV)
    _oracle_trajectory_check("embed_f16", w.X, w.C0, s.dtype, s.iters)


def test_full_size_batched_trajectory():
    s = workloads.spec("batched_bf16")
    w = workloads.make(s, device=DEV)
    _oracle_trajectory_check("batched_bf16", w.X, w.C0, s.dtype, s.iters)


def test_zipf_reduced_trajectory():
    """The Zipf recipe at 2^19 rows and K = 4,096 (as many centres), every
    row compared against the oracle's own trajectory for the configured 10
    iterations."""
    s = workloads.spec("zipf_bf16", N=1 << 19, K=4096, n_centers=4096)
    w = workloads.make(s, device=DEV)
    _oracle_trajectory_check("zipf_bf16 2^19 x 4096", w.X, w.C0, s.dtype, s.iters)


def test_zipf_full_size_steps():
    s = workloads.spec("zipf_bf16")
    w = workloads.make(s, device=DEV)
    X = w.X
    N, K = s.N, s.K
    step = BenchStep(X)
    rng = np.random.default_rng(11)
    C = w.C0.clone()
    for t in range(s.iters):
        _, labels, C_new, counts = step(C)
        # labels of sampled rows: the nearest of the centroids this step used
        rows = np.sort(rng.choice(N, size=SAMPLE_ROWS, replace=False))
        ridx = torch.as_tensor(rows, device=DEV)
        st = check_labels(f64(X[ridx]), oracle.round_to(s.dtype, f64(C)), labels[ridx], s.dtype, screened=True,
                          case=f"full size zipf_bf16 step {t} (sampled rows)")
        # counts: the label histogram, exactly
        lab = labels.long()
        assert int(counts.sum()) == N
        assert torch.equal(counts, torch.bincount(lab, minlength=K).to(torch.int32))
        # sampled clusters are the means of their members; the largest one at
        # the first and the last step
        cnt = counts.cpu().numpy()
        nonempty = np.nonzero(cnt)[0]
        ks = {int(k) for k in rng.choice(nonempty, size=min(SAMPLE_CLUSTERS, len(nonempty)), replace=False)}
        if t in (0, s.iters - 1):
            ks.add(int(np.argmax(cnt)))
        ks = np.array(sorted(ks))
        kidx = torch.as_tensor(ks, device=DEV)
        member = torch.isin(lab, kidx)
        remap = torch.full((K,), -1, dtype=torch.long, device=DEV)
        remap[kidx] = torch.arange(len(ks), device=DEV)
        C_or, cnt_or = oracle.update(f64(X[member]), remap[lab[member]].cpu().numpy().astype(np.int32), len(ks),
                                     f64(C[kidx]))
        assert np.array_equal(cnt_or, cnt[ks])
        r = rel_l2(f64(C_new[kidx]), C_or)
        assert r <= CENTROID_REL_L2, f"sampled-centroid rel-L2 {r:.3g}"
        st["centroid_rel_l2"] = r
        # every empty cluster keeps its centroid
        empty = counts == 0
        assert torch.equal(C_new[empty], C[empty])
        st["empty_clusters"] = int(empty.sum())
        C = C_new


def test_out_of_core_large_chunks():
    """fk_lloyd_ooc at the configured K and D with 16 M rows (4 GiB of pinned
    fp16 host memory; the configured 10^9 rows need 256 GB, more than the host
    has) in 4 chunks of 4 M rows, one iteration."""
    N, chunk = 1 << 24, 1 << 22
    s = workloads.spec("ooc_f16", N=N)
    Xh = torch.empty((N, s.D), dtype=torch.float16).pin_memory()
    for r0 in range(0, N, chunk):  # generated on the device block by block, same recipe
        Xh[r0:r0 + chunk].copy_(workloads.rows(s, r0, r0 + chunk, device=DEV))
    C0 = Xh[: s.K].float().clone()  # first K rows, the configured initialisation
    Ch = C0.clone()
    lab_h = torch.empty(N, dtype=torch.int32).pin_memory()
    cnt_h = torch.empty(s.K, dtype=torch.int32)
    fk.fk_lloyd_ooc(Xh, Ch, 1, chunk, lab_h, cnt_h)
    rng = np.random.default_rng(13)
    rows = np.sort(rng.choice(N, size=SAMPLE_ROWS, replace=False))
    C64 = oracle.round_to("f16", C0.numpy())
    check_labels(Xh[rows].double().numpy(), C64, lab_h[rows], "f16", screened=True,
                 case="out of core 2^24 rows (sampled rows)")
    assert int(cnt_h.sum()) == N
    assert torch.equal(cnt_h, torch.bincount(lab_h.long(), minlength=s.K).to(torch.int32))
    ks = np.sort(rng.choice(np.nonzero(cnt_h.numpy())[0], size=SAMPLE_CLUSTERS, replace=False))
    member = torch.isin(lab_h, torch.as_tensor(ks, dtype=torch.int32))
    remap = np.full(s.K, -1, np.int32)
    remap[ks] = np.arange(len(ks))
    C_or, cnt_or = oracle.update(Xh[member].double().numpy(), remap[lab_h[member].numpy()], len(ks),
                                 C0[ks].double().numpy())
    assert np.array_equal(cnt_or, cnt_h.numpy()[ks])
    assert rel_l2(Ch[ks].double().numpy(), C_or) <= CENTROID_REL_L2
    record("out of core 2^24 rows (sampled clusters)", centroid_rel_l2=rel_l2(Ch[ks].double().numpy(), C_or))
