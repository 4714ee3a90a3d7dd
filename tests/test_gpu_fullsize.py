"""Parity at the full sizes of the configured workloads.

Each case runs one Lloyd step the way bench.py times it: fk_prepare_centroids,
fk_assign_prepared and fk_update on inputs resident in HBM; the out-of-core
case runs fk_lloyd_ooc from pinned host memory.  The oracle cannot afford all
N x K distances at these sizes, so it checks:
  * the labels of a seeded sample of rows, against oracle.assign on the same
    rounded rows and centroids (the usual near-tie rule);
  * the counts, against a bincount of the GPU's labels (bit-exact);
  * the centroids of a sample of clusters (the largest one included), against
    oracle.update on their members, and an empty cluster keeping its centroid.
"""
import numpy as np
import pytest
import torch

import distance_argmin_flashassign_b200 as fk
import oracle
import workloads
from tests.parity import CENTROID_REL_L2, check_labels, f64, rel_l2

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
DT = {"f16": torch.float16, "bf16": torch.bfloat16}
SAMPLE_ROWS = 2048
SAMPLE_CLUSTERS = 16


def _bench_step(X, C):
    """One Lloyd step in bench.py's launch configuration; returns
    (rounded centroids, labels, new centroids, counts)."""
    C_dt, bias = fk.fk_prepare_centroids(C, X.dtype)
    labels = torch.empty(X.shape[:-1], dtype=torch.int32, device=X.device)
    fk.fk_assign_prepared(X, C_dt, bias, labels, xnorm=fk.fk_prepare_points(X))
    C_new = C.clone()
    counts = torch.empty(C.shape[:-1], dtype=torch.int32, device=X.device)
    fk.fk_update(X, labels, C_new, counts)
    torch.cuda.synchronize()
    return C_dt, labels, C_new, counts


def _check_problem(X, C_prev, C_dt, labels, C_new, counts, dtype, rng):
    """Sampled checks of one problem (X N x D on the device, the rest 1-problem views)."""
    N, D = X.shape
    K = C_prev.shape[0]
    # labels of sampled rows against the oracle on the same rounded values
    rows = np.sort(rng.choice(N, size=min(SAMPLE_ROWS, N), replace=False))
    ridx = torch.as_tensor(rows, device=X.device)
    X64 = f64(X[ridx])
    stats = check_labels(X64, f64(C_dt), labels[ridx], dtype)
    # counts: exact, from the labels
    lab = labels.long()
    assert int(counts.sum()) == N
    assert torch.equal(counts, torch.bincount(lab, minlength=K).to(torch.int32))
    # centroids of sampled clusters: the largest, random non-empty ones, and an empty one
    cnt = counts.cpu().numpy()
    nonempty = np.nonzero(cnt)[0]
    ks = {int(np.argmax(cnt))}
    ks.update(int(k) for k in rng.choice(nonempty, size=min(SAMPLE_CLUSTERS, len(nonempty)), replace=False))
    ks = np.array(sorted(ks))
    kidx = torch.as_tensor(ks, device=X.device)
    member = torch.isin(lab, kidx)
    Xm = f64(X[member])
    remap = torch.full((K,), -1, dtype=torch.long, device=X.device)
    remap[kidx] = torch.arange(len(ks), device=X.device)
    lm = remap[lab[member]].cpu().numpy().astype(np.int32)
    C_or, cnt_or = oracle.update(Xm, lm, len(ks), f64(C_prev[kidx]))
    assert np.array_equal(cnt_or, cnt[ks])
    r = rel_l2(f64(C_new[kidx]), C_or)
    assert r <= CENTROID_REL_L2, f"sampled-centroid rel-L2 {r:.3g}"
    empty = np.nonzero(cnt == 0)[0]
    if len(empty):
        k = int(empty[0])
        assert torch.equal(C_new[k], C_prev[k]), "an empty cluster must keep its centroid"
    return stats, r


@pytest.mark.parametrize("name", ["embed_f16", "zipf_bf16"])
def test_full_size_single_problem(name):
    s = workloads.spec(name)
    w = workloads.make(s, device=DEV)
    C_dt, labels, C_new, counts = _bench_step(w.X, w.C0.clone())
    stats, r = _check_problem(w.X, w.C0, C_dt, labels, C_new, counts, s.dtype, np.random.default_rng(11))
    assert stats["N"] == SAMPLE_ROWS


def test_full_size_batched():
    s = workloads.spec("batched_bf16")
    w = workloads.make(s, device=DEV)
    C_dt, labels, C_new, counts = _bench_step(w.X, w.C0.clone())
    rng = np.random.default_rng(12)
    for b in (0, s.B // 2, s.B - 1):  # first, middle and last problem of the one launch
        _check_problem(w.X[b], w.C0[b], C_dt[b], labels[b], C_new[b], counts[b], s.dtype, rng)


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
    check_labels(Xh[rows].double().numpy(), C64, lab_h[rows], "f16")
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
