"""The seeded input generators: deterministic, the stated shapes, and the
structure the recipes describe (no GPU)."""
import numpy as np
import pytest
import torch

import workloads


def test_deterministic_and_seeded():
    s = workloads.spec("tiny_f32", N=4096)
    a, b = workloads.make(s, seed=0), workloads.make(s, seed=0)
    c = workloads.make(s, seed=1)
    assert torch.equal(a.X, b.X) and torch.equal(a.C0, b.C0)
    assert not torch.equal(a.X, c.X)


@pytest.mark.parametrize("name,dt", [("tiny_f32", torch.float32), ("embed_f16", torch.float16),
                                     ("batched_bf16", torch.bfloat16), ("zipf_bf16", torch.bfloat16)])
def test_shapes_and_dtypes(name, dt):
    s = workloads.spec(name)
    small = s.replace(N=2048, K=min(s.K, 64), n_centers=min(s.n_centers, 64), B=min(s.B, 2))
    w = workloads.make(small)
    shape = (small.N, small.D) if small.B == 1 else (small.B, small.N, small.D)
    assert tuple(w.X.shape) == shape and w.X.dtype == dt and w.X.is_contiguous()
    assert w.C0.dtype == torch.float32
    assert tuple(w.C0.shape) == ((small.K, small.D) if small.B == 1 else (small.B, small.K, small.D))


def test_init_rows_are_exact_copies():
    s = workloads.spec("embed_f16", N=5000, K=100, n_centers=100)
    w = workloads.make(s)
    idx = workloads.init_indices(s)
    assert len(set(idx.tolist())) == s.K
    assert torch.equal(w.C0, w.X[idx].float())
    s3 = workloads.spec("batched_bf16", N=1000, K=50, n_centers=50, B=3)
    w3 = workloads.make(s3)
    assert torch.equal(w3.C0, w3.X[:, :50].float())


def test_row_ranges_match_whole(monkeypatch):
    monkeypatch.setattr(workloads, "BLOCK_ROWS", 1000)
    s = workloads.spec("tiny_f32", N=3500, K=8, n_centers=8)
    whole = workloads.rows(s, 0, s.N)
    assert torch.equal(workloads.rows(s, 900, 2100), whole[900:2100])
    assert torch.equal(workloads.rows(s, 3000, 3500), whole[3000:])


def test_embed_rows_unit_norm():
    w = workloads.make("embed_f16", N=4096, K=64, n_centers=64)
    n = w.X.float().norm(dim=1)
    assert torch.allclose(n, torch.ones_like(n), atol=2e-3)


def test_zipf_top_cluster_mass():
    # finite Zipf(1.2) over 65,536 centres: the hottest holds about 19.8 %
    k = np.arange(1, 65537, dtype=np.float64)
    p = k ** -1.2
    assert abs(p[0] / p.sum() - 0.198) < 0.002
    lab = workloads.labels(200000, 65536, kind="zipf")
    frac = (lab == 0).float().mean().item()
    assert abs(frac - 0.198) < 0.01
    assert lab.dtype == torch.int32 and int(lab.min()) >= 0 and int(lab.max()) < 65536


def test_label_kinds():
    for kind in ["uniform", "zipf", "one", "sparse"]:
        lab = workloads.labels(10000, 300, kind=kind)
        assert lab.dtype == torch.int32 and lab.min() >= 0 and lab.max() < 300
    assert torch.all(workloads.labels(100, 9, kind="one") == 8)
    assert torch.all(workloads.labels(1000, 50, kind="sparse") % 7 == 0)
