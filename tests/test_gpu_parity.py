"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle.

Small and ragged shapes span several tiles of every kernel (256-point units,
256-centroid tiles, 4096-key sort tiles, chunked segment sums) and their
tails; inputs come from the seeded generators only."""
import numpy as np
import pytest
import torch

import distance_argmin_flashassign_b200 as fk
import oracle
import workloads
from tests.parity import TORCH_DT, centroid_slack, check_centroids, check_labels, f64, rel_l2

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def mixture(N, D, K, dtype, seed=0, cfg="tiny_f32", n_centers=None):
    s = workloads.spec(cfg, N=N, D=D, K=K, dtype=dtype, n_centers=n_centers or max(K, 2), B=1)
    w = workloads.make(s, seed=seed)
    return w.X, w.C0


def c_in(C0, dtype):
    return C0.to(TORCH_DT[dtype])


ASSIGN_SHAPES = [  # (N, D, K): tails in N, D and K; tensor and CUDA-core paths
    (1000, 32, 10), (3001, 128, 300), (257, 8, 1), (5000, 64, 1024), (600, 100, 37),
    (2000, 120, 513), (1000, 16, 700), (4097, 128, 2048), (700, 40, 256), (300, 128, 1),
    (3000, 192, 300), (2500, 256, 700), (1000, 136, 37), (600, 248, 513),  # 3 and 4 k-blocks on the tensor path
]


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("shape", ASSIGN_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_assign_matches_oracle(shape, dtype):
    N, D, K = shape
    X, C0 = mixture(N, D, K, dtype, seed=N + D + K)
    C = c_in(C0, dtype)
    Xd, Cd = X.to(DEV), C.to(DEV)
    labels, mind = fk.fk_assign(Xd, Cd, want_mindist=True)
    fk.fk_sync()
    check_labels(f64(X), f64(C), labels, dtype, gpu_mindist=mind, case=f"assign {N}x{D}x{K} {dtype}")


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("path", [1, 2])
def test_near_ties_are_decided_exactly(dtype, path):
    """Centroids in pairs one rounding step apart (and exact duplicates): many
    points have two candidates whose distances differ by less than the fp32
    error of the kernels' scores.  The listed near-ties are re-decided in
    fp64 exactly as the oracle computes, so every label equals the oracle's."""
    g = torch.Generator().manual_seed(21)
    N, D, half = 6000, 128, 300
    base = (torch.randn(half, D, generator=g) * 2.0 + 3.0).to(TORCH_DT[dtype])
    twin = base.clone()
    # move one coordinate of each twin by one step of the input type
    bits = twin.view(torch.int16 if dtype != "f32" else torch.int32)
    col = torch.randint(0, D, (half,), generator=g)
    bits[torch.arange(half), col] += 1
    C = torch.cat([base, twin, base[:40]])  # and 40 exact duplicates
    idx = torch.randint(0, C.shape[0], (N,), generator=g)
    X = (C[idx].float() + 0.05 * torch.randn(N, D, generator=g)).to(TORCH_DT[dtype])
    try:
        fk.fk_set_assign_path(path)
        labels, mind = fk.fk_assign(X.to(DEV), C.to(DEV), want_mindist=True)
        fk.fk_sync()
    finally:
        fk.fk_set_assign_path(0)
    st = check_labels(f64(X), f64(C), labels, dtype, gpu_mindist=mind, exact=True,
                      case=f"near-tie pairs {dtype} path {path}")
    assert st["near_tie_points"] > 0


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_full_comparison_when_three_chunks_tie(dtype):
    """Every centroid of one group of five is an exact copy, placed in five
    different 32-centroid chunks: points near that group tie five ways, so
    the kernels list them for a comparison with every centroid; the label is
    the lowest index of the group, as in the oracle."""
    g = torch.Generator().manual_seed(33)
    N, D, K = 4000, 128, 700
    C = (torch.randn(K, D, generator=g) * 3.0).to(TORCH_DT[dtype])
    group = [37, 100, 260, 450, 699]
    C[group] = C[37].clone()
    X = (C[torch.randint(0, K, (N,), generator=g)].float() + 0.05 * torch.randn(N, D, generator=g))
    X[: N // 2] = (C[37].float() + 0.05 * torch.randn(N // 2, D, generator=g))
    X = X.to(TORCH_DT[dtype])
    labels, mind = fk.fk_assign(X.to(DEV), C.to(DEV), want_mindist=True)
    fk.fk_sync()
    check_labels(f64(X), f64(C), labels, dtype, gpu_mindist=mind, exact=True,
                 case=f"five-way ties {dtype}")
    assert not torch.isin(labels.cpu(), torch.tensor(group[1:], dtype=torch.int32)).any()


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_prepared_points_and_assign(dtype):
    """fk_prepare_points gives |x|^2 (fp32 sums of exact squares); the
    prepared assignment with and without it gives the same labels."""
    X, C0 = mixture(5000, 128, 600, dtype, seed=8, cfg="embed_f16")
    Xd = X.to(DEV)
    xn = fk.fk_prepare_points(Xd)
    ref = (f64(X) ** 2).sum(1)
    np.testing.assert_allclose(f64(xn), ref, rtol=2 * 128 * 2.0**-24, atol=0)
    C_dt, bias = fk.fk_prepare_centroids(C0.to(DEV), TORCH_DT[dtype])
    l1 = torch.empty(5000, dtype=torch.int32, device=DEV)
    l2 = torch.empty_like(l1)
    m1 = torch.empty(5000, device=DEV)
    m2 = torch.empty_like(m1)
    fk.fk_assign_prepared(Xd, C_dt, bias, l1, m1, xnorm=xn)
    fk.fk_assign_prepared(Xd, C_dt, bias, l2, m2)
    fk.fk_sync()
    assert torch.equal(l1, l2)
    check_labels(f64(X), f64(C_dt), l1, dtype, gpu_mindist=m1, exact=True, case=f"prepared points {dtype}")


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
def test_tensor_and_cuda_core_paths_agree(dtype):
    X, C0 = mixture(6000, 128, 777, dtype, seed=3)
    Xd, Cd = X.to(DEV), c_in(C0, dtype).to(DEV)
    try:
        fk.fk_set_assign_path(1)
        l1, m1 = fk.fk_assign(Xd, Cd, want_mindist=True)
        fk.fk_set_assign_path(2)
        l2, m2 = fk.fk_assign(Xd, Cd, want_mindist=True)
        fk.fk_sync()
    finally:
        fk.fk_set_assign_path(0)
    check_labels(f64(X), f64(Cd), l1, dtype, gpu_mindist=m1)
    check_labels(f64(X), f64(Cd), l2, dtype, gpu_mindist=m2)


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("path", [1, 2])
@pytest.mark.parametrize("K", [300, 200])
def test_integer_inputs_bit_exact_with_ties(dtype, path, K):
    """Small integers: products and fp32 sums are exact, so labels (including
    lowest-index tie-breaks on duplicated centroids) and mindist are exact.
    K = 200 fits one 256-centroid tile (each point's whole row of scores is
    read by one warp); K = 300 spans two."""
    g = torch.Generator().manual_seed(5)
    N, D = 3000, 64
    third = K // 3
    X = torch.randint(-8, 9, (N, D), generator=g).to(TORCH_DT[dtype])
    C = torch.cat([X[:third], X[:third], torch.randint(-8, 9, (K - 2 * third, D), generator=g).to(TORCH_DT[dtype])])
    C[K - 50] = C[10]  # later duplicate of an earlier centroid
    try:
        fk.fk_set_assign_path(path)
        labels, mind = fk.fk_assign(X.to(DEV), C.to(DEV), want_mindist=True)
        fk.fk_sync()
    finally:
        fk.fk_set_assign_path(0)
    lab, md, _ = oracle.assign(f64(X), f64(C))
    assert np.array_equal(labels.cpu().numpy(), lab)
    assert np.array_equal(mind.cpu().numpy().astype(np.float64), md)
    assert labels[:third].cpu().tolist() == list(range(third))


@pytest.mark.parametrize("K", [300, 256])
def test_assign_batched_matches_per_problem(K):
    B, N, D = 5, 1500, 128
    s = workloads.spec("batched_bf16", N=N, K=K, n_centers=64, B=B)
    w = workloads.make(s, seed=1)
    X, C = w.X, w.C0.to(torch.bfloat16)
    labels, mind = fk.fk_assign(X.to(DEV), C.to(DEV), want_mindist=True)
    fk.fk_sync()
    for b in range(B):
        check_labels(f64(X[b]), f64(C[b]), labels[b], "bf16", gpu_mindist=mind[b])


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("kind", ["uniform", "zipf", "one", "sparse"])
@pytest.mark.parametrize("ND", [(5000, 128, 300), (20000, 32, 2100), (3000, 100, 17), (9000, 8, 64), (100, 1, 300)],
                         ids=lambda s: "x".join(map(str, s)))
def test_update_matches_oracle(ND, kind, dtype):
    N, D, K = ND
    X, _ = mixture(N, D, 2, dtype, seed=N + K)
    labels = workloads.labels(N, K, seed=K, kind=kind)
    C_prev = workloads.perturb(torch.zeros(K, D), 1.0, seed=D)
    C = C_prev.clone().to(DEV)
    counts = torch.empty(K, dtype=torch.int32, device=DEV)
    fk.fk_update(X.to(DEV), labels.to(DEV), C, counts)
    fk.fk_sync()
    Cn, cnt = oracle.update(f64(X), labels.numpy(), K, f64(C_prev))
    assert np.array_equal(counts.cpu().numpy(), cnt)
    empty = cnt == 0
    assert torch.equal(C.cpu()[torch.from_numpy(empty)], C_prev[torch.from_numpy(empty)])
    check_centroids(C, Cn)


def test_update_is_deterministic():
    X, _ = mixture(50000, 128, 2, "bf16", seed=9)
    labels = workloads.labels(50000, 1000, kind="zipf").to(DEV)
    Xd = X.to(DEV)
    outs = []
    for _ in range(2):
        C = torch.zeros(1000, 128, device=DEV)
        fk.fk_update(Xd, labels, C)
        outs.append(C.clone())
    fk.fk_sync()
    assert torch.equal(outs[0], outs[1])


@pytest.mark.parametrize("B,N,D,K,kind", [
    (4, 3000, 64, 500, "zipf"),       # B*K fits one 11-bit sort pass
    (4, 8192, 64, 1000, "zipf"),      # B*K needs two passes; N is whole sort tiles: one pass per problem
    (3, 12288, 32, 700, "uniform"),   # the same with K not a power of two
    (3, 5000, 32, 1000, "uniform"),   # two passes; N not whole tiles: the two-pass sort
])
def test_update_batched(B, N, D, K, kind):
    s = workloads.spec("batched_bf16", N=N, D=D, K=K, n_centers=50, B=B)
    X = workloads.make(s, seed=2).X
    labels = torch.stack([workloads.labels(N, K, seed=b, kind=kind) for b in range(B)])
    C = torch.zeros(B, K, D, device=DEV)
    counts = torch.empty(B, K, dtype=torch.int32, device=DEV)
    fk.fk_update(X.to(DEV), labels.to(DEV), C, counts)
    fk.fk_sync()
    for b in range(B):
        Cn, cnt = oracle.update(f64(X[b]), labels[b].numpy(), K, np.zeros((K, D)))
        assert np.array_equal(counts[b].cpu().numpy(), cnt)
        check_centroids(C[b], Cn)


def test_update_reports_bad_label():
    X = torch.randn(1000, 32, device=DEV)
    labels = torch.zeros(1000, dtype=torch.int32, device=DEV)
    labels[17] = 40
    C = torch.zeros(8, 32, device=DEV)
    fk.fk_update(X, labels, C)
    with pytest.raises(fk.FKError) as e:
        fk.fk_sync()
    assert e.value.status == fk.FK_ERR_BAD_LABEL
    fk.fk_sync()  # the status word was cleared


def test_update_batched_reports_bad_label():
    B, N, D, K = 2, 4096, 16, 1500  # sorted in one pass per problem
    X = torch.randn(B, N, D, device=DEV)
    labels = torch.zeros(B, N, dtype=torch.int32, device=DEV)
    labels[1, 17] = K + 3
    C = torch.zeros(B, K, D, device=DEV)
    counts = torch.empty(B, K, dtype=torch.int32, device=DEV)
    fk.fk_update(X, labels, C, counts)
    with pytest.raises(fk.FKError) as e:
        fk.fk_sync()
    assert e.value.status == fk.FK_ERR_BAD_LABEL
    # the bad label was counted in its problem's cluster 0
    assert counts[0, 0].item() == N and counts[1, 0].item() == N
    fk.fk_sync()


LLOYD_CASES = [
    ("tiny_f32", 32768, 128, 5, 128),          # the tiny workload at full size
    ("embed_f16", 16384, 256, 3, 256),
    ("zipf_bf16", 16384, 1024, 2, 1024),
]


@pytest.mark.parametrize("cfg,N,K,iters,nc", LLOYD_CASES)
def test_lloyd_step_by_step(cfg, N, K, iters, nc):
    """One GPU Lloyd step at a time, each started from the oracle's centroids
    of that step (inputs flow from the oracle to the GPU only)."""
    s = workloads.spec(cfg, N=N, K=K, n_centers=nc)
    w = workloads.make(s, seed=0)
    X64 = f64(w.X)
    Xd = w.X.to(DEV)
    C = f64(w.C0)
    for t in range(iters):
        C_next, lab, mind, _, counts = oracle.lloyd_step(X64, C, s.dtype)
        Cg = torch.from_numpy(C.astype(np.float32)).to(DEV)
        Cg, labels, gmind, gcounts = fk.fk_lloyd(Xd, Cg, 1, want_mindist=True)
        st = check_labels(X64, oracle.round_to(s.dtype, C), labels, s.dtype, gpu_mindist=gmind,
                          case=f"lloyd {cfg} N={N} K={K} step {t}")
        # the gate: the oracle's centroids from the oracle's labels, flat 1e-4
        st["centroid_rel_l2"] = check_centroids(Cg, C_next)
        st["slack"] = centroid_slack(X64, lab, labels.cpu().numpy(), C_next, counts)  # diagnostic only
        assert int(gcounts.sum()) == N
        assert torch.equal(gcounts.cpu().long(), torch.bincount(labels.cpu().long(), minlength=K))
        C = C_next


@pytest.mark.parametrize("cfg,N,K,iters,nc", LLOYD_CASES[:2])
def test_lloyd_trajectory_matches_oracle(cfg, N, K, iters, nc):
    """Whole fk_lloyd runs against the oracle's own trajectory (workloads whose
    clusters are well separated, so the two trajectories cannot part)."""
    s = workloads.spec(cfg, N=N, K=K, n_centers=nc)
    w = workloads.make(s, seed=0)
    C = w.C0.clone().to(DEV)
    C, labels, mind, counts = fk.fk_lloyd(w.X.to(DEV), C, iters, want_mindist=True)
    out = oracle.lloyd(f64(w.X), f64(w.C0), iters, s.dtype)
    check_centroids(C, out["C"])
    Cprev = oracle.lloyd(f64(w.X), f64(w.C0), iters - 1, s.dtype)["C"] if iters > 1 else f64(w.C0)
    check_labels(f64(w.X), oracle.round_to(s.dtype, Cprev), labels, s.dtype, gpu_mindist=mind,
                 case=f"lloyd trajectory {cfg} N={N} K={K}")
    assert int(counts.sum()) == N


def test_lloyd_batched_matches_oracle():
    s = workloads.spec("batched_bf16", N=4096, K=256, n_centers=256, B=3)
    w = workloads.make(s, seed=0)
    C = w.C0.clone().to(DEV)
    C, labels, _, counts = fk.fk_lloyd(w.X.to(DEV), C, 3)
    for b in range(3):
        out = oracle.lloyd(f64(w.X[b]), f64(w.C0[b]), 3, "bf16")
        check_centroids(C[b], out["C"])
        assert int(counts[b].sum()) == 4096


@pytest.mark.parametrize("dtype", ["f16", "f32"])
def test_ooc_matches_in_core(dtype):
    N, D, K = 50001, 128 if dtype == "f16" else 32, 300
    cfg = "ooc_f16" if dtype == "f16" else "tiny_f32"
    s = workloads.spec(cfg, N=N, D=D, K=K, n_centers=K, dtype=dtype)
    w = workloads.make(s, seed=4)
    Xh = w.X.pin_memory()
    Ch = w.C0.clone()
    lab_h = torch.empty(N, dtype=torch.int32).pin_memory()
    cnt_h = torch.empty(K, dtype=torch.int32)
    fk.fk_lloyd_ooc(Xh, Ch, 2, 12345, lab_h, cnt_h)
    Cd = w.C0.clone().to(DEV)
    Cd, labels, _, counts = fk.fk_lloyd(w.X.to(DEV), Cd, 2)
    assert rel_l2(Ch.numpy(), f64(Cd)) <= 1e-5
    mism = int((lab_h != labels.cpu()).sum())
    assert mism <= 1e-4 * N
    out = oracle.lloyd(f64(w.X), f64(w.C0), 2, dtype)
    check_centroids(Ch, out["C"])
    assert int(cnt_h.sum()) == N


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_prepared_bias_is_an_exact_tf32_split(dtype):
    # Each centroid's prepared bias is 8 floats: three terms that tf32 holds
    # exactly (low 13 fraction bits zero), summing exactly to one fp32 value
    # that is -|c_dt|^2/2 up to the rounding of an fp32 sum of D squares;
    # then zeros.  Padded centroids hold (-inf, 0, ...).
    B, K, D = 2, 300, 64
    g = torch.Generator().manual_seed(3)
    C = torch.randn(B, K, D, generator=g) * torch.logspace(-3, 3, K).view(1, K, 1)
    C_dt, bias = fk.fk_prepare_centroids(C.to(DEV), dtype)
    Kpad = (K + 255) // 256 * 256
    terms = bias.view(B, Kpad, 8).cpu()
    bits = terms.view(torch.int32)
    real = terms[:, :K]
    assert torch.all((bits[:, :K, :3] & 0x1FFF) == 0)
    assert torch.all(real[..., 3:] == 0)
    s64 = real[..., :3].double().sum(-1)
    assert torch.equal(s64.float().double(), s64)  # the terms add up to an fp32 value
    ref = -0.5 * (C_dt.cpu().double() ** 2).sum(-1)
    assert torch.all((s64 - ref).abs() <= 2 * D * 2.0**-24 * ref.abs())
    assert torch.all(torch.isneginf(terms[:, K:, 0])) and torch.all(terms[:, K:, 1:] == 0)


def test_ooc_repeated_calls_and_workspace_release():
    # The out-of-core driver keeps its buffers, side stream and events in the
    # scratch cache: repeated calls reuse them, and a call after
    # fk_release_workspace builds them again.  Every call gives the same result.
    N, D, K = 20000, 64, 100
    s = workloads.spec("ooc_f16", N=N, D=D, K=K, n_centers=K, dtype="f16")
    w = workloads.make(s, seed=9)
    Xh = w.X.pin_memory()
    results = []
    for release in (False, False, True, False):
        if release:
            fk.fk_release_workspace()
        Ch = w.C0.clone()
        lab_h = torch.empty(N, dtype=torch.int32).pin_memory()
        fk.fk_lloyd_ooc(Xh, Ch, 1, 7000, lab_h)
        results.append((Ch, lab_h.clone()))
    for Ch, lab in results[1:]:
        assert torch.equal(Ch, results[0][0])
        assert torch.equal(lab, results[0][1])
    out = oracle.lloyd(f64(w.X), f64(w.C0), 1, "f16")
    check_centroids(results[0][0], out["C"])


def test_edge_cases():
    # K = 1: every label 0, centroid = mean
    X = torch.randn(777, 16, device=DEV, dtype=torch.float16)
    C = X[:1].float().clone()
    C, labels, _, counts = fk.fk_lloyd(X, C, 1)
    assert int(labels.abs().sum()) == 0 and counts.tolist() == [777]
    np.testing.assert_allclose(C.cpu().numpy()[0], f64(X).mean(0), rtol=1e-3, atol=1e-3)
    # K > N: empty clusters keep their centroid
    X = torch.randn(50, 24, device=DEV)
    C0 = torch.randn(300, 24, device=DEV)
    C = C0.clone()
    C, labels, _, counts = fk.fk_lloyd(X, C, 1)
    empty = counts == 0
    assert int(empty.sum()) >= 250 and torch.equal(C[empty], C0[empty])
    # N = 0: no-op
    lab = torch.empty(0, dtype=torch.int32, device=DEV)
    fk.fk_assign(torch.empty(0, 8, device=DEV, dtype=torch.float16), torch.zeros(3, 8, device=DEV,
                 dtype=torch.float16), labels=lab)
    # D = 1 and identical points
    X = torch.full((1000, 1), 2.5, device=DEV)
    labels, mind = fk.fk_assign(X, torch.tensor([[1.0], [4.0], [2.5], [2.5]], device=DEV), want_mindist=True)
    fk.fk_sync()
    assert torch.all(labels == 2) and torch.all(mind == 0)


def test_wait_timeout_mechanism_and_recovery():
    assert fk.fk_debug_wait_timeout(1_000_000) == fk.FK_ERR_TIMEOUT
    X = torch.randn(1000, 64, device=DEV, dtype=torch.float16)
    labels, _ = fk.fk_assign(X, X[:10].clone())
    fk.fk_sync()
    assert labels[:10].cpu().tolist() == list(range(10))


def test_launch_counter_counts_kernels():
    X = torch.randn(5000, 128, device=DEV, dtype=torch.float16)
    n0 = fk.fk_launch_count()
    fk.fk_assign(X, X[:300].clone())
    fk.fk_sync()
    assert fk.fk_launch_count() - n0 == 3  # norms + tensor-core assign + near-tie re-decision


TF32_SHAPES = [(1, 4, 1), (129, 1024, 129), (5000, 36, 4096), (300, 8, 2), (2048, 64, 257), (777, 4, 40)]


@pytest.mark.parametrize("shape", TF32_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_fp32_tensor_path_edges(shape):
    """The fp32 tensor-core path (three tf32 passes) at its edges: one row, the
    smallest and largest D it takes (4 and 1,024 = 32 k-blocks), ragged units
    and tiles (129 rows and centroids), K = 1 to 4,096.  Forced onto that path;
    labels must equal the oracle's."""
    N, D, K = shape
    X, C0 = mixture(N, D, K, "f32", seed=N * 7 + D + K)
    try:
        fk.fk_set_assign_path(1)
        labels, mind = fk.fk_assign(X.to(DEV), C0.to(DEV), want_mindist=True)
        fk.fk_sync()
    finally:
        fk.fk_set_assign_path(0)
    check_labels(f64(X), f64(C0), labels, "f32", gpu_mindist=mind, exact=True,
                 case=f"tf32 path {N}x{D}x{K}")


def test_fp32_unaligned_rows_fall_back():
    """X starting 4 bytes past a 16-byte boundary cannot feed the tensor maps:
    the assignment runs on the CUDA-core kernel, with the same exact labels."""
    X, C0 = mixture(3000, 64, 300, "f32", seed=77)
    base = torch.empty(X.numel() + 1, device=DEV)
    Xu = base[1:].view(X.shape)
    Xu.copy_(X.to(DEV))
    assert Xu.data_ptr() % 16 == 4
    labels, mind = fk.fk_assign(Xu, C0.to(DEV), want_mindist=True)
    fk.fk_sync()
    check_labels(f64(X), f64(C0), labels, "f32", gpu_mindist=mind, exact=True, case="fp32 unaligned rows")
