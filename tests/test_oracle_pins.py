"""Pins for the CPU oracle (no GPU).

The Flash-KMeans pages (arXiv 2603.09229 abstract; the Japanese HN summary,
section on what Flash-KMeans changes) print no worked example, so the oracle is
pinned to things other than itself:

* library routines that solve a special case: ``scipy.cluster.vq.vq`` (nearest
  code-book entry) and ``sklearn.cluster.KMeans`` limited to one Lloyd step;
* closed forms and hand-worked cases (K = 1 gives the global mean; a 1-D
  example; centroids equal to data rows);
* invariants of Lloyd's algorithm (counts sum to N, each centroid is the mean
  of its members, the objective never increases);
* recovery of a planted, well-separated mixture;
* the tie and empty-cluster readings (lowest index; keep previous centroid).

``test_mutants_are_caught`` plants plausible mistakes in a copy of the C
source and checks that the pins above reject every one of them.
"""
import os
import re
import tempfile

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


# ----------------------------------------------------------------- pins ----
def pin_vq(lib):
    from scipy.cluster.vq import vq
    rng = np.random.default_rng(1)
    for (N, D, K) in [(300, 3, 7), (257, 1, 5), (64, 33, 64), (50, 8, 1)]:
        X = rng.standard_normal((N, D))
        C = rng.standard_normal((K, D))
        lab, mind, second = oracle.assign(X, C, lib)
        code, dist = vq(X, C, check_finite=True)
        assert np.array_equal(lab, code.astype(np.int32)), (N, D, K)
        np.testing.assert_allclose(mind, dist ** 2, rtol=1e-9, atol=1e-12)
        full = ((X[:, None, :] - C[None, :, :]) ** 2).sum(-1)
        if K > 1:
            full[np.arange(N), lab] = np.inf
            np.testing.assert_allclose(second, full.min(1), rtol=1e-9, atol=1e-12)
        else:
            assert np.all(np.isinf(second))


def pin_sklearn_step(lib):
    from sklearn.cluster import KMeans
    rng = np.random.default_rng(2)
    for (N, D, K) in [(500, 5, 7), (400, 16, 20)]:
        X = rng.standard_normal((N, D)) + 3.0 * rng.integers(0, 4, (N, 1))
        C0 = X[:K].copy()
        lab, _, _ = oracle.assign(X, C0, lib)
        Cn, counts = oracle.update(X, lab, K, C0, lib)
        assert counts.min() > 0  # sklearn relocates empty clusters; avoid them here
        km = KMeans(n_clusters=K, init=C0, n_init=1, max_iter=1, algorithm="lloyd",
                    tol=0.0).fit(X)
        np.testing.assert_allclose(Cn, km.cluster_centers_, rtol=1e-10, atol=1e-12)


def pin_hand_1d(lib):
    # points 0,1,9,10,4 against centroids 0 and 10 (worked by hand):
    # squared distances (0,100) (1,81) (81,1) (100,0) (16,36)
    X = np.array([[0.0], [1.0], [9.0], [10.0], [4.0]])
    C = np.array([[0.0], [10.0]])
    lab, mind, second = oracle.assign(X, C, lib)
    assert lab.tolist() == [0, 0, 1, 1, 0]
    assert mind.tolist() == [0.0, 1.0, 1.0, 0.0, 16.0]
    assert second.tolist() == [100.0, 81.0, 81.0, 100.0, 36.0]
    Cn, counts = oracle.update(X, lab, 2, C, lib)
    assert counts.tolist() == [3, 2]
    assert Cn[0, 0] == pytest.approx(5.0 / 3.0, abs=1e-15) and Cn[1, 0] == 9.5
    # 2-D: x = (1, 2), c0 = (4, 6) -> 9 + 16 = 25, c1 = (1, -1) -> 0 + 9 = 9
    lab, mind, _ = oracle.assign(np.array([[1.0, 2.0]]), np.array([[4.0, 6.0], [1.0, -1.0]]), lib)
    assert lab.tolist() == [1] and mind.tolist() == [9.0]


def pin_ties(lib):
    # x = 5 is equidistant (25) from 0 and 10: the lower index wins, whatever the values
    X = np.array([[5.0], [5.0]])
    assert oracle.assign(X, np.array([[0.0], [10.0]]), lib)[0].tolist() == [0, 0]
    assert oracle.assign(X, np.array([[10.0], [0.0]]), lib)[0].tolist() == [0, 0]
    # duplicated centroids: the first copy wins
    C = np.array([[9.0, 9.0], [1.0, 1.0], [1.0, 1.0], [1.0, 1.0]])
    X = np.array([[1.0, 2.0], [0.0, 0.0], [9.0, 9.0]])
    assert oracle.assign(X, C, lib)[0].tolist() == [1, 1, 0]
    # small-integer lattice: ties exact in fp64, brute-force first minimum
    rng = np.random.default_rng(3)
    X = rng.integers(-3, 4, (200, 3)).astype(np.float64)
    C = rng.integers(-3, 4, (9, 3)).astype(np.float64)
    lab, mind, _ = oracle.assign(X, C, lib)
    for i in range(len(X)):
        d = [int(((X[i] - C[k]) ** 2).sum()) for k in range(len(C))]
        assert lab[i] == d.index(min(d)) and mind[i] == min(d)


def pin_k1_mean(lib):
    rng = np.random.default_rng(4)
    X = rng.standard_normal((123, 6))
    lab, mind, _ = oracle.assign(X, X[:1], lib)
    assert np.all(lab == 0)
    Cn, counts = oracle.update(X, lab, 1, X[:1], lib)
    assert counts.tolist() == [123]
    np.testing.assert_allclose(Cn[0], X.mean(0), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(mind, ((X - X[0]) ** 2).sum(1), rtol=1e-12, atol=1e-14)


def pin_prefix_identity(lib):
    rng = np.random.default_rng(5)
    X = rng.standard_normal((90, 4))
    K = 30
    lab, mind, second = oracle.assign(X, X[:K], lib)
    assert lab[:K].tolist() == list(range(K))
    assert np.all(mind[:K] == 0.0) and np.all(second[:K] > 0)


def pin_permutation(lib):
    rng = np.random.default_rng(6)
    X = rng.standard_normal((400, 5))
    C = rng.standard_normal((13, 5))
    perm = rng.permutation(13)
    l1, m1, _ = oracle.assign(X, C, lib)
    l2, m2, _ = oracle.assign(X, C[perm], lib)
    # centroid perm[j] sits at position j, so label l1 -> position inv[l1]
    inv = np.argsort(perm)
    assert np.array_equal(l2, inv[l1]) and np.array_equal(m1, m2)


def pin_empty_cluster(lib):
    X = np.array([[0.0, 0.0], [0.1, 0.0], [5.0, 5.0]])
    C = np.array([[0.0, 0.0], [100.0, 100.0], [5.0, 5.0]])
    lab, _, _ = oracle.assign(X, C, lib)
    assert lab.tolist() == [0, 0, 2]
    Cn, counts = oracle.update(X, lab, 3, C, lib)
    assert counts.tolist() == [2, 0, 1]
    assert Cn[1].tolist() == [100.0, 100.0]
    np.testing.assert_allclose(Cn[0], [0.05, 0.0], rtol=0, atol=1e-15)


def pin_invariants(lib):
    rng = np.random.default_rng(7)
    N, D, K = 600, 4, 9
    X = rng.standard_normal((N, D)) + 4.0 * rng.integers(0, 3, (N, D))
    out = None
    C = X[:K].copy()
    J_prev = np.inf
    for _ in range(8):
        lab, mind, _ = oracle.assign(X, C, lib)
        J = mind.sum()
        assert J <= J_prev * (1 + 1e-12)
        Cn, counts = oracle.update(X, lab, K, C, lib)
        assert counts.sum() == N
        sums = np.zeros((K, D))
        np.add.at(sums, lab, X)
        nz = counts > 0
        np.testing.assert_allclose(Cn[nz], sums[nz] / counts[nz, None], rtol=1e-12, atol=1e-13)
        # the update never increases the objective for fixed labels
        assert oracle.objective(X, lab, Cn, lib) <= J * (1 + 1e-12)
        J_prev, C = J, Cn
    out = oracle.lloyd(X, X[:K], 8, "f64", lib)
    h = out["objective"]
    assert all(b <= a * (1 + 1e-12) for a, b in zip(h, h[1:]))


def pin_objective(lib):
    # hand-worked: the 1-D case above, each point against its nearest centroid:
    # J = 0 + 1 + 1 + 0 + 16 = 18
    X = np.array([[0.0], [1.0], [9.0], [10.0], [4.0]])
    C = np.array([[0.0], [10.0]])
    assert oracle.objective(X, np.array([0, 0, 1, 1, 0], np.int32), C, lib) == 18.0
    # labels need not be the nearest: every point on centroid 1 gives
    # 100 + 81 + 1 + 0 + 36 = 218
    assert oracle.objective(X, np.ones(5, np.int32), C, lib) == 218.0
    # 2-D, worked by hand: (1,2)->(4,6): 25; (0,0)->(1,-1): 2; (3,3)->(4,6): 10
    X2 = np.array([[1.0, 2.0], [0.0, 0.0], [3.0, 3.0]])
    C2 = np.array([[4.0, 6.0], [1.0, -1.0]])
    assert oracle.objective(X2, np.array([0, 1, 0], np.int32), C2, lib) == 37.0
    # brute force with numpy on random data and random (not nearest) labels
    rng = np.random.default_rng(12)
    X = rng.standard_normal((700, 9))
    C = rng.standard_normal((23, 9))
    lab = rng.integers(0, 23, 700).astype(np.int32)
    ref = float(((X - C[lab]) ** 2).sum())
    assert oracle.objective(X, lab, C, lib) == pytest.approx(ref, rel=1e-12)
    # with the nearest labels it equals the sum of the assignment's distances
    lab, mind, _ = oracle.assign(X, C, lib)
    assert oracle.objective(X, lab, C, lib) == pytest.approx(float(mind.sum()), rel=1e-12)


def pin_gauss(lib):
    # one centre, unit weight: the closed form exp(-beta d)
    X = np.array([[0.0], [1.0], [3.0]])
    G, L = oracle.gauss_sum(X, np.array([[1.0]]), 0.5, lib=lib)
    np.testing.assert_allclose(G, np.exp(-0.5 * np.array([1.0, 0.0, 4.0])), rtol=1e-15)
    np.testing.assert_allclose(L, -0.5 * np.array([1.0, 0.0, 4.0]), rtol=0, atol=1e-15)
    # hand-worked: x = 0, centres 1 and 2, weights 3 and -1, beta 0.5:
    # 3 e^-0.5 - e^-2
    G, L = oracle.gauss_sum(np.zeros((1, 1)), np.array([[1.0], [2.0]]), 0.5, w=np.array([3.0, -1.0]), lib=lib)
    assert G[0] == pytest.approx(3 * np.exp(-0.5) - np.exp(-2.0), rel=1e-14)
    assert L[0] == pytest.approx(np.log(3 * np.exp(-0.5) - np.exp(-2.0)), rel=1e-14)
    # brute force with numpy (explicit differences, exp, weighted sum)
    rng = np.random.default_rng(15)
    X = rng.standard_normal((300, 7))
    C = rng.standard_normal((40, 7))
    w = rng.uniform(0.1, 2.0, 40)
    d = ((X[:, None, :] - C[None]) ** 2).sum(-1)
    G, L = oracle.gauss_sum(X, C, 0.3, w=w, lib=lib)
    np.testing.assert_allclose(G, (w[None] * np.exp(-0.3 * d)).sum(1), rtol=1e-12)
    # no weights means unit weights; a large beta is summed in log space
    G1, _ = oracle.gauss_sum(X, C, 0.3, lib=lib)
    np.testing.assert_allclose(G1, np.exp(-0.3 * d).sum(1), rtol=1e-12)
    _, L = oracle.gauss_sum(X, C, 400.0, w=w, lib=lib)
    e = np.log(w)[None] - 400.0 * d
    m = e.max(1)
    np.testing.assert_allclose(L, m + np.log(np.exp(e - m[:, None]).sum(1)), rtol=1e-12)
    # linearity in the weights; the sign parts combine as G(w+) - G(w-)
    w2 = rng.uniform(-1.0, 1.0, 40)
    Ga, _ = oracle.gauss_sum(X, C, 0.3, w=w, lib=lib)
    Gb, _ = oracle.gauss_sum(X, C, 0.3, w=w2, lib=lib)
    Gab, _ = oracle.gauss_sum(X, C, 0.3, w=w + w2, lib=lib)
    np.testing.assert_allclose(Gab, Ga + Gb, rtol=1e-10, atol=1e-13)
    # symmetry of the Gaussian kernel: u . (K v) = v . (K u) with C = X
    u, v = rng.standard_normal(300), rng.standard_normal(300)
    Kv, _ = oracle.gauss_sum(X, X, 0.3, w=v, lib=lib)
    Ku, _ = oracle.gauss_sum(X, X, 0.3, w=u, lib=lib)
    assert float(u @ Kv) == pytest.approx(float(v @ Ku), rel=1e-11)


def _kpp_python(X, K, u):
    """k-means++ with the same reproducible rule, written separately: pure
    Python sums in dimension order and Python integers for the weights."""
    import math
    N, D = X.shape
    rows = [list(map(float, r)) for r in X]
    def d2of(a, b):
        s = 0.0
        for j in range(D):
            t = a[j] - b[j]
            s += t * t
        return s
    cen = [min(int(math.floor(u[0] * N)), N - 1)]
    L = max(0, (N - 1).bit_length())
    d2 = None
    s = 0
    for t in range(1, K):
        c = rows[cen[-1]]
        d = [d2of(r, c) for r in rows]
        d2 = d if d2 is None else [min(a, b) for a, b in zip(d2, d)]
        if t == 1:
            m = max(d2)
            s = 61 - math.frexp(m)[1] - L if m > 0 else 0
        q = [int(math.floor(math.ldexp(v, s))) for v in d2]
        T = sum(q)
        if T == 0:
            cen.append(min(int(math.floor(u[t] * N)), N - 1))
            continue
        r = min(int(math.floor(u[t] * float(T))), T - 1)
        run = 0
        for i, qi in enumerate(q):
            run += qi
            if run > r:
                cen.append(i)
                break
    return cen


def pin_kmeanspp(lib):
    rng = np.random.default_rng(16)
    # one centre: point floor(u0 N)
    X = rng.standard_normal((100, 3))
    assert oracle.kmeanspp(X, 1, np.array([0.505]), lib).tolist() == [50]
    # two far clusters: the second centre lies in the other cluster
    X = np.concatenate([rng.standard_normal((50, 4)), 1000.0 + rng.standard_normal((50, 4))])
    for u1 in (0.01, 0.3, 0.999):  # cluster A holds about 1e-6 of the weight
        c = oracle.kmeanspp(X, 2, np.array([0.1, u1]), lib)
        assert c[0] == 10 and c[1] >= 50
    # the same rule written separately (Python sums and integers)
    X = rng.standard_normal((150, 5))
    u = rng.random(12)
    assert oracle.kmeanspp(X, 12, u, lib).tolist() == _kpp_python(X, 12, u)
    # probability proportional to D2: over a fine grid of u1 the second
    # centre is point i for a share q_i / T of the grid
    X = rng.standard_normal((40, 2))
    grid = (np.arange(20000) + 0.5) / 20000
    counts = np.zeros(40)
    for u1 in grid:
        counts[oracle.kmeanspp(X, 2, np.array([0.0, u1]), lib)[1]] += 1
    d2 = ((X - X[0]) ** 2).sum(1)
    np.testing.assert_allclose(counts / len(grid), d2 / d2.sum(), atol=2.0 / len(grid))
    # draws on a weight boundary: points 0, 1, 2 on a line, centre 0 first;
    # weights 0, 2^56, 2^58 (total 5 * 2^56); u1 = 0.2 gives r = 2^56, which
    # the running weight of point 1 reaches but does not exceed, so point 2;
    # u1 = 0 gives r = 0: the first point of positive weight, point 1
    X = np.array([[0.0], [1.0], [2.0]])
    assert oracle.kmeanspp(X, 2, np.array([0.0, 0.2]), lib).tolist() == [0, 2]
    assert oracle.kmeanspp(X, 2, np.array([0.0, 0.0]), lib).tolist() == [0, 1]
    # every point the same: all weights are zero, centre t is floor(u_t N)
    X = np.ones((30, 3))
    assert oracle.kmeanspp(X, 3, np.array([0.2, 0.5, 0.95]), lib).tolist() == [6, 15, 28]


def pin_planted(lib):
    rng = np.random.default_rng(8)
    K, D, per = 12, 6, 40
    centers = rng.uniform(-50, 50, (K, D))
    comp = np.repeat(np.arange(K), per)
    X = centers[comp] + 0.01 * rng.standard_normal((K * per, D))
    lab, _, _ = oracle.assign(X, centers, lib)
    assert np.array_equal(lab, comp)
    Cn, counts = oracle.update(X, lab, K, centers, lib)
    assert counts.tolist() == [per] * K
    for k in range(K):
        np.testing.assert_allclose(Cn[k], X[comp == k].mean(0), rtol=1e-12, atol=1e-12)


def pin_top2(lib):
    """The two nearest centroids: a hand-worked 1-D case with duplicated
    centroids (ties to the lowest index), K = 1, and brute force on integer
    data, where every distance is exact and a stable sort of each row's
    distances gives both labels."""
    X = np.array([[0.0], [1.0], [2.5], [10.0]])
    C = np.array([[0.0], [2.0], [3.0], [2.0]])
    l1, l2, d1, d2 = oracle.top2(X, C, lib)
    assert l1.tolist() == [0, 0, 1, 2]
    assert l2.tolist() == [1, 1, 2, 1]
    assert d1.tolist() == [0.0, 1.0, 0.25, 49.0]
    assert d2.tolist() == [4.0, 1.0, 0.25, 64.0]
    l1, l2, d1, d2 = oracle.top2(X, C[:1], lib)
    assert l1.tolist() == [0] * 4 and l2.tolist() == [-1] * 4 and np.all(np.isinf(d2))
    rng = np.random.default_rng(21)
    X = rng.integers(-3, 4, (300, 3)).astype(float)
    C = rng.integers(-3, 4, (25, 3)).astype(float)
    dm = ((X[:, None, :] - C[None, :, :]) ** 2).sum(-1)
    order = np.argsort(dm, axis=1, kind="stable")
    l1, l2, d1, d2 = oracle.top2(X, C, lib)
    rows = np.arange(300)
    assert np.array_equal(l1, order[:, 0]) and np.array_equal(l2, order[:, 1])
    assert np.array_equal(d1, dm[rows, order[:, 0]]) and np.array_equal(d2, dm[rows, order[:, 1]])


PINS = [pin_vq, pin_sklearn_step, pin_hand_1d, pin_ties, pin_k1_mean, pin_prefix_identity,
        pin_permutation, pin_empty_cluster, pin_invariants, pin_objective, pin_gauss, pin_kmeanspp,
        pin_planted, pin_top2]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(pin, oracle_lib):
    pin(oracle_lib)


def test_update_rejects_bad_label(oracle_lib):
    with pytest.raises(ValueError):
        oracle.update(np.zeros((3, 2)), np.array([0, 2, 1], np.int32), 2, np.zeros((2, 2)), oracle_lib)


# --------------------------------------------------------- screened assign --
def _screen_cases():
    rng = np.random.default_rng(14)
    yield "normal", rng.standard_normal((3000, 64)), rng.standard_normal((300, 64))
    X = rng.integers(-3, 4, (2000, 16)).astype(np.float64)
    C = rng.integers(-3, 4, (120, 16)).astype(np.float64)
    C[60:] = C[:60]  # every centroid twice: exact ties everywhere
    yield "integer ties", X, C
    import torch
    base = (rng.standard_normal((200, 128)) * 2 + 3).astype(np.float32)
    twin = torch.from_numpy(base).to(torch.bfloat16)
    bits = twin.view(torch.int16)
    bits[np.arange(200), rng.integers(0, 128, 200)] += 1
    Cb = np.concatenate([torch.from_numpy(base).to(torch.bfloat16).double().numpy(), twin.double().numpy()])
    Xb = torch.from_numpy(Cb[rng.integers(0, 400, 3000)] + 0.05 * rng.standard_normal((3000, 128))).to(
        torch.bfloat16).double().numpy()
    yield "one-ulp twins", Xb, Cb
    yield "large offset", 1000.0 + 0.01 * rng.standard_normal((2000, 32)), 1000.0 + 0.01 * rng.standard_normal((50, 32))
    yield "K = 1", rng.standard_normal((100, 8)), rng.standard_normal((1, 8))


@pytest.mark.parametrize("case", list(_screen_cases()), ids=lambda c: c[0])
def test_screened_assign_equals_plain(case, oracle_lib):
    """assign_screened must return exactly assign's labels and distances
    (brute force on the same inputs), including exact ties, near-ties one
    bf16 step apart and inputs whose expanded distances cancel badly."""
    _, X, C = case
    lab, mind, second = oracle.assign(X, C, oracle_lib)
    l2, m2, s2 = oracle.assign_screened(X, C, oracle_lib, block_elems=1 << 14)
    assert np.array_equal(lab, l2)
    assert np.array_equal(mind, m2)
    if C.shape[0] > 1:
        np.testing.assert_allclose(s2, second, rtol=1e-4, atol=1e-6 * float(np.abs(second).max()))


def test_screened_assign_margin_matters(oracle_lib):
    """With no rounding margin the screening decides near-ties in fp32 and
    disagrees with the plain oracle: the equality pin above would catch a
    screening that dropped its margin."""
    _, X, C = [c for c in _screen_cases() if c[0] == "one-ulp twins"][0]
    lab, _, _ = oracle.assign(X, C, oracle_lib)
    l0, _, _ = oracle.assign_screened(X, C, oracle_lib, margin=0.0)
    assert not np.array_equal(lab, l0)


# ------------------------------------------------------------- rounding ----
def test_bf16_rounding_nearest_even():
    import torch
    one = 1.0
    vals = np.array([one, one + 2 ** -8, one + 3 * 2 ** -8, -2.5, 3.0e38, 1e-40, 0.0, -0.0,
                     np.inf, -np.inf], np.float32)
    bits = oracle.bf16_bits_from_f32(vals)
    assert bits[0] == 0x3F80 and bits[1] == 0x3F80 and bits[2] == 0x3F82
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    assert np.array_equal(bits, ref)
    rng = np.random.default_rng(9)
    v = (rng.standard_normal(100000) * 10.0 ** rng.integers(-20, 20, 100000)).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    assert np.array_equal(oracle.bf16_bits_from_f32(v), ref)


def test_round_to_f16_matches_torch():
    import torch
    rng = np.random.default_rng(10)
    v = rng.standard_normal(50000) * 100
    ref = torch.from_numpy(v.astype(np.float32)).to(torch.float16).double().numpy()
    assert np.array_equal(oracle.round_to("f16", v), ref)


def test_lloyd_loop_against_independent_steps(oracle_lib):
    """oracle.lloyd against other implementations of each step: torch's
    round-to-nearest-even casts (fp32 master, then bf16), scipy's vq for the
    nearest centroid and numpy for the means (empty clusters keep the master)."""
    import torch
    from scipy.cluster.vq import vq
    rng = np.random.default_rng(11)
    X = torch.from_numpy(rng.standard_normal((300, 8))).to(torch.bfloat16).double().numpy()
    K = 5
    out = oracle.lloyd(X, X[:K], 3, "bf16", oracle_lib)
    C32 = torch.from_numpy(X[:K]).float()
    for _ in range(3):
        Cr = C32.to(torch.bfloat16).double().numpy()
        lab, dist = vq(X, Cr)
        nxt = C32.clone()
        for k in range(K):
            if (lab == k).any():
                nxt[k] = torch.from_numpy(X[lab == k].mean(0)).float()
        C32 = nxt
    assert np.array_equal(out["labels"], lab.astype(np.int32))
    np.testing.assert_allclose(out["C"], C32.double().numpy(), rtol=0, atol=2e-7)
    np.testing.assert_allclose(out["mindist"], dist ** 2, rtol=1e-12, atol=1e-12)


def test_lloyd_f64_matches_sklearn(oracle_lib):
    """Several fp64 Lloyd iterations against scikit-learn's Lloyd from the
    same initial centroids (a case without empty clusters)."""
    from sklearn.cluster import KMeans
    rng = np.random.default_rng(13)
    X = rng.standard_normal((800, 6)) + 4.0 * rng.integers(0, 3, (800, 1))
    C0 = X[:8].copy()
    out = oracle.lloyd(X, C0, 4, "f64", oracle_lib)
    assert out["counts"].min() > 0
    km = KMeans(n_clusters=8, init=C0, n_init=1, max_iter=4, algorithm="lloyd", tol=0.0).fit(X)
    np.testing.assert_allclose(out["C"], km.cluster_centers_, rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------- golden ---
def test_golden_fixture(oracle_lib):
    """Regression check, not a pin: the oracle against values an earlier build
    of itself wrote (tests/golden/make_golden.py, oracle only).  It catches an
    unintended change of the oracle's arithmetic; the pins above are what tie
    the oracle to the definition."""
    import json
    import workloads
    path = os.path.join(HERE, "golden", "tiny_f32_n512_k16.json")
    with open(path) as f:
        g = json.load(f)
    s = workloads.spec("tiny_f32", N=g["N"], K=g["K"], n_centers=g["n_centers"])
    w = workloads.make(s, seed=g["seed"])
    X = w.X.double().numpy()
    out = oracle.lloyd(X, w.C0.double().numpy(), g["iters"], "f32", oracle_lib)
    assert out["labels"].tolist() == g["labels"]
    assert out["counts"].tolist() == g["counts"]
    np.testing.assert_allclose(out["C"], np.array(g["C"]), rtol=0, atol=0)


# --------------------------------------------------------------- mutants ---
MUTANTS = [
    ("wrong sign", "double t = x[j] - c[j];", "double t = x[j] + c[j];"),
    ("no square", "s += t * t;", "s += fabs(t);"),
    ("dropped accumulation", "s += t * t;", "s = t * t;"),
    ("tie to highest index", "if (d < best) {", "if (d <= best) {"),
    ("centroid stride", "sqdist(x, C + (size_t)k * (size_t)D, D)", "sqdist(x, C + (size_t)k, D)"),
    ("runner-up not tracked", "runner = best;\n", "\n"),
    ("mean off by one", "out[j] = s[j] / (double)counts[k];", "out[j] = s[j] / (double)(counts[k] + 1);"),
    ("empty cluster zeroed", "for (int j = 0; j < D; ++j) out[j] = prev[j];",
     "for (int j = 0; j < D; ++j) out[j] = 0.0;"),
    ("objective on the wrong centroid", "C + (size_t)labels[i] * (size_t)D, D);",
     "C + (size_t)(labels[i] + 1 < 0 ? 0 : 0) * (size_t)D, D);"),
    ("objective drops the last point", "for (int64_t i = 0; i < N; ++i)\n        J +=",
     "for (int64_t i = 0; i + 1 < N; ++i)\n        J +="),
    ("objective not accumulated", "J += sqdist(", "J = sqdist("),
    ("Gauss exponent sign", "const double e = log(fabs(wk)) - beta *", "const double e = log(fabs(wk)) + beta *"),
    ("Gauss weight dropped", "const double e = log(fabs(wk)) - beta *", "const double e = 0.0 * log(fabs(wk)) - beta *"),
    ("Gauss negative part ignored", "if (G) G[i] = exp(lp) - exp(lq);", "if (G) G[i] = exp(lp);"),
    ("seeding weights by distance, not its square",
     "T += (int64_t)floor(ldexp(d2[i], s));", "T += (int64_t)floor(ldexp(sqrt(d2[i]), s));"),
    ("seeding without the running minimum", "d2[i] = (t == 1 || d < d2[i]) ? d : d2[i];", "d2[i] = d;"),
    ("seeding off by one in the draw", "if (run > r) break;", "if (run >= r) break;"),
    ("top-2 runner-up tie to the highest index", "} else if (d < runner || a2 < 0) {",
     "} else if (d <= runner || a2 < 0) {"),
    ("top-2 forgets the displaced best", "a2 = k == 0 ? -1 : a1;", "a2 = k;"),
    ("last point dropped", "for (int64_t i = 0; i < N; ++i) {\n        int32_t k = labels[i];",
     "for (int64_t i = 0; i + 1 < N; ++i) {\n        int32_t k = labels[i];"),
]


@pytest.mark.parametrize("mutant", MUTANTS, ids=lambda m: m[0])
def test_mutants_are_caught(mutant):
    name, old, new = mutant
    src = open(oracle._SRC).read()
    assert src.count(old) >= 1, name
    with tempfile.TemporaryDirectory() as td:
        path = os.path.join(td, "mutant.c")
        with open(path, "w") as f:
            f.write(src.replace(old, new))
        lib = oracle._bind(__import__("ctypes").CDLL(oracle.build(path, os.path.join(td, "m.so"), openmp=False)))
        caught = []
        for pin in PINS:
            try:
                pin(lib)
            except (AssertionError, ValueError):
                caught.append(pin.__name__)
        assert caught, f"mutant '{name}' passes every pin"
