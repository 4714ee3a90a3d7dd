"""Weighted Gauss sums (fk_gauss_sum) against the CPU oracle.

G[i] = sum_k w_k exp(-beta |x_i - c_k|^2) ("Fast Gauss Sums via Flash
Attention", abstract), and the matrix-free kernel-vector product Kv
(FlashDiffusion, Figure 4 caption: C = X, w = v).

Tolerance, from the arithmetic of the GPU path: the score of a centroid is an
fp32 sum of D + 16 terms (products, bias terms), each rounding adding at
most one fp32 unit of a magnitude below |x|^2 + |c|^2 + |ln w| / (2 beta),
so ln G moves by at most 2 beta (D + 16) 2^-24 times that; exp2/log2 and the
fp32 sum of K terms add (K + 16) 2^-23.  For signed weights, G = P - Q is
compared with that relative bound on P + Q (its cancellation is the input's,
not the method's)."""
import numpy as np
import pytest
import torch

import distance_argmin_flashassign_b200 as fk
import oracle
from tests.parity import TORCH_DT, f64, record

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
U = 2.0 ** -24


def _data(N, D, K, dtype, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    cen = torch.randn(max(K // 4, 1), D, generator=g) * scale
    X = (cen[torch.randint(0, cen.shape[0], (N,), generator=g)] + 0.5 * torch.randn(N, D, generator=g))
    C = (cen[torch.randint(0, cen.shape[0], (K,), generator=g)] + 0.5 * torch.randn(K, D, generator=g))
    return X.to(TORCH_DT[dtype]), C.to(TORCH_DT[dtype])


def _log_tol(X64, C64, beta, w, K):
    xn = (X64 ** 2).sum(1)
    cmax = float((C64 ** 2).sum(1).max())
    lw = 0.0 if w is None else float(np.abs(np.log(np.abs(w[w != 0]))).max())
    D = X64.shape[1]
    return 2 * beta * (D + 16) * U * (xn + cmax + lw / (2 * beta)) + (K + 16) * 2 * U


CASES = [  # (N, D, K, beta): several 256-centroid tiles, one tile, a ragged tail, one centroid
    (3000, 128, 700, 0.02), (5000, 64, 256, 0.05), (4097, 128, 2048, 0.01), (1000, 32, 1, 0.1), (2500, 96, 300, 1.0),
]


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c)))
def test_gauss_sum_matches_oracle(case, dtype):
    N, D, K, beta = case
    X, C = _data(N, D, K, dtype, seed=N + K)
    w = torch.rand(K, generator=torch.Generator().manual_seed(K)) + 0.1
    G, L = fk.fk_gauss_sum(X.to(DEV), C.to(DEV), beta, w=w.to(DEV))
    torch.cuda.synchronize()
    X64, C64, w64 = f64(X), f64(C), w.double().numpy()
    Go, Lo = oracle.gauss_sum(X64, C64, beta, w=w64)
    tol = _log_tol(X64, C64, beta, w64, K)
    err = np.abs(f64(L) - Lo)
    assert np.all(err <= tol), f"ln G off by {float((err / tol).max()):.3g} x tolerance"
    ok = Go > 1e-30  # G itself where fp32 holds it
    np.testing.assert_array_less(np.abs(f64(G)[ok] - Go[ok]), (np.expm1(tol) * Go + 1e-37)[ok] * 1.0001)
    record(f"gauss {N}x{D}x{K} beta {beta} {dtype}", N=N, max_log_err=float(err.max()), tol=float(tol.min()))


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_gauss_sum_tensor_and_cuda_core_paths(dtype):
    N, D, K, beta = 2000, 128, 500, 0.03
    X, C = _data(N, D, K, dtype, seed=4)
    outs = []
    try:
        for path in (1, 2):
            fk.fk_set_assign_path(path)
            outs.append(fk.fk_gauss_sum(X.to(DEV), C.to(DEV), beta)[1])
            torch.cuda.synchronize()
    finally:
        fk.fk_set_assign_path(0)
    X64, C64 = f64(X), f64(C)
    _, Lo = oracle.gauss_sum(X64, C64, beta)
    tol = _log_tol(X64, C64, beta, None, K)
    for L in outs:
        assert np.all(np.abs(f64(L) - Lo) <= tol)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_gauss_sum_signed_weights(dtype):
    N, D, K, beta = 3000, 64, 600, 0.05
    X, C = _data(N, D, K, dtype, seed=7)
    w = torch.randn(K, generator=torch.Generator().manual_seed(8))
    G, L = fk.fk_gauss_sum(X.to(DEV), C.to(DEV), beta, w=w.to(DEV), signed=True)
    torch.cuda.synchronize()
    X64, C64, w64 = f64(X), f64(C), w.double().numpy()
    Go, _ = oracle.gauss_sum(X64, C64, beta, w=w64)
    P, _ = oracle.gauss_sum(X64, C64, beta, w=np.maximum(w64, 0))
    Q, _ = oracle.gauss_sum(X64, C64, beta, w=np.maximum(-w64, 0))
    tol = _log_tol(X64, C64, beta, w64, K)
    err = np.abs(f64(G) - Go)
    assert np.all(err <= np.expm1(tol) * (P + Q) + 1e-37)
    pos = Go > 0
    assert np.all(np.isnan(f64(L)[~pos]) | (f64(G)[~pos] <= 0))


def test_kernel_vector_product():
    """Kv with the points as their own centres (C = X), signed v."""
    N, D, beta = 4000, 32, 0.2
    X, _ = _data(N, D, 8, "f16", seed=9)
    v = torch.randn(N, generator=torch.Generator().manual_seed(10))
    Xd = X.to(DEV)
    Kv, _ = fk.fk_gauss_sum(Xd, Xd, beta, w=v.to(DEV), signed=True)
    torch.cuda.synchronize()
    X64, v64 = f64(X), v.double().numpy()
    Ko, _ = oracle.gauss_sum(X64, X64, beta, w=v64)
    P, _ = oracle.gauss_sum(X64, X64, beta, w=np.maximum(v64, 0))
    Q, _ = oracle.gauss_sum(X64, X64, beta, w=np.maximum(-v64, 0))
    tol = _log_tol(X64, X64, beta, v64, N)
    assert np.all(np.abs(f64(Kv) - Ko) <= np.expm1(tol) * (P + Q))


def test_gauss_sum_argument_errors():
    X = torch.zeros(10, 8, device=DEV, dtype=torch.float16)
    with pytest.raises(fk.FKError):
        fk.fk_gauss_sum(X, X, 0.0)
    with pytest.raises(fk.FKError):
        fk.fk_gauss_sum(X, X, 1.0, signed=True)
