"""fk_update_noalloc, the centroid update for callers that cannot let a
library allocate device memory (code recorded under stream capture, engines
that hand all device memory to their own pool, allocation-free loops).

It must give what fk_update gives, on consecutive calls that share its one
static scratch array.  This file is collected last so that a run stopping at
the first failure has already run every other test; it also passes on its
own in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

import distance_argmin_flashassign_b200 as fk
import oracle
import workloads
from tests.parity import check_centroids, f64

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
DT = {torch.float32: fk.FK_F32, torch.float16: fk.FK_F16, torch.bfloat16: fk.FK_BF16}


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _noalloc(X, labels, C, counts):
    N, D = X.shape
    K = C.shape[0]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = fk.lib.fk_update_noalloc(_p(X), _p(labels), N, D, DT[X.dtype], K, _p(C), _p(counts), stream)
    assert st == fk.FK_OK, fk.lib.fk_last_error_message().decode()


CASES = [  # two different problems back to back on the same static scratch
    (200_000, 128, 1000, "zipf", "bf16"),
    (150_001, 64, 3000, "uniform", "f16"),
]


def test_no_alloc_update_matches_fk_update_on_two_calls_in_a_row():
    """The same kernels with the same arguments run on both entry points, so
    the results are bit-identical; the first case is also checked against
    the oracle's means."""
    for i, (N, D, K, kind, dtype) in enumerate(CASES):
        s = workloads.spec("tiny_f32", N=N, D=D, K=2, n_centers=64, dtype=dtype)
        Xc = workloads.make(s, seed=N).X
        X = Xc.to(DEV)
        labels_c = workloads.labels(N, K, seed=D, kind=kind)
        labels = labels_c.to(DEV)
        C0c = workloads.perturb(torch.zeros(K, D), 1.0, seed=K)
        C0 = C0c.to(DEV)
        C_ref, cnt_ref = C0.clone(), torch.empty(K, dtype=torch.int32, device=DEV)
        fk.fk_update(X, labels, C_ref, cnt_ref)
        C_na, cnt_na = C0.clone(), torch.full((K,), -1, dtype=torch.int32, device=DEV)
        _noalloc(X, labels, C_na, cnt_na)
        torch.cuda.synchronize()
        assert torch.equal(cnt_na, cnt_ref)
        assert torch.equal(C_na, C_ref)
        if i == 0:
            C_or, cnt_or = oracle.update(f64(Xc), labels_c.numpy(), K, f64(C0c))
            assert np.array_equal(cnt_na.cpu().numpy(), cnt_or)
            check_centroids(C_na, C_or)


def test_no_alloc_update_refuses_problems_beyond_its_scratch():
    p = ctypes.c_void_p(256)
    st = fk.lib.fk_update_noalloc(p, p, 3_000_000, 128, fk.FK_BF16, 1000, p, None, None)
    assert st == fk.FK_ERR_UNSUPPORTED
    assert "bytes of scratch" in fk.lib.fk_last_error_message().decode()
