"""Failure paths of the out-of-core driver and the scratch cache, made on the
host (fk_debug_inject): a chunk copy that is not issued, a scratch allocation
that fails.  Nothing faults, traps or waits forever on the device.  After
each failure the call has returned with the right status, no device error is
pending, and the next call gives the same result as an undisturbed one."""
import numpy as np
import pytest
import torch

import distance_argmin_flashassign_b200 as fk
import oracle
import workloads
from tests.parity import check_centroids, f64

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
N, D, K, CHUNK = 30000, 64, 200, 7000  # 5 chunks per iteration


@pytest.fixture(scope="module")
def ooc_case():
    s = workloads.spec("ooc_f16", N=N, D=D, K=K, n_centers=K)
    w = workloads.make(s, seed=21)
    Xh = w.X.pin_memory()
    Ch = w.C0.clone()
    lab = torch.empty(N, dtype=torch.int32).pin_memory()
    fk.fk_lloyd_ooc(Xh, Ch, 2, CHUNK, lab)  # the undisturbed result
    return w, Xh, Ch, lab


def _run(Xh, C0):
    Ch = C0.clone()
    lab = torch.empty(N, dtype=torch.int32).pin_memory()
    fk.fk_lloyd_ooc(Xh, Ch, 2, CHUNK, lab)
    return Ch, lab


@pytest.mark.parametrize("at", [0, 3, 7])  # first chunk, mid first iteration, mid second iteration
def test_chunk_copy_failure(ooc_case, at):
    w, Xh, C_ref, lab_ref = ooc_case
    fk.fk_debug_inject(fk.FK_INJECT_CHUNK_COPY, at)
    Ch = w.C0.clone()
    with pytest.raises(fk.FKError) as e:
        fk.fk_lloyd_ooc(Xh, Ch, 2, CHUNK)
    assert e.value.status == fk.FK_ERR_HOST_IO
    assert "injected" in str(e.value)
    assert torch.cuda.current_stream().query()  # the call left nothing running
    fk.fk_sync()  # no device-side error pending
    C2, lab2 = _run(Xh, w.C0)
    assert torch.equal(C2, C_ref) and torch.equal(lab2, lab_ref)


def test_scratch_allocation_failure(ooc_case):
    w, Xh, C_ref, lab_ref = ooc_case
    fk.fk_release_workspace()  # the next call must grow the cache
    fk.fk_debug_inject(fk.FK_INJECT_SCRATCH_ALLOC)
    Ch = w.C0.clone()
    with pytest.raises(fk.FKError) as e:
        fk.fk_lloyd_ooc(Xh, Ch, 2, CHUNK)
    assert e.value.status == fk.FK_ERR_OOM
    assert torch.equal(Ch, w.C0)  # nothing was written
    fk.fk_sync()
    C2, lab2 = _run(Xh, w.C0)
    assert torch.equal(C2, C_ref) and torch.equal(lab2, lab_ref)
    out = oracle.lloyd(f64(w.X), f64(w.C0), 2, "f16")
    check_centroids(C2, out["C"])


def test_update_scratch_allocation_failure():
    X = torch.randn(50000, 128, device=DEV, dtype=torch.bfloat16)
    labels = workloads.labels(50000, 300, seed=3).to(DEV)
    C_ref = torch.zeros(300, 128, device=DEV)
    fk.fk_update(X, labels, C_ref)
    fk.fk_release_workspace()
    fk.fk_debug_inject(fk.FK_INJECT_SCRATCH_ALLOC)
    C = torch.zeros(300, 128, device=DEV)
    with pytest.raises(fk.FKError) as e:
        fk.fk_update(X, labels, C)
    assert e.value.status == fk.FK_ERR_OOM
    fk.fk_update(X, labels, C)
    fk.fk_sync()
    assert torch.equal(C, C_ref)
