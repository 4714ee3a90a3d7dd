"""Comparison rules between the CUDA library and the CPU oracle.

Acceptance (Flash-KMeans is exact k-means, arXiv 2603.09229 abstract; the
tolerances are the project's stated bar):

* labels are bit-exact, except at near-ties: a point may carry another label
  than the oracle's only if, in fp64, its distance to the GPU's centroid
  exceeds the minimum by at most ``band * (|x|^2 + |c_best|^2)`` with
  band = 1e-4 for fp32 inputs and 1e-2 for fp16/bf16 inputs (c_best is the
  oracle's centroid); and such points are at most 0.01 % of N;
* centroids within 1e-4 relative L2 (Frobenius) of the oracle's;
* counts (integers) exact.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

BAND = {"f32": 1e-4, "f16": 1e-2, "bf16": 1e-2}
MINDIST_TOL = {"f32": 1e-5, "f16": 1e-3, "bf16": 1e-3}
MAX_MISMATCH_FRAC = 1e-4
CENTROID_REL_L2 = 1e-4

TORCH_DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def dtag(t: torch.Tensor) -> str:
    return {torch.float32: "f32", torch.float16: "f16", torch.bfloat16: "bf16"}[t.dtype]


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def check_labels(X64: np.ndarray, C64: np.ndarray, gpu_labels, dtype: str, gpu_mindist=None,
                 exact: bool = False, max_frac: float = MAX_MISMATCH_FRAC):
    """Compare GPU labels (and mindist) with the oracle on the same rounded inputs.

    Returns a dict of statistics; raises AssertionError when the bar is missed."""
    gl = np.asarray(gpu_labels.cpu() if torch.is_tensor(gpu_labels) else gpu_labels).astype(np.int64)
    lab, mind, second = oracle.assign(X64, C64)
    N = len(lab)
    assert gl.min(initial=0) >= 0 and gl.max(initial=0) < C64.shape[0], "label out of range"
    mism = np.nonzero(gl != lab)[0]
    stats = {"N": N, "mismatch": int(len(mism)), "near_tie_points": 0}
    scale = (X64 ** 2).sum(1) + (C64[lab] ** 2).sum(1)
    gap = second - mind
    stats["near_tie_points"] = int((gap <= BAND[dtype] * scale).sum())
    if exact:
        assert len(mism) == 0, f"{len(mism)} label mismatches where bit-exactness is required: {mism[:10]}"
    if len(mism):
        d_gpu = ((X64[mism] - C64[gl[mism]]) ** 2).sum(1)
        excess = d_gpu - mind[mism]
        bad = excess > BAND[dtype] * scale[mism]
        assert not bad.any(), (f"{int(bad.sum())} mismatches outside the near-tie band, e.g. row "
                               f"{mism[bad][0]}: excess {excess[bad][0]:.3g} vs band "
                               f"{BAND[dtype] * scale[mism][bad][0]:.3g}")
        assert len(mism) <= max(max_frac * N, 0), f"{len(mism)} near-tie mismatches > {max_frac:.2%} of {N}"
    if gpu_mindist is not None:
        gm = np.asarray(gpu_mindist.cpu() if torch.is_tensor(gpu_mindist) else gpu_mindist, np.float64)
        d_at = ((X64 - C64[gl]) ** 2).sum(1)
        err = np.abs(gm - d_at)
        tol = MINDIST_TOL[dtype] * ((X64 ** 2).sum(1) + (C64[gl] ** 2).sum(1)) + 1e-30
        assert np.all(err <= tol), f"mindist off by {float((err / tol).max()):.3g} x tolerance"
        assert np.all(gm >= 0)
    return stats


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def check_centroids(C_gpu, C_or, tol: float = CENTROID_REL_L2):
    r = rel_l2(f64(C_gpu) if torch.is_tensor(C_gpu) else C_gpu, C_or)
    assert r <= tol, f"centroid rel-L2 {r:.3g} > {tol}"
    return r
