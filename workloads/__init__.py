"""Seeded synthetic inputs for exact Lloyd k-means (Flash-KMeans workloads).

This module only draws random inputs.  It holds none of the method's
arithmetic: no distance, no argmin, no mean.  Both the CPU oracle (``oracle/``)
and the CUDA library are fed from here, so that they see identical values.

Flash-KMeans (arXiv 2603.09229, abstract) evaluates exact k-means on
"N points, K centroids" but publishes no dataset shapes; the five workloads
below are the synthetic stand-ins this project measures on:

====  ===================  ====================================================
 id    name                 recipe
====  ===================  ====================================================
 1     tiny_f32             N=32,768 D=32 fp32; 128 centres ~U[-1,1]^D, equal
                            weights, x = centre + 0.05 N(0,I); K=128, init =
                            first K rows; 5 iterations
 2     embed_f16            N=2^20 D=128 fp16; 1,024 centres = unit vectors,
                            x = centre + 0.15 N(0,I), then x <- x/|x|; K=1,024,
                            init = K distinct random rows; 20 iterations
 3     batched_bf16         B=32 problems, each N=32,768 D=128 bf16; token =
                            N(0,I) + one of 256 per-problem offsets ~0.5 N(0,I);
                            K=256 per problem, init = first K rows; 10 iters
 4     zipf_bf16            N=2^23 D=128 bf16; 65,536 centres ~2 N(0,I), centre
                            k (rank k+1) drawn with mass ~ (k+1)^-1.2, x =
                            centre + 0.3 N(0,I); K=65,536, init = first K rows;
                            10 iterations
 5     ooc_f16              N=1e9 D=128 fp16 in pinned host memory; 8,192
                            centres ~U[-1,1]^D, sigma 0.1; K=8,192, init =
                            first K rows; 3 iterations; 64 Mi-row chunks
====  ===================  ====================================================

Randomness: torch generators (Philox on CUDA, MT19937 on CPU), one generator
per (seed, workload id, stream tag, row block).  Values are drawn in fp32 and
rounded once to the workload dtype with round-to-nearest-even.  The same call
on a different device gives different (but equally seeded) values; a test
always compares the two implementations on one generated tensor.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

BLOCK_ROWS = 1 << 20  # rows per independently seeded generation block

DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@dataclasses.dataclass(frozen=True)
class Spec:
    cfg: int
    name: str
    N: int
    D: int
    K: int
    dtype: str
    iters: int
    B: int = 1
    n_centers: int = 0
    chunk_rows: int = 0

    def replace(self, **kw) -> "Spec":
        return dataclasses.replace(self, **kw)

    @property
    def bytes_per_elem(self) -> int:
        return 4 if self.dtype == "f32" else 2


SPECS = {
    "tiny_f32": Spec(1, "tiny_f32", 32768, 32, 128, "f32", 5, 1, 128),
    "embed_f16": Spec(2, "embed_f16", 1 << 20, 128, 1024, "f16", 20, 1, 1024),
    "batched_bf16": Spec(3, "batched_bf16", 32768, 128, 256, "bf16", 10, 32, 256),
    "zipf_bf16": Spec(4, "zipf_bf16", 1 << 23, 128, 65536, "bf16", 10, 1, 65536),
    "ooc_f16": Spec(5, "ooc_f16", 10**9, 128, 8192, "f16", 3, 1, 8192, 64 << 20),
}


def spec(name: str, **overrides) -> Spec:
    s = SPECS[name]
    if overrides:
        s = s.replace(**overrides)
    return s


def _seed(seed: int, cfg: int, tag: int, block: int = 0) -> int:
    """Mix (seed, workload, stream tag, block) into one 63-bit generator seed."""
    h = 0x9E3779B97F4A7C15
    for v in (seed, cfg, tag, block):
        h ^= (v + 0x632BE59BD9B4E019 + ((h << 6) & 0xFFFFFFFFFFFFFFFF) + (h >> 2)) & 0xFFFFFFFFFFFFFFFF
        h = (h * 0xBF58476D1CE4E5B9) & 0xFFFFFFFFFFFFFFFF
    return h & 0x7FFFFFFFFFFFFFFF


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


_TAG_CENTERS, _TAG_ROWS, _TAG_INIT, _TAG_LABELS = 1, 2, 3, 4


def centers(s: Spec, seed: int = 0, device="cpu", batch: int = 0) -> torch.Tensor:
    """Mixture centres (fp32) of workload ``s``; ``batch`` selects a problem."""
    g = _gen(device, _seed(seed, s.cfg, _TAG_CENTERS, batch))
    M, D = s.n_centers, s.D
    if s.cfg in (1, 5):
        return torch.rand((M, D), generator=g, device=device) * 2.0 - 1.0
    if s.cfg == 2:
        c = torch.randn((M, D), generator=g, device=device)
        return c / c.norm(dim=1, keepdim=True)
    if s.cfg == 3:
        return 0.5 * torch.randn((M, D), generator=g, device=device)
    if s.cfg == 4:
        return 2.0 * torch.randn((M, D), generator=g, device=device)
    raise ValueError(s.cfg)


def _zipf_cdf(M: int, device) -> torch.Tensor:
    k = torch.arange(1, M + 1, dtype=torch.float64, device=device)
    p = k.pow(-1.2)
    cdf = torch.cumsum(p / p.sum(), 0)
    cdf[-1] = 1.0
    return cdf


def _block_rows(s: Spec, cen: torch.Tensor, seed: int, block: int, n: int, device,
                batch: int = 0) -> torch.Tensor:
    g = _gen(device, _seed(seed, s.cfg, _TAG_ROWS, block + (batch << 32)))
    M = cen.shape[0]
    if s.cfg == 4:
        u = torch.rand((n,), generator=g, device=device, dtype=torch.float64)
        comp = torch.searchsorted(_zipf_cdf(M, device), u).clamp_(max=M - 1)
    else:
        comp = torch.randint(0, M, (n,), generator=g, device=device)
    noise = torch.randn((n, s.D), generator=g, device=device)
    sigma = {1: 0.05, 2: 0.15, 3: 1.0, 4: 0.3, 5: 0.1}[s.cfg]
    x = cen[comp] + sigma * noise
    if s.cfg == 2:
        x = x / x.norm(dim=1, keepdim=True)
    return x


def rows(s: Spec, start: int, stop: int, seed: int = 0, device="cpu",
         batch: int = 0, cen: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Rows [start, stop) of problem ``batch`` of ``s``, rounded to s.dtype."""
    if cen is None:
        cen = centers(s, seed, device, batch)
    out = []
    b0, b1 = start // BLOCK_ROWS, (max(stop, start + 1) - 1) // BLOCK_ROWS
    for b in range(b0, b1 + 1):
        lo = b * BLOCK_ROWS
        n_blk = min(BLOCK_ROWS, s.N - lo)
        blk = _block_rows(s, cen, seed, b, n_blk, device, batch)
        a, z = max(start, lo) - lo, min(stop, lo + n_blk) - lo
        out.append(blk[a:z])
    x = torch.cat(out, 0) if len(out) > 1 else out[0]
    return x.to(DTYPES[s.dtype]).contiguous()


def init_indices(s: Spec, seed: int = 0, device="cpu") -> torch.Tensor:
    """Row indices of the initial centroids (first K rows, or K distinct random rows)."""
    if s.cfg == 2:
        g = _gen(device, _seed(seed, s.cfg, _TAG_INIT))
        return torch.randperm(s.N, generator=g, device=device)[: s.K]
    return torch.arange(s.K, device=device)


@dataclasses.dataclass
class Workload:
    spec: Spec
    X: torch.Tensor        # [N, D] or [B, N, D], dtype of spec
    C0: torch.Tensor       # [K, D] or [B, K, D], fp32 (exact copies of rows of X)
    seed: int


def make(name_or_spec, seed: int = 0, device="cpu", **overrides) -> Workload:
    """Generate the whole input of a workload (X resident on ``device``)."""
    s = name_or_spec if isinstance(name_or_spec, Spec) else spec(name_or_spec, **overrides)
    if s.K > s.N:
        raise ValueError("K must not exceed N")
    xs, cs = [], []
    for b in range(s.B):
        cen = centers(s, seed, device, b)
        x = rows(s, 0, s.N, seed, device, b, cen)
        idx = init_indices(s, seed, device)
        xs.append(x)
        cs.append(x[idx].float())
    if s.B == 1:
        return Workload(s, xs[0], cs[0], seed)
    return Workload(s, torch.stack(xs), torch.stack(cs), seed)


def labels(N: int, K: int, seed: int = 0, kind: str = "uniform", device="cpu",
           s: float = 1.2) -> torch.Tensor:
    """Random cluster ids in [0, K) (int32) for update-only tests.

    ``kind``: "uniform", "zipf" (mass ~ (k+1)^-s, cluster 0 hottest), "one"
    (every point in cluster K-1), "sparse" (only every 7th cluster is used).
    """
    g = _gen(device, _seed(seed, 99, _TAG_LABELS, K))
    if kind == "uniform":
        lab = torch.randint(0, K, (N,), generator=g, device=device)
    elif kind == "zipf":
        k = torch.arange(1, K + 1, dtype=torch.float64, device=device)
        cdf = torch.cumsum(k.pow(-s) / k.pow(-s).sum(), 0)
        cdf[-1] = 1.0
        u = torch.rand((N,), generator=g, device=device, dtype=torch.float64)
        lab = torch.searchsorted(cdf, u).clamp_(max=K - 1)
    elif kind == "one":
        lab = torch.full((N,), K - 1, device=device)
    elif kind == "sparse":
        used = torch.arange(0, K, 7, device=device)
        lab = used[torch.randint(0, used.numel(), (N,), generator=g, device=device)]
    else:
        raise ValueError(kind)
    return lab.to(torch.int32)


def perturb(C: torch.Tensor, scale: float, seed: int = 0) -> torch.Tensor:
    """Seeded noise added to fp32 centroids (mid-trajectory-like starting points)."""
    g = _gen(C.device, _seed(seed, 98, _TAG_INIT, C.numel()))
    return (C + scale * torch.randn(C.shape, generator=g, device=C.device)).float()


def total_rows(s: Spec) -> int:
    return s.N * s.B


def n_blocks(s: Spec) -> int:
    return math.ceil(s.N / BLOCK_ROWS)
