"""k-means++ seeding on the GPU (fk_seed_kmeanspp) against the oracle's draw
with the same uniforms: the chosen indices must be identical (the distances
are the same fp64 sums and the weights integers, so every draw is)."""
import numpy as np
import pytest
import torch

import distance_argmin_flashassign_b200 as fk
import oracle
import workloads
from tests.parity import TORCH_DT, f64

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


# Row widths cover every warp layout of the 16-byte path (1 to 32 lanes per
# row, up to 8 vectors per lane) and the two fallbacks (rows not a multiple
# of 16 bytes, staged in shared memory or read directly).
CASES = [(5000, 32, 50, "f32"), (20000, 128, 100, "f16"), (3001, 64, 64, "bf16"), (257, 8, 40, "f16"),
         (1000, 100, 1, "f32"), (2048, 4, 25, "f32"), (3000, 16, 25, "f16"), (3000, 16, 25, "f32"),
         (3000, 512, 30, "bf16"), (1500, 1000, 10, "f16"), (2000, 1024, 12, "f32"), (4000, 100, 30, "f16"),
         (999, 3, 20, "bf16"), (65536, 128, 256, "f16")]


@pytest.mark.parametrize("N,D,K,dtype", CASES, ids=lambda v: str(v))
def test_seeding_matches_oracle(N, D, K, dtype):
    s = workloads.spec("embed_f16", N=N, D=D, K=2, n_centers=32, dtype=dtype)
    X = workloads.make(s, seed=N + K).X
    u = np.random.default_rng(K).random(K)
    c = fk.fk_seed_kmeanspp(X.to(DEV), K, u)
    assert c.cpu().numpy().tolist() == oracle.kmeanspp(f64(X), K, u).tolist()


def test_seeding_unaligned_rows():
    """X starting 2 bytes past an aligned address takes the unstaged path."""
    s = workloads.spec("embed_f16", N=3000, D=64, K=2, n_centers=32, dtype="f16")
    X = workloads.make(s, seed=5).X
    base = torch.empty(X.numel() + 1, dtype=X.dtype, device=DEV)
    Xu = base[1:].view(X.shape)
    Xu.copy_(X.to(DEV))
    assert Xu.data_ptr() % 4 == 2
    u = np.random.default_rng(6).random(40)
    assert fk.fk_seed_kmeanspp(Xu, 40, u).cpu().tolist() == oracle.kmeanspp(f64(X), 40, u).tolist()


def test_seeding_boundary_draw_and_duplicates():
    X = torch.tensor([[0.0], [1.0], [2.0]], device=DEV)
    assert fk.fk_seed_kmeanspp(X, 2, [0.0, 0.2]).cpu().tolist() == [0, 2]
    # many duplicated points: the weights run out, then centre t is floor(u_t N)
    g = torch.Generator().manual_seed(3)
    base = torch.randn(5, 16, generator=g)
    X = base[torch.randint(0, 5, (4000,), generator=g)].to(torch.bfloat16)
    u = np.random.default_rng(4).random(12)
    assert fk.fk_seed_kmeanspp(X.to(DEV), 12, u).cpu().tolist() == oracle.kmeanspp(f64(X), 12, u).tolist()


def test_seeding_argument_errors():
    X = torch.zeros(10, 4, device=DEV)
    with pytest.raises(fk.FKError):
        fk.fk_seed_kmeanspp(X, 2, [0.5, 1.0])
