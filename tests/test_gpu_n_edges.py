"""Degenerate and ragged inputs through the whole chain (Pipeline: permute ->
dense + entropy -> radius -> mask -> block-sparse attention -> inverse
permute), every output against the oracle, and empty problems.

  * one token (grid 1 x 1 x 1): the single key gets all the weight, so
    O = V, H = 0 (to rounding) and the one block pair is kept;
  * one column (1 x 37 x 1): every tile is truncated to 4 x 1;
  * wide rows whose width is no multiple of the tile (2 x 3 x 130), and a
    single frame with 16-token blocks (the eight-query-block tile kernel);
  * empty problems (no heads, no tokens): every call returns without error,
    the mask writes zero row offsets and nnz = 0, and nothing is reported."""
import numpy as np
import pytest
import torch

from entropy_adaptive_radius_b200 import tra, workloads
from tests.gpu_util import need_gpu, to64
from tests.test_gpu_k_chain import chain_every_element

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("grid,heads,d,block,vote,tau", [
    ((1, 1, 1), 2, 64, 16, 1, 0.5),
    ((1, 1, 1), 1, 128, 128, 1, 0.5),
    ((1, 37, 1), 2, 64, 16, 1, 0.3),
    ((1, 37, 1), 2, 128, 64, 2, 0.3),
    ((2, 3, 130), 2, 128, 64, 1, 0.02),
    ((1, 21, 19), 3, 64, 16, 3, 0.05),
])
def test_degenerate_grids_every_element(grid, heads, d, block, vote, tau):
    need_gpu()
    wl = workloads.Workload(name=f"edge_{grid}", F=grid[0], H=grid[1], W=grid[2], heads=heads,
                            d=d, dtype="bf16", block_q=block, block_k=block, gamma=0.4,
                            vote=vote, seed=31, tau=tau, sparse_calls=1)
    nnz, size = chain_every_element(wl)
    assert nnz > 0


def test_single_token_closed_form():
    """N = 1: softmax over one key is 1, so O = V exactly, H = 0 up to the
    rounding of the fused score offset (|x| ~ 1e-8 in the log2 domain), and
    LSE = scale * q . k."""
    need_gpu()
    heads, d = 3, 128
    g = torch.Generator().manual_seed(5)
    Q, K, V = (torch.randn(heads, 1, d, generator=g).to(torch.bfloat16).cuda() for _ in range(3))
    O_ = torch.empty_like(Q)
    H = torch.empty(heads, 1, dtype=torch.float32, device="cuda")
    L = torch.empty_like(H)
    tra.tra_dense_attn_entropy(Q, K, V, O_, H, L)
    torch.cuda.synchronize()
    assert tra.tra_get_device_error() == 0
    assert torch.equal(O_, V)
    assert float(H.abs().max()) <= 1e-6
    s = (to64(Q)[:, 0] * to64(K)[:, 0]).sum(axis=1) / np.sqrt(d)
    assert np.allclose(to64(L)[:, 0], s, atol=1e-3)


@pytest.mark.parametrize("heads,grid", [(0, (4, 8, 8)), (2, (0, 8, 8)), (2, (3, 0, 5))])
def test_empty_problems(heads, grid):
    need_gpu()
    F, Hh, W = grid
    N, d = F * Hh * W, 128
    bf = dict(dtype=torch.bfloat16, device="cuda")
    X = torch.zeros(heads, N, d, **bf)
    Q, K, V, Y, O_ = (torch.zeros(heads, N, d, **bf) for _ in range(5))
    H = torch.zeros(heads, N, dtype=torch.float32, device="cuda")
    r = torch.zeros_like(H)
    phi = torch.zeros(max(F, 1), dtype=torch.float32, device="cuda")
    nqb = -(-N // 128)
    row_ptr = torch.full((heads * (nqb + 1),), 7, dtype=torch.int32, device="cuda")
    col_idx = torch.zeros(1, dtype=torch.int32, device="cuda")
    nnz = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    ws = tra.workspace_tensor(max(1, tra.tra_workspace_size(heads, grid, 128, 128)))
    tra.tra_tile_major_permute(X, Y, grid)
    tra.tra_dense_attn_entropy(Q, K, V, O_, H)
    tra.tra_attn_entropy(Q, K, H)
    tra.tra_budget_radius(H, r, grid, 0.1, 0.3, phi_out=phi if F > 0 else None)
    tra.tra_build_block_mask(r, phi, grid, 128, 128, 1, row_ptr, col_idx, nnz, ws)
    tra.tra_block_sparse_attn(Q, K, V, O_, row_ptr, col_idx, 128, 128)
    tra.tra_inverse_permute(Y, X, grid)
    torch.cuda.synchronize()
    assert tra.tra_get_device_error() == 0
    assert int(nnz.item()) == 0
    assert torch.all(row_ptr == 0)
