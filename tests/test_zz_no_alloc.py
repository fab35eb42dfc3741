"""The allocation-free block-mask entry point.

tra_build_block_mask_noalloc serves callers that cannot allocate or pass
scratch memory (a plugin that only receives its tensors from a framework that
owns all device memory, or a caller that must not allocate mid-run): it uses
a buffer built into the library instead of a caller workspace.  Its result
must be the same CSR as tra_build_block_mask's, call after call, even though
every call reuses (and leaves data in) that one buffer.

This file is collected last so that, if it fails, a run that stops at the
first failure has already run every other test."""
import ctypes
import math

import numpy as np
import pytest
import torch

from entropy_adaptive_radius_b200 import inputs, tra, workloads
from oracle import tra_oracle as O
from tests.gpu_util import need_gpu

pytestmark = pytest.mark.gpu


def _csr_buffers(heads, nqb, nkb):
    row_ptr = torch.full((heads * (nqb + 1),), -3, dtype=torch.int32, device="cuda")
    col_idx = torch.full((heads * nqb * nkb,), -3, dtype=torch.int32, device="cuda")
    nnz = torch.full((1,), -3, dtype=torch.int32, device="cuda")
    return row_ptr, col_idx, nnz


def _radii(wl, heads, tau, seed):
    N = wl.N
    grid = (wl.F, wl.H, wl.W)
    Hs = inputs.synthetic_entropy(heads, N, seed, math.log(N) - 2.0, math.log(N))
    pi = O.tile_major_order(*grid, wl.tile)
    t_tm = O.token_coords(*grid)[pi][:, 2]
    r = np.stack([O.radius(Hs[h], t_tm, tau, wl.gamma, wl.F, N) for h in range(heads)])
    return torch.from_numpy(r.astype(np.float32)).cuda()


def _both(wl, heads, r, phi, vote):
    grid = (wl.F, wl.H, wl.W)
    bq, bk = wl.block_q, wl.block_k
    nqb, nkb = -(-wl.N // bq), -(-wl.N // bk)
    ref = _csr_buffers(heads, nqb, nkb)
    ws = tra.workspace_tensor(tra.tra_mask_workspace_size(heads, grid, bq, bk, wl.tile))
    tra.tra_build_block_mask(r, phi, grid, bq, bk, vote, *ref, ws, wl.tile)
    got = _csr_buffers(heads, nqb, nkb)
    tra.tra_build_block_mask_noalloc(r, phi, grid, bq, bk, vote, *got, wl.tile)
    torch.cuda.synchronize()
    assert tra.tra_get_device_error() == 0
    n_ref, n_got = int(ref[2].item()), int(got[2].item())
    assert n_got == n_ref
    assert torch.equal(got[0], ref[0])
    assert torch.equal(got[1][:n_got], ref[1][:n_ref])
    return n_got


@pytest.mark.parametrize("wl", [workloads.WAN14B, workloads.WAN13B, workloads.TINY],
                         ids=lambda w: w.name)
def test_noalloc_matches_workspace_entry_point_twice(wl):
    """Two calls in a row with different radii and vote thresholds: each
    must equal the workspace entry point's CSR (stale buffer contents from the
    first call must not leak into the second)."""
    need_gpu()
    heads = wl.heads
    phi = torch.from_numpy(O.phi(np.arange(wl.F), wl.gamma).astype(np.float32)).cuda()
    r1 = _radii(wl, heads, 0.05, seed=11)
    r2 = _radii(wl, heads, 0.5, seed=12)
    n1 = _both(wl, heads, r1, phi, 1)
    n2 = _both(wl, heads, r2, phi, 4 if wl.block_q >= 64 else 2)
    assert n1 > 0 and n2 > 0 and n1 != n2


def test_noalloc_refuses_problems_beyond_its_buffer():
    need_gpu()
    wl = workloads.WAN14B
    grid = tra.Grid(wl.F, wl.H, wl.W)
    tile = tra.Tile(*wl.tile)
    heads = 200
    need = tra.tra_mask_workspace_size(heads, (wl.F, wl.H, wl.W), 128, 128, wl.tile)
    assert need > tra.MASK_STATIC_SCRATCH_BYTES
    buf = torch.empty(64, dtype=torch.int32, device="cuda")
    p = ctypes.c_void_p(buf.data_ptr())
    s = tra.lib().tra_build_block_mask_noalloc(p, p, heads, grid, tile, 128, 128, 1, p, p, 1, p,
                                              ctypes.c_void_p(0))
    assert s == 3   # TRA_ERR_WORKSPACE, nothing launched
    with pytest.raises(tra.TraError):
        tra._check("tra_build_block_mask_noalloc", s)


def test_noalloc_empty_problem_follows_the_workspace_entry_point():
    """N = 0 (a grid with no frames): both entry points write zero row
    offsets and nnz = 0, and check only those two outputs, so an unused radius
    pointer that is not device memory is accepted by both."""
    need_gpu()
    heads = 3
    grid = tra.Grid(0, 45, 80)
    tile = tra.Tile(1, 4, 4)
    host_r = (ctypes.c_float * 4)()
    results = []
    for noalloc in (False, True):
        row_ptr = torch.full((heads,), 7, dtype=torch.int32, device="cuda")
        nnz = torch.full((1,), 7, dtype=torch.int32, device="cuda")
        rp, nz = ctypes.c_void_p(row_ptr.data_ptr()), ctypes.c_void_p(nnz.data_ptr())
        r = ctypes.cast(host_r, ctypes.c_void_p)
        if noalloc:
            s = tra.lib().tra_build_block_mask_noalloc(r, None, heads, grid, tile, 128, 128, 1, rp,
                                                      None, 0, nz, ctypes.c_void_p(0))
        else:
            s = tra.lib().tra_build_block_mask_ex(r, None, heads, grid, tile, 128, 128, 1, 0, rp,
                                                 None, 0, nz, None, 0, ctypes.c_void_p(0))
        torch.cuda.synchronize()
        results.append((s, row_ptr.cpu().tolist(), int(nnz.item())))
    assert results[0] == results[1] == (0, [0] * heads, 0)
