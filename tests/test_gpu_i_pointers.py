"""Entry points refuse memory that is not on the current device.

A host pointer handed to a kernel would fault the GPU, so every C entry point
asks the CUDA runtime where each of its pointers lives and returns
TRA_ERR_INVALID_ARGUMENT (1) before any launch when one is host memory
(pageable or pinned).  The Python binding refuses CPU tensors before the C
call.  Each C-level case first confirms, with a host-only runtime query, that
the runtime classes the pointer as host memory, so the call under test takes
the refusing branch."""
import ctypes

import numpy as np
import pytest
import torch

from entropy_adaptive_radius_b200 import tra
from tests.gpu_util import need_gpu

pytestmark = pytest.mark.gpu

GRID = (2, 8, 8)
TILE = (1, 4, 4)


def host_kind(ptr: int):
    from cuda.bindings import runtime as cudart
    err, attr = cudart.cudaPointerGetAttributes(ptr)
    if err != cudart.cudaError_t.cudaSuccess:
        return None
    t = attr.type
    if t == cudart.cudaMemoryType.cudaMemoryTypeUnregistered:
        return "pageable"
    if t == cudart.cudaMemoryType.cudaMemoryTypeHost:
        return "pinned"
    return None


def c_radial(r_ptr, phi_ptr, heads):
    return tra.lib().tra_radial_radius(r_ptr, phi_ptr, heads, tra._grid(GRID), tra._tile(TILE),
                                       ctypes.c_float(2.0), 0, tra._stream(None))


def test_binding_refuses_cpu_tensors():
    need_gpu()
    N = GRID[0] * GRID[1] * GRID[2]
    with pytest.raises(ValueError):
        tra.tra_radial_radius(torch.empty(1, N), GRID, 2.0)
    Q = torch.zeros(1, 128, 64, dtype=torch.bfloat16)
    O = torch.empty(1, 128, 64, dtype=torch.bfloat16, device="cuda")
    H = torch.empty(1, 128, device="cuda")
    with pytest.raises(ValueError):
        tra.tra_dense_attn_entropy(Q, Q.cuda(), Q.cuda(), O, H)


@pytest.mark.parametrize("kind", ["pageable", "pinned"])
def test_c_entry_points_refuse_host_pointers(kind):
    need_gpu()
    N = GRID[0] * GRID[1] * GRID[2]
    if kind == "pageable":
        host = np.zeros(N, np.float32)
        ptr = host.ctypes.data
    else:
        host = torch.zeros(N, dtype=torch.float32).pin_memory()
        ptr = host.data_ptr()
    if host_kind(ptr) != kind:
        pytest.skip("the runtime does not class this buffer as host memory")
    r = torch.full((1, N), -1.0, device="cuda")
    phi = torch.full((GRID[0],), -1.0, device="cuda")
    # host r, host phi_out, and a host pointer among device ones
    assert c_radial(ctypes.c_void_p(ptr), None, 1) == 1
    assert c_radial(None, ctypes.c_void_p(ptr), 0) == 1
    assert c_radial(ctypes.c_void_p(r.data_ptr()), ctypes.c_void_p(ptr), 1) == 1
    torch.cuda.synchronize()
    assert bool((r == -1.0).all()) and bool((phi == -1.0).all())   # nothing was launched
    # the same call on device memory runs
    assert c_radial(ctypes.c_void_p(r.data_ptr()), ctypes.c_void_p(phi.data_ptr()), 1) == 0
    torch.cuda.synchronize()
    assert bool((r == 2.0).all())
    assert tra.tra_get_device_error() == 0
