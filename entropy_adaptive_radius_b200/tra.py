"""ctypes binding of libtra.so, the C ABI declared in include/tra.h.

Argument marshalling only: every function takes torch tensors that already
live on the GPU, passes their device pointers, sizes and the current CUDA
stream to the C entry point of the same name, and raises TraError when the
call returns a non-zero status.  Nothing here computes any part of the
method, and there is no fallback: if libtra.so is missing the first call
raises.
"""
import ctypes
import math
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# The library this binding loads: libtra.so beside this file, or the build
# that TRA_LIBRARY names (the checked build, libtra_check.so, in the tests).
LIB_PATH = os.environ.get("TRA_LIBRARY") or os.path.join(_HERE, "libtra.so")
CHECK_LIB_PATH = os.path.join(_HERE, "libtra_check.so")

TRA_BF16, TRA_F32 = 0, 1
TRA_METRIC_DISK, TRA_METRIC_LINE = 0, 1
TRA_BUDGET_ENTROPY, TRA_BUDGET_SHARED = 0, 1
METRICS = {"disk": TRA_METRIC_DISK, "line": TRA_METRIC_LINE}
BUDGETS = {"entropy": TRA_BUDGET_ENTROPY, "shared": TRA_BUDGET_SHARED}
STATUS = {0: "TRA_OK", 1: "TRA_ERR_INVALID_ARGUMENT", 2: "TRA_ERR_UNSUPPORTED",
          3: "TRA_ERR_WORKSPACE", 4: "TRA_ERR_CAPACITY", 5: "TRA_ERR_CUDA",
          6: "TRA_ERR_DEVICE", 7: "TRA_ERR_TIMEOUT", 8: "TRA_ERR_BAD_INPUT"}


class TraError(RuntimeError):
    def __init__(self, fn: str, status: int, text: str):
        super().__init__(f"{fn}: {STATUS.get(status, status)} ({text})")
        self.status = status


class Grid(ctypes.Structure):
    _fields_ = [("F", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int)]


class Tile(ctypes.Structure):
    _fields_ = [("t", ctypes.c_int), ("y", ctypes.c_int), ("x", ctypes.c_int)]


_lib = None
_c_int, _c_ll, _c_size, _c_float, _vp = (ctypes.c_int, ctypes.c_longlong, ctypes.c_size_t,
                                         ctypes.c_float, ctypes.c_void_p)

_PROTOS = {
    "tra_status_string": (ctypes.c_char_p, [_c_int]),
    "tra_version": (_c_int, []),
    "tra_tile_major_permute": (_c_int, [_vp, _vp, _c_int, _c_int, _c_int, _c_int, Grid, Tile, _vp]),
    "tra_inverse_permute": (_c_int, [_vp, _vp, _c_int, _c_int, _c_int, Grid, Tile, _vp]),
    "tra_dense_attn_entropy": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int,
                                        _c_float, _vp]),
    "tra_attn_entropy": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_float, _vp]),
    "tra_budget_radius": (_c_int, [_vp, _vp, _vp, _c_int, Grid, Tile, _c_float, _c_float, _vp]),
    "tra_budget_radius_ex": (_c_int, [_vp, _vp, _vp, _c_int, Grid, Tile, _c_float, _c_float,
                                      _c_int, _c_int, _vp]),
    "tra_radial_radius": (_c_int, [_vp, _vp, _c_int, Grid, Tile, _c_float, _c_int, _vp]),
    "tra_mask_workspace_size": (_c_size, [_c_int, Grid, Tile, _c_int, _c_int]),
    "tra_workspace_size": (_c_size, [_c_int, Grid, _c_int, _c_int]),
    "tra_build_block_mask_ex": (_c_int, [_vp, _vp, _c_int, Grid, Tile, _c_int, _c_int, _c_int,
                                         _c_int, _vp, _vp, _c_ll, _vp, _vp, _c_size, _vp]),
    "tra_build_block_mask": (_c_int, [_vp, _vp, _c_int, Grid, Tile, _c_int, _c_int, _c_int, _vp,
                                      _vp, _c_ll, _vp, _vp, _c_size, _vp]),
    "tra_build_block_mask_noalloc": (_c_int, [_vp, _vp, _c_int, Grid, Tile, _c_int, _c_int, _c_int,
                                              _vp, _vp, _c_ll, _vp, _vp]),
    "tra_block_sparse_attn": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int,
                                       _c_int, _c_int, _c_float, _vp]),
    "tra_quantize_e4m3": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _vp]),
    "tra_block_sparse_attn_fp8": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int,
                                           _c_int, _c_int, _c_int, _c_int, _c_float, _vp]),
    "tra_selftest_wait_timeout": (_c_int, [_c_int, _vp, _vp]),
    "tra_get_device_error": (_c_int, [ctypes.POINTER(_c_int), _vp]),
}


def lib() -> ctypes.CDLL:
    """The loaded libtra.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m entropy_adaptive_radius_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _PROTOS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def status_string(s: int) -> str:
    return lib().tra_status_string(s).decode()


def _check(fn: str, s: int):
    if s != 0:
        raise TraError(fn, s, status_string(s))


def _p(t: Optional[torch.Tensor]):
    """Device pointer of a tensor on the current CUDA device (None stays None)."""
    if t is None:
        return None
    if not t.is_cuda or t.device.index != torch.cuda.current_device():
        raise ValueError(f"tensor on {t.device}: the library takes tensors on the current "
                         "CUDA device")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return TRA_BF16
    if t.dtype == torch.float32:
        return TRA_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _grid(grid: Sequence[int]) -> Grid:
    return Grid(*map(int, grid))


def _tile(tile: Sequence[int]) -> Tile:
    return Tile(*map(int, tile))


def _contig(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def _want(name: str, t: Optional[torch.Tensor], shape=None, dtypes=None, min_numel=None):
    """The C calls cannot see allocation sizes, so every tensor's shape and
    dtype is checked here against the call's dimensions before its pointer
    is passed on (a short tensor would send a kernel past its end)."""
    if t is None:
        return
    if dtypes is not None and t.dtype not in dtypes:
        raise TypeError(f"{name}: dtype {t.dtype}, expected one of {dtypes}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if min_numel is not None and t.numel() < min_numel:
        raise ValueError(f"{name}: {t.numel()} elements, at least {min_numel} needed")


_BF16 = (torch.bfloat16,)
_F32 = (torch.float32,)
_I32 = (torch.int32,)
_U8 = (torch.uint8,)


def _n_of(grid: Sequence[int]) -> int:
    F, H, W = (int(v) for v in grid)
    return F * H * W


def _qkv(Q) -> tuple:
    if Q.dim() != 3:
        raise ValueError(f"expected [heads, N, d], got shape {tuple(Q.shape)}")
    return tuple(Q.shape)


def tra_tile_major_permute(X, X_tm, grid, tile=(1, 4, 4), stream=None):
    """X_tm[h, p] = X[h, pi(p)] for X [heads, N, d] (bf16 or f32)."""
    _contig(X, X_tm)
    heads, N, d = _qkv(X)
    if N != _n_of(grid):
        raise ValueError(f"X has {N} tokens, the grid {tuple(grid)} has {_n_of(grid)}")
    _want("X", X, dtypes=_BF16 + _F32)
    _want("X_tm", X_tm, (heads, N, d), _BF16 + _F32)
    _check("tra_tile_major_permute", lib().tra_tile_major_permute(
        _p(X), _p(X_tm), _dtype(X), _dtype(X_tm), heads, d, _grid(grid), _tile(tile),
        _stream(stream)))
    return X_tm


def tra_inverse_permute(X_tm, X, grid, tile=(1, 4, 4), stream=None):
    """X[h, pi(p)] = X_tm[h, p]."""
    _contig(X, X_tm)
    if X.dtype != X_tm.dtype:
        raise TypeError("inverse permute keeps the dtype")
    heads, N, d = _qkv(X_tm)
    if N != _n_of(grid):
        raise ValueError(f"X_tm has {N} tokens, the grid {tuple(grid)} has {_n_of(grid)}")
    _want("X_tm", X_tm, dtypes=_BF16 + _F32)
    _want("X", X, (heads, N, d))
    _check("tra_inverse_permute", lib().tra_inverse_permute(
        _p(X_tm), _p(X), _dtype(X_tm), heads, d, _grid(grid), _tile(tile), _stream(stream)))
    return X


def tra_dense_attn_entropy(Q, K, V, O, H, lse=None, scale=None, stream=None):
    """Dense attention O, entropy H and (optionally) LSE of Q, K, V [heads, N, d] bf16."""
    _contig(Q, K, V, O, H, lse)
    heads, N, d = _qkv(Q)
    for name, t in (("Q", Q), ("K", K), ("V", V), ("O", O)):
        _want(name, t, (heads, N, d), _BF16)
    _want("H", H, (heads, N), _F32)
    _want("lse", lse, (heads, N), _F32)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    _check("tra_dense_attn_entropy", lib().tra_dense_attn_entropy(
        _p(Q), _p(K), _p(V), _p(O), _p(H), _p(lse), heads, N, d, scale, _stream(stream)))
    return O, H


def tra_attn_entropy(Q, K, H, lse=None, scale=None, stream=None):
    """Entropy H (and optionally LSE) of every query of Q, K [heads, N, d] bf16
    over all keys, without the PV product or an output."""
    _contig(Q, K, H, lse)
    heads, N, d = _qkv(Q)
    _want("Q", Q, (heads, N, d), _BF16)
    _want("K", K, (heads, N, d), _BF16)
    _want("H", H, (heads, N), _F32)
    _want("lse", lse, (heads, N), _F32)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    _check("tra_attn_entropy", lib().tra_attn_entropy(
        _p(Q), _p(K), _p(H), _p(lse), heads, N, d, scale, _stream(stream)))
    return H


def _radius_args(heads, grid, H, r, phi_out):
    N = _n_of(grid)
    _want("H", H, (heads, N), _F32)
    _want("r", r, (heads, N), _F32)
    _want("phi_out", phi_out, dtypes=_F32, min_numel=int(grid[0]))


def tra_budget_radius(H, r, grid, tau, gamma, tile=(1, 4, 4), phi_out=None, stream=None):
    """Per-query base radius r [heads, N] from entropy H (tile-major order)."""
    _contig(H, r, phi_out)
    heads = H.shape[0]
    _radius_args(heads, grid, H, r, phi_out)
    _check("tra_budget_radius", lib().tra_budget_radius(
        _p(H), _p(r), _p(phi_out), heads, _grid(grid), _tile(tile), float(tau), float(gamma),
        _stream(stream)))
    return r


def tra_budget_radius_ex(H, r, grid, tau, gamma, budget="entropy", metric="disk", tile=(1, 4, 4),
                         phi_out=None, stream=None):
    """Base radii from the entropy with a choice of budget ("entropy" per query,
    "shared" per head) and distance ("disk", "line")."""
    _contig(H, r, phi_out)
    heads = H.shape[0]
    _radius_args(heads, grid, H, r, phi_out)
    _check("tra_budget_radius_ex", lib().tra_budget_radius_ex(
        _p(H), _p(r), _p(phi_out), heads, _grid(grid), _tile(tile), float(tau), float(gamma),
        BUDGETS[budget], METRICS[metric], _stream(stream)))
    return r


def tra_radial_radius(r, grid, r0, metric="disk", tile=(1, 4, 4), phi_out=None, stream=None):
    """Radial Attention's static window: r = r0 everywhere and the band table in phi_out."""
    _contig(r, phi_out)
    heads = r.shape[0]
    _radius_args(heads, grid, None, r, phi_out)
    _check("tra_radial_radius", lib().tra_radial_radius(
        _p(r), _p(phi_out), heads, _grid(grid), _tile(tile), float(r0), METRICS[metric],
        _stream(stream)))
    return r


def _mask_args(heads, grid, block_q, block_k, r, phi, row_ptr, col_idx, nnz, workspace=None):
    N = _n_of(grid)
    nqb = -(-N // block_q) if block_q > 0 else 0
    _want("r", r, (heads, N), _F32)
    _want("phi", phi, dtypes=_F32, min_numel=int(grid[0]))
    _want("row_ptr", row_ptr, dtypes=_I32, min_numel=heads * (nqb + 1))
    _want("col_idx", col_idx, dtypes=_I32)
    _want("nnz", nnz, dtypes=_I32, min_numel=1)
    _want("workspace", workspace, dtypes=_U8)


def tra_mask_workspace_size(heads, grid, block_q, block_k, tile=(1, 4, 4)) -> int:
    return int(lib().tra_mask_workspace_size(heads, _grid(grid), _tile(tile), block_q, block_k))


def tra_workspace_size(heads, grid, block_q, block_k) -> int:
    """tra_mask_workspace_size for the default 1 x 4 x 4 tile."""
    return int(lib().tra_workspace_size(heads, _grid(grid), block_q, block_k))


def tra_build_block_mask(r, phi, grid, block_q, block_k, vote, row_ptr, col_idx, nnz, workspace,
                         tile=(1, 4, 4), stream=None):
    """Block-sparse CSR of the radius mask.  `workspace` is a uint8 CUDA tensor of
    at least tra_mask_workspace_size bytes (256-byte aligned)."""
    _contig(r, phi, row_ptr, col_idx, nnz, workspace)
    heads = r.shape[0]
    _mask_args(heads, grid, block_q, block_k, r, phi, row_ptr, col_idx, nnz, workspace)
    _check("tra_build_block_mask", lib().tra_build_block_mask(
        _p(r), _p(phi), heads, _grid(grid), _tile(tile), block_q, block_k, vote, _p(row_ptr),
        _p(col_idx), col_idx.numel(), _p(nnz), _p(workspace), workspace.numel(),
        _stream(stream)))
    return row_ptr, col_idx, nnz


def tra_build_block_mask_ex(r, phi, grid, block_q, block_k, vote, row_ptr, col_idx, nnz,
                            workspace, metric="disk", tile=(1, 4, 4), stream=None):
    """tra_build_block_mask with a choice of distance ("disk" or "line")."""
    _contig(r, phi, row_ptr, col_idx, nnz, workspace)
    heads = r.shape[0]
    _mask_args(heads, grid, block_q, block_k, r, phi, row_ptr, col_idx, nnz, workspace)
    _check("tra_build_block_mask_ex", lib().tra_build_block_mask_ex(
        _p(r), _p(phi), heads, _grid(grid), _tile(tile), block_q, block_k, vote, METRICS[metric],
        _p(row_ptr), _p(col_idx), col_idx.numel(), _p(nnz), _p(workspace), workspace.numel(),
        _stream(stream)))
    return row_ptr, col_idx, nnz


def tra_build_block_mask_noalloc(r, phi, grid, block_q, block_k, vote, row_ptr, col_idx, nnz,
                                 tile=(1, 4, 4), stream=None):
    """Same CSR as tra_build_block_mask, for callers that cannot pass scratch
    memory: the library uses its built-in buffer of TRA_MASK_STATIC_SCRATCH_BYTES
    (8 MiB per device).  Calls that overlap on the GPU share that buffer and
    race; issue them in order on one stream."""
    _contig(r, phi, row_ptr, col_idx, nnz)
    heads = r.shape[0]
    _mask_args(heads, grid, block_q, block_k, r, phi, row_ptr, col_idx, nnz)
    _check("tra_build_block_mask_noalloc", lib().tra_build_block_mask_noalloc(
        _p(r), _p(phi), heads, _grid(grid), _tile(tile), block_q, block_k, vote, _p(row_ptr),
        _p(col_idx), col_idx.numel(), _p(nnz), _stream(stream)))
    return row_ptr, col_idx, nnz


MASK_STATIC_SCRATCH_BYTES = 8 * 1024 * 1024


def _csr_args(heads, N, block_q, row_ptr, col_idx, lse):
    nqb = -(-N // block_q) if block_q > 0 else 0
    _want("row_ptr", row_ptr, dtypes=_I32, min_numel=heads * (nqb + 1))
    _want("col_idx", col_idx, dtypes=_I32)
    _want("lse", lse, (heads, N), _F32)


def tra_block_sparse_attn(Q, K, V, O, row_ptr, col_idx, block_q, block_k, lse=None, scale=None,
                          stream=None):
    """Exact attention over the kept blocks of the CSR mask."""
    _contig(Q, K, V, O, row_ptr, col_idx, lse)
    heads, N, d = _qkv(Q)
    for name, t in (("Q", Q), ("K", K), ("V", V), ("O", O)):
        _want(name, t, (heads, N, d), _BF16)
    _csr_args(heads, N, block_q, row_ptr, col_idx, lse)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    _check("tra_block_sparse_attn", lib().tra_block_sparse_attn(
        _p(Q), _p(K), _p(V), _p(O), _p(lse), _p(row_ptr), _p(col_idx), heads, N, d, block_q,
        block_k, scale, _stream(stream)))
    return O


def tra_quantize_e4m3(X, Xq, scales, block=128, stream=None):
    """Per-block E4M3 codes Xq (uint8 [heads, N, d]) and fp32 scales
    [heads, ceil(N / block)] of a bf16 X [heads, N, d]."""
    _contig(X, Xq, scales)
    heads, N, d = _qkv(X)
    _want("X", X, (heads, N, d), _BF16)
    _want("Xq", Xq, (heads, N, d), _U8)
    _want("scales", scales, (heads, -(-N // block) if block > 0 else 0), _F32)
    _check("tra_quantize_e4m3", lib().tra_quantize_e4m3(
        _p(X), _p(Xq), _p(scales), heads, N, d, block, _stream(stream)))
    return Xq, scales


def tra_block_sparse_attn_fp8(Q8, q_scales, K8, k_scales, V, O, row_ptr, col_idx, block_q=128,
                              block_k=128, lse=None, scale=None, stream=None):
    """Block-sparse attention with E4M3 Q and K (from tra_quantize_e4m3, block 128)."""
    _contig(Q8, q_scales, K8, k_scales, V, O, row_ptr, col_idx, lse)
    heads, N, d = _qkv(V)
    _want("Q8", Q8, (heads, N, d), _U8)
    _want("K8", K8, (heads, N, d), _U8)
    _want("V", V, (heads, N, d), _BF16)
    _want("O", O, (heads, N, d), _BF16)
    nsc = -(-N // 128)
    _want("q_scales", q_scales, (heads, nsc), _F32)
    _want("k_scales", k_scales, (heads, nsc), _F32)
    _csr_args(heads, N, block_q, row_ptr, col_idx, lse)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    _check("tra_block_sparse_attn_fp8", lib().tra_block_sparse_attn_fp8(
        _p(Q8), _p(q_scales), _p(K8), _p(k_scales), _p(V), _p(O), _p(lse), _p(row_ptr),
        _p(col_idx), heads, N, d, block_q, block_k, scale, _stream(stream)))
    return O


def tra_selftest_wait_timeout(limit_ms, completed=None, stream=None):
    """Launch the bounded-wait self-test (a wait that nothing completes, given
    up after limit_ms); read the outcome with tra_get_device_error."""
    _contig(completed)
    _want("completed", completed, dtypes=_I32, min_numel=1)
    _check("tra_selftest_wait_timeout", lib().tra_selftest_wait_timeout(
        int(limit_ms), _p(completed), _stream(stream)))


def tra_get_device_error(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device error code."""
    code = _c_int(0)
    s = lib().tra_get_device_error(ctypes.byref(code), _stream(stream))
    if s not in (0, 7, 8):
        _check("tra_get_device_error", s)
    return code.value


def workspace_tensor(nbytes: int, device="cuda") -> torch.Tensor:
    """A uint8 CUDA buffer of `nbytes` whose start is 256-byte aligned (torch's
    caching allocator returns 512-byte aligned blocks)."""
    t = torch.empty(max(1, nbytes), dtype=torch.uint8, device=device)
    if t.data_ptr() % 256:
        raise RuntimeError("allocator returned a misaligned workspace")
    return t
