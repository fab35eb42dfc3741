"""Shared helpers of the GPU parity tests: device checks, tolerance checks,
and the oracle-side reference of a CSR (built from the oracle's mask).
Nothing here computes a result of the CUDA path."""
import numpy as np
import pytest
import torch

# parity tolerances: attention output (bf16 inputs, fp32 accumulation),
# entropy; LSE follows entropy (both are ln Z up to a bounded term)
O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
H_ABS = 1e-3
LSE_ABS = 1e-3


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    major, _ = torch.cuda.get_device_capability()
    if major != 10:
        pytest.skip("needs an sm_100 GPU")


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def check_attention(O_gpu, O_ref, what=""):
    err = np.abs(to64(O_gpu) - O_ref)
    assert np.isfinite(err).all(), f"{what}: non-finite output"
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= O_MAX_ABS, f"{what}: max abs err {mx:.3e} > {O_MAX_ABS}"
    assert mean <= O_MEAN_ABS, f"{what}: mean abs err {mean:.3e} > {O_MEAN_ABS}"
    return mx, mean


def check_close(x_gpu, x_ref, tol, what=""):
    a = to64(x_gpu) if isinstance(x_gpu, torch.Tensor) else np.asarray(x_gpu, np.float64)
    b = np.asarray(x_ref, np.float64)
    both_inf = np.isinf(a) & np.isinf(b) & (np.sign(a) == np.sign(b))
    with np.errstate(invalid="ignore"):
        err = np.where(both_inf, 0.0, np.abs(a - b))
    mx = float(np.nanmax(err)) if err.size else 0.0
    assert not np.isnan(err).any(), f"{what}: NaN mismatch"
    assert mx <= tol, f"{what}: max abs err {mx:.3e} > {tol}"
    return mx


def csr_rows(row_ptr, col_idx, h, qb, nqb):
    """Kept key blocks of row (h, qb) of a CSR given as numpy arrays."""
    s = int(row_ptr[h * (nqb + 1) + qb])
    e = int(row_ptr[h * (nqb + 1) + qb + 1])
    return col_idx[s:e]


def check_csr_valid(row_ptr, col_idx, nnz, heads, nqb, nkb):
    rp = np.asarray(row_ptr).reshape(heads, nqb + 1)
    assert rp[0, 0] == 0
    for h in range(heads):
        assert np.all(np.diff(rp[h]) >= 0)
        if h + 1 < heads:
            assert rp[h, nqb] == rp[h + 1, 0]
    assert rp[heads - 1, nqb] == nnz
    c = np.asarray(col_idx[:nnz])
    assert c.min() >= 0 and c.max() < nkb
    flat = rp[:, :nqb].ravel()
    ends = rp[:, 1:].ravel()
    for s, e in zip(flat, ends):
        if e - s > 1:
            assert np.all(np.diff(c[s:e]) > 0), "col_idx not strictly ascending in a row"
