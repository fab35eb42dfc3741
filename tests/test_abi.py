"""C-ABI checks that need no GPU: the library loads, exports every entry
point that include/tra.h declares, and rejects bad arguments before touching
a device (and reports a missing device instead of falling back)."""
import ctypes
import os
import re

import pytest
import torch

from entropy_adaptive_radius_b200 import build as tra_build
from entropy_adaptive_radius_b200 import tra

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tra.h")

OK, INVALID, UNSUPPORTED, WORKSPACE, CAPACITY, CUDA, DEVICE = 0, 1, 2, 3, 4, 5, 6


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(tra.LIB_PATH):
        tra_build.build(quiet=True)
    return tra.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tra_[a-z_]+)\s*\(", text)))


def test_header_declares_the_six_calls():
    names = declared_functions()
    for n in ("tra_tile_major_permute", "tra_inverse_permute", "tra_dense_attn_entropy",
              "tra_budget_radius", "tra_build_block_mask", "tra_block_sparse_attn"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_checked_build_exports_every_declared_symbol():
    """The index-checked build (libtra_check.so) is the same library."""
    if not os.path.exists(tra.CHECK_LIB_PATH):
        tra_build.build(quiet=True, check=True)
    C = ctypes.CDLL(tra.CHECK_LIB_PATH)
    for name in declared_functions():
        assert hasattr(C, name), name


def test_status_strings(L):
    for s in range(8):
        assert len(tra.status_string(s)) > 0
    assert tra.status_string(99) == "unknown status"
    assert L.tra_version() >= 100


G = tra.Grid(21, 45, 80)
T = tra.Tile(1, 4, 4)
P = ctypes.c_void_p(4096)      # a 16-byte aligned stand-in address, never dereferenced
P2 = ctypes.c_void_p(8192)
MIS = ctypes.c_void_p(4104)    # misaligned
S0 = ctypes.c_void_p(0)


def test_permute_validation(L):
    f = L.tra_tile_major_permute
    assert f(None, P, 0, 0, 2, 128, G, T, S0) == INVALID
    assert f(P, None, 0, 0, 2, 128, G, T, S0) == INVALID
    assert f(MIS, P, 0, 0, 2, 128, G, T, S0) == INVALID
    assert f(P, P, 0, 0, 2, 128, G, T, S0) == INVALID
    assert f(P, P2, 5, 0, 2, 128, G, T, S0) == INVALID
    assert f(P, P2, 0, 0, 2, 100, G, T, S0) == UNSUPPORTED
    assert f(P, P2, 0, 0, -1, 128, G, T, S0) == INVALID
    assert f(P, P2, 0, 0, 2, 128, tra.Grid(-1, 2, 2), T, S0) == INVALID
    assert f(P, P2, 0, 0, 2, 128, G, tra.Tile(0, 4, 4), S0) == INVALID
    assert f(P, P2, 0, 0, 2, 128, tra.Grid(2000, 2, 2), T, S0) == INVALID   # F > 1024
    # empty problems are valid no-ops
    assert f(None, None, 0, 0, 0, 128, G, T, S0) == OK
    assert f(None, None, 0, 0, 2, 128, tra.Grid(0, 45, 80), T, S0) == OK
    g = L.tra_inverse_permute
    assert g(P, P2, 0, 2, 100, G, T, S0) == UNSUPPORTED
    assert g(P, None, 0, 2, 128, G, T, S0) == INVALID


def test_attention_validation(L):
    d = L.tra_dense_attn_entropy
    assert d(P, P, P, P, P, None, 2, 1000, 96, 0.1, S0) == UNSUPPORTED
    assert d(P, P, P, P, P, None, 2, 1000, 128, 0.0, S0) == INVALID
    assert d(P, P, P, P, P, None, 2, 1000, 128, float("nan"), S0) == INVALID
    assert d(P, P, P, P, None, None, 2, 1000, 128, 0.1, S0) == INVALID   # H required
    assert d(P, None, P, P, P, None, 2, 1000, 128, 0.1, S0) == INVALID
    assert d(P, P, MIS, P, P, None, 2, 1000, 128, 0.1, S0) == INVALID
    assert d(P, P, P, P, P, None, 0, 1000, 128, 0.1, S0) == OK
    assert d(P, P, P, P, P, None, 2, 0, 128, 0.1, S0) == OK
    assert d(P, P, P, P, P, None, 2, (1 << 24) + 1, 128, 0.1, S0) == UNSUPPORTED
    s = L.tra_block_sparse_attn
    assert s(P, P, P, P, None, P, P, 2, 1000, 128, 32, 128, 0.1, S0) == UNSUPPORTED
    assert s(P, P, P, P, None, P, P, 2, 1000, 128, 128, 48, 0.1, S0) == UNSUPPORTED
    assert s(P, P, P, P, None, None, P, 2, 1000, 128, 128, 128, 0.1, S0) == INVALID
    # 16-token query blocks merge lists of at most 1024 key blocks
    assert s(P, P, P, P, None, P, P, 2, 64 * 1025, 128, 16, 64, 0.1, S0) == UNSUPPORTED


def test_radius_and_mask_validation(L):
    b = L.tra_budget_radius
    assert b(P, P, None, 2, G, T, -1.0, 0.3, S0) == INVALID
    assert b(P, P, None, 2, G, T, 1.0, float("inf"), S0) == INVALID
    assert b(None, P, None, 2, G, T, 1.0, 0.3, S0) == INVALID
    assert b(None, None, None, 0, G, T, 1.0, 0.3, S0) == OK
    m = L.tra_build_block_mask
    ws = L.tra_mask_workspace_size(40, G, T, 128, 128)
    assert ws > 0
    assert m(P, P, 40, G, T, 128, 48, 1, P, P, 100, P, P, ws, S0) == UNSUPPORTED
    assert m(P, P, 40, G, T, 128, 128, 0, P, P, 100, P, P, ws, S0) == INVALID
    assert m(P, P, 40, G, T, 128, 128, 1, P, P, -1, P, P, ws, S0) == CAPACITY
    assert m(P, P, 40, G, T, 128, 128, 1, P, P, 100, None, P, ws, S0) == INVALID
    assert m(P, P, 40, G, T, 128, 128, 1, P, P, 100, P, P, ws - 1, S0) == WORKSPACE
    assert m(P, P, 40, G, T, 128, 128, 1, P, P, 100, P, ctypes.c_void_p(4096 + 128), ws, S0) == WORKSPACE
    assert m(None, P, 40, G, T, 128, 128, 1, P, P, 100, P, P, ws, S0) == INVALID
    # the threshold table of the mask kernel holds at most 384 key frames
    g400 = tra.Grid(400, 4, 4)
    assert m(P, P, 2, g400, T, 16, 16, 1, P, P, 100, P, P, 1 << 30, S0) == UNSUPPORTED


def test_workspace_size_grows_with_problem(L):
    small = L.tra_mask_workspace_size(2, tra.Grid(4, 8, 8), T, 16, 16)
    big = L.tra_mask_workspace_size(40, G, T, 128, 128)
    assert 0 < small < big
    assert L.tra_mask_workspace_size(2, G, T, 100, 128) == 0
    # bitmask rows dominate: heads * nqb * ceil(nkb/32) words
    nqb = -(-75600 // 128)
    assert big >= 40 * nqb * (-(-nqb // 32)) * 4


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU path")
def test_workspace_size_default_tile(L):
    """tra_workspace_size is tra_mask_workspace_size with the 1 x 4 x 4 tile,
    and the size does not depend on the tile."""
    for heads, grid, bq, bk in ((40, G, 128, 128), (12, tra.Grid(21, 30, 52), 64, 64),
                                (2, tra.Grid(4, 8, 8), 16, 16), (3, G, 96, 128)):
        assert L.tra_workspace_size(heads, grid, bq, bk) == L.tra_mask_workspace_size(
            heads, grid, T, bq, bk)
    for tile in (tra.Tile(1, 2, 8), tra.Tile(2, 3, 5), tra.Tile(1, 1, 1)):
        assert L.tra_workspace_size(40, G, 128, 128) == L.tra_mask_workspace_size(
            40, G, tile, 128, 128)


def test_static_scratch_size_matches_the_header():
    """The binding's copy of TRA_MASK_STATIC_SCRATCH_BYTES is the header's."""
    m = re.search(r"#define\s+TRA_MASK_STATIC_SCRATCH_BYTES\s+\(([^)]*)\)", open(HEADER).read())
    assert m, "macro not found"
    expr = re.sub(r"(\d+)u\b", r"\1", m.group(1))
    assert re.fullmatch(r"[\d\s*+()]+", expr)
    assert eval(expr) == tra.MASK_STATIC_SCRATCH_BYTES


def test_valid_call_without_gpu_reports_device_error(L):
    # No silent CPU fallback: a well-formed call on a machine without an
    # sm_100 GPU returns TRA_ERR_DEVICE and the binding raises.
    assert L.tra_tile_major_permute(P, P2, 0, 0, 2, 128, G, T, S0) == DEVICE
    with pytest.raises(tra.TraError):
        tra._check("x", DEVICE)


def test_variant_validation(L):
    b = L.tra_budget_radius_ex
    assert b(P, P, None, 2, G, T, 1.0, 0.3, 2, 0, S0) == INVALID       # unknown budget
    assert b(P, P, None, 2, G, T, 1.0, 0.3, 0, 9, S0) == INVALID       # unknown metric
    assert b(P, P, None, 2, G, T, -1.0, 0.3, 1, 1, S0) == INVALID
    assert b(None, P, None, 2, G, T, 1.0, 0.3, 1, 0, S0) == INVALID
    assert b(None, None, None, 0, G, T, 1.0, 0.3, 1, 1, S0) == OK
    rr = L.tra_radial_radius
    assert rr(P, None, 2, G, T, -1.0, 0, S0) == INVALID
    assert rr(P, None, 2, G, T, float("nan"), 0, S0) == INVALID
    assert rr(P, None, 2, G, T, 3.0, 4, S0) == INVALID
    assert rr(None, None, 2, G, T, 3.0, 0, S0) == INVALID
    assert rr(None, None, 0, G, T, 3.0, 1, S0) == OK
    assert rr(P, None, 2, tra.Grid(2000, 2, 2), T, 3.0, 0, S0) == INVALID   # F > 1024
    m = L.tra_build_block_mask_ex
    ws = L.tra_mask_workspace_size(40, G, T, 128, 128)
    assert m(P, P, 40, G, T, 128, 128, 1, 7, P, P, 100, P, P, ws, S0) == INVALID
    assert m(P, P, 40, G, T, 128, 48, 1, 1, P, P, 100, P, P, ws, S0) == UNSUPPORTED
    assert m(P, P, 40, G, T, 128, 128, 1, 1, P, P, 100, P, P, ws - 1, S0) == WORKSPACE


def test_fp8_validation(L):
    q = L.tra_quantize_e4m3
    assert q(P, P2, P, 2, 1000, 96, 128, S0) == UNSUPPORTED
    assert q(P, P2, P, 2, 1000, 128, 32, S0) == UNSUPPORTED
    assert q(None, P2, P, 2, 1000, 128, 128, S0) == INVALID
    assert q(P, MIS, P, 2, 1000, 128, 128, S0) == INVALID
    assert q(P, P2, None, 2, 1000, 128, 128, S0) == INVALID
    assert q(None, None, None, 0, 1000, 128, 128, S0) == OK
    a = L.tra_block_sparse_attn_fp8
    assert a(P, P, P, P, P, P, None, P, P, 2, 1000, 64, 128, 128, 0.1, S0) == UNSUPPORTED
    assert a(P, P, P, P, P, P, None, P, P, 2, 1000, 128, 64, 64, 0.1, S0) == UNSUPPORTED
    assert a(P, None, P, P, P, P, None, P, P, 2, 1000, 128, 128, 128, 0.1, S0) == INVALID
    assert a(P, P, P, P, P, P, None, None, P, 2, 1000, 128, 128, 128, 0.1, S0) == INVALID
    assert a(P, P, P, P, P, P, None, P, P, 2, 1000, 128, 128, 128, 0.0, S0) == INVALID


def test_selftest_validation(L):
    st = L.tra_selftest_wait_timeout
    assert st(0, None, S0) == INVALID
    assert st(3000, None, S0) == INVALID
    assert st(10, MIS, S0) == INVALID


def test_header_compiles_as_c99_and_host_calls_answer(L, tmp_path):
    """A plain C caller: include/tra.h compiles under -std=c99 -pedantic
    -Werror, links against libtra.so, and the host-side calls agree with the
    binding (status strings, workspace size, argument checks)."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    exe = tmp_path / "abi_host"
    libdir = os.path.dirname(tra.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror",
                    "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c", "abi_host.c"),
                    "-o", str(exe), "-L", libdir, "-ltra", "-Wl,-rpath," + libdir], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.splitlines()
    kv = {}
    statuses = []
    for line in out:
        key, rest = line.split(" ", 1)
        if key == "status":
            statuses.append(rest.split(" ", 1)[1])
        else:
            kv[key] = rest
    assert int(kv["version"]) == L.tra_version()
    assert statuses == [tra.status_string(s) for s in range(9)] and len(set(statuses)) == 9
    assert int(kv["workspace"]) == tra.tra_mask_workspace_size(40, (21, 45, 80), 128, 128) > 0
    assert int(kv["workspace_bad"]) == 0
    assert int(kv["workspace_default_tile"]) == int(kv["workspace"])
    assert int(kv["permute_null"]) == INVALID
