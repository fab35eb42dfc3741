"""The Python binding checks every tensor's shape and dtype against the
call's dimensions before any pointer reaches the C ABI, which cannot see
allocation sizes (CPU: the checks fire before the device check, so CPU
tensors exercise them)."""
import pytest
import torch

from entropy_adaptive_radius_b200 import tra

GRID = (2, 8, 8)
N = 128
h, d = 2, 64


def bf(*s):
    return torch.zeros(*s, dtype=torch.bfloat16)


def f32(*s):
    return torch.zeros(*s, dtype=torch.float32)


def i32(*s):
    return torch.zeros(*s, dtype=torch.int32)


def test_permute_checks_tokens_against_the_grid_and_output_shape():
    with pytest.raises(ValueError, match="tokens"):
        tra.tra_tile_major_permute(bf(h, N + 1, d), bf(h, N + 1, d), GRID)
    with pytest.raises(ValueError, match="X_tm"):
        tra.tra_tile_major_permute(bf(h, N, d), bf(h, N - 1, d), GRID)
    with pytest.raises(TypeError):
        tra.tra_tile_major_permute(torch.zeros(h, N, d, dtype=torch.float16), bf(h, N, d), GRID)
    with pytest.raises(ValueError, match="X:"):
        tra.tra_inverse_permute(bf(h, N, d), bf(h, N, d - 8), GRID)


@pytest.mark.parametrize("which", ["K", "V", "O"])
def test_dense_checks_every_operand(which):
    t = {"Q": bf(h, N, d), "K": bf(h, N, d), "V": bf(h, N, d), "O": bf(h, N, d)}
    t[which] = bf(h, N - 16, d)
    with pytest.raises(ValueError, match=which):
        tra.tra_dense_attn_entropy(t["Q"], t["K"], t["V"], t["O"], f32(h, N))
    with pytest.raises(ValueError, match="H"):
        tra.tra_dense_attn_entropy(bf(h, N, d), bf(h, N, d), bf(h, N, d), bf(h, N, d), f32(h, N - 1))
    with pytest.raises(TypeError):
        tra.tra_dense_attn_entropy(bf(h, N, d), f32(h, N, d), bf(h, N, d), bf(h, N, d), f32(h, N))


def test_entropy_only_and_sparse_checks():
    with pytest.raises(ValueError, match="K"):
        tra.tra_attn_entropy(bf(h, N, d), bf(h + 1, N, d), f32(h, N))
    with pytest.raises(ValueError, match="lse"):
        tra.tra_attn_entropy(bf(h, N, d), bf(h, N, d), f32(h, N), lse=f32(h, N - 1))
    nqb = N // 64
    with pytest.raises(ValueError, match="row_ptr"):
        tra.tra_block_sparse_attn(bf(h, N, d), bf(h, N, d), bf(h, N, d), bf(h, N, d),
                                  i32(h * (nqb + 1) - 1), i32(8), 64, 64)
    with pytest.raises(TypeError, match="col_idx"):
        tra.tra_block_sparse_attn(bf(h, N, d), bf(h, N, d), bf(h, N, d), bf(h, N, d),
                                  i32(h * (nqb + 1)), torch.zeros(8, dtype=torch.int64), 64, 64)


def test_radius_and_mask_checks():
    with pytest.raises(ValueError, match="r"):
        tra.tra_budget_radius(f32(h, N), f32(h, N - 1), GRID, 0.1, 0.3)
    with pytest.raises(ValueError, match="phi_out"):
        tra.tra_budget_radius(f32(h, N), f32(h, N), GRID, 0.1, 0.3, phi_out=f32(GRID[0] - 1))
    with pytest.raises(ValueError, match="r"):
        tra.tra_radial_radius(f32(h, N + 1), GRID, 2.0)
    ws = torch.zeros(1024, dtype=torch.uint8)
    nqb = N // 64
    with pytest.raises(ValueError, match="row_ptr"):
        tra.tra_build_block_mask(f32(h, N), f32(GRID[0]), GRID, 64, 64, 1, i32(h * (nqb + 1) - 1),
                                 i32(64), i32(1), ws)
    with pytest.raises(ValueError, match="phi"):
        tra.tra_build_block_mask_noalloc(f32(h, N), f32(1), GRID, 64, 64, 1, i32(h * (nqb + 1)),
                                         i32(64), i32(1))
    with pytest.raises(TypeError, match="workspace"):
        tra.tra_build_block_mask_ex(f32(h, N), f32(GRID[0]), GRID, 64, 64, 1, i32(h * (nqb + 1)),
                                    i32(64), i32(1), f32(256))


def test_fp8_checks():
    Xq = torch.zeros(h, N, 128, dtype=torch.uint8)
    with pytest.raises(ValueError, match="scales"):
        tra.tra_quantize_e4m3(bf(h, N, 128), Xq, f32(h, 2), block=128)
    with pytest.raises(TypeError, match="Xq"):
        tra.tra_quantize_e4m3(bf(h, N, 128), bf(h, N, 128), f32(h, 1), block=128)
    with pytest.raises(ValueError, match="k_scales"):
        tra.tra_block_sparse_attn_fp8(Xq, f32(h, 1), Xq, f32(h, 2), bf(h, N, 128), bf(h, N, 128),
                                      i32(h * 2), i32(4))


def test_valid_arguments_reach_the_device_check():
    # well-formed CPU tensors pass every shape check and are refused only
    # because they are not on the GPU
    with pytest.raises(ValueError, match="CUDA device"):
        tra.tra_dense_attn_entropy(bf(h, N, d), bf(h, N, d), bf(h, N, d), bf(h, N, d), f32(h, N))
