"""GPU parity of the FP8 score path: per-block E4M3 quantization bit for bit
against the oracle (codes and scales), and the block-sparse attention with
E4M3 Q and K against the oracle's FP8-score attention within the attention
tolerances (max abs 2e-2, mean abs 2e-3; LSE 1e-3)."""
import math

import numpy as np
import pytest
import torch

from entropy_adaptive_radius_b200 import inputs, tra, workloads
from oracle import tra_oracle as O
from tests.gpu_util import LSE_ABS, check_attention, check_close, need_gpu, to64

pytestmark = pytest.mark.gpu


def gpu_quant(X, block=128):
    heads, N, d = X.shape
    Xq = torch.empty(heads, N, d, dtype=torch.uint8, device="cuda")
    sc = torch.empty(heads, -(-N // block), dtype=torch.float32, device="cuda")
    tra.tra_quantize_e4m3(X.cuda(), Xq, sc, block)
    return Xq, sc


def codes_to_float(Xq):
    return Xq.view(torch.float8_e4m3fn).float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("heads,N,d,block", [(2, 300, 128, 128), (1, 1000, 64, 64), (3, 129, 128, 64),
                                             (1, 128, 128, 128)])
def test_quantize_bitexact(heads, N, d, block):
    need_gpu()
    g = torch.Generator().manual_seed(N + d)
    X = (torch.randn(heads, N, d, generator=g) * torch.logspace(-3, 1, heads)[:, None, None]).to(torch.bfloat16)
    X[0, :min(N, block)] = 0                          # an all-zero block: scale 1, codes 0
    Xq, sc = gpu_quant(X, block)
    codes, scales = O.quantize_e4m3_blocks(to64(X), block)
    assert np.array_equal(sc.cpu().numpy(), scales)
    assert np.array_equal(codes_to_float(Xq), codes)


def fp8_case(heads, N, seed, density, qscale=2.0):
    g = torch.Generator().manual_seed(seed)
    Q = (torch.randn(heads, N, 128, generator=g) * qscale).to(torch.bfloat16)
    K = torch.randn(heads, N, 128, generator=g).to(torch.bfloat16)
    V = torch.randn(heads, N, 128, generator=g).to(torch.bfloat16)
    nb = -(-N // 128)
    mask = inputs.synthetic_block_mask(heads, nb, nb, seed=seed, density=density)
    return Q, K, V, mask


def run_fp8(Q, K, V, mask):
    Q8, qs = gpu_quant(Q)
    K8, ks = gpu_quant(K)
    rp, ci = inputs.csr_from_block_mask(mask)
    O_ = torch.empty(V.shape, dtype=torch.bfloat16, device="cuda")
    L = torch.empty(V.shape[:2], dtype=torch.float32, device="cuda")
    tra.tra_block_sparse_attn_fp8(Q8, qs, K8, ks, V.cuda(), O_, torch.from_numpy(rp.ravel()).cuda(),
                                  torch.from_numpy(ci if ci.size else np.zeros(1, np.int32)).cuda(), lse=L)
    assert tra.tra_get_device_error() == 0
    return O_, L


@pytest.mark.parametrize("heads,N,density", [(2, 1000, 0.3), (1, 3000, 0.1), (2, 256, 1.0), (1, 130, 0.5)])
def test_fp8_sparse_attention_matches_oracle(heads, N, density):
    need_gpu()
    Q, K, V, mask = fp8_case(heads, N, seed=N, density=density)
    O_, L = run_fp8(Q, K, V, mask)
    Q8, qs = O.quantize_e4m3_blocks(to64(Q), 128)
    K8, ks = O.quantize_e4m3_blocks(to64(K), 128)
    Or, Lr = O.sparse_attention_fp8qk(Q8, qs, K8, ks, to64(V), mask, 128, 128, 1.0 / math.sqrt(128))
    check_attention(O_, Or, "O fp8")
    check_close(L, Lr, LSE_ABS, "LSE fp8")


def test_fp8_full_size_sampled_and_distance_to_bf16():
    """Wan2.1-14B-shaped launch (all heads): sampled rows against the oracle's
    FP8 attention; the distance to the bf16-score path is reported, not
    bounded by the parity tolerance (it is the cost of the reading)."""
    need_gpu()
    wl = workloads.WAN14B
    Q, K, V = inputs.make_qkv(wl.F, wl.H, wl.W, wl.heads, wl.d, wl.seed, wl.q_scale, "bf16")
    nb = -(-wl.N // 128)
    mask = inputs.synthetic_block_mask(wl.heads, nb, nb, seed=wl.seed, density=0.12)
    O_, L = run_fp8(Q, K, V, mask)
    rng = np.random.default_rng(wl.seed)
    last = (wl.N - 1) // 128 * 128
    rows = np.unique(np.concatenate([np.arange(0, 64), np.arange(last, wl.N), rng.integers(0, wl.N, 64)]))
    scale = 1.0 / math.sqrt(wl.d)
    for h in sorted({0, wl.heads - 1}):
        q8, qs = O.quantize_e4m3_blocks(to64(Q[h:h + 1]), 128)
        k8, ks = O.quantize_e4m3_blocks(to64(K[h:h + 1]), 128)
        Or, Lr = O.sparse_attention_fp8qk(q8, qs, k8, ks, to64(V[h:h + 1]), mask[h:h + 1], 128, 128,
                                          scale, rows=rows, head=0)
        check_attention(O_[h][rows], Or, f"O fp8 h{h}")
        check_close(to64(L)[h, rows], Lr, LSE_ABS, f"LSE fp8 h{h}")
    # the bf16-score path on the same mask, for the record
    rp, ci = inputs.csr_from_block_mask(mask)
    Ob = torch.empty_like(O_)
    tra.tra_block_sparse_attn(Q.cuda(), K.cuda(), V.cuda(), Ob, torch.from_numpy(rp.ravel()).cuda(),
                              torch.from_numpy(ci).cuda(), 128, 128)
    diff = (O_.float() - Ob.float()).abs()
    print(f"fp8 vs bf16 scores: max abs {diff.max().item():.4f}, mean abs {diff.mean().item():.5f}")
    assert bool(torch.isfinite(O_).all())
