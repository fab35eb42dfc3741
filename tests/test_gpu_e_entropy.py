"""GPU parity of the entropy-only pass (the entropy refresh of cross-step
reuse, Token Radius Attention summary §2 "TRA pipeline"): H and LSE against
the fp64 oracle within 1e-3, and against the dense warm-up kernel's H."""
import math

import numpy as np
import pytest
import torch

from entropy_adaptive_radius_b200 import inputs, tra, workloads
from oracle import tra_oracle as O
from tests.gpu_util import H_ABS, LSE_ABS, check_close, need_gpu, to64

pytestmark = pytest.mark.gpu


def gpu_entropy(Q, K, with_lse=True):
    Qd, Kd = Q.cuda(), K.cuda()
    heads, N, _ = Q.shape
    H = torch.full((heads, N), -7.0, dtype=torch.float32, device="cuda")
    L = torch.full_like(H, -7.0) if with_lse else None
    tra.tra_attn_entropy(Qd, Kd, H, L)
    assert tra.tra_get_device_error() == 0
    return H, L


def rand_qk(heads, N, d, seed, qscale=1.0):
    g = torch.Generator().manual_seed(seed)
    Q = (torch.randn(heads, N, d, generator=g) * qscale).to(torch.bfloat16)
    K = torch.randn(heads, N, d, generator=g).to(torch.bfloat16)
    return Q, K


def oracle_h_lse(Q, K):
    d = Q.shape[2]
    V = np.zeros(Q.shape)
    _, Hr, Lr = O.dense_attention_entropy(to64(Q), to64(K), V, 1.0 / math.sqrt(d))
    return Hr, Lr


@pytest.mark.parametrize("heads,N,d", [(1, 128, 64), (1, 128, 128), (2, 256, 64), (2, 1000, 128),
                                       (1, 60, 64), (1, 1, 128), (3, 777, 64), (1, 2560, 128),
                                       (2, 129, 128), (1, 383, 64)])
def test_entropy_only_random(heads, N, d):
    need_gpu()
    Q, K = rand_qk(heads, N, d, seed=N + 3 * d, qscale=2.0)
    H, L = gpu_entropy(Q, K)
    Hr, Lr = oracle_h_lse(Q, K)
    check_close(H, Hr, H_ABS, "H")
    check_close(L, Lr, LSE_ABS, "LSE")


def test_entropy_only_without_lse_and_special_cases():
    need_gpu()
    # uniform scores: H = ln N
    for N, d in ((300, 64), (5000, 128)):
        _, K = rand_qk(2, N, d, seed=1)
        H, _ = gpu_entropy(torch.zeros(2, N, d, dtype=torch.bfloat16), K, with_lse=False)
        check_close(H, np.full((2, N), math.log(N)), H_ABS, "H uniform")
    # one-hot rows: H = 0
    N, d = 700, 64
    Q = torch.zeros(1, N, d)
    K = torch.zeros(1, N, d)
    Q[0, :, 0] = 400.0
    K[0, 123, 0] = 1.0
    H, L = gpu_entropy(Q.to(torch.bfloat16), K.to(torch.bfloat16))
    check_close(H, np.zeros((1, N)), H_ABS, "H one-hot")
    check_close(L, np.full((1, N), 50.0), LSE_ABS, "LSE one-hot")


def test_entropy_only_large_score_range_rescales():
    need_gpu()
    heads, N, d = 2, 1500, 128
    g = torch.Generator().manual_seed(9)
    K = torch.randn(heads, N, d, generator=g) * torch.linspace(0.1, 6.0, N)[None, :, None]
    Q = torch.randn(heads, N, d, generator=g) * 2
    Q, K = Q.to(torch.bfloat16), K.to(torch.bfloat16)
    H, L = gpu_entropy(Q, K)
    Hr, Lr = oracle_h_lse(Q, K)
    check_close(H, Hr, H_ABS, "H")
    check_close(L, Lr, LSE_ABS, "LSE")


@pytest.mark.parametrize("wl", [workloads.WAN13B, workloads.WAN14B], ids=lambda w: w.name)
def test_entropy_only_full_size(wl):
    """Full-size launch (all heads): sampled rows against the oracle, every
    row against the dense warm-up kernel's entropy."""
    need_gpu()
    Q, K, V = inputs.make_qkv(wl.F, wl.H, wl.W, wl.heads, wl.d, wl.seed, wl.q_scale, "bf16")
    H, L = gpu_entropy(Q, K)
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    Hd = torch.empty_like(H)
    tra.tra_dense_attn_entropy(Qd, Kd, Vd, torch.empty_like(Qd), Hd)
    assert tra.tra_get_device_error() == 0
    # both are within 1e-3 of the exact entropy
    assert float((H - Hd).abs().max()) <= 2 * H_ABS
    N = wl.N
    rng = np.random.default_rng(wl.seed)
    last = (N - 1) // 128 * 128
    rows = np.unique(np.concatenate([np.arange(0, 64), np.arange(last, N), rng.integers(0, N, 64)]))
    scale = 1.0 / math.sqrt(wl.d)
    Hn, Ln = to64(H), to64(L)
    for h in sorted({0, wl.heads - 1}):
        q, k = to64(Q[h]), to64(K[h])
        _, Hr, Lr = O.attention_rows(q, k, np.zeros((N, 8)), scale, rows)
        check_close(Hn[h, rows], Hr, H_ABS, f"H h{h}")
        check_close(Ln[h, rows], Lr, LSE_ABS, f"LSE h{h}")
