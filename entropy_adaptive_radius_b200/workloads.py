"""Named synthetic workloads shaped like the video-DiT attention layers that
Token Radius Attention is evaluated on (Token Radius Attention for Efficient
Video Generation, section 3 "Comprehensive validation": Wan2.1 and
HunyuanVideo at 1.3B-14B parameters).

A workload fixes the latent grid (F frames x H rows x W columns), the number
of heads, the head dimension, the tile and block shapes, the TRA parameters
(gamma, vote threshold, a kept-block target that tau is calibrated to) and
the seed of the synthetic inputs.  Nothing here computes any part of the
method; the module is plain data shared by the tests, the bench and the
smoke entry.
"""
from dataclasses import dataclass, field
from typing import Optional, Tuple


@dataclass(frozen=True)
class Workload:
    name: str
    F: int
    H: int
    W: int
    heads: int
    d: int
    dtype: str              # "f32" or "bf16": element type of Q, K, V as generated
    block_q: int
    block_k: int
    gamma: float
    vote: int
    seed: int
    tau: Optional[float] = None          # fixed tau, else calibrated to kept_target
    kept_target: Optional[float] = None  # target fraction of kept blocks
    q_scale: Tuple[float, float] = (0.5, 4.0)  # log-uniform range of the per-query scale
    tile: Tuple[int, int, int] = (1, 4, 4)     # (frames, rows, cols) of a tile
    sparse_calls: int = 1                # sparse calls that reuse one warm-up
    sweep: Tuple[float, ...] = field(default=())
    sweep_votes: Tuple[int, ...] = field(default=())

    @property
    def N(self) -> int:
        return self.F * self.H * self.W

    @property
    def nqb(self) -> int:
        return -(-self.N // self.block_q)

    @property
    def nkb(self) -> int:
        return -(-self.N // self.block_k)


TINY = Workload(
    name="tiny_4x8x8_h2_d64_f32", F=4, H=8, W=8, heads=2, d=64, dtype="f32",
    block_q=16, block_k=16, gamma=0.5, vote=1, seed=0, tau=4.0)

WAN13B = Workload(
    name="wan2.1-1.3b_480p_21x30x52_h12_d128_bf16", F=21, H=30, W=52, heads=12,
    d=128, dtype="bf16", block_q=64, block_k=64, gamma=0.3, vote=1, seed=1,
    kept_target=0.15)

WAN14B = Workload(
    name="wan2.1-14b_720p_21x45x80_h40_d128_bf16", F=21, H=45, W=80, heads=40,
    d=128, dtype="bf16", block_q=128, block_k=128, gamma=0.3, vote=1, seed=2,
    kept_target=0.12, sparse_calls=4)

HUNYUAN = Workload(
    name="hunyuanvideo-13b_720p_33x45x80_h24_d128_bf16", F=33, H=45, W=80,
    heads=24, d=128, dtype="bf16", block_q=128, block_k=128, gamma=0.2, vote=1,
    seed=3, kept_target=0.09, q_scale=(0.25, 8.0))

SWEEP = Workload(
    name="density-sweep_21x45x80_h40_d128_bf16", F=21, H=45, W=80, heads=40,
    d=128, dtype="bf16", block_q=128, block_k=128, gamma=0.3, vote=1, seed=4,
    sweep=(0.05, 0.09, 0.19, 0.40, 1.00), sweep_votes=(1, 4, 16))

ALL = (TINY, WAN13B, WAN14B, HUNYUAN, SWEEP)
BY_NAME = {w.name: w for w in ALL}
