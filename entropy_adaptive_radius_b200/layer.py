"""One Token Radius Attention layer across the denoising steps of a video
diffusion model (Token Radius Attention summary, §2 "TRA pipeline": entropy
from a dense warm-up phase, budget -> radius -> block mask, and cross-step
reuse of the entropy by the later sparse steps).

`TraLayer` owns the device buffers of one layer: the tile-major copies of
Q, K, V and O, the entropy, radii, decay table, the CSR block mask and the
mask's scratch space.  Its `forward` runs one step through the C ABI; which
kind of step it is follows the `ReusePolicy`:

  * the first `warmup` steps are dense: dense attention with entropy, then
    radius and mask from that entropy;
  * every later step is sparse: block-sparse attention over the current mask;
  * with `refresh_every = k > 0`, every k-th step after the warm-up also
    refreshes the entropy from its own Q and K and rebuilds the mask for the
    steps that follow: `refresh = "entropy"` keeps the sparse output and adds
    an entropy-only pass (no PV product); `refresh = "dense"` makes the step a
    dense one.

The mask may also come from the variants the summary's §4 ablations and
Radial Attention describe: `budget="shared"` gives every query of a head the
head's mean budget, `metric="line"` measures distance along the in-frame
raster order, and `radial_r0=r0` replaces the entropy by Radial Attention's
static window (base radius r0, window halving per doubling of the temporal
distance); the sparse steps are unchanged.

With `layout="tile_major"` the layer takes and returns tensors that are
already in tile-major order and runs no permutation: a model that keeps the
tokens of a whole transformer block in tile-major order permutes once on the
way in and once on the way out (`to_tile_major` / `from_tile_major`) instead
of around every attention call.

This module only sequences calls and holds buffers; every step of the method
runs in the CUDA kernels behind `tra`.
"""
from dataclasses import dataclass
from typing import Optional, Sequence

import torch

from . import tra


@dataclass(frozen=True)
class ReusePolicy:
    warmup: int = 1
    refresh_every: int = 0
    refresh: str = "entropy"  # "entropy" (entropy-only pass) or "dense"

    def __post_init__(self):
        if self.warmup < 1:
            raise ValueError("the first step must be dense: warmup >= 1")
        if self.refresh_every < 0:
            raise ValueError("refresh_every >= 0")
        if self.refresh not in ("entropy", "dense"):
            raise ValueError("refresh is 'entropy' or 'dense'")

    def kind(self, step: int) -> str:
        """"dense", "sparse" or "sparse+entropy" for step index `step`."""
        if step < self.warmup:
            return "dense"
        k = step - self.warmup + 1  # 1-based index in the sparse phase
        if self.refresh_every and k % self.refresh_every == 0:
            return "dense" if self.refresh == "dense" else "sparse+entropy"
        return "sparse"


class TraLayer:
    """Buffers and step sequencing of one attention layer on one GPU."""

    def __init__(self, grid: Sequence[int], heads: int, d: int, *, tau: float, gamma: float,
                 tile=(1, 4, 4), block_q: int = 128, block_k: int = 128, vote: int = 1,
                 policy: ReusePolicy = ReusePolicy(), layout: str = "original",
                 budget: str = "entropy", metric: str = "disk", radial_r0: Optional[float] = None,
                 device="cuda"):
        if layout not in ("original", "tile_major"):
            raise ValueError("layout is 'original' or 'tile_major'")
        if budget not in tra.BUDGETS or metric not in tra.METRICS:
            raise ValueError("budget is 'entropy' or 'shared'; metric is 'disk' or 'line'")
        if radial_r0 is not None and not radial_r0 >= 0:
            raise ValueError("radial_r0 >= 0")
        self.layout = layout
        self.budget, self.metric, self.radial_r0 = budget, metric, radial_r0
        self.grid = tuple(int(v) for v in grid)
        F, H, W = self.grid
        self.N = F * H * W
        self.heads, self.d = heads, d
        self.tile = tuple(tile)
        self.block_q, self.block_k = block_q, block_k
        self.tau, self.gamma, self.vote = float(tau), float(gamma), int(vote)
        self.policy = policy
        bf = dict(dtype=torch.bfloat16, device=device)
        # tile-major copies of Q, K, V, O (the resident layout needs none)
        n_buf = 4 if layout == "original" else 0
        self.Qtm, self.Ktm, self.Vtm, self.Otm = (
            [torch.empty(heads, self.N, d, **bf) for _ in range(n_buf)] or [None] * 4)
        self.H = torch.empty(heads, self.N, dtype=torch.float32, device=device)
        self.r = torch.empty_like(self.H)
        self.phi = torch.empty(F, dtype=torch.float32, device=device)
        self.nqb = -(-self.N // block_q)
        self.nkb = -(-self.N // block_k)
        self.row_ptr = torch.empty(heads * (self.nqb + 1), dtype=torch.int32, device=device)
        self.col_idx = torch.empty(max(1, heads * self.nqb * self.nkb), dtype=torch.int32,
                                   device=device)
        self.nnz = torch.zeros(1, dtype=torch.int32, device=device)
        self.ws = tra.workspace_tensor(
            tra.tra_mask_workspace_size(heads, self.grid, block_q, block_k, self.tile), device)
        self.step_index = 0

    def reset(self):
        """Start a new denoising run (the next step is a warm-up step again)."""
        self.step_index = 0

    def _meta(self):
        return {"grid": list(self.grid), "heads": self.heads, "d": self.d, "tile": list(self.tile),
                "block_q": self.block_q, "block_k": self.block_k, "tau": self.tau,
                "gamma": self.gamma, "vote": self.vote, "budget": self.budget,
                "metric": self.metric, "radial_r0": self.radial_r0}

    def state_dict(self) -> dict:
        """What the following steps reuse: the entropy of the last refresh, the
        radii, the decay table, the CSR mask and the step index (copies, on the
        layer's device), with the settings they were built under.  Save it with
        torch.save to resume a denoising run without a new warm-up."""
        nnz = int(self.nnz.item())
        return {"meta": self._meta(), "step_index": self.step_index, "H": self.H.clone(),
                "r": self.r.clone(), "phi": self.phi.clone(), "row_ptr": self.row_ptr.clone(),
                "col_idx": self.col_idx[:nnz].clone(), "nnz": nnz}

    def load_state_dict(self, state: dict):
        """Restore a state_dict taken from a layer with the same settings."""
        if state["meta"] != self._meta():
            raise ValueError("state was taken from a layer with other settings")
        nnz = int(state["nnz"])
        if nnz > self.col_idx.numel() or state["row_ptr"].numel() != self.row_ptr.numel():
            raise ValueError("state does not fit this layer's mask buffers")
        self.H.copy_(state["H"])
        self.r.copy_(state["r"])
        self.phi.copy_(state["phi"])
        self.row_ptr.copy_(state["row_ptr"])
        self.col_idx[:nnz].copy_(state["col_idx"])
        self.nnz.fill_(nnz)
        self.step_index = int(state["step_index"])

    def _rebuild_mask(self):
        if self.radial_r0 is not None:
            tra.tra_radial_radius(self.r, self.grid, self.radial_r0, self.metric, self.tile,
                                  phi_out=self.phi)
        else:
            tra.tra_budget_radius_ex(self.H, self.r, self.grid, self.tau, self.gamma, self.budget,
                                     self.metric, self.tile, phi_out=self.phi)
        tra.tra_build_block_mask_ex(self.r, self.phi, self.grid, self.block_q, self.block_k,
                                    self.vote, self.row_ptr, self.col_idx, self.nnz, self.ws,
                                    self.metric, self.tile)

    def to_tile_major(self, X: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
        """[heads, N, d] from the original token order to tile-major order (bf16)."""
        if out is None:
            out = torch.empty(X.shape, dtype=torch.bfloat16, device=X.device)
        return tra.tra_tile_major_permute(X, out, self.grid, self.tile)

    def from_tile_major(self, X_tm: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
        """[heads, N, d] from tile-major order back to the original order."""
        if out is None:
            out = torch.empty_like(X_tm)
        return tra.tra_inverse_permute(X_tm, out, self.grid, self.tile)

    def forward(self, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                O: Optional[torch.Tensor] = None) -> torch.Tensor:
        """One denoising step.  Q, K, V: [heads, N, d], bf16 (or fp32 in the
        original layout, rounded to bf16 by the permute), in the original
        (t, y, x) token order, or in tile-major order with layout="tile_major".
        Returns O [heads, N, d] bf16 in the same order as the inputs."""
        kind = self.policy.kind(self.step_index)
        if O is None:
            O = torch.empty(self.heads, self.N, self.d, dtype=torch.bfloat16, device=Q.device)
        if self.layout == "original":
            for X, Y in ((Q, self.Qtm), (K, self.Ktm), (V, self.Vtm)):
                tra.tra_tile_major_permute(X, Y, self.grid, self.tile)
            q, k, v, o = self.Qtm, self.Ktm, self.Vtm, self.Otm
        else:
            q, k, v, o = Q, K, V, O
        if kind == "dense":
            tra.tra_dense_attn_entropy(q, k, v, o, self.H)
            self._rebuild_mask()
        else:
            tra.tra_block_sparse_attn(q, k, v, o, self.row_ptr, self.col_idx, self.block_q,
                                      self.block_k)
            if kind == "sparse+entropy":
                tra.tra_attn_entropy(q, k, self.H)
                self._rebuild_mask()
        if self.layout == "original":
            tra.tra_inverse_permute(self.Otm, O, self.grid, self.tile)
        self.step_index += 1
        return O

    __call__ = forward
