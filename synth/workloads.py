"""The seeded synthetic workloads: shapes, value recipe and mask parameters.

All grids are token grids T x H x W cut into 4x4x4 tiles (64 tokens = one
attention block), so the tile grid is (T/4, H/4, W/4) and S = T*H*W.
Q and K are pos_weight * e(t,h,w) + noise_weight * z with e a fixed 3D
sinusoidal embedding and z ~ N(0,1); V ~ N(0,1).  ``iid_normal`` workloads
draw Q, K, V ~ N(0,1) and use externally supplied Bernoulli block masks.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional, Tuple


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    d: int
    grid: Tuple[int, int, int]          # token grid (T, H, W)
    thr: float = 0.2
    sta: Optional[Tuple[int, int, int]] = None   # half-window in tiles (wt, wh, ww)
    pos_weight: float = 1.0
    noise_weight: float = 0.5
    iid_normal: bool = False
    densities: Tuple[float, ...] = field(default_factory=tuple)  # static-mask Bernoulli p values

    @property
    def S(self) -> int:
        T, H, W = self.grid
        return T * H * W

    @property
    def nb(self) -> int:
        return self.S // 64

    @property
    def tile_grid(self) -> Tuple[int, int, int]:
        T, H, W = self.grid
        return (T // 4, H // 4, W // 4)


WORKLOADS = {
    # 1024 tokens, 16 blocks: the case the oracle finishes instantly
    "tiny": Workload("tiny", B=1, H=2, d=64, grid=(4, 16, 16), thr=0.2, sta=None),
    # 8192 tokens, 128 blocks, STA window +-1 tile on every axis
    "small": Workload("small", B=1, H=12, d=64, grid=(8, 32, 32), thr=0.2, sta=(1, 1, 1)),
    # Wan 2.1 14B 720p-shaped layer: 76,800 tokens, 1200 blocks
    "wan720p": Workload("wan720p", B=1, H=40, d=128, grid=(20, 48, 80), thr=0.2, sta=(1, 2, 2)),
    # HunyuanVideo 720p-shaped layer: 107,520 tokens, 1680 blocks, more diffuse rows
    "hunyuan720p": Workload("hunyuan720p", B=1, H=24, d=128, grid=(28, 48, 80), thr=0.4, sta=None,
                            noise_weight=1.0),
    # static-mask density sweep: 32,768 tokens, 512 blocks, i.i.d. N(0,1) inputs
    "sweep": Workload("sweep", B=1, H=24, d=128, grid=(8, 64, 64), iid_normal=True,
                      pos_weight=0.0, noise_weight=1.0,
                      densities=(0.05, 0.1, 0.2, 0.4, 0.7, 1.0)),
}
