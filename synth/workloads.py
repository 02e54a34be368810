"""The five VMoBA layer workloads (shapes, block boxes, thresholds).

Grids follow the pages' video sizes after a 4x temporal / 16x16 spatial latent
compression (e.g. 93x576x1024 frames -> a 24x36x64 latent), 12 heads of
head_dim 128 (the Wan 2.1 1.3B attention shape), and block counts near the
paper's "8-48-72" setting (VMoBA page 1, training strategy).

``boxes[mode]`` is the full (bt, bh, bw) block box of each partition mode,
stored as plain data: mode 0 = 1D temporal, 1 = 2D spatial, 2 = 3D local.
"""
from __future__ import annotations

from dataclasses import dataclass, field


@dataclass(frozen=True)
class Workload:
    wid: int
    name: str
    T: int
    H: int
    W: int
    n_heads: int
    head_dim: int
    dtype: str                      # "f32" or "bf16" (I/O and storage type)
    kind: str                       # "iid" or "smooth"
    boxes: tuple                    # full (bt, bh, bw) for modes 0, 1, 2
    taus: tuple
    backward: bool
    head_gain: bool = False
    layers: int = 3
    notes: str = field(default="", compare=False)

    @property
    def s(self) -> int:
        return self.T * self.H * self.W


WORKLOADS = {
    1: Workload(1, "tiny-256tok", 4, 8, 8, 2, 64, "f32", "iid",
                ((1, 8, 8), (4, 4, 4), (2, 4, 4)), (0.5,), False,
                notes="oracle-scale case, fp32 I/O, forward only"),
    2: Workload(2, "small-2048tok", 8, 16, 16, 4, 64, "bf16", "smooth",
                ((1, 16, 16), (8, 4, 4), (2, 4, 4)), (0.25, 0.5, 0.75), True),
    3: Workload(3, "wan1.3b-32760tok", 21, 30, 52, 12, 128, "bf16", "smooth",
                ((1, 30, 52), (21, 5, 4), (3, 5, 4)), (0.25,), False,
                notes="inference setting, forward only"),
    4: Workload(4, "train-55296tok", 24, 36, 64, 12, 128, "bf16", "smooth",
                ((1, 36, 64), (24, 6, 8), (4, 6, 8)), (0.25,), True,
                notes="headline: 93x576x1024 video, batch 1, fwd+bwd"),
    5: Workload(5, "stack30-75600tok", 21, 45, 80, 12, 128, "bf16", "smooth",
                ((1, 45, 80), (21, 9, 8), (3, 9, 8)), (0.1, 0.25, 0.5), True,
                head_gain=True, layers=30, notes="30-layer sweep, mode = layer mod 3"),
}

# The paper's own block counts on the 55296-token latent: 8 / 48 / 72 blocks
# for 1D / 2D / 3D (VMoBA notes, training strategy).  The pages give counts,
# not boxes: 1D is 3 frames per block; 2D is the 6x8 spatial box of workload
# 4; 3D is workload 4's 4x6x8 box doubled in height and width (4x12x16).
BOXES_8_48_72 = ((3, 36, 64), (24, 6, 8), (4, 12, 16))


# The 10-48-60 setting of the pages' pre-training runs (digest, App. C: 11K
# and 46K tokens, 1D / 2D / 3D block counts 10, 48 and 60, tau 0.25, the Wan
# 2.1 architecture).  The pages give neither the latents' T, H, W nor the
# boxes; these latents are chosen so that the three counts come out exactly:
#   11520 tokens = T10 x H32 x W36: 1D one frame (10 blocks of 1152), 2D 4x6
#     (8 x 6 = 48 blocks of 240), 3D 2x8x12 (5 x 4 x 3 = 60 blocks of 192);
#   46080 tokens = T30 x H32 x W48: 1D three frames (10 blocks of 4608), 2D
#     4x8 (8 x 6 = 48 blocks of 960), 3D 6x8x16 (5 x 4 x 3 = 60 blocks of 768).
# 12 heads of 128 (the Wan 2.1 1.3B attention shape), bf16, fwd + bwd.
PAPER_10_48_60 = {
    "11520tok": Workload(60, "pretrain-11520tok", 10, 32, 36, 12, 128, "bf16", "smooth",
                         ((1, 32, 36), (10, 4, 6), (2, 8, 12)), (0.25,), True,
                         notes="10-48-60 block counts at 11K tokens"),
    "46080tok": Workload(61, "pretrain-46080tok", 30, 32, 48, 12, 128, "bf16", "smooth",
                         ((3, 32, 48), (30, 4, 8), (6, 8, 16)), (0.25,), True,
                         notes="10-48-60 block counts at 46K tokens"),
}
