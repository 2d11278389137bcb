"""Seeded synthetic inputs for the attention workloads.

This module is shared by the tests, the bench and the oracle checks.  It holds
no attention arithmetic: it only draws i.i.d. normal numbers from a seeded
numpy PCG64 stream, scales them by a power of two, and rounds them to the
16-bit or 8-bit (E4M3) type the GPU receives (round-to-nearest-even, done by torch's CPU cast).
The oracle is then fed exactly those rounded values widened to fp64.

Workloads follow the shapes the pages measure: detector feature maps flattened
into sequences (20x20 -> N=400, 80x80 -> N=6400), and the long-sequence case
(N=8192, d=128) from the LLM explainer page, and the 160x160 first stage of
the YOLOv12 image page (N=25600, d=96).  The pages measure on trained
detectors and image datasets; the seeded N(0,1) draws stand in for those
feature maps at the same shapes.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

DTYPES = {"bf16": torch.bfloat16, "fp16": torch.float16, "fp8": torch.float8_e4m3fn}


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    N: int
    H: int
    d: int
    dtype: str           # element type handed to the GPU ("bf16", "fp16" or "fp8": E4M3)
    seed: int
    std: float = 1.0     # the draws are N(0,1) * std (std is a power of two)
    backward: bool = False
    note: str = ""

    @property
    def scale(self) -> float:
        """1/sqrt(d) rounded to fp32: the exact value both sides receive."""
        return float(np.float32(1.0 / math.sqrt(self.d)))

    @property
    def fwd_flop(self) -> float:
        """4 B H N^2 d: two N x N x d products (S = Q K^T and O = P V)."""
        return 4.0 * self.B * self.H * self.N * self.N * self.d

    @property
    def bwd_flop(self) -> float:
        """2.5 x the forward count: five N x N x d products (S, dP, dV, dK, dQ)."""
        return 2.5 * self.fwd_flop


# The five workloads and the N sweep.  Seeds are 1000 + workload index; the
# sweep uses 1000 + N.
WORKLOADS = {
    "c1": Workload("c1_tiny_n400_h2_d64", 1, 400, 2, 64, "bf16", 1001,
                   note="20x20 map, fp32 draws rounded to bf16"),
    "c2": Workload("c2_detector_deep_b32_n400_h4_d64", 32, 400, 4, 64, "bf16", 1002,
                   note="20x20 map, 256 channels as 4 heads of 64"),
    "c3": Workload("c3_detector_neck_n6400_h1_d256", 1, 6400, 1, 256, "fp16", 1003, std=0.5,
                   note="80x80 map, 256 channels as one head"),
    "c4": Workload("c4_long_n8192_h8_d128", 1, 8192, 8, 128, "bf16", 1004),
    "c5": Workload("c5_train_b4_n4096_h8_d64", 4, 4096, 8, 64, "bf16", 1005, backward=True),
}
for _n in (1024, 2048, 4096, 8192):
    WORKLOADS[f"sweep{_n}"] = Workload(f"c4_sweep_n{_n}_h8_d64", 1, _n, 8, 64, "bf16", 1000 + _n)
# Not one of the pages' configurations: the long-sequence shape with a
# backward, to measure and test the d = 128 backward at full size.
WORKLOADS["c4train"] = Workload("c4_train_n8192_h8_d128", 1, 8192, 8, 128, "bf16", 1006,
                                backward=True, note="long-sequence shape, forward + backward")
# The detector neck shape with a backward (not one of the pages'
# configurations): measures and tests the d = 256 backward.
WORKLOADS["c3train"] = Workload("c3_train_n6400_h1_d256", 1, 6400, 1, 256, "fp16", 1009, std=0.5,
                                backward=True, note="detector neck shape, forward + backward")
# The first stage of the YOLOv12 image page's network: a 160x160 feature map
# (N = 25600 tokens) with 96 channels, attended as one head of d = 96, fp16,
# Q, K, V packed per token.
# The long-sequence shape on 8-bit (E4M3) inputs, forward only.
WORKLOADS["c4fp8"] = Workload("c4_long_fp8_n8192_h8_d128", 1, 8192, 8, 128, "fp8", 1008,
                              note="long-sequence shape, E4M3 Q, K, V, descale factors 1")
WORKLOADS["y12s1"] = Workload("yolov12_stage1_n25600_h1_d96", 1, 25600, 1, 96, "fp16", 1007,
                              backward=True, note="160x160 map, 96 channels as one head")


def draw(B: int, N: int, H: int, d: int, dtype: str, seed: int, count: int = 3,
         std: float = 1.0, device: str | torch.device = "cpu"):
    """Draw `count` tensors [B, N, H, d] in order Q, K, V, dO from one stream.

    Returns a list of torch tensors of the 16-bit `dtype` on `device`.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    out = []
    for _ in range(count):
        x = rng.standard_normal((B, N, H, d), dtype=np.float32)
        if std != 1.0:
            x = x * np.float32(std)
        t = torch.from_numpy(x).to(DTYPES[dtype])
        out.append(t.to(device) if str(device) != "cpu" else t)
    return out


def draw_workload(w: Workload, count: int | None = None, device="cpu"):
    if count is None:
        count = 4 if w.backward else 3
    return draw(w.B, w.N, w.H, w.d, w.dtype, w.seed, count=count, std=w.std, device=device)


def draw_fp32(B: int, N: int, H: int, d: int, seed: int, count: int = 3, std: float = 1.0):
    """The unrounded fp32 draws of `draw` (same stream), for reporting the
    input-quantisation error only."""
    rng = np.random.Generator(np.random.PCG64(seed))
    out = []
    for _ in range(count):
        x = rng.standard_normal((B, N, H, d), dtype=np.float32)
        if std != 1.0:
            x = x * np.float32(std)
        out.append(x)
    return out


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Widen a (CPU or GPU) 16-bit tensor to a float64 numpy array, exactly."""
    return t.detach().to("cpu", torch.float64).numpy()
