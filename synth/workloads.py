"""The synthetic workloads, as plain numbers (shapes, pattern parameters,
tile size, seed).  Both the oracle side and the CUDA side read them; nothing
here computes attention.

Q, K, V are iid N(0, 1) rounded to bf16 (see ``synth.normal_bf16``), seed 0,
scale 1/sqrt(D), layout [B, H, N, D].
"""
from __future__ import annotations

import math
from dataclasses import dataclass


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    D: int
    window: int
    sinks: int
    stride: int
    n_global: int
    block: int
    seed: int = 0
    causal: int = 1
    area: int = 0
    summary: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    def pattern_args(self) -> dict:
        return dict(window=self.window, sinks=self.sinks, stride=self.stride, n_global=self.n_global,
                    causal=self.causal, area=self.area, summary=self.summary)


WORKLOADS = {
    # tiny window + sinks, 64-wide tiles
    "tiny_w128_s4": Workload("tiny_w128_s4", 1, 2, 2, 512, 64, 128, 4, 0, 0, 64),
    # the pages' example: N = 8192, window 1024, 4 sinks, 128 x 128 tiles
    "w1024_s4_n8192": Workload("w1024_s4_n8192", 1, 16, 16, 8192, 128, 1024, 4, 0, 0, 128),
    # long sliding window with grouped kv heads
    "w4096_gqa_n32768": Workload("w4096_gqa_n32768", 1, 32, 8, 32768, 128, 4096, 0, 0, 0, 128),
    # narrow window, many heads, d = 64
    "w128_s4_h64_n16384": Workload("w128_s4_h64_n16384", 2, 64, 8, 16384, 64, 128, 4, 0, 0, 128),
    # local 128 + every 128th prior token + 16 global tokens
    "strided_global_n16384": Workload("strided_global_n16384", 1, 16, 16, 16384, 128, 128, 0, 128, 16, 128),
    # Area Attention: 1,600 tokens (a 40 x 40 feature map) in four stripes of 400, no causality;
    # heads, head size and batch are not on the pages (8 heads of 64, a batch of 16 images)
    "area_n1600": Workload("area_n1600", 16, 8, 8, 1600, 64, -1, 0, 0, 0, 128, causal=0, area=400),
}

# The workload the throughput metric is quoted on.
HEADLINE = "w1024_s4_n8192"
