"""Workload shapes of the fused MoE layer forward.

Each entry is one synthetic workload: T tokens of hidden size d routed to
top-k of E experts (expert intermediate I) plus, when Is > 0, one shared
expert of intermediate Is.  The layer shape (256 routed experts, top-8, one
shared expert) is Hy4-preview's ("PR #54160 完整报告", section 功能与动机);
hidden sizes 4096 / 6144 and FP8 128x128 block scales come from the same
page (section 实现拆解, items 4 and 5).
"""
from __future__ import annotations

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int
    d: int
    E: int
    k: int
    I: int
    Is: int = 0
    wdtype: int = 0          # 0 bf16 weights, 1 fp8 e4m3 with 128x128 block scales, 2 MXFP8,
                             # 3 FP8 per tensor with static (calibrated) activation scales
    zipf_bias: bool = False  # skewed routing: per-expert Zipf(s=1.2) logit bias
    seed: int = 0
    renorm: bool = True

    def rows(self) -> int:
        """Rows of the permuted activation matrices: T*k routed + T shared."""
        return self.T * self.k + (self.T if self.Is > 0 else 0)

    def with_T(self, T: int) -> "MoEConfig":
        return replace(self, T=T)

    def flops(self) -> float:
        """Algorithmic FLOPs of one forward: the two router GEMMs, the routed
        and shared expert FFNs (gate, up, down), multiply-adds counted as 2."""
        router = 2.0 * 2 * self.T * self.d * self.E
        routed = 2.0 * self.T * self.k * 3 * self.d * self.I
        shared = 2.0 * self.T * 3 * self.d * self.Is
        return router + routed + shared


CONFIGS = {
    # 16 tokens, d 256, 8 experts top-2, I 128, no shared expert
    "tiny": MoEConfig("tiny", T=16, d=256, E=8, k=2, I=128, Is=0, seed=0),
    # decode-shaped Hy4-like layer: 64 tokens, 256 experts top-8 + shared, I 1536
    "decode": MoEConfig("decode", T=64, d=4096, E=256, k=8, I=1536, Is=1536, seed=1),
    # prefill-shaped layer: 8192 tokens, same layer
    "prefill": MoEConfig("prefill", T=8192, d=4096, E=256, k=8, I=1536, Is=1536, seed=2),
    # FP8 block-scaled layer: 4096 tokens, d 6144, I 2048
    "fp8": MoEConfig("fp8", T=4096, d=6144, E=256, k=8, I=2048, Is=2048, wdtype=1, seed=3),
    # the FP8 layer in MXFP8: e4m3 weights and activations, E8M0 scale per 1x32
    # (the MXFP8 weight format of the same page, section 实现拆解 item 4)
    "mxfp8": MoEConfig("mxfp8", T=4096, d=6144, E=256, k=8, I=2048, Is=2048, wdtype=2, seed=3),
    # the FP8 layer with per-tensor scales: one scale per weight matrix, static
    # activation scales ("HPC-Ops" GroupGEMM FP8 per-tensor; the Hunyuan page's
    # static FP8 scheme)
    "fp8t": MoEConfig("fp8t", T=4096, d=6144, E=256, k=8, I=2048, Is=2048, wdtype=3, seed=3),
    # skewed routing: 16384 tokens, Zipf-biased router logits
    "skew": MoEConfig("skew", T=16384, d=4096, E=256, k=8, I=1536, Is=1536,
                      zipf_bias=True, seed=4),
}
