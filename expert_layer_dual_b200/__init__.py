"""B200-native fused Mixture-of-Experts layer forward (sm_100a).

y = sum_k w_k * E_{e_k}(x) + S(x) for a Hunyuan-style MoE layer (256 routed
experts, top-8, one shared expert), with FP32-accurate router logits from a
dual-BF16 weight split.  Every stage runs in hand-written CUDA kernels behind
the C ABI declared in ``include/moe.h``; ``expert_layer_dual_b200.moe`` is the
thin ctypes binding over it (argument marshalling only).

Importing the package is cheap: the shared library is loaded on first use of
``expert_layer_dual_b200.moe`` and a missing library raises immediately.
"""
from .configs import CONFIGS, MoEConfig  # noqa: F401

__all__ = ["CONFIGS", "MoEConfig"]
