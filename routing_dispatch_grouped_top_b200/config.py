"""Layer shapes of the routed MoE workloads this library is measured on.

Notation follows the pages' statement of the problem: T tokens, E experts,
top-K, H dispatch width, F expert width, b bytes per activation (bf16: 2),
P logical expert-parallel partitions (a buffer layout only: one GPU, no
transfer).  ``d_model`` is set only for the latent layer, whose dispatch width H
is reached by a down-projection from ``d_model``.
"""
from __future__ import annotations

from dataclasses import dataclass, replace
from typing import Optional


@dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int
    H: int
    E: int
    K: int
    F: int
    P: int = 1
    renormalize: bool = True
    zipf_s: Optional[float] = None      # per-expert logit bias drawn from rank-Zipf popularity
    d_model: Optional[int] = None       # latent layer: model width before the down-projection
    group_limit: int = 0                # node-limited routing: experts from the M best partitions
    F_shared: int = 0                   # width of a shared expert every token passes through (0: none)
    fp8_dispatch: bool = False          # E4M3 dispatch with per-token scales, E4M3 gate/up weights
    seed: int = 0

    @property
    def TK(self) -> int:
        return self.T * self.K

    @property
    def d_in(self) -> int:
        return self.d_model if self.d_model else self.H

    def with_(self, **kw) -> "MoEConfig":
        return replace(self, **kw)

    # ---- algorithmic work (what the method must move or compute) ----
    def expert_flops(self) -> int:
        """SwiGLU FFN over every assignment: gate+up 4*H*F, down 2*H*F per row."""
        return 6 * self.H * self.F * self.TK

    def gate_up_flops(self) -> int:
        return 4 * self.H * self.F * self.TK

    def down_flops(self) -> int:
        return 2 * self.H * self.F * self.TK

    def dispatch_bytes(self, b: int = 2) -> int:
        """T x K x H x b: activation payload of one dispatch (no padding)."""
        return self.T * self.K * self.H * b

    def dispatch_bytes_actual(self) -> int:
        """Bytes the dispatch writes: bf16 rows, or E4M3 rows plus one fp32 scale per row."""
        return self.dispatch_bytes(1) + 4 * self.TK if self.fp8_dispatch else self.dispatch_bytes(2)

    def expert_weight_bytes(self, b: int = 2) -> int:
        return 3 * self.H * self.F * self.E * b


# The five workloads: a tiny layer, two prefill layers, one decode step with a
# skewed router and one latent-dispatch layer.
TINY = MoEConfig("tiny_T64_H256_E8_K2_F512", T=64, H=256, E=8, K=2, F=512)
QWEN3_30B_A3B_PREFILL = MoEConfig("qwen3_30b_a3b_prefill_T4096_H2048_E128_K8_F768",
                                  T=4096, H=2048, E=128, K=8, F=768)
DEEPSEEK_R1_PREFILL = MoEConfig("deepseek_r1_prefill_T8192_H7168_E256_K8_F2048_P8",
                                T=8192, H=7168, E=256, K=8, F=2048, P=8)
DEEPSEEK_R1_DECODE = MoEConfig("deepseek_r1_decode_T128_H7168_E256_K8_F2048_zipf1.1",
                               T=128, H=7168, E=256, K=8, F=2048, zipf_s=1.1)
LATENT_896E = MoEConfig("latent_T4096_D7168_H2048_E896_K16_F1024_P64",
                        T=4096, H=2048, E=896, K=16, F=1024, P=64, d_model=7168)

ALL = {c.name: c for c in (TINY, QWEN3_30B_A3B_PREFILL, DEEPSEEK_R1_PREFILL,
                           DEEPSEEK_R1_DECODE, LATENT_896E)}
SHORT = {"tiny": TINY, "qwen3": QWEN3_30B_A3B_PREFILL, "r1_prefill": DEEPSEEK_R1_PREFILL,
         "r1_decode": DEEPSEEK_R1_DECODE, "latent": LATENT_896E}


def get(name: str) -> MoEConfig:
    if name in SHORT:
        return SHORT[name]
    return ALL[name]
