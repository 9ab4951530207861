"""The five synthetic DSA workloads (shapes, dtypes, seeds).

Shapes follow the pages: the indexer width/heads and top-k of the A.X-K2 DSA layer
(index_head_dim, index_n_heads, index_topk), the MLA head widths qk_nope + qk_rope / v of
the DeepSeek-V2 attention parameter guide, and the DSA-SWA-SWA hybrid with a 512-token
window of the openPangu-2.0 report (§3.2).
"""
from __future__ import annotations

from dataclasses import dataclass


@dataclass(frozen=True)
class DSAConfig:
    name: str
    B: int            # batch rows
    S: int            # queries per row
    T: int            # keys per row (queries are the last S positions: q_off = T - S)
    HI: int           # indexer heads
    DI: int           # indexer head dim
    scale: float      # indexer softmax_scale
    K: int            # top-k
    H: int            # attention heads
    d_nope: int       # qk_nope_head_dim
    d_rope: int       # qk_rope_head_dim
    dv: int           # v_head_dim
    dtype: str        # "f32" or "bf16"
    gate: str         # "off" or "sigmoid"
    seed: int
    swa_layers: int = 0   # extra sliding-window layers (hybrid block)
    swa_kv_heads: int = 0
    window: int = 0
    description: str = ""

    @property
    def dqk(self) -> int:
        return self.d_nope + self.d_rope

    @property
    def q_off(self) -> int:
        return self.T - self.S

    @property
    def k_eff(self) -> int:
        return min(self.K, self.T)


CONFIGS = {
    "c1": DSAConfig("c1", 1, 256, 256, 4, 32, 1.0 / 8, 16, 4, 32, 32, 64, "f32", "off", 0,
                    description="tiny DSA forward, fp32, S=256"),
    "c2": DSAConfig("c2", 1, 4096, 4096, 16, 64, 2.0 ** -4, 512, 20, 64, 64, 128, "bf16", "off",
                    1, description="DSA prefill, bf16, S=4096, MLA 20 heads 64+64/128"),
    "c3": DSAConfig("c3", 1, 32768, 32768, 32, 128, 2.0 ** -5, 2048, 32, 128, 64, 128, "bf16",
                    "sigmoid", 2, description="long DSA prefill, bf16, S=32768, gated"),
    "c4": DSAConfig("c4", 64, 1, 131072, 32, 128, 2.0 ** -5, 2048, 32, 128, 64, 128, "bf16",
                    "off", 3, description="DSA decode, bf16, batch 64 x 1 query, 131072 cached"),
    "c5": DSAConfig("c5", 1, 65536, 65536, 32, 128, 2.0 ** -5, 2048, 32, 128, 64, 128, "bf16",
                    "sigmoid", 4, swa_layers=2, swa_kv_heads=8, window=512,
                    description="hybrid DSA-SWA-SWA block, bf16, S=65536, gated"),
}


def get_config(name: str) -> DSAConfig:
    try:
        return CONFIGS[name]
    except KeyError:
        raise ValueError(f"unknown config {name!r}; known: {sorted(CONFIGS)}") from None
