"""Model shapes for the oracle (its own copy; the CUDA library has another).

Notation (per expert): N blocks, widths d_v / d_a, H heads of Dh channels
(A = H*Dh), FFN widths F_v / F_a, L_c conditioning + L_vid video tokens
(L_v = L_c + L_vid), L_a action tokens of dimension P_a, batch B.

The presets are the synthetic MoT shapes the method is benchmarked on:
1 tiny fp32 check model; 2 a Fast-WAM-shaped one-step model; 3 the same with a
10-step Euler teacher schedule; 4 batch 8 with 8-frame video; 5 a
Flash-WAM-like joint one-step model with patch input, consistency endpoints
and a rank-128 LoRA on the action expert.  The Fast-WAM page gives no depth
or widths, so all shapes are synthetic stand-ins.
"""
from __future__ import annotations

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class WamConfig:
    n_blocks: int
    d_video: int
    d_action: int
    n_heads: int
    head_dim: int
    ffn_video: int
    ffn_action: int
    l_cond: int
    l_video: int
    l_action: int
    action_dim: int = 30
    video_patch_dim: int = 0      # 0: video tokens arrive embedded at d_video
    batch: int = 1
    lora_rank: int = 0
    lora_scale: float = 1.0
    video_has_output: bool = False  # joint variant: video endpoint is produced
    dtype: str = "fp32"           # "fp32" or "bf16" (parameter rounding)
    default_steps: int = 1

    @property
    def attn_dim(self) -> int:
        return self.n_heads * self.head_dim

    @property
    def l_v(self) -> int:
        return self.l_cond + self.l_video

    def with_(self, **kw) -> "WamConfig":
        return replace(self, **kw)


_FASTWAM = dict(n_blocks=28, d_video=1536, d_action=768, n_heads=24, head_dim=64,
                ffn_video=6144, ffn_action=3072, l_cond=64, l_video=1024, l_action=32,
                dtype="bf16")

PRESETS = {
    1: WamConfig(n_blocks=2, d_video=64, d_action=64, n_heads=4, head_dim=16,
                 ffn_video=256, ffn_action=256, l_cond=0, l_video=64, l_action=16,
                 dtype="fp32"),
    2: WamConfig(**_FASTWAM),
    3: WamConfig(**_FASTWAM, default_steps=10),
    4: WamConfig(**{**_FASTWAM, "l_video": 2048, "batch": 8}),
    5: WamConfig(n_blocks=30, d_video=1536, d_action=1536, n_heads=24, head_dim=64,
                 ffn_video=6144, ffn_action=6144, l_cond=0, l_video=1024, l_action=16,
                 video_patch_dim=192, lora_rank=128, lora_scale=1.0,
                 video_has_output=True, dtype="bf16"),
}


def preset(k: int) -> WamConfig:
    return PRESETS[k]
