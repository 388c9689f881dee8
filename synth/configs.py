"""Workload shapes of the Ideogram 4 DiT block.

The full-width model follows the "Model spec" table of the Ideogram 4.0 survey
page (emb_dim 4608, 18 heads, intermediate 12288, adaln_dim 512,
mrope_section (24, 20, 20), rope_theta 5e6, 128 latent channels, at most 2048
text tokens, 256-2048 px per side in multiples of 16, aspect ratio up to 6:1,
a 1024 px image = a 64 x 64 token grid).  The tiny width is a test size.
"""

from __future__ import annotations

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class Config:
    name: str
    B: int
    T_text: int
    grid_t: int
    grid_h: int
    grid_w: int
    D: int = 4608
    H: int = 18
    head_dim: int = 256
    I: int = 12288
    adaln_dim: int = 512
    rope_theta: float = 5.0e6
    sections: tuple = (24, 20, 20)
    eps: float = 1e-6
    x_dtype: str = "bf16"     # residual stream storage: "f32" or "bf16"
    w_dtype: str = "bf16"     # linear weight storage: "bf16", "e4m3" or "nvfp4_mixed"
    n_blocks: int = 1         # > 1 only for the stack workload
    latent_ch: int = 128

    @property
    def L(self) -> int:
        return self.T_text + self.grid_t * self.grid_h * self.grid_w

    @property
    def n_img(self) -> int:
        return self.grid_t * self.grid_h * self.grid_w

    @property
    def M(self) -> int:
        return self.B * self.L

    def with_(self, **kw) -> "Config":
        return replace(self, **kw)


CONFIGS = {
    # tiny single block: fp32 residual stream in/out, bf16 compute
    "tiny": Config("tiny", B=1, T_text=32, grid_t=1, grid_h=8, grid_w=8, D=1024, H=4, I=2816,
                   x_dtype="f32"),
    # full width, 512 px: 128 text + 32x32 image tokens
    "512px": Config("512px", B=1, T_text=128, grid_t=1, grid_h=32, grid_w=32),
    # full width, 1024 px: 512 text + 64x64 image tokens (the measured workload)
    "1024px": Config("1024px", B=1, T_text=512, grid_t=1, grid_h=64, grid_w=64),
    "1024px_fp8": Config("1024px_fp8", B=1, T_text=512, grid_t=1, grid_h=64, grid_w=64,
                         w_dtype="e4m3"),
    # full width, largest size: 2048 text + 128x128 image tokens
    "2048px": Config("2048px", B=1, T_text=2048, grid_t=1, grid_h=128, grid_w=128),
    # 6:1 aspect, 2048 x 352 px: 2048 text + 128x22 image tokens
    "2048x352": Config("2048x352", B=1, T_text=2048, grid_t=1, grid_h=128, grid_w=22),
    # one denoiser step of the 34-block stack, FP8 weights, batch 2 at 1024 px
    "stack_1024px_fp8": Config("stack_1024px_fp8", B=2, T_text=512, grid_t=1, grid_h=64,
                               grid_w=64, w_dtype="e4m3", n_blocks=34),
    # one sampler step at 1024 px: the conditional 34-block stack over 512 text +
    # 64x64 image tokens and the separate image-only unconditional stack, FP8
    "step_1024px_fp8": Config("step_1024px_fp8", B=1, T_text=512, grid_t=1, grid_h=64,
                              grid_w=64, w_dtype="e4m3", n_blocks=34),
    # the block's FFN linears with NVFP4 weights (the NVFP4 Mixed scheme keeps
    # the attention projections in FP8): gate/up and down at 1024 px
    "ffn_1024px_nvfp4": Config("ffn_1024px_nvfp4", B=1, T_text=512, grid_t=1, grid_h=64,
                               grid_w=64, w_dtype="nvfp4"),
    # the whole block with the NVFP4 Mixed weights: FFN linears in NVFP4, the
    # AdaLN and attention projections in FP8 (1024 px, and a small case with
    # 64 text + 12x12 image tokens at D = 1024)
    "1024px_nvfp4": Config("1024px_nvfp4", B=1, T_text=512, grid_t=1, grid_h=64, grid_w=64,
                           w_dtype="nvfp4_mixed"),
    "small_nvfp4": Config("small_nvfp4", B=1, T_text=64, grid_t=1, grid_h=12, grid_w=12, D=1024,
                          H=4, I=2816, w_dtype="nvfp4_mixed"),
    # the text conditioning projection of a 2048-token caption (13 x 4096 = 53248
    # raw features per token -> 4608), FP8 weights as released
    "textcond_2048_fp8": Config("textcond_2048_fp8", B=1, T_text=2048, grid_t=1, grid_h=0,
                                grid_w=0, w_dtype="e4m3"),
}


def get_config(name: str) -> Config:
    return CONFIGS[name]
