"""The five synthetic layer shapes this library is measured and checked on.

T tokens, hidden size d, N_r routed experts with K of them active per token,
N_s shared experts, SwiGLU intermediate size I.  The V3 shape (d 7168, 256
routed experts, 8 active, 1 shared, I 2048) is the DeepSeek-V3 layer that the
"DeepSeek-V3 技術報告" summary describes in section 核心概念 (1 shared + 256
routed experts, 8 active).
"""
from dataclasses import dataclass, replace


@dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int
    d: int
    N_r: int
    K: int
    N_s: int
    I: int
    dtype: str            # "f32" | "bf16" | "e4m3" (FFN arithmetic); router stays f32/bf16
    seed: int
    bias: str = "zero"    # "zero" | "uniform" (U(-0.01, 0.01))
    zipf: float = 0.0     # > 0: expert popularity skewed to Zipf(zipf) (input recipe)
    steps: int = 1        # forward + bias-update steps per run
    outlier_frac: float = 0.0
    outlier_scale: float = 1.0
    n_groups: int = 1        # > 1: expert groups for the per-token group (node) limit
    topk_groups: int = 1     # groups a token may use when n_groups > 1

    @property
    def R(self):
        return self.T * self.K

    def flops(self):
        """Algorithmic FLOPs of one forward: router logits + routed + shared SwiGLU FFNs."""
        return 2 * self.T * self.d * self.N_r + (self.K + self.N_s) * self.T * 6 * self.d * self.I

    def weight_bytes(self):
        el = 1 if self.dtype == "e4m3" else (4 if self.dtype == "f32" else 2)
        return (self.N_r + self.N_s) * 3 * self.I * self.d * el

    def with_T(self, T):
        return replace(self, T=T)


CONFIGS = {
    "tiny_f32": LayerConfig("tiny_f32", T=128, d=256, N_r=16, K=4, N_s=1, I=128,
                            dtype="f32", seed=0),
    "small_bf16": LayerConfig("small_bf16", T=4096, d=2048, N_r=64, K=6, N_s=2, I=1408,
                              dtype="bf16", seed=1, bias="uniform"),
    "v3_bf16": LayerConfig("v3_bf16", T=8192, d=7168, N_r=256, K=8, N_s=1, I=2048,
                           dtype="bf16", seed=2),
    "v3_zipf_bf16": LayerConfig("v3_zipf_bf16", T=8192, d=7168, N_r=256, K=8, N_s=1, I=2048,
                                dtype="bf16", seed=2, zipf=1.2, steps=100),
    # decode-shaped batch at the V3 shape: ~8 tokens per expert, so the expert
    # GEMMs stream all weights for little arithmetic (HBM-bound)
    "v3_decode_bf16": LayerConfig("v3_decode_bf16", T=256, d=7168, N_r=256, K=8, N_s=1, I=2048,
                                  dtype="bf16", seed=5),
    # V3 shape with the node limit: 8 groups of 32 experts, at most 4 per token
    "v3_grouped_bf16": LayerConfig("v3_grouped_bf16", T=8192, d=7168, N_r=256, K=8, N_s=1,
                                   I=2048, dtype="bf16", seed=6, n_groups=8, topk_groups=4),
    "v3_fp8": LayerConfig("v3_fp8", T=16384, d=7168, N_r=256, K=8, N_s=1, I=2048,
                          dtype="e4m3", seed=4, outlier_frac=0.001, outlier_scale=50.0),
}
