"""Named layer workloads: the shapes of the models the pages serve and train.

Each entry is one MoE layer (one fused gate_up stack and one fused down stack)
with its routing, token counts and synthetic-input recipe.  Weights are
random (there are no checkpoints here); only the shapes and value
distributions follow the models.
"""
from dataclasses import dataclass, field
from typing import Optional, Tuple


@dataclass(frozen=True)
class Workload:
    name: str
    fmt: str                     # "nf4" or "mxfp4"
    E: int                       # experts
    H: int                       # hidden size
    I: int                       # expert intermediate size (gate_up has 2I outputs)
    k: int                       # experts per token
    tokens: Tuple[int, ...]      # token counts T the layer is run at
    exp_range: Tuple[int, int] = (-4, 2)   # MXFP4: E8M0 exponent range of the scales
    weight_std: float = 0.02              # NF4: std of the fp32 weights before quantisation
    lora_rank: int = 0
    lora_alpha: float = 0.0
    zipf_s: Optional[float] = None        # skewed routing when set
    glu: Optional[Tuple[float, float, float]] = None   # clamped GLU (alpha, limit, beta); None = SwiGLU
    bias_std: float = 0.0                 # > 0: per-expert fp32 biases N(0, bias_std) on both stacks
    interleaved: bool = False             # gate_up drawn with gate/up rows interleaved, de-interleaved at load
    gating: str = "topk"                  # router weights: "topk" (softmax over the picks) or "all"
    absmax_dq: bool = False               # NF4: absmax stored double-quantised (nested form)
    zero_block_every: int = 0             # NF4: every n-th 64-value block of the fp32 weights is zero
    scales: str = "uniform"               # MXFP4: "uniform" (exp_range) or "extreme" (synth.expert_mxfp4_extreme)
    seed: int = 0
    notes: str = field(default="", compare=False)

    @property
    def lora_scale(self):
        return self.lora_alpha / self.lora_rank if self.lora_rank else 0.0

    def gate_up_bytes_per_expert(self):
        n = 2 * self.I * self.H
        return n // 2 + (n // 64 * 4 if self.fmt == "nf4" else n // 32)

    def down_bytes_per_expert(self):
        n = self.I * self.H
        return n // 2 + (n // 64 * 4 if self.fmt == "nf4" else n // 32)

    def flops(self, T):
        """Algorithmic flops of one forward: real routed rows only, no padding."""
        R = T * self.k
        f = 2 * R * (self.H * 2 * self.I + self.I * self.H)
        if self.lora_rank:
            f += 2 * R * (self.H * self.lora_rank + self.lora_rank * 2 * self.I)
        return f


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny_mxfp4", "mxfp4", E=8, H=256, I=128, k=2, tokens=(64,), exp_range=(-4, 2),
                 notes="tiny MXFP4 layer for correctness"),
        Workload("qwen3_30b_a3b_nf4_decode", "nf4", E=128, H=2048, I=768, k=8, tokens=(1, 8, 32, 64),
                 notes="Qwen3-30B-A3B-shaped NF4 layer, decode batches"),
        Workload("qwen3_30b_a3b_nf4_lora", "nf4", E=128, H=2048, I=768, k=8, tokens=(512,),
                 lora_rank=8, lora_alpha=16.0,
                 notes="Qwen3-30B-A3B-shaped NF4 layer with per-expert LoRA r=8 alpha=16 on gate_up"),
        Workload("gptoss_20b_mxfp4", "mxfp4", E=32, H=2880, I=2880, k=4, tokens=(1, 16, 4096),
                 exp_range=(-6, 1), notes="gpt-oss-20b-shaped MXFP4 layer"),
        Workload("gptoss_120b_mxfp4_zipf", "mxfp4", E=128, H=2880, I=2880, k=4, tokens=(16384,),
                 exp_range=(-6, 1), zipf_s=1.1,
                 notes="gpt-oss-120b-shaped MXFP4 layer, prefill, Zipf(1.1)-skewed expert load"),
    ]
}
