"""Layer shapes: the five synthetic MoE layers plus the smaller shapes the parity tests use.

A shape is plain data (sizes, activation, gate normalisation, capacity factor, dtype, how the
synthetic logit bias is drawn).  Nothing here computes any part of the layer.

The five named layers stand in for the models the pages measure on (GPT-2, BERT-Large, Mixtral
and DeepSeek-V2 style expert shapes: FlowMoE notes, results table; FSMoE summary, abstract), with
random weights of those shapes: no dataset or trained checkpoint is involved.
"""
from __future__ import annotations

from dataclasses import dataclass, replace
from typing import Optional

GELU = 0
SWIGLU = 1

FP32 = 0
BF16 = 1

# capacity sentinel meaning "no capacity limit" (dropless routing); mirrors MOE_DROPLESS in moe.h
DROPLESS = 2**31 - 1


@dataclass(frozen=True)
class LayerShape:
    name: str
    T: int                    # tokens in the batch
    d: int                    # hidden (model) dimension
    E: int                    # routed experts
    k: int                    # experts chosen per token
    d_ff: int                 # expert FFN inner dimension
    n_shared: int = 0         # always-on shared experts (every token, weight 1, no capacity)
    act: int = GELU           # GELU (erf form) or SwiGLU
    gate_norm: int = 0        # 0: softmax over all E logits; 1: softmax over the k selected logits
    capacity_factor: Optional[float] = 1.25   # None: dropless
    dtype: int = BF16
    bias: str = "none"        # synthetic per-expert logit offset: "none" | "zipf" | "normal"
    fwd_only: bool = False
    aux_loss_coef: float = 0.0   # weight of the load-balancing loss (0: not computed)
    choice_major: bool = False   # drop priority: all first choices, then second, ... (else token order)

    @property
    def E_tot(self) -> int:
        return self.E + self.n_shared

    @property
    def dropless(self) -> bool:
        return self.capacity_factor is None

    def with_(self, **kw) -> "LayerShape":
        return replace(self, **kw)


# The five layers, in order.  Workload text for each is in the dict below.
SWITCH_TINY = LayerShape("switch_tiny", T=256, d=64, E=4, k=1, d_ff=128, act=GELU, gate_norm=0,
                         capacity_factor=1.25, dtype=FP32, fwd_only=True)
GPT2_GSHARD = LayerShape("gpt2_gshard", T=4096, d=768, E=16, k=2, d_ff=3072, act=GELU,
                         gate_norm=0, capacity_factor=1.25, dtype=BF16)
BERT_LARGE_SKEW = LayerShape("bert_large_skew", T=8192, d=1024, E=32, k=2, d_ff=4096, act=GELU,
                             gate_norm=0, capacity_factor=1.0, dtype=BF16, bias="zipf")
MIXTRAL_DROPLESS = LayerShape("mixtral_dropless", T=16384, d=4096, E=8, k=2, d_ff=14336,
                              act=SWIGLU, gate_norm=1, capacity_factor=None, dtype=BF16)
DEEPSEEK_V2 = LayerShape("deepseek_v2", T=16384, d=2048, E=64, k=6, d_ff=1408, n_shared=2,
                         act=SWIGLU, gate_norm=0, capacity_factor=1.5, dtype=BF16, bias="normal")

LAYERS = [SWITCH_TINY, GPT2_GSHARD, BERT_LARGE_SKEW, MIXTRAL_DROPLESS, DEEPSEEK_V2]
BY_NAME = {s.name: s for s in LAYERS}

WORKLOAD_TEXT = {
    "switch_tiny": "Switch top-1 fwd fp32 T=256 d=64 E=4 F=128 GELU cf=1.25",
    "gpt2_gshard": "GPT-2-style GShard top-2 fwd+bwd bf16 T=4096 d=768 E=16 F=3072 GELU cf=1.25",
    "bert_large_skew": "BERT-Large-style top-2 fwd+bwd bf16 T=8192 d=1024 E=32 F=4096 GELU cf=1.0 Zipf bias",
    "mixtral_dropless": "Mixtral-style dropless top-2 fwd+bwd bf16 T=16384 d=4096 E=8 SwiGLU F=14336",
    "deepseek_v2": "DeepSeek-V2-style top-6 of 64 + 2 shared fwd+bwd bf16 T=16384 d=2048 SwiGLU F=1408 cf=1.5",
}

# Reduced shapes, same structure as the five layers, small enough for the full (unsampled)
# oracle comparison in seconds.  Each spans several 128-row tiles with a ragged tail.
PARITY_SMALL = [
    SWITCH_TINY,
    LayerShape("gpt2_small", T=1000, d=256, E=8, k=2, d_ff=384, act=GELU, gate_norm=0,
               capacity_factor=1.25, dtype=BF16),
    LayerShape("bert_skew_small", T=1100, d=128, E=16, k=2, d_ff=512, act=GELU, gate_norm=0,
               capacity_factor=1.0, dtype=BF16, bias="zipf"),
    LayerShape("mixtral_small", T=777, d=256, E=4, k=2, d_ff=640, act=SWIGLU, gate_norm=1,
               capacity_factor=None, dtype=BF16),
    LayerShape("deepseek_small", T=600, d=128, E=16, k=6, d_ff=192, n_shared=2, act=SWIGLU,
               gate_norm=0, capacity_factor=1.5, dtype=BF16, bias="normal"),
]

# fp32 shapes: the GPU's fp32 path is held to the tight fp32 tolerance, which pins the
# backward formulas on the device as closely as the oracle's own finite differences do.
PARITY_FP32 = [
    LayerShape("fp32_gelu", T=300, d=64, E=4, k=2, d_ff=96, act=GELU, gate_norm=0,
               capacity_factor=1.0, dtype=FP32, bias="zipf"),
    LayerShape("fp32_swiglu_shared", T=200, d=32, E=6, k=3, d_ff=48, n_shared=1, act=SWIGLU,
               gate_norm=0, capacity_factor=1.25, dtype=FP32, bias="normal"),
    LayerShape("fp32_renorm_dropless", T=150, d=48, E=5, k=2, d_ff=40, act=SWIGLU, gate_norm=1,
               capacity_factor=None, dtype=FP32),
]
