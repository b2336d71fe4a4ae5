"""The synthetic workloads the layer is checked and measured on.

Shapes follow the pages' workloads: a Switch-Base FFN slot (d_model 768, d_ff
3072; "From Switch Transformer to GLaM" and the Switch results pages), a
sparsely-gated top-2 layer, a skewed-routing overflow stress, and a
Mixtral-shaped SwiGLU layer (d_model 4096, d_ff 14336, 8 experts, top-2; CMU
10-423 Lecture 16 section 3 and exercise 1).  The capacity C is not stored here:
it is computed from (T, N, k, cf) by the library's ``moe_capacity``.
"""
from dataclasses import dataclass, replace
from typing import Optional


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d_model: int
    d_ff: int
    n_experts: int
    top_k: int
    capacity_factor: float
    act: str            # "relu" | "swiglu"
    dtype: str          # "f32" | "bf16"
    norm: str           # "layernorm" | "rmsnorm"
    biases: bool = False
    zipf_exponent: Optional[float] = None   # router bias 3*ln(popularity), popularity ~ (i+1)^-s
    alpha: float = 1e-2
    seed: int = 0

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", T=512, d_model=64, d_ff=256, n_experts=8, top_k=1,
                         capacity_factor=1.0, act="relu", dtype="f32", norm="layernorm",
                         biases=True),
    "switch_base": Workload("switch_base", T=65536, d_model=768, d_ff=3072, n_experts=64,
                            top_k=1, capacity_factor=1.25, act="relu", dtype="bf16",
                            norm="layernorm"),
    "top2": Workload("top2", T=32768, d_model=1024, d_ff=4096, n_experts=32, top_k=2,
                     capacity_factor=2.0, act="relu", dtype="bf16", norm="layernorm"),
    "skew": Workload("skew", T=65536, d_model=768, d_ff=3072, n_experts=128, top_k=1,
                     capacity_factor=1.0, act="relu", dtype="bf16", norm="layernorm",
                     zipf_exponent=1.2),
    "mixtral": Workload("mixtral", T=16384, d_model=4096, d_ff=14336, n_experts=8, top_k=2,
                        capacity_factor=1.25, act="swiglu", dtype="bf16", norm="rmsnorm"),
}

ORDER = ["tiny_f32", "switch_base", "top2", "skew", "mixtral"]
