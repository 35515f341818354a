"""The five LISA workloads, as shapes and generation parameters.

Shapes follow the Qwen2.5-1.5B / 7B attention geometry named on the LISA pages
(arXiv 2607.19358, abstract: DeepSeek-distilled Qwen models; experiment design
in the gptget.net digest: M = 256).  The indexer geometry (4 heads of dim 64)
and every distribution below are stated definitions of this library, because
the pages give neither.

Dimension names:
  B     batch (independent sequences)
  Hq    query heads, Hkv key/value heads, G = Hq / Hkv query heads per KV head
  d     head dim of q / k / v
  HI    indexer heads, R = HI / Hkv indexer heads per KV head
  dI    indexer head dim
  M     tokens kept by the top-M selection
"""

from dataclasses import dataclass, field


@dataclass(frozen=True)
class LisaConfig:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    HI: int
    dI: int
    M: int
    dtype: str                 # "bf16" or "fp32": storage dtype of q/k/v/caches/out
    kind: str                  # "prefill_decode" | "decode" | "prefill" | "ragged_decode" | "long_decode"
    seed: int
    T: int = 0                 # prefill length (kind prefill / prefill_decode)
    n_decode: int = 0          # decode steps (prefill_decode / long_decode)
    L: int = 0                 # decode: tokens in the cache including the new one
    L_lo: int = 0              # ragged_decode: per-sequence L drawn uniformly in [L_lo, L_hi]
    L_hi: int = 0
    layers: int = 1            # long_decode: independent stacked layers
    S0: str = "zeros"          # initial linear state: "zeros" or "normal" (N(0,1))
    description: str = field(default="", compare=False)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def R(self) -> int:
        return self.HI // self.Hkv

    @property
    def L_max(self) -> int:
        """Rows every cache buffer holds."""
        if self.kind == "prefill_decode":
            return self.T + self.n_decode
        if self.kind == "prefill":
            return self.T
        if self.kind == "decode":
            return self.L
        if self.kind == "ragged_decode":
            return self.L_hi
        if self.kind == "long_decode":
            return self.L + self.n_decode
        raise ValueError(self.kind)


CONFIGS = {
    "tiny_fp32": LisaConfig(
        name="tiny_fp32", B=1, Hq=2, Hkv=1, d=64, HI=1, dI=32, M=32, dtype="fp32",
        kind="prefill_decode", seed=0, T=512, n_decode=16, S0="zeros",
        description="tiny single layer, fp32: causal prefill of 512 tokens then 16 decode steps",
    ),
    "decode_1p5b_16k": LisaConfig(
        name="decode_1p5b_16k", B=1, Hq=12, Hkv=2, d=128, HI=4, dI=64, M=256, dtype="bf16",
        kind="decode", seed=1, L=16384, S0="normal",
        description="Qwen2.5-1.5B-shaped single-layer decode step at 16384 cached tokens",
    ),
    "prefill_1p5b_16k": LisaConfig(
        name="prefill_1p5b_16k", B=1, Hq=12, Hkv=2, d=128, HI=4, dI=64, M=256, dtype="bf16",
        kind="prefill", seed=2, T=16384, S0="zeros",
        description="Qwen2.5-1.5B-shaped causal prefill of 16384 tokens",
    ),
    "ragged_7b_b32": LisaConfig(
        name="ragged_7b_b32", B=32, Hq=28, Hkv=4, d=128, HI=4, dI=64, M=256, dtype="bf16",
        kind="ragged_decode", seed=3, L_lo=4096, L_hi=16384, S0="normal",
        description="Qwen2.5-7B-shaped batched decode step, per-sequence length uniform in [4096, 16384]",
    ),
    "longcot_7b_28l": LisaConfig(
        name="longcot_7b_28l", B=8, Hq=28, Hkv=4, d=128, HI=4, dI=64, M=256, dtype="bf16",
        kind="long_decode", seed=4, L=16384, n_decode=1024, layers=28, S0="normal",
        description="Qwen2.5-7B-shaped 28 independent layers, 16384 prefilled rows, 1024 decode steps",
    ),
}

# Positional order of the workloads (index = seed).
CONFIG_ORDER = ["tiny_fp32", "decode_1p5b_16k", "prefill_1p5b_16k", "ragged_7b_b32", "longcot_7b_28l"]


def get_config(key) -> LisaConfig:
    if isinstance(key, int):
        return CONFIGS[CONFIG_ORDER[key]]
    return CONFIGS[key]
