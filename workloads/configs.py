"""Workload shapes.

The five benchmark workloads are the synthetic single-layer shapes the MHA2MLA
decode path is measured on: a tiny fp32 layer, a SmolLM-135M-shaped GQA layer
and three Llama-2-7B-shaped layers (bf16 latent d_c=256; ragged long context
with d_c=64; int4 latent with d_c=128).  The models the pages evaluate are
SmolLM and Llama-2-7B (GitHub README "MHA2MLA", §Models); their hidden sizes,
head counts and head dims are the public architecture figures of those models.

PARITY_WORKLOADS are reduced shapes with the same head geometry, small enough
for the float64 oracle to check every output, yet spanning several 64/128-token
tiles and a ragged tail.
"""

from dataclasses import dataclass, field, replace
from typing import Optional, Tuple


@dataclass(frozen=True)
class Workload:
    name: str
    dtype: str                 # arithmetic/storage dtype of weights, activations, cache: "f32" | "bf16"
    cache: str                 # latent cache encoding: "same" (dtype) | "int4_g32" | "int2_g32"
    hidden: int                # d
    n_heads: int               # H
    n_kv_heads: int            # n_kv
    head_dim: int              # d_h
    r_pairs: int               # r: RoPE frequency pairs kept per KV head
    d_c: int                   # joint latent width
    batch: int                 # B
    ctx: Optional[int]         # fixed context length L (None => ragged)
    ctx_range: Optional[Tuple[int, int]] = None   # inclusive U[lo, hi] for ragged lengths
    t_cal: int = 1024          # calibration tokens for the 2-norm statistics
    rope_base: float = 10000.0
    seed: int = 0
    fixed_lens: Optional[Tuple[int, ...]] = field(default=None)  # explicit lengths (parity cases)
    resid: int = 0             # int4 cache: unquantised residual window of the most recent tokens (0 or 128)

    @property
    def group(self) -> int:
        return self.n_heads // self.n_kv_heads

    @property
    def rope_width(self) -> int:
        """Retained RoPE key dims per token: n_kv * 2r."""
        return self.n_kv_heads * 2 * self.r_pairs

    @property
    def nope_dim(self) -> int:
        return self.head_dim - 2 * self.r_pairs

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = [
    Workload("tiny_f32", "f32", "same", hidden=128, n_heads=4, n_kv_heads=4, head_dim=32,
             r_pairs=2, d_c=32, batch=1, ctx=64, t_cal=256),
    Workload("smollm135m_gqa_bf16", "bf16", "same", hidden=576, n_heads=9, n_kv_heads=3,
             head_dim=64, r_pairs=4, d_c=32, batch=16, ctx=2048),
    Workload("llama2_7b_bf16", "bf16", "same", hidden=4096, n_heads=32, n_kv_heads=32,
             head_dim=128, r_pairs=4, d_c=256, batch=32, ctx=4096),
    Workload("llama2_7b_ragged_bf16", "bf16", "same", hidden=4096, n_heads=32, n_kv_heads=32,
             head_dim=128, r_pairs=4, d_c=64, batch=8, ctx=None, ctx_range=(1024, 32768)),
    Workload("llama2_7b_int4", "bf16", "int4_g32", hidden=4096, n_heads=32, n_kv_heads=32,
             head_dim=128, r_pairs=4, d_c=128, batch=64, ctx=8192),
]

# Reduced shapes for element-by-element parity against the oracle.  Head geometry
# matches the workloads above; hidden is cut so the SVD and prefill stay fast.
# Lengths include 1 (single cached token), a tail that is not a tile multiple,
# and an empty sequence where the cache layout allows it.
PARITY_WORKLOADS = [
    WORKLOADS[0],
    WORKLOADS[1].with_(name="smollm_gqa_small", batch=3, ctx=None, fixed_lens=(300, 1, 777), t_cal=512),
    WORKLOADS[2].with_(name="llama_dc256_small", hidden=512, batch=3, ctx=None,
                       fixed_lens=(1000, 1, 333), t_cal=512),
    WORKLOADS[3].with_(name="llama_dc64_ragged_small", hidden=512, batch=4, ctx=None,
                       ctx_range=None, fixed_lens=(2500, 129, 64, 1), t_cal=512),
    WORKLOADS[4].with_(name="llama_int4_small", hidden=512, batch=3, ctx=None,
                       fixed_lens=(700, 65, 1), t_cal=512),
    # the int4 cache with the 128-token residual window: a window across a tile boundary, a
    # window covering the whole sequence, a single token; 32 heads and 9 GQA heads
    WORKLOADS[4].with_(name="llama_int4_r128_small", hidden=512, batch=4, ctx=None,
                       fixed_lens=(700, 200, 128, 1), t_cal=512, resid=128),
    WORKLOADS[1].with_(name="smollm_int4_r128_small", cache="int4_g32", batch=3, ctx=None,
                       fixed_lens=(300, 129, 5), t_cal=512, resid=128),
    # the 2-bit latent cache
    WORKLOADS[4].with_(name="llama_int2_small", cache="int2_g32", hidden=512, batch=3, ctx=None,
                       fixed_lens=(700, 65, 1), t_cal=512),
]

# The int4 workload as the pages deploy the 4-bit cache: with a residual window of the 128
# most recent tokens kept unquantised (README "MHA2MLA", LongBench evaluation of the
# quantised cache).
EXTRA_WORKLOADS = [
    WORKLOADS[4].with_(name="llama2_7b_int4_r128", resid=128),
    # the same shape with the 2-bit latent (Notes §关键设计: 4- or 2-bit quantisation of the latent)
    WORKLOADS[4].with_(name="llama2_7b_int2", cache="int2_g32"),
]


def get(name_or_index) -> Workload:
    if isinstance(name_or_index, int):
        return WORKLOADS[name_or_index]
    for w in WORKLOADS + PARITY_WORKLOADS + EXTRA_WORKLOADS:
        if w.name == name_or_index:
            return w
    raise KeyError(name_or_index)
