"""Workload shapes for the FusedBitLinear projection, named by model size and regime.

Shapes follow the HGRNBit model zoo described on the pages (hidden size per model size, 24 or
32 layers) and the block layout: four attention-side projections H -> H (i, f, g, o), the MLP
gate_proj H -> 2I whose output feeds the SiLU-GLU, and down_proj I -> H.  I is the GLU half
width (2816 / 5632 / 7040 for hidden 1024 / 2048 / 2560).
"""
from dataclasses import dataclass, field
from typing import List, Tuple


@dataclass(frozen=True)
class Projection:
    name: str       # i_proj, f_proj, g_proj, o_proj, gate_proj, down_proj, proj
    K: int          # in_features
    N: int          # out_features (2I for gate_proj)
    glu: bool       # SiLU-GLU epilogue (gate_proj only): output is T x N/2
    src: str        # which activation feeds it: x_attn, x_o, x_mlp, h (the GLU output)


def block(H: int, I: int) -> Tuple[Projection, ...]:
    return (
        Projection("i_proj", H, H, False, "x_attn"),
        Projection("f_proj", H, H, False, "x_attn"),
        Projection("g_proj", H, H, False, "x_attn"),
        Projection("o_proj", H, H, False, "x_o"),
        Projection("gate_proj", H, 2 * I, True, "x_mlp"),
        Projection("down_proj", I, H, False, "h"),
    )


@dataclass(frozen=True)
class Workload:
    name: str
    T: int                          # tokens per step
    layers: int                     # distinct layers whose weights one step streams
    projections: Tuple[Projection, ...]
    x_dtype: str = "f16"            # activations in
    y_dtype: str = "f16"            # projection outputs
    outlier_frac: float = 0.0       # fraction of activation entries scaled by outlier_scale
    outlier_scale: float = 20.0
    w_std: float = 0.02
    notes: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def weights_per_layer(self) -> int:
        return sum(p.N * p.K for p in self.projections)

    @property
    def packed_bytes_per_layer(self) -> int:
        return self.weights_per_layer // 4


TINY = Workload("tiny_single_t16", 16, 1, (Projection("proj", 256, 512, False, "x_attn"),),
                x_dtype="f32", y_dtype="f32",
                notes="single FusedBitLinear 256->512, 16 tokens, fp32 in/out")

HGRN_370M_T64 = Workload("hgrn370m_block_t64", 64, 1, block(1024, 2816),
                         notes="370M-shaped block projections, hidden 1024, 64 tokens")


def hgrn_1p3b_decode(T: int) -> Workload:
    return Workload(f"hgrn1p3b_decode_t{T}", T, 24, block(2048, 5632),
                    notes="1.3B-shaped decode, 24 layers of packed weights per step")


HGRN_1P3B_PREFILL = Workload("hgrn1p3b_prefill_t32768", 32768, 1, block(2048, 5632),
                             outlier_frac=0.01, outlier_scale=20.0,
                             notes="1.3B-shaped prefill, 16 x 2048 tokens, 1% outliers x20")

HGRN_2P7B_DECODE_T8 = Workload("hgrn2p7b_decode_t8", 8, 32, block(2560, 7040),
                               notes="2.7B-shaped decode, 8 tokens, 32 layers")
HGRN_2P7B_PREFILL = Workload("hgrn2p7b_prefill_t8192", 8192, 1, block(2560, 7040),
                             notes="2.7B-shaped prefill, 8192 tokens, one layer")

WORKLOADS = {w.name: w for w in [
    TINY, HGRN_370M_T64,
    hgrn_1p3b_decode(1), hgrn_1p3b_decode(8), hgrn_1p3b_decode(64),
    HGRN_1P3B_PREFILL, HGRN_2P7B_DECODE_T8, HGRN_2P7B_PREFILL,
]}

# the largest configuration that fits one GPU: the benchmark's headline workload
DEFAULT = HGRN_1P3B_PREFILL.name
# the decode configurations the benchmark reports beside it (HBM-bound regime)
DECODE_SUITE = ("hgrn1p3b_decode_t1", "hgrn1p3b_decode_t8", "hgrn1p3b_decode_t64",
                "hgrn2p7b_decode_t8")
