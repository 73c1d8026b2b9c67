"""Named MoE-layer shapes.

The five full-size layers:

* ``tiny_fp32``        T=256,   d=256,  E=16,  h=128,  k=4,  FP32
* ``dsmoe16b_bf16``    T=4096,  d=2048, E=64,  h=1408, k=6,  BF16  (DeepSeek-MoE-16B-like)
* ``dsv3_bf16``        T=8192,  d=7168, E=256, h=2048, k=8,  BF16  (DeepSeek-V3-like) + RBD map 8 experts/device, 4 devices/node
* ``dsv3_zipf_bf16``   as ``dsv3_bf16`` with a Zipf(s=1.1) per-expert logit bias (skewed load)
* ``finegrained_bf16`` T=16384, d=4096, E=512, h=512,  k=16, BF16  + RBD map 16 experts/device, 8 devices/node

Fine-grained expert segmentation (split each expert m ways, raise k by m) is the
architecture the X-MoE article (adg.csdn.net) describes in §1 "专家混合架构的技术演进与核心挑战";
``finegrained_bf16`` is the 1/m split with k=16 named there.

The ``small_*`` shapes are parity cases: BF16 layers the CPU oracle finishes in
seconds whose row counts span several 128-row GEMM tiles and end in ragged tails.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Optional


@dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int                 # tokens
    d: int                 # model (hidden) width
    E: int                 # routed experts
    h: int                 # expert FFN width (SwiGLU inner size)
    k: int                 # experts per token
    dtype: str             # "f32" or "bf16": storage type of x, W*, activations
    zipf_c: float = 0.0    # >0: add bias_e = -zipf_c * zipf_s * ln(perm(e) + 1) to the gate logits
    zipf_s: float = 1.1
    rbd_epd: Optional[int] = None   # RBD virtual map: experts per device
    rbd_dpn: Optional[int] = None   # RBD virtual map: devices per node
    note: str = field(default="", compare=False)

    @property
    def N(self) -> int:
        """Number of (token, expert) assignments = rows of the padding-free buffer."""
        return self.T * self.k

    @property
    def has_rbd(self) -> bool:
        return self.rbd_epd is not None and self.rbd_dpn is not None

    def with_(self, **kw) -> "LayerConfig":
        return replace(self, **kw)


CONFIGS = {
    "tiny_fp32": LayerConfig("tiny_fp32", T=256, d=256, E=16, h=128, k=4, dtype="f32",
                             note="tiny FP32 layer, random balanced gate"),
    "dsmoe16b_bf16": LayerConfig("dsmoe16b_bf16", T=4096, d=2048, E=64, h=1408, k=6, dtype="bf16",
                                 rbd_epd=8, rbd_dpn=4,
                                 note="DeepSeek-MoE-16B-like layer; RBD map reuses dsv3's 8 experts/device, 4 devices/node"),
    "dsv3_bf16": LayerConfig("dsv3_bf16", T=8192, d=7168, E=256, h=2048, k=8, dtype="bf16",
                             rbd_epd=8, rbd_dpn=4, note="DeepSeek-V3-like layer, balanced"),
    "dsv3_zipf_bf16": LayerConfig("dsv3_zipf_bf16", T=8192, d=7168, E=256, h=2048, k=8, dtype="bf16",
                                  zipf_c=1.5, note="DeepSeek-V3-like layer, Zipf(1.1) expert skew"),
    "finegrained_bf16": LayerConfig("finegrained_bf16", T=16384, d=4096, E=512, h=512, k=16, dtype="bf16",
                                    rbd_epd=16, rbd_dpn=8, note="fine-grained 1/m split, k=16"),
}

# Parity shapes the oracle runs in full on the CPU (seconds).  They exercise the
# BF16 tensor-core path with several M tiles per expert, ragged segment tails,
# h and d that are not multiples of the N tile, empty experts and k = E.
SMALL = {
    "small_bf16": LayerConfig("small_bf16", T=300, d=256, E=16, h=192, k=3, dtype="bf16",
                              rbd_epd=2, rbd_dpn=2),
    "small_ragged_bf16": LayerConfig("small_ragged_bf16", T=517, d=200, E=24, h=136, k=5, dtype="bf16",
                                     rbd_epd=3, rbd_dpn=2),
    "small_skew_bf16": LayerConfig("small_skew_bf16", T=700, d=320, E=16, h=256, k=4, dtype="bf16",
                                   zipf_c=1.5, rbd_epd=2, rbd_dpn=4),
    "small_kE_bf16": LayerConfig("small_kE_bf16", T=130, d=128, E=8, h=64, k=8, dtype="bf16",
                                 rbd_epd=1, rbd_dpn=2),
    "small_f32": LayerConfig("small_f32", T=333, d=96, E=9, h=40, k=3, dtype="f32",
                             rbd_epd=3, rbd_dpn=1),
    "one_token_bf16": LayerConfig("one_token_bf16", T=1, d=64, E=8, h=64, k=2, dtype="bf16",
                                  rbd_epd=2, rbd_dpn=2),
    # >= 256 rows per expert on average: full 256-token tiles of the token-as-N GEMMs next to
    # ragged tails, and d, h that are not multiples of the feature tile.
    "small_pairs_bf16": LayerConfig("small_pairs_bf16", T=1100, d=320, E=8, h=136, k=2, dtype="bf16",
                                    rbd_epd=2, rbd_dpn=2),
    # rows wider than 16 column chunks: the gather-sum kernels take 4 chunks per work item,
    # and the last item of every row is partial (17 and 18 chunks).
    "wide_d_bf16": LayerConfig("wide_d_bf16", T=96, d=4160, E=8, h=64, k=3, dtype="bf16"),
    "wide_d_f32": LayerConfig("wide_d_f32", T=40, d=2200, E=6, h=40, k=2, dtype="f32"),
    # k > 16: the RBD per-token kernels use whole 32-lane groups; 8 nodes of 8 experts.
    "big_k_bf16": LayerConfig("big_k_bf16", T=96, d=64, E=64, h=64, k=20, dtype="bf16", rbd_epd=4, rbd_dpn=2),
}


# Profiling shapes: slices of a full layer with the same d, h and rows per expert but fewer
# experts, so that a multi-pass ncu capture holds a few GB on the device instead of ~50 GB.
# Per-launch traffic scales with the number of experts (each expert's rows, weights and
# weight gradients are distinct).
PROFILE = {
    "dsv3_slice_bf16": LayerConfig("dsv3_slice_bf16", T=512, d=7168, E=16, h=2048, k=8, dtype="bf16",
                                   note="1/16 of the DeepSeek-V3-like layer: 16 experts, ~256 rows each"),
}


def get_config(name: str) -> LayerConfig:
    for table in (CONFIGS, SMALL, PROFILE):
        if name in table:
            return table[name]
    raise KeyError(f"unknown layer config {name!r}; known: {sorted(CONFIGS) + sorted(SMALL) + sorted(PROFILE)}")


def small_configs():
    return list(SMALL.values())
