"""Workload shapes of the frozen AWQ routed-experts FFN.

Each workload is named for what it is.  Sizes follow the five synthetic
workloads the method is measured on: a tiny parity case, a decode-shaped
batch that is bound by packed-weight bytes, a prefill-shaped batch that is
bound by the tensor cores, a wide 512-expert bank with a selection bias, and a
skewed (Zipf-offset) routing case that also runs the backward chain.

Nothing here computes any part of the method; it only fixes sizes,
dtypes and the seeded value distributions (see ``inputs.py``).
"""
from dataclasses import dataclass, field
from typing import Optional


@dataclass(frozen=True)
class Workload:
    name: str
    T: int            # tokens
    H: int            # hidden width (gate/up input, down output)
    I: int            # intermediate width (gate/up output, down input)
    E: int            # experts in the resident bank
    top_k: int
    group: int        # AWQ input-channel group size
    scale_dtype: str  # "f16" | "bf16" | "f32"
    bias: bool = False            # per-expert FP32 bias on gate, up and down
    bias_std: float = 0.02
    logit_std: float = 1.0
    sel_bias_std: Optional[float] = None   # selection-only router bias
    zipf_s: Optional[float] = None         # per-expert Zipf rank offset
    backward: bool = False                 # upstream gradient + input VJPs
    expert_start: int = 0
    seed: int = 0
    renormalize: int = 1

    @property
    def A(self) -> int:
        return self.T * self.top_k


WORKLOADS = {
    "tiny": Workload("tiny", T=16, H=256, I=512, E=8, top_k=2, group=64,
                     scale_dtype="f16"),
    "decode": Workload("decode", T=32, H=2048, I=768, E=128, top_k=8,
                       group=128, scale_dtype="f16"),
    "prefill": Workload("prefill", T=8192, H=2048, I=768, E=128, top_k=8,
                        group=128, scale_dtype="bf16", bias=True),
    "wide": Workload("wide", T=4096, H=2048, I=512, E=512, top_k=10,
                     group=128, scale_dtype="f16", logit_std=1.5,
                     sel_bias_std=0.1),
    "skewed": Workload("skewed", T=16384, H=4096, I=1408, E=64, top_k=6,
                       group=128, scale_dtype="f16", zipf_s=1.2,
                       backward=True),
}


def scaled(w: Workload, **kw) -> Workload:
    """A copy of ``w`` with some fields replaced (smaller parity cases)."""
    d = dict(w.__dict__)
    d.update(kw)
    return Workload(**d)
