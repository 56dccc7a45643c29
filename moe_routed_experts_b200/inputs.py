"""Seeded synthetic inputs shared by the CUDA path's tests, the bench and the
CPU oracle's tests.

This module holds no arithmetic of the method itself: it only draws numbers
(NumPy ``default_rng``) and stores them in the storage dtypes the operation
consumes.  BF16 values are produced by a library conversion (torch CPU,
round-to-nearest-even from float32) and F16 values by NumPy's float16 cast.

Draw order (one generator, seeded once): x, router logits, selection bias,
Zipf rank permutation, then for each projection gate, up, down: qweight words,
qzeros words, scales, bias; finally the upstream gradient dOut.

Packed words are drawn as uniform 32-bit integers.  Eight independent codes
uniform on 0..15 packed into one word in any fixed nibble order give exactly
a uniform 32-bit word, so drawing the word directly yields the stated
code/zero distribution without the generator having to know the packing
order (that order belongs to the method and lives in the oracle and in the
kernels).
"""
import math
from typing import Dict, Optional

import numpy as np
import torch

from .configs import Workload

_DT_BITS = {"bf16": np.uint16, "f16": np.uint16, "f32": np.float32}


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def f32_to_f16_bits(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32).astype(np.float16).view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(b, dtype=np.uint16).view(np.float16).astype(np.float32)


def to_storage(a: np.ndarray, dt: str) -> np.ndarray:
    if dt == "bf16":
        return f32_to_bf16_bits(a)
    if dt == "f16":
        return f32_to_f16_bits(a)
    if dt == "f32":
        return np.ascontiguousarray(a, dtype=np.float32)
    raise ValueError(dt)


def random_words(rng: np.random.Generator, shape) -> np.ndarray:
    """Uniform 32-bit words, returned as int32 (the storage type of qweight/qzeros)."""
    return rng.integers(0, 2**32, size=shape, dtype=np.uint32).view(np.int32)


def draw_projection(rng: np.random.Generator, E: int, K_in: int, N: int, group: int,
                    scale_dtype: str, bias: bool, bias_std: float) -> Dict[str, np.ndarray]:
    qweight = random_words(rng, (E, K_in, N // 8))
    qzeros = random_words(rng, (E, K_in // group, N // 8))
    s = rng.uniform(0.5, 1.5, size=(E, K_in // group, N)).astype(np.float32)
    s = s / np.float32(8.0 * math.sqrt(K_in))
    scales = to_storage(s, scale_dtype)
    out = {"qweight": qweight, "qzeros": qzeros, "scales": scales, "bias": None}
    if bias:
        out["bias"] = (rng.standard_normal((E, N), dtype=np.float32) * np.float32(bias_std)).astype(np.float32)
    return out


def generate(w: Workload, with_grad: Optional[bool] = None) -> Dict[str, object]:
    """All inputs of one workload, as NumPy arrays in storage dtypes.

    Activations are BF16 bit patterns (uint16), logits FP32, scales in the
    workload's scale dtype (uint16 bit patterns for F16/BF16).
    """
    rng = np.random.default_rng(w.seed)
    T, H, I, E = w.T, w.H, w.I, w.E
    x = f32_to_bf16_bits(rng.standard_normal((T, H), dtype=np.float32))
    logits = (rng.standard_normal((T, E), dtype=np.float32) * np.float32(w.logit_std)).astype(np.float32)
    sel_bias = None
    if w.sel_bias_std is not None:
        sel_bias = (rng.standard_normal(E, dtype=np.float32) * np.float32(w.sel_bias_std)).astype(np.float32)
    if w.zipf_s is not None:
        # Expert e gets Zipf rank r_e = 1 + perm[e]; its logit offset is
        # 2*log(r_e^-s) = -2*s*log(r_e), added to every token's logit.
        rank = 1.0 + rng.permutation(E).astype(np.float64)
        offset = (-2.0 * w.zipf_s * np.log(rank)).astype(np.float32)
        logits = (logits + offset[None, :]).astype(np.float32)
    proj = {}
    for name, K_in, N in (("gate", H, I), ("up", H, I), ("down", I, H)):
        proj[name] = draw_projection(rng, E, K_in, N, w.group, w.scale_dtype, w.bias, w.bias_std)
    d_out = None
    if with_grad or (with_grad is None and w.backward):
        d_out = f32_to_bf16_bits(rng.standard_normal((T, H), dtype=np.float32))
    return {"workload": w, "x": x, "logits": logits, "sel_bias": sel_bias,
            "gate": proj["gate"], "up": proj["up"], "down": proj["down"], "d_out": d_out}


def random_bf16(rng: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    return f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32) * np.float32(std))


def nf4_codebook() -> np.ndarray:
    """The 16 values of the 4-bit NormalFloat data type (Dettmers et al.,
    "QLoRA", 2023, section 3): quantiles of N(0, 1) at evenly spaced
    probabilities, 8 on the positive side and 7 on the negative side plus an
    exact zero, scaled so the extremes are -1 and 1.  The outermost
    probability is the midpoint of 1 - 1/(2*15) and 1 - 1/(2*16) (the two
    halves' own outermost quantiles).  A payload input: the operation takes
    whatever codebook the caller passes (tests pin this construction against
    the paper's table)."""
    from scipy.stats import norm
    top = 1.0 - 0.5 * (1.0 / 30.0 + 1.0 / 32.0)
    pos = norm.ppf(np.linspace(top, 0.5, 9)[:-1])
    neg = -norm.ppf(np.linspace(top, 0.5, 8)[:-1])
    v = np.sort(np.concatenate([pos, [0.0], neg]))
    return (v / np.max(np.abs(v))).astype(np.float32)


def draw_nf4_projection(rng: np.random.Generator, E: int, K_in: int, N: int, block: int, bias: bool = False,
                        bias_std: float = 0.02) -> Dict[str, np.ndarray]:
    """NF4 payload of E experts ([K_in, N] each): uniform random code bytes
    (two uniform 4-bit codes per byte), absmax scales uniform[0.5, 1.5) /
    sqrt(K_in) per block of `block` flat elements, the NF4 codebook."""
    codes = rng.integers(0, 256, size=(E, K_in * N // 2), dtype=np.uint8)
    absmax = (rng.uniform(0.5, 1.5, size=(E, K_in * N // block)) / math.sqrt(K_in)).astype(np.float32)
    out = {"codes": codes, "absmax": absmax, "codebook": nf4_codebook(), "block": block, "N": N, "bias": None}
    if bias:
        out["bias"] = (rng.standard_normal((E, N), dtype=np.float32) * np.float32(bias_std)).astype(np.float32)
    return out
