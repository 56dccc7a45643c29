"""Brute-force NumPy cross-check of the C oracle on tiny inputs.

TEST INFRASTRUCTURE ONLY.  An independent second statement of the grouped
projection: dequantize a whole expert bank at once with array operations
(ruda-tensor 0.21.34 src/packed_experts.rs, AwqExpertPayload; ruda-tensor
0.21.33 src/frozen_awq.rs, FrozenAwqOps: AWQ nibble order and scale-dtype
coefficient rounding), then a dense float64 matmul per expert.  The rounding
of the coefficient to FP16 is NumPy's float16 cast and to BF16 is torch's
float32 -> bfloat16 cast (the exact product (q - z) * s has at most 12
significant bits for a BF16 scale, so the float32 step is exact).  It shares
no code with moe_oracle.c.
"""
import numpy as np
import torch

# logical column of nibble slot s within a word (packing order 0,2,4,6,1,3,5,7)
_COLUMN_OF_SLOT = np.array([0, 2, 4, 6, 1, 3, 5, 7])


def unpack_bank(words: np.ndarray) -> np.ndarray:
    """[..., W] int32 words -> [..., 8W] codes in logical column order."""
    u = words.astype(np.int64) & 0xFFFFFFFF
    out = np.zeros(words.shape[:-1] + (words.shape[-1], 8), np.int64)
    for s in range(8):
        out[..., _COLUMN_OF_SLOT[s]] = (u >> (4 * s)) & 0xF
    return out.reshape(words.shape[:-1] + (words.shape[-1] * 8,))


def scales_to_f64(scales: np.ndarray, sdt: str) -> np.ndarray:
    if sdt == "f16":
        return scales.view(np.float16).astype(np.float64)
    if sdt == "bf16":
        return (scales.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return scales.astype(np.float64)


def round_coefficients(exact: np.ndarray, sdt: str) -> np.ndarray:
    if sdt == "f16":
        return exact.astype(np.float16).astype(np.float64)
    if sdt == "bf16":
        t = torch.from_numpy(exact.astype(np.float32))
        return t.to(torch.bfloat16).to(torch.float64).numpy()
    return exact.astype(np.float32).astype(np.float64)


def dequant_bank(proj: dict, sdt: str, group: int) -> np.ndarray:
    """[E, K, N] float64 coefficients of a whole bank."""
    q = unpack_bank(proj["qweight"])                     # [E, K, N]
    z = unpack_bank(proj["qzeros"])                      # [E, K/g, N]
    s = scales_to_f64(np.asarray(proj["scales"]), sdt)   # [E, K/g, N]
    z_full = np.repeat(z, group, axis=1)
    s_full = np.repeat(s, group, axis=1)
    return round_coefficients((q - z_full).astype(np.float64) * s_full, sdt)


def grouped_matmul(x: np.ndarray, offsets: np.ndarray, W: np.ndarray, bias=None) -> np.ndarray:
    """Rows offsets[e]:offsets[e+1] of x times W[e] (+ bias[e]), float64, no rounding."""
    E = W.shape[0]
    out = np.zeros((x.shape[0], W.shape[2]), np.float64)
    for e in range(E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if b > a:
            out[a:b] = x[a:b] @ W[e]
            if bias is not None:
                out[a:b] += bias[e][None, :].astype(np.float64)
    return out
