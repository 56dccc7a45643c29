"""Pins of the oracle's NF4 payload (reading of ruda-tensor 0.21.34
PackedExpertPayload::Nf4, "high-nibble-first flat-block NF4", with the
4-bit NormalFloat data type of Dettmers et al., "QLoRA", 2023):

- the codebook the generator builds from the paper's construction equals the
  paper's table (tests/golden/nf4_codebook.txt);
- hand-worked bytes: the high nibble is the even flat element;
- hand-worked coefficients, one a double-rounding witness
  (tests/golden/nf4_coefficients.txt): the F32 x F32 product is rounded once;
- the projection and its input VJP against an independent NumPy
  dequantize-then-matmul, and the adjoint identity.
"""
import os

import numpy as np
import pytest

import oracle
from moe_routed_experts_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _codebook_table():
    with open(os.path.join(GOLDEN, "nf4_codebook.txt")) as f:
        return np.array([float(l) for l in f if l.strip() and not l.startswith("#")], np.float64)


def test_codebook_construction_matches_the_published_table():
    table = _codebook_table()
    assert table.shape == (16,) and table[7] == 0.0 and table[0] == -1.0 and table[15] == 1.0
    assert np.max(np.abs(inputs.nf4_codebook().astype(np.float64) - table)) <= 2e-7


def test_high_nibble_first():
    codes = np.array([0x1F, 0x80, 0xC3], np.uint8)
    assert [oracle.nf4_code(codes, f) for f in range(6)] == [1, 15, 8, 0, 12, 3]


def test_hand_worked_coefficients():
    cb = _codebook_table().astype(np.float32)
    n = 0
    with open(os.path.join(GOLDEN, "nf4_coefficients.txt")) as f:
        for line in f:
            if not line.strip() or line.startswith("#"):
                continue
            q, a, dt, want = line.split()
            absmax = np.array([int(a, 16)], np.uint32).view(np.float32)
            codes = np.array([(int(q) << 4) | int(q)], np.uint8)  # both elements of the block use code q
            _, bits = oracle.nf4_dequant(codes, absmax, cb, 1, 2, 2, dt)
            assert bits.tolist() == [[int(want, 16)] * 2], line
            n += 1
    assert n == 7


def _numpy_dequant(payload, e, K, N, cdt):
    """Independent: unpack high-nibble-first bytes, look up, scale in double, round in NumPy."""
    b = payload["codes"][e].astype(np.int64)
    q = np.empty(K * N, np.int64)
    q[0::2] = b >> 4
    q[1::2] = b & 15
    a = np.repeat(payload["absmax"][e].astype(np.float64), payload["block"])
    v = payload["codebook"].astype(np.float64)[q] * a
    if cdt == "f16":
        w = v.astype(np.float16).astype(np.float64)  # NumPy rounds double -> half once, to nearest even
    else:  # 8 significant bits, round half to even (np.rint), from the double itself
        m, ex = np.frexp(v)
        w = np.ldexp(np.rint(m * 256.0) / 256.0, ex)
    return w.reshape(K, N)


@pytest.mark.parametrize("cdt", ["f16", "bf16"])
def test_dequant_matches_numpy(cdt):
    rng = np.random.default_rng(31)
    E, K, N, B = 2, 64, 48, 64
    p = inputs.draw_nf4_projection(rng, E, K, N, B)
    for e in range(E):
        W, _ = oracle.nf4_dequant(p["codes"][e], p["absmax"][e], p["codebook"], K, N, B, cdt)
        assert np.array_equal(W, _numpy_dequant(p, e, K, N, cdt))


@pytest.mark.parametrize("cdt", ["f16", "bf16"])
def test_projection_and_vjp_against_numpy(cdt):
    rng = np.random.default_rng(32)
    E, K, N, B, R = 3, 64, 32, 32, 13
    p = inputs.draw_nf4_projection(rng, E, K, N, B, bias=True)
    rexp = rng.integers(0, E, R).astype(np.int32)
    x = inputs.random_bf16(rng, (R, K))
    xd = inputs.bf16_bits_to_f32(x).astype(np.float64)
    y = oracle.nf4_project(x, "bf16", rexp, p, cdt, exact=True)
    g = rng.standard_normal((R, N))
    dx = oracle.nf4_input_backward(g, "f64", rexp, p, K, cdt, exact=True)
    for r in range(R):
        W = _numpy_dequant(p, rexp[r], K, N, cdt)
        assert np.allclose(y[r], xd[r] @ W + p["bias"][rexp[r]], rtol=1e-12, atol=1e-12)
        assert np.allclose(dx[r], W @ g[r], rtol=1e-12, atol=1e-12)
    # the adjoint identity <J x, g> = <x, J^T g> (bias off)
    p["bias"] = None
    Jx = oracle.nf4_project(xd, "f64", rexp, p, cdt, exact=True)
    lhs, rhs = np.sum(Jx * g), np.sum(xd * dx)
    assert abs(lhs - rhs) <= 1e-12 * (abs(lhs) + np.sum(np.abs(Jx * g)))


def test_bad_block_layout_is_rejected():
    rng = np.random.default_rng(33)
    p = inputs.draw_nf4_projection(rng, 1, 8, 8, 16)
    p["block"] = 24  # 64 elements are not whole blocks of 24
    with pytest.raises(ValueError):
        oracle.nf4_project(np.zeros((1, 8), np.uint16), "bf16", np.zeros(1, np.int32), p, "bf16")
