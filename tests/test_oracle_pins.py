"""Pins of the CPU oracle against hand-worked values and library routines.

Each check ties one oracle step to something other than the oracle itself:
hand-worked words and coefficients (tests/golden/), the IEEE rounding of
NumPy's float16 cast and of float32 arithmetic, closed-form softmax values,
and hand-worked routing cases.
"""
import math
import os
import struct

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line.split()


def test_unpack_hand_worked_words():
    n = 0
    for parts in _lines("unpack_words.txt"):
        word = int(parts[0], 16)
        want = [int(v) for v in parts[1:9]]
        assert list(oracle.unpack_word(word)) == want, parts[0]
        assert oracle.pack_word(want) == word, parts[0]
        n += 1
    assert n >= 9


def test_unpack_signed_word_is_read_unsigned():
    # int32 -2147483648 is the word 0x80000000: only column 7 holds 8
    assert list(oracle.unpack_word(np.int32(-2147483648).view(np.uint32))) == [0] * 7 + [8]
    assert list(oracle.unpack_word(np.int32(-1).view(np.uint32))) == [15] * 8


def test_pack_unpack_round_trip_random():
    rng = np.random.default_rng(7)
    for _ in range(500):
        codes = rng.integers(0, 16, 8)
        assert list(oracle.unpack_word(oracle.pack_word(codes))) == list(codes)
    for word in rng.integers(0, 2**32, 500, dtype=np.uint64):
        assert oracle.pack_word(oracle.unpack_word(int(word))) == int(word)


def test_hand_worked_coefficients():
    n = 0
    for parts in _lines("coefficients.txt"):
        sdt, sbits, q, z, want = parts[0], int(parts[1], 16), int(parts[2]), int(parts[3]), int(parts[4], 16)
        v, bits = oracle.coefficient(q, z, sbits, sdt)
        assert bits == want, (parts, hex(bits))
        n += 1
    assert n >= 12


def test_f16_rounding_matches_numpy_cast():
    # NumPy's float64 -> float16 cast is an independent IEEE nearest-even conversion.
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.integers(-9, 5, 20000),
        np.array([65504.0, 65519.99, 65520.0, 1e6, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26, 2.0 ** -14]),
    ])
    for v in vals:
        want = int(np.array(v, np.float64).astype(np.float16).view(np.uint16))
        assert oracle.encode(v, "f16") == want, v
        assert oracle.encode(-v, "f16") == (want ^ 0x8000), v


def test_f32_rounding_matches_hardware_cast():
    rng = np.random.default_rng(2)
    vals = rng.standard_normal(20000) * 10.0 ** rng.integers(-40, 38, 20000)
    for v in vals:
        want = struct.unpack("<I", struct.pack("<f", v))[0] if abs(v) < 3.4e38 else None
        if want is not None:
            assert oracle.encode(v, "f32") == want, v


def test_bf16_rounding_of_float32_values():
    # BF16 nearest-even from float32 values; torch's CPU conversion is the library routine.
    import torch
    rng = np.random.default_rng(3)
    vals = (rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000)).astype(np.float32)
    want = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    for v, w in zip(vals, want):
        assert oracle.encode(float(v), "bf16") == int(w), v


def test_bf16_rounding_from_double_is_single_rounding():
    # 1 + 2^-8 + 2^-30 lies just above the BF16 midpoint 1 + 2^-8; a direct rounding
    # goes up.  Going through FP32 first (which drops 2^-30) would give the tie and
    # round down to 1.0: the oracle must not double-round.
    v = 1.0 + 2.0 ** -8 + 2.0 ** -30
    assert oracle.encode(v, "bf16") == 0x3F81
    assert oracle.encode(1.0 + 2.0 ** -8, "bf16") == 0x3F80


def test_decode_round_trip_all_16bit_patterns():
    for dt in ("f16", "bf16"):
        for b in range(0, 65536, 7):
            v = oracle.decode(b, dt)
            if math.isnan(v):
                continue
            assert oracle.encode(v, dt) == b, (dt, hex(b))


def test_coefficient_exhaustive_against_numpy_f16():
    # Every (q, z) pair times random F16 scales: RNE((q-z)*s) must equal NumPy's
    # float16 cast of the exact float64 product.
    rng = np.random.default_rng(4)
    scales = rng.integers(0, 0x7C00, 300).astype(np.uint16)
    for sb in scales:
        s = float(np.array(sb, np.uint16).view(np.float16))
        for q in range(16):
            for z in range(16):
                want = int(np.array((q - z) * s, np.float64).astype(np.float16).view(np.uint16))
                _, bits = oracle.coefficient(q, z, int(sb), "f16")
                assert bits == want or (q == z and bits in (0, 0x8000) and want in (0, 0x8000)), (q, z, hex(sb))


def test_route_hand_cases():
    # ruda-tensor 0.21.38 src/moe_exchange.rs, MoeDispatched: FP32 [tokens,top_k]
    # weights and U32 selected IDs.  Tie at 3,3 goes to the lower ID.
    sel, w = oracle.route(np.array([[1.0, 3.0, 3.0, 0.0]], np.float32), None, 2)
    assert sel.tolist() == [[1, 2]]
    assert np.allclose(w, [[0.5, 0.5]], atol=0)
    # selection bias chooses the set, weights come from the unbiased logits
    logits = np.array([[0.0, 1.0, 2.0, 0.5]], np.float32)
    bias = np.array([-100.0, 10.0, -100.0, 5.0], np.float32)
    sel, w = oracle.route(logits, bias, 2)
    assert sel.tolist() == [[1, 3]]
    e1, e3 = math.exp(1.0), math.exp(0.5)
    assert w[0, 0] == np.float32(e1 / (e1 + e3)) and w[0, 1] == np.float32(e3 / (e1 + e3))
    # expert_start offsets the global IDs
    sel, _ = oracle.route(np.array([[1.0, 3.0, 3.0, 0.0]], np.float32), None, 2, expert_start=40)
    assert sel.tolist() == [[41, 42]]


def test_route_signed_zero_and_nan_scores():
    # -0 and +0 are the same score: the tie goes to the lower ID, whichever
    # sign it carries (IEEE comparison, not the bit pattern)
    sel, w = oracle.route(np.array([[-0.0, 0.0, -1.0]], np.float32), None, 1)
    assert sel.tolist() == [[0]]
    sel, _ = oracle.route(np.array([[0.0, -0.0, -1.0]], np.float32), None, 2)
    assert sel.tolist() == [[0, 1]]
    # scores that are zero only after the selection bias: -0 + -0 = -0 for
    # expert 0, 1 + (-1) = +0 for expert 1; still a tie, lower ID first
    logits = np.array([[-0.0, 1.0, -2.0]], np.float32)
    bias = np.array([-0.0, -1.0, 0.0], np.float32)
    sel, w = oracle.route(logits, bias, 1)
    assert sel.tolist() == [[0]]
    # a NaN score (invalid input) ranks as -inf: chosen only when nothing
    # else is left, and then before a real -inf with a higher ID
    sel, _ = oracle.route(np.array([[np.nan, 0.5, -np.inf, 2.0]], np.float32), None, 3)
    assert sel.tolist() == [[3, 1, 0]]


def test_route_top_k_equals_e_is_full_softmax():
    rng = np.random.default_rng(5)
    logits = rng.standard_normal((6, 9)).astype(np.float32)
    sel, w = oracle.route(logits, None, 9)
    for t in range(6):
        ex = [math.exp(float(v)) for v in logits[t]]
        den = sum(ex)
        for j in range(9):
            assert abs(w[t, j] - ex[sel[t, j]] / den) <= 1e-7
        assert list(sel[t]) == sorted(range(9), key=lambda e: (-logits[t, e], e))


def test_route_without_renormalisation_is_full_softmax_of_selected():
    logits = np.array([[0.0, 1.0, 2.0, 3.0]], np.float32)
    sel, w = oracle.route(logits, None, 2, renormalize=0)
    den = sum(math.exp(v) for v in (0.0, 1.0, 2.0, 3.0))
    assert sel.tolist() == [[3, 2]]
    assert abs(w[0, 0] - math.exp(3.0) / den) < 1e-7 and abs(w[0, 1] - math.exp(2.0) / den) < 1e-7


def test_route_rejects_bad_top_k():
    with pytest.raises(ValueError):
        oracle.route(np.zeros((1, 4), np.float32), None, 5)
    with pytest.raises(ValueError):
        oracle.route(np.zeros((1, 4), np.float32), None, 0)


def test_dispatch_hand_case():
    # tokens 0..2 with top_k=2 over E=3: rows grouped by expert, each expert's rows
    # ascending by token (ruda-tensor 0.21.38, MoeDispatched: expert-sorted rows).
    sel = np.array([[2, 0], [0, 1], [2, 1]], np.uint32)
    off, rexp, src, row_of = oracle.dispatch(sel, 3)
    assert off.tolist() == [0, 2, 4, 6]
    assert rexp.tolist() == [0, 0, 1, 1, 2, 2]
    assert src.tolist() == [0, 1, 1, 2, 0, 2]
    assert row_of.tolist() == [[4, 0], [1, 2], [5, 3]]
    with pytest.raises(ValueError):
        oracle.dispatch(np.array([[3, 0]], np.uint32), 3)
