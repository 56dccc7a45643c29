"""The C oracle's grouped projections against the NumPy brute force on tiny
inputs (E <= 4, K_in <= 64, N <= 32, group in {8, 16, 32}), plus the
special case E = 1, top_k = 1 where the routed FFN is a dense SwiGLU MLP."""
import numpy as np
import pytest

import oracle
from oracle import bruteforce as bf
from moe_routed_experts_b200 import inputs


def _bank(rng, E, K, N, g, sdt, bias=False):
    return inputs.draw_projection(rng, E, K, N, g, sdt, bias, 0.05)


def _bf16_to_f64(a):
    return inputs.bf16_bits_to_f32(a).astype(np.float64)


@pytest.mark.parametrize("sdt", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("E,K,N,g", [(1, 8, 8, 8), (3, 32, 16, 16), (4, 64, 32, 32), (2, 64, 24, 8)])
def test_dequant_matches_bruteforce_bitwise(sdt, E, K, N, g):
    rng = np.random.default_rng(11 + E * K + N)
    proj = _bank(rng, E, K, N, g, sdt)
    Wbf = bf.dequant_bank(proj, sdt, g)
    for e in range(E):
        W, _ = oracle.dequant(proj["qweight"][e], proj["qzeros"][e], proj["scales"][e], sdt, K, N, g)
        assert np.array_equal(W, Wbf[e])


@pytest.mark.parametrize("sdt", ["f16", "bf16"])
@pytest.mark.parametrize("bias", [False, True])
@pytest.mark.parametrize("E,K,N,g,R", [(1, 16, 8, 8, 3), (3, 32, 16, 16, 10), (4, 64, 32, 32, 17)])
def test_project_matches_bruteforce(sdt, bias, E, K, N, g, R):
    rng = np.random.default_rng(100 + R)
    proj = _bank(rng, E, K, N, g, sdt, bias)
    x = inputs.random_bf16(rng, (R, K))
    counts = rng.multinomial(R, np.ones(E) / E)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    rexp = np.repeat(np.arange(E), counts).astype(np.int32)
    want = bf.grouped_matmul(_bf16_to_f64(x), offsets, bf.dequant_bank(proj, sdt, g), proj["bias"])
    got = oracle.project(x, "bf16", rexp, proj, sdt, g, exact=True)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)
    stored = oracle.project(x, "bf16", rexp, proj, sdt, g)
    got_r = _bf16_to_f64(stored)
    want_r = inputs.bf16_bits_to_f32(inputs.f32_to_bf16_bits(want.astype(np.float32))).astype(np.float64)
    # within one BF16 ulp of the brute force's rounding (double->float->bf16 there)
    ulp = np.maximum(np.abs(want_r), 1e-30) * 2.0 ** -7
    assert np.all(np.abs(got_r - want_r) <= ulp)


@pytest.mark.parametrize("sdt", ["f16", "bf16"])
def test_input_backward_matches_bruteforce_transpose(sdt):
    rng = np.random.default_rng(5)
    E, K, N, g, R = 3, 64, 32, 16, 12
    p1, p2 = _bank(rng, E, K, N, g, sdt), _bank(rng, E, K, N, g, sdt)
    g1, g2 = inputs.random_bf16(rng, (R, N)), inputs.random_bf16(rng, (R, N))
    counts = np.array([5, 0, 7])
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    rexp = np.repeat(np.arange(E), counts).astype(np.int32)
    W1, W2 = bf.dequant_bank(p1, sdt, g), bf.dequant_bank(p2, sdt, g)
    want = np.zeros((R, K))
    for e in range(E):
        a, b = offsets[e], offsets[e + 1]
        want[a:b] = _bf16_to_f64(g1[a:b]) @ W1[e].T + _bf16_to_f64(g2[a:b]) @ W2[e].T
    got = oracle.input_backward(g1, "bf16", rexp, p1, sdt, g, grad2=g2, proj2=p2, exact=True)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("sdt", ["f16", "bf16"])
def test_single_expert_top1_is_dense_swiglu_mlp(sdt):
    """E = 1, top_k = 1: weight 1.0 for every token, so out = y = down(silu(gate x) * up x)."""
    from moe_routed_experts_b200.configs import Workload
    w = Workload("one", T=9, H=32, I=16, E=1, top_k=1, group=16, scale_dtype=sdt)
    inp = inputs.generate(w)
    res = oracle.forward(inp)
    assert np.all(res["weights"] == 1.0)
    assert np.array_equal(res["src_token"], np.arange(9))
    x = _bf16_to_f64(inp["x"])
    Wg = bf.dequant_bank(inp["gate"], sdt, 16)[0]
    Wu = bf.dequant_bank(inp["up"], sdt, 16)[0]
    Wd = bf.dequant_bank(inp["down"], sdt, 16)[0]

    def rb(a):
        return inputs.bf16_bits_to_f32(inputs.f32_to_bf16_bits(np.asarray(a, np.float32))).astype(np.float64)

    G, U = rb(x @ Wg), rb(x @ Wu)
    assert np.array_equal(_bf16_to_f64(res["G"]), G) or np.max(np.abs(_bf16_to_f64(res["G"]) - G)) <= 2.0 ** -7 * np.max(np.abs(G))
    h = rb(G / (1.0 + np.exp(-G)) * U)
    y = rb(_bf16_to_f64(res["h"]) @ Wd)
    out = _bf16_to_f64(res["out"])
    assert np.array_equal(out, _bf16_to_f64(res["y"]))            # weight exactly 1
    assert np.max(np.abs(_bf16_to_f64(res["h"]) - h)) <= 2.0 ** -7 * np.max(np.abs(h)) + 1e-30
    assert np.max(np.abs(out - y)) <= 2.0 ** -7 * np.max(np.abs(y))
