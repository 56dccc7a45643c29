"""The rounded coefficients, bit for bit, through the kernels that run.

[FA] FrozenAwqOps keeps the scale-dtype rounding of each coefficient
W = RNE_sdt((q - z) s); every projection kernel forms W in its own code
(the streaming decode tile, the tcgen05 dequant
warps, the warp-level tiles, the input-VJP tiles).  Fed one-hot rows, a
kernel's output IS its coefficients: with activations in the scale dtype and
no bias, row r = e_kk makes the FP32 accumulation hold the single exact
product 1 * W[kk, n] (every other product is an exact zero, split-K partial
sums add zeros), and the output, stored in the scale dtype, is W[kk, n]
unchanged.  So the forward output of the identity batch is the whole
coefficient matrix, and the input VJP of one-hot gradient rows is its
transpose; both must equal the oracle's dequantization bit for bit.

Paths: 1 = warp-level tiles (the streaming tile when the shape allows, the
plain warp tile otherwise), 2 = 128-row tcgen05 tiles, 3 = 256-row CTA-pair
tcgen05 tiles.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import bits
from moe_routed_experts_b200 import binding as B
from moe_routed_experts_b200 import ffn, inputs

pytestmark = pytest.mark.gpu

TORCH_DT = {"f16": torch.float16, "bf16": torch.bfloat16}


@pytest.fixture(params=[1, 2, 3], ids=["warp_tiles", "tcgen05_tiles", "tcgen05_pair_tiles"])
def path(request):
    try:
        prev = B.set_projection_path(request.param)
    except ValueError:
        pytest.skip("projection path %d not available" % request.param)
    yield request.param
    B.set_projection_path(prev)


def _scales(rng, shape, sdt, wide):
    """Scales of the workloads (uniform[0.5, 1.5) / (8 sqrt(K)) in the scale
    dtype), or, with `wide`, F16/BF16 bit patterns over many binades: for F16
    subnormal scales (products rounded on the subnormal grid) and scales up
    to 4096, while |15 s| stays finite."""
    if not wide:
        return None
    if sdt == "f16":
        raw = rng.integers(0x0001, 0x6C00, size=shape).astype(np.uint16)  # up to 4096: 15 s stays finite
        raw[..., 0, :] = rng.integers(0x0001, 0x0400, size=raw[..., 0, :].shape)  # group 0: subnormal scales
    else:
        raw = rng.integers(0x2000, 0x6000, size=shape).astype(np.uint16)  # 2^-63 .. 2^65
    return raw


def _payload(rng, E, K, N, g, sdt, wide):
    proj = inputs.draw_projection(rng, E, K, N, g, sdt, False, 0.0)
    sc = _scales(rng, proj["scales"].shape, sdt, wide)
    if sc is not None:
        proj["scales"] = sc
    return proj


def _want(proj, sdt, K, N, g):
    E = proj["qweight"].shape[0]
    return [oracle.dequant(proj["qweight"][e], proj["qzeros"][e], proj["scales"][e], sdt, K, N, g)[1].astype(np.uint16)
            for e in range(E)]


def _one_hot(R, width, dt):
    """Rows e_{r mod width} in dtype dt."""
    x = torch.zeros((R, width), dtype=TORCH_DT[dt], device="cuda")
    r = torch.arange(R, device="cuda")
    x[r, r % width] = 1
    return x


def _first_mismatch(got, want):
    m = np.nonzero(got != want)
    return list(zip(*[a[:4].tolist() for a in m]))


# (K, N, group): one full group, the decode/prefill gate-up and down shapes
# (several groups, full tile counts), and a shape only the plain warp tile takes
SHAPES = [(128, 256, 128), (2048, 768, 128), (768, 2048, 128), (48, 40, 16)]


@pytest.mark.parametrize("sdt", ["f16", "bf16"])
@pytest.mark.parametrize("wide", [False, True], ids=["workload_scales", "wide_scales"])
@pytest.mark.parametrize("K,N,g", SHAPES)
def test_forward_outputs_are_the_coefficients(K, N, g, sdt, wide, path):
    rng = np.random.default_rng(K + N + (7 if wide else 0))
    E = 2
    gate, up = _payload(rng, E, K, N, g, sdt, wide), _payload(rng, E, K, N, g, sdt, wide)
    # every expert gets the identity batch: rows kk = 0..K-1, so A = E K
    x = _one_hot(E * K, K, sdt)
    off = torch.arange(0, E * K + 1, K, dtype=torch.int32, device="cuda")
    st = B.new_status()
    h, G, U = B.awq_grouped_gate_up_swiglu(x, off, ffn.projection_to_device(gate, sdt),
                                           ffn.projection_to_device(up, sdt), g, want_gu=True, device_status=st)
    y = B.awq_grouped_down(x, off, ffn.projection_to_device(gate, sdt), g, device_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    wg, wu = _want(gate, sdt, K, N, g), _want(up, sdt, K, N, g)
    Gb, Ub, yb = bits(G), bits(U), bits(y)
    for e in range(E):
        rows = slice(e * K, (e + 1) * K)
        for name, got, want in (("G", Gb[rows], wg[e]), ("U", Ub[rows], wu[e]), ("single", yb[rows], wg[e])):
            assert np.array_equal(got, want), "%s expert %d: first mismatches (kk, n) %s" % (
                name, e, _first_mismatch(got, want))


BWD_SHAPES = [(128, 256, 128), (2048, 768, 128), (768, 2048, 128), (64, 48, 16)]


@pytest.mark.parametrize("sdt", ["f16", "bf16"])
@pytest.mark.parametrize("wide", [False, True], ids=["workload_scales", "wide_scales"])
@pytest.mark.parametrize("K,N,g", BWD_SHAPES)
def test_input_vjp_outputs_are_the_transposed_coefficients(K, N, g, sdt, wide, path):
    rng = np.random.default_rng(3 * K + N + (5 if wide else 0))
    E = 2
    p1, p2 = _payload(rng, E, K, N, g, sdt, wide), _payload(rng, E, K, N, g, sdt, wide)
    d1, d2 = ffn.projection_to_device(p1, sdt), ffn.projection_to_device(p2, sdt)
    # gradient rows e_n (n = 0..N-1) per expert: dinput row n is column n of W
    onehot = _one_hot(E * N, N, sdt)
    zero = torch.zeros_like(onehot)
    off = torch.arange(0, E * N + 1, N, dtype=torch.int32, device="cuda")
    st = B.new_status()
    d_single = B.awq_input_backward(onehot, off, d1, g, device_status=st)
    d_first = B.awq_input_backward(onehot, off, d1, g, grad2=zero, proj2=d2, device_status=st)
    d_second = B.awq_input_backward(zero, off, d1, g, grad2=onehot, proj2=d2, device_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    w1, w2 = _want(p1, sdt, K, N, g), _want(p2, sdt, K, N, g)
    for e in range(E):
        rows = slice(e * N, (e + 1) * N)
        for name, got, want in (("single", bits(d_single)[rows], w1[e].T), ("pair/first", bits(d_first)[rows], w1[e].T),
                                ("pair/second", bits(d_second)[rows], w2[e].T)):
            assert np.array_equal(got, want), "%s expert %d: first mismatches (n, kk) %s" % (
                name, e, _first_mismatch(got, want))
