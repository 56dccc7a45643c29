"""GPU parity of the NF4 payload path (nf4_grouped_projection,
nf4_input_backward) against the oracle: the coefficients bit for bit through
the kernels that run (one-hot rows and gradients), and random batches within
the tolerance of tests/helpers.py (2e-2 * rms, beyond it only justified
rounding flips)."""
import numpy as np
import pytest
import torch

import oracle
from helpers import U32_ROUNDOFF, bits, check_close
from moe_routed_experts_b200 import binding as B
from moe_routed_experts_b200 import inputs

pytestmark = pytest.mark.gpu

TORCH_DT = {"f16": torch.float16, "bf16": torch.bfloat16}


def _one_hot(R, width, dt):
    x = torch.zeros((R, width), dtype=TORCH_DT[dt], device="cuda")
    r = torch.arange(R, device="cuda")
    x[r, r % width] = 1
    return x


@pytest.mark.parametrize("cdt", ["f16", "bf16"])
@pytest.mark.parametrize("K,N,block", [(64, 64, 64), (256, 192, 32), (768, 2048, 64)])
def test_nf4_coefficients_bit_exact_through_the_kernels(K, N, block, cdt):
    rng = np.random.default_rng(K + N + block)
    E = 2
    p = inputs.draw_nf4_projection(rng, E, K, N, block)
    dp = B.nf4_payload_to_device(p)
    # forward: the identity batch of each expert outputs W; VJP: one-hot gradients output W^T
    x = _one_hot(E * K, K, cdt)
    off = torch.arange(0, E * K + 1, K, dtype=torch.int32, device="cuda")
    st = B.new_status()
    y = B.nf4_grouped_projection(x, off, dp, cdt, device_status=st)
    g = _one_hot(E * N, N, cdt)
    offg = torch.arange(0, E * N + 1, N, dtype=torch.int32, device="cuda")
    d = B.nf4_input_backward(g, offg, dp, K, cdt, device_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    yb, db = bits(y), bits(d)
    for e in range(E):
        _, want = oracle.nf4_dequant(p["codes"][e], p["absmax"][e], p["codebook"], K, N, block, cdt)
        want = want.astype(np.uint16)
        assert np.array_equal(yb[e * K:(e + 1) * K], want), "forward coefficients differ (expert %d)" % e
        assert np.array_equal(db[e * N:(e + 1) * N], want.T), "transposed coefficients differ (expert %d)" % e


def _j_nf4(x, xdt, rexp, p, cdt, K_red, transpose=False, K=None):
    def justify(rows, cols):
        ur, inv = np.unique(rows, return_inverse=True)
        if transpose:
            ex = oracle.nf4_input_backward(x[ur], xdt, rexp[ur], p, K, cdt, exact=True)
            mag = oracle.nf4_input_backward(x[ur], xdt, rexp[ur], p, K, cdt, magnitude=True)
        else:
            ex = oracle.nf4_project(x[ur], xdt, rexp[ur], p, cdt, exact=True)
            mag = oracle.nf4_project(x[ur], xdt, rexp[ur], p, cdt, magnitude=True)
        conv = 2.0 ** -9 if (xdt == "f16" and cdt == "bf16") else 0.0
        return ex[inv, cols], ((K_red + 8) * U32_ROUNDOFF + conv) * mag[inv, cols]
    return justify


@pytest.mark.parametrize("cdt", ["f16", "bf16"])
@pytest.mark.parametrize("E,K,N,block,counts", [(4, 256, 128, 64, [5, 0, 17, 40]),
                                                 (128, 768, 2048, 64, None)])
def test_nf4_projection_and_vjp_against_oracle(E, K, N, block, counts, cdt):
    rng = np.random.default_rng(E + K)
    p = inputs.draw_nf4_projection(rng, E, K, N, block, bias=True)
    if counts is None:  # the decode down projection's shape: about two rows per expert, some empty
        counts = rng.integers(0, 5, E)
    counts = np.asarray(counts)
    A = int(counts.sum())
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    rexp = np.repeat(np.arange(E), counts).astype(np.int32)
    x = inputs.random_bf16(rng, (A, K))
    g = inputs.random_bf16(rng, (A, N))
    dp = B.nf4_payload_to_device(p)
    xd = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    gd = torch.from_numpy(g.view(np.int16)).view(torch.bfloat16).cuda()
    offd = torch.from_numpy(off).cuda()
    st = B.new_status()
    y = B.nf4_grouped_projection(xd, offd, dp, cdt, device_status=st)
    d = B.nf4_input_backward(gd, offd, dp, K, cdt, device_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    want_y = oracle.nf4_project(x, "bf16", rexp, p, cdt)
    check_close(bits(y), want_y, "nf4/y", justify=_j_nf4(x, "bf16", rexp, p, cdt, K))
    pb = dict(p, bias=None)
    want_d = oracle.nf4_input_backward(g, "bf16", rexp, pb, K, cdt)
    check_close(bits(d), want_d, "nf4/dinput", justify=_j_nf4(g, "bf16", rexp, pb, cdt, N, transpose=True, K=K))


def test_nf4_rejects_unsupported_layouts():
    rng = np.random.default_rng(1)
    p = B.nf4_payload_to_device(inputs.draw_nf4_projection(rng, 1, 64, 64, 64))
    x = torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda")
    off = torch.tensor([0, 4], dtype=torch.int32, device="cuda")
    p_bad = dict(p, block=48)
    with pytest.raises(B.MoeError):
        B.nf4_grouped_projection(x, off, p_bad, "bf16")
