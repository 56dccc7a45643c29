"""The gather mode of the dispatch: routing without the COPY (moe_route) and a
gate/up projection that reads each expert-sorted row from the tokens
through src_token (awq_grouped_gate_up_swiglu_gather).

[MX] MoeDispatchOps::moe_dispatch states a device COPY; the gather mode
departs from it only in where the rows are read, so every output must be
bit-identical to the COPY mode's on the same inputs, on every tile path
(the tcgen05 tiles load the rows with TMA tile::gather4, the small-batch
tiles with per-row bulk copies or loads), and match the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import bits, check_forward_steps, check_routing, dt_name, generated, u32
from moe_routed_experts_b200 import binding as B
from moe_routed_experts_b200 import ffn

pytestmark = pytest.mark.gpu


@pytest.fixture(params=[1, 2, 3], ids=["warp_tiles", "tcgen05_tiles", "tcgen05_pair_tiles"])
def path(request):
    try:
        prev = B.set_projection_path(request.param)
    except ValueError:
        pytest.skip("projection path %d not available" % request.param)
    yield request.param
    B.set_projection_path(prev)


SHAPES = {
    "tiny": {},
    "decode": {},
    "prefill_small": ("prefill", dict(T=1024, H=256, I=128, E=16)),
    "wide_small": ("wide", dict(T=512, H=256, I=128, E=64)),
    "prefill": ("prefill", {}),
}


def _inp(key):
    spec = SHAPES[key]
    name, kw = (key, spec) if isinstance(spec, dict) else spec
    return generated(name, **kw)


def _run(inp, gather):
    dev = ffn.to_device(inp)
    buf = ffn.alloc(inp["workload"], keep_gu=True)
    ffn.forward(dev, buf, gather=gather)
    torch.cuda.synchronize()
    r = buf.route
    res = {"selected": u32(r["selected_experts"]), "weights": r["weights"].cpu().numpy(),
           "offsets": r["offsets"].cpu().numpy(), "row_experts": u32(r["row_experts"]),
           "src_token": r["src_token"].cpu().numpy(), "row_of": r["row_of"].cpu().numpy(),
           "G": bits(buf.G), "U": bits(buf.U), "h": bits(buf.h), "h_dt": dt_name(buf.h.dtype), "y": bits(buf.y),
           "out": bits(buf.out), "status": int(buf.status.item())}
    if not gather:
        res["values"] = bits(r["values"])
        res["values_dt"] = dt_name(r["values"].dtype)
    return res


@pytest.mark.parametrize("key", list(SHAPES))
def test_gather_mode_is_bit_identical_to_copy_mode(key, path):
    inp = _inp(key)
    a, b = _run(inp, gather=False), _run(inp, gather=True)
    assert a["status"] == 0 and b["status"] == 0
    for k in ("selected", "weights", "offsets", "row_experts", "src_token", "row_of", "G", "U", "h", "y", "out"):
        assert np.array_equal(a[k], b[k]), "%s differs between the COPY and the gather mode" % k


@pytest.mark.parametrize("key", ["tiny", "prefill_small", "wide_small"])
def test_gather_mode_against_oracle(key, path):
    inp = _inp(key)
    res = _run(inp, gather=True)
    want = oracle.forward(inp)
    check_routing(res, want, key)
    res["values"] = want["values"]  # the rows the gather reads (bit copies of x, checked in the routing tests)
    res["values_dt"] = "bf16"
    check_forward_steps(inp, res, want, key + "/gather")
    assert res["status"] == 0


def test_gather_row_out_of_range_is_flagged(path):
    inp = _inp("prefill_small")
    w = inp["workload"]
    dev = ffn.to_device(inp)
    r = B.moe_route(dev["logits"], w.top_k, E=w.E)
    src = r["src_token"].clone()
    src[5] = w.T + 3
    src[w.A - 1] = -1
    st = B.new_status()
    B.awq_grouped_gate_up_swiglu_gather(dev["x"], src, r["offsets"], dev["gate"], dev["up"], w.group,
                                        device_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 4  # MOE_DEVICE_ERR_ROW_RANGE, nothing else
