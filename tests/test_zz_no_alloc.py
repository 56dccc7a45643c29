"""The allocation-free routing entry point (moe_route_dispatch_noalloc).

Some callers cannot allocate a device workspace (serving loops that must not
call cudaMalloc/cudaFree, or frameworks that own all device memory); this
entry point uses scratch compiled into the library instead.  It must give
exactly the results of moe_route_dispatch, on every call, because every call
reuses the same scratch.  This file runs last so that a failure here leaves
every other test already run; it also passes on its own in a fresh process.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from moe_routed_experts_b200 import binding as B
from moe_routed_experts_b200 import build as libbuild
from moe_routed_experts_b200 import ffn, inputs
from moe_routed_experts_b200.configs import WORKLOADS, scaled

pytestmark = pytest.mark.gpu

KEYS = ("values", "weights", "selected_experts", "row_experts", "offsets", "src_token", "row_of")


def _fresh_outputs(T, H, E, k):
    A = T * k
    return {
        "values": torch.full((A, H), 7, dtype=torch.bfloat16, device="cuda"),
        "weights": torch.full((T, k), -1.0, dtype=torch.float32, device="cuda"),
        "selected_experts": torch.full((T, k), -1, dtype=torch.int32, device="cuda"),
        "row_experts": torch.full((A,), -1, dtype=torch.int32, device="cuda"),
        "offsets": torch.full((E + 1,), -1, dtype=torch.int32, device="cuda"),
        "src_token": torch.full((A,), -1, dtype=torch.int32, device="cuda"),
        "row_of": torch.full((T, k), -1, dtype=torch.int32, device="cuda"),
    }


@pytest.mark.parametrize("name,kw", [("decode", {}), ("wide", dict(T=1024, H=256)), ("skewed", dict(T=2048, H=512))])
def test_noalloc_matches_workspace_entry_point_on_two_calls(name, kw):
    libbuild.build()
    w = scaled(WORKLOADS[name], **kw) if kw else WORKLOADS[name]
    inp = inputs.generate(w, with_grad=False)
    dev = ffn.to_device(inp)
    ref = B.moe_route_dispatch(dev["x"], dev["logits"], w.top_k, E=w.E, sel_bias=dev["sel_bias"],
                               expert_start=w.expert_start, renormalize=w.renormalize)
    torch.cuda.synchronize()
    for call in range(2):  # the second call runs over the scratch the first one left behind
        out = _fresh_outputs(w.T, w.H, w.E, w.top_k)
        st = B.new_status()
        B.moe_route_dispatch_noalloc(dev["x"], dev["logits"], w.top_k, out, E=w.E, sel_bias=dev["sel_bias"],
                                     expert_start=w.expert_start, renormalize=w.renormalize, device_status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        for key in KEYS:  # the same kernels on the same inputs: bit-identical, weights included
            assert torch.equal(out[key], ref[key]), (call, key)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    L = B.lib()
    T, E, k = 200000, 64, 8  # needs far more than the built-in 1 MiB
    need = L.moe_route_dispatch_workspace_size(T, E, k)
    assert need > (1 << 20)
    fake = 0x10000
    rc = L.moe_route_dispatch_noalloc(fake, B.MOE_BF16, T, 16, fake, None, E, 0, k, 1, fake, fake, fake, fake, fake,
                                      fake, fake, None, None)
    assert rc == 3  # MOE_ERR_WORKSPACE, before any launch
    assert b"1048576" in L.moe_last_error_string()
    # an invalid argument is reported as such, before the scratch-size check
    rc = L.moe_route_dispatch_noalloc(fake, B.MOE_BF16, T, 16, fake, None, E, 0, E + 1, 1, fake, fake, fake, fake,
                                      fake, fake, fake, None, None)
    assert rc == 1  # MOE_ERR_INVALID_ARGUMENT (top_k > E)
    rc = L.moe_route_dispatch_noalloc(fake, B.MOE_BF16, T, 16, fake, None, MOE_TOO_MANY_EXPERTS, 0, k, 1, fake,
                                      fake, fake, fake, fake, fake, fake, None, None)
    assert rc == 1  # MOE_ERR_INVALID_ARGUMENT (E > MOE_MAX_EXPERTS)


MOE_TOO_MANY_EXPERTS = 4097
