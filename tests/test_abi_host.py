"""The C-ABI library loads without a GPU, exports exactly what
include/moe_awq.h declares, and rejects bad arguments on the host before any
launch (the argument-validation pattern: a valid layout is accepted, a wrong
packing or shape is rejected with a typed error)."""
import ctypes as C

import pytest

from moe_routed_experts_b200 import binding as B
from moe_routed_experts_b200 import build as libbuild


@pytest.fixture(scope="module")
def L():
    libbuild.build()
    return B.lib()


def test_library_exports_every_header_function(L):
    names = B.header_functions()
    assert len(names) >= 13
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(B._SIGS), "binding signatures and header disagree"


def test_only_the_abi_is_exported():
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True, text=True).stdout
    text = [ln.split()[-1] for ln in out.splitlines() if " T " in ln]
    assert set(text) == set(B.header_functions())


def test_version_and_error_string(L):
    assert "sm_100a" in B.version()
    assert isinstance(L.moe_last_error_string(), bytes)


def test_projection_workspace_query(L):
    # nothing for an empty batch or an invalid count of projections
    assert L.awq_projection_workspace_size(0, 2048, 768, 128, 128, 2) == 0
    assert L.awq_projection_workspace_size(256, 2048, 768, 128, 128, 3) == 0


def test_workspace_size_query(L):
    assert L.moe_route_dispatch_workspace_size(0, 8, 2) >= 256
    a = L.moe_route_dispatch_workspace_size(8192, 128, 8)
    b = L.moe_route_dispatch_workspace_size(16384, 64, 6)
    assert a >= 8192 * 8 * 4 and b >= 16384 * 6 * 4
    assert L.moe_route_dispatch_workspace_size(-1, 8, 2) == 0


FAKE = 0x10000  # a 16-byte aligned non-null address; never dereferenced (validation fails first)


def _route(L, T=4, H=8, E=8, k=2, xdt=B.MOE_BF16, ws_bytes=1 << 20, expert_start=0):
    return L.moe_route_dispatch(FAKE, xdt, T, H, FAKE, None, E, expert_start, k, 1, FAKE, FAKE, FAKE, FAKE, FAKE,
                                FAKE, FAKE, FAKE, ws_bytes, None, None)


def test_route_dispatch_rejects_bad_arguments(L):
    assert _route(L, k=0) == 1
    assert _route(L, k=9) == 1            # top_k > E
    assert _route(L, k=33, E=64) == 1     # above the 32-lane selection limit
    assert _route(L, E=0) == 1
    assert _route(L, E=5000) == 1
    assert _route(L, T=-1) == 1
    assert _route(L, H=0) == 1
    assert _route(L, xdt=7) == 2
    assert _route(L, ws_bytes=16) == 3
    assert _route(L, expert_start=-3) == 1


def _gate_up(L, A=16, H=64, I=32, E=2, g=16, adt=B.MOE_BF16, sdt=B.MOE_F16, values=FAKE):
    return L.awq_grouped_gate_up_swiglu(values, adt, A, H, I, FAKE, E, FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE,
                                        None, sdt, B.MOE_F32, g, FAKE, None, None, None, 0, None, None)


def test_projection_rejects_bad_geometry_and_dtypes(L):
    assert _gate_up(L, I=30) == 1            # N not divisible by 8
    assert _gate_up(L, g=24) == 1            # group not a multiple of 16
    assert _gate_up(L, H=80, g=32) == 1      # incomplete group
    assert _gate_up(L, sdt=B.MOE_F32) == 2   # FP32 scales are not run
    assert _gate_up(L, adt=B.MOE_F32) == 2
    assert _gate_up(L, E=0) == 1
    assert _gate_up(L, values=FAKE + 2) == 1  # misaligned activations
    assert _gate_up(L, A=0) == 0             # nothing to do
    assert L.awq_grouped_down(FAKE, B.MOE_BF16, 4, 64, 12, FAKE, 1, FAKE, FAKE, FAKE, None, B.MOE_F16, B.MOE_F32, 16,
                              FAKE, None, 0, None, None) == 1
    assert L.awq_input_backward(FAKE, B.MOE_BF16, 4, 16, 64, FAKE, 1, FAKE, FAKE, FAKE, B.MOE_BF16, 48, None, None,
                                None, None, FAKE, None, 0, None, None) == 1


def test_combine_family_rejects_bad_arguments(L):
    assert L.moe_combine(FAKE, B.MOE_BF16, 8, FAKE, FAKE, FAKE, 4, 16, 0, FAKE, None, None) == 1
    assert L.moe_combine(FAKE, B.MOE_F32, 8, FAKE, FAKE, FAKE, 4, 16, 2, FAKE, None, None) == 2
    assert L.moe_combine(FAKE, B.MOE_BF16, 8, FAKE, FAKE, FAKE, 0, 16, 2, FAKE, None, None) == 0
    assert L.moe_dispatch_backward(FAKE, B.MOE_BF16, 8, FAKE, FAKE, 4, 16, 40, FAKE, None, None) == 1
    assert L.moe_combine_backward(FAKE, FAKE, B.MOE_BF16, 8, FAKE, FAKE, 4, 16, 2, None, None, None, None) == 0
    assert L.moe_swiglu_backward(FAKE, FAKE, FAKE, B.MOE_BF16, -1, 8, FAKE, FAKE, None) == 1


def test_dtype_choosing_forward_forms_reject_bad_dtypes(L):
    def route_dt(xdt, vdt, k=2):
        return L.moe_route_dispatch_dt(FAKE, xdt, 4, 8, FAKE, None, 8, 0, k, 1, FAKE, vdt, FAKE, FAKE, FAKE, FAKE,
                                       FAKE, FAKE, FAKE, 1 << 20, None, None)
    assert route_dt(B.MOE_F16, B.MOE_BF16) == 2   # only BF16 -> F16 converts
    assert route_dt(B.MOE_BF16, B.MOE_F32) == 2
    assert route_dt(B.MOE_BF16, B.MOE_F16, k=0) == 1

    def gate_up_dt(odt, hdt=B.MOE_F16, A=16):
        return L.awq_grouped_gate_up_swiglu_dt(FAKE, B.MOE_F16, A, 64, 32, FAKE, 2, FAKE, FAKE, FAKE, None, FAKE,
                                               FAKE, FAKE, None, B.MOE_F16, B.MOE_F32, 16, FAKE, hdt, None, None,
                                               odt, None, 0, None, None)
    assert gate_up_dt(B.MOE_F32) == 2
    assert gate_up_dt(B.MOE_BF16, hdt=B.MOE_F32) == 2
    assert gate_up_dt(B.MOE_BF16, A=0) == 0

    def gather_dt(odt, hdt=B.MOE_F16, A=16):
        return L.awq_grouped_gate_up_swiglu_gather_dt(FAKE, B.MOE_BF16, 8, FAKE, A, 64, 32, FAKE, 2, FAKE, FAKE, FAKE,
                                                      None, FAKE, FAKE, FAKE, None, B.MOE_F16, B.MOE_F32, 16, FAKE,
                                                      hdt, None, None, odt, None, 0, None, None)
    assert gather_dt(B.MOE_F32) == 2
    assert gather_dt(B.MOE_BF16, hdt=B.MOE_F32) == 2
    assert gather_dt(B.MOE_BF16, A=0) == 0

    def down_dt(odt, A=4):
        return L.awq_grouped_down_dt(FAKE, B.MOE_F16, A, 64, 16, FAKE, 1, FAKE, FAKE, FAKE, None, B.MOE_F16,
                                     B.MOE_F32, 16, FAKE, odt, None, 0, None, None)
    assert down_dt(B.MOE_F32) == 2
    assert down_dt(B.MOE_BF16, A=0) == 0


def test_dtype_choosing_backward_forms_reject_bad_dtypes(L):
    # the _dt forms check the output dtype on the host (2 = unsupported dtype)
    assert L.moe_combine_backward_dt(FAKE, FAKE, B.MOE_BF16, 8, FAKE, FAKE, 4, 16, 2, FAKE, B.MOE_F32, None, None,
                                     None) == 2
    assert L.moe_combine_backward_dt(FAKE, FAKE, B.MOE_BF16, 8, FAKE, FAKE, 4, 16, 0, FAKE, B.MOE_F16, None, None,
                                     None) == 1
    assert L.moe_combine_backward_dt(FAKE, FAKE, B.MOE_BF16, 8, FAKE, FAKE, 0, 16, 2, FAKE, B.MOE_F16, None, None,
                                     None) == 0
    assert L.moe_swiglu_backward_dt(FAKE, FAKE, FAKE, B.MOE_BF16, 4, 8, FAKE, FAKE, B.MOE_F32, None, None) == 2
    assert L.moe_swiglu_backward_dt(FAKE, FAKE, FAKE, B.MOE_BF16, -1, 8, FAKE, FAKE, B.MOE_F16, None, None) == 1
    assert L.moe_swiglu_backward_dt(FAKE, FAKE, FAKE, B.MOE_BF16, 0, 8, FAKE, FAKE, B.MOE_F16, None, None) == 0
    assert L.awq_input_backward_dt(FAKE, B.MOE_F16, 4, 16, 64, FAKE, 1, FAKE, FAKE, FAKE, B.MOE_F16, 16, None, None,
                                   None, None, FAKE, B.MOE_F32, None, 0, None, None) == 2
    assert L.awq_input_backward_dt(FAKE, B.MOE_F16, 4, 16, 64, FAKE, 1, FAKE, FAKE, FAKE, B.MOE_F16, 48, None, None,
                                   None, None, FAKE, B.MOE_BF16, None, 0, None, None) == 1
    assert L.awq_input_backward_dt(FAKE, B.MOE_F16, 0, 16, 64, FAKE, 1, FAKE, FAKE, FAKE, B.MOE_F16, 16, None, None,
                                   None, None, FAKE, B.MOE_BF16, None, 0, None, None) == 0


def test_projection_path_knob(L):
    assert L.moe_set_projection_path(7) == -1
    prev = L.moe_set_projection_path(1)
    assert prev in (0, 1, 2, 3)
    assert L.moe_set_projection_path(3) == 1
    assert L.moe_set_projection_path(1) == 3
    assert L.moe_set_projection_path(prev) == 1


def test_router_backward_rejects_bad_arguments(L):
    # (logits, selected, d_weights, T, E, top_k, renormalize, expert_start, d_logits, status, stream)
    assert L.moe_router_backward(FAKE, FAKE, FAKE, 4, 8, 0, 1, 0, FAKE, None, None) == 1      # top_k < 1
    assert L.moe_router_backward(FAKE, FAKE, FAKE, 4, 8, 9, 1, 0, FAKE, None, None) == 1      # top_k > E
    assert L.moe_router_backward(FAKE, FAKE, FAKE, 4, 64, 33, 1, 0, FAKE, None, None) == 1    # above 32 lanes
    assert L.moe_router_backward(FAKE, FAKE, FAKE, 4, 0, 1, 1, 0, FAKE, None, None) == 1      # E < 1
    assert L.moe_router_backward(FAKE, FAKE, FAKE, 4, 8, 2, 1, -1, FAKE, None, None) == 1     # expert_start
    assert L.moe_router_backward(FAKE, None, FAKE, 4, 8, 2, 1, 0, FAKE, None, None) == 1      # NULL tensor
    assert L.moe_router_backward(FAKE, FAKE, FAKE, 0, 8, 2, 1, 0, FAKE, None, None) == 0      # nothing to do


def test_projection_path_knob_accepts_every_path(L):
    prev = L.moe_set_projection_path(0)
    for path in (1, 2, 3, 0):
        L.moe_set_projection_path(path)
    assert L.moe_set_projection_path(4) == -1
    L.moe_set_projection_path(prev)
