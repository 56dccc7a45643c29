"""Edge cases and device-side data errors.

Degenerate shapes (one token, one expert, one word column, K equal to the
group, every row on one expert, empty experts), other dtype combinations,
and inconsistent mappings injected on the host: the kernels must flag them
in the device status word, skip the offending rows, and never fault."""
import numpy as np
import pytest
import torch

import oracle
from helpers import (bits, check_close, check_forward_steps, check_routing, gpu_forward_numpy, j_chain,
                     j_input_backward, j_project, j_swiglu, j_swiglu_backward)
from moe_routed_experts_b200 import binding as B
from moe_routed_experts_b200 import ffn, inputs
from moe_routed_experts_b200.configs import Workload

pytestmark = pytest.mark.gpu


@pytest.fixture(params=[1, 2, 3], ids=["warp_tiles", "tcgen05_tiles", "tcgen05_pair_tiles"])
def path(request):
    try:
        prev = B.set_projection_path(request.param)
    except ValueError:
        pytest.skip("projection path %d not available" % request.param)
    yield request.param
    B.set_projection_path(prev)


def _run(w, logits_fn=None):
    inp = inputs.generate(w)
    if logits_fn is not None:
        inp["logits"] = logits_fn(inp["logits"])
    res, dev, buf = gpu_forward_numpy(inp)
    want = oracle.forward(inp)
    check_routing(res, want, w.name)
    check_forward_steps(inp, res, want, w.name)
    assert res["status"] == 0
    return res, want


def test_one_token_one_expert(path):
    _run(Workload("min", T=1, H=16, I=16, E=1, top_k=1, group=16, scale_dtype="f16"))


def test_k_equals_group_and_ragged_feature_slab(path):
    # gate/up: K = H = group = 16; I = 80 (ten word columns: a ragged slab)
    _run(Workload("kgroup", T=37, H=16, I=80, E=5, top_k=3, group=16, scale_dtype="bf16", bias=True))


@pytest.mark.parametrize("N", [8, 24, 136])
def test_single_projection_narrow_outputs(N, path):
    # one word column (N = 8) and ragged slabs, through the grouped projection alone
    rng = np.random.default_rng(N)
    A, K, g, E = 29, 64, 16, 3
    proj = inputs.draw_projection(rng, E, K, N, g, "f16", True, 0.1)
    x = inputs.random_bf16(rng, (A, K))
    counts = np.array([10, 0, 19])
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    xd = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    y = B.awq_grouped_down(xd, torch.from_numpy(off).cuda(), ffn.projection_to_device(proj, "f16"), g)
    re = np.repeat(np.arange(E), counts).astype(np.int32)
    want = oracle.project(x, "bf16", re, proj, "f16", g)
    check_close(bits(y), want, "narrow", justify=j_project(x, "bf16", re, proj, "f16", g))


def test_every_row_on_one_expert(path):
    def hot(l):
        l = l.copy()
        l[:, 3] += 100.0
        return l
    res, _ = _run(Workload("hot", T=300, H=128, I=64, E=8, top_k=1, group=32, scale_dtype="f16"), hot)
    counts = np.diff(res["offsets"])
    assert counts[3] == 300 and counts.sum() == 300


def test_many_empty_experts(path):
    def few(l):
        l = l.copy()
        l[:, 6:] -= 50.0
        return l
    res, _ = _run(Workload("empty", T=64, H=128, I=64, E=40, top_k=2, group=64, scale_dtype="f16"), few)
    assert np.all(np.diff(res["offsets"])[6:] == 0)


def test_expert_start_offset(path):
    _run(Workload("start", T=50, H=128, I=64, E=6, top_k=2, group=32, scale_dtype="f16", expert_start=12))


@pytest.mark.parametrize("act,sdt", [("f16", "f16"), ("f16", "bf16"), ("bf16", "bf16")])
def test_activation_and_scale_dtypes(act, sdt, path):
    w = Workload("dt", T=40, H=128, I=64, E=4, top_k=2, group=32, scale_dtype=sdt)
    inp = inputs.generate(w)
    x32 = inputs.bf16_bits_to_f32(inp["x"])
    xs = inputs.to_storage(x32, act)
    sel, wts = oracle.route(inp["logits"], None, w.top_k)
    off, rexp, src, row_of = oracle.dispatch(sel, w.E)
    values = xs[src]
    re = rexp.astype(np.int32)
    dt_t = torch.float16 if act == "f16" else torch.bfloat16
    vd = torch.from_numpy(values.view(np.int16)).view(dt_t).cuda()
    offd = torch.from_numpy(off).cuda()
    gate, up = ffn.projection_to_device(inp["gate"], sdt), ffn.projection_to_device(inp["up"], sdt)
    h, G, U = B.awq_grouped_gate_up_swiglu(vd, offd, gate, up, w.group, want_gu=True)
    torch.cuda.synchronize()
    oG = oracle.project(values, act, re, inp["gate"], sdt, w.group)
    oU = oracle.project(values, act, re, inp["up"], sdt, w.group)
    oh = oracle.swiglu(oG, oU, act)
    check_close(bits(G), oG, "G", dt=act, justify=j_project(values, act, re, inp["gate"], sdt, w.group))
    check_close(bits(U), oU, "U", dt=act, justify=j_project(values, act, re, inp["up"], sdt, w.group))
    check_close(bits(h), oracle.swiglu(bits(G), bits(U), act), "h", dt=act,
                justify=j_swiglu(bits(G), bits(U), act))
    check_close(bits(h), oh, "h(end-to-end)", dt=act,
                justify=j_chain(j_swiglu(oG, oU, act), j_swiglu(bits(G), bits(U), act)))
    down = ffn.projection_to_device(inp["down"], sdt)
    y = B.awq_grouped_down(h, offd, down, w.group)
    oy = oracle.project(bits(h), act, re, inp["down"], sdt, w.group)
    check_close(bits(y), oy, "y", dt=act, justify=j_project(bits(h), act, re, inp["down"], sdt, w.group))
    dx = B.awq_input_backward(y, offd, down, w.group)
    odx = oracle.input_backward(bits(y), act, re, inp["down"], sdt, w.group)
    check_close(bits(dx), odx, "dinput", dt=act, justify=j_input_backward(bits(y), act, re, inp["down"], sdt, w.group))


def test_single_frozen_linear_is_one_expert(path):
    # the frozen AWQ linear is the grouped projection with E = 1, offsets {0, A}
    rng = np.random.default_rng(8)
    A, K, N, g = 77, 256, 40, 64
    proj = inputs.draw_projection(rng, 1, K, N, g, "f16", True, 0.1)
    x = inputs.random_bf16(rng, (A, K))
    xd = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    off = torch.tensor([0, A], dtype=torch.int32, device="cuda")
    y = B.awq_grouped_down(xd, off, ffn.projection_to_device(proj, "f16"), g)
    want = oracle.project(x, "bf16", np.zeros(A, np.int32), proj, "f16", g)
    check_close(bits(y), want, "linear", justify=j_project(x, "bf16", np.zeros(A, np.int32), proj, "f16", g))


def test_inconsistent_offsets_are_flagged_not_faulted(path):
    w = Workload("bad", T=64, H=128, I=64, E=4, top_k=2, group=32, scale_dtype="f16")
    inp = inputs.generate(w)
    dev = ffn.to_device(inp)
    A = w.A
    values = torch.zeros((A, w.H), dtype=torch.bfloat16, device="cuda")
    for bad in ([0, 40, 20, 100, A], [5, 30, 60, 90, A], [0, 30, 60, 90, A - 1], [0, 30, 60, 90, A + 50]):
        st = B.new_status()
        off = torch.tensor(bad, dtype=torch.int32, device="cuda")
        h = torch.full((A, w.I), 7.0, dtype=torch.bfloat16, device="cuda")
        B.awq_grouped_gate_up_swiglu(values, off, dev["gate"], dev["up"], w.group, device_status=st, out=h)
        torch.cuda.synchronize()
        assert int(st.item()) & 2, bad


@pytest.mark.parametrize("value,flagged", [(70000.0, True), (float("nan"), True), (1e-7, False), (2.0 ** -16, False),
                                           (65280.0, False), (float("inf"), False)],
                         ids=["overflow", "nan", "below_f16_subnormal_grid", "on_f16_subnormal_grid",
                              "bf16_max_below_65504", "inf_converts_exactly"])
def test_f16_range_overflow_is_flagged(value, flagged, path):
    # F16 scales with BF16 inputs: the tensor-core operand is F16; a finite
    # BF16 activation or gradient above F16's range (it would become inf) or
    # a NaN is reported by the projection and the input VJP, and only those
    # (tiny values keep what F16's subnormal grid holds: under 2^-25 absolute)
    rng = np.random.default_rng(11)
    E, K, N, g, A = 2, 256, 128, 64, 256
    proj = inputs.draw_projection(rng, E, K, N, g, "f16", False, 0.0)
    dproj = ffn.projection_to_device(proj, "f16")
    off = torch.tensor([0, A // 2, A], dtype=torch.int32, device="cuda")
    x = torch.from_numpy(inputs.random_bf16(rng, (A, K)).view(np.int16)).view(torch.bfloat16).cuda()
    st = B.new_status()
    B.awq_grouped_down(x, off, dproj, g, device_status=st)
    gr = torch.from_numpy(inputs.random_bf16(rng, (A, N)).view(np.int16)).view(torch.bfloat16).cuda()
    B.awq_input_backward(gr, off, dproj, g, device_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0  # in-range inputs: nothing reported
    want = 16 if flagged else 0  # MOE_DEVICE_ERR_ACT_RANGE
    x[A - 3, K - 5] = value
    st = B.new_status()
    B.awq_grouped_down(x, off, dproj, g, device_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == want, int(st.item())
    gr[7, 3] = -value
    st = B.new_status()
    B.awq_input_backward(gr, off, dproj, g, device_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == want, int(st.item())


def _bf16_cuda(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("value,flagged", [(4.0e5, True), (float("nan"), True), (float("inf"), False),
                                           (1.2e5, False)],
                         ids=["overflow", "nan", "inf_stays_inf", "in_range"])
@pytest.mark.parametrize("H", [72, 70], ids=["vector_rows", "element_rows"])
def test_f16_dy_from_bf16_inputs(value, flagged, H):
    # moe_combine_backward writing F16 dy from BF16 inputs: one rounding of
    # the FP32 product, bit for bit the oracle's F16 rounding here (w = 0.5
    # makes the product exact), and a value that is not inf but overflows
    # F16 (or a NaN) is reported like the BF16 -> F16 input conversion
    rng = np.random.default_rng(5)
    T, k = 6, 2
    A = T * k
    d_out = inputs.random_bf16(rng, (T, H))
    y = inputs.random_bf16(rng, (A, H))
    wts = np.full((T, k), 0.5, np.float32)
    row_of = np.arange(A, dtype=np.int32).reshape(T, k)
    args = (_bf16_cuda(y), torch.from_numpy(wts).cuda(), torch.from_numpy(row_of).cuda())
    for planted in (False, True):
        if planted:
            d_out[3, 17] = bits(torch.tensor([value], dtype=torch.bfloat16))[0]
        st = B.new_status()
        dy, _ = B.moe_combine_backward(_bf16_cuda(d_out), *args, device_status=st, dy_dtype=torch.float16)
        torch.cuda.synchronize()
        assert dy.dtype == torch.float16
        assert int(st.item()) == (16 if planted and flagged else 0), int(st.item())
        o_dy, _ = oracle.combine_backward(d_out, y, "bf16", wts, row_of, dy_dt="f16")
        got = bits(dy)
        same = (got == o_dy) | (np.isnan(got.view(np.float16)) & np.isnan(o_dy.view(np.float16)))
        assert np.all(same)


@pytest.mark.parametrize("value,flagged", [(2.0e5, True), (float("nan"), True), (float("inf"), False),
                                           (6.0e4, False)],
                         ids=["overflow", "nan", "inf_stays_inf", "in_range"])
@pytest.mark.parametrize("A,I,r,c", [(16, 40, 2, 3), (15, 39, 14, 38)], ids=["vectors", "tail_element"])
def test_f16_swiglu_grads_from_bf16_inputs(value, flagged, A, I, r, c):
    # moe_swiglu_backward writing F16 dG/dU from BF16 dh, G, U (8-element
    # vectors, and the scalar tail when A*I is not a multiple of 8); at
    # G = 0.5, U = 1 the planted dh gives dG = 0.74 dh and dU = 0.31 dh
    rng = np.random.default_rng(6)
    dh, G, U = (inputs.random_bf16(rng, (A, I)) for _ in range(3))
    G[r, c] = bits(torch.tensor([0.5], dtype=torch.bfloat16))[0]
    U[r, c] = bits(torch.tensor([1.0], dtype=torch.bfloat16))[0]
    for planted in (False, True):
        if planted:
            dh[r, c] = bits(torch.tensor([value], dtype=torch.bfloat16))[0]
        st = B.new_status()
        dG, dU = B.moe_swiglu_backward(_bf16_cuda(dh), _bf16_cuda(G), _bf16_cuda(U), out_dtype=torch.float16,
                                       device_status=st)
        torch.cuda.synchronize()
        assert dG.dtype == dU.dtype == torch.float16
        assert int(st.item()) == (16 if planted and flagged else 0), int(st.item())
        if not planted:
            o_dG, o_dU = oracle.swiglu_backward(dh, G, U, "bf16", odt="f16")
            check_close(bits(dG), o_dG, "swiglu_dt/dG", dt="f16", justify=j_swiglu_backward(dh, G, U, which=0))
            check_close(bits(dU), o_dU, "swiglu_dt/dU", dt="f16", justify=j_swiglu_backward(dh, G, U, which=1))


def test_row_index_out_of_range_is_flagged():
    T, H, k, A = 8, 64, 2, 16
    y = torch.ones((A, H), dtype=torch.bfloat16, device="cuda")
    wts = torch.full((T, k), 0.5, dtype=torch.float32, device="cuda")
    sel = torch.tensor([[0, 1]] * T, dtype=torch.int32, device="cuda")
    row_of = torch.arange(T * k, dtype=torch.int32, device="cuda").view(T, k).clone()
    row_of[3, 1] = A + 5
    row_of[5, 0] = -1
    st = B.new_status()
    out = B.moe_combine(y, wts, sel, row_of, device_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & 4
    o = out.float().cpu().numpy()
    assert np.all(o[0] == 1.0) and np.all(o[3] == 0.5) and np.all(o[5] == 0.5)
    st2 = B.new_status()
    B.moe_dispatch_backward(y, row_of, sel, device_status=st2)
    B.moe_combine_backward(out, y, wts, row_of, device_status=st2)
    torch.cuda.synchronize()
    assert int(st2.item()) & 4


def test_zero_tokens():
    x = torch.empty((0, 32), dtype=torch.bfloat16, device="cuda")
    logits = torch.empty((0, 8), dtype=torch.float32, device="cuda")
    r = B.moe_route_dispatch(x, logits, 2, E=8)
    torch.cuda.synchronize()
    assert r["offsets"].cpu().tolist() == [0] * 9
