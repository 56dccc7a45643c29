"""GPU parity of every C-ABI entry point against the CPU oracle, on the same
seeded inputs.  Indices, dispatch order, offsets and the rounded
coefficients bit for bit; FP32 weights within 2e-6; BF16/F16 outputs and
gradients within 2e-2 * rms(oracle)."""
import numpy as np
import pytest
import torch

import oracle
from helpers import (TOL, as_f64, bits, check_close, check_forward_steps, check_routing, generated, gpu_forward,
                     gpu_forward_numpy, sample_rows, u32, values_in)
from moe_routed_experts_b200 import binding as B
from moe_routed_experts_b200 import ffn, inputs
from moe_routed_experts_b200.configs import WORKLOADS, Workload, scaled

pytestmark = pytest.mark.gpu

PATHS = [1, 2, 3]


@pytest.fixture(params=PATHS, ids=["warp_tiles", "tcgen05_tiles", "tcgen05_pair_tiles"])
def path(request):
    p = request.param
    try:
        prev = B.set_projection_path(p)
    except ValueError:
        pytest.skip("projection path %d not available" % p)
    yield p
    B.set_projection_path(prev)


# ------------------------------------------------------------------ coefficients

@pytest.mark.parametrize("sdt", ["f16", "bf16"])
@pytest.mark.parametrize("pairing", [0, 1])
def test_coefficients_bit_exact(sdt, pairing):
    rng = np.random.default_rng(21)
    K, N, g = 512, 512, 16
    proj = inputs.draw_projection(rng, 1, K, N, g, sdt, False, 0.0)
    # widen the scale range well beyond the workloads', including F16 subnormals
    raw = rng.integers(0, 0x7B00 if sdt == "f16" else 0x7F00, size=proj["scales"].shape).astype(np.uint16)
    raw[0, 0, :64] = np.arange(64, dtype=np.uint16)  # smallest magnitudes / subnormals
    proj["scales"] = raw
    dev = ffn.projection_to_device(proj, sdt)
    got = bits(B.awq_dequant_coefficients(dev["qweight"][0], dev["qzeros"][0], dev["scales"][0], g, pairing))
    _, want = oracle.dequant(proj["qweight"][0], proj["qzeros"][0], proj["scales"][0], sdt, K, N, g)
    mism = np.nonzero(got != want.astype(np.uint16))
    assert mism[0].size == 0, "first mismatches at %s" % (list(zip(*[m[:5] for m in mism])),)


# ------------------------------------------------------------------ routing and dispatch

@pytest.mark.parametrize("name", list(WORKLOADS))
def test_route_dispatch_full_size(name):
    inp = generated(name)
    w = inp["workload"]
    dev = ffn.to_device(inp)
    st = B.new_status()
    r = B.moe_route_dispatch(dev["x"], dev["logits"], w.top_k, E=w.E, sel_bias=dev["sel_bias"], device_status=st)
    torch.cuda.synchronize()
    sel, wts = oracle.route(inp["logits"], inp["sel_bias"], w.top_k)
    off, rexp, src, row_of = oracle.dispatch(sel, w.E)
    got = {"selected": u32(r["selected_experts"]), "weights": r["weights"].cpu().numpy(),
           "offsets": r["offsets"].cpu().numpy(), "row_experts": u32(r["row_experts"]),
           "src_token": r["src_token"].cpu().numpy(), "row_of": r["row_of"].cpu().numpy()}
    check_routing(got, {"selected": sel, "weights": wts, "offsets": off, "row_experts": rexp, "src_token": src,
                        "row_of": row_of}, name)
    src_t = torch.from_numpy(src.astype(np.int64)).cuda()
    assert torch.equal(r["values"], dev["x"][src_t]), "values are not bit copies of x[src_token]"
    assert int(st.item()) == 0
    # the F16 form of the COPY: each row's exact F16 image (torch's cast rounds to nearest even)
    r16 = B.moe_route_dispatch(dev["x"], dev["logits"], w.top_k, E=w.E, sel_bias=dev["sel_bias"], device_status=st,
                               values_dtype=torch.float16)
    torch.cuda.synchronize()
    assert r16["values"].dtype == torch.float16
    assert torch.equal(r16["values"].view(torch.int16), dev["x"][src_t].to(torch.float16).view(torch.int16))
    assert torch.equal(r16["row_of"], r["row_of"]) and torch.equal(r16["offsets"], r["offsets"])
    assert int(st.item()) == 0


@pytest.mark.parametrize("renorm,expert_start", [(0, 0), (1, 7), (0, 100)])
def test_route_dispatch_options(renorm, expert_start):
    w = Workload("opt", T=300, H=64, I=32, E=40, top_k=5, group=16, scale_dtype="f16", sel_bias_std=0.3,
                 expert_start=expert_start, renormalize=renorm)
    inp = inputs.generate(w)
    dev = ffn.to_device(inp)
    r = B.moe_route_dispatch(dev["x"], dev["logits"], w.top_k, E=w.E, sel_bias=dev["sel_bias"],
                             expert_start=expert_start, renormalize=renorm)
    sel, wts = oracle.route(inp["logits"], inp["sel_bias"], w.top_k, renorm, expert_start)
    off, rexp, src, row_of = oracle.dispatch(sel, w.E, expert_start)
    got = {"selected": u32(r["selected_experts"]), "weights": r["weights"].cpu().numpy(),
           "offsets": r["offsets"].cpu().numpy(), "row_experts": u32(r["row_experts"]),
           "src_token": r["src_token"].cpu().numpy(), "row_of": r["row_of"].cpu().numpy()}
    check_routing(got, {"selected": sel, "weights": wts, "offsets": off, "row_experts": rexp, "src_token": src,
                        "row_of": row_of}, "options")


@pytest.mark.parametrize("H", [20, 64], ids=["two_byte_rows", "sixteen_byte_rows"])
@pytest.mark.parametrize("value,flagged", [(None, False), (70000.0, True), (float("nan"), True),
                                           (float("inf"), False), (1e-7, False)],
                         ids=["plain", "overflow", "nan", "inf_converts_exactly", "below_f16_subnormal_grid"])
def test_route_dispatch_f16_rows(H, value, flagged):
    # the F16 form of the COPY on both copy paths (H = 20: 40-byte rows, one
    # 2-byte element per lane; H = 64: 16-byte vectors): each row is the F16
    # image of the BF16 token row (torch's cast rounds to nearest even), the
    # row maps equal the plain COPY's, and only a finite value above F16's
    # range or a NaN is reported (MOE_DEVICE_ERR_ACT_RANGE)
    T, E, k = 150, 12, 3
    rng = np.random.default_rng(H)
    logits = rng.standard_normal((T, E), dtype=np.float32)
    x = inputs.random_bf16(rng, (T, H))
    if value is not None:
        x[37, H - 3] = bits(torch.tensor([value], dtype=torch.bfloat16))[0]
    xd = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    ld = torch.from_numpy(logits).cuda()
    st, st16 = B.new_status(), B.new_status()
    r = B.moe_route_dispatch(xd, ld, k, E=E, device_status=st)
    r16 = B.moe_route_dispatch(xd, ld, k, E=E, device_status=st16, values_dtype=torch.float16)
    torch.cuda.synchronize()
    assert r16["values"].dtype == torch.float16
    for key in ("selected_experts", "weights", "offsets", "row_experts", "src_token", "row_of"):
        assert torch.equal(r16[key], r[key]), key
    want = r["values"].to(torch.float16)
    nan = torch.isnan(want)  # NaN payloads may differ: compare NaN-ness there
    assert torch.equal(torch.isnan(r16["values"]), nan)
    assert torch.equal(r16["values"].view(torch.int16)[~nan], want.view(torch.int16)[~nan])
    assert int(st.item()) == 0
    assert int(st16.item()) == (16 if flagged else 0), int(st16.item())


def test_route_ties_and_empty_experts():
    # many exact ties (logits on a coarse grid) and experts nobody picks
    T, E, k = 700, 96, 4
    rng = np.random.default_rng(3)
    logits = (rng.integers(0, 3, (T, E)).astype(np.float32))
    logits[:, 50:] = -5.0
    x = inputs.random_bf16(rng, (T, 24))
    xd = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    r = B.moe_route_dispatch(xd, torch.from_numpy(logits).cuda(), k, E=E)
    sel, wts = oracle.route(logits, None, k)
    off, rexp, src, row_of = oracle.dispatch(sel, E)
    assert np.array_equal(u32(r["selected_experts"]), sel)
    assert np.array_equal(r["offsets"].cpu().numpy(), off)
    assert np.array_equal(r["src_token"].cpu().numpy(), src)
    assert np.array_equal(r["row_of"].cpu().numpy(), row_of)
    assert np.all(np.diff(off)[50:] == 0)


@pytest.mark.parametrize("with_bias", [False, True])
def test_route_signed_zero_ties(with_bias):
    # scores of -0 and +0 are equal (a tie, lower ID first) on both sides;
    # with the selection bias, zero sums arise as x + (-x) = +0 and
    # (-0) + (-0) = -0.  A few NaN logits (invalid input) rank as -inf.
    T, E, k = 257, 40, 6
    rng = np.random.default_rng(5)
    logits = rng.choice(np.array([-0.0, 0.0, -1.0, 1.0, -np.inf], np.float32), size=(T, E))
    logits[rng.integers(0, T, 20), rng.integers(0, E, 20)] = np.nan
    bias = None
    if with_bias:
        bias = rng.choice(np.array([-0.0, 0.0, -1.0, 1.0], np.float32), size=E)
    x = inputs.random_bf16(rng, (T, 16))
    xd = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    r = B.moe_route_dispatch(xd, torch.from_numpy(logits).cuda(), k, E=E,
                             sel_bias=None if bias is None else torch.from_numpy(bias).cuda())
    sel, wts = oracle.route(logits, bias, k)
    off, rexp, src, row_of = oracle.dispatch(sel, E)
    assert np.array_equal(u32(r["selected_experts"]), sel)
    assert np.array_equal(r["offsets"].cpu().numpy(), off)
    assert np.array_equal(r["src_token"].cpu().numpy(), src)
    assert np.array_equal(r["row_of"].cpu().numpy(), row_of)
    ok = np.all(np.isfinite(wts), axis=1)  # tokens whose selection holds no NaN
    assert np.max(np.abs(r["weights"].cpu().numpy()[ok] - wts[ok])) <= 2e-6


def test_route_large_expert_count_and_top_k_32():
    T, E, k = 130, 4096, 32
    rng = np.random.default_rng(4)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    x = inputs.random_bf16(rng, (T, 8))
    xd = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    r = B.moe_route_dispatch(xd, torch.from_numpy(logits).cuda(), k, E=E)
    sel, wts = oracle.route(logits, None, k)
    off, rexp, src, row_of = oracle.dispatch(sel, E)
    assert np.array_equal(u32(r["selected_experts"]), sel)
    assert np.max(np.abs(r["weights"].cpu().numpy() - wts)) <= 2e-6
    assert np.array_equal(r["offsets"].cpu().numpy(), off)
    assert np.array_equal(r["row_of"].cpu().numpy(), row_of)


# ------------------------------------------------------------------ forward, every row

SMALL = {
    "tiny": {},
    "decode": {},
    "prefill": dict(T=512, H=256, I=128, E=16),
    "wide": dict(T=256, H=256, I=128, E=64),
    "skewed": dict(T=1024, H=512, I=256, E=16),
}


def _oracle_forward_all(inp):
    return oracle.forward(inp)


@pytest.mark.parametrize("name", list(SMALL))
def test_forward_every_row(name, path):
    inp = generated(name, **SMALL[name])
    res, dev, buf = gpu_forward_numpy(inp)
    want = _oracle_forward_all(inp)
    check_routing(res, want, name)
    assert np.array_equal(res["values"], values_in(res["values_dt"], want["values"]))
    check_forward_steps(inp, res, want, name)
    assert res["status"] == 0


def test_forward_is_deterministic(path):
    inp = generated("prefill", **SMALL["prefill"])
    a, _, _ = gpu_forward_numpy(inp)
    b, _, _ = gpu_forward_numpy(inp)
    for key in ("values", "G", "U", "h", "y", "out"):
        assert np.array_equal(a[key], b[key]), key


# ------------------------------------------------------------------ forward, full size, sampled rows

@pytest.mark.parametrize("name", ["decode", "prefill", "wide", "skewed"])
def test_forward_full_size_sampled(name, path):
    inp = generated(name)
    w = inp["workload"]
    res, dev, buf = gpu_forward_numpy(inp)
    rows = sample_rows(res["offsets"], n_experts=4, rows_per=6)
    tokens = np.array([0, w.T // 3, w.T - 1], np.int64)
    want = oracle.forward(inp, rows=rows, tokens=tokens)
    check_forward_steps(inp, res, want, name, rows=want["rows_used"], tokens=tokens)
    assert res["status"] == 0
