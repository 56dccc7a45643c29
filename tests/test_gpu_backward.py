"""GPU parity of the backward chain: combine VJP (expert rows and FP32
weights), the down and gate+up input VJPs (transpose of the same rounded
coefficients), the SwiGLU VJP and the COPY-dispatch VJP.  Each step is fed
the device's own inputs and compared with the oracle on the same values."""
import numpy as np
import pytest
import torch

import oracle
from helpers import (bits, check_close, generated, gpu_forward, j_chain, j_combine_backward_dy, j_dispatch_backward,
                     j_input_backward, j_swiglu_backward, sample_rows)
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


def _chain(name, kw, rows=None, tokens=None):
    inp = generated(name, **kw)
    w = inp["workload"]
    dev, buf = gpu_forward(inp, keep_gu=True)
    d_out = dev["d_out"]
    g = ffn.backward(dev, buf, d_out)
    torch.cuda.synchronize()
    r = buf.route
    row_of = r["row_of"].cpu().numpy()
    sel = r["selected_experts"].cpu().numpy().view(np.uint32)
    wts = r["weights"].cpu().numpy()
    offsets = r["offsets"].cpu().numpy()
    rexp_all = (r["row_experts"].cpu().numpy().view(np.uint32).astype(np.int64) - w.expert_start).astype(np.int32)
    y, G, U = bits(buf.y), bits(buf.G), bits(buf.U)
    dy, dh, dG, dU, dv, dx = (bits(g[k]) for k in ("dy", "dh", "dG", "dU", "dvalues", "dx"))
    dw = g["dweights"].cpu().numpy()
    dout = inp["d_out"]
    if rows is None:
        rows = np.arange(w.A)
    if tokens is None:
        tokens = np.arange(w.T)
    # the chain writes dy, dG and dU in the scale dtype when it is F16
    cdt = ffn.operand_dtype(w.scale_dtype)
    assert g["dy"].dtype == g["dG"].dtype == g["dU"].dtype == ffn._SDT[cdt]
    assert g["dh"].dtype == g["dvalues"].dtype == g["dx"].dtype == torch.bfloat16
    # combine VJP on the sampled tokens
    o_dy, o_dw = oracle.combine_backward(dout[tokens], y, "bf16", wts[tokens], row_of[tokens], dy_dt=cdt)
    dy_rows = row_of[tokens].reshape(-1)
    check_close(dy[dy_rows], o_dy[dy_rows], name + "/dy", dt=cdt,
                justify=j_combine_backward_dy(dout[tokens], "bf16", wts[tokens], row_of[tokens], dy_rows))
    assert np.max(np.abs(dw[tokens] - o_dw)) <= 2e-2 * np.sqrt(np.mean(o_dw.astype(np.float64) ** 2)), "dweights"
    # down input VJP, SwiGLU VJP, gate+up input VJP on the sampled rows
    re = rexp_all[rows]
    sdt, gs = w.scale_dtype, w.group
    o_dh = oracle.input_backward(dy[rows], cdt, re, inp["down"], sdt, gs, odt="bf16")
    check_close(dh[rows], o_dh, name + "/dh", justify=j_input_backward(dy[rows], cdt, re, inp["down"], sdt, gs))
    o_dG, o_dU = oracle.swiglu_backward(dh[rows], G[rows], U[rows], "bf16", odt=cdt)
    check_close(dG[rows], o_dG, name + "/dG", dt=cdt, justify=j_swiglu_backward(dh[rows], G[rows], U[rows], which=0))
    check_close(dU[rows], o_dU, name + "/dU", dt=cdt, justify=j_swiglu_backward(dh[rows], G[rows], U[rows], which=1))
    o_dv = oracle.input_backward(dG[rows], cdt, re, inp["gate"], sdt, gs, grad2=dU[rows], proj2=inp["up"],
                                 odt="bf16")
    check_close(dv[rows], o_dv, name + "/dvalues",
                justify=j_input_backward(dG[rows], cdt, re, inp["gate"], sdt, gs, dU[rows], inp["up"]))
    o_dx = oracle.dispatch_backward(dv, "bf16", sel[tokens], row_of[tokens])
    check_close(dx[tokens], o_dx, name + "/dx", justify=j_dispatch_backward(dv, "bf16", sel[tokens], row_of[tokens]))
    # router-logit VJP from the device dweights (FP32 softmax algebra)
    dl = g["dlogits"].cpu().numpy()
    o_dl = oracle.router_backward(inp["logits"][tokens], sel[tokens], dw[tokens], renormalize=w.renormalize,
                                  expert_start=w.expert_start)
    assert np.max(np.abs(dl[tokens] - o_dl)) <= ROUTER_TOL * max(1.0, float(np.max(np.abs(dw[tokens])))), "dlogits"
    assert int(buf.status.item()) == 0
    return w, offsets


# d_logits = w (dw - <w, dw>) in FP32: a few ulps of max|dw| (weights <= 1)
ROUTER_TOL = 1e-5


@pytest.mark.parametrize("renorm", [1, 0])
@pytest.mark.parametrize("E,k", [(8, 2), (64, 6), (512, 10), (4096, 32)])
def test_router_backward_against_oracle(renorm, E, k):
    rng = np.random.default_rng(E + k)
    T = 37
    logits = (rng.standard_normal((T, E)) * 1.5).astype(np.float32)
    sel, _ = oracle.route(logits, None, k, renormalize=renorm, expert_start=3)
    dw = rng.standard_normal((T, k)).astype(np.float32)
    o_dl = oracle.router_backward(logits, sel, dw, renormalize=renorm, expert_start=3)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    dl = B.moe_router_backward(torch.from_numpy(logits).cuda(), torch.from_numpy(sel.view(np.int32)).cuda(),
                               torch.from_numpy(dw).cuda(), renormalize=renorm, expert_start=3, device_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert np.max(np.abs(dl.cpu().numpy() - o_dl)) <= ROUTER_TOL * max(1.0, float(np.max(np.abs(dw))))
    if renorm:  # unselected experts get exactly zero
        mask = np.ones((T, E), bool)
        np.put_along_axis(mask, (sel.astype(np.int64) - 3), False, axis=1)
        assert np.all(dl.cpu().numpy()[mask] == 0)


SMALL = {"skewed": dict(T=1024, H=512, I=256, E=16), "prefill": dict(T=512, H=256, I=128, E=16, backward=True),
         "decode": dict(backward=True), "tiny": dict(backward=True),
         # output widths that end inside a 256-column tile, four zero/scale groups per tile
         "ragged": dict(T=512, H=320, I=192, E=8, group=64),
         # pair-tile input VJP with an output width ending mid-tile and two group rows per CTA
         "ragged_pair": dict(T=512, H=384, I=256, E=8, group=64)}


@pytest.mark.parametrize("name", list(SMALL))
def test_backward_chain_every_row(name, path):
    _chain("skewed" if name.startswith("ragged") else name, SMALL[name])


def test_backward_full_size_skewed_sampled(path):
    inp = generated("skewed")
    w = inp["workload"]
    sel, _ = oracle.route(inp["logits"], None, w.top_k)
    off, _, _, _ = oracle.dispatch(sel, w.E)
    rows = sample_rows(off, n_experts=3, rows_per=4)
    tokens = np.array([0, 5, w.T // 2, w.T - 1])
    _chain("skewed", {}, rows=rows, tokens=tokens)


def test_backward_skewed_hot_median_smallest_experts_every_row(path):
    # every row of the hottest, a median and the smallest non-empty expert of
    # the full-size skewed workload, and the tokens that select them
    from test_gpu_full_size import skewed_rows_and_tokens
    inp = generated("skewed")
    w = inp["workload"]
    sel, _ = oracle.route(inp["logits"], None, w.top_k)
    off, _, _, row_of = oracle.dispatch(sel, w.E)
    rows, tokens, _ = skewed_rows_and_tokens(off, row_of, sel, w.expert_start)
    _chain("skewed", {}, rows=rows, tokens=tokens)


def test_whole_chain_against_oracle_chain():
    """Oracle forward + backward from scratch vs the device chain (no shared intermediates)."""
    inp = generated("skewed", T=256, H=256, I=128, E=8)
    w = inp["workload"]
    dev, buf = gpu_forward(inp, keep_gu=True)
    g = ffn.backward(dev, buf, dev["d_out"])
    torch.cuda.synchronize()
    f = oracle.forward(inp)
    rexp = (f["row_experts"].astype(np.int64) - w.expert_start).astype(np.int32)
    cdt = ffn.operand_dtype(w.scale_dtype)  # dy, dG, dU: F16 with F16 scales
    o_dy, o_dw = oracle.combine_backward(inp["d_out"], f["y"], "bf16", f["weights"], f["row_of"], dy_dt=cdt)
    o_dh = oracle.input_backward(o_dy, cdt, rexp, inp["down"], w.scale_dtype, w.group, odt="bf16")
    o_dG, o_dU = oracle.swiglu_backward(o_dh, f["G"], f["U"], "bf16", odt=cdt)
    o_dv = oracle.input_backward(o_dG, cdt, rexp, inp["gate"], w.scale_dtype, w.group, grad2=o_dU,
                                 proj2=inp["up"], odt="bf16")
    o_dx = oracle.dispatch_backward(o_dv, "bf16", f["selected"], f["row_of"])
    # end to end: a flip is justified by the last step's FP32 bound plus the
    # measured difference between the exact values on the device's upstream
    # tensors and on the oracle's (each step is checked on its own elsewhere)
    dG, dU, dv = bits(g["dG"]), bits(g["dU"]), bits(g["dvalues"])
    j_dv = j_chain(j_input_backward(o_dG, cdt, rexp, inp["gate"], w.scale_dtype, w.group, o_dU, inp["up"]),
                   j_input_backward(dG, cdt, rexp, inp["gate"], w.scale_dtype, w.group, dU, inp["up"]))
    j_dx = j_chain(j_dispatch_backward(o_dv, "bf16", f["selected"], f["row_of"]),
                   j_dispatch_backward(dv, "bf16", f["selected"], f["row_of"]))
    check_close(bits(g["dx"]), o_dx, "chain/dx", justify=j_dx)
    check_close(dv, o_dv, "chain/dvalues", justify=j_dv)


@pytest.mark.parametrize("group", [256, 512])
def test_backward_chain_large_groups(group, path):
    # zero/scale groups spanning two or four 128-deep steps of the tcgen05 tiles
    _chain("skewed", dict(T=300, H=1024, I=512, E=8, group=group))
