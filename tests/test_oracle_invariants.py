"""Invariants, adjoint identities and finite differences of the CPU oracle.

- routing/dispatch invariants on workload-shaped data (counts sum to T*k,
  distinct IDs per token, weights >= 0 summing to 1, expert-sorted rows with
  ascending tokens, row_of a bijection);
- combine special cases (top_k = 1, one-hot weights, order independence);
- <J x, g> = <x, J^T g> for each projection in exact mode;
- a central finite difference of the exact-mode whole FFN against the
  exact-mode VJP chain (combine VJP -> down VJP -> SwiGLU VJP -> gate/up VJP
  -> COPY VJP);
- dweights in closed form; the logit VJP against finite differences.
"""
import numpy as np
import pytest

import oracle
from moe_routed_experts_b200 import inputs
from moe_routed_experts_b200.configs import WORKLOADS, scaled


def _f(a):
    return inputs.bf16_bits_to_f32(a).astype(np.float64)


@pytest.mark.parametrize("name", ["tiny", "decode", "wide", "skewed"])
def test_route_dispatch_invariants(name):
    w = WORKLOADS[name]
    if w.T > 2048:
        w = scaled(w, T=2048)
    inp = inputs.generate(scaled(w, H=64, I=64, E=w.E), with_grad=False)
    sel, wts = oracle.route(inp["logits"], inp["sel_bias"], w.top_k)
    T, k, E = w.T, w.top_k, w.E
    assert sel.shape == (T, k)
    for t in range(T):
        assert len(set(sel[t].tolist())) == k
        assert np.all(sel[t] < E)
    assert np.all(wts >= 0)
    assert np.all(np.abs(wts.astype(np.float64).sum(1) - 1.0) <= 2e-6)
    # selection is the k best scores, descending, ties to the lower ID
    score = inp["logits"] + (inp["sel_bias"] if inp["sel_bias"] is not None else 0)
    for t in range(0, T, max(1, T // 64)):
        order = sorted(range(E), key=lambda e: (-float(score[t, e]), e))[:k]
        assert sel[t].tolist() == order
    off, rexp, src, row_of = oracle.dispatch(sel, E)
    A = T * k
    assert off[0] == 0 and off[-1] == A and np.all(np.diff(off) >= 0)
    counts = np.bincount(sel.reshape(-1), minlength=E)
    assert np.array_equal(np.diff(off), counts)
    for e in range(E):
        rows = slice(off[e], off[e + 1])
        assert np.all(rexp[rows] == e)
        assert np.all(np.diff(src[rows]) > 0)
    assert np.array_equal(np.sort(row_of.reshape(-1)), np.arange(A))
    for t in range(T):
        for j in range(k):
            r = row_of[t, j]
            assert src[r] == t and rexp[r] == sel[t, j]
    values = oracle.copy_rows(inp["x"], src)
    assert np.array_equal(values, inp["x"][src])


def test_skewed_routing_is_heavily_imbalanced():
    w = WORKLOADS["skewed"]
    inp = inputs.generate(scaled(w, H=64, I=64), with_grad=False)
    sel, _ = oracle.route(inp["logits"], None, w.top_k)
    counts = np.bincount(sel.reshape(-1), minlength=w.E)
    assert counts.max() > 10 * w.A / w.E
    assert (counts == 0).sum() >= 10


def test_combine_special_cases():
    rng = np.random.default_rng(3)
    T, H, k = 5, 16, 3
    y = inputs.random_bf16(rng, (T * k, H))
    sel = np.array([[4, 1, 7], [0, 2, 3], [9, 8, 5], [1, 2, 0], [6, 3, 4]], np.uint32)
    row_of = rng.permutation(T * k).reshape(T, k).astype(np.int32)
    # one-hot weights pick a single row exactly
    w1 = np.zeros((T, k), np.float32)
    w1[:, 1] = 1.0
    out = oracle.combine(y, "bf16", w1, sel, row_of)
    assert np.array_equal(out, y[row_of[:, 1]])
    # permuting the selections inside a token changes nothing (ascending-ID rule)
    wts = rng.uniform(0, 1, (T, k)).astype(np.float32)
    out_a = oracle.combine(y, "bf16", wts, sel, row_of)
    perm = np.array([2, 0, 1])
    out_b = oracle.combine(y, "bf16", wts[:, perm], sel[:, perm], row_of[:, perm])
    assert np.array_equal(out_a, out_b)
    # top_k = 1 with weight 1 is the row itself
    out1 = oracle.combine(y[:T], "bf16", np.ones((T, 1), np.float32), sel[:, :1], np.arange(T, dtype=np.int32)[:, None])
    assert np.array_equal(out1, y[:T])
    # top_k = 1 COPY VJP is the identity permutation
    dx = oracle.dispatch_backward(y[:T], "bf16", sel[:, :1], np.arange(T, dtype=np.int32)[::-1].copy()[:, None])
    assert np.array_equal(dx, y[:T][::-1])


def test_dispatch_backward_hand_worked_top3():
    """COPY VJP with top_k = 3 ([MX] moe_dispatch_backward sums the selected
    expert-row seeds of each token, no routing weights).  Two tokens, six
    distinct rows; every sum is exact in BF16, so dx is known by hand:
      token 0 selects experts (5, 2, 9) in rows (3, 0, 5):
        dx[0] = dv[3] + dv[0] + dv[5] = (0.5 + 1 + 64, -1 + 2 - 128) = (65.5, -127)
      token 1 selects experts (1, 7, 3) in rows (2, 4, 1):
        dx[1] = dv[2] + dv[4] + dv[1] = (16 - 3 + 4, 32 + 0.25 + 8) = (17, 40.25)"""
    dv = np.array([[1, 2], [4, 8], [16, 32], [0.5, -1], [-3, 0.25], [64, -128]], np.float32)
    sel = np.array([[5, 2, 9], [1, 7, 3]], np.uint32)
    row_of = np.array([[3, 0, 5], [2, 4, 1]], np.int32)
    dx = oracle.dispatch_backward(inputs.f32_to_bf16_bits(dv), "bf16", sel, row_of)
    assert np.array_equal(_f(dx), np.array([[65.5, -127.0], [17.0, 40.25]]))
    # the same in exact mode, and with the selections of a token permuted
    dx64 = oracle.dispatch_backward(dv.astype(np.float64), "f64", sel, row_of)
    assert np.array_equal(dx64, np.array([[65.5, -127.0], [17.0, 40.25]]))
    perm = np.array([2, 0, 1])
    dxp = oracle.dispatch_backward(inputs.f32_to_bf16_bits(dv), "bf16", sel[:, perm].copy(), row_of[:, perm].copy())
    assert np.array_equal(dxp, dx)


def test_dweights_closed_form_and_dy():
    rng = np.random.default_rng(4)
    T, H, k = 6, 32, 2
    y = inputs.random_bf16(rng, (T * k, H))
    d_out = inputs.random_bf16(rng, (T, H))
    wts = rng.uniform(0, 1, (T, k)).astype(np.float32)
    row_of = rng.permutation(T * k).reshape(T, k).astype(np.int32)
    dy, dw = oracle.combine_backward(d_out, y, "bf16", wts, row_of)
    for t in range(T):
        for j in range(k):
            r = row_of[t, j]
            assert dw[t, j] == np.float32(np.dot(_f(d_out[t]), _f(y[r])))
            want = inputs.f32_to_bf16_bits((wts[t, j].astype(np.float64) * _f(d_out[t])).astype(np.float32))
            # the product of an f32 and a bf16 is exact in double; double->f32->bf16 may
            # double-round only on exact ties, which random data does not hit
            assert np.array_equal(dy[r], want)
    only_dw = oracle.combine_backward(d_out, y, "bf16", wts, row_of, want_dy=False)
    assert only_dw[0] is None and np.array_equal(only_dw[1], dw)


def test_incomplete_group_is_rejected():
    rng = np.random.default_rng(1)
    proj = inputs.draw_projection(rng, 1, 48, 16, 16, "f16", False, 0.0)
    with pytest.raises(ValueError):
        oracle.project(np.zeros((1, 48), np.uint16), "bf16", np.zeros(1, np.int32), proj, "f16", 32)


@pytest.mark.parametrize("sdt", ["f16", "bf16"])
def test_projection_adjoint_identity(sdt):
    rng = np.random.default_rng(8)
    E, K, N, g, R = 3, 64, 48, 16, 11
    proj = inputs.draw_projection(rng, E, K, N, g, sdt, False, 0.0)
    rexp = rng.integers(0, E, R).astype(np.int32)
    x = rng.standard_normal((R, K))
    gy = rng.standard_normal((R, N))
    Jx = oracle.project(x, "f64", rexp, proj, sdt, g, exact=True)
    JTg = oracle.input_backward(gy, "f64", rexp, proj, sdt, g, exact=True)
    lhs, rhs = np.sum(Jx * gy), np.sum(x * JTg)
    assert abs(lhs - rhs) <= 1e-12 * (abs(lhs) + np.sum(np.abs(Jx * gy)))


def _exact_chain(inp, xs, route_res):
    """Exact-mode forward of tokens xs (float64 [T,H]) at a fixed routing."""
    w = inp["workload"]
    sel, wts, off, rexp, src, row_of = route_res
    vals = xs[src]
    re = rexp.astype(np.int32)
    G = oracle.project(vals, "f64", re, inp["gate"], w.scale_dtype, w.group, exact=True)
    U = oracle.project(vals, "f64", re, inp["up"], w.scale_dtype, w.group, exact=True)
    s = 1.0 / (1.0 + np.exp(-G))
    h = G * s * U
    y = oracle.project(h, "f64", re, inp["down"], w.scale_dtype, w.group, exact=True)
    out = np.zeros_like(xs)
    for t in range(xs.shape[0]):
        for j in np.argsort(sel[t]):
            out[t] += float(wts[t, j]) * y[row_of[t, j]]
    return out, (G, U, h, y)


@pytest.mark.parametrize("sdt", ["f16", "bf16"])
def test_whole_ffn_vjp_matches_finite_difference(sdt):
    w = scaled(WORKLOADS["tiny"], T=6, H=32, I=48, E=4, top_k=2, group=16, scale_dtype=sdt)
    inp = inputs.generate(w)
    rng = np.random.default_rng(9)
    sel, wts = oracle.route(inp["logits"], None, w.top_k)
    off, rexp, src, row_of = oracle.dispatch(sel, w.E)
    rr = (sel, wts, off, rexp, src, row_of)
    x0 = _f(inp["x"])
    d_out = rng.standard_normal(x0.shape)
    out, (G, U, h, y) = _exact_chain(inp, x0, rr)
    # the oracle's own VJP chain, every step in exact (unrounded double) mode
    dy, _ = oracle.combine_backward(d_out, y, "f64", wts, row_of, want_dw=False)
    re = rexp.astype(np.int32)
    dh = oracle.input_backward(dy, "f64", re, inp["down"], sdt, w.group, exact=True)
    dG, dU = oracle.swiglu_backward(dh, G, U, "f64")
    dvals = oracle.input_backward(dG, "f64", re, inp["gate"], sdt, w.group, grad2=dU, proj2=inp["up"], exact=True)
    dx = oracle.dispatch_backward(dvals, "f64", sel, row_of)
    v = rng.standard_normal(x0.shape)
    eps = 1e-6
    fp = np.sum(_exact_chain(inp, x0 + eps * v, rr)[0] * d_out)
    fm = np.sum(_exact_chain(inp, x0 - eps * v, rr)[0] * d_out)
    fd = (fp - fm) / (2 * eps)
    an = np.sum(dx * v)
    assert abs(fd - an) <= 1e-6 * max(1.0, abs(an))


def test_swiglu_backward_storage_matches_exact_formula():
    rng = np.random.default_rng(10)
    n = 4096
    G, U, dh = (inputs.random_bf16(rng, (n,), 2.0) for _ in range(3))
    dG, dU = oracle.swiglu_backward(dh, G, U)
    g, u, d = _f(G), _f(U), _f(dh)
    # finite difference of h = silu(G) U in double
    eps = 1e-7
    hf = lambda a, b: a / (1.0 + np.exp(-a)) * b
    fdG = (hf(g + eps, u) - hf(g - eps, u)) / (2 * eps) * d
    fdU = (hf(g, u + eps) - hf(g, u - eps)) / (2 * eps) * d
    assert np.max(np.abs(_f(dG) - fdG)) <= 2.0 ** -7 * np.max(np.abs(fdG)) + 1e-6
    assert np.max(np.abs(_f(dU) - fdU)) <= 2.0 ** -7 * np.max(np.abs(fdU)) + 1e-6


@pytest.mark.parametrize("renorm", [1, 0])
def test_router_backward_matches_finite_difference(renorm):
    rng = np.random.default_rng(12)
    T, E, k = 4, 7, 3
    logits = rng.standard_normal((T, E)).astype(np.float32)
    sel, _ = oracle.route(logits, None, k, renormalize=renorm)
    dw = rng.standard_normal((T, k)).astype(np.float32)
    dl = oracle.router_backward(logits, sel, dw, renormalize=renorm)

    def weights(l):  # float64 weights at the fixed selection
        out = np.zeros((T, k))
        for t in range(T):
            ex = np.exp(l[t] - l[t].max())
            den = ex[sel[t]].sum() if renorm else ex.sum()
            out[t] = ex[sel[t]] / den
        return out

    l0 = logits.astype(np.float64)
    eps = 1e-6
    for t in range(T):
        for e in range(E):
            lp, lm = l0.copy(), l0.copy()
            lp[t, e] += eps
            lm[t, e] -= eps
            fd = np.sum((weights(lp) - weights(lm))[t] * dw[t]) / (2 * eps)
            assert abs(dl[t, e] - fd) <= 1e-5 * max(1.0, abs(fd)), (t, e)
        if renorm:
            unsel = np.setdiff1d(np.arange(E), sel[t])
            assert np.all(dl[t, unsel] == 0)
