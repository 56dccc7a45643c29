"""Shared helpers of the GPU parity tests: device runs through the C ABI,
oracle runs on the same seeded inputs, and the tolerance checks.

Tolerance (floating outputs and gradients): |got - oracle| <= 2e-2 *
rms(oracle) per tensor.  An element beyond that bound passes only when its
difference is a rounding flip that the arithmetic explains: the device
accumulates in FP32 (the oracle in double), so when the exact result lies
within the FP32 error bound of a rounding midpoint of the storage format,
the device may store the other neighbour of the exact value.  With 8
significant bits, one such step at |v| > ~2.6 rms already exceeds 2e-2 rms.
For each such element the oracle supplies the unrounded value v and an
error bound b (from the magnitudes of the summed terms, computed by the
oracle in the same pass): the element passes iff got is the RNE image of a
real within b of v (for a step bound: the neighbour of RNE(v) on v's side,
with v within b of their midpoint).  End-to-end checks widen b by the
measured difference between the exact values on the device's upstream
tensors and on the oracle's.
Every check records its max err/rms and the count of such flips (printed in
the pytest summary).  Integer and index outputs, and the rounded
coefficients, must match bit for bit; FP32 routing weights within 2e-6.
"""
import functools

import numpy as np
import torch

import oracle
from moe_routed_experts_b200 import binding as B
from moe_routed_experts_b200 import ffn, inputs
from moe_routed_experts_b200.configs import WORKLOADS, scaled

TOL = 2e-2
WEIGHT_TOL = 2e-6
# unit roundoff of an FP32 accumulation step; 2^-23 rather than 2^-24 so the
# bound also holds for an adder that truncates instead of rounding
U32_ROUNDOFF = 2.0 ** -23
# relative error of the FP32 elementwise steps (fast exponential and division
# of silu and its VJP: a few ulps of FP32), with margin
ELEMWISE_REL = 2.0 ** -17

# (name, max err / rms, elements beyond the strict bound, elements) per check
REPORT = []


def bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def u32(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().cpu().numpy().view(np.uint32)


def as_f64(b: np.ndarray, dt: str = "bf16") -> np.ndarray:
    if dt == "bf16":
        return inputs.bf16_bits_to_f32(b).astype(np.float64)
    if dt == "f16":
        return inputs.f16_bits_to_f32(b).astype(np.float64)
    return np.asarray(b, np.float64)


def _ordered(b: np.ndarray) -> np.ndarray:
    """16-bit float bits -> integers in the order of the values (+-0 -> 0)."""
    b = np.asarray(b).astype(np.int64)
    mag = b & 0x7FFF
    return np.where(b & 0x8000, -mag, mag)


def _from_ordered(o: np.ndarray) -> np.ndarray:
    o = np.asarray(o, np.int64)
    return np.where(o < 0, (-o) | 0x8000, o).astype(np.uint16)


def rounding_justified(got_b, exact, bound, dt="bf16"):
    """Element-wise: got is the round-to-nearest-even image of some real within
    `bound` of `exact`, i.e. the distance from `exact` to the interval of reals
    that round to got (between got's midpoints with its two storage
    neighbours) is at most `bound`.  With an FP32-accumulation bound this
    admits exactly the rounding flips that bound explains (got is RNE(exact)'s
    neighbour on the side of `exact` and `exact` lies within `bound` of their
    midpoint); with an end-to-end bound widened by measured upstream
    differences it admits what those differences explain, and no more."""
    og = _ordered(got_b)
    g = as_f64(got_b, dt)
    with np.errstate(over="ignore", invalid="ignore"):
        lo = 0.5 * (g + as_f64(_from_ordered(og - 1), dt))
        hi = 0.5 * (g + as_f64(_from_ordered(og + 1), dt))
    dist = np.maximum(0.0, np.maximum(lo - exact, exact - hi))
    return dist <= bound


def check_close(got, want, name, dt="bf16", tol=TOL, justify=None):
    """got/want: storage bits (16-bit) of the same shape.  justify(rows, cols)
    -> (exact, bound) for the listed elements of a 2-D tensor; without it the
    strict bound alone applies."""
    got, want = np.asarray(got), np.asarray(want)
    g, w = as_f64(got, dt), as_f64(want, dt)
    assert g.shape == w.shape, (name, g.shape, w.shape)
    assert np.all(np.isfinite(g)), name + ": non-finite values"
    if not w.size:
        return 0.0
    rms = float(np.sqrt(np.mean(w * w)))
    err = np.abs(g - w)
    strict = tol * rms
    over = np.nonzero(err.reshape(-1) > strict)[0]
    if over.size:
        worst = int(over[np.argmax(err.reshape(-1)[over])])
        msg = "%s: err %.4g at value %.4g > %.3g * rms %.4g" % (name, err.reshape(-1)[worst], w.reshape(-1)[worst],
                                                                 tol, rms)
        assert justify is not None, msg + " (%d elements, no flip justification available)" % over.size
        shape2 = got.shape if got.ndim == 2 else (1, got.size)
        rows, cols = np.unravel_index(over, shape2)
        exact, bound = justify(rows, cols)
        ok = rounding_justified(got.reshape(-1)[over], exact, bound, dt)
        if not np.all(ok):
            i = int(np.nonzero(~ok)[0][0])
            raise AssertionError(msg + "; not a justified rounding flip at [%d, %d]: got %.6g, oracle %.6g, exact "
                                 "%.9g, bound %.3g (%d of %d elements beyond the bound unexplained)" % (
                                     rows[i], cols[i], g.reshape(-1)[over[i]], w.reshape(-1)[over[i]], exact[i],
                                     bound[i], int((~ok).sum()), over.size))
    ratio = float(err.max()) / max(rms, 1e-30)
    REPORT.append((name, ratio, int(over.size), int(w.size)))
    return ratio


# ---------------------------------------------------------------- flip justifications
#
# Each factory returns justify(rows, cols) for check_close: the oracle's
# unrounded value of the listed elements and the bound of the device's FP32
# evaluation error there.  Only rows holding a flagged element are recomputed.

def _rowwise(fn):
    def justify(rows, cols):
        ur, inv = np.unique(rows, return_inverse=True)
        exact, bound = fn(ur)
        return exact[inv, cols], bound[inv, cols]
    return justify


def _conversion_rel(xdt, sdt):
    """Relative error of converting the activations to the scale dtype for
    the tensor-core product: none for BF16 -> F16 in F16's normal range, one
    rounding to 8 significant bits for F16 -> BF16."""
    return 2.0 ** -9 if (xdt == "f16" and sdt == "bf16") else 0.0


def j_project(x, xdt, rexp, proj, sdt, g, bias_dt="f32"):
    """Rows of a grouped projection: K products + bias + split-K partials."""
    K = x.shape[1]

    def fn(ur):
        ex = oracle.project(x[ur], xdt, rexp[ur], proj, sdt, g, exact=True, bias_dt=bias_dt)
        mag = oracle.project(x[ur], xdt, rexp[ur], proj, sdt, g, magnitude=True, bias_dt=bias_dt)
        return ex, ((K + 8) * U32_ROUNDOFF + _conversion_rel(xdt, sdt)) * mag
    return _rowwise(fn)


def j_input_backward(grad, gdt, rexp, proj, sdt, g, grad2=None, proj2=None):
    N = grad.shape[1] * (2 if grad2 is not None else 1)

    def fn(ur):
        g2 = None if grad2 is None else grad2[ur]
        ex = oracle.input_backward(grad[ur], gdt, rexp[ur], proj, sdt, g, grad2=g2, proj2=proj2, exact=True)
        mag = oracle.input_backward(grad[ur], gdt, rexp[ur], proj, sdt, g, grad2=g2, proj2=proj2, magnitude=True)
        return ex, ((N + 8) * U32_ROUNDOFF + _conversion_rel(gdt, sdt)) * mag
    return _rowwise(fn)


def j_swiglu(G, U, dt="bf16"):
    def fn(ur):
        ex = oracle.swiglu(G[ur], U[ur], dt, "f64")
        return ex, ELEMWISE_REL * np.abs(ex)
    return _rowwise(fn)


def j_swiglu_backward(dh, G, U, dt="bf16", which=0):
    """dG (which=0) or dU (which=1); the bound scales with the magnitude of
    the formula's terms, |dh| (|U| (1 + |G|) + |G|)."""
    def fn(ur):
        ex = oracle.swiglu_backward(dh[ur], G[ur], U[ur], dt, "f64")[which]
        a, gg, uu = (np.abs(as_f64(t[ur], dt)) for t in (dh, G, U))
        return ex, ELEMWISE_REL * a * (uu * (1.0 + gg) + gg)
    return _rowwise(fn)


def _abs_bits(b):
    return (np.asarray(b) & np.uint16(0x7FFF)).astype(np.uint16)


def j_combine(y, dt, weights, selected, row_of):
    """Rows are tokens (indices into the given weights/selected/row_of)."""
    k = weights.shape[1]

    def fn(ut):
        ex = oracle.combine(y, dt, weights[ut], selected[ut], row_of[ut], "f64")
        mag = oracle.combine(_abs_bits(y), dt, np.abs(weights[ut]), selected[ut], row_of[ut], "f64")
        return ex, (2 * k + 2) * U32_ROUNDOFF * mag
    return _rowwise(fn)


def j_dispatch_backward(dv, dt, selected, row_of):
    k = selected.shape[1]

    def fn(ut):
        ex = oracle.dispatch_backward(dv, dt, selected[ut], row_of[ut], "f64")
        mag = oracle.dispatch_backward(_abs_bits(dv), dt, selected[ut], row_of[ut], "f64")
        return ex, (k + 2) * U32_ROUNDOFF * mag
    return _rowwise(fn)


def j_combine_backward_dy(d_out, dt, weights, row_of, rows_listed):
    """dy rows listed in `rows_listed` (dy[row_of[t, j]] = RNE(w[t, j] dOut[t]):
    one FP32 product, then the storage rounding)."""
    T, k = weights.shape
    tok_of, slot_of = {}, {}
    for t in range(T):
        for j in range(k):
            tok_of[int(row_of[t, j])] = t
            slot_of[int(row_of[t, j])] = j

    def fn(ur):
        ts = np.array([tok_of[int(rows_listed[r])] for r in ur])
        js = np.array([slot_of[int(rows_listed[r])] for r in ur])
        wv = weights[ts, js].astype(np.float64)[:, None]
        ex = wv * as_f64(d_out[ts], dt)  # the product of an FP32 and a 16-bit float is exact in double
        return ex, 2 * U32_ROUNDOFF * np.abs(ex)
    return _rowwise(fn)


def j_chain(j_oracle_inputs, j_device_inputs):
    """End to end: the exact value from the oracle's own upstream chain, with
    the bound of the last step widened by the measured difference between
    the exact values on the device's upstream tensors and on the oracle's
    (upstream flips, each checked in its own step)."""
    def justify(rows, cols):
        ex_o, b_o = j_oracle_inputs(rows, cols)
        ex_d, _ = j_device_inputs(rows, cols)
        return ex_o, b_o + np.abs(ex_d - ex_o)
    return justify


@functools.lru_cache(maxsize=4)
def generated(name: str, **kw):
    w = WORKLOADS[name]
    if kw:
        w = scaled(w, **kw)
    return inputs.generate(w)


def workload_inputs(w):
    return inputs.generate(w)


def gpu_forward(inp, keep_gu=True):
    dev = ffn.to_device(inp)
    buf = ffn.alloc(inp["workload"], keep_gu=keep_gu)
    ffn.forward(dev, buf)
    torch.cuda.synchronize()
    return dev, buf


def gpu_forward_numpy(inp):
    dev, buf = gpu_forward(inp)
    r = buf.route
    res = {"selected": u32(r["selected_experts"]), "weights": r["weights"].cpu().numpy(),
           "offsets": r["offsets"].cpu().numpy(), "row_experts": u32(r["row_experts"]),
           "src_token": r["src_token"].cpu().numpy(), "row_of": r["row_of"].cpu().numpy(),
           "values": bits(r["values"]), "values_dt": dt_name(r["values"].dtype), "G": bits(buf.G), "U": bits(buf.U),
           "h": bits(buf.h), "h_dt": dt_name(buf.h.dtype), "y": bits(buf.y), "out": bits(buf.out),
           "status": int(buf.status.item())}
    return res, dev, buf


def dt_name(dtype) -> str:
    return {torch.bfloat16: "bf16", torch.float16: "f16"}[dtype]


def values_in(dt: str, bf16_rows: np.ndarray) -> np.ndarray:
    """The dispatched rows as the COPY writes them in dtype dt: the BF16 bits
    themselves, or their F16 images (exact in F16's normal range; numpy's
    float16 cast rounds to nearest even)."""
    if dt == "bf16":
        return bf16_rows
    return as_f64(bf16_rows, "bf16").astype(np.float16).view(np.uint16)


def check_forward_steps(inp, res, want, name, rows=None, tokens=None):
    """Each forward step against the oracle on the device's inputs of that
    step (one storage rounding apart), then the end-to-end output against the
    oracle's own chain (flips justified by the upstream differences)."""
    w = inp["workload"]
    if rows is None:
        rows = np.arange(w.A)
    rexp = (res["row_experts"][rows].astype(np.int64) - w.expert_start).astype(np.int32)
    values, vdt = res["values"][rows], res.get("values_dt", "bf16")
    G, U, h = res["G"][rows], res["U"][rows], res["h"][rows]
    sdt, g = w.scale_dtype, w.group
    check_close(G, want["G"], name + "/G", justify=j_project(values, vdt, rexp, inp["gate"], sdt, g))
    check_close(U, want["U"], name + "/U", justify=j_project(values, vdt, rexp, inp["up"], sdt, g))
    hdt = res.get("h_dt", "bf16")  # h in the down projection's operand dtype
    check_close(h, oracle.swiglu(G, U, "bf16", hdt), name + "/h", dt=hdt, justify=j_swiglu(G, U))
    y = oracle.project(h, hdt, rexp, inp["down"], sdt, g, odt="bf16")
    check_close(res["y"][rows], y, name + "/y", justify=j_project(h, hdt, rexp, inp["down"], sdt, g))
    if tokens is None:
        tokens = np.arange(w.T)
        y_orc_rows = want["y"] if want["y"].shape[0] == w.A else None
    else:
        y_orc_rows = None
    sel_t, w_t, ro_t = res["selected"][tokens], res["weights"][tokens], res["row_of"][tokens]
    out = oracle.combine(res["y"], "bf16", w_t, sel_t, ro_t)
    j_dev = j_combine(res["y"], "bf16", w_t, sel_t, ro_t)
    check_close(res["out"][tokens], out, name + "/out", justify=j_dev)
    if "out" in want:
        if y_orc_rows is not None:
            j_orc = j_combine(y_orc_rows, "bf16", want["weights"][tokens], want["selected"][tokens],
                              want["row_of"][tokens])
        else:  # the oracle ran on a sample: its y rows sit at the sample positions
            pos = {int(r): i for i, r in enumerate(want["rows_used"])}
            ro_s = np.array([[pos[int(want["row_of"][t, j])] for j in range(w.top_k)] for t in tokens], np.int32)
            j_orc = j_combine(want["y"], "bf16", want["weights"][tokens], want["selected"][tokens], ro_s)
        check_close(res["out"][tokens], want["out"], name + "/out(end-to-end)", justify=j_chain(j_orc, j_dev))


def check_routing(res, want, name):
    assert np.array_equal(res["selected"], want["selected"]), name + ": selected_experts"
    assert np.max(np.abs(res["weights"].astype(np.float64) - want["weights"])) <= WEIGHT_TOL, name + ": weights"
    for key in ("offsets", "row_experts", "src_token", "row_of"):
        assert np.array_equal(res[key].astype(np.int64), want[key].astype(np.int64)), name + ": " + key


def sample_rows(offsets, n_experts=6, rows_per=8, seed=0):
    """Rows from a few non-empty experts (first, last, largest, random)."""
    rng = np.random.default_rng(seed)
    counts = np.diff(offsets)
    nz = np.nonzero(counts)[0]
    pick = {int(nz[0]), int(nz[-1]), int(nz[np.argmax(counts[nz])])}
    while len(pick) < min(n_experts, len(nz)):
        pick.add(int(rng.choice(nz)))
    rows = []
    for e in sorted(pick):
        a, b = int(offsets[e]), int(offsets[e + 1])
        k = min(rows_per, b - a)
        rows.extend([a, b - 1] + list(rng.choice(np.arange(a, b), size=k, replace=False)))
    return np.array(sorted(set(rows)), np.int64)
