"""Shared helpers of the GPU parity tests: device runs through the C ABI,
oracle runs on the same seeded inputs, and the tolerance checks.

Tolerance (floating outputs and gradients): |got - oracle| <= 2e-2 *
rms(oracle) per tensor, widened at each element by one unit in the last
place of the storage dtype at the oracle's value.  The widening covers the
one case the rms bound cannot: the device accumulates in FP32 and the oracle
in double, so when the exact result lies within the FP32 error of a BF16
rounding boundary the two stored values are adjacent BF16 numbers, and with
8 significant bits one such step at |v| > ~2.6 rms already exceeds 2e-2 rms.
The share of elements that need the widening is reported and bounded.
Integer and index outputs, and the rounded coefficients, must match bit for
bit; FP32 routing weights within 2e-6.
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


def ulp(v: np.ndarray, dt: str) -> np.ndarray:
    """Spacing of the storage format at |v| (normal range; subnormal floor)."""
    mant, emin = (7, -126) if dt == "bf16" else (10, -14)
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, emin)
    return np.ldexp(1.0, (e - mant).astype(np.int64))


def check_close(got, want, name, dt="bf16", tol=TOL, max_widened=2e-3, ulps=1):
    g, w = as_f64(got, dt), as_f64(want, dt)
    assert g.shape == w.shape, (name, g.shape, w.shape)
    assert np.all(np.isfinite(g)), name + ": non-finite values"
    if not w.size:
        return 0.0
    rms = float(np.sqrt(np.mean(w * w)))
    err = np.abs(g - w)
    strict = tol * rms
    bound = strict + ulps * ulp(w, dt)
    worst = int(np.argmax(err - bound))
    assert np.all(err <= bound), "%s: err %.4g at value %.4g > %.3g * rms %.4g + 1 ulp" % (
        name, err.reshape(-1)[worst], w.reshape(-1)[worst], tol, rms)
    widened = float(np.mean(err > strict))
    assert widened <= max_widened, "%s: %.2e of elements beyond %.3g * rms" % (name, widened, tol)
    return float(err.max()) / max(rms, 1e-30)


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
           "values": bits(r["values"]), "G": bits(buf.G), "U": bits(buf.U), "h": bits(buf.h), "y": bits(buf.y),
           "out": bits(buf.out), "status": int(buf.status.item())}
    return res, dev, buf


def check_forward_steps(inp, res, want, name, rows=None, tokens=None):
    """Each forward step against the oracle on the device's inputs of that
    step (one storage rounding apart), then the end-to-end output against the
    oracle's own chain (two roundings may compound: two-ulp slack)."""
    w = inp["workload"]
    if rows is None:
        rows = np.arange(w.A)
    rexp = (res["row_experts"][rows].astype(np.int64) - w.expert_start).astype(np.int32)
    G, U, h = res["G"][rows], res["U"][rows], res["h"][rows]
    check_close(G, want["G"], name + "/G")
    check_close(U, want["U"], name + "/U")
    check_close(h, oracle.swiglu(G, U, "bf16"), name + "/h")
    y = oracle.project(h, "bf16", rexp, inp["down"], w.scale_dtype, w.group)
    check_close(res["y"][rows], y, name + "/y")
    if tokens is None:
        out = oracle.combine(res["y"], "bf16", res["weights"], res["selected"], res["row_of"])
        check_close(res["out"], out, name + "/out")
        check_close(res["out"], want["out"], name + "/out(end-to-end)", ulps=2)
    else:
        sel_t, w_t = res["selected"][tokens], res["weights"][tokens]
        out = oracle.combine(res["y"], "bf16", w_t, sel_t, res["row_of"][tokens])
        check_close(res["out"][tokens], out, name + "/out")
        check_close(res["out"][tokens], want["out"], name + "/out(end-to-end)", ulps=2)


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
