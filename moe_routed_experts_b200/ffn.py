"""The routed-experts FFN as a sequence of C-ABI calls.

``forward`` = moe_route_dispatch -> awq_grouped_gate_up_swiglu ->
awq_grouped_down -> moe_combine; ``backward`` = moe_combine_backward ->
awq_input_backward(down) -> moe_swiglu_backward -> awq_input_backward(gate
+ up, one accumulation) -> moe_dispatch_backward, and moe_router_backward
for the router logits.  The ``_dt`` forms of the dispatch, the projections
and the first three backward steps write the tensors that only feed a
tensor-core product (values, h, dy, dG, dU) in the scale dtype.  Only
argument marshalling happens here; every step runs in the library's
kernels.
"""
from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch

from . import binding as B

_SDT = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}


def _t16(a: np.ndarray, dt: torch.dtype, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(dt).to(device)


def projection_to_device(proj: dict, scale_dtype: str, device="cuda") -> dict:
    out = {"qweight": torch.from_numpy(np.ascontiguousarray(proj["qweight"])).to(device),
           "qzeros": torch.from_numpy(np.ascontiguousarray(proj["qzeros"])).to(device)}
    if scale_dtype == "f32":
        out["scales"] = torch.from_numpy(np.ascontiguousarray(proj["scales"], np.float32)).to(device)
    else:
        out["scales"] = _t16(proj["scales"], _SDT[scale_dtype], device)
    out["bias"] = None if proj.get("bias") is None else torch.from_numpy(proj["bias"]).to(device)
    return out


def to_device(inp: dict, device="cuda") -> dict:
    """Generated NumPy inputs (moe_routed_experts_b200.inputs) -> device tensors."""
    w = inp["workload"]
    d = {"workload": w,
         "x": _t16(inp["x"], torch.bfloat16, device),
         "logits": torch.from_numpy(inp["logits"]).to(device),
         "sel_bias": None if inp["sel_bias"] is None else torch.from_numpy(inp["sel_bias"]).to(device)}
    for name in ("gate", "up", "down"):
        d[name] = projection_to_device(inp[name], w.scale_dtype, device)
    d["d_out"] = None if inp.get("d_out") is None else _t16(inp["d_out"], torch.bfloat16, device)
    return d


@dataclass
class Buffers:
    """Preallocated device outputs and scratch for one workload."""
    route: dict
    workspace: torch.Tensor
    h: torch.Tensor
    G: Optional[torch.Tensor]
    U: Optional[torch.Tensor]
    y: torch.Tensor
    out: torch.Tensor
    status: torch.Tensor
    proj_ws: Optional[torch.Tensor] = None


def alloc(w, device="cuda", keep_gu: bool = False) -> Buffers:
    T, H, I, E, k = w.T, w.H, w.I, w.E, w.top_k
    A = T * k
    vdt = _SDT[operand_dtype(w.scale_dtype)]  # values and h: the projections' operand dtype
    route = {
        "values": torch.empty((A, H), dtype=vdt, device=device),
        "weights": torch.empty((T, k), dtype=torch.float32, device=device),
        "selected_experts": torch.empty((T, k), dtype=torch.int32, device=device),
        "row_experts": torch.empty((A,), dtype=torch.int32, device=device),
        "offsets": torch.empty((E + 1,), dtype=torch.int32, device=device),
        "src_token": torch.empty((A,), dtype=torch.int32, device=device),
        "row_of": torch.empty((T, k), dtype=torch.int32, device=device),
    }
    ws = torch.empty(max(B.route_dispatch_workspace_size(T, E, k), 256), dtype=torch.uint8, device=device)
    h = torch.empty((A, I), dtype=vdt, device=device)
    G = torch.empty((A, I), dtype=torch.bfloat16, device=device) if keep_gu else None
    U = torch.empty((A, I), dtype=torch.bfloat16, device=device) if keep_gu else None
    y = torch.empty((A, H), dtype=torch.bfloat16, device=device)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=device)
    sdt = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}[w.scale_dtype]
    pws = max(B.projection_workspace_size(A, H, I, E, w.group, 2, vdt, sdt),
              B.projection_workspace_size(A, H, I, E, w.group, 2, torch.bfloat16, sdt),  # gather mode reads x
              B.projection_workspace_size(A, I, H, E, w.group, 1, vdt, sdt))
    proj_ws = torch.empty(pws, dtype=torch.uint8, device=device) if pws else None
    return Buffers(route, ws, h, G, U, y, out, torch.zeros(1, dtype=torch.int32, device=device), proj_ws)


def forward(dev: dict, buf: Buffers, gather: bool = False) -> torch.Tensor:
    """One forward pass of the whole hot path into ``buf``; returns buf.out.
    gather: route without the COPY and let the gate/up projection read each
    row from x through src_token (buf.route["values"] is then not written)."""
    w = dev["workload"]
    if gather:
        r = B.moe_route(dev["logits"], w.top_k, E=w.E, sel_bias=dev["sel_bias"], expert_start=w.expert_start,
                        renormalize=w.renormalize, workspace=buf.workspace, device_status=buf.status, out=buf.route)
    else:
        r = B.moe_route_dispatch(dev["x"], dev["logits"], w.top_k, E=w.E, sel_bias=dev["sel_bias"],
                                 expert_start=w.expert_start, renormalize=w.renormalize, workspace=buf.workspace,
                                 device_status=buf.status, out=buf.route)
    lib, st = B.lib(), B._stream()
    gate, up, down = dev["gate"], dev["up"], dev["down"]
    A = w.A
    # values and h in the operand dtype (F16 with F16 scales); G, U, y and out in BF16
    pay = (B._ptr(gate["qweight"]), B._ptr(gate["qzeros"]), B._ptr(gate["scales"]), B._ptr(gate["bias"]),
           B._ptr(up["qweight"]), B._ptr(up["qzeros"]), B._ptr(up["scales"]), B._ptr(up["bias"]),
           B._dt(gate["scales"].dtype), B.MOE_F32, w.group, B._ptr(buf.h), B._dt(buf.h.dtype), B._ptr(buf.G),
           B._ptr(buf.U), B.MOE_BF16)
    tail = (B._ptr(buf.proj_ws), 0 if buf.proj_ws is None else buf.proj_ws.numel(), B._ptr(buf.status), st)
    if gather:
        s = lib.awq_grouped_gate_up_swiglu_gather_dt(B._ptr(dev["x"]), B.MOE_BF16, w.T, B._ptr(r["src_token"]), A,
                                                     w.H, w.I, B._ptr(r["offsets"]), w.E, *pay, *tail)
        B._check("awq_grouped_gate_up_swiglu_gather", s)
    else:
        s = lib.awq_grouped_gate_up_swiglu_dt(B._ptr(r["values"]), B._dt(r["values"].dtype), A, w.H, w.I,
                                              B._ptr(r["offsets"]), w.E, *pay, *tail)
        B._check("awq_grouped_gate_up_swiglu", s)
    s = lib.awq_grouped_down_dt(
        B._ptr(buf.h), B._dt(buf.h.dtype), A, w.I, w.H, B._ptr(r["offsets"]), w.E, B._ptr(down["qweight"]),
        B._ptr(down["qzeros"]), B._ptr(down["scales"]), B._ptr(down["bias"]), B._dt(down["scales"].dtype),
        B.MOE_F32, w.group, B._ptr(buf.y), B.MOE_BF16, B._ptr(buf.proj_ws),
        0 if buf.proj_ws is None else buf.proj_ws.numel(), B._ptr(buf.status), st)
    B._check("awq_grouped_down", s)
    s = lib.moe_combine(B._ptr(buf.y), B.MOE_BF16, A, B._ptr(r["weights"]), B._ptr(r["selected_experts"]),
                        B._ptr(r["row_of"]), w.T, w.H, w.top_k, B._ptr(buf.out), B._ptr(buf.status), st)
    B._check("moe_combine", s)
    return buf.out


def operand_dtype(scale_dtype: str, act_dtype: str = "bf16") -> str:
    """dtype of the tensors that only feed a projection's tensor-core
    product: the dispatched rows (values), h, and the gradients of the input
    VJPs (dy, dG, dU).

    The products run in the scale dtype, so with F16 scales the step before
    writes F16 directly (the COPY converts while copying; the other steps
    round their FP32 values once) instead of the activation dtype plus a
    conversion pass; G, U, y, out and the activation gradients (dh,
    dvalues, dx) stay in act_dtype."""
    return "f16" if scale_dtype == "f16" else act_dtype


def backward(dev: dict, buf: Buffers, d_out: torch.Tensor) -> dict:
    """Input VJP of the forward held in ``buf`` (needs G and U kept)."""
    w = dev["workload"]
    r = buf.route
    assert buf.G is not None and buf.U is not None, "allocate with keep_gu=True"
    act = buf.y.dtype
    gdt = _SDT[operand_dtype(w.scale_dtype, "bf16" if act == torch.bfloat16 else "f16")]
    dy, dw = B.moe_combine_backward(d_out, buf.y, r["weights"], r["row_of"], device_status=buf.status, dy_dtype=gdt)
    dh = B.awq_input_backward(dy, r["offsets"], dev["down"], w.group, device_status=buf.status, out_dtype=act)
    dG, dU = B.moe_swiglu_backward(dh, buf.G, buf.U, out_dtype=gdt, device_status=buf.status)
    dvalues = B.awq_input_backward(dG, r["offsets"], dev["gate"], w.group, grad2=dU, proj2=dev["up"],
                                   device_status=buf.status, out_dtype=act)
    dx = B.moe_dispatch_backward(dvalues, r["row_of"], r["selected_experts"], device_status=buf.status)
    dlogits = B.moe_router_backward(dev["logits"], r["selected_experts"], dw, renormalize=w.renormalize,
                                    expert_start=w.expert_start, device_status=buf.status)
    return {"dy": dy, "dweights": dw, "dh": dh, "dG": dG, "dU": dU, "dvalues": dvalues, "dx": dx,
            "dlogits": dlogits}
