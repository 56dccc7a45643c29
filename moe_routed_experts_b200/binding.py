"""Thin ctypes binding of libmoe_awq.so (include/moe_awq.h).

Argument marshalling only: PyTorch allocates the device tensors and supplies
the current CUDA stream; every step of the operation runs in the library's
CUDA kernels.  There is no other execution path: if the library is missing
or a call fails, an exception is raised.

Unsigned 32-bit outputs (selected_experts, row_experts) are held in int32
tensors carrying the same bit patterns.
"""
import ctypes as C
import os
import re

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe_awq.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "moe_awq.h")

MOE_F32, MOE_F16, MOE_BF16 = 0, 1, 2
STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARGUMENT", 2: "MOE_ERR_UNSUPPORTED_DTYPE", 3: "MOE_ERR_WORKSPACE",
          4: "MOE_ERR_CUDA"}
DEVICE_ERR = {1: "EXPERT_RANGE", 2: "OFFSETS", 4: "ROW_RANGE", 8: "TIMEOUT", 16: "ACT_RANGE"}

_TORCH_DT = {torch.float32: MOE_F32, torch.float16: MOE_F16, torch.bfloat16: MOE_BF16}
_NAME_DT = {"f32": MOE_F32, "f16": MOE_F16, "bf16": MOE_BF16}


class MoeError(RuntimeError):
    def __init__(self, fn, status, msg):
        super().__init__("%s -> %s: %s" % (fn, STATUS.get(status, status), msg))
        self.status = status


_lib = None

P, I64, I32, SZ = C.c_void_p, C.c_int64, C.c_int32, C.c_size_t

_SIGS = {
    "moe_last_error_string": (C.c_char_p, []),
    "moe_version": (C.c_char_p, []),
    "moe_route_dispatch_workspace_size": (SZ, [I64, I64, I32]),
    "moe_route_dispatch": (C.c_int, [P, C.c_int, I64, I64, P, P, I64, I32, I32, I32, P, P, P, P, P, P, P, P, SZ, P, P]),
    "moe_route_dispatch_noalloc": (C.c_int, [P, C.c_int, I64, I64, P, P, I64, I32, I32, I32, P, P, P, P, P, P, P, P,
                                             P]),
    "moe_route": (C.c_int, [P, P, I64, I64, I32, I32, I32, P, P, P, P, P, P, P, SZ, P, P]),
    "awq_grouped_gate_up_swiglu": (C.c_int, [P, C.c_int, I64, I64, I64, P, I64, P, P, P, P, P, P, P, P, C.c_int,
                                             C.c_int, I64, P, P, P, P, SZ, P, P]),
    "awq_grouped_gate_up_swiglu_gather": (C.c_int, [P, C.c_int, I64, P, I64, I64, I64, P, I64, P, P, P, P, P, P, P,
                                                    P, C.c_int, C.c_int, I64, P, P, P, P, SZ, P, P]),
    "awq_projection_workspace_size": (SZ, [I64, I64, I64, I64, I64, I32]),
    "awq_projection_workspace_size_dt": (SZ, [I64, I64, I64, I64, I64, I32, C.c_int, C.c_int]),
    "awq_input_backward_workspace_size": (SZ, [I64, I64, I64, I64, I64, I32, C.c_int, C.c_int]),
    "awq_grouped_down": (C.c_int, [P, C.c_int, I64, I64, I64, P, I64, P, P, P, P, C.c_int, C.c_int, I64, P, P, SZ, P,
                                   P]),
    "moe_combine": (C.c_int, [P, C.c_int, I64, P, P, P, I64, I64, I32, P, P, P]),
    "moe_combine_backward": (C.c_int, [P, P, C.c_int, I64, P, P, I64, I64, I32, P, P, P, P]),
    "awq_input_backward": (C.c_int, [P, C.c_int, I64, I64, I64, P, I64, P, P, P, C.c_int, I64, P, P, P, P, P, P, SZ,
                                     P, P]),
    "moe_swiglu_backward": (C.c_int, [P, P, P, C.c_int, I64, I64, P, P, P]),
    "moe_route_dispatch_dt": (C.c_int, [P, C.c_int, I64, I64, P, P, I64, I32, I32, I32, P, C.c_int, P, P, P, P, P,
                                         P, P, SZ, P, P]),
    "awq_grouped_gate_up_swiglu_dt": (C.c_int, [P, C.c_int, I64, I64, I64, P, I64, P, P, P, P, P, P, P, P, C.c_int,
                                                C.c_int, I64, P, C.c_int, P, P, C.c_int, P, SZ, P, P]),
    "awq_grouped_gate_up_swiglu_gather_dt": (C.c_int, [P, C.c_int, I64, P, I64, I64, I64, P, I64, P, P, P, P, P, P,
                                                       P, P, C.c_int, C.c_int, I64, P, C.c_int, P, P, C.c_int, P, SZ,
                                                       P, P]),
    "awq_grouped_down_dt": (C.c_int, [P, C.c_int, I64, I64, I64, P, I64, P, P, P, P, C.c_int, C.c_int, I64, P,
                                      C.c_int, P, SZ, P, P]),
    "moe_combine_backward_dt": (C.c_int, [P, P, C.c_int, I64, P, P, I64, I64, I32, P, C.c_int, P, P, P]),
    "awq_input_backward_dt": (C.c_int, [P, C.c_int, I64, I64, I64, P, I64, P, P, P, C.c_int, I64, P, P, P, P, P,
                                        C.c_int, P, SZ, P, P]),
    "moe_swiglu_backward_dt": (C.c_int, [P, P, P, C.c_int, I64, I64, P, P, C.c_int, P, P]),
    "moe_dispatch_backward": (C.c_int, [P, C.c_int, I64, P, P, I64, I64, I32, P, P, P]),
    "moe_router_backward": (C.c_int, [P, P, P, I64, I64, I32, I32, I32, P, P, P]),
    "awq_dequant_coefficients": (C.c_int, [P, P, P, C.c_int, I64, I64, I64, I32, P, P]),
    "moe_set_projection_path": (I32, [I32]),
    "nf4_grouped_projection": (C.c_int, [P, C.c_int, I64, I64, I64, P, I64, P, P, P, I64, C.c_int, P, C.c_int, P, P,
                                         P]),
    "nf4_input_backward": (C.c_int, [P, C.c_int, I64, I64, I64, P, I64, P, P, P, I64, C.c_int, P, P, P]),
}


def header_functions():
    """Names of the functions include/moe_awq.h declares."""
    with open(HEADER) as f:
        src = f.read()
    return sorted(set(re.findall(r"^MOE_API\s+[\w\s\*]*?\b(\w+)\s*\(", src, flags=re.M)))


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libmoe_awq.so is not built (run __graft_entry__.build() or "
                               "python moe_routed_experts_b200/build.py); there is no other execution path")
        L = C.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(fn, status):
    if status != 0:
        raise MoeError(fn, status, lib().moe_last_error_string().decode())


def _ptr(t):
    if t is None:
        return None
    assert t.is_cuda and t.is_contiguous(), "tensors passed to the library must be contiguous CUDA tensors"
    return t.data_ptr()


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _dt(x):
    if isinstance(x, str):
        return _NAME_DT[x]
    return _TORCH_DT[x]


def version():
    return lib().moe_version().decode()


def set_projection_path(path: int) -> int:
    prev = lib().moe_set_projection_path(int(path))
    if prev < 0:
        raise ValueError("projection path %d is not available" % path)
    return prev


def new_status(device=None):
    return torch.zeros(1, dtype=torch.int32, device=device or "cuda")


def route_dispatch_workspace_size(T, E, top_k):
    return int(lib().moe_route_dispatch_workspace_size(T, E, top_k))


def moe_route_dispatch(x, logits, top_k, E=None, sel_bias=None, expert_start=0, renormalize=1, workspace=None,
                       device_status=None, out=None, values_dtype=None):
    """Routing, row maps and the expert-sorted rows in values_dtype (default:
    x's dtype; F16 for BF16 x converts while copying; ``out["values"]``'s
    dtype when out is given)."""
    T, H = x.shape
    E = E if E is not None else logits.shape[1]
    A = T * top_k
    dev = x.device
    if out is not None:
        values_dtype = out["values"].dtype
    values_dtype = values_dtype or x.dtype
    if out is None:
        out = {
            "values": torch.empty((A, H), dtype=values_dtype, device=dev),
            "weights": torch.empty((T, top_k), dtype=torch.float32, device=dev),
            "selected_experts": torch.empty((T, top_k), dtype=torch.int32, device=dev),
            "row_experts": torch.empty((A,), dtype=torch.int32, device=dev),
            "offsets": torch.empty((E + 1,), dtype=torch.int32, device=dev),
            "src_token": torch.empty((A,), dtype=torch.int32, device=dev),
            "row_of": torch.empty((T, top_k), dtype=torch.int32, device=dev),
        }
    if workspace is None:
        workspace = torch.empty(max(route_dispatch_workspace_size(T, E, top_k), 256), dtype=torch.uint8, device=dev)
    st = lib().moe_route_dispatch_dt(
        _ptr(x), _dt(x.dtype), T, H, _ptr(logits), _ptr(sel_bias), E, expert_start, top_k, renormalize,
        _ptr(out["values"]), _dt(values_dtype), _ptr(out["weights"]), _ptr(out["selected_experts"]),
        _ptr(out["row_experts"]), _ptr(out["offsets"]), _ptr(out["src_token"]), _ptr(out["row_of"]), _ptr(workspace),
        workspace.numel(), _ptr(device_status), _stream())
    _check("moe_route_dispatch", st)
    return out


def moe_route(logits, top_k, E=None, sel_bias=None, expert_start=0, renormalize=1, workspace=None,
              device_status=None, out=None):
    """Routing and row maps without the COPY (the gather mode of the dispatch)."""
    T = logits.shape[0]
    E = E if E is not None else logits.shape[1]
    A = T * top_k
    dev = logits.device
    if out is None:
        out = {
            "weights": torch.empty((T, top_k), dtype=torch.float32, device=dev),
            "selected_experts": torch.empty((T, top_k), dtype=torch.int32, device=dev),
            "row_experts": torch.empty((A,), dtype=torch.int32, device=dev),
            "offsets": torch.empty((E + 1,), dtype=torch.int32, device=dev),
            "src_token": torch.empty((A,), dtype=torch.int32, device=dev),
            "row_of": torch.empty((T, top_k), dtype=torch.int32, device=dev),
        }
    if workspace is None:
        workspace = torch.empty(max(route_dispatch_workspace_size(T, E, top_k), 256), dtype=torch.uint8, device=dev)
    st = lib().moe_route(
        _ptr(logits), _ptr(sel_bias), T, E, expert_start, top_k, renormalize, _ptr(out["weights"]),
        _ptr(out["selected_experts"]), _ptr(out["row_experts"]), _ptr(out["offsets"]), _ptr(out["src_token"]),
        _ptr(out["row_of"]), _ptr(workspace), workspace.numel(), _ptr(device_status), _stream())
    _check("moe_route", st)
    return out


def moe_route_dispatch_noalloc(x, logits, top_k, out, E=None, sel_bias=None, expert_start=0, renormalize=1,
                               device_status=None):
    """moe_route_dispatch with the library's built-in scratch; `out` holds
    preallocated outputs (same keys as moe_route_dispatch returns)."""
    T, H = x.shape
    E = E if E is not None else logits.shape[1]
    st = lib().moe_route_dispatch_noalloc(
        _ptr(x), _dt(x.dtype), T, H, _ptr(logits), _ptr(sel_bias), E, expert_start, top_k, renormalize,
        _ptr(out["values"]), _ptr(out["weights"]), _ptr(out["selected_experts"]), _ptr(out["row_experts"]),
        _ptr(out["offsets"]), _ptr(out["src_token"]), _ptr(out["row_of"]), _ptr(device_status), _stream())
    _check("moe_route_dispatch_noalloc", st)
    return out


def _bias_dt(*biases):
    for b in biases:
        if b is not None:
            return _dt(b.dtype)
    return MOE_F32


def projection_workspace_size(A, K, N, E, group, nproj, act_dtype=None, scale_dtype=None):
    """Workspace bytes of a projection; with the dtypes (torch dtypes), the
    bytes for exactly those (else enough for any)."""
    if act_dtype is None or scale_dtype is None:
        return int(lib().awq_projection_workspace_size(A, K, N, E, group, nproj))
    return int(lib().awq_projection_workspace_size_dt(A, K, N, E, group, nproj, _dt(act_dtype), _dt(scale_dtype)))


def input_backward_workspace_size(A, N, K, E, group, nproj, grad_dtype, scale_dtype):
    return int(lib().awq_input_backward_workspace_size(A, N, K, E, group, nproj, _dt(grad_dtype), _dt(scale_dtype)))


def _workspace(nbytes, device, workspace=None):
    if nbytes == 0:
        return None
    if workspace is not None and workspace.numel() >= nbytes:
        return workspace
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def awq_grouped_gate_up_swiglu(values, offsets, gate, up, group, want_gu=False, device_status=None, out=None,
                               workspace=None, out_dtype=None, h_dtype=None):
    """G, U in out_dtype (default: values' dtype) and h in h_dtype (default:
    ``out``'s dtype when given, else out_dtype)."""
    A, H = values.shape
    E = offsets.numel() - 1
    I = gate["qweight"].shape[2] * 8
    sdt = _dt(gate["scales"].dtype)
    out_dtype = out_dtype or values.dtype
    h_dtype = out.dtype if out is not None else (h_dtype or out_dtype)
    h = out if out is not None else torch.empty((A, I), dtype=h_dtype, device=values.device)
    G = torch.empty((A, I), dtype=out_dtype, device=values.device) if want_gu else None
    U = torch.empty((A, I), dtype=out_dtype, device=values.device) if want_gu else None
    ws = _workspace(projection_workspace_size(A, H, I, E, group, 2, values.dtype, gate["scales"].dtype), values.device,
                    workspace)
    st = lib().awq_grouped_gate_up_swiglu_dt(
        _ptr(values), _dt(values.dtype), A, H, I, _ptr(offsets), E,
        _ptr(gate["qweight"]), _ptr(gate["qzeros"]), _ptr(gate["scales"]), _ptr(gate.get("bias")),
        _ptr(up["qweight"]), _ptr(up["qzeros"]), _ptr(up["scales"]), _ptr(up.get("bias")),
        sdt, _bias_dt(gate.get("bias"), up.get("bias")), group, _ptr(h), _dt(h_dtype), _ptr(G), _ptr(U), _dt(out_dtype),
        _ptr(ws), 0 if ws is None else ws.numel(), _ptr(device_status), _stream())
    _check("awq_grouped_gate_up_swiglu", st)
    return (h, G, U) if want_gu else h


def awq_grouped_gate_up_swiglu_gather(x, src_token, offsets, gate, up, group, want_gu=False, device_status=None,
                                      out=None, workspace=None, out_dtype=None, h_dtype=None):
    """Gate/up on expert-sorted rows read as x[src_token[r]] (no COPY); dtypes
    as in awq_grouped_gate_up_swiglu (defaults: x's dtype)."""
    T, H = x.shape
    A = src_token.numel()
    E = offsets.numel() - 1
    I = gate["qweight"].shape[2] * 8
    sdt = _dt(gate["scales"].dtype)
    out_dtype = out_dtype or x.dtype
    h_dtype = out.dtype if out is not None else (h_dtype or out_dtype)
    h = out if out is not None else torch.empty((A, I), dtype=h_dtype, device=x.device)
    G = torch.empty((A, I), dtype=out_dtype, device=x.device) if want_gu else None
    U = torch.empty((A, I), dtype=out_dtype, device=x.device) if want_gu else None
    ws = _workspace(projection_workspace_size(A, H, I, E, group, 2, x.dtype, gate["scales"].dtype), x.device, workspace)
    st = lib().awq_grouped_gate_up_swiglu_gather_dt(
        _ptr(x), _dt(x.dtype), T, _ptr(src_token), A, H, I, _ptr(offsets), E,
        _ptr(gate["qweight"]), _ptr(gate["qzeros"]), _ptr(gate["scales"]), _ptr(gate.get("bias")),
        _ptr(up["qweight"]), _ptr(up["qzeros"]), _ptr(up["scales"]), _ptr(up.get("bias")),
        sdt, _bias_dt(gate.get("bias"), up.get("bias")), group, _ptr(h), _dt(h_dtype), _ptr(G), _ptr(U),
        _dt(out_dtype), _ptr(ws), 0 if ws is None else ws.numel(), _ptr(device_status), _stream())
    _check("awq_grouped_gate_up_swiglu_gather", st)
    return (h, G, U) if want_gu else h


def awq_grouped_down(inp, offsets, proj, group, device_status=None, out=None, workspace=None, out_dtype=None):
    """y in out_dtype (default: ``out``'s dtype when given, else the input's)."""
    A, K = inp.shape
    E = offsets.numel() - 1
    N = proj["qweight"].shape[2] * 8
    out_dtype = out.dtype if out is not None else (out_dtype or inp.dtype)
    y = out if out is not None else torch.empty((A, N), dtype=out_dtype, device=inp.device)
    ws = _workspace(projection_workspace_size(A, K, N, E, group, 1, inp.dtype, proj["scales"].dtype), inp.device,
                    workspace)
    st = lib().awq_grouped_down_dt(
        _ptr(inp), _dt(inp.dtype), A, K, N, _ptr(offsets), E, _ptr(proj["qweight"]), _ptr(proj["qzeros"]),
        _ptr(proj["scales"]), _ptr(proj.get("bias")), _dt(proj["scales"].dtype), _bias_dt(proj.get("bias")), group,
        _ptr(y), _dt(out_dtype), _ptr(ws), 0 if ws is None else ws.numel(), _ptr(device_status), _stream())
    _check("awq_grouped_down", st)
    return y


def moe_combine(y, weights, selected_experts, row_of, device_status=None, out=None):
    A, H = y.shape
    T, k = weights.shape
    o = out if out is not None else torch.empty((T, H), dtype=y.dtype, device=y.device)
    st = lib().moe_combine(_ptr(y), _dt(y.dtype), A, _ptr(weights), _ptr(selected_experts), _ptr(row_of), T, H, k,
                           _ptr(o), _ptr(device_status), _stream())
    _check("moe_combine", st)
    return o


def moe_combine_backward(d_out, y, weights, row_of, want_dy=True, want_dw=True, device_status=None, dy_dtype=None):
    """dy in dy_dtype (default: y's dtype) and the FP32 weight VJP."""
    A, H = y.shape
    T, k = weights.shape
    dy_dtype = dy_dtype or y.dtype
    dy = torch.empty((A, H), dtype=dy_dtype, device=y.device) if want_dy else None
    dw = torch.empty((T, k), dtype=torch.float32, device=y.device) if want_dw else None
    st = lib().moe_combine_backward_dt(_ptr(d_out), _ptr(y), _dt(y.dtype), A, _ptr(weights), _ptr(row_of), T, H, k,
                                       _ptr(dy), _dt(dy_dtype), _ptr(dw), _ptr(device_status), _stream())
    _check("moe_combine_backward", st)
    return dy, dw


def awq_input_backward(grad, offsets, proj, group, grad2=None, proj2=None, device_status=None, out=None,
                       workspace=None, out_dtype=None):
    """Input VJP in out_dtype (default: the gradients' dtype; ``out``'s dtype when given)."""
    A, N = grad.shape
    E = offsets.numel() - 1
    K = proj["qweight"].shape[1]
    if out is not None:
        out_dtype = out.dtype
    out_dtype = out_dtype or grad.dtype
    d = out if out is not None else torch.empty((A, K), dtype=out_dtype, device=grad.device)
    p2 = proj2 or {}
    nbytes = input_backward_workspace_size(A, N, K, E, group, 2 if grad2 is not None else 1, grad.dtype,
                                           proj["scales"].dtype)
    ws = _workspace(nbytes, grad.device, workspace)
    st = lib().awq_input_backward_dt(
        _ptr(grad), _dt(grad.dtype), A, N, K, _ptr(offsets), E, _ptr(proj["qweight"]), _ptr(proj["qzeros"]),
        _ptr(proj["scales"]), _dt(proj["scales"].dtype), group, _ptr(grad2), _ptr(p2.get("qweight")),
        _ptr(p2.get("qzeros")), _ptr(p2.get("scales")), _ptr(d), _dt(out_dtype), _ptr(ws),
        0 if ws is None else ws.numel(), _ptr(device_status), _stream())
    _check("awq_input_backward", st)
    return d


def moe_swiglu_backward(dh, G, U, out_dtype=None, device_status=None):
    """dG, dU in out_dtype (default: G's dtype); dh, G and U share one dtype."""
    A, I = G.shape
    out_dtype = out_dtype or G.dtype
    dG = torch.empty((A, I), dtype=out_dtype, device=G.device)
    dU = torch.empty((A, I), dtype=out_dtype, device=G.device)
    st = lib().moe_swiglu_backward_dt(_ptr(dh), _ptr(G), _ptr(U), _dt(G.dtype), A, I, _ptr(dG), _ptr(dU),
                                      _dt(out_dtype), _ptr(device_status), _stream())
    _check("moe_swiglu_backward", st)
    return dG, dU


def moe_dispatch_backward(dvalues, row_of, selected_experts, device_status=None):
    A, H = dvalues.shape
    T, k = row_of.shape
    dx = torch.empty((T, H), dtype=dvalues.dtype, device=dvalues.device)
    st = lib().moe_dispatch_backward(_ptr(dvalues), _dt(dvalues.dtype), A, _ptr(row_of), _ptr(selected_experts), T,
                                     H, k, _ptr(dx), _ptr(device_status), _stream())
    _check("moe_dispatch_backward", st)
    return dx


def moe_router_backward(logits, selected_experts, d_weights, renormalize=1, expert_start=0, device_status=None):
    T, E = logits.shape
    k = selected_experts.shape[1]
    dl = torch.empty((T, E), dtype=torch.float32, device=logits.device)
    st = lib().moe_router_backward(_ptr(logits), _ptr(selected_experts), _ptr(d_weights), T, E, k, int(renormalize),
                                   int(expert_start), _ptr(dl), _ptr(device_status), _stream())
    _check("moe_router_backward", st)
    return dl


def awq_dequant_coefficients(qweight, qzeros, scales, group, pairing=0):
    K, NW = qweight.shape
    N = NW * 8
    out = torch.empty((K, N), dtype=torch.int16, device=qweight.device)
    st = lib().awq_dequant_coefficients(_ptr(qweight), _ptr(qzeros), _ptr(scales), _dt(scales.dtype), K, N, group,
                                        pairing, _ptr(out), _stream())
    _check("awq_dequant_coefficients", st)
    return out


def nf4_payload_to_device(payload: dict, device="cuda") -> dict:
    """NF4 payload (codes uint8 [E, K*N/2], absmax f32, codebook f32 [16]) -> device tensors."""
    d = {"codes": torch.from_numpy(payload["codes"]).to(device), "absmax": torch.from_numpy(payload["absmax"]).to(device),
         "codebook": torch.from_numpy(payload["codebook"]).to(device), "block": int(payload["block"]),
         "N": int(payload["N"]), "bias": None}
    if payload.get("bias") is not None:
        d["bias"] = torch.from_numpy(payload["bias"]).to(device)
    return d


def nf4_grouped_projection(inp, offsets, payload, coef_dtype="bf16", device_status=None, out=None):
    A, K = inp.shape
    E = offsets.numel() - 1
    N = payload["N"]
    y = out if out is not None else torch.empty((A, N), dtype=inp.dtype, device=inp.device)
    st = lib().nf4_grouped_projection(
        _ptr(inp), _dt(inp.dtype), A, K, N, _ptr(offsets), E, _ptr(payload["codes"]), _ptr(payload["absmax"]),
        _ptr(payload["codebook"]), payload["block"], _NAME_DT[coef_dtype], _ptr(payload.get("bias")),
        _bias_dt(payload.get("bias")), _ptr(y), _ptr(device_status), _stream())
    _check("nf4_grouped_projection", st)
    return y


def nf4_input_backward(grad, offsets, payload, K, coef_dtype="bf16", device_status=None, out=None):
    A, N = grad.shape
    E = offsets.numel() - 1
    d = out if out is not None else torch.empty((A, K), dtype=grad.dtype, device=grad.device)
    st = lib().nf4_input_backward(
        _ptr(grad), _dt(grad.dtype), A, N, K, _ptr(offsets), E, _ptr(payload["codes"]), _ptr(payload["absmax"]),
        _ptr(payload["codebook"]), payload["block"], _NAME_DT[coef_dtype], _ptr(d), _ptr(device_status), _stream())
    _check("nf4_input_backward", st)
    return d
