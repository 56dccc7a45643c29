"""CPU oracle of the frozen AWQ routed-experts FFN (ctypes over moe_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
bench's CPU-baseline leg, never by the product path.  It shares no code with
the CUDA library; see moe_oracle.c for what each step computes and which
statement of the method it follows.

Arrays are NumPy; 16-bit floats are passed as uint16 bit patterns.
"""
import ctypes as C
import os

import numpy as np

from .build import build as _build_library

DT = {"f32": 0, "f16": 1, "bf16": 2, "f64": 3}

_lib = None


def lib():
    global _lib
    if _lib is None:
        # ORACLE_LIB: a planted-mistake build for the mutant test (tests only)
        path = os.environ.get("ORACLE_LIB") or _build_library()
        _lib = C.CDLL(path)
        _declare(_lib)
    return _lib


P = C.c_void_p
I64 = C.c_int64
I32 = C.c_int32
U32 = C.c_uint32


def _declare(L):
    L.oracle_round.restype = C.c_double
    L.oracle_round.argtypes = [C.c_double, C.c_int]
    L.oracle_encode.restype = U32
    L.oracle_encode.argtypes = [C.c_double, C.c_int]
    L.oracle_decode.restype = C.c_double
    L.oracle_decode.argtypes = [U32, C.c_int]
    L.oracle_unpack_word.argtypes = [U32, P]
    L.oracle_pack_word.restype = U32
    L.oracle_pack_word.argtypes = [P]
    L.oracle_coefficient.restype = C.c_double
    L.oracle_coefficient.argtypes = [I32, I32, U32, C.c_int, P]
    L.oracle_dequant.argtypes = [P, P, P, C.c_int, I64, I64, I64, P, P]
    L.oracle_route.restype = C.c_int
    L.oracle_route.argtypes = [P, P, I64, I64, I32, I32, U32, P, P]
    L.oracle_dispatch.restype = C.c_int
    L.oracle_dispatch.argtypes = [P, I64, I32, I64, U32, P, P, P, P]
    L.oracle_copy_rows.argtypes = [P, I64, I64, P, I64, P]
    L.oracle_project.restype = C.c_int
    L.oracle_project.argtypes = [P, C.c_int, I64, I64, I64, P, I64, P, P, P, C.c_int, P, C.c_int,
                                 I64, C.c_int, P, C.c_int]
    L.oracle_swiglu.argtypes = [P, P, C.c_int, I64, P, C.c_int]
    L.oracle_combine.argtypes = [P, C.c_int, P, P, P, I64, I64, I32, P, C.c_int]
    L.oracle_combine_backward.argtypes = [P, P, C.c_int, P, P, I64, I64, I32, P, P, C.c_int]
    L.oracle_input_backward.restype = C.c_int
    L.oracle_input_backward.argtypes = [P, C.c_int, I64, I64, I64, P, I64, P, P, P, C.c_int, I64,
                                        P, P, P, P, C.c_int, P, C.c_int]
    L.oracle_swiglu_backward.argtypes = [P, P, P, C.c_int, I64, P, P, C.c_int]
    L.oracle_dispatch_backward.argtypes = [P, C.c_int, P, P, I64, I64, I32, P, C.c_int]
    L.oracle_router_backward.argtypes = [P, P, P, I64, I64, I32, I32, U32, P]
    L.oracle_num_threads.restype = C.c_int
    L.oracle_nf4_code.restype = I32
    L.oracle_nf4_code.argtypes = [P, I64]
    L.oracle_nf4_dequant.argtypes = [P, P, P, I64, I64, I64, C.c_int, P, P]
    L.oracle_nf4_project.restype = C.c_int
    L.oracle_nf4_project.argtypes = [P, C.c_int, I64, I64, I64, P, I64, P, P, P, I64, C.c_int, P, C.c_int, C.c_int,
                                     P, C.c_int]
    L.oracle_nf4_input_backward.restype = C.c_int
    L.oracle_nf4_input_backward.argtypes = [P, C.c_int, I64, I64, I64, P, I64, P, P, P, I64, C.c_int, C.c_int, P,
                                            C.c_int]


def _p(a):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(C.c_void_p)


def _c(a, dtype=None):
    if a is None:
        return None
    return np.ascontiguousarray(a, dtype=dtype) if dtype is not None else np.ascontiguousarray(a)


def _sdt_array(a, dt):
    return _c(a, np.float32 if dt == "f32" else np.uint16)


def _out_dtype(dt):
    """NumPy storage of a tensor of oracle dtype dt (16-bit formats as bits)."""
    return {"f32": np.float32, "f64": np.float64}.get(dt, np.uint16)


def num_threads() -> int:
    return int(lib().oracle_num_threads())


# ---------------------------------------------------------------- scalars

def round_to(v: float, dt: str) -> float:
    return float(lib().oracle_round(float(v), DT[dt]))


def encode(v: float, dt: str) -> int:
    return int(lib().oracle_encode(float(v), DT[dt]))


def decode(bits: int, dt: str) -> float:
    return float(lib().oracle_decode(int(bits), DT[dt]))


def decode_array(a: np.ndarray, dt: str) -> np.ndarray:
    """Storage array -> float64 values (through the oracle's own decoder)."""
    a = np.asarray(a)
    if dt == "f32":
        return a.astype(np.float64)
    f = np.vectorize(lambda b: lib().oracle_decode(int(b), DT[dt]), otypes=[np.float64])
    return f(a) if a.size else a.astype(np.float64)


def unpack_word(word: int) -> np.ndarray:
    codes = np.zeros(8, np.int32)
    lib().oracle_unpack_word(int(word) & 0xFFFFFFFF, _p(codes))
    return codes


def pack_word(codes) -> int:
    c = _c(codes, np.int32)
    assert c.shape == (8,)
    return int(lib().oracle_pack_word(_p(c)))


def coefficient(q: int, z: int, scale_bits: int, sdt: str):
    bits = np.zeros(1, np.uint32)
    v = lib().oracle_coefficient(int(q), int(z), int(scale_bits), DT[sdt], _p(bits))
    return float(v), int(bits[0])


def dequant(qw, qz, sc, sdt: str, K: int, N: int, g: int):
    """One expert's coefficients: (W float64 [K,N], bits uint32 [K,N])."""
    if g < 1 or K % g or N % 8:
        raise ValueError("dequant: incomplete group or N % 8 != 0")
    qw, qz, sc = _c(qw, np.int32), _c(qz, np.int32), _sdt_array(sc, sdt)
    W = np.zeros((K, N), np.float64)
    Wb = np.zeros((K, N), np.uint32)
    lib().oracle_dequant(_p(qw), _p(qz), _p(sc), DT[sdt], K, N, g, _p(W), _p(Wb))
    return W, Wb


# ---------------------------------------------------------------- routing

def route(logits, sel_bias, k: int, renormalize: int = 1, expert_start: int = 0):
    logits = _c(logits, np.float32)
    T, E = logits.shape
    sb = _c(sel_bias, np.float32)
    sel = np.zeros((T, k), np.uint32)
    w = np.zeros((T, k), np.float32)
    rc = lib().oracle_route(_p(logits), _p(sb), T, E, k, renormalize, expert_start, _p(sel), _p(w))
    if rc != 0:
        raise ValueError("oracle_route: invalid arguments")
    return sel, w


def dispatch(selected, E: int, expert_start: int = 0):
    selected = _c(selected, np.uint32)
    T, k = selected.shape
    A = T * k
    offsets = np.zeros(E + 1, np.int32)
    row_experts = np.zeros(A, np.uint32)
    src_token = np.zeros(A, np.int32)
    row_of = np.zeros((T, k), np.int32)
    rc = lib().oracle_dispatch(_p(selected), T, k, E, expert_start, _p(offsets), _p(row_experts),
                               _p(src_token), _p(row_of))
    if rc != 0:
        raise ValueError("oracle_dispatch: expert ID out of range")
    return offsets, row_experts, src_token, row_of


def copy_rows(x, src_token):
    x = _c(x)
    src = _c(src_token, np.int32)
    T, H = x.shape
    out = np.zeros((src.shape[0], H), x.dtype)
    lib().oracle_copy_rows(_p(x), H, x.dtype.itemsize, _p(src), src.shape[0], _p(out))
    return out


# ---------------------------------------------------------------- projections

def project(x, xdt: str, row_expert, proj: dict, sdt: str, g: int, exact: bool = False,
            odt: str = None, bias_dt: str = "f32", magnitude: bool = False):
    """Rows of x through their experts' projection (see oracle_project).
    exact: the unrounded double sums; magnitude: the double sums of the
    products' magnitudes (|x W|, plus |bias|)."""
    x = _c(x)
    R, K = x.shape
    qw = _c(proj["qweight"], np.int32)
    E, K2, NW = qw.shape
    assert K2 == K
    N = NW * 8
    qz = _c(proj["qzeros"], np.int32)
    sc = _sdt_array(proj["scales"], sdt)
    bias = proj.get("bias")
    if bias is not None:
        bias = _c(bias, np.float32 if bias_dt == "f32" else np.uint16)
    re = _c(row_expert, np.int32)
    odt = odt or xdt
    mode = 2 if magnitude else 1 if exact else 0
    out = np.zeros((R, N), np.float64 if mode else _out_dtype(odt))
    rc = lib().oracle_project(_p(x), DT[xdt], R, K, N, _p(re), E, _p(qw), _p(qz), _p(sc), DT[sdt],
                              _p(bias), DT[bias_dt], g, mode, _p(out), DT[odt])
    if rc != 0:
        raise ValueError("oracle_project: " + ("incomplete group or N % 8 != 0" if rc == -2 else "expert index out of range"))
    return out


def swiglu(G, U, dt: str = "bf16", odt: str = None):
    """h from stored G and U (dtype dt); odt "f64" gives the unrounded h."""
    G, U = _c(G), _c(U)
    odt = odt or dt
    h = np.zeros(G.shape, _out_dtype(odt))
    lib().oracle_swiglu(_p(G), _p(U), DT[dt], G.size, _p(h), DT[odt])
    return h


def combine(y, dt: str, weights, selected, row_of, odt: str = None):
    """Per-token ascending-ID combine; odt "f64" gives the unrounded sums."""
    y = _c(y)
    w, sel, ro = _c(weights, np.float32), _c(selected, np.uint32), _c(row_of, np.int32)
    T, k = w.shape
    H = y.shape[1]
    odt = odt or dt
    out = np.zeros((T, H), _out_dtype(odt))
    lib().oracle_combine(_p(y), DT[dt], _p(w), _p(sel), _p(ro), T, H, k, _p(out), DT[odt])
    return out


def combine_backward(d_out, y, dt: str, weights, row_of, want_dy=True, want_dw=True, dy_dt: str = None):
    d_out, y = _c(d_out), _c(y)
    w, ro = _c(weights, np.float32), _c(row_of, np.int32)
    T, k = w.shape
    H = y.shape[1]
    dy_dt = dy_dt or dt
    dy = np.zeros(y.shape, _out_dtype(dy_dt)) if want_dy else None
    dw = np.zeros((T, k), np.float32) if want_dw else None
    lib().oracle_combine_backward(_p(d_out), _p(y), DT[dt], _p(w), _p(ro), T, H, k, _p(dy), _p(dw), DT[dy_dt])
    return dy, dw


def input_backward(grad, gdt: str, row_expert, proj: dict, sdt: str, g: int, grad2=None, proj2=None,
                   exact: bool = False, odt: str = None, magnitude: bool = False):
    grad = _c(grad)
    R, N = grad.shape
    qw = _c(proj["qweight"], np.int32)
    E, K, NW = qw.shape
    assert NW * 8 == N
    qz = _c(proj["qzeros"], np.int32)
    sc = _sdt_array(proj["scales"], sdt)
    g2 = qw2 = qz2 = sc2 = None
    if grad2 is not None:
        g2 = _c(grad2)
        qw2 = _c(proj2["qweight"], np.int32)
        qz2 = _c(proj2["qzeros"], np.int32)
        sc2 = _sdt_array(proj2["scales"], sdt)
    re = _c(row_expert, np.int32)
    odt = odt or gdt
    mode = 2 if magnitude else 1 if exact else 0
    out = np.zeros((R, K), np.float64 if mode else _out_dtype(odt))
    rc = lib().oracle_input_backward(_p(grad), DT[gdt], R, N, K, _p(re), E, _p(qw), _p(qz), _p(sc), DT[sdt], g,
                                     _p(g2), _p(qw2), _p(qz2), _p(sc2), mode, _p(out), DT[odt])
    if rc != 0:
        raise ValueError("oracle_input_backward: " + ("incomplete group or N % 8 != 0" if rc == -2 else "expert index out of range"))
    return out


def swiglu_backward(dh, G, U, dt: str = "bf16", odt: str = None):
    dh, G, U = _c(dh), _c(G), _c(U)
    odt = odt or dt
    dG, dU = np.zeros(G.shape, _out_dtype(odt)), np.zeros(U.shape, _out_dtype(odt))
    lib().oracle_swiglu_backward(_p(dh), _p(G), _p(U), DT[dt], G.size, _p(dG), _p(dU), DT[odt])
    return dG, dU


def dispatch_backward(dvalues, dt: str, selected, row_of, odt: str = None):
    dv = _c(dvalues)
    sel, ro = _c(selected, np.uint32), _c(row_of, np.int32)
    T, k = sel.shape
    H = dv.shape[1]
    odt = odt or dt
    dx = np.zeros((T, H), _out_dtype(odt))
    lib().oracle_dispatch_backward(_p(dv), DT[dt], _p(sel), _p(ro), T, H, k, _p(dx), DT[odt])
    return dx


def router_backward(logits, selected, d_weights, renormalize: int = 1, expert_start: int = 0):
    logits = _c(logits, np.float32)
    T, E = logits.shape
    sel, dw = _c(selected, np.uint32), _c(d_weights, np.float32)
    k = sel.shape[1]
    dl = np.zeros((T, E), np.float32)
    lib().oracle_router_backward(_p(logits), _p(sel), _p(dw), T, E, k, renormalize, expert_start, _p(dl))
    return dl


# ---------------------------------------------------------------- whole chain

def forward(inp: dict, rows=None, tokens=None):
    """Storage-rounded forward of a generated workload.

    Routing and dispatch always cover every token (they fix the row order).
    ``rows`` (indices into the A dispatched rows) restricts the projections to
    a sample; ``tokens`` restricts the combine (their rows are added to the
    sample automatically).  Returns a dict; sampled tensors are indexed by the
    sample order given in ``rows_used`` / ``tokens_used``.
    """
    w = inp["workload"]
    sdt, g = w.scale_dtype, w.group
    sel, wts = route(inp["logits"], inp["sel_bias"], w.top_k, w.renormalize, w.expert_start)
    offsets, row_experts, src_token, row_of = dispatch(sel, w.E, w.expert_start)
    A = w.A
    if tokens is not None:
        tokens = np.asarray(tokens, np.int64)
        need = set(int(r) for r in row_of[tokens].reshape(-1))
        if rows is not None:
            need |= set(int(r) for r in rows)
        rows = np.array(sorted(need), np.int64)
    if rows is None:
        rows = np.arange(A, dtype=np.int64)
    rows = np.asarray(rows, np.int64)
    values = copy_rows(inp["x"], src_token[rows])
    rexp = (row_experts[rows].astype(np.int64) - w.expert_start).astype(np.int32)
    G = project(values, "bf16", rexp, inp["gate"], sdt, g)
    U = project(values, "bf16", rexp, inp["up"], sdt, g)
    h = swiglu(G, U, "bf16")
    y = project(h, "bf16", rexp, inp["down"], sdt, g)
    res = {"selected": sel, "weights": wts, "offsets": offsets, "row_experts": row_experts,
           "src_token": src_token, "row_of": row_of, "rows_used": rows, "values": values,
           "G": G, "U": U, "h": h, "y": y}
    if tokens is not None:
        pos = {int(r): i for i, r in enumerate(rows)}
        T, k = row_of.shape
        H = w.H
        y_full_idx = np.array([[pos[int(row_of[t, j])] for j in range(k)] for t in tokens], np.int32)
        out = combine(y, "bf16", wts[tokens], sel[tokens], y_full_idx)
        res["tokens_used"] = tokens
        res["out"] = out
    elif rows.shape[0] == A:
        res["out"] = combine(y, "bf16", wts, sel, row_of)
    return res


# ---------------------------------------------------------------- NF4 payloads

def nf4_code(codes, f: int) -> int:
    codes = _c(codes, np.uint8)
    return int(lib().oracle_nf4_code(_p(codes), int(f)))


def nf4_dequant(codes, absmax, codebook, K: int, N: int, B: int, cdt: str):
    """One expert's NF4 coefficients: (W float64 [K,N], bits uint32 [K,N])."""
    codes, absmax, cb = _c(codes, np.uint8), _c(absmax, np.float32), _c(codebook, np.float32)
    W = np.zeros((K, N), np.float64)
    Wb = np.zeros((K, N), np.uint32)
    lib().oracle_nf4_dequant(_p(codes), _p(absmax), _p(cb), K, N, B, DT[cdt], _p(W), _p(Wb))
    return W, Wb


def nf4_project(x, xdt: str, row_expert, payload: dict, cdt: str, exact: bool = False, odt: str = None,
                bias_dt: str = "f32", magnitude: bool = False):
    """Rows of x through their experts' NF4 projection (see oracle_nf4_project).
    payload: codes uint8 [E, K*N/2], absmax f32 [E, K*N/B], codebook f32 [16],
    block B, N; optional bias [E, N]."""
    x = _c(x)
    R, K = x.shape
    N, B = payload["N"], payload["block"]
    codes, absmax = _c(payload["codes"], np.uint8), _c(payload["absmax"], np.float32)
    cb = _c(payload["codebook"], np.float32)
    E = codes.shape[0]
    bias = payload.get("bias")
    if bias is not None:
        bias = _c(bias, np.float32 if bias_dt == "f32" else np.uint16)
    re = _c(row_expert, np.int32)
    odt = odt or xdt
    mode = 2 if magnitude else 1 if exact else 0
    out = np.zeros((R, N), np.float64 if mode else _out_dtype(odt))
    rc = lib().oracle_nf4_project(_p(x), DT[xdt], R, K, N, _p(re), E, _p(codes), _p(absmax), _p(cb), B, DT[cdt],
                                  _p(bias), DT[bias_dt], mode, _p(out), DT[odt])
    if rc != 0:
        raise ValueError("oracle_nf4_project: " + ("bad block layout" if rc == -2 else "expert index out of range"))
    return out


def nf4_input_backward(grad, gdt: str, row_expert, payload: dict, K: int, cdt: str, exact: bool = False,
                       odt: str = None, magnitude: bool = False):
    grad = _c(grad)
    R, N = grad.shape
    B = payload["block"]
    codes, absmax = _c(payload["codes"], np.uint8), _c(payload["absmax"], np.float32)
    cb = _c(payload["codebook"], np.float32)
    E = codes.shape[0]
    re = _c(row_expert, np.int32)
    odt = odt or gdt
    mode = 2 if magnitude else 1 if exact else 0
    out = np.zeros((R, K), np.float64 if mode else _out_dtype(odt))
    rc = lib().oracle_nf4_input_backward(_p(grad), DT[gdt], R, N, K, _p(re), E, _p(codes), _p(absmax), _p(cb), B,
                                         DT[cdt], mode, _p(out), DT[odt])
    if rc != 0:
        raise ValueError("oracle_nf4_input_backward: " + ("bad block layout" if rc == -2 else "expert index out of range"))
    return out
