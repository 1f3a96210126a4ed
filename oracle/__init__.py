"""CPU oracle for the MACaQ W4A4 / MXFP4 linear layer (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this package. The CUDA library never calls it and shares no code with it.

The arithmetic lives in ``macaq_oracle.c`` (plain C, compiled with ``-O2 -ffp-contract=off`` so
that no multiply-add is contracted); this module only marshals numpy arrays into it. Every
function cites, in the C source, the passage of the pages (or of OCP MX v1.0) it follows.

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py`` against closed forms,
brute force and the OCP E2M1 table; model-level quality (perplexity, KL) is not computed here and
stays unpinned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "macaq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

MX_GROUP = 32

_u8p = ctypes.POINTER(ctypes.c_uint8)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)
_i64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile liboracle.so next to its source (gcc, -O2 -ffp-contract=off)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11", "-fPIC", "-shared",
            "-o", tmp, _SRC, "-lm",
        ])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            lib.oracle_fwht_f32.argtypes = [_f32p, ctypes.c_int]
            lib.oracle_transform_rows.argtypes = [_u16p, _f32p, _i64, _i64, ctypes.c_int, ctypes.c_int, _f32p]
            lib.oracle_e8m0_exponent.argtypes = [ctypes.c_float]
            lib.oracle_e8m0_exponent.restype = ctypes.c_int
            lib.oracle_e2m1_code.argtypes = [ctypes.c_float]
            lib.oracle_e2m1_code.restype = ctypes.c_uint8
            lib.oracle_e2m1_value.argtypes = [ctypes.c_uint8]
            lib.oracle_e2m1_value.restype = ctypes.c_double
            lib.oracle_mxfp4_quantize_row.argtypes = [_f32p, _i64, _u8p, _u8p]
            lib.oracle_prep_weights.argtypes = [_u16p, _f32p, _i64, _i64, ctypes.c_int, _u8p, _u8p, _f32p, _f32p]
            lib.oracle_act_quant.argtypes = [_u16p, _f32p, _i64, _i64, ctypes.c_int, _i32p, ctypes.c_int32,
                                             _u8p, _u8p, _f32p]
            lib.oracle_dequant_row.argtypes = [_u8p, _u8p, _i64, _f64p]
            lib.oracle_linear.argtypes = [_u8p, _u8p, _i64p, _i64, _u8p, _u8p, _i64, _i64, _f64p, _f64p, _f64p]
            lib.oracle_grouped_linear.argtypes = [_u8p, _u8p, _i32p, ctypes.c_int32, _i64p, _i64, _u8p, _u8p,
                                                  _i64, _i64, _f64p, _f64p, _f64p]
            lib.oracle_bf16_rne.argtypes = [ctypes.c_float]
            lib.oracle_bf16_rne.restype = ctypes.c_uint16
            lib.oracle_moe_combine.argtypes = [_u16p, _i64, _i64, _i32p, _f32p, _i64, ctypes.c_int32, _f32p]
            lib.oracle_exp_f32.argtypes = [ctypes.c_float]
            lib.oracle_exp_f32.restype = ctypes.c_float
            lib.oracle_swiglu_f32.argtypes = [ctypes.c_float, ctypes.c_float]
            lib.oracle_swiglu_f32.restype = ctypes.c_float
            lib.oracle_swiglu_act_quant.argtypes = [_f32p, _f32p, _f32p, _i64, _i64, ctypes.c_int, _u8p, _u8p, _f32p]
            lib.oracle_act_transform_bf16.argtypes = [_u16p, _f32p, _i64, _i64, ctypes.c_int, _u16p, _f32p]
            lib.oracle_flip_refine.argtypes = [_u16p, _f32p, _i64, _i64, ctypes.c_int, _f32p, ctypes.c_int, _u8p, _u8p,
                                               _i32p, _f32p, _f64p]
            _lib = lib
    return _lib


def _p(a: np.ndarray | None, ptype):
    if a is None:
        return ctypes.cast(None, ptype)
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ptype)


def _bits16(x) -> np.ndarray:
    """bf16 data as its uint16 bit pattern (accepts a CPU torch bf16 tensor or a uint16 array)."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch

    assert x.dtype == torch.bfloat16 and x.device.type == "cpu"
    return np.ascontiguousarray(x.contiguous().view(torch.int16).numpy().view(np.uint16))


def _f32(a) -> np.ndarray | None:
    if a is None:
        return None
    if not isinstance(a, np.ndarray):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(a, dtype=np.float32)


def fwht_f32(v: np.ndarray) -> np.ndarray:
    """Fixed-order fp32 Walsh-Hadamard butterfly over one block (returns a new array)."""
    out = np.array(v, dtype=np.float32, copy=True)
    _load().oracle_fwht_f32(_p(out, _f32p), out.shape[-1])
    return out


def transform_rows(x_bf16, mul, b: int, absorb: bool) -> np.ndarray:
    """fl32(x * mul) then H_b per aligned block (then * 1/b when absorb). Returns fp32 [rows, K]."""
    x = _bits16(x_bf16)
    rows, K = x.shape
    m = _f32(mul)
    out = np.empty((rows, K), np.float32)
    _load().oracle_transform_rows(_p(x, _u16p), _p(m, _f32p), rows, K, int(b), int(bool(absorb)), _p(out, _f32p))
    return out


def e8m0_exponent(amax: float) -> int:
    return int(_load().oracle_e8m0_exponent(ctypes.c_float(amax)))


def e2m1_code(t: float) -> int:
    return int(_load().oracle_e2m1_code(ctypes.c_float(t)))


def e2m1_value(code: int) -> float:
    return float(_load().oracle_e2m1_value(ctypes.c_uint8(code)))


def mxfp4_quantize(y: np.ndarray):
    """MXFP4 of fp32 rows [rows, K] -> (codes u8 [rows, K/2], sf u8 [rows, K/32])."""
    y = np.ascontiguousarray(y, dtype=np.float32)
    if y.ndim == 1:
        y = y[None, :]
    rows, K = y.shape
    codes = np.empty((rows, K // 2), np.uint8)
    sf = np.empty((rows, K // MX_GROUP), np.uint8)
    lib = _load()
    for r in range(rows):
        lib.oracle_mxfp4_quantize_row(_p(y[r], _f32p), K, _p(codes[r], _u8p), _p(sf[r], _u8p))
    return codes, sf


def prep_weights(W_bf16, s, b: int):
    """W' = MXFP4(W diag(s) H_b / b) -> (Wq [N, K/2], Wsf [N, K/32] row-major, inv_s [K] or None)."""
    w = _bits16(W_bf16)
    N, K = w.shape
    s32 = _f32(s)
    Wq = np.empty((N, K // 2), np.uint8)
    Wsf = np.empty((N, K // MX_GROUP), np.uint8)
    inv_s = np.empty(K, np.float32) if s32 is not None else None
    work = np.empty((N, K), np.float32)
    _load().oracle_prep_weights(_p(w, _u16p), _p(s32, _f32p), N, K, int(b), _p(Wq, _u8p), _p(Wsf, _u8p),
                                _p(inv_s, _f32p), _p(work, _f32p))
    return Wq, Wsf, inv_s


def act_quant(X_bf16, inv_s, b: int, offsets=None):
    """MXFP4(X diag(inv_s) H_b) -> (Xq [M, K/2], Xsf [M, K/32] row-major).

    offsets (int32 [E+1]) selects the grouped form: rows of expert e use inv_s[e] ([E, K])."""
    x = _bits16(X_bf16)
    M, K = x.shape
    inv = _f32(inv_s)
    off = None if offsets is None else np.ascontiguousarray(np.asarray(offsets, dtype=np.int32))
    E = 0 if off is None else len(off) - 1
    Xq = np.empty((M, K // 2), np.uint8)
    Xsf = np.empty((M, K // MX_GROUP), np.uint8)
    work = np.empty(K, np.float32)
    _load().oracle_act_quant(_p(x, _u16p), _p(inv, _f32p), M, K, int(b), _p(off, _i32p), E, _p(Xq, _u8p),
                             _p(Xsf, _u8p), _p(work, _f32p))
    return Xq, Xsf


def dequant(codes: np.ndarray, sf: np.ndarray) -> np.ndarray:
    """MXFP4 rows -> float64 values (exact)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    rows = codes.shape[0]
    K = codes.shape[1] * 2
    out = np.empty((rows, K), np.float64)
    lib = _load()
    for r in range(rows):
        lib.oracle_dequant_row(_p(codes[r], _u8p), _p(sf[r], _u8p), K, _p(out[r], _f64p))
    return out


def linear(Aq, Asf, Wq, Wsf, rows=None):
    """Y = dq(A) dq(W)^T and T = |dq(A)| |dq(W)|^T in float64, for the listed rows of A."""
    Aq = np.ascontiguousarray(Aq, dtype=np.uint8)
    Asf = np.ascontiguousarray(Asf, dtype=np.uint8)
    Wq = np.ascontiguousarray(Wq, dtype=np.uint8)
    Wsf = np.ascontiguousarray(Wsf, dtype=np.uint8)
    M, K = Aq.shape[0], Aq.shape[1] * 2
    N = Wq.shape[0]
    r = None if rows is None else np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    n_rows = M if r is None else len(r)
    Y = np.empty((n_rows, N), np.float64)
    T = np.empty((n_rows, N), np.float64)
    work = np.empty((n_rows + 1) * K, np.float64)
    _load().oracle_linear(_p(Aq, _u8p), _p(Asf, _u8p), _p(r, _i64p), n_rows, _p(Wq, _u8p), _p(Wsf, _u8p), N, K,
                          _p(Y, _f64p), _p(T, _f64p), _p(work, _f64p))
    return Y, T


def grouped_linear(Aq, Asf, offsets, Wq, Wsf, rows=None):
    """Grouped form: Wq [E, N, K/2], Wsf [E, N, K/32]; rows of expert e use its weights."""
    Aq = np.ascontiguousarray(Aq, dtype=np.uint8)
    Asf = np.ascontiguousarray(Asf, dtype=np.uint8)
    Wq = np.ascontiguousarray(Wq, dtype=np.uint8)
    Wsf = np.ascontiguousarray(Wsf, dtype=np.uint8)
    off = np.ascontiguousarray(np.asarray(offsets, dtype=np.int32))
    E = len(off) - 1
    M, K = Aq.shape[0], Aq.shape[1] * 2
    N = Wq.shape[1]
    r = None if rows is None else np.ascontiguousarray(np.sort(np.asarray(rows, dtype=np.int64)))
    n_rows = M if r is None else len(r)
    Y = np.empty((n_rows, N), np.float64)
    T = np.empty((n_rows, N), np.float64)
    work = np.empty(2 * K, np.float64)
    _load().oracle_grouped_linear(_p(Aq, _u8p), _p(Asf, _u8p), _p(off, _i32p), E, _p(r, _i64p), n_rows,
                                  _p(Wq, _u8p), _p(Wsf, _u8p), N, K, _p(Y, _f64p), _p(T, _f64p), _p(work, _f64p))
    return Y, T


def _dequant_rows(codes: np.ndarray, sf: np.ndarray, rows=None) -> np.ndarray:
    """dequant() of the listed rows (all rows when None)."""
    if rows is None:
        return dequant(codes, sf)
    rows = np.asarray(rows, dtype=np.int64)
    return dequant(codes[rows], sf[rows])


def linear_matmul(Aq, Asf, Wq, Wsf, rows=None, n_chunk: int = 4096):
    """The quantity linear() computes, Y = dq(A) dq(W)^T and T = |dq(A)| |dq(W)|^T in float64, for the
    listed rows of A, with the sum over k taken by a float64 library matmul instead of the ordered C
    loop. The dequantization is the same exact C routine (OCP MX v1.0 element and scale values); the
    sums differ from linear()'s only by float64 rounding, at most about K * 2^-53 of T, far inside the
    1e-5 * T tolerance the GPU is held to. W is dequantized n_chunk rows at a time."""
    Aq = np.ascontiguousarray(Aq, dtype=np.uint8)
    Asf = np.ascontiguousarray(Asf, dtype=np.uint8)
    a = _dequant_rows(Aq, Asf, rows)
    a_abs = np.abs(a)
    N = Wq.shape[0]
    Y = np.empty((a.shape[0], N), np.float64)
    T = np.empty((a.shape[0], N), np.float64)
    for n0 in range(0, N, n_chunk):
        w = dequant(np.ascontiguousarray(Wq[n0:n0 + n_chunk]), np.ascontiguousarray(Wsf[n0:n0 + n_chunk]))
        Y[:, n0:n0 + w.shape[0]] = a @ w.T
        T[:, n0:n0 + w.shape[0]] = a_abs @ np.abs(w).T
    return Y, T


def grouped_linear_matmul(Aq, Asf, offsets, Wq, Wsf, rows=None):
    """grouped_linear() with the k-sums by a float64 library matmul (see linear_matmul): row m of expert
    e (offsets[e] <= m < offsets[e+1]) is multiplied by W'_e = Wq[e], Wsf[e] (row-major SF [N, K/32])."""
    off = np.asarray(offsets, dtype=np.int64)
    M = int(off[-1])
    rows = np.arange(M) if rows is None else np.sort(np.asarray(rows, dtype=np.int64))
    N = Wq.shape[1]
    Y = np.empty((len(rows), N), np.float64)
    T = np.empty((len(rows), N), np.float64)
    expert = np.searchsorted(off, rows, side="right") - 1
    for e in np.unique(expert):
        sel = np.nonzero(expert == e)[0]
        a = _dequant_rows(np.ascontiguousarray(Aq, dtype=np.uint8), np.ascontiguousarray(Asf, dtype=np.uint8),
                          rows[sel])
        w = dequant(np.ascontiguousarray(Wq[e]), np.ascontiguousarray(Wsf[e]))
        Y[sel] = a @ w.T
        T[sel] = np.abs(a) @ np.abs(w).T
    return Y, T


def bf16_rne(values) -> np.ndarray:
    """fp32 values -> bf16 bit patterns (uint16), round to nearest even."""
    v = np.ascontiguousarray(np.asarray(values, dtype=np.float32)).ravel()
    lib = _load()
    return np.array([lib.oracle_bf16_rne(float(x)) for x in v], dtype=np.uint16).reshape(np.shape(values))


def moe_combine(Y_bf16, pos, w) -> np.ndarray:
    """out[t, n] = sum_j fl32(w[t, j] * Y[pos[t, j], n]) in fp32, j in order from +0 (pos outside the
    rows of Y skipped). Y: bf16 [y_rows, N] (torch CPU tensor or uint16 bits); pos int32 and w fp32
    [T, topk]. Returns fp32 [T, N]."""
    y = _bits16(Y_bf16)
    y_rows, N = y.shape
    pos = np.ascontiguousarray(np.asarray(pos, dtype=np.int32))
    w = np.ascontiguousarray(np.asarray(w, dtype=np.float32))
    T, topk = pos.shape
    out = np.empty((T, N), np.float32)
    _load().oracle_moe_combine(_p(y, _u16p), y_rows, N, _p(pos, _i32p), _p(w, _f32p), T, topk, _p(out, _f32p))
    return out


def exp_f32(x: float) -> float:
    """The fixed fp32 exp of the fused SwiGLU (Cody-Waite reduction, degree-6 Taylor, x in [-100, 88])."""
    return float(_load().oracle_exp_f32(ctypes.c_float(x)))


def swiglu_f32(g: float, u: float) -> float:
    return float(_load().oracle_swiglu_f32(ctypes.c_float(g), ctypes.c_float(u)))


def swiglu_act_quant(G, U, inv_s, b: int):
    """MXFP4(swiglu(G, U) diag(inv_s) H_b) of fp32 [M, I] gate and up outputs -> (Hq [M, I/2], Hsf [M, I/32])."""
    G = np.ascontiguousarray(G, dtype=np.float32)
    U = np.ascontiguousarray(U, dtype=np.float32)
    M, I = G.shape
    inv = _f32(inv_s)
    Hq = np.empty((M, I // 2), np.uint8)
    Hsf = np.empty((M, I // MX_GROUP), np.uint8)
    work = np.empty(I, np.float32)
    _load().oracle_swiglu_act_quant(_p(G, _f32p), _p(U, _f32p), _p(inv, _f32p), M, I, int(b), _p(Hq, _u8p),
                                    _p(Hsf, _u8p), _p(work, _f32p))
    return Hq, Hsf


def flip_refine(W_bf16, s, b: int, H, sweeps: int, Wq, Wsf):
    """Flip-Refinement of prepared codes (see macaq_oracle.c): W bf16 [N, K], s [K] or None, H fp32 [K, K]
    symmetric, Wq [N, K/2] and Wsf [N, K/32] row-major from prep_weights. Returns (refined Wq, flips [N])."""
    w = _bits16(W_bf16)
    N, K = w.shape
    s32 = _f32(s)
    Hh = np.ascontiguousarray(H, dtype=np.float32)
    q = np.array(Wq, dtype=np.uint8, copy=True, order="C")
    sf = np.ascontiguousarray(Wsf, dtype=np.uint8)
    flips = np.empty(N, np.int32)
    wrow = np.empty(K, np.float32)
    g = np.empty(K, np.float64)
    _load().oracle_flip_refine(_p(w, _u16p), _p(s32, _f32p), N, K, int(b), _p(Hh, _f32p), int(sweeps), _p(q, _u8p),
                               _p(sf, _u8p), _p(flips, _i32p), _p(wrow, _f32p), _p(g, _f64p))
    return q, flips


def act_transform_bf16(X_bf16, inv_s, b: int) -> np.ndarray:
    """bf16 bits [M, K] of X diag(inv_s) H_b computed in fp32 and rounded once (weight-only activations)."""
    x = _bits16(X_bf16)
    M, K = x.shape
    inv = _f32(inv_s)
    out = np.empty((M, K), np.uint16)
    work = np.empty(K, np.float32)
    _load().oracle_act_transform_bf16(_p(x, _u16p), _p(inv, _f32p), M, K, int(b), _p(out, _u16p), _p(work, _f32p))
    return out


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact float64 values of bf16 bit patterns."""
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


def w4a16_linear(X_bf16, inv_s, b: int, Wq, Wsf, rows=None, n_chunk: int = 4096):
    """The weight-only layer: Y = bf16(X diag(inv_s) H_b) dq(W')^T and T = |.| |.|^T in float64 (the k-sum by a
    library matmul, as linear_matmul), for the listed rows of X."""
    xt = act_transform_bf16(X_bf16 if rows is None else _rows16(X_bf16, rows), inv_s, b)
    a = bf16_bits_to_f64(xt)
    a_abs = np.abs(a)
    N = Wq.shape[0]
    Y = np.empty((a.shape[0], N), np.float64)
    T = np.empty((a.shape[0], N), np.float64)
    for n0 in range(0, N, n_chunk):
        w = dequant(np.ascontiguousarray(Wq[n0:n0 + n_chunk]), np.ascontiguousarray(Wsf[n0:n0 + n_chunk]))
        Y[:, n0:n0 + w.shape[0]] = a @ w.T
        T[:, n0:n0 + w.shape[0]] = a_abs @ np.abs(w).T
    return Y, T


def _rows16(X_bf16, rows):
    return np.ascontiguousarray(_bits16(X_bf16)[np.asarray(rows, dtype=np.int64)])
