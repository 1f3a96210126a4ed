"""W4A4 / MXFP4 linear layer of MACaQ on NVIDIA B200 (sm_100a).

A thin ctypes binding over ``libmacaq.so`` (C ABI in ``include/macaq.h``). Every function here only
marshals torch CUDA tensors into pointers and sizes, allocates outputs with torch when the caller
does not pass them, and raises on a non-zero status: all arithmetic runs in the library's CUDA
kernels. There is no CPU fallback; calling without the built library raises.

Method (page "Huawei's research lab in Switzerland open-sources the four-bit quantization tool
MACaQ for running models locally", aipolix.com, paragraphs 2-3; page "MACaQ quantizer from
huawei-csl targets GGUF, vLLM and Diffusers models", glonce.com, paragraph 5):
    W' = MXFP4(W diag(s) H_b / b)      prep_weights (offline)
    X' = MXFP4(X diag(1/s) H_b)        act_quant (online)
    Y  = X' W'^T                       linear / grouped_linear
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

__all__ = [
    "MacaqError", "OUT_BF16", "OUT_F32", "A_QUANTIZED", "A_BF16_FUSED", "A_BF16_ONE_LAUNCH",
    "sf_bytes", "grouped_sf_bytes", "workspace_bytes", "fused_workspace_bytes", "WORKSPACE_COUNTER_BYTES",
    "status_str",
    "prep_weights", "act_quant", "linear", "linear_fixed_scratch", "grouped_linear", "device_status",
    "set_wait_limit_ns", "check_group_offsets", "act_quant_gather", "moe_combine",
    "linear_swiglu", "swiglu_act_quant", "interleave_gate_up", "flip_refine", "act_transform", "linear_w4a16",
    "library_path", "lib",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libmacaq.so")
_lock = threading.Lock()
_lib = None

OUT_BF16, OUT_F32 = 0, 1
WORKSPACE_COUNTER_BYTES = 65536  # MACAQ_WORKSPACE_COUNTER_BYTES: the zero-between-calls counter region
A_QUANTIZED, A_BF16_FUSED, A_BF16_ONE_LAUNCH = 0, 1, 2

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_i32 = ctypes.c_int32
_sz = ctypes.c_size_t

_SIGNATURES = {
    "macaq_status_str": ([ctypes.c_int], ctypes.c_char_p),
    "macaq_last_cuda_error": ([], ctypes.c_int),
    "macaq_sf_bytes": ([_i64, _i64], _sz),
    "macaq_grouped_sf_bytes": ([_i64, _i32, _i64], _sz),
    "macaq_workspace_bytes": ([_i64, _i64, _i64, _i32], _sz),
    "macaq_fused_workspace_bytes": ([_i64, _i64, _i64, _i32], _sz),
    "macaq_prep_weights": ([_vp, _vp, _i64, _i64, _i32, _vp, _vp, _vp, _vp], ctypes.c_int),
    "macaq_act_quant": ([_vp, _vp, _i64, _i64, _i32, _vp, _i32, _vp, _vp, _vp], ctypes.c_int),
    "macaq_linear": ([_i32, _vp, _vp, _vp, _i64, _i64, _i64, _i32, _vp, _vp, _vp, _i32, _vp, _sz, _vp],
                     ctypes.c_int),
    "macaq_linear_fixed_scratch": ([_i32, _vp, _vp, _vp, _i64, _i64, _i64, _i32, _vp, _vp, _vp, _i32, _vp],
                                   ctypes.c_int),
    "macaq_grouped_linear": ([_i32, _vp, _vp, _vp, _vp, _i32, _i64, _i64, _i64, _i32, _vp, _vp, _vp, _i32, _vp,
                              _sz, _vp], ctypes.c_int),
    "macaq_device_status": ([ctypes.POINTER(ctypes.c_int32), _i32], ctypes.c_int),
    "macaq_set_wait_limit_ns": ([ctypes.c_uint64], None),
    "macaq_check_group_offsets": ([_vp, _i32, _i64], ctypes.c_int),
    "macaq_act_quant_gather": ([_vp, _i64, _vp, _vp, _i64, _i64, _i32, _vp, _i32, _vp, _vp, _vp], ctypes.c_int),
    "macaq_moe_combine": ([_vp, _i64, _i64, _vp, _vp, _i64, _i32, _vp, _i32, _vp], ctypes.c_int),
    "macaq_linear_swiglu_workspace_bytes": ([_i64, _i64, _i64], _sz),
    "macaq_linear_swiglu": ([_vp, _vp, _i64, _i64, _i64, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _sz, _vp], ctypes.c_int),
    "macaq_swiglu_act_quant": ([_vp, _i64, _i64, _vp, _i32, _vp, _vp, _vp], ctypes.c_int),
    "macaq_flip_refine": ([_vp, _vp, _i64, _i64, _i32, _vp, _i32, _vp, _vp, _vp, _vp], ctypes.c_int),
    "macaq_act_transform": ([_vp, _vp, _i64, _i64, _i32, _vp, _vp], ctypes.c_int),
    "macaq_linear_w4a16_workspace_bytes": ([_i64, _i64, _i64], _sz),
    "macaq_linear_w4a16": ([_vp, _vp, _i64, _i64, _i64, _i32, _vp, _vp, _vp, _i32, _vp, _sz, _vp], ctypes.c_int),
}


class MacaqError(RuntimeError):
    """A libmacaq call returned a non-zero status."""

    def __init__(self, fn: str, status: int):
        self.status = status
        name = status_str(status)
        extra = ""
        if name == "MACAQ_ERR_CUDA":
            extra = f" (cudaError {lib().macaq_last_cuda_error()})"
        super().__init__(f"{fn} failed: {name}{extra}")


def library_path() -> str:
    return _LIB_PATH


def lib():
    """The loaded libmacaq.so (raises if it has not been built: there is no fallback)."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(_LIB_PATH):
                    raise RuntimeError(
                        f"libmacaq.so is missing at {_LIB_PATH}; build it with "
                        "`python -m w4a4_mxfp4_quantized_b200.build` (nvcc, sm_100a)")
                L = ctypes.CDLL(_LIB_PATH)
                for name, (args, res) in _SIGNATURES.items():
                    f = getattr(L, name)
                    f.argtypes = args
                    f.restype = res
                _lib = L
    return _lib


def status_str(status: int) -> str:
    return lib().macaq_status_str(int(status)).decode()


def _check(fn: str, status: int):
    if status != 0:
        raise MacaqError(fn, status)


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libmacaq takes CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("libmacaq takes contiguous tensors")
    return t.data_ptr()


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


_ws_cache: dict = {}


def _workspace(dev, nbytes: int) -> torch.Tensor:
    """A scratch buffer per device, zero-initialised, grown on demand and reused across calls (the
    kernels leave its counter region zero). Calls that may overlap on different streams need their
    own buffers."""
    key = torch.device(dev).index
    buf = _ws_cache.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
        _ws_cache[key] = buf
    return buf


def sf_bytes(rows: int, K: int) -> int:
    """Bytes of the tiled scale-factor buffer of `rows` rows of K elements."""
    return int(lib().macaq_sf_bytes(rows, K))


def grouped_sf_bytes(total_rows: int, E: int, K: int) -> int:
    return int(lib().macaq_grouped_sf_bytes(total_rows, E, K))


def workspace_bytes(M: int, N: int, K: int, E: int = 0) -> int:
    return int(lib().macaq_workspace_bytes(M, N, K, E))


def fused_workspace_bytes(M: int, N: int, K: int, E: int = 0) -> int:
    return int(lib().macaq_fused_workspace_bytes(M, N, K, E))


def prep_weights(W: torch.Tensor, s: torch.Tensor | None, had_block: int = 32, *, Wq=None, Wsf=None,
                 inv_s=None):
    """Offline W' = MXFP4(W diag(s) H_b / b). Returns (Wq u8 [N, K/2], Wsf u8 tiled, inv_s fp32 [K] or None)."""
    assert W.dtype == torch.bfloat16 and W.dim() == 2
    N, K = W.shape
    dev = W.device
    Wq = torch.empty(N, K // 2, dtype=torch.uint8, device=dev) if Wq is None else Wq
    Wsf = torch.empty(max(sf_bytes(N, K), 16), dtype=torch.uint8, device=dev) if Wsf is None else Wsf
    if s is not None and inv_s is None:
        inv_s = torch.empty(K, dtype=torch.float32, device=dev)
    _check("macaq_prep_weights", lib().macaq_prep_weights(
        _ptr(W), _ptr(s), N, K, had_block, _ptr(Wq), _ptr(Wsf), _ptr(inv_s) if s is not None else None,
        _stream(dev)))
    return Wq, Wsf, (inv_s if s is not None else None)


def act_quant(X: torch.Tensor, inv_s: torch.Tensor | None, had_block: int = 32, *, group_offsets=None,
              Xq=None, Xsf=None):
    """Online X' = MXFP4(X diag(inv_s) H_b). Returns (Xq u8 [M, K/2], Xsf u8 tiled).

    group_offsets (int32 CUDA [E+1]) selects the grouped form: inv_s is then [E, K]."""
    assert X.dtype == torch.bfloat16 and X.dim() == 2
    M, K = X.shape
    dev = X.device
    E = 0 if group_offsets is None else group_offsets.numel() - 1
    Xq = torch.empty(M, K // 2, dtype=torch.uint8, device=dev) if Xq is None else Xq
    if Xsf is None:
        n = grouped_sf_bytes(M, E, K) if group_offsets is not None else sf_bytes(M, K)
        Xsf = torch.empty(max(n, 16), dtype=torch.uint8, device=dev)
    _check("macaq_act_quant", lib().macaq_act_quant(
        _ptr(X), _ptr(inv_s), M, K, had_block, _ptr(group_offsets), E, _ptr(Xq), _ptr(Xsf), _stream(dev)))
    return Xq, Xsf


def act_quant_gather(X: torch.Tensor, row_index: torch.Tensor, inv_s: torch.Tensor | None, had_block: int = 32, *,
                     group_offsets=None, Xq=None, Xsf=None):
    """act_quant of the gathered rows X[row_index] without writing that copy: row m of the output is
    the transform and MXFP4 of X[row_index[m]] (row_index int32 CUDA [M]). Grouped form as act_quant."""
    assert X.dtype == torch.bfloat16 and X.dim() == 2 and row_index.dtype == torch.int32
    x_rows, K = X.shape
    M = row_index.numel()
    dev = X.device
    E = 0 if group_offsets is None else group_offsets.numel() - 1
    Xq = torch.empty(M, K // 2, dtype=torch.uint8, device=dev) if Xq is None else Xq
    if Xsf is None:
        n = grouped_sf_bytes(M, E, K) if group_offsets is not None else sf_bytes(M, K)
        Xsf = torch.empty(max(n, 16), dtype=torch.uint8, device=dev)
    _check("macaq_act_quant_gather", lib().macaq_act_quant_gather(
        _ptr(X), x_rows, _ptr(row_index), _ptr(inv_s), M, K, had_block, _ptr(group_offsets), E, _ptr(Xq), _ptr(Xsf),
        _stream(dev)))
    return Xq, Xsf


def moe_combine(Y: torch.Tensor, pos: torch.Tensor, weights: torch.Tensor, *, out_dtype: int = OUT_BF16, out=None):
    """out[t] = sum_j weights[t, j] * Y[pos[t, j]] in fp32, j in order (pos outside Y's rows skipped).
    Y bf16 CUDA [rows, N] (N % 8 == 0); pos int32 and weights fp32 CUDA [T, topk]."""
    assert Y.dtype == torch.bfloat16 and pos.dtype == torch.int32 and weights.dtype == torch.float32
    y_rows, N = Y.shape
    T, topk = pos.shape
    dev = Y.device
    out = _out(T, N, out_dtype, dev, out)
    _check("macaq_moe_combine", lib().macaq_moe_combine(
        _ptr(Y), y_rows, N, _ptr(pos), _ptr(weights), T, topk, _ptr(out), out_dtype, _stream(dev)))
    return out


def interleave_gate_up(W_gate: torch.Tensor, W_up: torch.Tensor, block: int = 64) -> torch.Tensor:
    """Stacks gate and up weights [I, K] into the [2I, K] layout linear_swiglu expects: gate rows
    64j..64j+63, then up rows 64j..64j+63, for every j (pure indexing)."""
    I, K = W_gate.shape
    return torch.stack([W_gate.view(I // block, block, K), W_up.view(I // block, block, K)], dim=1).reshape(2 * I, K)


def linear_swiglu(A: torch.Tensor, Asf: torch.Tensor, Wq: torch.Tensor, Wsf: torch.Tensor,
                  inv_s_down: torch.Tensor | None, had_block_down: int = 32, *, Hq=None, Hsf=None, workspace=None):
    """Gate/up linear (weights interleaved by interleave_gate_up, then prep_weights) followed by SwiGLU and
    the down projection's activation quantization. Returns (Hq u8 [M, I/2], Hsf u8 tiled), the down
    projection's A operand."""
    N = Wq.shape[0]
    K = Wq.shape[1] * 2
    M = A.shape[0]
    I = N // 2
    dev = A.device
    Hq = torch.empty(M, I // 2, dtype=torch.uint8, device=dev) if Hq is None else Hq
    Hsf = torch.empty(max(sf_bytes(M, I), 16), dtype=torch.uint8, device=dev) if Hsf is None else Hsf
    need = int(lib().macaq_linear_swiglu_workspace_bytes(M, N, K))
    if workspace is None and need > 0:
        workspace = _workspace(dev, need)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("macaq_linear_swiglu", lib().macaq_linear_swiglu(
        _ptr(A), _ptr(Asf), M, N, K, _ptr(Wq), _ptr(Wsf), _ptr(inv_s_down), had_block_down, _ptr(Hq), _ptr(Hsf),
        _ptr(workspace), ws_bytes, _stream(dev)))
    return Hq, Hsf


def swiglu_act_quant(GU: torch.Tensor, inv_s: torch.Tensor | None, had_block: int = 32, *, Hq=None, Hsf=None):
    """MXFP4(silu(G) U diag(inv_s) H_b) from an fp32 gate/up output [M, 2I] (64-interleaved columns)."""
    assert GU.dtype == torch.float32 and GU.dim() == 2
    M, N = GU.shape
    I = N // 2
    dev = GU.device
    Hq = torch.empty(M, I // 2, dtype=torch.uint8, device=dev) if Hq is None else Hq
    Hsf = torch.empty(max(sf_bytes(M, I), 16), dtype=torch.uint8, device=dev) if Hsf is None else Hsf
    _check("macaq_swiglu_act_quant", lib().macaq_swiglu_act_quant(
        _ptr(GU), M, I, _ptr(inv_s), had_block, _ptr(Hq), _ptr(Hsf), _stream(dev)))
    return Hq, Hsf


def flip_refine(W: torch.Tensor, s: torch.Tensor | None, H: torch.Tensor, Wq: torch.Tensor, Wsf: torch.Tensor,
                had_block: int = 32, sweeps: int = 1, flips: torch.Tensor | None = None):
    """Refines the prepared codes Wq in place (Hessian-guided moves to neighbouring FP4 values, scales
    fixed). H: fp32 CUDA [K, K] symmetric. Returns the per-row count of accepted moves (int32 [N])."""
    assert W.dtype == torch.bfloat16 and H.dtype == torch.float32
    N, K = W.shape
    dev = W.device
    flips = torch.empty(N, dtype=torch.int32, device=dev) if flips is None else flips
    _check("macaq_flip_refine", lib().macaq_flip_refine(
        _ptr(W), _ptr(s), N, K, had_block, _ptr(H), sweeps, _ptr(Wq), _ptr(Wsf), _ptr(flips), _stream(dev)))
    return flips


def act_transform(X: torch.Tensor, inv_s: torch.Tensor | None, had_block: int = 32, *, Xt=None):
    """bf16(X diag(inv_s) H_b): the weight-only mode's activations (the act_quant transform, no MXFP4)."""
    assert X.dtype == torch.bfloat16 and X.dim() == 2
    M, K = X.shape
    Xt = torch.empty(M, K, dtype=torch.bfloat16, device=X.device) if Xt is None else Xt
    _check("macaq_act_transform", lib().macaq_act_transform(_ptr(X), _ptr(inv_s), M, K, had_block, _ptr(Xt),
                                                            _stream(X.device)))
    return Xt


def linear_w4a16(X: torch.Tensor, inv_s: torch.Tensor | None, Wq: torch.Tensor, Wsf: torch.Tensor, *,
                 had_block: int = 32, out_dtype: int = OUT_BF16, Y=None, workspace=None):
    """Weight-only layer for decode (M <= 64): Y = bf16(X diag(inv_s) H_b) dq(W')^T, fp32 accumulation."""
    N = Wq.shape[0]
    K = Wq.shape[1] * 2
    M = X.shape[0]
    dev = X.device
    Y = _out(M, N, out_dtype, dev, Y)
    need = int(lib().macaq_linear_w4a16_workspace_bytes(M, N, K))
    if workspace is None and need > 0:
        workspace = _workspace(dev, need)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("macaq_linear_w4a16", lib().macaq_linear_w4a16(
        _ptr(X), _ptr(inv_s), M, N, K, had_block, _ptr(Wq), _ptr(Wsf), _ptr(Y), out_dtype, _ptr(workspace), ws_bytes,
        _stream(dev)))
    return Y


def _out(M, N, out_dtype, dev, Y):
    if Y is not None:
        return Y
    return torch.empty(M, N, dtype=torch.float32 if out_dtype == OUT_F32 else torch.bfloat16, device=dev)


def linear(A: torch.Tensor, Asf: torch.Tensor | None, Wq: torch.Tensor, Wsf: torch.Tensor, *,
           mode: int = A_QUANTIZED, inv_s: torch.Tensor | None = None, had_block: int = 32,
           out_dtype: int = OUT_BF16, Y=None, workspace=None, use_workspace: bool = True):
    """Dense W4A4 linear Y = dq(A) dq(W')^T (fp32 accumulate; bf16 or fp32 out).

    mode=A_QUANTIZED: A, Asf from act_quant. With few rows (M <= 128) a workspace selects the skinny
    kernel (weights in the MMA's M slot, split over all SMs); use_workspace=False runs the general
    kernel instead.
    mode=A_BF16_FUSED: A is bf16 X [M, K]; the call applies inv_s, H_b and MXFP4 itself (inside the
    GEMM kernel for M <= 4, else a quantizer pass then the GEMM) and needs a workspace.
    mode=A_BF16_ONE_LAUNCH: the same result; M > 128 (N, K % 256 == 0) runs as one launch in which
    the 2-SM GEMM quantizes X itself."""
    N = Wq.shape[0]
    K = Wq.shape[1] * 2
    M = A.shape[0]
    dev = A.device
    Y = _out(M, N, out_dtype, dev, Y)
    fused = mode in (A_BF16_FUSED, A_BF16_ONE_LAUNCH)
    if fused:
        ws_need = fused_workspace_bytes(M, N, K, 0)
    else:
        ws_need = workspace_bytes(M, N, K, 0) if use_workspace else 0
    if workspace is None and ws_need > 0:
        workspace = _workspace(dev, ws_need)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("macaq_linear", lib().macaq_linear(
        mode, _ptr(A), None if fused else _ptr(Asf), _ptr(inv_s) if fused else None, M, N, K, had_block, _ptr(Wq),
        _ptr(Wsf), _ptr(Y), out_dtype, _ptr(workspace), ws_bytes, _stream(dev)))
    return Y


def linear_fixed_scratch(A: torch.Tensor, Asf: torch.Tensor, Wq: torch.Tensor, Wsf: torch.Tensor, *,
                         out_dtype: int = OUT_BF16, Y=None):
    """linear() on the library's fixed per-device scratch: the C call allocates no device memory
    (pass Y to allocate nothing here either). Calls that may overlap on one device race."""
    N = Wq.shape[0]
    K = Wq.shape[1] * 2
    M = A.shape[0]
    dev = A.device
    Y = _out(M, N, out_dtype, dev, Y)
    _check("macaq_linear_fixed_scratch", lib().macaq_linear_fixed_scratch(
        A_QUANTIZED, _ptr(A), _ptr(Asf), None, M, N, K, 32, _ptr(Wq), _ptr(Wsf), _ptr(Y), out_dtype, _stream(dev)))
    return Y


def grouped_linear(A: torch.Tensor, Asf: torch.Tensor | None, group_offsets: torch.Tensor, Wq: torch.Tensor,
                   Wsf: torch.Tensor, *, mode: int = A_QUANTIZED, inv_s: torch.Tensor | None = None,
                   had_block: int = 32, out_dtype: int = OUT_BF16, Y=None, workspace=None):
    """Grouped W4A4 linear: rows of expert e times W'_e. Wq [E, N, K/2], Wsf [E, sf_bytes(N, K)].

    mode=A_BF16_FUSED: A is bf16 X [total_rows, K] and inv_s [E, K]; the call quantizes it per
    expert into the workspace, then runs the grouped GEMM."""
    E, N, K2 = Wq.shape
    K = K2 * 2
    M = A.shape[0]
    dev = A.device
    Y = _out(M, N, out_dtype, dev, Y)
    fused = mode in (A_BF16_FUSED, A_BF16_ONE_LAUNCH)
    ws_need = fused_workspace_bytes(M, N, K, E) if fused else workspace_bytes(M, N, K, E)
    if workspace is None and ws_need > 0:
        workspace = _workspace(dev, ws_need)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("macaq_grouped_linear", lib().macaq_grouped_linear(
        mode, _ptr(A), None if fused else _ptr(Asf), _ptr(inv_s) if fused else None, _ptr(group_offsets), E, M, N,
        K, had_block, _ptr(Wq), _ptr(Wsf), _ptr(Y), out_dtype, _ptr(workspace), ws_bytes, _stream(dev)))
    return Y


def device_status(reset: bool = False) -> int:
    """The sticky device status word (0, or 6 = a bounded wait ran out). Synchronize first."""
    v = ctypes.c_int32(0)
    _check("macaq_device_status", lib().macaq_device_status(ctypes.byref(v), 1 if reset else 0))
    return int(v.value)


def set_wait_limit_ns(ns: int):
    lib().macaq_set_wait_limit_ns(int(ns))


def check_group_offsets(offsets, total_rows: int) -> None:
    """Host-side check of grouped row offsets (a CPU tensor or array of E + 1 int32 values): they must
    start at 0, end at total_rows and never decrease. Raises MacaqError(MACAQ_ERR_SHAPE) otherwise.
    The device-side reads clamp malformed offsets instead of failing, so callers that hold a host
    copy check it here before launching."""
    import numpy as np

    a = np.ascontiguousarray(np.asarray(offsets.cpu() if isinstance(offsets, torch.Tensor) else offsets,
                                        dtype=np.int32))
    if a.ndim != 1 or a.size < 2:
        raise MacaqError("macaq_check_group_offsets", 2)
    _check("macaq_check_group_offsets", lib().macaq_check_group_offsets(
        a.ctypes.data_as(ctypes.c_void_p), a.size - 1, int(total_rows)))
