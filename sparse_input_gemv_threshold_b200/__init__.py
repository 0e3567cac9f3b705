"""Python binding of libsig.so, the activation-sparse linear layer for B200.

Argument marshalling only: every function checks dtypes and devices, takes
``data_ptr()`` of the torch tensors and the current CUDA stream, and calls the
C ABI declared in ``include/sig.h``.  Every step of the computation runs in the
library's CUDA kernels; there is no other implementation behind these calls.
Importing this module fails loudly when ``libsig.so`` has not been built.

fp16 tensors are ``torch.float16``; masks are ``torch.int32`` tensors holding
the uint32 bit words (bit i % 32 of word i // 32); index lists are int32.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

__all__ = [
    "LIB_PATH", "SigError", "OP_SPARSE_GEMV", "OP_TOPK", "OP_GATED_MLP", "OP_NM_GEMM",
    "MAX_D_IN", "abi_version", "workspace_bytes", "workspace", "sparsify_threshold",
    "sparsify_topk", "sparsify_nm", "sparse_gemv", "gated_mlp_sparse", "row_norms",
    "nm_act_gemm", "take_device_error", "status_string", "gated_mlp_sparse_noalloc",
    "sparse_gemv_multi", "workspace_bytes_multi", "OP_RANK_ADAPTER", "rank_adapter_sparse",
    "OP_SPARSE_GEMV_BATCH", "MAX_BATCH", "sparse_gemv_batch", "OP_SPARSE_GEMV_Q8",
    "sparse_gemv_q8", "sparsify_nm_ex", "nm_act_gemm_ex", "col_sums", "teal_mlp_sparse",
    "nm_packed_bytes", "sparsify_nm_packed", "nm_act_gemm_packed", "sparse_gemv_f8",
    "OP_SPARSE_GEMV_F8", "set_wait_limit", "sparse_gemv_q4", "OP_SPARSE_GEMV_Q4",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsig.so")

OP_SPARSE_GEMV, OP_TOPK, OP_GATED_MLP, OP_NM_GEMM, OP_RANK_ADAPTER = 1, 2, 3, 4, 5
OP_SPARSE_GEMV_BATCH = 6
OP_SPARSE_GEMV_Q8 = 7
OP_SPARSE_GEMV_F8 = 8
OP_SPARSE_GEMV_Q4 = 9
MAX_BATCH = 16
MAX_D_IN = 131072

_p, _i64, _i32, _f32, _sz = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                             ctypes.c_float, ctypes.c_size_t)

_SIGNATURES = {
    "sig_status_string": (ctypes.c_char_p, [_i32]),
    "sig_abi_version": (_i32, []),
    "sig_workspace_bytes": (_sz, [_i32, _i64, _i64, _i64]),
    "sig_workspace_init": (_i32, [_p, _sz, _p]),
    "sparsify_threshold": (_i32, [_p, _i64, _f32, _p, _p, _p, _p]),
    "sparsify_topk": (_i32, [_p, _i64, _i64, _p, _p, _p, _p, _sz, _p]),
    "sparsify_nm": (_i32, [_p, _i64, _i64, _i32, _i32, _p, _p, _p, _p]),
    "sig_nm_packed_bytes": (_sz, [_i64, _i64]),
    "nm_act_gemm_packed": (_i32, [_p, _i64, _i64, _p, _i64, _p, _p]),
    "sparse_gemv": (_i32, [_p, _i64, _i64, _p, _f32, _p, _p, _p, _p, _sz, _p]),
    "gated_mlp_sparse": (_i32, [_p, _p, _p, _p, _p, _i64, _i64, _f32, _p, _p, _p, _p, _sz, _p]),
    "sig_row_norms": (_i32, [_p, _i64, _i64, _p, _p]),
    "nm_act_gemm": (_i32, [_p, _i64, _i64, _p, _i64, _i32, _i32, _p, _p, _sz, _p]),
    "sig_take_device_error": (_i32, [ctypes.POINTER(ctypes.c_uint), _p]),
    "sig_set_wait_limit": (_i32, [ctypes.c_longlong]),
    "gated_mlp_sparse_noalloc": (_i32, [_p, _p, _p, _p, _p, _i64, _i64, _f32, _p, _p, _p, _p]),
    "sparse_gemv_multi": (_i32, [_i32, _p, _p, _i64, _p, _f32, _p, _p, _p, _p, _sz, _p]),
    "sig_workspace_bytes_multi": (_sz, [_i32, _p, _i64]),
    "rank_adapter_sparse": (_i32, [_p, _p, _p, _i64, _i64, _i64, _f32, _p, _p, _p, _p, _sz, _p]),
    "sparse_gemv_batch": (_i32, [_p, _i64, _i64, _p, _i64, _f32, _p, _p, _sz, _p]),
    "sparse_gemv_q8": (_i32, [_p, _p, _i64, _i64, _p, _f32, _p, _p, _sz, _p]),
    "sparse_gemv_f8": (_i32, [_p, _p, _i64, _i64, _p, _f32, _p, _p, _sz, _p]),
    "sparse_gemv_q4": (_i32, [_p, _p, _i64, _i64, _p, _f32, _p, _p, _sz, _p]),
    "sparsify_nm_ex": (_i32, [_p, _i64, _i64, _i32, _i32, _p, _p, _i32, _p, _p, _p, _p]),
    "nm_act_gemm_ex": (_i32, [_p, _i64, _i64, _p, _i64, _i32, _i32, _p, _p, _i32, _p, _p, _p, _sz,
                              _p]),
    "sig_col_sums": (_i32, [_p, _i64, _i64, _p, _p]),
    "teal_mlp_sparse": (_i32, [_p, _p, _p, _p, _i64, _i64, _f32, _f32, _p, _p, _p, _p, _sz, _p]),
}


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is not built; run `python sparse_input_gemv_threshold_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    return lib


_lib = _load()


class SigError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {status_string(status)} (status {status})")
        self.status = status


def status_string(status: int) -> str:
    return _lib.sig_status_string(status).decode()


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise SigError(fn, status)


def abi_version() -> int:
    return _lib.sig_abi_version()


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t):
    return None if t is None else t.data_ptr()


def _need(t, dtype, name, dev=None):
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dev is not None and t.device != dev:
        raise ValueError(f"{name} is on {t.device}, expected {dev}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def workspace_bytes(op: int, d_in: int, d_out: int = 0, rows: int = 0) -> int:
    return int(_lib.sig_workspace_bytes(op, d_in, d_out, rows))


_ws_cache = {}
_ws_lock = threading.Lock()


def workspace(op: int, d_in: int, d_out: int = 0, rows: int = 0, device=None,
              stream=None) -> torch.Tensor:
    """A zeroed workspace for ``op`` at these sizes, cached per (device, stream).

    The kernels leave their counters ready for the next call (returned to
    zero, or advanced to the next epoch), so a cached workspace can be reused
    by later calls on the same stream.  Calls on different streams get
    different workspaces.
    """
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    nbytes = workspace_bytes(op, d_in, d_out, rows)
    key = (dev, _stream(stream), op, d_in, d_out, rows)
    with _ws_lock:
        ws = _ws_cache.get(key)
        if ws is None:
            ws = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=dev)
            _ws_cache[key] = ws
    return ws


def sparsify_threshold(x, t: float, mask_bits=None, idx=None, nnz=None, stream=None):
    """Threshold mask |x_i| >= t.  Returns (mask_bits, idx, nnz) device tensors."""
    _need(x, torch.float16, "x")
    d = x.numel()
    words = (d + 31) // 32
    mask_bits = torch.empty(words, dtype=torch.int32, device=x.device) if mask_bits is None else mask_bits
    idx = torch.empty(d, dtype=torch.int32, device=x.device) if idx is None else idx
    nnz = torch.empty(1, dtype=torch.int32, device=x.device) if nnz is None else nnz
    _check("sparsify_threshold", _lib.sparsify_threshold(
        _ptr(x), d, float(t), _ptr(mask_bits), _ptr(idx), _ptr(nnz), _stream(stream)))
    return mask_bits, idx, nnz


def sparsify_topk(x, k: int, mask_bits=None, idx=None, nnz=None, stream=None):
    """Top-k mask by |x| (ties by lower index).  Returns (mask_bits, idx, nnz)."""
    _need(x, torch.float16, "x")
    d = x.numel()
    mask_bits = torch.empty((d + 31) // 32, dtype=torch.int32, device=x.device) if mask_bits is None else mask_bits
    idx = torch.empty(d, dtype=torch.int32, device=x.device) if idx is None else idx
    nnz = torch.empty(1, dtype=torch.int32, device=x.device) if nnz is None else nnz
    _check("sparsify_topk", _lib.sparsify_topk(
        _ptr(x), d, int(k), _ptr(mask_bits), _ptr(idx), _ptr(nnz), None, 0, _stream(stream)))
    return mask_bits, idx, nnz


def sparsify_nm(X, n: int, m: int, X_masked=None, mask_bits=None, want_masked=True,
                want_bits=True, stream=None):
    """Per-row N:M mask of a 2-D fp16 ``X``.  Returns (X_masked, mask_bits)."""
    _need(X, torch.float16, "X")
    rows, d = X.shape
    if want_masked and X_masked is None:
        X_masked = torch.empty_like(X)
    if want_bits and mask_bits is None:
        mask_bits = torch.empty((rows, (d + 31) // 32), dtype=torch.int32, device=X.device)
    _check("sparsify_nm", _lib.sparsify_nm(
        _ptr(X), rows, d, int(n), int(m), _ptr(X_masked), _ptr(mask_bits), None, _stream(stream)))
    return X_masked, mask_bits


def nm_packed_bytes(rows: int, d: int) -> int:
    return int(_lib.sig_nm_packed_bytes(rows, d))


def sparsify_nm_packed(X, n: int = 2, out=None, stream=None):
    """The packed 2:4 operand of ``X`` (n = 2: 2:4; n = 1: 1:4 padded to 2:4),
    as a uint8 tensor of sig_nm_packed_bytes(rows, d) bytes (values, then the
    tensor-core metadata; layout in include/sig.h)."""
    _need(X, torch.float16, "X")
    rows, d = X.shape
    nbytes = nm_packed_bytes(rows, d)
    if nbytes == 0:
        raise SigError("sparsify_nm", 2)
    if out is None:
        out = torch.empty(nbytes, dtype=torch.uint8, device=X.device)
    _check("sparsify_nm", _lib.sparsify_nm(
        _ptr(X), rows, d, int(n), 4, None, None, _ptr(out), _stream(stream)))
    return out


def nm_act_gemm_packed(packed, rows: int, K: int, WT, Y=None, stream=None):
    """Y = A WT with A (rows x K) given as sparsify_nm's packed 2:4 operand."""
    _need(packed, torch.uint8, "packed")
    _need(WT, torch.float16, "WT", packed.device)
    N = WT.shape[1]
    if Y is None:
        Y = torch.empty((rows, N), dtype=torch.float16, device=packed.device)
    _check("nm_act_gemm_packed", _lib.nm_act_gemm_packed(
        _ptr(packed), rows, K, _ptr(WT), N, _ptr(Y), _stream(stream)))
    return Y


def sparse_gemv(WT, x, t: float = 0.0, idx=None, nnz=None, y=None, ws=None, stream=None):
    """y = W (m . x) with WT (d_in, d_out) fp16.  idx/nnz select rows; else |x| >= t."""
    _need(WT, torch.float16, "WT")
    _need(x, torch.float16, "x", WT.device)
    d_in, d_out = WT.shape
    if x.numel() != d_in:
        raise ValueError("x length must equal WT.shape[0]")
    if y is None:
        y = torch.empty(d_out, dtype=torch.float16, device=WT.device)
    if ws is None:
        ws = workspace(OP_SPARSE_GEMV, d_in, d_out, device=WT.device, stream=stream)
    _check("sparse_gemv", _lib.sparse_gemv(
        _ptr(WT), d_in, d_out, _ptr(x), float(t), _ptr(idx), _ptr(nnz), _ptr(y),
        _ptr(ws), ws.numel(), _stream(stream)))
    return y


def _ptr_array(ts):
    return (ctypes.c_void_p * len(ts))(*[t.data_ptr() for t in ts])


def workspace_bytes_multi(d_outs, d_in: int) -> int:
    arr = (ctypes.c_int64 * len(d_outs))(*d_outs)
    return int(_lib.sig_workspace_bytes_multi(len(d_outs), arr, d_in))


def sparse_gemv_multi(WTs, x, t: float = 0.0, idx=None, nnz=None, ys=None, ws=None, stream=None):
    """y_p = W_p (m . x) for weights that read the same x, one mask, one launch."""
    _need(x, torch.float16, "x")
    d_in = x.numel()
    for i, w in enumerate(WTs):
        _need(w, torch.float16, f"WT[{i}]", x.device)
        if w.shape[0] != d_in:
            raise ValueError("every WT must have d_in rows")
    d_outs = [int(w.shape[1]) for w in WTs]
    if ys is None:
        ys = [torch.empty(n, dtype=torch.float16, device=x.device) for n in d_outs]
    if ws is None:
        nbytes = workspace_bytes_multi(d_outs, d_in)
        key = (x.device, _stream(stream), "multi", d_in, tuple(d_outs))
        with _ws_lock:
            ws = _ws_cache.get(key)
            if ws is None:
                ws = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=x.device)
                _ws_cache[key] = ws
    wt_arr, y_arr = _ptr_array(WTs), _ptr_array(ys)
    d_arr = (ctypes.c_int64 * len(d_outs))(*d_outs)
    _check("sparse_gemv_multi", _lib.sparse_gemv_multi(
        len(WTs), wt_arr, d_arr, d_in, _ptr(x), float(t), _ptr(idx), _ptr(nnz), y_arr,
        _ptr(ws), ws.numel(), _stream(stream)))
    return ys


def gated_mlp_sparse(x, WgT, WuT, WdT, down_norms, t: float, y=None, h_out=None,
                     mask_out=None, ws=None, stream=None):
    """RaNA gated MLP (Eqn. 12 masker then sparse down projection).  Returns y."""
    for name, w in (("WgT", WgT), ("WuT", WuT), ("WdT", WdT), ("x", x)):
        _need(w, torch.float16, name, x.device)
    _need(down_norms, torch.float32, "down_norms", x.device)
    d_model, d_ff = WgT.shape
    if y is None:
        y = torch.empty(d_model, dtype=torch.float16, device=x.device)
    if ws is None:
        ws = workspace(OP_GATED_MLP, d_model, d_ff, device=x.device, stream=stream)
    _check("gated_mlp_sparse", _lib.gated_mlp_sparse(
        _ptr(x), _ptr(WgT), _ptr(WuT), _ptr(WdT), _ptr(down_norms), d_model, d_ff, float(t),
        _ptr(y), _ptr(h_out), _ptr(mask_out), _ptr(ws), ws.numel(), _stream(stream)))
    return y


def sparsify_nm_ex(X, n: int, m: int, shift=None, norms=None, var: bool = False,
                   X_masked=None, want_bits=True, want_gamma=False, stream=None):
    """N:M mask with the per-token shift (PTS), the weight-aware score (WT:
    norms = ||W_i||) and the variance correction (VAR).  Returns
    (X_masked, mask_bits or None, gamma or None)."""
    _need(X, torch.float16, "X")
    rows, d = X.shape
    for name, v, size in (("shift", shift, rows), ("norms", norms, d)):
        if v is not None:
            _need(v, torch.float32, name, X.device)
            if v.numel() != size:
                raise ValueError(f"{name} must have {size} entries")
    if X_masked is None:
        X_masked = torch.empty_like(X)
    bits = (torch.empty((rows, (d + 31) // 32), dtype=torch.int32, device=X.device)
            if want_bits else None)
    gamma = torch.empty(rows, dtype=torch.float32, device=X.device) if want_gamma else None
    _check("sparsify_nm_ex", _lib.sparsify_nm_ex(
        _ptr(X), rows, d, n, m, _ptr(shift), _ptr(norms), int(bool(var)), _ptr(X_masked),
        _ptr(bits), _ptr(gamma), _stream(stream)))
    return X_masked, bits, gamma


def nm_act_gemm_ex(X, WT, n: int, m: int, shift=None, norms=None, var: bool = False,
                   col_sums=None, Y=None, ws=None, stream=None):
    """Y = X_masked WT + shift col_sums^T on the tensor cores (see sparsify_nm_ex)."""
    _need(X, torch.float16, "X")
    _need(WT, torch.float16, "WT", X.device)
    rows, K = X.shape
    N = WT.shape[1]
    if shift is not None and col_sums is None:
        col_sums = col_sums_of(WT, stream=stream)
    if Y is None:
        Y = torch.empty((rows, N), dtype=torch.float16, device=X.device)
    if ws is None:
        ws = workspace(OP_NM_GEMM, K, N, rows, device=X.device, stream=stream)
    _check("nm_act_gemm_ex", _lib.nm_act_gemm_ex(
        _ptr(X), rows, K, _ptr(WT), N, n, m, _ptr(shift), _ptr(norms), int(bool(var)),
        _ptr(col_sums), _ptr(Y), _ptr(ws), ws.numel(), _stream(stream)))
    return Y


def col_sums_of(WT, sums=None, stream=None):
    """r_j = sum_i WT[i, j] (float64 accumulation, float32 out)."""
    _need(WT, torch.float16, "WT")
    rows, cols = WT.shape
    if sums is None:
        sums = torch.empty(cols, dtype=torch.float32, device=WT.device)
    _check("sig_col_sums", _lib.sig_col_sums(_ptr(WT), rows, cols, _ptr(sums), _stream(stream)))
    return sums


col_sums = col_sums_of


def sparse_gemv_q8(QT, scale, x, t: float, y=None, ws=None, stream=None):
    """y = W (m . x) with int8 weights QT (d_in x d_out) and float32 column scales."""
    _need(QT, torch.int8, "QT")
    _need(scale, torch.float32, "scale", QT.device)
    _need(x, torch.float16, "x", QT.device)
    d_in, d_out = QT.shape
    if x.numel() != d_in or scale.numel() != d_out:
        raise ValueError("shapes: QT (d_in, d_out), scale (d_out), x (d_in)")
    if y is None:
        y = torch.empty(d_out, dtype=torch.float16, device=QT.device)
    if ws is None:
        ws = workspace(OP_SPARSE_GEMV_Q8, d_in, d_out, device=QT.device, stream=stream)
    _check("sparse_gemv_q8", _lib.sparse_gemv_q8(
        _ptr(QT), _ptr(scale), d_in, d_out, _ptr(x), float(t), _ptr(y), _ptr(ws), ws.numel(),
        _stream(stream)))
    return y


def sparse_gemv_f8(QT, scale, x, t: float, y=None, ws=None, stream=None):
    """y = W (m . x) with fp8 e4m3 weight codes QT (uint8, d_in x d_out) and
    float32 column scales."""
    _need(QT, torch.uint8, "QT")
    _need(scale, torch.float32, "scale", QT.device)
    _need(x, torch.float16, "x", QT.device)
    d_in, d_out = QT.shape
    if x.numel() != d_in or scale.numel() != d_out:
        raise ValueError("shapes: QT (d_in, d_out), scale (d_out), x (d_in)")
    if y is None:
        y = torch.empty(d_out, dtype=torch.float16, device=QT.device)
    if ws is None:
        ws = workspace(OP_SPARSE_GEMV_F8, d_in, d_out, device=QT.device, stream=stream)
    _check("sparse_gemv_f8", _lib.sparse_gemv_f8(
        _ptr(QT), _ptr(scale), d_in, d_out, _ptr(x), float(t), _ptr(y), _ptr(ws), ws.numel(),
        _stream(stream)))
    return y


def sparse_gemv_q4(QT4, scale, x, t: float, y=None, ws=None, stream=None):
    """y = W (m . x) with int4 weights packed two to a byte (QT4: uint8,
    d_in x d_out / 2; the even column in the low nibble) and float32 column
    scales."""
    _need(QT4, torch.uint8, "QT4")
    _need(scale, torch.float32, "scale", QT4.device)
    _need(x, torch.float16, "x", QT4.device)
    d_in, half = QT4.shape
    d_out = 2 * half
    if x.numel() != d_in or scale.numel() != d_out:
        raise ValueError("shapes: QT4 (d_in, d_out / 2), scale (d_out), x (d_in)")
    if y is None:
        y = torch.empty(d_out, dtype=torch.float16, device=QT4.device)
    if ws is None:
        ws = workspace(OP_SPARSE_GEMV_Q4, d_in, d_out, device=QT4.device, stream=stream)
    _check("sparse_gemv_q4", _lib.sparse_gemv_q4(
        _ptr(QT4), _ptr(scale), d_in, d_out, _ptr(x), float(t), _ptr(y), _ptr(ws), ws.numel(),
        _stream(stream)))
    return y


def sparse_gemv_batch(WT, X, t: float, Y=None, ws=None, stream=None):
    """Y[b] = W (m_b . X[b]), m_b = |X[b]| >= t, for B <= MAX_BATCH tokens in one launch."""
    _need(WT, torch.float16, "WT")
    _need(X, torch.float16, "X", WT.device)
    if X.dim() != 2 or X.shape[1] != WT.shape[0]:
        raise ValueError("X must be (B, d_in) with d_in = WT.shape[0]")
    B, d_in = X.shape
    d_out = WT.shape[1]
    if Y is None:
        Y = torch.empty((B, d_out), dtype=torch.float16, device=WT.device)
    if ws is None:
        ws = workspace(OP_SPARSE_GEMV_BATCH, d_in, d_out, B, device=WT.device, stream=stream)
    _check("sparse_gemv_batch", _lib.sparse_gemv_batch(
        _ptr(WT), d_in, d_out, _ptr(X), B, float(t), _ptr(Y), _ptr(ws), ws.numel(),
        _stream(stream)))
    return Y


def teal_mlp_sparse(x, WgT, WuT, WdT, t_x: float, t_h: float, y=None, h_out=None, mask_out=None,
                    ws=None, stream=None):
    """Gated MLP with the magnitude threshold on x (gate and up) and on h (down).  Returns y."""
    for name, w in (("WgT", WgT), ("WuT", WuT), ("WdT", WdT), ("x", x)):
        _need(w, torch.float16, name, x.device)
    d_model, d_ff = WgT.shape
    if y is None:
        y = torch.empty(d_model, dtype=torch.float16, device=x.device)
    if ws is None:
        ws = workspace(OP_GATED_MLP, d_model, d_ff, device=x.device, stream=stream)
    _check("teal_mlp_sparse", _lib.teal_mlp_sparse(
        _ptr(x), _ptr(WgT), _ptr(WuT), _ptr(WdT), d_model, d_ff, float(t_x), float(t_h), _ptr(y),
        _ptr(h_out), _ptr(mask_out), _ptr(ws), ws.numel(), _stream(stream)))
    return y


def rank_adapter_sparse(x, BT, AT, t: float, y=None, v_out=None, mask_out=None, ws=None,
                        stream=None):
    """RaNA rank adapter y = A (m . v), v = fp16(B x), m_i = v_i^2 >= t.  Returns y.

    ``BT`` is B transposed (d_in x r), ``AT`` is A transposed (r x d_out).
    """
    for name, w in (("BT", BT), ("AT", AT), ("x", x)):
        _need(w, torch.float16, name, x.device)
    d_in, r = BT.shape
    if AT.shape[0] != r or x.numel() != d_in:
        raise ValueError("shapes: x (d_in), BT (d_in, r), AT (r, d_out)")
    d_out = AT.shape[1]
    if y is None:
        y = torch.empty(d_out, dtype=torch.float16, device=x.device)
    if ws is None:
        ws = workspace(OP_RANK_ADAPTER, d_in, d_out, r, device=x.device, stream=stream)
    _check("rank_adapter_sparse", _lib.rank_adapter_sparse(
        _ptr(x), _ptr(BT), _ptr(AT), d_in, r, d_out, float(t), _ptr(y), _ptr(v_out),
        _ptr(mask_out), _ptr(ws), ws.numel(), _stream(stream)))
    return y


def gated_mlp_sparse_noalloc(x, WgT, WuT, WdT, down_norms, t: float, y=None, h_out=None,
                             mask_out=None, stream=None):
    """gated_mlp_sparse with no workspace: for callers that cannot allocate
    device memory at the call site.  Its scratch is a fixed array inside the
    library (SIG_NOALLOC_SCRATCH_BYTES per GPU); calls that overlap on the GPU
    race on it.  Make the first call on a device before any stream capture."""
    for name, w in (("WgT", WgT), ("WuT", WuT), ("WdT", WdT), ("x", x)):
        _need(w, torch.float16, name, x.device)
    _need(down_norms, torch.float32, "down_norms", x.device)
    d_model, d_ff = WgT.shape
    if y is None:
        y = torch.empty(d_model, dtype=torch.float16, device=x.device)
    _check("gated_mlp_sparse_noalloc", _lib.gated_mlp_sparse_noalloc(
        _ptr(x), _ptr(WgT), _ptr(WuT), _ptr(WdT), _ptr(down_norms), d_model, d_ff, float(t),
        _ptr(y), _ptr(h_out), _ptr(mask_out), _stream(stream)))
    return y


def row_norms(WT, out=None, stream=None):
    """float32 l2 norm of every row of a 2-D fp16 matrix (float64 accumulation)."""
    _need(WT, torch.float16, "WT")
    rows, cols = WT.shape
    out = torch.empty(rows, dtype=torch.float32, device=WT.device) if out is None else out
    _check("sig_row_norms", _lib.sig_row_norms(_ptr(WT), rows, cols, _ptr(out), _stream(stream)))
    return out


def nm_act_gemm(X, WT, n: int, m: int, Y=None, ws=None, stream=None):
    """Y = (M . X) WT with M the per-row n:m mask of X, on the tensor cores."""
    _need(X, torch.float16, "X")
    _need(WT, torch.float16, "WT", X.device)
    rows, K = X.shape
    N = WT.shape[1]
    if Y is None:
        Y = torch.empty((rows, N), dtype=torch.float16, device=X.device)
    if ws is None:
        ws = workspace(OP_NM_GEMM, K, N, rows, device=X.device, stream=stream)
    _check("nm_act_gemm", _lib.nm_act_gemm(
        _ptr(X), rows, K, _ptr(WT), N, int(n), int(m), _ptr(Y), _ptr(ws), ws.numel(),
        _stream(stream)))
    return Y


def take_device_error(stream=None) -> int:
    """Read and clear the device error word (0 = no kernel gave up on a wait)."""
    code = ctypes.c_uint(0)
    st = _lib.sig_take_device_error(ctypes.byref(code), _stream(stream))
    if st not in (0, 6):
        raise SigError("sig_take_device_error", st)
    return int(code.value)


def set_wait_limit(cycles: int) -> None:
    """Cycles after which a tensor-core GEMM wait gives up (<= 0: the default)."""
    _check("sig_set_wait_limit", _lib.sig_set_wait_limit(int(cycles)))
