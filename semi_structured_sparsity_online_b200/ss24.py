"""ctypes binding of ``libss24.so`` (declared in ``include/ss24.h``).

Argument marshalling only: every step of the pass runs in the library's CUDA
kernels. PyTorch supplies device memory (outputs are allocated as torch
tensors) and the current CUDA stream. The raw C functions are available as
``lib().ss24_*``; the helpers below wrap them for torch tensors.

The library must have been built (``semi_structured_sparsity_online_b200.build``
or ``__graft_entry__.build()``); loading fails loudly otherwise. There is no
CPU fallback.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libss24.so")

# enums (include/ss24.h)
OK = 0
STATUS_NAMES = {0: "SS24_OK", 1: "SS24_ERR_NULL", 2: "SS24_ERR_SHAPE", 3: "SS24_ERR_ALIGN",
                4: "SS24_ERR_DTYPE", 5: "SS24_ERR_FORMAT", 6: "SS24_ERR_WORKSPACE", 7: "SS24_ERR_CUDA",
                8: "SS24_ERR_ARG"}
STATUS_NAMES_INV = {v: k for k, v in STATUS_NAMES.items()}
BF16, F32 = 0, 1
MAG, WANDA = 0, 1
DENSE, SPARSE_24, SPARSE_48 = 0, 24, 48
FMT_NONE, FMT_FP8, FMT_INT, FMT_NVFP4, FMT_MXFP4 = 0, 1, 2, 3, 4
_FMT = {"none": FMT_NONE, "fp8": FMT_FP8, "int": FMT_INT, "nvfp4": FMT_NVFP4, "mxfp4": FMT_MXFP4}
_SCORE = {"mag": MAG, "wanda": WANDA}


class Format(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("bits", ctypes.c_int32), ("group", ctypes.c_int32),
                ("pack4", ctypes.c_int32)]


class Operand(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("axis", ctypes.c_int32),
                ("rows", ctypes.c_int64), ("k", ctypes.c_int64), ("ld", ctypes.c_int64),
                ("batch", ctypes.c_int64), ("batch_stride", ctypes.c_int64),
                ("hadamard", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class Outputs(ctypes.Structure):
    _fields_ = [("values", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("tensor_scale", ctypes.c_void_p), ("meta", ctypes.c_void_p)]


class SS24Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


_lib = None
_P = ctypes.c_void_p
_S = ctypes.c_size_t
_OP = ctypes.POINTER(Operand)
_OUT = ctypes.POINTER(Outputs)

_SIGNATURES = {
    "ss24_workspace_bytes": (ctypes.c_size_t, []),
    "ss24_workspace_init": (ctypes.c_int, [_P, _S, _P]),
    "ss24_workspace_error": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_int32), _P]),
    "ss24_prune24_compress": (ctypes.c_int, [_OP, ctypes.c_int, _P, _P, _P, _P, _P, _S, _P]),
    "ss24_quantize_fp8": (ctypes.c_int, [_OP, _P, _OUT, _P, _P, _S, _P]),
    "ss24_quantize_int": (ctypes.c_int, [_OP, Format, _OUT, _P, _P, _S, _P]),
    "ss24_quantize_nvfp4": (ctypes.c_int, [_OP, _P, _OUT, _P, _P, _S, _P]),
    "ss24_quantize_mxfp4": (ctypes.c_int, [_OP, _OUT, _P, _P, _S, _P]),
    "ss24_prune24_quant_fused": (ctypes.c_int, [_OP, ctypes.c_int, _P, Format, _P, _OUT, _P, _P, _S, _P]),
    "ss24_prune24_quant_fused_noalloc": (ctypes.c_int, [_OP, ctypes.c_int, _P, Format, _P, _OUT, _P, _P]),
    "ss24_prune48_pairwise_quant_fused": (ctypes.c_int,
                                          [_OP, ctypes.c_int, _P, Format, _P, _OUT, _P, _P, _S, _P]),
    "ss24_error_energy": (ctypes.c_int, [_OP, ctypes.c_int, ctypes.c_int, _P, Format, Format, _P, _P, _P, _P,
                                         _S, _P]),
    "ss24_amax": (ctypes.c_int, [_OP, ctypes.c_int, ctypes.c_int, _P, _P, _P, _S, _P]),
    "ss24_tensor_scale": (ctypes.c_int, [_OP, ctypes.c_int, ctypes.c_int, _P, ctypes.c_int32, _P, _P, _S, _P]),
    "ss24_predicted_ratio": (ctypes.c_int, [_P, _P, _P, ctypes.c_int64, _P]),
    "ss24_bits_per_element": (ctypes.c_double, [Format, ctypes.c_int, ctypes.c_int64, ctypes.c_int32]),
    "ss24_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "ss24_selfcheck_division": (ctypes.c_int, [ctypes.c_int32, ctypes.c_uint32, ctypes.c_uint32, _P, _P]),
    "ss24_amax_rows": (ctypes.c_int, [_OP, ctypes.c_int, ctypes.c_int, _P, _P, ctypes.c_int32, _P, _P, _S, _P]),
    "ss24_quantize_int_rows": (ctypes.c_int, [_OP, ctypes.c_int, ctypes.c_int, _P, Format, _P, _OUT, _P, _P, _S,
                                              _P]),
    "ss24_dequantize": (ctypes.c_int, [_OP, ctypes.c_int, Format, _OUT, _P, _P]),
    "ss24_hadamard": (ctypes.c_int, [_OP, ctypes.c_int32, _P, _P]),
    "ss24_softmax_prune": (ctypes.c_int, [_OP, ctypes.c_float, ctypes.c_int, Format, _P, _OUT, _P, _P,
                                          ctypes.c_size_t, _P]),
    "ss24_scale_tiles_bytes": (ctypes.c_int64, [ctypes.c_int64, ctypes.c_int64]),
    "ss24_scale_tiles": (ctypes.c_int, [_P, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, _P, _P]),
    "ss24_selfcheck_encoder": (ctypes.c_int, [ctypes.c_int32, _P, ctypes.c_int32, ctypes.c_uint32, ctypes.c_uint32,
                                              _P, _P]),
    "ss24_sparse_gemm_fp8": (ctypes.c_int, [_P, _P, _P, _P, _P, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                            _P, _P, _S, _P]),
    "ss24_encode_e4m3": (ctypes.c_int, [_P, _P, ctypes.c_int64, _P]),
    "ss24_decode_e4m3": (ctypes.c_int, [_P, _P, ctypes.c_int64, _P]),
    "ss24_encode_e2m1": (ctypes.c_int, [_P, _P, ctypes.c_int64, _P]),
    "ss24_decode_e2m1": (ctypes.c_int, [_P, _P, ctypes.c_int64, _P]),
}


def lib():
    """Load libss24.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build the CUDA library first "
                               "(python -m semi_structured_sparsity_online_b200.build)")
        h = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            f = getattr(h, name)
            f.restype = res
            f.argtypes = args
        _lib = h
    return _lib


def _check(status: int, where: str):
    if status != OK:
        raise SS24Error(status, where)


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def make_format(fmt="none", bits=8, group=0, pack4=False) -> Format:
    kind = _FMT[fmt] if isinstance(fmt, str) else int(fmt)
    return Format(kind, int(bits), int(group), int(bool(pack4)))


def make_operand(x: torch.Tensor, axis: int = 1, rows=None, k=None, hadamard: int = 0) -> Operand:
    """Operand descriptor of a CUDA tensor. 2-D: one operand; axis 1: x is
    [rows, ld] with k contiguous; axis 0: x is [k, ld] holding A[r][c] at
    x[c][r]. 3-D [B, ., .]: a batch of B such operands (x.stride(0) apart).
    hadamard: 0, or the block of the rotation the pass applies along k first."""
    if x.dtype == torch.bfloat16:
        dt = BF16
    elif x.dtype == torch.float32:
        dt = F32
    else:
        raise TypeError("operand must be bfloat16 or float32")
    if x.dim() not in (2, 3) or x.stride(-1) != 1:
        raise ValueError("operand must be 2-D or 3-D with a contiguous last dimension")
    batch, bstride = (x.shape[0], x.stride(0)) if x.dim() == 3 else (1, 0)
    m = x[0] if x.dim() == 3 else x
    if axis == 1:
        r = m.shape[0] if rows is None else rows
        kk = m.shape[1] if k is None else k
    else:
        kk = m.shape[0] if k is None else k
        r = m.shape[1] if rows is None else rows
    return Operand(x.data_ptr(), dt, axis, r, kk, m.stride(0), batch, bstride, int(hadamard), 0)


class Workspace:
    """Device workspace for the library's calls (allocated by torch, cleared once)."""

    def __init__(self, device=None, stream=None):
        n = lib().ss24_workspace_bytes()
        self.buf = torch.empty(n + 256, dtype=torch.uint8, device=device or "cuda")
        off = (-self.buf.data_ptr()) % 256
        self.tensor = self.buf[off:off + n]
        self.nbytes = n
        _check(lib().ss24_workspace_init(self.ptr, n, _stream(stream)), "ss24_workspace_init")

    @property
    def ptr(self):
        return ctypes.c_void_p(self.tensor.data_ptr())

    def error(self, stream=None) -> int:
        code = ctypes.c_int32(0)
        _check(lib().ss24_workspace_error(self.ptr, ctypes.byref(code), _stream(stream)), "ss24_workspace_error")
        return code.value


_default_ws = {}


def default_workspace(device=None) -> Workspace:
    dev = torch.device(device or "cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    if dev not in _default_ws:
        _default_ws[dev] = Workspace(dev)
    return _default_ws[dev]


def _alloc_outputs(x_rows, k, pattern, fmt: Format, in_dtype, device, batch=None):
    """Output tensors of a pass; with `batch` every output gets a leading
    [batch] dimension (the per-operand outputs packed one after the other)."""
    sparse = pattern != DENSE
    n = k // 2 if sparse else k
    lead = () if batch is None else (batch,)
    out = {}

    def empty(shape, dtype):
        return torch.empty(lead + shape, dtype=dtype, device=device)

    if fmt.kind == FMT_NONE:
        out["values"] = empty((x_rows, n), in_dtype)
    elif fmt.kind == FMT_FP8:
        out["values"] = empty((x_rows, n), torch.uint8)
    elif fmt.kind == FMT_INT:
        if fmt.pack4:
            out["values"] = empty((x_rows, n // 2), torch.uint8)
        else:
            out["values"] = empty((x_rows, n), torch.int16 if fmt.bits > 8 else torch.int8)
        g = fmt.group or n
        out["scales"] = empty((x_rows, n // g), torch.float32)
    elif fmt.kind in (FMT_NVFP4, FMT_MXFP4):
        out["values"] = empty((x_rows, n // 2), torch.uint8)
        blk = 16 if fmt.kind == FMT_NVFP4 else 32
        out["scales"] = empty((x_rows, n // blk), torch.uint8)
    if fmt.kind in (FMT_FP8, FMT_NVFP4):
        out["tensor_scale"] = empty((1,), torch.float32) if batch is None else torch.empty(
            (batch,), dtype=torch.float32, device=device)
    if sparse:
        out["meta"] = empty((x_rows, k // (16 if pattern == SPARSE_48 else 8)), torch.uint8)
    return out


def _lead(op):
    return None if op.batch <= 1 and op.batch_stride == 0 else op.batch


def _energy(op, device):
    b = _lead(op)
    return torch.zeros((4,) if b is None else (b, 4), dtype=torch.float64, device=device)


def run(x: torch.Tensor, pattern=SPARSE_24, fmt="none", bits=8, group=0, pack4=False, score="mag",
        col_norms=None, tensor_scale=None, energy=True, axis=1, ws=None, stream=None, out=None, hadamard=0):
    """One pass through the matching C entry point. Returns a dict of output
    tensors (``values``, ``scales``, ``tensor_scale``, ``meta``) and ``energy``
    (float64[4] on the device: e_total, e_prune, e_quant, e_quant_dense). A
    3-D x is a batch: every output and the energies get a leading [B].
    hadamard=b rotates x along k in the pass first (block Hadamard of b, the
    result rounded to bf16; bf16 input, magnitude score), and so do the amax
    passes behind a derived tensor scale."""
    f = make_format(fmt, bits, group, pack4)
    op = make_operand(x, axis, hadamard=hadamard)
    sc = _SCORE[score] if isinstance(score, str) else int(score)
    if out is None:
        out = _alloc_outputs(op.rows, op.k, pattern, f, x.dtype, x.device, _lead(op))
    e = _energy(op, x.device) if energy is True else energy
    if e is not None and e is not False:
        out["energy"] = e
    else:
        e = None
    ws = ws or default_workspace(x.device)
    o = Outputs(*(_ptr(out.get(key)) for key in ("values", "scales", "tensor_scale", "meta")))
    s = _stream(stream)
    L = lib()
    if pattern == DENSE:
        if f.kind == FMT_FP8:
            st = L.ss24_quantize_fp8(ctypes.byref(op), _ptr(tensor_scale), ctypes.byref(o), _ptr(e), ws.ptr,
                                     ws.nbytes, s)
        elif f.kind == FMT_INT:
            st = L.ss24_quantize_int(ctypes.byref(op), f, ctypes.byref(o), _ptr(e), ws.ptr, ws.nbytes, s)
        elif f.kind == FMT_NVFP4:
            st = L.ss24_quantize_nvfp4(ctypes.byref(op), _ptr(tensor_scale), ctypes.byref(o), _ptr(e), ws.ptr,
                                       ws.nbytes, s)
        elif f.kind == FMT_MXFP4:
            st = L.ss24_quantize_mxfp4(ctypes.byref(op), ctypes.byref(o), _ptr(e), ws.ptr, ws.nbytes, s)
        else:
            raise ValueError("dense pattern needs a quantization format")
        _check(st, "ss24_quantize")
    elif pattern == SPARSE_24 and f.kind == FMT_NONE and tensor_scale is None:
        _check(L.ss24_prune24_compress(ctypes.byref(op), sc, _ptr(col_norms), _ptr(out["values"]),
                                       _ptr(out["meta"]), _ptr(e), ws.ptr, ws.nbytes, s), "ss24_prune24_compress")
    else:
        fn = L.ss24_prune24_quant_fused if pattern == SPARSE_24 else L.ss24_prune48_pairwise_quant_fused
        _check(fn(ctypes.byref(op), sc, _ptr(col_norms), f, _ptr(tensor_scale), ctypes.byref(o), _ptr(e),
                  ws.ptr, ws.nbytes, s), "ss24_prune_quant_fused")
    return out


def error_energy(x, pattern=SPARSE_24, sparse_fmt=("none",), dense_fmt=("int", 8, 0), score="mag",
                 col_norms=None, sparse_scale=None, dense_scale=None, axis=1, ws=None, stream=None, energy=None,
                 hadamard=0):
    """Read-only energy pass; returns float64[4] (or [B, 4]) on the device."""
    sf = make_format(*sparse_fmt) if isinstance(sparse_fmt, tuple) else sparse_fmt
    df = make_format(*dense_fmt) if isinstance(dense_fmt, tuple) else dense_fmt
    op = make_operand(x, axis, hadamard=hadamard)
    e = energy if energy is not None else _energy(op, x.device)
    ws = ws or default_workspace(x.device)
    _check(lib().ss24_error_energy(ctypes.byref(op), pattern, _SCORE[score] if isinstance(score, str) else score,
                                   _ptr(col_norms), sf, df, _ptr(sparse_scale), _ptr(dense_scale), _ptr(e), ws.ptr,
                                   ws.nbytes, _stream(stream)), "ss24_error_energy")
    return e


def amax(x, pattern=SPARSE_24, score="mag", col_norms=None, axis=1, ws=None, stream=None, hadamard=0):
    op = make_operand(x, axis, hadamard=hadamard)
    out = torch.empty(max(op.batch, 1), dtype=torch.float32, device=x.device)
    ws = ws or default_workspace(x.device)
    _check(lib().ss24_amax(ctypes.byref(op), pattern, _SCORE[score] if isinstance(score, str) else score,
                           _ptr(col_norms), _ptr(out), ws.ptr, ws.nbytes, _stream(stream)), "ss24_amax")
    return out


def tensor_scale(x, fmt="fp8", pattern=SPARSE_24, score="mag", col_norms=None, axis=1, ws=None, stream=None,
                 out=None, hadamard=0):
    """The per-tensor scale (FP8: amax / 448, NVFP4: amax / 2688) as a device
    float32[1] (float32[B] for a batch)."""
    op = make_operand(x, axis, hadamard=hadamard)
    out = out if out is not None else torch.empty(max(op.batch, 1), dtype=torch.float32, device=x.device)
    ws = ws or default_workspace(x.device)
    _check(lib().ss24_tensor_scale(ctypes.byref(op), pattern, _SCORE[score] if isinstance(score, str) else score,
                                   _ptr(col_norms), _FMT[fmt] if isinstance(fmt, str) else fmt, _ptr(out), ws.ptr,
                                   ws.nbytes, _stream(stream)), "ss24_tensor_scale")
    return out


def amax_rows(x, pattern=DENSE, score="mag", col_norms=None, scale_fmt=None, ws=None, stream=None, out=None,
              scale_out=None, hadamard=0):
    """Per-row amax of the values a pass with this pattern / score quantizes,
    float32 [rows] (or [B, rows]) on the device, and, with scale_fmt ("fp8" or
    "nvfp4"), the per-tensor scale from the same read: returns (rows, scale)."""
    op = make_operand(x, 1, hadamard=hadamard)
    lead = _lead(op)
    shape = (op.rows,) if lead is None else (lead, op.rows)
    out = out if out is not None else torch.empty(shape, dtype=torch.float32, device=x.device)
    if scale_fmt is not None and scale_out is None:
        scale_out = torch.empty(max(op.batch, 1), dtype=torch.float32, device=x.device)
    kind = 0 if scale_fmt is None else (_FMT[scale_fmt] if isinstance(scale_fmt, str) else int(scale_fmt))
    ws = ws or default_workspace(x.device)
    _check(lib().ss24_amax_rows(ctypes.byref(op), pattern, _SCORE[score] if isinstance(score, str) else score,
                                _ptr(col_norms), _ptr(out), kind, _ptr(scale_out), ws.ptr, ws.nbytes,
                                _stream(stream)), "ss24_amax_rows")
    return out, scale_out


def run_int_rows(x, row_amax, pattern=DENSE, bits=8, pack4=False, score="mag", col_norms=None, energy=True,
                 ws=None, stream=None, out=None, hadamard=0):
    """INT-b with one scale per row from a given per-row amax (ss24_quantize_int_rows);
    returns the same dict as run()."""
    f = make_format("int", bits, 0, pack4)
    op = make_operand(x, 1, hadamard=hadamard)
    if out is None:
        out = _alloc_outputs(op.rows, op.k, pattern, f, x.dtype, x.device, _lead(op))
    e = _energy(op, x.device) if energy is True else energy
    if e is not None and e is not False:
        out["energy"] = e
    else:
        e = None
    ws = ws or default_workspace(x.device)
    o = Outputs(*(_ptr(out.get(key)) for key in ("values", "scales", "tensor_scale", "meta")))
    _check(lib().ss24_quantize_int_rows(ctypes.byref(op), pattern, _SCORE[score] if isinstance(score, str) else score,
                                        _ptr(col_norms), f, _ptr(row_amax), ctypes.byref(o), _ptr(e), ws.ptr,
                                        ws.nbytes, _stream(stream)), "ss24_quantize_int_rows")
    return out


def dequantize(out, rows, k, pattern=SPARSE_24, fmt="none", bits=8, group=0, pack4=False, dtype=torch.bfloat16,
               batch=None, stream=None, xhat=None):
    """The dense float32 operand [rows, k] (or [B, rows, k]) that the outputs of a
    pass (the dict run() returns) stand for: dequantized values on kept
    positions, zero on dropped ones."""
    f = make_format(fmt, bits, group, pack4)
    dev = out["values"].device
    op = Operand(None, BF16 if dtype == torch.bfloat16 else F32, 1, rows, k, k, batch or 0, 0)
    shape = (rows, k) if batch is None else (batch, rows, k)
    xhat = xhat if xhat is not None else torch.empty(shape, dtype=torch.float32, device=dev)
    o = Outputs(*(_ptr(out.get(key)) for key in ("values", "scales", "tensor_scale", "meta")))
    _check(lib().ss24_dequantize(ctypes.byref(op), pattern, f, ctypes.byref(o), _ptr(xhat), _stream(stream)),
           "ss24_dequantize")
    return xhat


def softmax_prune(s: torch.Tensor, alpha: float, pattern=SPARSE_24, fmt="fp8", bits=8, group=0, pack4=False,
                  tensor_scale=None, energy=True, ws=None, stream=None, out=None):
    """P = softmax(alpha * s) per row, pruned / quantized in the same pass
    (ss24_softmax_prune): the same dict as run() for the bf16 operand P, which
    is never stored. s: logits [rows, keys] or [B, rows, keys], bf16 or fp32."""
    f = make_format(fmt, bits, group, pack4)
    op = make_operand(s, 1)
    if out is None:
        out = _alloc_outputs(op.rows, op.k, pattern, f, torch.bfloat16, s.device, _lead(op))
    e = _energy(op, s.device) if energy is True else energy
    if e is not None and e is not False:
        out["energy"] = e
    else:
        e = None
    ws = ws or default_workspace(s.device)
    o = Outputs(*(_ptr(out.get(key)) for key in ("values", "scales", "tensor_scale", "meta")))
    _check(lib().ss24_softmax_prune(ctypes.byref(op), float(alpha), pattern, f, _ptr(tensor_scale), ctypes.byref(o),
                                    _ptr(e), ws.ptr, ws.nbytes, _stream(stream)),
           "ss24_softmax_prune")
    return out


def hadamard(x: torch.Tensor, block: int, out=None, stream=None):
    """Block Hadamard rotation of x [rows, k] or [B, rows, k] (bf16 or fp32,
    k contiguous) along k (ss24_hadamard): fp32 of the same shape, packed."""
    op = make_operand(x, 1)
    out = out if out is not None else torch.empty(x.shape, dtype=torch.float32, device=x.device)
    _check(lib().ss24_hadamard(ctypes.byref(op), int(block), _ptr(out), _stream(stream)), "ss24_hadamard")
    return out


def scale_tiles(scales, rows, cols, batch=None, out=None, stream=None):
    """NVFP4 / MXFP4 scale bytes (uint8 [rows, cols] or [B, rows, cols] on the
    device, packed) in the block-scaled MMA's 128 x 4 tile layout
    (ss24_scale_tiles): uint8 [B * ss24_scale_tiles_bytes(rows, cols)]."""
    nb = batch or 1
    per = lib().ss24_scale_tiles_bytes(rows, cols)
    if per < 0:
        raise ValueError("negative scale matrix size")
    out = out if out is not None else torch.empty(nb * per, dtype=torch.uint8, device=scales.device)
    _check(lib().ss24_scale_tiles(_ptr(scales), rows, cols, batch or 0, _ptr(out), _stream(stream)),
           "ss24_scale_tiles")
    return out


def predicted_ratio(sparse_energy, dense_energy, out=None, stream=None):
    """float64[..., 4] on the device: loss, rel_err_sparse, rel_err_dense, R_hat,
    for each pair of energy records (float64[..., 4], contiguous)."""
    count = sparse_energy.numel() // 4
    r = out if out is not None else torch.empty_like(sparse_energy)
    _check(lib().ss24_predicted_ratio(_ptr(sparse_energy), _ptr(dense_energy), _ptr(r), count, _stream(stream)),
           "ss24_predicted_ratio")
    return r


def sparse_gemm_fp8(a, b, y=None, ws=None, stream=None):
    """Y = s_a s_b A B^T on the tensor cores' 2:4-sparse FP8 MMA
    (ss24_sparse_gemm_fp8). a: the dict of a 2:4 + FP8 pass over [m, k]
    (``values`` [m, k/2], ``meta`` [m, k/8], ``tensor_scale``); b: the dict of a
    dense FP8 pass over [n, k] (``values`` [n, k], ``tensor_scale``). Returns
    float32 [m, n] on the device."""
    m, n, k = a["values"].shape[0], b["values"].shape[0], b["values"].shape[1]
    y = y if y is not None else torch.empty((m, n), dtype=torch.float32, device=a["values"].device)
    ws = ws or default_workspace(a["values"].device)
    _check(lib().ss24_sparse_gemm_fp8(_ptr(a["values"]), _ptr(a["meta"]), _ptr(a["tensor_scale"]),
                                      _ptr(b["values"]), _ptr(b["tensor_scale"]), m, n, k, _ptr(y), ws.ptr,
                                      ws.nbytes, _stream(stream)), "ss24_sparse_gemm_fp8")
    return y


def bits_per_element(fmt="none", bits=8, group=0, pattern=SPARSE_24, k=4096, with_scales=False) -> float:
    return lib().ss24_bits_per_element(make_format(fmt, bits, group), pattern, k, int(with_scales))


def status_string(status: int) -> str:
    return lib().ss24_status_string(status).decode()


def selfcheck_division(mode=0, b_first=0, b_count=1 << 23, chunk=1 << 16, stream=None):
    """Mismatches between the kernels' corrected division and IEEE division
    (see ss24_selfcheck_division); returns (count, first mismatch or None)."""
    res = torch.tensor([0, -1], dtype=torch.int64, device="cuda")
    for b0 in range(b_first, b_first + b_count, chunk):
        n = min(chunk, b_first + b_count - b0)
        _check(lib().ss24_selfcheck_division(mode, b0, n, _ptr(res), _stream(stream)), "ss24_selfcheck_division")
    r = res.cpu().numpy().view("uint64")
    return int(r[0]), (None if r[1] == 0xFFFFFFFFFFFFFFFF else (int(r[1]) >> 32, int(r[1]) & 0xFFFFFFFF))


def selfcheck_encoder(kind, bounds, chunk=1 << 12, stream=None):
    """Mismatches between the kernels' E4M3 ("fp8") or E2M1 ("nvfp4") encoder
    and the step table `bounds` (see ss24_selfcheck_encoder) over every finite
    fp32 bit pattern; returns (count, first mismatching bit pattern or None)."""
    k = _FMT[kind] if isinstance(kind, str) else int(kind)
    b = torch.as_tensor(np.asarray(bounds, dtype=np.uint32).view(np.int32)).cuda()
    res = torch.tensor([0, -1], dtype=torch.int64, device="cuda")
    for h0 in range(0, 1 << 16, chunk):
        n = min(chunk, (1 << 16) - h0)
        _check(lib().ss24_selfcheck_encoder(k, _ptr(b), b.numel(), h0, n, _ptr(res), _stream(stream)),
               "ss24_selfcheck_encoder")
    r = res.cpu().numpy().view("uint64")
    return int(r[0]), (None if r[1] == 0xFFFFFFFFFFFFFFFF else int(r[1]))


def _convert(name, t_in, out_dtype, stream=None):
    out = torch.empty(t_in.shape, dtype=out_dtype, device=t_in.device)
    _check(getattr(lib(), name)(_ptr(t_in), _ptr(out), t_in.numel(), _stream(stream)), name)
    return out


def encode_e4m3(t, stream=None):
    return _convert("ss24_encode_e4m3", t.contiguous(), torch.uint8, stream)


def decode_e4m3(t, stream=None):
    return _convert("ss24_decode_e4m3", t.contiguous(), torch.float32, stream)


def encode_e2m1(t, stream=None):
    return _convert("ss24_encode_e2m1", t.contiguous(), torch.uint8, stream)


def decode_e2m1(t, stream=None):
    return _convert("ss24_decode_e2m1", t.contiguous(), torch.float32, stream)
