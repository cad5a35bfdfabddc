"""ctypes wrapper of the ss24 oracle (``oracle/ss24_oracle.c``).

TEST INFRASTRUCTURE. The oracle is a plain, slow CPU statement of the online
2:4 prune / compress / quantize pass and of its error energies ("Is 2:4 Sparsity
Still Worth It? Semi-Structured Sparsity versus Quantization in LLM Inference",
§2-§4 and §6). Only the test suite, the package smoke check and the benchmark's
CPU-baseline leg may import this module. It shares no code with the CUDA path.

Arrays are numpy: a bf16 operand is passed as its raw ``uint16`` bit patterns,
an fp32 operand as ``float32``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ss24_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

BF16, F32 = 0, 1
MAG, WANDA = 0, 1
DENSE, SPARSE_24, SPARSE_48 = 0, 24, 48
FMT_NONE, FMT_FP8, FMT_INT, FMT_NVFP4, FMT_MXFP4 = 0, 1, 2, 3, 4

_FMT_NAMES = {"none": FMT_NONE, "fp8": FMT_FP8, "int": FMT_INT, "nvfp4": FMT_NVFP4, "mxfp4": FMT_MXFP4}


def build(force: bool = False) -> str:
    """Compile the oracle with gcc: binary32 arithmetic, no contraction, no fast-math."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-Wall", "-ffp-contract=off", "-fno-fast-math",
               "-fPIC", "-shared", "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


class _Args(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("axis", ctypes.c_int32),
                ("rows", ctypes.c_int64), ("k", ctypes.c_int64), ("ld", ctypes.c_int64),
                ("pattern", ctypes.c_int32), ("score", ctypes.c_int32),
                ("norms", ctypes.c_void_p), ("fmt", ctypes.c_int32), ("bits", ctypes.c_int32),
                ("group", ctypes.c_int32), ("pack4", ctypes.c_int32),
                ("tensor_scale_in", ctypes.c_void_p)]


class _Outputs(ctypes.Structure):
    _fields_ = [("values", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("tensor_scale", ctypes.c_void_p), ("meta", ctypes.c_void_p)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _lib.oracle_run.restype = ctypes.c_int
        _lib.oracle_run.argtypes = [ctypes.POINTER(_Args), ctypes.POINTER(_Outputs), ctypes.c_void_p]
        _lib.oracle_dequantize.restype = ctypes.c_int
        _lib.oracle_dequantize.argtypes = [ctypes.POINTER(_Args), ctypes.POINTER(_Outputs), ctypes.c_void_p]
        _lib.oracle_amax.restype = ctypes.c_float
        _lib.oracle_scale_tiles_bytes.restype = ctypes.c_int64
        _lib.oracle_scale_tiles_bytes.argtypes = [ctypes.c_int64, ctypes.c_int64]
        _lib.oracle_scale_tiles.restype = ctypes.c_int
        _lib.oracle_scale_tiles.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                            ctypes.c_void_p]
        _lib.oracle_hadamard_scale.restype = ctypes.c_float
        _lib.oracle_hadamard_scale.argtypes = [ctypes.c_int32]
        _lib.oracle_hadamard.restype = ctypes.c_int
        _lib.oracle_hadamard.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                         ctypes.c_int32, ctypes.c_void_p]
        _lib.oracle_exp_ss.restype = ctypes.c_float
        _lib.oracle_exp_ss.argtypes = [ctypes.c_float]
        _lib.oracle_softmax_bf16.restype = ctypes.c_int
        _lib.oracle_softmax_bf16.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                             ctypes.c_float, ctypes.c_void_p]
        _lib.oracle_softmax_f64_bf16.restype = ctypes.c_int
        _lib.oracle_softmax_f64_bf16.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                                 ctypes.c_float, ctypes.c_void_p]
        _lib.oracle_hadamard_bf16.restype = ctypes.c_int
        _lib.oracle_hadamard_bf16.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                              ctypes.c_int32, ctypes.c_void_p]
        _lib.oracle_amax.argtypes = [ctypes.POINTER(_Args)]
        _lib.oracle_tensor_scale.restype = ctypes.c_float
        _lib.oracle_tensor_scale.argtypes = [ctypes.POINTER(_Args)]
        _lib.oracle_scale_of_amax.restype = ctypes.c_float
        _lib.oracle_scale_of_amax.argtypes = [ctypes.c_float, ctypes.c_int32]
        _lib.oracle_select24.restype = ctypes.c_int
        _lib.oracle_select24.argtypes = [ctypes.c_void_p]
        _lib.oracle_select48.restype = ctypes.c_int
        _lib.oracle_select48.argtypes = [ctypes.c_void_p]
        _lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        _lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        _lib.oracle_e4m3_decode.restype = ctypes.c_float
        _lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        _lib.oracle_e2m1_encode.restype = ctypes.c_uint8
        _lib.oracle_e2m1_encode.argtypes = [ctypes.c_float]
        _lib.oracle_e2m1_decode.restype = ctypes.c_float
        _lib.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
        _lib.oracle_floor_log2.restype = ctypes.c_int
        _lib.oracle_floor_log2.argtypes = [ctypes.c_float]
        _lib.oracle_ratio.restype = None
        _lib.oracle_ratio.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        _lib.oracle_bits_per_element.restype = ctypes.c_double
        _lib.oracle_bits_per_element.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                                 ctypes.c_int32, ctypes.c_int64, ctypes.c_int32]
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


def _make_args(x, dtype, rows, k, ld, axis, pattern, score, norms, fmt, bits, group, pack4, scale_arr):
    return _Args(_ptr(x), dtype, axis, rows, k, ld, pattern, score, _ptr(norms), fmt, bits, group,
                 pack4, _ptr(scale_arr))


def _operand_shape(x, axis, rows, k, ld):
    """Infer (rows, k, ld) of the logical operand A[rows][k] from a 2-D array."""
    if axis == 1:
        r, kk = x.shape
        return (rows if rows is not None else r), (k if k is not None else kk), (ld if ld is not None else kk)
    kk, r = x.shape  # axis 0: stored [k][rows]
    return (rows if rows is not None else r), (k if k is not None else kk), (ld if ld is not None else r)


def run(x, *, pattern=SPARSE_24, score=MAG, norms=None, fmt="none", bits=8, group=0, pack4=False,
        tensor_scale=None, axis=1, rows=None, k=None, ld=None):
    """Run the oracle pass. ``x`` is a 2-D uint16 (bf16 bits) or float32 array,
    stored [rows][ld] (axis 1) or [k][ld] (axis 0). Returns a dict with the
    outputs that the format produces and ``energy`` = [E_total, E_prune, E_q, E_q_dense]."""
    x = np.ascontiguousarray(x)
    dtype = BF16 if x.dtype == np.uint16 else F32
    if dtype == F32 and x.dtype != np.float32:
        raise TypeError("x must be uint16 (bf16 bits) or float32")
    rows, k, ld = _operand_shape(x, axis, rows, k, ld)
    fmt_id = _FMT_NAMES[fmt] if isinstance(fmt, str) else fmt
    n = k if pattern == DENSE else k // 2
    if norms is not None:
        norms = np.ascontiguousarray(norms, dtype=np.float32)
    out = {}
    if fmt_id == FMT_NONE:
        out["values"] = np.zeros((rows, n), dtype=x.dtype)
    elif fmt_id == FMT_FP8:
        out["values"] = np.zeros((rows, n), dtype=np.uint8)
    elif fmt_id == FMT_INT:
        if pack4:
            out["values"] = np.zeros((rows, n // 2), dtype=np.uint8)
        else:
            out["values"] = np.zeros((rows, n), dtype=np.int16 if bits > 8 else np.int8)
        g = group if group else n
        out["scales"] = np.zeros((rows, n // g), dtype=np.float32)
    elif fmt_id == FMT_NVFP4:
        out["values"] = np.zeros((rows, n // 2), dtype=np.uint8)
        out["scales"] = np.zeros((rows, n // 16), dtype=np.uint8)
    elif fmt_id == FMT_MXFP4:
        out["values"] = np.zeros((rows, n // 2), dtype=np.uint8)
        out["scales"] = np.zeros((rows, n // 32), dtype=np.uint8)
    if fmt_id in (FMT_FP8, FMT_NVFP4):
        out["tensor_scale"] = np.zeros(1, dtype=np.float32)
    if pattern != DENSE:
        out["meta"] = np.zeros((rows, k // (16 if pattern == SPARSE_48 else 8)), dtype=np.uint8)
    scale_arr = None if tensor_scale is None else np.array([tensor_scale], dtype=np.float32)
    args = _make_args(x, dtype, rows, k, ld, axis, pattern, score, norms, fmt_id, bits, group,
                      int(pack4), scale_arr)
    outs = _Outputs(_ptr(out.get("values")), _ptr(out.get("scales")), _ptr(out.get("tensor_scale")),
                    _ptr(out.get("meta")))
    energy = np.zeros(4, dtype=np.float64)
    rc = lib().oracle_run(ctypes.byref(args), ctypes.byref(outs), energy.ctypes.data)
    if rc != 0:
        raise ValueError(f"oracle_run rejected its arguments (code {rc})")
    out["energy"] = energy
    return out


def dequantize(out, *, rows, k, pattern=SPARSE_24, fmt="none", bits=8, group=0, pack4=False, dtype=BF16):
    """The dense float32 operand [rows][k] that the outputs of a pass (a dict as
    run() returns it) stand for: dequantized values on kept positions, zero on
    dropped ones."""
    fmt_id = _FMT_NAMES[fmt] if isinstance(fmt, str) else fmt
    dummy = np.zeros(1, dtype=np.uint16 if dtype == BF16 else np.float32)
    args = _make_args(dummy, dtype, rows, k, k, 1, pattern, MAG, None, fmt_id, bits, group, int(pack4), None)
    keep = {key: np.ascontiguousarray(out[key]) for key in ("values", "scales", "tensor_scale", "meta") if key in out}
    outs = _Outputs(_ptr(keep.get("values")), _ptr(keep.get("scales")), _ptr(keep.get("tensor_scale")),
                    _ptr(keep.get("meta")))
    xhat = np.zeros((rows, k), dtype=np.float32)
    if lib().oracle_dequantize(ctypes.byref(args), ctypes.byref(outs), xhat.ctypes.data) != 0:
        raise ValueError("oracle_dequantize rejected its arguments")
    return xhat


def amax(x, *, pattern=SPARSE_24, score=MAG, norms=None, axis=1, rows=None, k=None, ld=None):
    """Largest |value| among the values a pass would quantize (kept, or all when dense)."""
    x = np.ascontiguousarray(x)
    dtype = BF16 if x.dtype == np.uint16 else F32
    rows, k, ld = _operand_shape(x, axis, rows, k, ld)
    if norms is not None:
        norms = np.ascontiguousarray(norms, dtype=np.float32)
    args = _make_args(x, dtype, rows, k, ld, axis, pattern, score, norms, FMT_NONE, 8, 0, 0, None)
    return float(lib().oracle_amax(ctypes.byref(args)))


def tensor_scale(x, fmt, *, pattern=SPARSE_24, score=MAG, norms=None, axis=1, rows=None, k=None, ld=None):
    """The per-tensor scale (FP8: amax / 448, NVFP4: amax / 2688) a pass over the
    whole operand derives when none is given."""
    x = np.ascontiguousarray(x)
    dtype = BF16 if x.dtype == np.uint16 else F32
    rows, k, ld = _operand_shape(x, axis, rows, k, ld)
    if norms is not None:
        norms = np.ascontiguousarray(norms, dtype=np.float32)
    fmt_id = _FMT_NAMES[fmt] if isinstance(fmt, str) else fmt
    args = _make_args(x, dtype, rows, k, ld, axis, pattern, score, norms, fmt_id, 8, 0, 0, None)
    return float(lib().oracle_tensor_scale(ctypes.byref(args)))


def host_threads():
    """Host cores this process may run on (the thread count of run_parallel)."""
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        return os.cpu_count() or 1


def _row_blocks(rows, threads, block_rows):
    if block_rows is None:
        block_rows = max(1, -(-rows // (4 * threads)))
    return [(r0, min(rows, r0 + block_rows)) for r0 in range(0, rows, block_rows)]


def run_parallel(x, *, threads=None, block_rows=None, pattern=SPARSE_24, score=MAG, norms=None, fmt="none",
                 bits=8, group=0, pack4=False, tensor_scale=None):
    """run() on host threads: the rows of an axis-1 operand x [rows][k] cut into
    contiguous blocks, each block one run() call (the C oracle, which releases
    the interpreter lock while it runs). Each row's outputs depend on that row
    alone once the tensor scale is fixed, so the blocks' outputs, concatenated,
    are run()'s outputs on the whole operand. A per-tensor scale that is not
    given is derived first, exactly as run() derives it: the amax of every
    block (amax(), an exact maximum), their maximum, then scale_of_amax. The
    energies are the blocks' binary64 sums added in block order (run() adds
    the same terms in row order: equal up to the order of binary64 additions).
    Returns run()'s dict."""
    from concurrent.futures import ThreadPoolExecutor
    x = np.ascontiguousarray(x)
    rows = x.shape[0]
    threads = threads or host_threads()
    blocks = _row_blocks(rows, threads, block_rows)
    fmt_id = _FMT_NAMES[fmt] if isinstance(fmt, str) else fmt
    with ThreadPoolExecutor(max_workers=threads) as ex:
        if fmt_id in (FMT_FP8, FMT_NVFP4) and tensor_scale is None:
            am = list(ex.map(lambda b: amax(x[b[0]:b[1]], pattern=pattern, score=score, norms=norms), blocks))
            tensor_scale = float(lib().oracle_scale_of_amax(max(am) if am else 0.0, fmt_id))
        parts = list(ex.map(lambda b: run(x[b[0]:b[1]], pattern=pattern, score=score, norms=norms, fmt=fmt,
                                          bits=bits, group=group, pack4=pack4, tensor_scale=tensor_scale),
                            blocks))
    if not parts:
        return run(x, pattern=pattern, score=score, norms=norms, fmt=fmt, bits=bits, group=group, pack4=pack4,
                   tensor_scale=tensor_scale)
    out = {}
    for key in parts[0]:
        if key == "energy":
            e = np.zeros(4, dtype=np.float64)
            for p in parts:
                e += p["energy"]
            out[key] = e
        elif key == "tensor_scale":
            out[key] = parts[0][key]
        else:
            out[key] = np.concatenate([p[key] for p in parts], axis=0)
    return out


def scale_of_amax(a, fmt):
    """The per-tensor scale of an amax (FP8: a / 448, NVFP4: a / 2688)."""
    return float(lib().oracle_scale_of_amax(float(a), _FMT_NAMES[fmt] if isinstance(fmt, str) else fmt))


def select24(s):
    s = np.ascontiguousarray(s, dtype=np.float32)
    return lib().oracle_select24(s.ctypes.data)


def select48(s):
    s = np.ascontiguousarray(s, dtype=np.float32)
    return lib().oracle_select48(s.ctypes.data)


def e4m3_encode(v):
    return lib().oracle_e4m3_encode(float(v))


def e4m3_decode(c):
    return lib().oracle_e4m3_decode(int(c))


def e2m1_encode(v):
    return lib().oracle_e2m1_encode(float(v))


def e2m1_decode(c):
    return lib().oracle_e2m1_decode(int(c))


def floor_log2(a):
    return lib().oracle_floor_log2(float(a))


def hadamard(x, block):
    """Block Hadamard rotation along k (see oracle_hadamard) of an operand given
    as bf16 bits (uint16) or float32, [rows, k] or [batch, rows, k]: float32 of
    the same shape."""
    a = np.asarray(x)
    if a.dtype == np.uint16:
        f = (a.astype(np.uint32) << 16).view(np.float32)   # bf16 bits widened exactly
    else:
        f = a.astype(np.float32)
    f = np.ascontiguousarray(f, dtype=np.float32)
    k = f.shape[-1]
    rows = f.size // k if k else 0
    out = np.empty_like(f)
    if f.size and lib().oracle_hadamard(f.ctypes.data, rows, k, k, int(block), out.ctypes.data) != 0:
        raise ValueError("oracle_hadamard rejected its arguments")
    return out


def hadamard_bf16(x, block):
    """The rotation as a fused pass applies it (see oracle_hadamard_bf16): bf16
    bits of the same shape as x (bf16 bits or float32, [rows, k] or [B, rows, k])."""
    a = np.asarray(x)
    f = (a.astype(np.uint32) << 16).view(np.float32) if a.dtype == np.uint16 else a.astype(np.float32)
    f = np.ascontiguousarray(f, dtype=np.float32)
    k = f.shape[-1]
    out = np.empty(f.shape, dtype=np.uint16)
    if f.size and lib().oracle_hadamard_bf16(f.ctypes.data, f.size // k, k, k, int(block), out.ctypes.data) != 0:
        raise ValueError("oracle_hadamard_bf16 rejected its arguments")
    return out


def softmax_bf16(s, alpha):
    """P = softmax(alpha * s) per row as bf16 bits (see oracle_softmax_bf16) of
    logits given as bf16 bits (uint16) or float32, [rows, k] or [batch, rows, k]."""
    a = np.asarray(s)
    f = (a.astype(np.uint32) << 16).view(np.float32) if a.dtype == np.uint16 else a.astype(np.float32)
    f = np.ascontiguousarray(f, dtype=np.float32)
    k = f.shape[-1]
    rows = f.size // k
    out = np.empty(f.shape, dtype=np.uint16)
    if lib().oracle_softmax_bf16(f.ctypes.data, rows, k, k, float(alpha), out.ctypes.data) != 0:
        raise ValueError("oracle_softmax_bf16 rejected its arguments")
    return out


def softmax_f64_bf16(s, alpha, threads=1):
    """P = softmax(alpha * s) per row from the plain definition in binary64
    (libm exp, index-order sum), rounded once to bf16 (see
    oracle_softmax_f64_bf16): bf16 bits of the same shape as the logits (bf16
    bits or float32, [rows, k] or [batch, rows, k]). threads > 1 runs row
    blocks on host threads (each row depends on itself alone)."""
    a = np.asarray(s)
    f = (a.astype(np.uint32) << 16).view(np.float32) if a.dtype == np.uint16 else a.astype(np.float32)
    f = np.ascontiguousarray(f, dtype=np.float32)
    k = f.shape[-1]
    rows = f.size // k
    out = np.empty(f.shape, dtype=np.uint16)
    f2, o2 = f.reshape(rows, k), out.reshape(rows, k)

    def block(b):
        r0, r1 = b
        if lib().oracle_softmax_f64_bf16(f2[r0:r1].ctypes.data, r1 - r0, k, k, float(alpha),
                                         o2[r0:r1].ctypes.data) != 0:
            raise ValueError("oracle_softmax_f64_bf16 rejected its arguments")

    blocks = _row_blocks(rows, threads, None)
    if threads > 1:
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(block, blocks))
    else:
        for b in blocks:
            block(b)
    return out


def scale_tiles(scales, rows, cols, batch=1):
    """Scale bytes [batch, rows, cols] (or [rows, cols]) in the block-scaled MMA's
    128 x 4 tile layout (see oracle_scale_tiles): uint8[batch * tiles_bytes]."""
    src = np.ascontiguousarray(scales, dtype=np.uint8).reshape(-1)
    if src.size != batch * rows * cols:
        raise ValueError("scales do not hold batch * rows * cols bytes")
    per = lib().oracle_scale_tiles_bytes(rows, cols)
    out = np.empty(batch * per, dtype=np.uint8)
    if lib().oracle_scale_tiles(src.ctypes.data if src.size else None, rows, cols, batch, out.ctypes.data) != 0:
        raise ValueError("oracle_scale_tiles rejected its arguments")
    return out


def ratio(sparse_energy, dense_energy):
    """[loss, rel_err_sparse, rel_err_dense, R_hat] from two energy vectors."""
    s = np.ascontiguousarray(sparse_energy, dtype=np.float64)
    d = np.ascontiguousarray(dense_energy, dtype=np.float64)
    out = np.zeros(4, dtype=np.float64)
    lib().oracle_ratio(s.ctypes.data, d.ctypes.data, out.ctypes.data)
    return out


def bits_per_element(fmt, bits=8, group=0, pattern=SPARSE_24, k=4096, with_scales=False):
    fmt_id = _FMT_NAMES[fmt] if isinstance(fmt, str) else fmt
    return lib().oracle_bits_per_element(fmt_id, bits, group, pattern, k, int(with_scales))
