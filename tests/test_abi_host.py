"""Host-side checks of the C ABI: the library loads, exports every function the
header declares, and rejects invalid arguments before touching the GPU.
No test here launches a kernel."""
import ctypes
import os
import re

import pytest

import oracle
from semi_structured_sparsity_online_b200 import ss24

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "ss24.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return sorted(set(re.findall(r"\b(ss24_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert len(names) >= 19
    L = ss24.lib()
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(ss24._SIGNATURES)


def test_workspace_bytes_and_status_strings():
    assert ss24.lib().ss24_workspace_bytes() >= 256 + 32 * 1024
    for s in range(9):
        assert ss24.status_string(s)
    assert ss24.status_string(99) == "unknown status"


def test_bits_per_element_matches_oracle_accounting():
    for fmt, bits, group in [("none", 16, 0), ("fp8", 8, 0), ("int", 3, 0), ("int", 8, 128), ("int", 16, 64),
                             ("nvfp4", 4, 0), ("mxfp4", 4, 0)]:
        for pattern in (ss24.DENSE, ss24.SPARSE_24, ss24.SPARSE_48):
            for ws in (False, True):
                a = ss24.bits_per_element(fmt, bits, group, pattern, 4096, ws)
                b = oracle.bits_per_element(fmt, bits, group, pattern, 4096, ws)
                assert a == b, (fmt, bits, group, pattern, ws)
    # equal-bit identity: 2:4 on 2m bits == dense m+1 bits
    for m in range(1, 9):
        assert ss24.bits_per_element("int", 2 * m) == ss24.bits_per_element("int", m + 1, pattern=ss24.DENSE)
    assert ss24.bits_per_element("int", 1) < 0


# Fake, never-dereferenced pointer values: every call below fails validation,
# so nothing is launched and no pointer is read.
ALIGNED = 0x7F0000000000
MISALIGNED = ALIGNED + 8
WS_BYTES = None


def _ws_bytes():
    return ss24.lib().ss24_workspace_bytes()


def op(x=ALIGNED, dtype=ss24.BF16, axis=1, rows=16, k=64, ld=64, batch=0, batch_stride=0):
    return ss24.Operand(x, dtype, axis, rows, k, ld, batch, batch_stride)


def outs(values=ALIGNED, scales=ALIGNED, tscale=ALIGNED, meta=ALIGNED):
    return ss24.Outputs(values, scales, tscale, meta)


def fused(o, fmt=None, ws=ALIGNED, ws_bytes=None, score=ss24.MAG, norms=None, out=None):
    fmt = fmt or ss24.make_format("nvfp4")
    out = out or outs()
    return ss24.lib().ss24_prune24_quant_fused(ctypes.byref(o) if o is not None else None, score, norms, fmt,
                                               None, ctypes.byref(out), None, ws,
                                               _ws_bytes() if ws_bytes is None else ws_bytes, None)


@pytest.mark.parametrize("case,expected", [
    ("null_operand", 1), ("null_x", 1), ("bad_dtype", 4), ("bad_axis", 8), ("neg_rows", 2), ("zero_k", 2),
    ("ld_lt_k", 2), ("misaligned_x", 3), ("odd_ld", 3), ("k_not_mult8", 2), ("nvfp4_k", 2),
    ("bad_kind", 5), ("int_bits", 5), ("int_pack4", 5), ("int_group_np2", 5), ("int_group_big", 5),
    ("ws_null", 6), ("ws_small", 6), ("ws_misaligned", 6), ("null_values", 1), ("null_meta", 1),
    ("null_scales", 1), ("null_tscale", 1), ("wanda_no_norms", 1), ("wanda_misaligned_norms", 3),
    ("bad_score", 8), ("misaligned_values", 3), ("neg_batch", 2), ("huge_batch", 2), ("overlapping_batch", 2),
    ("misaligned_batch_stride", 3),
])
def test_validation_rejects_before_launch(case, expected):
    f = None
    o = op()
    kw = {}
    if case == "null_operand":
        o = None
    elif case == "null_x":
        o = op(x=0)
    elif case == "bad_dtype":
        o = op(dtype=7)
    elif case == "bad_axis":
        o = op(axis=2)
    elif case == "neg_rows":
        o = op(rows=-1)
    elif case == "zero_k":
        o = op(k=0)
    elif case == "ld_lt_k":
        o = op(ld=32)
    elif case == "misaligned_x":
        o = op(x=MISALIGNED)
    elif case == "odd_ld":
        o = op(ld=68 + 1)
    elif case == "k_not_mult8":
        o = op(k=60, ld=64)
    elif case == "nvfp4_k":
        o = op(k=48, ld=64)
    elif case == "bad_kind":
        f = ss24.Format(9, 8, 0, 0)
    elif case == "int_bits":
        f = ss24.make_format("int", 17)
    elif case == "int_pack4":
        f = ss24.make_format("int", 8, 0, True)
    elif case == "int_group_np2":
        f = ss24.make_format("int", 8, 24)
    elif case == "int_group_big":
        f = ss24.make_format("int", 8, 256)
    elif case == "ws_null":
        kw["ws"] = None
    elif case == "ws_small":
        kw["ws_bytes"] = 64
    elif case == "ws_misaligned":
        kw["ws"] = ALIGNED + 16
    elif case == "null_values":
        kw["out"] = outs(values=0)
    elif case == "null_meta":
        kw["out"] = outs(meta=0)
    elif case == "null_scales":
        kw["out"] = outs(scales=0)
    elif case == "null_tscale":
        kw["out"] = outs(tscale=0)
    elif case == "wanda_no_norms":
        kw["score"] = ss24.WANDA
    elif case == "wanda_misaligned_norms":
        kw["score"] = ss24.WANDA
        kw["norms"] = MISALIGNED
    elif case == "bad_score":
        kw["score"] = 5
    elif case == "misaligned_values":
        kw["out"] = outs(values=MISALIGNED)
    elif case == "neg_batch":
        o = op(batch=-1)
    elif case == "huge_batch":
        o = op(batch=1025, batch_stride=16 * 64)
    elif case == "overlapping_batch":
        o = op(batch=2, batch_stride=16 * 64 - 8)
    elif case == "misaligned_batch_stride":
        o = op(batch=2, batch_stride=16 * 64 + 4)
    assert fused(o, f, **kw) == expected


def test_other_entry_points_validate():
    L = ss24.lib()
    o = op()
    out = outs()
    wsb = _ws_bytes()
    assert L.ss24_quantize_fp8(ctypes.byref(op(k=12, ld=16)), None, ctypes.byref(out), None, ALIGNED, wsb, None) == 2
    assert L.ss24_quantize_int(ctypes.byref(o), ss24.make_format("fp8"), ctypes.byref(out), None, ALIGNED, wsb,
                               None) == 5
    assert L.ss24_quantize_nvfp4(ctypes.byref(op(k=8, ld=8)), None, ctypes.byref(out), None, ALIGNED, wsb,
                                 None) == 2
    assert L.ss24_quantize_mxfp4(ctypes.byref(op(k=16, ld=16)), ctypes.byref(out), None, ALIGNED, wsb, None) == 2
    assert L.ss24_prune24_compress(ctypes.byref(o), ss24.MAG, None, ALIGNED, None, None, ALIGNED, wsb, None) == 1
    assert L.ss24_prune48_pairwise_quant_fused(ctypes.byref(op(k=24, ld=24)), ss24.MAG, None,
                                               ss24.make_format("none"), None, ctypes.byref(out), None, ALIGNED,
                                               wsb, None) == 2
    assert L.ss24_error_energy(ctypes.byref(o), ss24.DENSE, ss24.MAG, None, ss24.make_format("none"),
                               ss24.make_format("int", 5), None, None, ALIGNED, ALIGNED, wsb, None) == 8
    assert L.ss24_error_energy(ctypes.byref(o), ss24.SPARSE_24, ss24.MAG, None, ss24.make_format("none"),
                               ss24.make_format("none"), None, None, ALIGNED, ALIGNED, wsb, None) == 5
    assert L.ss24_error_energy(ctypes.byref(o), ss24.SPARSE_24, ss24.MAG, None, ss24.make_format("none"),
                               ss24.make_format("int", 5), None, None, None, ALIGNED, wsb, None) == 1
    assert L.ss24_amax(ctypes.byref(o), ss24.SPARSE_24, ss24.MAG, None, None, ALIGNED, wsb, None) == 1
    assert L.ss24_amax_rows(ctypes.byref(o), ss24.DENSE, ss24.MAG, None, None, 0, None, ALIGNED, wsb, None) == 1
    assert L.ss24_amax_rows(ctypes.byref(o), ss24.DENSE, ss24.MAG, None, ALIGNED, 2, ALIGNED, ALIGNED, wsb,
                            None) == 5                                        # INT has no tensor scale
    assert L.ss24_amax_rows(ctypes.byref(op(axis=0)), ss24.DENSE, ss24.MAG, None, ALIGNED, 0, None, ALIGNED, wsb,
                            None) == 8
    assert L.ss24_quantize_int_rows(ctypes.byref(o), ss24.DENSE, ss24.MAG, None, ss24.make_format("int", 8, 32),
                                    ALIGNED, ctypes.byref(out), None, ALIGNED, wsb, None) == 5   # group must be 0
    assert L.ss24_quantize_int_rows(ctypes.byref(o), ss24.DENSE, ss24.MAG, None, ss24.make_format("int", 8, 0),
                                    None, ctypes.byref(out), None, ALIGNED, wsb, None) == 1
    assert L.ss24_quantize_int_rows(ctypes.byref(op(axis=0)), ss24.DENSE, ss24.MAG, None,
                                    ss24.make_format("int", 8, 0), ALIGNED, ctypes.byref(out), None, ALIGNED, wsb,
                                    None) == 8
    assert L.ss24_predicted_ratio(None, ALIGNED, ALIGNED, 1, None) == 1
    assert L.ss24_predicted_ratio(ALIGNED, ALIGNED, ALIGNED, -1, None) == 2
    assert L.ss24_selfcheck_division(3, 0, 1, ALIGNED, None) == 8
    assert L.ss24_selfcheck_encoder(1, None, 126, 0, 1, ALIGNED, None) == 1            # null table
    assert L.ss24_selfcheck_encoder(2, ALIGNED, 126, 0, 1, ALIGNED, None) == 5         # INT: no encoder
    assert L.ss24_selfcheck_encoder(1, ALIGNED, 7, 0, 1, ALIGNED, None) == 2           # E4M3 wants 126
    assert L.ss24_selfcheck_encoder(3, ALIGNED, 7, 65535, 2, ALIGNED, None) == 2       # hi range
    assert L.ss24_selfcheck_division(2, 1 << 15, 1, ALIGNED, None) == 2
    assert L.ss24_selfcheck_division(2, 100, (1 << 15) - 99, ALIGNED, None) == 2
    assert L.ss24_selfcheck_division(0, 1 << 23, 1, ALIGNED, None) == 2
    assert L.ss24_selfcheck_division(0, 0, 1, None, None) == 1
    assert L.ss24_encode_e4m3(None, None, 5, None) == 1
    assert L.ss24_decode_e2m1(ALIGNED, ALIGNED, -1, None) == 2
    assert L.ss24_workspace_init(None, wsb, None) == 6
    assert L.ss24_workspace_error(None, None, None) == 1


def test_scale_tiles_validation():
    L = ss24.lib()
    assert L.ss24_scale_tiles_bytes(130, 5) == oracle.lib().oracle_scale_tiles_bytes(130, 5) == 2048
    assert L.ss24_scale_tiles_bytes(0, 5) == 0 and L.ss24_scale_tiles_bytes(5, 0) == 0
    assert L.ss24_scale_tiles_bytes(-1, 5) == -1
    assert L.ss24_scale_tiles(None, -1, 4, 0, ALIGNED, None) == 2          # SS24_ERR_SHAPE
    assert L.ss24_scale_tiles(ALIGNED, 4, 4, 1025, ALIGNED, None) == 2     # batch beyond 1024
    assert L.ss24_scale_tiles(None, 4, 4, 0, ALIGNED, None) == 1           # SS24_ERR_NULL
    assert L.ss24_scale_tiles(ALIGNED, 4, 4, 0, None, None) == 1
    assert L.ss24_scale_tiles(ALIGNED, 4, 4, 0, MISALIGNED, None) == 3     # SS24_ERR_ALIGN
    assert L.ss24_scale_tiles(None, 0, 4, 0, None, None) == 0              # empty: nothing to write


def test_hadamard_validation():
    L = ss24.lib()

    def op(rows=4, k=64, ld=None, axis=1, ptr=ALIGNED, dtype=ss24.BF16):
        return ss24.Operand(ptr, dtype, axis, rows, k, ld or k, 0, 0)
    call = lambda o, b, out=ALIGNED: L.ss24_hadamard(ctypes.byref(o), b, out, None)
    assert call(op(), 3) == 8 and call(op(), 1) == 8 and call(op(), 512) == 8       # SS24_ERR_ARG
    assert call(op(axis=0, ld=8), 16) == 8
    assert call(op(k=48), 32) == 2                                                 # k % block
    assert call(op(k=4, ld=8), 2) == 2                                             # k % 8
    assert call(op(), 16, None) == 1                                               # SS24_ERR_NULL
    assert call(op(), 16, MISALIGNED) == 3                                         # SS24_ERR_ALIGN
    assert call(op(rows=0, ptr=None), 16, None) == 0                               # empty operand


def test_softmax_prune_validation():
    L = ss24.lib()
    ws = ctypes.c_void_p(ALIGNED)

    def op(rows=4, k=512, ld=None, axis=1, ptr=ALIGNED, dtype=ss24.BF16):
        return ss24.Operand(ptr, dtype, axis, rows, k, ld or k, 0, 0)
    outs = ss24.Outputs(ALIGNED, ALIGNED, ALIGNED, ALIGNED)

    def call(o, alpha=0.1, pattern=ss24.SPARSE_24, fmt=("fp8",), scale=ALIGNED, wsb=None):
        f = ss24.make_format(*fmt)
        return L.ss24_softmax_prune(ctypes.byref(o), alpha, pattern, f, scale, ctypes.byref(outs), None, ws,
                                    wsb if wsb is not None else _ws_bytes(), None)
    assert call(op(axis=0, ld=8)) == 8                           # SS24_ERR_ARG: axis 0
    assert call(op(), alpha=float("nan")) == 8                   # alpha not finite
    assert call(op(k=264)) == 2                                  # SS24_ERR_SHAPE: keys % 256
    assert call(op(), fmt=("int", 8, 0)) == 5                    # SS24_ERR_FORMAT: one INT scale per row
    assert call(op(), fmt=("fp8",), scale=None) == 1             # SS24_ERR_NULL: FP8 needs the given scale
    assert call(op(), fmt=("none",), pattern=ss24.DENSE) == 5    # dense needs a quantization format
    assert call(op(), wsb=16) == 6                               # SS24_ERR_WORKSPACE


def test_rotated_operand_validation():
    """The operand's hadamard field: checked before anything is launched."""
    L = ss24.lib()
    ws = ctypes.c_void_p(ALIGNED)
    outs = ss24.Outputs(ALIGNED, ALIGNED, ALIGNED, ALIGNED)

    def op(rows=4, k=1024, ld=None, axis=1, dtype=ss24.BF16, had=16):
        return ss24.Operand(ALIGNED, dtype, axis, rows, k, ld or k, 0, 0, had, 0)

    def fused(o, score=ss24._SCORE["mag"], fmt=("fp8",)):
        return L.ss24_prune24_quant_fused(ctypes.byref(o), score, ALIGNED, ss24.make_format(*fmt), ALIGNED,
                                          ctypes.byref(outs), None, ws, _ws_bytes(), None)
    assert fused(op(had=3)) == 8 and fused(op(had=512)) == 8 and fused(op(had=1)) == 8   # SS24_ERR_ARG
    assert fused(op(dtype=ss24.F32)) == 8                                                # bf16 only
    assert fused(op(axis=0, ld=8)) == 8                                                  # axis 1 only
    assert fused(op(k=1040, had=32)) == 2                                                # SS24_ERR_SHAPE: k % block
    assert fused(op(), score=ss24._SCORE["wanda"]) == 8                                  # magnitude only
    assert L.ss24_quantize_int(ctypes.byref(op(k=4096)), ss24.make_format("int", 8, 0), ctypes.byref(outs), None,
                               ws, _ws_bytes(), None) == 8                               # the row-block INT pass
    assert L.ss24_hadamard(ctypes.byref(op()), 16, ALIGNED, None) == 8                   # no second rotation
    assert L.ss24_softmax_prune(ctypes.byref(op(k=1024)), 0.1, ss24.SPARSE_24, ss24.make_format("fp8"), ALIGNED,
                                ctypes.byref(outs), None, ws, _ws_bytes(), None) == 8


def test_algorithmic_bytes_match_the_stored_layouts():
    """The bytes the benchmark and run_case count per launch, from the layouts:
    input 2 bytes per bf16 element; FP8 codes 1 byte per stored value; metadata
    1/8 byte per element (2:4) or 1/16 (4:8); E4M3 block scales 1 byte per 16
    stored values, E8M0 per 32; INT scales 4 bytes per group or row; packed
    INT4 / INT3 codes half a byte per stored value."""
    import bench
    import run_case
    m = k = 4096
    n = m * k
    pb = run_case.pass_bytes
    assert pb("fused_24_fp8", m, k) == 2 * n + n // 2 + n // 8 == 44_040_192
    assert pb("dense_fp8", m, k) == 3 * n == 50_331_648
    assert pb("fused_24_none", m, k) == 2 * n + n + n // 8 == 52_428_800
    assert pb("fused_24_nvfp4", m, k) == 2 * n + n // 4 + n // 32 + n // 8 == 40_370_176
    assert pb("fused_24_mxfp4", m, k) == 2 * n + n // 4 + n // 64 + n // 8 == 40_108_032
    assert pb("fused_48_nvfp4", m, k) == 2 * n + n // 4 + n // 32 + n // 16 == 39_321_600
    assert pb("fused_24_int8g128", m, k) == 2 * n + n // 2 + 4 * (n // 2 // 128) + n // 8 == 44_302_336
    assert pb("dense_nvfp4", m, k) == 2 * n + n // 2 + n // 16 == 42_991_616
    assert pb("hadamard128", m, k) == 6 * n
    assert pb("softmax_24_fp8", m, k) == pb("fused_24_fp8", m, k)
    ab = bench.pass_bytes()
    ns = bench.SWEEP_M * bench.SWEEP_K
    assert ab["sweep_fused_24_nvfp4"] == pb("fused_24_nvfp4", bench.SWEEP_M, bench.SWEEP_K) == 565_182_464
    assert ab["sweep_fused_48_nvfp4"] == pb("fused_48_nvfp4", bench.SWEEP_M, bench.SWEEP_K)
    assert ab["sweep_compress_24"] == pb("fused_24_none", bench.SWEEP_M, bench.SWEEP_K)
    assert ab["sweep_dense_nvfp4"] == pb("dense_nvfp4", bench.SWEEP_M, bench.SWEEP_K)
    assert ab["sweep_scale"] == 2 * ns
    assert ab["linear_fused_24_fp8"] == 8 * pb("fused_24_fp8", m, k)
    assert ab["linear_dense_fp8"] == 8 * pb("dense_fp8", m, k)
    assert ab["linear_dense_int8_row"] == 8 * (2 * n + 4 * m + n + 4 * m)
    nw = bench.W_M * bench.W_K
    assert ab["weight_wanda_24_int4"] == 2 * nw + 4 * bench.W_K + nw // 4 + 4 * (nw // 256) + nw // 8
    assert ab["weight_dense_int3"] == 2 * nw + nw // 2 + 4 * (nw // 128)


def test_bench_traffic_is_tied_to_the_kernel_sources(tmp_path, monkeypatch):
    """The bench reports a kernel's ncu DRAM bytes only while the kernel
    sources hash to the value recorded beside them: any change to a source
    makes the figure stale, and the bench reports none."""
    import json
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    src = tmp_path / "semi_structured_sparsity_online_b200" / "csrc"
    src.mkdir(parents=True)
    (src / "a.cu").write_text("kernel a")
    (src / "b.cuh").write_text("header b")
    (src / "notes.txt").write_text("not a source")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    sha = bench.kernel_source_sha()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"source_sha": sha, "sweep_fused_24_nvfp4": 123}))
    assert bench.measured_traffic("sweep_fused_24_nvfp4") == 123
    assert bench.measured_traffic("sweep_dense_nvfp4") is None
    (src / "notes.txt").write_text("edited, still not a source")
    assert bench.measured_traffic("sweep_fused_24_nvfp4") == 123
    (src / "b.cuh").write_text("header b, changed")
    assert bench.measured_traffic("sweep_fused_24_nvfp4") is None
