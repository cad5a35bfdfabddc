"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs. Codes, scales, metadata and kept values must match bit for
bit; energies to 1e-6 relative (the bound the library states for its binary32
per-element terms summed in binary64)."""
import math

import numpy as np
import pytest
import torch

import oracle
from semi_structured_sparsity_online_b200 import synth

pytestmark = pytest.mark.gpu

RTOL = 1e-6


@pytest.fixture(scope="module")
def ss():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from semi_structured_sparsity_online_b200 import ss24
    ss24.lib()
    return ss24


@pytest.fixture(scope="module")
def ws(ss):
    return ss.Workspace()


def to_dev(a):
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(a).cuda()


def to_np(t):
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def bits_equal(a, b):
    a = np.ascontiguousarray(a)
    b = np.ascontiguousarray(b)
    if a.dtype == np.float32:
        return a.shape == b.shape and np.array_equal(a.view(np.uint32), b.view(np.uint32))
    return a.shape == b.shape and np.array_equal(a, b)


def assert_same(got, ref, what):
    if not bits_equal(got, ref):
        bad = np.argwhere(np.asarray(got) != np.asarray(ref))
        raise AssertionError(f"{what}: {len(bad)} mismatches, first at {bad[:3].tolist()}: "
                             f"gpu {np.asarray(got)[tuple(bad[0])] if len(bad) else None} "
                             f"oracle {np.asarray(ref)[tuple(bad[0])] if len(bad) else None}")


def assert_energy(got, ref, fields=(0, 1, 2, 3), atol=0.0):
    g = got.cpu().numpy()
    for f in fields:
        assert abs(g[f] - ref[f]) <= RTOL * abs(ref[f]) + atol, (f, g[f], ref[f])


def compare(ss, ws, xh, *, pattern, fmt, bits=8, group=0, pack4=False, score="mag", norms=None,
            tensor_scale=None, k=None, axis=1, rows=None):
    """Run both sides on the host array xh and compare: axis 1, xh is [rows][ld]
    (k <= ld); axis 0, xh is [k][ld] holding A[r][c] at xh[c][r] (rows <= ld)."""
    x = to_dev(xh)
    if axis == 1 and k is not None and k != xh.shape[1]:
        xd = x[:, :k]
    elif axis == 0 and rows is not None and rows != xh.shape[1]:
        xd = x[:, :rows]
    else:
        xd = x
    nd = to_dev(norms) if norms is not None else None
    sd = torch.tensor([tensor_scale], dtype=torch.float32, device="cuda") if tensor_scale is not None else None
    opat = {0: oracle.DENSE, 24: oracle.SPARSE_24, 48: oracle.SPARSE_48}[pattern]
    out = ss.run(xd, pattern=pattern, fmt=fmt, bits=bits, group=group, pack4=pack4, score=score, col_norms=nd,
                 tensor_scale=sd, ws=ws, axis=axis)
    torch.cuda.synchronize()
    ref = oracle.run(xh, pattern=opat, fmt=fmt, bits=bits, group=group, pack4=pack4,
                     score=oracle.WANDA if score == "wanda" else oracle.MAG, norms=norms,
                     tensor_scale=tensor_scale, k=k, axis=axis, rows=rows)
    for key in ("values", "scales", "meta", "tensor_scale"):
        if key in ref:
            assert_same(to_np(out[key]), ref[key], key)
    assert_energy(out["energy"], ref["energy"], atol=1e-30)
    assert ws.error() == 0
    return out, ref


# --------------------------------------------------------------------------
# converters: the kernels' own cvt-based encoders against the oracle's
# --------------------------------------------------------------------------

def probe_values(n_random=1 << 22, seed=0):
    rng = np.random.default_rng(seed)
    allbf = synth.bf16_to_f32(np.arange(65536, dtype=np.uint16))
    rnd = rng.integers(0, 2 ** 32, size=n_random, dtype=np.uint64).astype(np.uint32).view(np.float32)
    small = (rng.standard_normal(n_random) * 4).astype(np.float32)
    v = np.concatenate([allbf, rnd, small])
    return v[np.isfinite(v)].astype(np.float32)


def oracle_encode_vec(fn, v):
    return np.fromiter((fn(float(t)) for t in v), dtype=np.uint8, count=len(v))


def test_e4m3_encoder_matches_oracle(ss):
    rng = np.random.default_rng(2)
    allbf = synth.bf16_to_f32(np.arange(65536, dtype=np.uint16))
    rnd = probe_values(n_random=1 << 18, seed=2)
    # midpoints between neighbouring E4M3 values and one ulp either side
    dec = np.array([oracle.e4m3_decode(c) for c in range(127)], dtype=np.float64)
    mids = ((dec[1:] + dec[:-1]) / 2).astype(np.float32)
    ext = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9))])
    v = np.concatenate([allbf, ext, -ext, rng.choice(rnd, 300000)]).astype(np.float32)
    v = v[np.isfinite(v)]
    got = ss.encode_e4m3(torch.from_numpy(v).cuda()).cpu().numpy()
    ref = oracle_encode_vec(oracle.e4m3_encode, v)
    assert_same(got, ref, "e4m3 encode")
    codes = np.arange(256, dtype=np.uint8)
    d = ss.decode_e4m3(torch.from_numpy(codes).cuda()).cpu().numpy()
    for c in range(256):
        r = oracle.e4m3_decode(c)
        if np.isnan(r):
            assert np.isnan(d[c])
        else:
            assert d[c] == r and np.signbit(d[c]) == np.signbit(r)


def test_e2m1_encoder_matches_oracle(ss):
    v = probe_values(n_random=1 << 18, seed=1)
    grid = np.arange(-8, 8, 0.03125, dtype=np.float32)
    v = np.concatenate([v, grid, np.nextafter(grid, np.float32(0)),
                        np.nextafter(grid, np.float32(100))]).astype(np.float32)
    got = ss.encode_e2m1(torch.from_numpy(v).cuda()).cpu().numpy()
    ref = oracle_encode_vec(oracle.e2m1_encode, v)
    assert_same(got, ref, "e2m1 encode")
    codes = np.arange(16, dtype=np.uint8)
    d = ss.decode_e2m1(torch.from_numpy(codes).cuda()).cpu().numpy()
    for c in range(16):
        assert d[c] == oracle.e2m1_decode(c) and np.signbit(d[c]) == np.signbit(oracle.e2m1_decode(c))


def test_encoders_match_the_oracle_on_every_fp32_pattern(ss):
    """The kernels' E4M3 and E2M1 encoders against the oracle's step tables for
    all 2^32 fp32 bit patterns (NaN and infinity excluded)."""
    import encoder_bounds as eb
    for kind, bounds in (("fp8", eb.e4m3_bounds()), ("nvfp4", eb.e2m1_bounds())):
        bad, first = ss.selfcheck_encoder(kind, bounds)
        assert bad == 0, f"{kind}: {bad} mismatches, first bit pattern {first:#010x}"


# --------------------------------------------------------------------------
# the pass: every pattern x score x format, ragged shapes
# --------------------------------------------------------------------------

FORMATS = [("none", 8, 0, False), ("fp8", 8, 0, False), ("int", 8, 64, False), ("int", 4, 32, True),
           ("int", 12, 128, False), ("int", 3, 16, False), ("nvfp4", 4, 0, False), ("mxfp4", 4, 0, False)]


@pytest.mark.parametrize("pattern", [24, 48])
@pytest.mark.parametrize("score", ["mag", "wanda"])
@pytest.mark.parametrize("fmt,bits,group,pack4", FORMATS)
def test_sparse_pass_bf16(ss, ws, pattern, score, fmt, bits, group, pack4):
    rows, k = 100, 512     # 4 row tiles (ragged), 2 column tiles
    xh = synth.sweep_operand(rows, k, seed=3 + pattern)
    norms = np.exp(np.random.default_rng(5).standard_normal(k)).astype(np.float32) if score == "wanda" else None
    compare(ss, ws, xh, pattern=pattern, fmt=fmt, bits=bits, group=group, pack4=pack4, score=score, norms=norms)


@pytest.mark.parametrize("k", [2048, 4608])
@pytest.mark.parametrize("pattern", [24, 48])
@pytest.mark.parametrize("score", ["mag", "wanda"])
@pytest.mark.parametrize("fmt,bits,group,pack4", FORMATS)
def test_sparse_pass_full_width(ss, ws, pattern, score, fmt, bits, group, pack4, k):
    """k >= 1024: units of 1024 columns of one row (k = 4608: a ragged last unit)."""
    xh = synth.sweep_operand(37, k, seed=6 + pattern)
    norms = np.exp(np.random.default_rng(7).standard_normal(k)).astype(np.float32) if score == "wanda" else None
    compare(ss, ws, xh, pattern=pattern, fmt=fmt, bits=bits, group=group, pack4=pack4, score=score, norms=norms)


@pytest.mark.parametrize("k", [2048, 4608])
@pytest.mark.parametrize("fmt,bits,group,pack4", [f for f in FORMATS if f[0] != "none"])
def test_dense_pass_full_width(ss, ws, fmt, bits, group, pack4, k):
    xh = synth.linear_input(29, k, seed=9, n_outlier=8)[0]
    compare(ss, ws, xh, pattern=0, fmt=fmt, bits=bits, group=group, pack4=pack4)


@pytest.mark.parametrize("k", [1024, 4608])
@pytest.mark.parametrize("bits,group,pack4", [(8, 8, False), (5, 256, False), (4, 256, True), (2, 8, True),
                                              (16, 32, False), (7, 128, False)])
def test_dense_int_every_group_span_full_width(ss, ws, bits, group, pack4, k):
    """Dense INT on full-width bf16 rows: groups of 8 (four per lane of 32
    values) up to 256 (eight lanes), every code width and storage."""
    xh = synth.linear_input(21, k, seed=19 + bits, n_outlier=8)[0]
    compare(ss, ws, xh, pattern=0, fmt="int", bits=bits, group=group, pack4=pack4)


@pytest.mark.parametrize("pattern", [0, 24, 48])
@pytest.mark.parametrize("fmt,bits,group,pack4", [("none", 8, 0, False), ("fp8", 8, 0, False), ("nvfp4", 4, 0, False),
                                                  ("int", 3, 16, False), ("mxfp4", 4, 0, False)])
def test_full_width_rows_not_a_multiple_of_64(ss, ws, pattern, fmt, bits, group, pack4):
    """bf16 by magnitude with k = 4128 (a multiple of 32, not of 64; a ragged
    last unit of 32 columns): the full-width stream kernel with a chunk per
    lane and segment, where k = 2048 / 4608 take one lane per 32 elements."""
    k = 4128
    if (pattern == 0 and fmt == "none") or (pattern and fmt == "mxfp4"):
        pytest.skip("format not defined for this pattern / k")
    xh = synth.sweep_operand(23, k, seed=12 + pattern)
    compare(ss, ws, xh, pattern=pattern, fmt=fmt, bits=bits, group=group, pack4=pack4)


@pytest.mark.parametrize("fmt,bits,group,pack4", FORMATS)
def test_sparse_pass_fp32(ss, ws, fmt, bits, group, pack4):
    xh = synth.gaussian_f32(37, 1024, seed=0)
    compare(ss, ws, xh, pattern=24, fmt=fmt, bits=bits, group=group, pack4=pack4)


@pytest.mark.parametrize("fmt,bits,group,pack4", [f for f in FORMATS if f[0] != "none"] + [("int", 8, 256, False)])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_dense_pass(ss, ws, fmt, bits, group, pack4, dtype):
    xh = synth.sweep_operand(70, 768, seed=9) if dtype == "bf16" else synth.gaussian_f32(70, 768, seed=9)
    compare(ss, ws, xh, pattern=0, fmt=fmt, bits=bits, group=group, pack4=pack4)


@pytest.mark.parametrize("pattern", [0, 24, 48])
@pytest.mark.parametrize("k", [128, 256, 1024, 4096, 96, 400])
def test_int_one_scale_per_row(ss, ws, pattern, k):
    """Group 0: one scale per row; tile mode when k is a power of two <= 256,
    row mode (two sweeps over whole rows) otherwise."""
    if pattern == 48 and k % 16:
        pytest.skip("4:8 needs k % 16 == 0")
    xh, _ = synth.linear_input(45, k, seed=2, n_outlier=min(8, k // 16))
    compare(ss, ws, xh, pattern=pattern, fmt="int", bits=8, group=0)
    compare(ss, ws, xh, pattern=pattern, fmt="int", bits=4, group=0, pack4=True)


AXIS0_FORMATS = [("none", 8, 0, False), ("fp8", 8, 0, False), ("int", 8, 32, False), ("int", 4, 16, True),
                 ("int", 12, 64, False), ("nvfp4", 4, 0, False), ("mxfp4", 4, 0, False)]


@pytest.mark.parametrize("pattern", [24, 48])
@pytest.mark.parametrize("fmt,bits,group,pack4", AXIS0_FORMATS)
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_strided_axis(ss, ws, pattern, fmt, bits, group, pack4, dtype):
    """Reduction axis strided in memory (rows contiguous): k = 512 spans four
    128-wide tiles, 104 rows are ragged against the 64 / 32-row tile."""
    xh = synth.sweep_operand(512, 104, seed=31) if dtype == "bf16" else synth.gaussian_f32(512, 104, seed=31)
    compare(ss, ws, xh, pattern=pattern, fmt=fmt, bits=bits, group=group, pack4=pack4, axis=0)
    norms = np.exp(np.random.default_rng(2).standard_normal(512)).astype(np.float32)
    compare(ss, ws, xh, pattern=pattern, fmt=fmt, bits=bits, group=group, pack4=pack4, axis=0, score="wanda",
            norms=norms)


@pytest.mark.parametrize("fmt,bits,group", [("fp8", 8, 0), ("int", 8, 128), ("int", 5, 0), ("nvfp4", 4, 0),
                                            ("mxfp4", 4, 0)])
def test_strided_axis_dense_and_v_along_keys(ss, ws, fmt, bits, group):
    """Dense partner along the strided axis, and V (keys x d, row-major) pruned
    along the key axis of P.V: the logical operand is A[d][keys]."""
    v = synth.attention_qkv(heads=1, seq=2048, d=128, seed=6)      # [keys, d]
    if fmt == "int" and group == 0:
        with pytest.raises(ss.SS24Error):                              # a 2048-long row does not fit a tile
            ss.run(to_dev(v), pattern=0, fmt="int", bits=bits, group=0, axis=0, ws=ws)
    else:
        compare(ss, ws, v, pattern=0, fmt=fmt, bits=bits, group=group, axis=0)
    compare(ss, ws, v, pattern=24, fmt="fp8", axis=0)
    compare(ss, ws, v[:, :96].copy(), pattern=24, fmt="nvfp4", axis=0)      # 96 rows: ragged tile


def test_strided_axis_limits_and_energy_pass(ss, ws):
    x = to_dev(synth.gaussian_bf16(512, 64, seed=3))
    with pytest.raises(ss.SS24Error) as e:
        ss.run(x, pattern=24, fmt="int", bits=8, group=128, axis=0, ws=ws)   # 256-element groups
    assert e.value.status == 5
    with pytest.raises(ss.SS24Error):
        ss.run(x, pattern=0, fmt="int", bits=8, group=0, axis=0, ws=ws)       # one scale per 512-long row
    xh = synth.sweep_operand(256, 80, seed=4)
    xd = to_dev(xh)
    e_gpu = ss.error_energy(xd, pattern=24, sparse_fmt=("nvfp4",), dense_fmt=("int", 3, 64), axis=0, ws=ws)
    sp = oracle.run(xh, fmt="nvfp4", axis=0)["energy"]
    de = oracle.run(xh, pattern=oracle.DENSE, fmt="int", bits=3, group=64, axis=0)["energy"]
    assert_energy(e_gpu, np.array([sp[0], sp[1], sp[2], de[3]]))
    w = synth.gaussian_bf16(256, 64, seed=5, std=0.02)               # k = 256, 64 rows
    norms = np.exp(np.random.default_rng(6).standard_normal(256)).astype(np.float32)
    a = ss.amax(to_dev(w), pattern=24, score="wanda", col_norms=to_dev(norms), axis=0, ws=ws)
    assert a.item() == oracle.amax(w, score=oracle.WANDA, norms=norms, axis=0)


# --------------------------------------------------------------------------
# batches: B same-shaped operands in one call, each exactly as alone
# --------------------------------------------------------------------------

def test_bounded_wait_runs_out_and_is_reported(ss, monkeypatch):
    """A wait that runs out, made on purpose (the SS24_TEST_SKIP_TILE hook: the
    first CTA of the strided-axis kernel skips its third tile copy, and waits
    give up after 10 ms): the call returns, the kernel ends without hanging,
    the workspace's error word is set; after ss24_workspace_init the same call
    is exact against the oracle again."""
    import time
    xh = synth.sweep_operand(4096, 4096, seed=31)      # A[r][c] at xh[c][r]: k = 4096 positions x 4096 rows
    ts = oracle.tensor_scale(xh, "fp8", pattern=oracle.SPARSE_24, axis=0)
    sd = torch.tensor([ts], dtype=torch.float32, device="cuda")
    x = to_dev(xh)
    ws = ss.Workspace()
    ss.run(x, pattern=24, fmt="fp8", tensor_scale=sd, ws=ws, axis=0)      # first call: module and attributes
    torch.cuda.synchronize()
    assert ws.error() == 0
    monkeypatch.setenv("SS24_TEST_SKIP_TILE", "2")
    t0 = time.perf_counter()
    ss.run(x, pattern=24, fmt="fp8", tensor_scale=sd, ws=ws, axis=0)
    code = ws.error()                                   # synchronizes the stream
    elapsed = time.perf_counter() - t0
    assert code != 0, "the skipped tile did not make a wait run out"
    assert elapsed < 1.5, elapsed                       # the 10 ms limit, not two seconds
    monkeypatch.delenv("SS24_TEST_SKIP_TILE")
    assert ss.lib().ss24_workspace_init(ws.ptr, ws.nbytes, None) == 0
    assert ws.error() == 0
    out = ss.run(x, pattern=24, fmt="fp8", tensor_scale=sd, ws=ws, axis=0)
    torch.cuda.synchronize()
    ref = oracle.run(xh, pattern=oracle.SPARSE_24, fmt="fp8", tensor_scale=ts, axis=0)
    for key in ("values", "meta"):
        assert_same(to_np(out[key]), ref[key], key)
    assert_energy(out["energy"], ref["energy"], atol=1e-30)
    assert ws.error() == 0


def compare_batch(ss, ws, xs, *, pattern, fmt, bits=8, group=0, pack4=False, axis=1, pad_rows=0, tensor_scale=None):
    """xs: host arrays of one shape; they are placed pad_rows apart (a strided
    batch when pad_rows > 0) and processed in one call; each operand's outputs
    are compared with the oracle run on that operand alone."""
    B = len(xs)
    shape = xs[0].shape
    full = np.zeros((B, shape[0] + pad_rows, shape[1]), dtype=xs[0].dtype)
    for b in range(B):
        full[b, :shape[0]] = xs[b]
    xd = to_dev(full)[:, :shape[0]]
    sd = torch.tensor(tensor_scale, dtype=torch.float32, device="cuda") if tensor_scale is not None else None
    out = ss.run(xd, pattern=pattern, fmt=fmt, bits=bits, group=group, pack4=pack4, axis=axis, tensor_scale=sd,
                 ws=ws)
    torch.cuda.synchronize()
    opat = {0: oracle.DENSE, 24: oracle.SPARSE_24, 48: oracle.SPARSE_48}[pattern]
    for b in range(B):
        ref = oracle.run(xs[b], pattern=opat, fmt=fmt, bits=bits, group=group, pack4=pack4, axis=axis,
                         tensor_scale=None if tensor_scale is None else tensor_scale[b])
        for key in ("values", "scales", "meta"):
            if key in ref:
                assert_same(to_np(out[key][b]), ref[key], f"{key}[{b}]")
        if "tensor_scale" in ref:
            assert_same(to_np(out["tensor_scale"][b:b + 1]), ref["tensor_scale"], f"tensor_scale[{b}]")
        assert_energy(out["energy"][b], ref["energy"], atol=1e-30)
    assert ws.error() == 0


@pytest.mark.parametrize("pattern,fmt,bits,group", [(24, "fp8", 8, 0), (24, "nvfp4", 4, 0), (48, "mxfp4", 4, 0),
                                                    (24, "int", 8, 64), (24, "none", 8, 0), (0, "fp8", 8, 0),
                                                    (0, "int", 8, 0), (24, "int", 4, 0), (0, "int", 8, 0)])
@pytest.mark.parametrize("pad_rows", [0, 5])
def test_batch_of_operands(ss, ws, pattern, fmt, bits, group, pad_rows):
    xs = [synth.sweep_operand(100, 1024, seed=40 + b) for b in range(3)]  # distinct operands and scales
    compare_batch(ss, ws, xs, pattern=pattern, fmt=fmt, bits=bits, group=group, pad_rows=pad_rows)


def test_batch_given_scales_axis0_and_long_rows(ss, ws):
    xs = [synth.sweep_operand(64, 512, seed=50 + b) for b in range(4)]
    scales = [oracle.tensor_scale(x, "fp8") * (1 + b) for b, x in enumerate(xs)]
    compare_batch(ss, ws, xs, pattern=24, fmt="fp8", tensor_scale=scales)
    xa = [synth.sweep_operand(256, 72, seed=60 + b) for b in range(3)]        # axis 0: [k][rows]
    compare_batch(ss, ws, xa, pattern=24, fmt="nvfp4", axis=0)
    compare_batch(ss, ws, xa, pattern=0, fmt="int", bits=8, group=32, axis=0)
    xl = [synth.linear_input(20, 5120, seed=70 + b, n_outlier=8)[0] for b in range(2)]
    compare_batch(ss, ws, xl, pattern=24, fmt="int", bits=8, group=0, pad_rows=3)


@pytest.mark.parametrize("pattern,fmt,bits,group", [(24, "nvfp4", 4, 0), (0, "nvfp4", 4, 0), (24, "mxfp4", 4, 0),
                                                    (0, "mxfp4", 4, 0), (48, "nvfp4", 4, 0), (24, "int", 8, 128),
                                                    (48, "fp8", 8, 0)])
@pytest.mark.parametrize("rows,k,batch,pad", [(1, 1024, 1, 0), (2, 4160, 3, 2), (5, 2048, 4, 0)])
def test_lane_block_few_units_and_batches(ss, ws, pattern, fmt, bits, group, rows, k, batch, pad):
    """The lane-block kernels (with and without their one-unit-ahead loads) on
    operands with fewer units than warps, a last unit with two lanes inside
    the row (k = 4160), and strided batches: every output and energy of every
    operand against the oracle."""
    if fmt == "int" and (k // 2) % group:
        pytest.skip("the rows hold no whole number of groups")
    xs = [synth.sweep_operand(rows, k, seed=150 + 7 * b + rows) for b in range(batch)]
    compare_batch(ss, ws, xs, pattern=pattern, fmt=fmt, bits=bits, group=group, pad_rows=pad)


def test_batch_amax_scale_energy_and_empty(ss, ws):
    xs = [synth.gaussian_bf16(40, 256, seed=80 + b, std=1.0 + b) for b in range(5)]
    xd = to_dev(np.stack(xs))
    a = ss.amax(xd, pattern=24, ws=ws).cpu().numpy()
    t = ss.tensor_scale(xd, "nvfp4", ss.SPARSE_24, ws=ws).cpu().numpy()
    e = ss.error_energy(xd, pattern=24, sparse_fmt=("fp8",), dense_fmt=("int", 5, 32), ws=ws).cpu().numpy()
    for b, x in enumerate(xs):
        assert a[b] == np.float32(oracle.amax(x))
        assert t[b] == np.float32(oracle.tensor_scale(x, "nvfp4"))
        sp = oracle.run(x, fmt="fp8")["energy"]
        de = oracle.run(x, pattern=oracle.DENSE, fmt="int", bits=5, group=32)["energy"]
        g = e[b]
        for f, r in zip(range(4), [sp[0], sp[1], sp[2], de[3]]):
            assert abs(g[f] - r) <= RTOL * abs(r)
    empty = torch.zeros((3, 0, 64), dtype=torch.bfloat16, device="cuda")
    out = ss.run(empty, pattern=24, fmt="fp8", ws=ws)
    torch.cuda.synchronize()
    assert out["energy"].shape == (3, 4) and out["energy"].abs().sum().item() == 0.0
    assert ws.error() == 0


@pytest.mark.parametrize("k", [14336, 16400])
def test_int_one_scale_per_very_long_row(ss, ws, k):
    """k = 14336: eight chunks per thread of a 256-thread row block; k = 16400
    (over 2048 chunks): the two-sweep warp-per-row kernel."""
    for pattern in (0, 24, 48):
        xh, _ = synth.linear_input(7, k, seed=8)
        compare(ss, ws, xh, pattern=pattern, fmt="int", bits=8, group=0)
        xf = synth.gaussian_f32(5, k, seed=9)
        compare(ss, ws, xf, pattern=pattern, fmt="int", bits=5, group=0)
    xh, _ = synth.linear_input(6, k, seed=10)
    norms = synth.linear_weight(1, k, seed=11)[1]
    compare(ss, ws, xh, pattern=24, fmt="int", bits=4, group=0, pack4=True, score="wanda", norms=norms)


ROWS_CASES = [("linear", 45, 4096), ("linear", 13, 1000), ("linear", 33, 96), ("gauss32", 9, 5120),
              ("linear", 7, 14336)]


@pytest.mark.parametrize("pattern,score", [(0, "mag"), (24, "mag"), (24, "wanda"), (48, "mag")])
@pytest.mark.parametrize("case", ROWS_CASES)
def test_row_amax_and_int_from_given_row_amax(ss, ws, pattern, score, case):
    """ss24_amax_rows (per-row amax and the tensor scale in one read) and
    ss24_quantize_int_rows (one scale per row from that amax) against the oracle."""
    kind, rows, k = case
    if pattern == 48 and k % 16:
        pytest.skip("4:8 needs k % 16 == 0")
    xh = synth.linear_input(rows, k, seed=12, n_outlier=min(8, k // 16))[0] if kind == "linear" \
        else synth.gaussian_f32(rows, k, seed=13)
    norms = synth.linear_weight(1, k, seed=14)[1] if score == "wanda" else None
    opat = {0: oracle.DENSE, 24: oracle.SPARSE_24, 48: oracle.SPARSE_48}[pattern]
    osc = oracle.WANDA if score == "wanda" else oracle.MAG
    x, nd = to_dev(xh), (to_dev(norms) if norms is not None else None)
    ra, sc = ss.amax_rows(x, pattern=pattern, score=score, col_norms=nd, scale_fmt="fp8", ws=ws)
    torch.cuda.synchronize()
    want = np.array([oracle.amax(np.ascontiguousarray(xh[r:r + 1]), pattern=opat, score=osc, norms=norms)
                     for r in range(rows)], dtype=np.float32)
    assert_same(to_np(ra), want, "row amax")
    assert_same(to_np(sc), np.array([oracle.tensor_scale(xh, "fp8", pattern=opat, score=osc, norms=norms)],
                                    dtype=np.float32), "tensor scale")
    for bits, pack4 in ((8, False), (4, True)):
        out = ss.run_int_rows(x, ra, pattern=pattern, bits=bits, pack4=pack4, score=score, col_norms=nd, ws=ws)
        torch.cuda.synchronize()
        ref = oracle.run(xh, pattern=opat, fmt="int", bits=bits, group=0, pack4=pack4, score=osc, norms=norms)
        for key in ("values", "scales", "meta"):
            if key in ref:
                assert_same(to_np(out[key]), ref[key], key)
        assert_energy(out["energy"], ref["energy"], atol=1e-30)
    assert ws.error() == 0


def test_row_amax_batch_and_empty(ss, ws):
    xs = [synth.sweep_operand(40, 2048, seed=80 + b) for b in range(3)]
    x = torch.stack([to_dev(v) for v in xs])
    ra, _ = ss.amax_rows(x, ws=ws)
    out = ss.run_int_rows(x, ra, bits=8, ws=ws)
    torch.cuda.synchronize()
    for b, xh in enumerate(xs):
        ref = oracle.run(xh, pattern=oracle.DENSE, fmt="int", bits=8, group=0)
        assert_same(to_np(out["values"][b]), ref["values"], "values")
        assert_same(to_np(out["scales"][b]), ref["scales"], "scales")
        assert_energy(out["energy"][b], ref["energy"], atol=1e-30)
    empty = torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda")
    ra0, sc0 = ss.amax_rows(empty, scale_fmt="fp8", ws=ws)
    torch.cuda.synchronize()
    assert ra0.numel() == 0 and sc0.item() == 0.0
    assert ws.error() == 0


DEQ_FORMATS = [("none", 8, 0, False), ("fp8", 8, 0, False), ("int", 8, 64, False), ("int", 4, 0, True),
               ("int", 12, 32, False), ("int", 5, 0, False), ("nvfp4", 4, 0, False), ("mxfp4", 4, 0, False)]


@pytest.mark.parametrize("pattern", [0, 24, 48])
@pytest.mark.parametrize("fmt,bits,group,pack4", DEQ_FORMATS)
@pytest.mark.parametrize("shape", [(37, 512), (9, 2048), (13, 1536)])
def test_dequantize_matches_oracle(ss, ws, pattern, fmt, bits, group, pack4, shape):
    """ss24_dequantize of the pass's own outputs against the oracle's
    reconstruction, bit for bit (fp32 and bf16 kept values for format NONE)."""
    if fmt == "none" and pattern == 0:
        pytest.skip("format NONE is the plain 2:4 compression")
    rows, k = shape
    opat = {0: oracle.DENSE, 24: oracle.SPARSE_24, 48: oracle.SPARSE_48}[pattern]
    for xh in ((synth.sweep_operand(rows, k, seed=40),) if fmt != "none"
               else (synth.sweep_operand(rows, k, seed=40), synth.gaussian_f32(rows, k, seed=41))):
        out, ref = compare(ss, ws, xh, pattern=pattern, fmt=fmt, bits=bits, group=group, pack4=pack4)
        dt = torch.bfloat16 if xh.dtype == np.uint16 else torch.float32
        got = ss.dequantize(out, rows, k, pattern=pattern, fmt=fmt, bits=bits, group=group, pack4=pack4, dtype=dt)
        torch.cuda.synchronize()
        want = oracle.dequantize(ref, rows=rows, k=k, pattern=opat, fmt=fmt, bits=bits, group=group, pack4=pack4,
                                 dtype=oracle.BF16 if xh.dtype == np.uint16 else oracle.F32)
        assert_same(to_np(got), want, "x_hat")


@pytest.mark.parametrize("pattern", [0, 24, 48])
@pytest.mark.parametrize("fmt,bits,group,pack4", [("fp8", 8, 0, False), ("nvfp4", 4, 0, False),
                                                  ("int", 8, 0, False), ("int", 4, 0, True), ("mxfp4", 4, 0, False)])
@pytest.mark.parametrize("rows,k,batch", [(20, 1024, 3), (3, 64, 7), (1, 8, 5)])
def test_dequantize_batch(ss, ws, pattern, fmt, bits, group, pack4, rows, k, batch):
    """Batches: one tensor scale per operand (FP8, NVFP4) and one INT scale per
    row, including operands much smaller than the kernel's unit of work."""
    if k % 16 and pattern == 48:
        pytest.skip("4:8 needs k % 16 == 0")
    n = k // 2 if pattern else k
    if (fmt == "nvfp4" and n % 16) or (fmt == "mxfp4" and n % 32):
        pytest.skip("block longer than the row")
    opat = {0: oracle.DENSE, 24: oracle.SPARSE_24, 48: oracle.SPARSE_48}[pattern]
    xs = [synth.sweep_operand(rows, k, seed=90 + b) for b in range(batch)]
    x = torch.stack([to_dev(v) for v in xs])
    out = ss.run(x, pattern=pattern, fmt=fmt, bits=bits, group=group, pack4=pack4, ws=ws)
    got = ss.dequantize(out, rows, k, pattern=pattern, fmt=fmt, bits=bits, group=group, pack4=pack4, batch=batch)
    torch.cuda.synchronize()
    for b, xh in enumerate(xs):
        ref = oracle.run(xh, pattern=opat, fmt=fmt, bits=bits, group=group, pack4=pack4)
        want = oracle.dequantize(ref, rows=rows, k=k, pattern=opat, fmt=fmt, bits=bits, group=group, pack4=pack4)
        assert_same(to_np(got[b]), want, f"x_hat[{b}]")


@pytest.mark.parametrize("pattern", [0, 24, 48])
@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
@pytest.mark.parametrize("rows,k,batch", [(37, 512, 0), (130, 1536, 0), (20, 1024, 3), (1, 64, 2)])
def test_scale_tiles_of_pass_scales(ss, ws, pattern, fmt, rows, k, batch):
    """The pass's own block scales, rearranged into the block-scaled MMA's tiles,
    against the oracle's rearrangement of the oracle's scales, byte for byte."""
    n = k // 2 if pattern else k
    blk = 16 if fmt == "nvfp4" else 32
    if n % blk:
        pytest.skip("block longer than the row")
    cols = n // blk
    opat = {0: oracle.DENSE, 24: oracle.SPARSE_24, 48: oracle.SPARSE_48}[pattern]
    nb = max(batch, 1)
    xs = [synth.sweep_operand(rows, k, seed=60 + b) for b in range(nb)]
    x = torch.stack([to_dev(v) for v in xs]) if batch else to_dev(xs[0])
    out = ss.run(x, pattern=pattern, fmt=fmt, ws=ws)
    got = ss.scale_tiles(out["scales"], rows, cols, batch=batch or None)
    torch.cuda.synchronize()
    want = np.concatenate([oracle.scale_tiles(oracle.run(xh, pattern=opat, fmt=fmt)["scales"], rows, cols)
                           for xh in xs])
    assert np.array_equal(got.cpu().numpy(), want)


@pytest.mark.parametrize("rows,cols,batch", [(1, 1, 0), (300, 17, 0), (129, 5, 4), (128, 4, 0), (4096, 256, 2)])
def test_scale_tiles_random_bytes(ss, rows, cols, batch):
    """Every byte value, ragged rows and columns, and zero padding written."""
    nb = max(batch, 1)
    src = np.random.default_rng(rows + cols).integers(0, 256, size=(nb, rows, cols), dtype=np.uint8)
    per = oracle.lib().oracle_scale_tiles_bytes(rows, cols)
    out = torch.full((nb * per,), 0x5A, dtype=torch.uint8, device="cuda")   # stale bytes must be overwritten
    got = ss.scale_tiles(torch.from_numpy(src).cuda(), rows, cols, batch=batch or None, out=out)
    torch.cuda.synchronize()
    assert np.array_equal(got.cpu().numpy(), oracle.scale_tiles(src, rows, cols, nb))


@pytest.mark.parametrize("b", [2, 4, 8, 16, 32, 64, 128, 256])
def test_hadamard_matches_oracle(ss, b):
    """Rotation bit for bit: bf16 and fp32 inputs, several rows, a ragged last
    warp, rows with ld > k, and a batch."""
    for rows, k in ((37, 512), (5, 256), (3, 768)):
        if k % b:
            continue
        for xh in (synth.sweep_operand(rows, k, seed=80 + b), synth.gaussian_f32(rows, k, seed=81 + b)):
            got = ss.hadamard(to_dev(xh), b)
            torch.cuda.synchronize()
            assert_same(to_np(got), oracle.hadamard(xh, b), f"rot b={b} {rows}x{k}")
    xh = synth.sweep_operand(9, 512, seed=82)
    wide = torch.zeros((9, 640), dtype=torch.bfloat16, device="cuda")
    wide[:, :512] = to_dev(xh)
    got = ss.hadamard(wide[:, :512], b)
    torch.cuda.synchronize()
    assert_same(to_np(got), oracle.hadamard(xh, b), "rot ld > k")
    # an output 16 but not 32 bytes aligned (the two-store path)
    buf = torch.empty(9 * 512 + 4, dtype=torch.float32, device="cuda")
    got = ss.hadamard(to_dev(xh), b, out=buf[4:].view(9, 512))
    torch.cuda.synchronize()
    assert got.data_ptr() % 32 == 16
    assert_same(to_np(got), oracle.hadamard(xh, b), "rot out 16-byte aligned")
    xs = [synth.sweep_operand(6, 256, seed=83 + i) for i in range(3)]
    got = ss.hadamard(torch.stack([to_dev(v) for v in xs]), b)
    torch.cuda.synchronize()
    for i, v in enumerate(xs):
        assert_same(to_np(got[i]), oracle.hadamard(v, b), f"rot batch {i}")


@pytest.mark.parametrize("fmt,bits,group", [("fp8", 8, 0), ("nvfp4", 4, 0), ("int", 8, 0)])
def test_rotated_pass_matches_oracle(ss, ws, fmt, bits, group):
    """A rotated pass: the rotation on the GPU feeding a fused 2:4 pass on the
    rotated fp32 operand, against the oracle's pass on its own rotation."""
    xh = synth.linear_input(64, 1024, seed=84)[0]
    rot = ss.hadamard(to_dev(xh), 128)
    out = ss.run(rot, pattern=24, fmt=fmt, bits=bits, group=group, ws=ws)
    torch.cuda.synchronize()
    ref = oracle.run(oracle.hadamard(xh, 128), pattern=oracle.SPARSE_24, fmt=fmt, bits=bits, group=group)
    assert_same(to_np(out["values"]), ref["values"], "values")
    assert_same(to_np(out["meta"]), ref["meta"], "meta")
    assert_energy(out["energy"], ref["energy"])


def test_rotation_raises_predicted_ratio(ss, ws):
    """The pages' direction (§4): on a linear input with outlier channels,
    rotation makes 2:4 relatively worse (R_hat grows), for 2:4 + FP8 against
    dense FP8 and for 2:4 INT8 against dense INT5 (one scale per row)."""
    x = to_dev(synth.linear_input(512, 4096, seed=85)[0])
    rot = ss.hadamard(x, 128)
    for sp, de in ((("fp8", 8), ("fp8", 8)), (("int", 8), ("int", 5))):
        r = []
        for inp in (x, rot):
            es = ss.run(inp, pattern=24, fmt=sp[0], bits=sp[1], ws=ws)["energy"]
            ed = ss.run(inp, pattern=0, fmt=de[0], bits=de[1], ws=ws)["energy"]
            r.append(ss.predicted_ratio(es, ed)[3].item())
        assert r[1] > r[0], (sp, de, r)
    # i.i.d. Gaussian data is rotation invariant in distribution: R_hat unchanged
    g = to_dev(synth.gaussian_bf16(32768, 128, seed=86))
    for inp_pair in ((g, ss.hadamard(g, 128)),):
        r = []
        for inp in inp_pair:
            es = ss.run(inp, pattern=24, fmt="fp8", ws=ws)["energy"]
            ed = ss.run(inp, pattern=0, fmt="int", bits=5, ws=ws)["energy"]
            r.append(ss.predicted_ratio(es, ed)[3].item())
        assert abs(r[1] / r[0] - 1) < 0.02, r


def test_pairwise48_drops_the_largest_value(ss, ws):
    """Pairwise 4:8 ranks pairs by energy, so a tensor's or row's largest value
    can be dropped (pairs (0.8, 0.8) and (0.75, 0.75) outrank (1.0, 0)): the
    derived tensor scales and the per-row INT scales take the kept amax."""
    pat8 = synth.bf16_bits(np.array([0.8, 0.8, 0.75, 0.75, 1.0, 0.0, 0.1, 0.1], dtype=np.float32))
    for rows, k in ((16, 2048), (3, 20480), (5, 256)):
        xh = np.tile(pat8, (rows, k // 8))
        for fmt, bits in (("fp8", 8), ("nvfp4", 4), ("int", 8)):
            compare(ss, ws, xh, pattern=48, fmt=fmt, bits=bits, group=0)
    xh = np.tile(pat8, (8, 1024 // 8))
    ra, _ = ss.amax_rows(to_dev(xh), pattern=48, ws=ws)
    torch.cuda.synchronize()
    assert np.all(ra.cpu().numpy() == np.float32(synth.bf16_to_f32(pat8)[0]))   # 0.8 in bf16, not 1.0


ROT_CASES = [(24, "none", 8, 0), (24, "fp8", 8, 0), (24, "nvfp4", 4, 0), (24, "mxfp4", 4, 0), (24, "int", 8, 64),
             (48, "nvfp4", 4, 0), (48, "fp8", 8, 0), (0, "fp8", 8, 0), (0, "nvfp4", 4, 0), (0, "int", 5, 128)]


@pytest.mark.parametrize("pattern,fmt,bits,group", ROT_CASES)
@pytest.mark.parametrize("b", [16, 128, 256])
def test_rotated_pass_fused_matches_oracle(ss, ws, pattern, fmt, bits, group, b):
    """The rotation inside the pass (operand field hadamard = b) against the
    oracle's rotation rounded to bf16 followed by the oracle's pass: full-width
    rows, a partial last unit and narrow rows; FP8 / NVFP4 with the derived
    tensor scale (the amax pass rotates too) and FP8 with a given one."""
    opat = {0: oracle.DENSE, 24: oracle.SPARSE_24, 48: oracle.SPARSE_48}[pattern]
    for rows, k in ((37, 1024), (5, 1280), (9, 512), (6, 256)):
        if k % b:
            continue
        xh = synth.sweep_operand(rows, k, seed=100 + b)
        rot = oracle.hadamard_bf16(xh, b)
        out = ss.run(to_dev(xh), pattern=pattern, fmt=fmt, bits=bits, group=group, ws=ws, hadamard=b)
        torch.cuda.synchronize()
        ts = oracle.tensor_scale(rot, fmt, pattern=opat) if fmt in ("fp8", "nvfp4") else None
        ref = oracle.run(rot, pattern=opat, fmt=fmt, bits=bits, group=group,
                         **({"tensor_scale": ts} if ts is not None else {}))
        for key in ("values", "scales", "meta"):
            if key in ref and out.get(key) is not None:
                assert_same(to_np(out[key]), ref[key], f"{key} {rows}x{k}")
        assert_energy(out["energy"], ref["energy"], atol=1e-30)
        if fmt == "fp8":
            given = torch.tensor([np.float32(0.05)], device="cuda")
            out = ss.run(to_dev(xh), pattern=pattern, fmt=fmt, tensor_scale=given, ws=ws, hadamard=b)
            torch.cuda.synchronize()
            ref = oracle.run(rot, pattern=opat, fmt=fmt, tensor_scale=float(np.float32(0.05)))
            assert_same(to_np(out["values"]), ref["values"], f"values given scale {rows}x{k}")
    assert ws.error() == 0


@pytest.mark.parametrize("pattern,fmt,bits,group", [(24, "fp8", 8, 0), (24, "nvfp4", 4, 0), (24, "int", 4, 32),
                                                    (24, "none", 8, 0), (48, "mxfp4", 4, 0), (0, "mxfp4", 4, 0),
                                                    (0, "fp8", 8, 0)])
@pytest.mark.parametrize("b", [2, 4, 8, 32, 64])
def test_rotated_pass_every_block_full_width(ss, ws, pattern, fmt, bits, group, b):
    """The rotation inside the pass on full-width rows (k = 4608: four whole
    units and a ragged fifth) for blocks inside one lane's 32 values (b <= 32)
    and across two lanes (b = 64), against the oracle's rotation rounded to
    bf16 and its pass."""
    opat = {0: oracle.DENSE, 24: oracle.SPARSE_24, 48: oracle.SPARSE_48}[pattern]
    xh = synth.sweep_operand(11, 4608, seed=130 + b)
    rot = oracle.hadamard_bf16(xh, b)
    out = ss.run(to_dev(xh), pattern=pattern, fmt=fmt, bits=bits, group=group, ws=ws, hadamard=b)
    torch.cuda.synchronize()
    ts = oracle.tensor_scale(rot, fmt, pattern=opat) if fmt in ("fp8", "nvfp4") else None
    ref = oracle.run(rot, pattern=opat, fmt=fmt, bits=bits, group=group,
                     **({"tensor_scale": ts} if ts is not None else {}))
    for key in ("values", "scales", "meta"):
        if key in ref and out.get(key) is not None:
            assert_same(to_np(out[key]), ref[key], key)
    assert_energy(out["energy"], ref["energy"], atol=1e-30)
    assert ws.error() == 0


@pytest.mark.parametrize("b", [8, 32, 128])
def test_rotated_error_energy_format_pairs(ss, ws, b):
    """The read-only energy pass over the operand rotated in registers (full-
    width rows, k = 4608), against the oracle's passes on its own rotation."""
    xh = synth.sweep_operand(9, 4608, seed=140 + b)
    rot = oracle.hadamard_bf16(xh, b)
    x = to_dev(xh)
    for sf, df in ((("nvfp4",), ("mxfp4",)), (("mxfp4",), ("int", 3, 64)), (("int", 4, 16, True), ("fp8",))):
        e = ss.error_energy(x, pattern=24, sparse_fmt=sf, dense_fmt=df, ws=ws, hadamard=b)
        sp = oracle.run(rot, **_fmt_kw(sf))["energy"]
        de = oracle.run(rot, pattern=oracle.DENSE, **_fmt_kw(df))["energy"]
        assert_energy(e, [sp[0], sp[1], sp[2], de[3]])
    assert ws.error() == 0


def test_rotated_rows_energy_and_batch(ss, ws):
    """Rotated per-row INT (the row amax pass and the INT pass from it), the
    rotated energy pass, and a rotated batch."""
    b = 64
    xh = synth.linear_input(40, 2048, seed=105)[0]
    rot = oracle.hadamard_bf16(xh, b)
    x = to_dev(xh)
    ra, _ = ss.amax_rows(x, ws=ws, hadamard=b)
    out = ss.run_int_rows(x, ra, bits=8, ws=ws, hadamard=b)
    torch.cuda.synchronize()
    ref = oracle.run(rot, pattern=oracle.DENSE, fmt="int", bits=8, group=0)
    assert_same(to_np(out["values"]), ref["values"], "int rows values")
    assert_same(to_np(out["scales"]), ref["scales"], "int rows scales")
    e = ss.error_energy(x, pattern=24, sparse_fmt=("fp8",), dense_fmt=("int", 5, 128), ws=ws, hadamard=b)
    torch.cuda.synchronize()
    ts = oracle.tensor_scale(rot, "fp8", pattern=oracle.SPARSE_24)
    sp = oracle.run(rot, pattern=oracle.SPARSE_24, fmt="fp8", tensor_scale=ts)["energy"]
    de = oracle.run(rot, pattern=oracle.DENSE, fmt="int", bits=5, group=128)["energy"]
    assert_energy(e, np.array([sp[0], sp[1], sp[2], de[3]]), atol=1e-30)
    xs = [synth.sweep_operand(7, 1024, seed=106 + i) for i in range(3)]
    out = ss.run(torch.stack([to_dev(v) for v in xs]), pattern=24, fmt="mxfp4", ws=ws, hadamard=32)
    torch.cuda.synchronize()
    for i, v in enumerate(xs):
        ref = oracle.run(oracle.hadamard_bf16(v, 32), pattern=oracle.SPARSE_24, fmt="mxfp4")
        assert_same(to_np(out["values"][i]), ref["values"], f"batch values {i}")
        assert_energy(out["energy"][i], ref["energy"], atol=1e-30)


SOFTMAX_CASES = [(24, "none", 8, 0), (24, "fp8", 8, 0), (24, "nvfp4", 4, 0), (24, "mxfp4", 4, 0),
                 (24, "int", 8, 32), (48, "nvfp4", 4, 0), (48, "fp8", 8, 0), (0, "fp8", 8, 0), (0, "mxfp4", 4, 0),
                 (0, "int", 4, 64)]


def _logits(rows, keys, seed):
    return (np.random.default_rng(seed).standard_normal((rows, keys)) * 3.0).astype(np.float32)


def _p_scale(fmt):
    # P <= 1: the FP8 scale 1/448 and the NVFP4 tensor scale 1 / (6 * 448)
    return {"fp8": np.float32(1.0 / 448.0), "nvfp4": np.float32(1.0 / 2688.0)}.get(fmt)


@pytest.mark.parametrize("pattern,fmt,bits,group", SOFTMAX_CASES)
@pytest.mark.parametrize("logits", ["bf16", "f32"])
def test_softmax_prune_matches_oracle(ss, ws, pattern, fmt, bits, group, logits):
    """P = softmax(alpha s) pruned in its producer, against the oracle's softmax
    followed by the oracle's pass on that bf16 P: outputs bit for bit,
    energies within 1e-6 (5 slices of 256 keys: a ragged last unit)."""
    rows, keys, alpha = 37, 1280, float(np.float32(1.0 / math.sqrt(128)))
    s = _logits(rows, keys, 90 + pattern)
    sh = synth.bf16_bits(s) if logits == "bf16" else s
    ts = _p_scale(fmt)
    tsd = torch.tensor([ts], device="cuda") if ts is not None else None
    out = ss.softmax_prune(to_dev(sh), alpha, pattern=pattern, fmt=fmt, bits=bits, group=group, tensor_scale=tsd,
                           ws=ws)
    torch.cuda.synchronize()
    P = oracle.softmax_bf16(sh, alpha)
    opat = {0: oracle.DENSE, 24: oracle.SPARSE_24, 48: oracle.SPARSE_48}[pattern]
    ref = oracle.run(P, pattern=opat, fmt=fmt, bits=bits, group=group,
                     **({"tensor_scale": float(ts)} if ts is not None else {}))
    assert_same(to_np(out["values"]), ref["values"], "values")
    if pattern:
        assert_same(to_np(out["meta"]), ref["meta"], "meta")
    if "scales" in ref and ref["scales"] is not None and out.get("scales") is not None:
        assert_same(to_np(out["scales"]), ref["scales"], "scales")
    assert_energy(out["energy"], ref["energy"], atol=1e-30)
    assert ws.error() == 0


def test_softmax_prune_batch_and_shapes(ss, ws):
    """A batch of three operands, one slice per row, and a long row of 8192 keys."""
    alpha = float(np.float32(1.0 / math.sqrt(128)))
    xs = [synth.bf16_bits(_logits(8, 512, 95 + b)) for b in range(3)]
    ts = torch.full((3,), 1.0 / 448.0, device="cuda")
    out = ss.softmax_prune(torch.stack([to_dev(v) for v in xs]), alpha, pattern=24, fmt="fp8", tensor_scale=ts, ws=ws)
    torch.cuda.synchronize()
    for b, sh in enumerate(xs):
        ref = oracle.run(oracle.softmax_bf16(sh, alpha), pattern=oracle.SPARSE_24, fmt="fp8",
                         tensor_scale=float(np.float32(1.0 / 448.0)))
        assert_same(to_np(out["values"][b]), ref["values"], f"values[{b}]")
        assert_same(to_np(out["meta"][b]), ref["meta"], f"meta[{b}]")
        assert_energy(out["energy"][b], ref["energy"], atol=1e-30)
    # wide logits: arguments below -104 (clamped), subnormal e, quotients below
    # 2^-40 (the IEEE-division chunks)
    wide = (np.random.default_rng(98).standard_normal((16, 512)) * 40.0).astype(np.float32)
    for a in (1.0, alpha):
        out = ss.softmax_prune(to_dev(wide), a, pattern=24, fmt="fp8", tensor_scale=ts[:1], ws=ws)
        torch.cuda.synchronize()
        ref = oracle.run(oracle.softmax_bf16(wide, a), pattern=oracle.SPARSE_24, fmt="fp8",
                         tensor_scale=float(np.float32(1.0 / 448.0)))
        assert_same(to_np(out["values"]), ref["values"], f"wide values alpha={a}")
        assert_same(to_np(out["meta"]), ref["meta"], f"wide meta alpha={a}")
    for rows, keys in ((3, 256), (2, 8192)):
        sh = synth.bf16_bits(_logits(rows, keys, 97))
        out = ss.softmax_prune(to_dev(sh), alpha, pattern=24, fmt="none", ws=ws)
        torch.cuda.synchronize()
        ref = oracle.run(oracle.softmax_bf16(sh, alpha), pattern=oracle.SPARSE_24, fmt="none")
        assert_same(to_np(out["values"]), ref["values"], f"values {rows}x{keys}")
        assert_same(to_np(out["meta"]), ref["meta"], f"meta {rows}x{keys}")


@pytest.mark.parametrize("sparse,dense", [(("fp8",), ("int", 5, 128)), (("nvfp4",), ("mxfp4",)),
                                          (("int", 8, 0), ("int", 5, 0))])
def test_measured_ratio_against_oracle_and_prediction(ss, ws, sparse, dense):
    """Operator-level R (errors of X_hat W^T): the GPU value against the same
    quantity built from the oracle's outputs in fp64, and against R_hat, which
    it matches in expectation for a weight with i.i.d. entries."""
    from semi_structured_sparsity_online_b200 import operator_error
    xh = synth.linear_input(256, 1024, seed=51, n_outlier=8)[0]
    wf = synth.gaussian_f32(512, 1024, seed=52)
    got = operator_error.measured_ratio(to_dev(xh), torch.from_numpy(wf).cuda(), sparse=sparse, dense=dense, ws=ws)

    def side(pattern, spec):
        fmt, bits, group = (spec + (8, 0))[:3]
        ref = oracle.run(xh, pattern=pattern, fmt=fmt, bits=bits, group=group)
        xhat = oracle.dequantize(ref, rows=256, k=1024, pattern=pattern, fmt=fmt, bits=bits, group=group)
        return xhat.astype(np.float64), ref["energy"]

    x = synth.bf16_to_f32(xh).astype(np.float64)
    y = x @ wf.astype(np.float64).T
    xs, es = side(oracle.SPARSE_24, sparse)
    xd, ed = side(oracle.DENSE, dense)
    err_s = np.linalg.norm((xs - x) @ wf.astype(np.float64).T) / np.linalg.norm(y)
    err_d = np.linalg.norm((xd - x) @ wf.astype(np.float64).T) / np.linalg.norm(y)
    assert abs(got["err_sparse"] / err_s - 1) < 1e-3 and abs(got["err_dense"] / err_d - 1) < 1e-3
    r_hat = oracle.ratio(es, ed)[3]
    assert abs(got["r_predicted"] / r_hat - 1) < 1e-6
    assert abs(got["r_measured"] / got["r_predicted"] - 1) < 0.1


def test_int_one_scale_per_long_row(ss, ws):
    """Rows of several hundred chunks: the row-block kernel with 256 threads per row."""
    for pattern in (0, 24, 48):
        xh, _ = synth.linear_input(21, 4352, seed=5)
        compare(ss, ws, xh, pattern=pattern, fmt="int", bits=8, group=0)
        xf = synth.gaussian_f32(13, 3072, seed=6)
        compare(ss, ws, xf, pattern=pattern, fmt="int", bits=6, group=0)


def test_division_matches_ieee_for_every_significand_pair(ss):
    """The kernels' corrected-reciprocal division against IEEE division: every
    pair of significands (2^46 quotients), then pairs spread over the exponent
    range where the kernels use it."""
    bad, first = ss.selfcheck_division(mode=0)
    assert bad == 0, f"first mismatch a, b bits = {first}"
    bad, first = ss.selfcheck_division(mode=1, b_count=1 << 12, chunk=1 << 12)
    assert bad == 0, f"first mismatch a, b bits = {first}"


def test_packed_bf16_operations_for_every_pair_of_magnitudes(ss):
    """The packed comparison, maximum, conversion and squares behind the bf16
    2:4 selection and amax, for every pair of finite bf16 magnitudes."""
    bad, first = ss.selfcheck_division(mode=2, b_first=0, b_count=1 << 15, chunk=1 << 15)
    assert bad == 0, f"first mismatch (a, b) = {first}"


@pytest.mark.parametrize("k", [8, 16, 24, 40, 96, 136, 264])
@pytest.mark.parametrize("pattern", [0, 24])
def test_small_and_ragged_k(ss, ws, pattern, k):
    """k below the tile width (zero-filled box) and k with a partial last tile."""
    xh = synth.ties_and_specials(33, k, seed=k) if k >= 12 else synth.gaussian_bf16(33, k, seed=k)
    fmt = "fp8" if pattern == 24 else "int"
    compare(ss, ws, xh, pattern=pattern, fmt=fmt, bits=8, group=8 if pattern == 0 else 4)
    if pattern == 24:
        compare(ss, ws, xh, pattern=24, fmt="none")


@pytest.mark.parametrize("rows", [1, 2, 31, 33, 257])
def test_ragged_rows(ss, ws, rows):
    xh = synth.gaussian_bf16(rows, 64, seed=rows)
    compare(ss, ws, xh, pattern=24, fmt="nvfp4")
    compare(ss, ws, xh, pattern=48, fmt="mxfp4")


def test_ties_specials_every_format(ss, ws):
    xh = synth.ties_and_specials(64, 256, seed=4)
    for fmt, bits, group, pack4 in FORMATS:
        compare(ss, ws, xh, pattern=24, fmt=fmt, bits=bits, group=group, pack4=pack4)
        compare(ss, ws, xh, pattern=48, fmt=fmt, bits=bits, group=group, pack4=pack4)


def test_row_stride_larger_than_k(ss, ws):
    full = synth.sweep_operand(50, 640, seed=12)
    compare(ss, ws, full, pattern=24, fmt="nvfp4", k=512)
    compare(ss, ws, full, pattern=0, fmt="int", bits=8, group=0, k=512)


def test_given_tensor_scale_and_saturation(ss, ws):
    xh = synth.sweep_operand(64, 512, seed=13)
    # a scale 16x too small saturates the largest values to +-448 / +-6
    s_fp8 = oracle.tensor_scale(xh, "fp8") / 16.0
    compare(ss, ws, xh, pattern=24, fmt="fp8", tensor_scale=s_fp8)
    compare(ss, ws, xh, pattern=0, fmt="fp8", tensor_scale=s_fp8)
    s_nv = oracle.tensor_scale(xh, "nvfp4") / 1e4
    compare(ss, ws, xh, pattern=24, fmt="nvfp4", tensor_scale=s_nv)
    compare(ss, ws, xh, pattern=0, fmt="nvfp4", tensor_scale=0.0)


def test_fp8_given_scale_overflow_guard(ss, ws):
    """Given FP8 scales tiny enough that v / s leaves the binary32 range for
    part of the values: the per-chunk guard (a bf16 threshold for bf16 input)
    must send exactly those chunks to IEEE division."""
    rng = np.random.default_rng(21)
    mag = np.exp2(rng.uniform(-10.0, 20.0, size=(40, 512))).astype(np.float32)
    xf = (mag * rng.choice([-1.0, 1.0], size=mag.shape)).astype(np.float32)
    xh = synth.bf16_bits(xf)
    for s in (2.0 ** -120, 2.0 ** -108, 2.0 ** -100, 2.0 ** -61, 2.0 ** -59, 3.0, 5.0):
        compare(ss, ws, xh, pattern=24, fmt="fp8", tensor_scale=s)
        compare(ss, ws, xh, pattern=0, fmt="fp8", tensor_scale=s)
    compare(ss, ws, xf, pattern=24, fmt="fp8", tensor_scale=2.0 ** -110)


def test_int_with_tiny_and_subnormal_scales(ss, ws):
    """Groups whose amax is tiny give subnormal scales: the IEEE-division path
    and the clamp of the definition."""
    rng = np.random.default_rng(17)
    x = rng.standard_normal((16, 256)).astype(np.float32)
    x[0::2] *= np.float32(2.0 ** -135)        # subnormal values, subnormal scales
    x[1::4] *= np.float32(2.0 ** -100)        # tiny normal values
    for pattern in (0, 24):
        compare(ss, ws, x, pattern=pattern, fmt="int", bits=8, group=32 if pattern == 0 else 16)
        compare(ss, ws, x, pattern=pattern, fmt="int", bits=4, group=0)
        compare(ss, ws, x, pattern=pattern, fmt="mxfp4")


def test_signed_zeros_keep_their_sign(ss, ws):
    """-0 and +0 quantize to the signed-zero codes IEEE division gives them."""
    x = np.zeros((8, 64), dtype=np.uint16)
    x[:, 0::3] = 0x8000                       # -0
    x[:, 1::5] = synth.bf16_bits(np.float32([[1.5]]))[0, 0]
    x[:, 2::7] = synth.bf16_bits(np.float32([[-3.0]]))[0, 0]
    for fmt in ("fp8", "nvfp4", "int", "mxfp4"):
        compare(ss, ws, x, pattern=24, fmt=fmt, bits=8, group=16)
        compare(ss, ws, x, pattern=0, fmt=fmt, bits=8, group=16)


def test_all_zero_operand(ss, ws):
    xh = np.zeros((40, 256), dtype=np.uint16)
    for fmt, bits, group, pack4 in FORMATS:
        compare(ss, ws, xh, pattern=24, fmt=fmt, bits=bits, group=group, pack4=pack4)
    compare(ss, ws, xh, pattern=0, fmt="nvfp4")
    compare(ss, ws, xh, pattern=0, fmt="mxfp4")


def test_empty_operand(ss, ws):
    x = torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda")
    out = ss.run(x, pattern=24, fmt="fp8", ws=ws)
    torch.cuda.synchronize()
    assert out["energy"].abs().sum().item() == 0.0
    assert out["tensor_scale"].item() == 0.0


def test_amax_and_error_energy_and_ratio(ss, ws):
    w, norms = synth.linear_weight(96, 512, seed=2)
    wd, nd = to_dev(w), to_dev(norms)
    for score, nrm in (("mag", None), ("wanda", norms)):
        sc = oracle.WANDA if score == "wanda" else oracle.MAG
        a = ss.amax(wd, pattern=24, score=score, col_norms=nd if nrm is not None else None, ws=ws)
        assert a.item() == oracle.amax(w, score=sc, norms=nrm)
        for sfmt, dfmt in [(("int", 8, 128), ("int", 5, 128)), (("fp8",), ("nvfp4",)), (("none",), ("mxfp4",)),
                           (("nvfp4",), ("fp8",)), (("int", 4, 64, True), ("int", 3, 64))]:
            e = ss.error_energy(wd, pattern=24, sparse_fmt=sfmt, dense_fmt=dfmt, score=score,
                                col_norms=nd if nrm is not None else None, ws=ws)
            sp = oracle.run(w, fmt=sfmt[0], bits=(sfmt[1] if len(sfmt) > 1 else 8),
                            group=(sfmt[2] if len(sfmt) > 2 else 0), pack4=(len(sfmt) > 3 and sfmt[3]),
                            score=sc, norms=nrm)["energy"]
            de = oracle.run(w, pattern=oracle.DENSE, fmt=dfmt[0], bits=(dfmt[1] if len(dfmt) > 1 else 8),
                            group=(dfmt[2] if len(dfmt) > 2 else 0))["energy"]
            ref = np.array([sp[0], sp[1], sp[2], de[3]])
            assert_energy(e, ref)
            r = ss.predicted_ratio(e, e)
            rr = oracle.ratio(ref, ref)
            r2 = ss.predicted_ratio(torch.stack([e, e]), torch.stack([e, e]))
            assert torch.equal(r2[0], r) and torch.equal(r2[1], r)
            np.testing.assert_allclose(r.cpu().numpy(), rr, rtol=2e-6)
    assert ws.error() == 0


# the read-only energy pass on bf16 full-width rows (k >= 1024, a multiple of
# 64): every pair of a 2:4 side's format and a dense side's format, with INT
# groups inside one lane and across lanes, a ragged last unit (k = 4608) and
# given per-tensor scales, one of them small enough that the quotients leave
# the fast division's range
LB_SPARSE = [("none",), ("fp8",), ("nvfp4",), ("mxfp4",), ("int", 8, 4), ("int", 8, 128), ("int", 4, 16, True),
             ("int", 12, 64)]
LB_DENSE = [("fp8",), ("nvfp4",), ("mxfp4",), ("int", 8, 8), ("int", 5, 256), ("int", 3, 32), ("int", 16, 64)]


def _fmt_kw(f):
    return dict(fmt=f[0], bits=(f[1] if len(f) > 1 else 8), group=(f[2] if len(f) > 2 else 0),
                pack4=(len(f) > 3 and f[3]))


@pytest.mark.parametrize("k", [1024, 4608, 5120])
def test_error_energy_every_format_pair_full_width(ss, ws, k):
    xh, _ = synth.linear_input(24, k, seed=90 + k, n_outlier=16)
    x = to_dev(xh)
    sp = {f: oracle.run(xh, **_fmt_kw(f))["energy"] for f in LB_SPARSE}
    de = {f: oracle.run(xh, pattern=oracle.DENSE, **_fmt_kw(f))["energy"] for f in LB_DENSE}
    for sf in LB_SPARSE:
        for df in LB_DENSE:
            e = ss.error_energy(x, pattern=24, sparse_fmt=sf, dense_fmt=df, ws=ws)
            assert_energy(e, [sp[sf][0], sp[sf][1], sp[sf][2], de[df][3]])
    for s_given in (0.37, 2.0 ** -120):
        ts = torch.tensor([s_given], dtype=torch.float32, device="cuda")
        for sf, df in ((("fp8",), ("fp8",)), (("nvfp4",), ("nvfp4",)), (("fp8",), ("nvfp4",))):
            e = ss.error_energy(x, pattern=24, sparse_fmt=sf, dense_fmt=df, sparse_scale=ts, dense_scale=ts, ws=ws)
            a = oracle.run(xh, fmt=sf[0], tensor_scale=np.float32(s_given))["energy"]
            b = oracle.run(xh, pattern=oracle.DENSE, fmt=df[0], tensor_scale=np.float32(s_given))["energy"]
            assert_energy(e, [a[0], a[1], a[2], b[3]])
    assert ws.error() == 0


def test_repeated_calls_are_deterministic(ss, ws):
    xh, _ = synth.linear_input(300, 1024, seed=1)
    x = to_dev(xh)
    outs = [ss.run(x, pattern=24, fmt="fp8", ws=ws) for _ in range(3)]
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert torch.equal(o["values"], outs[0]["values"])
        assert torch.equal(o["energy"], outs[0]["energy"])


# --------------------------------------------------------------------------
# full-size configurations: every output of the whole tensor against the
# oracle (run on all host cores, row blocks), all four energies to 1e-6
# --------------------------------------------------------------------------

def full_check(ss, ws, xh, *, pattern, fmt, bits=8, group=0, pack4=False, score="mag", norms=None):
    """One pass over the whole operand on the GPU (tensor scale derived by the
    library when the format has one) against oracle.run_parallel on the same
    bytes: codes, scales, metadata and tensor scale bit for bit, the four
    energies within 1e-6 relative."""
    x = to_dev(xh)
    nd = to_dev(norms) if norms is not None else None
    out = ss.run(x, pattern=pattern, fmt=fmt, bits=bits, group=group, pack4=pack4, score=score, col_norms=nd, ws=ws)
    torch.cuda.synchronize()
    assert ws.error() == 0
    got = {key: to_np(t) for key, t in out.items() if key != "energy"}
    energy = out["energy"]
    del out, x
    sc = oracle.WANDA if score == "wanda" else oracle.MAG
    opat = {0: oracle.DENSE, 24: oracle.SPARSE_24, 48: oracle.SPARSE_48}[pattern]
    ref = oracle.run_parallel(xh, pattern=opat, fmt=fmt, bits=bits, group=group, pack4=pack4, score=sc,
                              norms=norms)
    for key in ("values", "scales", "meta", "tensor_scale"):
        if key in ref:
            assert_same(got[key], ref[key], key)
    assert_energy(energy, ref["energy"], atol=1e-30)
    return energy.cpu().numpy()


def test_full_linear_input_fp8_and_int8_per_row(ss, ws):
    """Linear input X 4096 x 4096 (Student-t, 8 outlier channels x50): fused
    2:4 + FP8 and its dense FP8 and INT8-per-row partners."""
    xh, _ = synth.linear_input(4096, 4096, seed=1)
    e = full_check(ss, ws, xh, pattern=24, fmt="fp8")
    assert 0.0 < e[1] / e[0] < 0.5
    full_check(ss, ws, xh, pattern=0, fmt="fp8")
    full_check(ss, ws, xh, pattern=0, fmt="int", bits=8, group=0)


def test_full_weight_wanda_int(ss, ws):
    """Linear weight W 14336 x 4096 with Wanda scores: 2:4 + INT(2m) g128 against
    dense INT(m+1) g128, m = 2, 4, 8 (INT4 packed, INT8, INT16; INT3 packed,
    INT5, INT9)."""
    w, norms = synth.linear_weight(14336, 4096, seed=2)
    for m in (2, 4, 8):
        full_check(ss, ws, w, pattern=24, fmt="int", bits=2 * m, group=128, pack4=m == 2, score="wanda",
                   norms=norms)
        full_check(ss, ws, w, pattern=0, fmt="int", bits=m + 1, group=128, pack4=m == 2)


def test_full_attention_operands(ss, ws):
    """Q (32 heads x 8192 x 128) pruned along d: 2:4 + FP8 against dense NVFP4
    and MXFP4; P (32 x 2048 x 2048) pruned along the keys: 2:4 + FP8."""
    q = synth.attention_qkv(seed=4)
    full_check(ss, ws, q, pattern=24, fmt="fp8")
    full_check(ss, ws, q, pattern=0, fmt="nvfp4")
    full_check(ss, ws, q, pattern=0, fmt="mxfp4")
    p = synth.attention_probs(seed=7)
    full_check(ss, ws, p, pattern=24, fmt="fp8")


def test_full_attention_softmax_prune(ss, ws):
    """P = softmax(logits / sqrt(128)) for 32 heads x 2048 x 2048 keys, pruned
    2:4 + FP8 in its producer: sampled rows against the oracle's softmax and
    pass, bit for bit; energies by properties."""
    s = synth.attention_logits(seed=9)
    alpha = float(np.float32(1.0 / math.sqrt(128)))
    ts = torch.tensor([1.0 / 448.0], device="cuda")
    out = ss.softmax_prune(to_dev(s), alpha, pattern=24, fmt="fp8", tensor_scale=ts, ws=ws)
    torch.cuda.synchronize()
    rng = np.random.default_rng(10)
    rows = np.unique(np.concatenate([[0, s.shape[0] - 1], rng.integers(0, s.shape[0], 16)]))
    ref = oracle.run(oracle.softmax_bf16(s[rows], alpha), pattern=oracle.SPARSE_24, fmt="fp8",
                     tensor_scale=float(np.float32(1.0 / 448.0)))
    sel = torch.from_numpy(rows).cuda()
    assert_same(to_np(out["values"][sel]), ref["values"], "values")
    assert_same(to_np(out["meta"][sel]), ref["meta"], "meta")
    e = out["energy"].cpu().numpy()
    # each row of P sums to ~1 with 2048 near-equal entries: E_total ~ rows / 2048
    assert 0.5 * s.shape[0] / 2048 < e[0] < 2.0 * s.shape[0] / 2048
    assert 0.0 < e[1] / e[0] < 0.5 and 0.0 < e[2] < e[1]
    assert ws.error() == 0


def _bf16_ulp(v):
    """Spacing of bf16 values at |v| (2^-133 below the normal range)."""
    e = np.floor(np.log2(np.maximum(np.abs(v), 2.0 ** -126)))
    return np.exp2(e - 7.0)


def _meta24_of(p):
    """Metadata of 2:4 selection by magnitude on p [rows, k] (ties keep the lower
    index): one nibble i0 | i1 << 2 per group, two groups per byte."""
    g = np.abs(p.reshape(p.shape[0], -1, 4))
    beaten = np.zeros(g.shape, dtype=np.int32)
    for i in range(4):
        for j in range(4):
            if i != j:
                beaten[..., i] += (g[..., j] > g[..., i]) | ((g[..., j] == g[..., i]) & (j < i))
    kept = beaten < 2
    idx = np.argsort(~kept, axis=-1, kind="stable")[..., :2]            # kept positions, ascending
    nib = (idx[..., 0] | (idx[..., 1] << 2)).astype(np.uint8)
    return (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)


def test_full_softmax_prune_against_binary64_softmax(ss, ws):
    """The softmax producer checked against the plain definition, independently
    of the exponential and summation order it fixes: P for 32 heads x 2048 x
    2048 keys (logits N(0, 3^2), alpha = 1/sqrt(128)) pruned 2:4 with bf16
    kept values, against softmax in binary64 (libm exp, index-order sum)
    rounded once to bf16:
      - every kept value within one bf16 ulp of the binary64 P at its position;
      - the metadata equal to the selection on the binary64 P in every group
        whose second and third largest values are further apart than the sum
        of their ulps (where one ulp of error each cannot swap them);
      - E_total within 2^-6 relative of the binary64 P's energy."""
    import oracle as orc
    s = synth.attention_logits(seed=9)
    alpha = float(np.float32(1.0 / math.sqrt(128)))
    out = ss.softmax_prune(to_dev(s), alpha, pattern=24, fmt="none", ws=ws)
    torch.cuda.synchronize()
    assert ws.error() == 0
    kept = (to_np(out["values"]).astype(np.uint32) << 16).view(np.float32)
    meta = to_np(out["meta"])
    e_total = out["energy"].cpu().numpy()[0]
    del out
    pref = orc.softmax_f64_bf16(s, alpha, threads=orc.host_threads())
    rows, k = pref.shape
    checked = total = 0
    e_ref = 0.0
    for r0 in range(0, rows, 4096):
        r1 = min(rows, r0 + 4096)
        p = (pref[r0:r1].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        e_ref += float(np.einsum("ij,ij->", p, p))
        m = meta[r0:r1]
        nib = np.stack([m & 0xF, m >> 4], axis=-1).reshape(r1 - r0, -1)      # [rows, groups]
        i0, i1 = nib & 3, nib >> 2
        g = p.reshape(r1 - r0, -1, 4)
        at = np.stack([np.take_along_axis(g, i0[..., None], -1)[..., 0],
                       np.take_along_axis(g, i1[..., None], -1)[..., 0]], axis=-1).reshape(r1 - r0, -1)
        kv = kept[r0:r1].astype(np.float64)
        assert np.all(np.abs(kv - at) <= _bf16_ulp(at)), "a kept value is more than one bf16 ulp off"
        srt = -np.sort(-g, axis=-1)
        sep = (srt[..., 1] - srt[..., 2]) > _bf16_ulp(srt[..., 1]) + _bf16_ulp(srt[..., 2])
        ref_meta = _meta24_of(p)
        ref_nib = np.stack([ref_meta & 0xF, ref_meta >> 4], axis=-1).reshape(r1 - r0, -1)
        assert np.array_equal(nib[sep], ref_nib[sep]), "selection differs where the order is not in doubt"
        checked += int(sep.sum())
        total += sep.size
    assert checked > 0.9 * total
    assert abs(e_total - e_ref) <= 2.0 ** -6 * e_ref


@pytest.mark.parametrize("tokens,k", [(2048, 4096), (16384, 14336)])
def test_full_sweep_nvfp4(ss, ws, tokens, k):
    """The throughput sweep's smallest and largest shapes (0.1% outliers x100):
    2:4 + NVFP4, pairwise 4:8 + NVFP4 and 2:4 with bf16 kept values, whole
    tensors."""
    xh = synth.sweep_operand(tokens, k, seed=8)
    full_check(ss, ws, xh, pattern=24, fmt="nvfp4")
    full_check(ss, ws, xh, pattern=48, fmt="nvfp4")
    full_check(ss, ws, xh, pattern=24, fmt="none")
    full_check(ss, ws, xh, pattern=0, fmt="nvfp4")
    full_check(ss, ws, xh, pattern=24, fmt="mxfp4")
    full_check(ss, ws, xh, pattern=0, fmt="mxfp4")


def test_full_sweep_error_energy(ss, ws):
    """The read-only energy pass over the largest sweep operand (16384 x
    14336) for two format pairs, against the oracle's sparse and dense passes
    over the whole tensor: all four energies within 1e-6 relative."""
    xh = synth.sweep_operand(16384, 14336, seed=9)
    x = to_dev(xh)
    for sf, df in ((("nvfp4",), ("nvfp4",)), (("fp8",), ("int", 5, 128))):
        e = ss.error_energy(x, pattern=24, sparse_fmt=sf, dense_fmt=df, ws=ws)
        torch.cuda.synchronize()
        sp = oracle.run_parallel(xh, pattern=oracle.SPARSE_24, **_fmt_kw(sf))["energy"]
        de = oracle.run_parallel(xh, pattern=oracle.DENSE, **_fmt_kw(df))["energy"]
        assert_energy(e, [sp[0], sp[1], sp[2], de[3]])
    assert ws.error() == 0
