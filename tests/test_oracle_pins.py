"""Pins of the CPU oracle to things other than itself.

Each test checks one oracle function against brute force, a library routine,
a closed form, an invariant, or a figure printed on the pages ("Is 2:4
Sparsity Still Worth It? Semi-Structured Sparsity versus Quantization in LLM
Inference"; figures in tests/golden/). None of these tests needs a GPU.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy import integrate, special

import oracle
from semi_structured_sparsity_online_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
FIG = json.load(open(os.path.join(GOLDEN, "paper_figures.json")))


# --------------------------------------------------------------------------
# helpers written independently of the oracle (decoders and brute force)
# --------------------------------------------------------------------------

def brute_keep24(s):
    """Brute force over the six 2-of-4 masks: a mask is valid when every kept
    score is >= every dropped score; the lexicographically smallest valid
    (i0, i1) is the lower-index tie rule. Comparisons only."""
    for i0, i1 in itertools.combinations(range(4), 2):
        kept = (s[i0], s[i1])
        dropped = [s[j] for j in range(4) if j not in (i0, i1)]
        if all(a >= b for a in kept for b in dropped):
            return i0, i1
    raise AssertionError("no valid mask")


def unpack_meta(meta, k, group):
    """Decode metadata bytes [rows, k/(2*group)] to kept index pairs per group."""
    rows = meta.shape[0]
    ng = k // group
    nib = np.zeros((rows, ng), dtype=np.uint8)
    nib[:, 0::2] = meta & 0xF
    nib[:, 1::2] = meta >> 4
    return nib & 3, nib >> 2


def mask24_from_meta(meta, k):
    i0, i1 = unpack_meta(meta, k, 4)
    rows, ng = i0.shape
    mask = np.zeros((rows, k), dtype=bool)
    base = np.arange(ng) * 4
    r = np.arange(rows)[:, None]
    mask[r, base + i0] = True
    mask[r, base + i1] = True
    return mask


def mask48_from_meta(meta, k):
    p0, p1 = unpack_meta(meta, k, 8)
    rows, no = p0.shape
    mask = np.zeros((rows, k), dtype=bool)
    base = np.arange(no) * 8
    r = np.arange(rows)[:, None]
    for p in (p0, p1):
        mask[r, base + 2 * p] = True
        mask[r, base + 2 * p + 1] = True
    return mask


def e4m3_decode_torch(codes):
    return torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn).float().numpy()


def e2m1_value(code):
    """E2M1 from its bit fields: normal (-1)^s 2^(e-1) (1 + m/2), subnormal (-1)^s m/2."""
    s, e, m = (code >> 3) & 1, (code >> 1) & 3, code & 1
    mag = (m / 2.0) if e == 0 else 2.0 ** (e - 1) * (1 + m / 2.0)
    return -mag if s else mag


E2M1_TABLE = np.array([e2m1_value(c) for c in range(16)], dtype=np.float64)


def gaussian_loss_closed_form():
    """(E[Y(1)] + E[Y(2)]) / 4 for the order statistics of four i.i.d. chi^2_1
    variables (the squares of N(0,1) draws), by numerical integration over the
    half-normal magnitude t: F(t) = erf(t/sqrt 2), density 2 phi(t)."""
    def order_mean(j, n=4):
        c = math.factorial(n) / (math.factorial(j - 1) * math.factorial(n - j))
        def f(t):
            F = special.erf(t / math.sqrt(2.0))
            dens = 2.0 * math.exp(-t * t / 2.0) / math.sqrt(2.0 * math.pi)
            return t * t * c * F ** (j - 1) * (1.0 - F) ** (n - j) * dens
        return integrate.quad(f, 0.0, np.inf, epsabs=1e-13, epsrel=1e-12)[0]
    return (order_mean(1) + order_mean(2)) / 4.0


# --------------------------------------------------------------------------
# selection
# --------------------------------------------------------------------------

def test_select24_exhaustive_small_alphabet():
    alphabet = [0.0, -0.0, 1.0, -1.0, 2.0, -2.0, 3.0, -3.0]
    for t in itertools.product(alphabet, repeat=4):
        s = [abs(v) for v in t]
        nib = oracle.select24(s)
        assert (nib & 3, nib >> 2) == brute_keep24(s), t


def test_select24_random_scores_brute_force():
    rng = np.random.default_rng(5)
    for _ in range(4000):
        s = np.abs(rng.standard_normal(4).astype(np.float32))
        if rng.random() < 0.3:  # force ties
            s[rng.integers(4)] = s[rng.integers(4)]
        nib = oracle.select24(s)
        assert (nib & 3, nib >> 2) == brute_keep24(list(s))


def test_select48_brute_force_over_pair_masks():
    rng = np.random.default_rng(6)
    for trial in range(3000):
        if trial % 3 == 0:
            s = rng.integers(0, 3, size=8).astype(np.float32)
        else:
            s = np.abs(rng.standard_normal(8).astype(np.float32))
        e = (s[0::2] * s[0::2] + s[1::2] * s[1::2]).astype(np.float32)
        nib = oracle.select48(s)
        assert (nib & 3, nib >> 2) == brute_keep24(list(e))


def test_worked_example_layout():
    """Hand-derived example: kept order, nibble order and byte order."""
    lines = {}
    for ln in open(os.path.join(GOLDEN, "worked_example_24.txt")):
        if ln.startswith("#") or ":" not in ln:
            continue
        key, val = ln.split(":", 1)
        lines[key.strip()] = val.split()
    x = np.array([float(v) for v in lines["x"]], dtype=np.float32)[None, :]
    out = oracle.run(synth.bf16_bits(x), fmt="none")
    kept = synth.bf16_to_f32(out["values"])[0]
    assert kept.tolist() == [float(v) for v in lines["kept"]]
    assert out["meta"][0].tolist() == [int(v, 16) for v in lines["meta"]]
    assert out["energy"][0] == float(lines["e_total"][0])
    assert out["energy"][1] == float(lines["e_prune"][0])
    out32 = oracle.run(x, fmt="none")
    assert out32["values"][0].tolist() == [float(v) for v in lines["kept"]]


def test_compress_roundtrip_and_nibble_codes():
    x = synth.ties_and_specials(24, 256, seed=3)
    out = oracle.run(x, fmt="none")
    mask = mask24_from_meta(out["meta"], 256)
    assert (mask.sum(axis=1) == 128).all()
    # decompress(kept, meta) == x * mask, bit for bit
    dense = np.zeros_like(x)
    dense[mask] = out["values"].reshape(-1)
    assert np.array_equal(dense, np.where(mask, x, 0))
    nibs = np.concatenate([(out["meta"] & 0xF).ravel(), (out["meta"] >> 4).ravel()])
    assert set(np.unique(nibs).tolist()) <= {0x4, 0x8, 0xC, 0x9, 0xD, 0xE}


def test_wanda_scores_select_by_product():
    rng = np.random.default_rng(9)
    x = synth.gaussian_bf16(16, 64, seed=4)
    norms = np.exp(rng.standard_normal(64)).astype(np.float32)
    out = oracle.run(x, score=oracle.WANDA, norms=norms, fmt="none")
    s = np.abs(synth.bf16_to_f32(x)) * norms[None, :]
    i0, i1 = unpack_meta(out["meta"], 64, 4)
    for r in range(16):
        for g in range(16):
            assert (i0[r, g], i1[r, g]) == brute_keep24(list(s[r, 4 * g:4 * g + 4]))
    # unit norms reduce Wanda to magnitude
    ones = np.ones(64, dtype=np.float32)
    a = oracle.run(x, score=oracle.WANDA, norms=ones, fmt="none")
    b = oracle.run(x, fmt="none")
    assert np.array_equal(a["meta"], b["meta"]) and np.array_equal(a["values"], b["values"])


def test_axis0_is_the_transpose():
    x = synth.gaussian_bf16(64, 40, seed=12)         # logical A[40 rows][64 k], stored [k][rows]
    a = oracle.run(x, axis=0, fmt="nvfp4")
    b = oracle.run(np.ascontiguousarray(x.T), axis=1, fmt="nvfp4")
    for key in ("values", "scales", "meta", "tensor_scale", "energy"):
        assert np.array_equal(a[key], b[key]), key


# --------------------------------------------------------------------------
# number formats
# --------------------------------------------------------------------------

def _probe_floats(n_random=200000, limit=None, seed=0):
    rng = np.random.default_rng(seed)
    allbf = synth.bf16_to_f32(np.arange(65536, dtype=np.uint16))
    allbf = allbf[np.isfinite(allbf)]
    rnd = rng.integers(0, 2 ** 32, size=n_random, dtype=np.uint64).astype(np.uint32).view(np.float32)
    rnd = rnd[np.isfinite(rnd)]
    v = np.concatenate([allbf, rnd]).astype(np.float32)
    if limit is not None:
        v = v[np.abs(v) <= limit]
    return v


def test_e4m3_encode_matches_torch_rounding():
    """Below the saturation edge the encoder equals torch's float8_e4m3fn cast
    (round to nearest even); midpoints and +-1 ulp around them included."""
    v = _probe_floats(limit=464.0)
    codes = np.arange(256, dtype=np.uint8)
    vals = e4m3_decode_torch(codes).astype(np.float32)
    fin = np.sort(np.unique(np.abs(vals[np.isfinite(vals)])))
    mids = ((fin[1:].astype(np.float64) + fin[:-1]) / 2).astype(np.float32)
    around = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9))])
    v = np.concatenate([v, around, -around]).astype(np.float32)
    want = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(t) for t in v], dtype=np.uint8)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(float(v[i]), int(got[i]), int(want[i])) for i in bad[:5]]


def test_e4m3_saturates_and_decodes():
    for t in (448.0, 464.0, 465.0, 1e6, 3e38):
        assert oracle.e4m3_encode(t) == 0x7E and oracle.e4m3_encode(-t) == 0xFE
    vals = e4m3_decode_torch(np.arange(256, dtype=np.uint8))
    for c in range(256):
        d = oracle.e4m3_decode(c)
        if np.isnan(vals[c]):
            assert math.isnan(d)
        else:
            assert d == vals[c] and math.copysign(1, d) == math.copysign(1, vals[c])
            assert oracle.e4m3_encode(d) == c


def test_e2m1_encode_is_nearest_even_saturating():
    v = np.concatenate([_probe_floats(n_random=50000, limit=20.0, seed=1),
                        np.arange(-7.0, 7.0, 0.125, dtype=np.float32)]).astype(np.float32)
    for t in v:
        c = oracle.e2m1_encode(t)
        mags = np.abs(E2M1_TABLE[:8])
        a = min(abs(float(t)), 6.0)
        d = np.abs(mags - a)
        best = np.nonzero(d == d.min())[0]
        want = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]
        assert (c & 7) == want, (t, c)
        assert (c >> 3) == (1 if math.copysign(1.0, float(t)) < 0 else 0)
    for c in range(16):
        assert oracle.e2m1_decode(c) == E2M1_TABLE[c]


def test_floor_log2_bracket():
    v = np.abs(_probe_floats(n_random=100000, seed=2))
    v = v[(v > 0) & np.isfinite(v)]
    for a in v[::7]:
        e = oracle.floor_log2(a)
        assert math.ldexp(1.0, e) <= float(a) < math.ldexp(1.0, e + 1)


# --------------------------------------------------------------------------
# quantizers
# --------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [2, 3, 4, 5, 8, 12, 16])
@pytest.mark.parametrize("group", [0, 32, 128])
def test_int_codes_are_nearest_grid_points(bits, group):
    x = synth.gaussian_bf16(8, 512, seed=bits)
    out = oracle.run(x, pattern=oracle.DENSE, fmt="int", bits=bits, group=group)
    v = synth.bf16_to_f32(x)
    g = group or 512
    qmax = 2 ** (bits - 1) - 1
    scales = out["scales"]
    codes = out["values"].astype(np.int64)
    for r in range(8):
        for j in range(512):
            s = np.float32(scales[r, j // g])
            amax = np.float32(np.abs(v[r, (j // g) * g:(j // g + 1) * g]).max())
            assert s == np.float32(amax / np.float32(qmax))
            q = np.float64(np.float32(v[r, j]) / s)            # the binary32 quotient
            cand = np.arange(-qmax, qmax + 1)
            d = np.abs(cand - q)
            best = cand[d == d.min()]
            want = best[0] if len(best) == 1 else best[best % 2 == 0][0]
            assert codes[r, j] == want


def test_int_special_cases_and_packing():
    x = np.zeros((2, 64), dtype=np.float32)
    x[0, :32] = 0.75
    x[0, 32:] = -0.75
    out = oracle.run(x, pattern=oracle.DENSE, fmt="int", bits=4, group=32)
    assert (out["values"][0, :32] == 7).all() and (out["values"][0, 32:] == -7).all()
    assert (out["values"][1] == 0).all() and (out["scales"][1] == 0).all()
    assert out["energy"][3] == 0.0
    p = oracle.run(x, pattern=oracle.DENSE, fmt="int", bits=4, group=32, pack4=True)
    lo = (p["values"] & 0xF).astype(np.int8)
    hi = (p["values"] >> 4).astype(np.int8)
    lo = np.where(lo > 7, lo - 16, lo)
    hi = np.where(hi > 7, hi - 16, hi)
    unpacked = np.stack([lo, hi], axis=-1).reshape(2, 64)
    assert np.array_equal(unpacked, out["values"])


def test_fp8_codes_are_nearest_and_scaled_by_amax():
    x = synth.gaussian_bf16(16, 256, seed=21)
    out = oracle.run(x, fmt="fp8")
    kept = synth.bf16_to_f32(oracle.run(x, fmt="none")["values"])
    amax = np.float32(np.abs(kept).max())
    s = out["tensor_scale"][0]
    assert s == np.float32(amax / np.float32(448.0))
    dec = e4m3_decode_torch(np.arange(256, dtype=np.uint8)).astype(np.float64)
    fin = np.isfinite(dec)
    q = (kept / s).astype(np.float32).astype(np.float64)
    codes = out["values"]
    for qq, c in zip(q.ravel()[::5], codes.ravel()[::5]):
        d = np.where(fin, np.abs(dec - qq), np.inf)
        best = np.nonzero(d == d.min())[0]
        if len(best) > 1:
            best = [b for b in best if b % 2 == 0 and math.copysign(1, dec[b]) == math.copysign(1, qq)]
        assert dec[c] == dec[best[0]]
    # the largest kept magnitude maps to +-448
    assert abs(e4m3_decode_torch(codes).astype(np.float64)).max() == 448.0


def test_nvfp4_block_scales_and_codes_brute_force():
    x = synth.sweep_operand(8, 512, seed=30)
    out = oracle.run(x, pattern=oracle.DENSE, fmt="nvfp4")
    v = synth.bf16_to_f32(x).astype(np.float32)
    st = np.float32(out["tensor_scale"][0])
    assert st == np.float32(np.float32(np.abs(v).max()) / np.float32(2688.0))
    dec8 = e4m3_decode_torch(np.arange(128, dtype=np.uint8)).astype(np.float64)
    codes = np.stack([out["values"] & 0xF, out["values"] >> 4], axis=-1).reshape(8, 512)
    for r in range(8):
        for b in range(32):
            blk = v[r, 16 * b:16 * b + 16]
            bf = np.float32(np.float32(np.abs(blk).max() / np.float32(6.0)) / st)
            d = np.where(np.isfinite(dec8), np.abs(dec8 - np.float64(min(bf, 448.0))), np.inf)
            best = np.nonzero(d == d.min())[0]
            best = best[0] if len(best) == 1 else [c for c in best if c % 2 == 0][0]
            sb = out["scales"][r, b]
            assert sb == best
            denom = np.float32(dec8[sb] * st)
            for j in range(16):
                q = abs(float(np.float32(blk[j] / denom)))
                c = codes[r, 16 * b + j] & 7
                dd = np.abs(np.abs(E2M1_TABLE[:8]) - min(q, 6.0))
                cand = np.nonzero(dd == dd.min())[0]
                want = cand[0] if len(cand) == 1 else [t for t in cand if t % 2 == 0][0]
                assert c == want


def test_mxfp4_shared_exponent_and_exact_powers_of_two():
    x = synth.gaussian_bf16(4, 256, seed=31)
    out = oracle.run(x, pattern=oracle.DENSE, fmt="mxfp4")
    v = synth.bf16_to_f32(x)
    for r in range(4):
        for b in range(8):
            amax = float(np.abs(v[r, 32 * b:32 * b + 32]).max())
            e = int(out["scales"][r, b]) - 127
            assert 2.0 ** (e + 2) <= amax < 2.0 ** (e + 3)
    # powers of two within a block's range are exact: zero quantization error
    p = np.array([[2.0 ** j * s for j in range(-1, 3) for s in (1, -1)] * 4], dtype=np.float32)
    o = oracle.run(p, pattern=oracle.DENSE, fmt="mxfp4")
    assert o["energy"][3] == 0.0
    z = oracle.run(np.zeros((1, 64), np.float32), pattern=oracle.DENSE, fmt="mxfp4")
    assert (z["scales"] == 0).all() and (z["values"] == 0).all()


# --------------------------------------------------------------------------
# energies and the page figures
# --------------------------------------------------------------------------

def _decode_values(out, fmt, rows, n, bits=8, group=0):
    """Dequantize codes independently of the oracle (decoders above). The
    dequantized value is a binary32 product (code value times scale, rounded
    once), so each product is formed in float32 here too."""
    f32 = np.float32
    if fmt == "fp8":
        return (e4m3_decode_torch(out["values"]) * f32(out["tensor_scale"][0])).astype(np.float64)
    if fmt == "int":
        g = group or n
        return (out["values"].astype(f32) * np.repeat(out["scales"], g, axis=1)).astype(np.float64)
    codes = np.stack([out["values"] & 0xF, out["values"] >> 4], axis=-1).reshape(rows, n)
    mag = E2M1_TABLE[codes].astype(f32)
    if fmt == "nvfp4":
        denom = e4m3_decode_torch(out["scales"]) * f32(out["tensor_scale"][0])
        return (mag * np.repeat(denom, 16, axis=1)).astype(np.float64)
    return (mag * np.repeat(np.exp2(out["scales"].astype(f32) - f32(127.0)), 32, axis=1)).astype(np.float64)


@pytest.mark.parametrize("fmt,bits,group", [("fp8", 8, 0), ("int", 8, 64), ("int", 4, 0),
                                            ("nvfp4", 4, 0), ("mxfp4", 4, 0)])
def test_error_energies_add_exactly(fmt, bits, group):
    """E_total, E_prune and E_q against sums computed here from the decoded
    outputs; and (§4) E_prune + E_q equals the total 2:4 error energy."""
    rows, k = 16, 512
    x = synth.sweep_operand(rows, k, seed=40)
    out = oracle.run(x, fmt=fmt, bits=bits, group=group)
    xf = synth.bf16_to_f32(x).astype(np.float64)
    mask = mask24_from_meta(out["meta"], k)
    deq = _decode_values(out, fmt, rows, k // 2, bits, group)
    xhat = np.zeros_like(xf)
    xhat[mask] = deq.reshape(-1)
    e = out["energy"]
    assert e[0] == pytest.approx(np.sum(xf * xf), rel=1e-12)
    assert e[1] == pytest.approx(np.sum((xf * ~mask) ** 2), rel=1e-12)
    assert e[2] == pytest.approx(np.sum(((xf - xhat) * mask) ** 2), rel=1e-12)
    assert e[1] + e[2] == pytest.approx(np.sum((xf - xhat) ** 2), rel=1e-12)


def test_gaussian_energy_loss_closed_form_and_page_figure():
    closed = gaussian_loss_closed_form()
    assert closed == pytest.approx(FIG["energy_loss_24_gaussian"]["value"], abs=0.0005)
    x = synth.gaussian_f32(256, 1024, seed=0)
    e = oracle.run(x, fmt="none")["energy"]
    loss = e[1] / e[0]
    assert abs(loss - closed) < 0.003
    assert math.sqrt(loss) == pytest.approx(FIG["rel_err_24_from_loss"]["value"], abs=0.006)


def test_pairwise48_energy_loss_closed_form_and_page_figure():
    """Pair energies of Gaussian data are chi^2_2 (exponential, mean 2); the two
    smallest of four have means 2(1/4) and 2(1/4 + 1/3), so the loss is
    (5/3) / 8 = 5/24."""
    closed = 5.0 / 24.0
    assert closed == pytest.approx(FIG["energy_loss_48_pairwise_gaussian"]["value"], abs=0.0005)
    x = synth.gaussian_f32(1024, 1024, seed=1)
    e = oracle.run(x, pattern=oracle.SPARSE_48, fmt="none")["energy"]
    assert abs(e[1] / e[0] - closed) < 0.004
    out = oracle.run(x[:4], pattern=oracle.SPARSE_48, fmt="none")
    mask = mask48_from_meta(out["meta"], 1024)
    assert np.array_equal(out["values"].reshape(-1), x[:4][mask])


def test_dense_equal_bit_errors_match_page_figures():
    """Dense INT8 and INT3 (group 128) relative error on Gaussian data against
    the page's 0.6% and 27.4% (loose: the pages do not fix the scaling)."""
    x = synth.gaussian_f32(512, 1024, seed=2)
    for bits, key in ((8, "rel_err_dense_int8_gaussian"), (3, "rel_err_dense_int3_gaussian")):
        e = oracle.run(x, pattern=oracle.DENSE, fmt="int", bits=bits, group=128)["energy"]
        rel = math.sqrt(e[3] / e[0])
        assert rel == pytest.approx(FIG[key]["value"], rel=0.15)


def test_sparse_side_error_and_predicted_r_on_gaussian():
    """2:4 side stays at 36-37% across budgets; R_hat > 1 down to INT3 (§4:
    the two cross only below 3 bits); R_hat = rel_err_sparse / rel_err_dense."""
    x = synth.gaussian_f32(256, 1024, seed=3)
    lo, hi = FIG["rel_err_24_side_gaussian"]["low"], FIG["rel_err_24_side_gaussian"]["high"]
    for m in range(2, 9):
        sp = oracle.run(x, fmt="int", bits=2 * m, group=128)["energy"]
        de = oracle.run(x, pattern=oracle.DENSE, fmt="int", bits=m + 1, group=128)["energy"]
        loss, rs, rd, rhat = oracle.ratio(sp, de)
        assert lo - 0.01 <= rs <= hi + 0.01
        assert rhat > 1.0
        assert rhat == pytest.approx(rs / rd, rel=1e-12)
        assert loss == pytest.approx(sp[1] / sp[0], rel=1e-15)
        if m == 2:
            assert 1.25 < rhat < 1.45


def test_format_orderings():
    """§3: finer scales beat coarser (NVFP4 < MXFP4, INT8 g128 < INT8 per row);
    §6: pairwise 4:8 drops more energy than element-wise 2:4."""
    x, _ = synth.linear_input(256, 1024, seed=1)
    g = synth.gaussian_bf16(256, 1024, seed=5)
    for t in (x, g):
        nv = oracle.run(t, pattern=oracle.DENSE, fmt="nvfp4")["energy"][3]
        mx = oracle.run(t, pattern=oracle.DENSE, fmt="mxfp4")["energy"][3]
        assert nv < mx
        i128 = oracle.run(t, pattern=oracle.DENSE, fmt="int", bits=8, group=128)["energy"][3]
        irow = oracle.run(t, pattern=oracle.DENSE, fmt="int", bits=8, group=0)["energy"][3]
        assert i128 < irow
        l24 = oracle.run(t, fmt="none")["energy"]
        l48 = oracle.run(t, pattern=oracle.SPARSE_48, fmt="none")["energy"]
        assert l48[1] / l48[0] > l24[1] / l24[0]


def test_equal_bit_identity():
    """§2: half the values at 2m bits plus a 1-bit index per element equals
    m + 1 bits per element; 2:4 with 16-bit values costs more than FP8."""
    for m in range(1, 9):
        sp = oracle.bits_per_element("int", bits=2 * m, pattern=oracle.SPARSE_24)
        de = oracle.bits_per_element("int", bits=m + 1, pattern=oracle.DENSE)
        assert sp == de == m + 1
    for kept, dense in FIG["equal_bits_pairs"]["pairs"]:
        assert oracle.bits_per_element("int", bits=kept) == oracle.bits_per_element(
            "int", bits=dense, pattern=oracle.DENSE)
    assert oracle.bits_per_element("none") > oracle.bits_per_element("fp8", pattern=oracle.DENSE)
    # with scales: NVFP4 dense adds 8 bits per 16 values
    assert oracle.bits_per_element("nvfp4", pattern=oracle.DENSE, with_scales=True) == 4.5


def test_amax_of_kept_equals_amax_of_all_for_magnitude():
    x, _ = synth.linear_input(64, 512, seed=1)
    assert oracle.amax(x) == oracle.amax(x, pattern=oracle.DENSE)
    w, n = synth.linear_weight(64, 512)
    assert oracle.amax(w, score=oracle.WANDA, norms=n) <= oracle.amax(w, pattern=oracle.DENSE)


def test_encoder_step_tables_are_round_to_nearest_even_midpoints():
    """The bisected step tables (used to check the GPU encoders over all fp32
    patterns) sit exactly at the midpoints between neighbouring codes, the
    midpoint itself going to the code with an even significand."""
    import encoder_bounds as eb
    for bounds, decode, n in ((eb.e4m3_bounds(), oracle.e4m3_decode, 127),
                              (eb.e2m1_bounds(), oracle.e2m1_decode, 8)):
        vals = [decode(c) for c in range(n)]
        assert np.all(np.diff(bounds.astype(np.int64)) > 0)
        for i in range(n - 1):
            mid = np.float32((vals[i] + vals[i + 1]) / 2)          # exact: a few significant bits
            assert float(mid) == (vals[i] + vals[i + 1]) / 2
            mbits = int(np.array([mid], dtype=np.float32).view(np.uint32)[0])
            want = mbits if (i + 1) % 2 == 0 else mbits + 1         # tie goes to the even code
            assert int(bounds[i]) == want, (n, i)


DEQ_FORMATS = [("none", 8, 0, False), ("fp8", 8, 0, False), ("int", 8, 16, False), ("int", 4, 0, True),
               ("int", 12, 32, False), ("nvfp4", 4, 0, False), ("mxfp4", 4, 0, False)]


@pytest.mark.parametrize("pattern", [oracle.DENSE, oracle.SPARSE_24, oracle.SPARSE_48])
@pytest.mark.parametrize("fmt,bits,group,pack4", DEQ_FORMATS)
def test_dequantize_reproduces_the_error_energies(pattern, fmt, bits, group, pack4):
    """x_hat from the stored outputs: sum (x - x_hat)^2 is E_prune + E_q (sparse)
    or E_q,dense (dense), the energies the pass accumulated element by element
    (§4: the two errors land on disjoint elements). A wrong position, code,
    scale or product shows up as a different sum."""
    if fmt == "none" and pattern == oracle.DENSE:
        pytest.skip("format NONE is the plain 2:4 compression")
    xh = synth.linear_input(24, 256, seed=31, n_outlier=4)[0]
    out = oracle.run(xh, pattern=pattern, fmt=fmt, bits=bits, group=group, pack4=pack4)
    xhat = oracle.dequantize(out, rows=24, k=256, pattern=pattern, fmt=fmt, bits=bits, group=group, pack4=pack4)
    x = synth.bf16_to_f32(xh).astype(np.float64)
    err = float(np.sum((x - xhat.astype(np.float64)) ** 2))
    e = out["energy"]
    want = e[3] if pattern == oracle.DENSE else e[1] + e[2]
    assert abs(err - want) <= 1e-12 * want
    if pattern != oracle.DENSE:
        per_group = 4 if pattern == oracle.SPARSE_24 else 8
        nz = (xhat.reshape(24, -1, per_group) != 0).sum(axis=2)
        assert nz.max() <= per_group // 2      # at most the kept half of each group is non-zero
    if fmt == "none":
        kept = xhat != 0
        assert np.array_equal(xhat[kept], x[kept].astype(np.float32))


def _golden_scale_tiles(name):
    pts, total = [], None
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            if line.startswith("# total_bytes"):
                total = int(line.split()[2])
            elif line.strip() and not line.startswith("#"):
                pts.append(tuple(int(v) for v in line.split()))
    return total, pts


def test_scale_tiles_golden_offsets():
    """Hand-computed byte offsets of the block-scale tile layout."""
    total, pts = _golden_scale_tiles("scale_tiles_130x5.txt")
    assert oracle.lib().oracle_scale_tiles_bytes(130, 5) == total
    for r, c, off in pts:
        src = np.zeros((130, 5), dtype=np.uint8)
        src[r, c] = 0xA5
        out = oracle.scale_tiles(src, 130, 5)
        assert out.size == total
        assert np.flatnonzero(out).tolist() == [off], (r, c)


def test_scale_tiles_reshape_statement_and_padding():
    """The oracle's index arithmetic against the layout stated as tensor
    reshapes (pad, split rows into tiles of 4 x 32, swap the 4 and the 32),
    plus: zero padding, and every input byte stored exactly once."""
    rng = np.random.default_rng(5)
    for rows, cols, batch in ((1, 1, 1), (128, 4, 1), (130, 5, 2), (300, 17, 3), (7, 64, 1)):
        src = rng.integers(1, 256, size=(batch, rows, cols), dtype=np.uint8)
        got = oracle.scale_tiles(src, rows, cols, batch)
        rp, cp = -(-rows // 128) * 128, -(-cols // 4) * 4
        pad = np.zeros((batch, rp, cp), dtype=np.uint8)
        pad[:, :rows, :cols] = src
        t = pad.reshape(batch, rp // 128, 4, 32, cp // 4, 4)      # [b, rt, a, b32, ct, j]
        t = t.transpose(0, 1, 4, 3, 2, 5)                          # [b, rt, ct, b32, a, j]
        assert np.array_equal(got, t.reshape(-1)), (rows, cols, batch)
        assert np.count_nonzero(got) == src.size
        assert sorted(got[got != 0].tolist()) == sorted(src.reshape(-1).tolist())


def test_scale_tiles_rejects_bad_arguments():
    assert oracle.lib().oracle_scale_tiles_bytes(-1, 4) == -1
    assert oracle.lib().oracle_scale_tiles(None, 4, 4, 1, None) == -1
    assert oracle.lib().oracle_scale_tiles_bytes(0, 7) == 0


HADAMARD_BLOCKS = [2, 4, 8, 16, 32, 64, 128, 256]


@pytest.mark.parametrize("b", HADAMARD_BLOCKS)
def test_hadamard_unit_vectors_closed_form(b):
    """Each unit vector maps to a column of the Sylvester matrix, whose entry
    (j, i) is (-1)^popcount(i & j), times RN(1/sqrt(b)); other blocks stay 0."""
    k = 2 * b
    cb = np.float32(1.0 / math.sqrt(b))
    assert oracle.lib().oracle_hadamard_scale(b) == cb
    for i in sorted({0, 1, b // 2, b - 1, b, k - 1}):
        x = np.zeros((1, k), dtype=np.float32)
        x[0, i] = 1.0
        got = oracle.hadamard(x, b)[0]
        blk = (i // b) * b
        want = np.zeros(k, dtype=np.float32)
        for j in range(b):
            want[blk + j] = cb if bin((i - blk) & j).count("1") % 2 == 0 else -cb
        assert np.array_equal(got, want), (b, i)


@pytest.mark.parametrize("b", HADAMARD_BLOCKS)
def test_hadamard_against_library_matrix(b):
    """Against scipy.linalg.hadamard in binary64, within the rounding bound of
    log2(b) butterfly stages and the final scaling; and energy preserved."""
    from scipy.linalg import hadamard
    xh, _ = synth.linear_input(16, 1024, seed=71)
    x = ((xh.astype(np.uint32) << 16).view(np.float32)).astype(np.float64)
    got = oracle.hadamard(xh, b).astype(np.float64)
    H = hadamard(b).astype(np.float64) / math.sqrt(b)
    want = (x.reshape(16, -1, b) @ H.T).reshape(16, 1024)
    absx = np.abs(x).reshape(16, -1, b).sum(axis=2, keepdims=True) / math.sqrt(b)
    bound = ((math.log2(b) + 2) * 2.0 ** -24 * np.broadcast_to(absx, (16, 1024 // b, b))).reshape(16, 1024)
    assert np.all(np.abs(got - want) <= bound + 1e-45)
    assert abs((got ** 2).sum() / (x ** 2).sum() - 1) < 1e-5


def test_hadamard_is_an_involution_and_rejects_bad_blocks():
    xf = synth.gaussian_f32(8, 512, seed=72)
    for b in (8, 128):
        twice = oracle.hadamard(oracle.hadamard(xf, b), b)
        assert np.allclose(twice, xf, rtol=0, atol=1e-5 * np.abs(xf).max())
    for b in (0, 1, 3, 512):
        with pytest.raises(ValueError):
            oracle.hadamard(xf, b)
    with pytest.raises(ValueError):
        oracle.hadamard(synth.gaussian_f32(2, 24, seed=1), 16)   # k not a multiple of b


def test_exp_ss_within_one_ulp_of_libm():
    """The softmax exponential (Cody-Waite reduction, degree-7 Taylor
    polynomial) against libm's exp in binary64: at most 1 ulp of the binary32
    result where it is normal, one subnormal unit below; exact at 0; zero at
    and below -104."""
    L = oracle.lib()
    rng = np.random.default_rng(0)
    xs = np.concatenate([np.linspace(-104, 0, 20001, dtype=np.float32), -rng.exponential(4, 20000).astype(np.float32),
                         np.float32([-1e-30, -1e-8, -0.34657359, -0.34657362, -86.9, -87.0, -102.99, -103.5])])
    for x in xs[xs >= -104]:
        f, ref = L.oracle_exp_ss(float(x)), math.exp(float(x))
        if ref >= 2.0 ** -126:
            assert abs(f - ref) <= 2.0 ** (math.floor(math.log2(f)) - 23), x
        else:
            assert abs(f - ref) <= 2.0 ** -149, x
    assert L.oracle_exp_ss(0.0) == 1.0 and L.oracle_exp_ss(-104.0) == 0.0 and L.oracle_exp_ss(-1e30) == 0.0


def test_softmax_bf16_against_library_and_closed_forms():
    """P against scipy's softmax in binary64 (within bf16 rounding plus the
    binary32 steps), rows summing to 1, and two closed forms: a constant row
    gives exactly 1/k, and a row with one logit far above the rest gives 1 there."""
    from scipy.special import softmax
    rng = np.random.default_rng(3)
    s = (rng.standard_normal((6, 512)) * 3).astype(np.float32)
    alpha = 1.0 / math.sqrt(128)
    p = ((oracle.softmax_bf16(s, alpha).astype(np.uint32) << 16).view(np.float32)).astype(np.float64)
    ref = softmax(s.astype(np.float64) * np.float32(alpha), axis=1)
    assert np.all(np.abs(p - ref) <= 2.0 ** -8 * ref + 1e-38)
    assert np.all(np.abs(p.sum(axis=1) - 1) < 512 * 2.0 ** -9 * ref.max())
    const = oracle.softmax_bf16(np.full((2, 1024), 0.7, dtype=np.float32), 1.0)
    assert np.all(const == 0x3A80)                                 # 1/1024 = 2^-10 in bf16
    spike = np.zeros((1, 256), dtype=np.float32)
    spike[0, 77] = 200.0
    ps = (oracle.softmax_bf16(spike, 1.0).astype(np.uint32) << 16).view(np.float32)[0]
    assert ps[77] == 1.0 and np.count_nonzero(ps) == 1
    with pytest.raises(ValueError):
        oracle.softmax_bf16(np.zeros((2, 200), dtype=np.float32), 1.0)   # k not a multiple of 256


def test_hadamard_bf16_is_the_nearest_bf16_of_the_rotation():
    """The fused pass's rotation: each output is the bf16 nearest to the binary32
    rotation (ties to even), checked against both bf16 neighbours; exact where
    the rotation is itself a bf16 value (unit vectors, b a power of 4)."""
    xh = synth.sweep_operand(8, 512, seed=73)
    for b in (16, 32, 128):
        rot = oracle.hadamard(xh, b).astype(np.float64)
        got = ((oracle.hadamard_bf16(xh, b).astype(np.uint32) << 16).view(np.float32)).astype(np.float64)
        bits = (oracle.hadamard(xh, b).view(np.uint32) >> 16).astype(np.uint32)
        lo = ((bits << 16).view(np.float32)).astype(np.float64)                  # truncation toward zero
        hi = (((bits + 1) << 16).view(np.float32)).astype(np.float64)            # next bf16 away from zero
        d_got, d_lo, d_hi = np.abs(got - rot), np.abs(lo - rot), np.abs(hi - rot)
        assert np.all(d_got <= np.minimum(d_lo, d_hi))
        tie = d_lo == d_hi
        assert np.all(((oracle.hadamard_bf16(xh, b)[tie] & 1) == 0))
    e = np.zeros((1, 64), dtype=np.float32)
    e[0, 5] = 1.0
    got = (oracle.hadamard_bf16(e, 16).astype(np.uint32) << 16).view(np.float32)[0]
    assert np.array_equal(np.abs(got[:16]), np.full(16, 0.25, dtype=np.float32)) and not got[16:].any()


@pytest.mark.parametrize("pattern,fmt,bits,group,score", [
    (oracle.SPARSE_24, "nvfp4", 4, 0, "mag"), (oracle.SPARSE_48, "nvfp4", 4, 0, "mag"),
    (oracle.SPARSE_24, "fp8", 8, 0, "mag"), (oracle.DENSE, "fp8", 8, 0, "mag"),
    (oracle.DENSE, "int", 8, 0, "mag"), (oracle.SPARSE_24, "int", 4, 128, "wanda"),
    (oracle.SPARSE_48, "fp8", 8, 0, "wanda"), (oracle.DENSE, "mxfp4", 4, 0, "mag"),
    (oracle.SPARSE_24, "none", 8, 0, "mag")])
def test_threaded_driver_equals_the_plain_oracle(pattern, fmt, bits, group, score):
    """run_parallel (row blocks on host threads; the tensor scale from the
    blocks' amax) against one plain run() over the whole operand: outputs bit
    for bit, energies equal up to the order of the binary64 additions. Ragged
    blocks of 37 rows, and one block per row."""
    xh = synth.sweep_operand(300, 1024, seed=81)
    norms = synth.linear_weight(4, 1024, seed=82)[1] if score == "wanda" else None
    kw = dict(pattern=pattern, fmt=fmt, bits=bits, group=group, norms=norms,
              score=oracle.WANDA if score == "wanda" else oracle.MAG)
    ref = oracle.run(xh, **kw)
    for block_rows in (37, 1):
        got = oracle.run_parallel(xh, block_rows=block_rows, threads=4, **kw)
        assert set(got) == set(ref)
        for key in ref:
            if key == "energy":
                np.testing.assert_allclose(got[key], ref[key], rtol=1e-10, atol=0.0)
            else:
                assert np.array_equal(np.ascontiguousarray(got[key]).view(np.uint8),
                                      np.ascontiguousarray(ref[key]).view(np.uint8)), key


def test_binary64_softmax_is_the_nearest_bf16_of_the_library_softmax():
    """oracle.softmax_f64_bf16 against scipy's softmax in binary64 of the same
    binary32 scaled logits: every output is the nearer of the two bf16 values
    around scipy's (ties, to within 1e-12, may go either way; an exact tie goes
    to the even pattern); a constant row gives exactly 1/k; a row with one
    dominant logit gives 1 there and 0 elsewhere; row blocks on threads give
    the same bits."""
    rng = np.random.default_rng(61)
    s = (rng.standard_normal((48, 1024)) * 3.0).astype(np.float32)
    alpha = np.float32(1.0 / math.sqrt(128.0))
    got = oracle.softmax_f64_bf16(s, float(alpha))
    assert np.array_equal(got, oracle.softmax_f64_bf16(s, float(alpha), threads=4))
    ref = special.softmax((s * alpha).astype(np.float32).astype(np.float64), axis=1)
    g = (got.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    t = (ref.astype(np.float32).view(np.uint32) >> 16).astype(np.uint32)      # a bf16 pattern near ref
    cands = [((np.clip(t.astype(np.int64) + d, 0, 0x7f7f).astype(np.uint32) << 16).view(np.float32))
             .astype(np.float64) for d in (-1, 0, 1)]
    dist = np.stack([np.abs(c - ref) for c in cands])
    best = dist.min(axis=0)
    assert np.all(np.abs(g - ref) <= best * (1 + 1e-12) + 1e-300)
    const = oracle.softmax_f64_bf16(np.full((2, 1024), -1.25, dtype=np.float32), 1.0)
    assert np.all(const == 0x3A80)                                   # 2^-10, exactly
    spike = np.zeros((1, 256), dtype=np.float32)
    spike[0, 9] = 900.0
    ps = (oracle.softmax_f64_bf16(spike, 1.0).astype(np.uint32) << 16).view(np.float32)[0]
    assert ps[9] == 1.0 and np.count_nonzero(ps) == 1
