"""The fused 2:4 pass without caller scratch (ss24_prune24_quant_fused_noalloc).

Some callers cannot allocate device memory: code running where cudaMalloc is
not allowed, or a host that hands the library only the operand and the output
buffers. They use this entry point, whose scratch lives in a device array owned
by the library. The tests call it through the C ABI twice in a row (different
operands and formats, so the second call runs on the array the first one left
behind) and compare each result with the workspace entry point's and with the
CPU oracle's: codes, scales and metadata bit for bit, energies to the suite's
1e-6 relative. Rejected calls (axis 0, bad arguments) must return their status,
write nothing, and leave the next accepted call exact.
This file is collected last; it passes alone in a fresh process too.
"""
import ctypes

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


def _to_dev(a):
    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()


def _call(ss, x, fmt, ws=None, axis=1, expect=0, fill=None):
    """One fused call through the C ABI: the workspace entry point when `ws` is
    given, otherwise the no-allocation one. `fill`: a byte every output buffer
    starts with (to see that a rejected call wrote nothing)."""
    f = ss.make_format(*fmt)
    op = ss.make_operand(x, axis)
    sptr = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    out = ss._alloc_outputs(op.rows, op.k, ss.SPARSE_24, f, x.dtype, x.device)
    e = torch.zeros(4, dtype=torch.float64, device=x.device)
    if fill is not None:
        for t in list(out.values()) + [e]:
            t.view(torch.uint8).fill_(fill)
    o = ss.Outputs(*(ctypes.c_void_p(out[key].data_ptr()) if key in out else None
                     for key in ("values", "scales", "tensor_scale", "meta")))
    if ws is not None:
        st = ss.lib().ss24_prune24_quant_fused(ctypes.byref(op), ss.MAG, None, f, None, ctypes.byref(o),
                                               ctypes.c_void_p(e.data_ptr()), ws.ptr, ws.nbytes, sptr)
    else:
        st = ss.lib().ss24_prune24_quant_fused_noalloc(ctypes.byref(op), ss.MAG, None, f, None, ctypes.byref(o),
                                                       ctypes.c_void_p(e.data_ptr()), sptr)
    assert st == expect, ss.status_string(st)
    out["energy"] = e
    return out


def _assert_same(a, b):
    for key in ("values", "scales", "meta", "tensor_scale"):
        if key in a:
            assert torch.equal(a[key], b[key]), key
    ea, eb = a["energy"].cpu().numpy(), b["energy"].cpu().numpy()
    np.testing.assert_allclose(eb, ea, rtol=RTOL, atol=0.0)


def _assert_oracle(got, xh, fmt):
    ref = oracle.run(xh, pattern=oracle.SPARSE_24, fmt=fmt[0], **({"bits": fmt[1], "group": fmt[2]}
                                                                    if fmt[0] == "int" else {}))
    for key in ("values", "scales", "meta", "tensor_scale"):
        if key in ref:
            g = got[key].cpu().numpy()
            assert np.array_equal(g.view(np.uint8), np.ascontiguousarray(ref[key]).view(np.uint8)), key
    e = got["energy"].cpu().numpy()
    for f in range(4):
        assert abs(e[f] - ref["energy"][f]) <= RTOL * abs(ref["energy"][f]), (f, e[f], ref["energy"][f])


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row(ss):
    ws = ss.Workspace()
    x1h = synth.linear_input(1000, 4096, seed=21)[0]
    x2h = synth.sweep_operand(333, 2048, seed=22)
    x1, x2 = _to_dev(x1h), _to_dev(x2h)
    ref1 = _call(ss, x1, ("fp8",), ws)
    ref2 = _call(ss, x2, ("nvfp4",), ws)
    torch.cuda.synchronize()
    assert ws.error() == 0
    got1 = _call(ss, x1, ("fp8",))       # two no-allocation calls back to back
    got2 = _call(ss, x2, ("nvfp4",))
    torch.cuda.synchronize()
    _assert_same(ref1, got1)
    _assert_same(ref2, got2)
    _assert_oracle(got1, x1h, ("fp8",))
    _assert_oracle(got2, x2h, ("nvfp4",))


def test_noalloc_rejects_axis0_and_bad_arguments_without_writing(ss):
    """Rejected calls return their status and write nothing; the next accepted
    call (here INT8 with groups of 64, after the rejections) is exact."""
    xh = synth.sweep_operand(96, 512, seed=23)
    x = _to_dev(xh)
    # axis 0: the strided-axis kernel's time-limited waits report through the
    # scratch, which this entry point's callers cannot read
    bad = _call(ss, x, ("fp8",), axis=0, expect=ss.STATUS_NAMES_INV["SS24_ERR_ARG"], fill=0xA5)
    # k not a multiple of 8 (a view of 500 columns): a shape error
    bad2 = _call(ss, x[:, :500], ("nvfp4",), expect=ss.STATUS_NAMES_INV["SS24_ERR_SHAPE"], fill=0x5A)
    torch.cuda.synchronize()
    for out, byte in ((bad, 0xA5), (bad2, 0x5A)):
        for key, t in out.items():
            assert bool((t.view(torch.uint8) == byte).all()), f"a rejected call wrote {key}"
    got = _call(ss, x, ("int", 8, 64))
    torch.cuda.synchronize()
    _assert_oracle(got, xh, ("int", 8, 64))
