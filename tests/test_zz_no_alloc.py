"""The fused 2:4 pass without caller scratch (ss24_prune24_quant_fused_noalloc).

Some callers cannot allocate device memory: code running where cudaMalloc is
not allowed, or a host that hands the library only the operand and the output
buffers. They use this entry point, whose scratch lives in a device array owned
by the library. The test calls it through the C ABI twice in a row (different
operands and formats, so the second call runs on the array the first one left
behind) and compares each result with the workspace entry point's: codes,
scales and metadata bit for bit, energies to the suite's 1e-6 relative.
This file is collected last; it passes alone in a fresh process too.
"""
import ctypes

import numpy as np
import pytest
import torch

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


def _call(ss, x, fmt, ws=None):
    """One fused call through the C ABI: the workspace entry point when `ws` is
    given, otherwise the no-allocation one."""
    f = ss.make_format(*fmt)
    op = ss.make_operand(x)
    sptr = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    out = ss._alloc_outputs(op.rows, op.k, ss.SPARSE_24, f, x.dtype, x.device)
    e = torch.zeros(4, dtype=torch.float64, device=x.device)
    o = ss.Outputs(*(ctypes.c_void_p(out[key].data_ptr()) if key in out else None
                     for key in ("values", "scales", "tensor_scale", "meta")))
    if ws is not None:
        st = ss.lib().ss24_prune24_quant_fused(ctypes.byref(op), ss.MAG, None, f, None, ctypes.byref(o),
                                               ctypes.c_void_p(e.data_ptr()), ws.ptr, ws.nbytes, sptr)
    else:
        st = ss.lib().ss24_prune24_quant_fused_noalloc(ctypes.byref(op), ss.MAG, None, f, None, ctypes.byref(o),
                                                       ctypes.c_void_p(e.data_ptr()), sptr)
    assert st == 0, ss.status_string(st)
    out["energy"] = e
    return out


def _assert_same(a, b):
    for key in ("values", "scales", "meta", "tensor_scale"):
        if key in a:
            assert torch.equal(a[key], b[key]), key
    ea, eb = a["energy"].cpu().numpy(), b["energy"].cpu().numpy()
    np.testing.assert_allclose(eb, ea, rtol=RTOL, atol=0.0)


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row(ss):
    ws = ss.Workspace()
    x1 = _to_dev(synth.linear_input(1000, 4096, seed=21)[0])
    x2 = _to_dev(synth.sweep_operand(333, 2048, seed=22))
    ref1 = _call(ss, x1, ("fp8",), ws)
    ref2 = _call(ss, x2, ("nvfp4",), ws)
    torch.cuda.synchronize()
    assert ws.error() == 0
    got1 = _call(ss, x1, ("fp8",))       # two no-allocation calls back to back
    got2 = _call(ss, x2, ("nvfp4",))
    torch.cuda.synchronize()
    _assert_same(ref1, got1)
    _assert_same(ref2, got2)
