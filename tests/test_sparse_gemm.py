"""The consumer: the tensor cores' 2:4-sparse FP8 GEMM on the pass's outputs
("Is 2:4 Sparsity Still Worth It?" §1, §3: the sparse GEMM reads the kept
values and their indices), checked against the product of the dense operands
the oracle reconstructs, in binary64.

A wrong metadata layout (which value a nibble names, or which row or k step
a byte belongs to) moves products onto the wrong columns of B and shows as an
error of the size of the result; the bound below is the binary32 accumulation
of k products."""
import numpy as np
import pytest
import torch

import oracle
from semi_structured_sparsity_online_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ss():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from semi_structured_sparsity_online_b200 import ss24
    ss24.lib()
    return ss24


def _dev(a):
    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()


def _e4m3_table():
    return np.array([oracle.e4m3_decode(c) for c in range(256)], dtype=np.float64)


@pytest.mark.parametrize("m,n,k", [(128, 128, 256), (256, 384, 1024), (384, 256, 2048)])
def test_sparse_gemm_matches_the_dense_product_of_the_oracle_operands(ss, m, n, k):
    xh = synth.linear_input(m, k, seed=41, n_outlier=4)[0]
    wh = synth.gaussian_bf16(n, k, seed=42, std=0.02)
    ws = ss.Workspace()
    a = ss.run(_dev(xh), pattern=ss.SPARSE_24, fmt="fp8", ws=ws)
    b = ss.run(_dev(wh), pattern=ss.DENSE, fmt="fp8", ws=ws)
    y = ss.sparse_gemm_fp8(a, b, ws=ws)
    torch.cuda.synchronize()
    assert ws.error() == 0
    # the operands as the oracle writes them (bit-exact with the pass) and
    # their dense reconstruction in binary64
    ra = oracle.run(xh, pattern=oracle.SPARSE_24, fmt="fp8")
    rb = oracle.run(wh, pattern=oracle.DENSE, fmt="fp8")
    assert np.array_equal(a["values"].cpu().numpy(), ra["values"]) and np.array_equal(a["meta"].cpu().numpy(),
                                                                                        ra["meta"])
    assert np.array_equal(b["values"].cpu().numpy(), rb["values"])
    t = _e4m3_table()
    sa, sb = float(ra["tensor_scale"][0]), float(rb["tensor_scale"][0])
    ad = np.zeros((m, k))
    kept = t[ra["values"]].reshape(m, k // 4, 2)
    nib = np.stack([ra["meta"] & 0xF, ra["meta"] >> 4], axis=-1).reshape(m, k // 4)
    for j, sh in ((0, 0), (1, 2)):
        idx = (nib >> sh) & 3
        ad.reshape(m, k // 4, 4)[np.arange(m)[:, None], np.arange(k // 4)[None, :], idx] = kept[..., j]
    bd = t[rb["values"]]
    ref = (ad @ bd.T) * (np.float32(sa) * np.float32(sb))
    bound = (np.abs(ad) @ np.abs(bd).T) * abs(sa * sb)
    got = y.cpu().numpy().astype(np.float64)
    err = np.abs(got - ref)
    assert np.all(err <= 2.0 ** -20 * k * bound + 1e-30), float((err / (bound + 1e-30)).max())
    # and against the library's own dequantized operand, as a second route
    xhat = ss.dequantize(a, m, k, pattern=ss.SPARSE_24, fmt="fp8").cpu().numpy().astype(np.float64)
    rel = np.linalg.norm(xhat @ (bd * sb).T - got) / np.linalg.norm(got)
    assert rel < 1e-5


def test_sparse_gemm_rejects_bad_shapes(ss):
    ws = ss.Workspace()
    z = torch.zeros(16, dtype=torch.uint8, device="cuda")
    s = torch.ones(1, dtype=torch.float32, device="cuda")
    y = torch.zeros(16, dtype=torch.float32, device="cuda")
    import ctypes
    L = ss.lib()
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    for m, n, k in ((100, 128, 256), (128, 100, 256), (128, 128, 200), (-128, 128, 256), (128, 128, 0)):
        assert L.ss24_sparse_gemm_fp8(p(z), p(z), p(s), p(z), p(s), m, n, k, p(y), ws.ptr, ws.nbytes,
                                      None) == ss.STATUS_NAMES_INV["SS24_ERR_SHAPE"]
    assert L.ss24_sparse_gemm_fp8(None, p(z), p(s), p(z), p(s), 128, 128, 256, p(y), ws.ptr, ws.nbytes,
                                  None) == ss.STATUS_NAMES_INV["SS24_ERR_NULL"]
    assert L.ss24_sparse_gemm_fp8(p(z), p(z), p(s), p(z), p(s), 0, 128, 256, p(y), ws.ptr, ws.nbytes, None) == 0
