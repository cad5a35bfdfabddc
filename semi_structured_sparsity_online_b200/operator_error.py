"""Operator-level error of a pruned and quantized operand.

"Is 2:4 Sparsity Still Worth It?" (§4) compares the two sides of an equal-bit
budget through the error they cause in the GEMM that consumes the operand, and
predicts the ratio R of those errors from energies alone,
R_hat = sqrt((E_prune + E_q,2m) / E_q,m+1). This module measures R on an
operand X [M, K] (pruned along K) and a weight W [N, K]:

    Y   = X W^T                (X as stored, fp32)
    Y_s = X_hat_s W^T          (2:4 side: pruned, kept values quantized)
    Y_d = X_hat_d W^T          (dense side: every value quantized)
    err = ||Y_side - Y||_F / ||Y||_F,   R = err_s / err_d

with Y_side - Y formed as (X_hat_side - X) W^T, free of cancellation.

The passes and the reconstructions X_hat (ss24_dequantize) run in this
library's kernels; the three products are plain fp32 library GEMMs (TF32 off).
For W with i.i.d. entries, E||E W^T||^2 = ||E||^2 sigma^2 N, so R tends to
R_hat: the prediction is exact in expectation for such weights.
"""
from __future__ import annotations

import torch

from . import ss24


def _fmt(spec):
    spec = tuple(spec) if isinstance(spec, (tuple, list)) else (spec,)
    fmt = spec[0]
    bits = spec[1] if len(spec) > 1 else 8
    group = spec[2] if len(spec) > 2 else 0
    pack4 = spec[3] if len(spec) > 3 else False
    return fmt, bits, group, pack4


def measured_ratio(x: torch.Tensor, w: torch.Tensor, *, pattern=ss24.SPARSE_24, sparse=("fp8",),
                   dense=("int", 8, 0), score="mag", col_norms=None, ws=None):
    """Measured and predicted R for operand x [M, K] (bf16 or fp32, device) and
    weight w [N, K]. sparse / dense: (format, bits, group, pack4) of each side.
    Returns a dict of floats: err_sparse, err_dense, r_measured, r_predicted."""
    rows, k = x.shape
    sf, sb, sg, sp = _fmt(sparse)
    df, db, dg, dp = _fmt(dense)
    ws = ws or ss24.default_workspace(x.device)
    out_s = ss24.run(x, pattern=pattern, fmt=sf, bits=sb, group=sg, pack4=sp, score=score, col_norms=col_norms,
                     ws=ws)
    out_d = ss24.run(x, pattern=ss24.DENSE, fmt=df, bits=db, group=dg, pack4=dp, ws=ws)
    xs = ss24.dequantize(out_s, rows, k, pattern=pattern, fmt=sf, bits=sb, group=sg, pack4=sp, dtype=x.dtype)
    xd = ss24.dequantize(out_d, rows, k, pattern=ss24.DENSE, fmt=df, bits=db, group=dg, pack4=dp, dtype=x.dtype)
    ratio = ss24.predicted_ratio(out_s["energy"], out_d["energy"])
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    try:
        wt = w.float().t()
        xf = x.float()
        y = xf @ wt
        es = (xs - xf) @ wt
        ed = (xd - xf) @ wt
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev
    ny = torch.linalg.vector_norm(y.double())
    err_s = (torch.linalg.vector_norm(es.double()) / ny).item()
    err_d = (torch.linalg.vector_norm(ed.double()) / ny).item()
    return {"err_sparse": err_s, "err_dense": err_d, "r_measured": err_s / err_d,
            "r_predicted": float(ratio[3].item())}
