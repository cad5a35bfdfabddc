"""Run one pass of the library on one synthetic operand, a few times.

A small, self-contained driver for profiling a single kernel (for example under
Nsight Compute) or for a quick timing of one configuration:

    python run_case.py --pass fused_24_fp8 --m 4096 --k 4096 --iters 3

With --batch B the pass runs as one batched launch over B operands of that
shape (a [B, m, k] tensor).

Passes: tensor_scale, amax_rows (tensor scale and per-row amax),
fused_24_{none,fp8,nvfp4,mxfp4,int8g128}, fused_48_nvfp4,
dense_{fp8,nvfp4,mxfp4,int8_row,int8g128}, dense_int8_given_rows (one scale per
row from a given row amax), error_energy. Prints the mean CUDA-event
time per launch and the GB/s of the pass's algorithmic bytes.
"""
from __future__ import annotations

import argparse
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from semi_structured_sparsity_online_b200 import ss24, synth  # noqa: E402

# (pattern, format, bits, group): the stored format of each pass
PASSES = {
    "fused_24_none": (ss24.SPARSE_24, "none", 8, 0),
    "fused_24_fp8": (ss24.SPARSE_24, "fp8", 8, 0),
    "fused_24_nvfp4": (ss24.SPARSE_24, "nvfp4", 4, 0),
    "fused_24_mxfp4": (ss24.SPARSE_24, "mxfp4", 4, 0),
    "fused_24_int8g128": (ss24.SPARSE_24, "int", 8, 128),
    "fused_48_nvfp4": (ss24.SPARSE_48, "nvfp4", 4, 0),
    "fused_48_fp8": (ss24.SPARSE_48, "fp8", 8, 0),
    "fused_24_int4g128": (ss24.SPARSE_24, "int", 4, 128),
    "dense_int3g128": (ss24.DENSE, "int", 3, 128),
    "dense_fp8": (ss24.DENSE, "fp8", 8, 0),
    "dense_nvfp4": (ss24.DENSE, "nvfp4", 4, 0),
    "dense_mxfp4": (ss24.DENSE, "mxfp4", 4, 0),
    "dense_int8_row": (ss24.DENSE, "int", 8, 0),
    "dense_int8g128": (ss24.DENSE, "int", 8, 128),
}


def pass_bytes(name, m, k):
    """Algorithmic bytes of one launch on a bf16 [m, k] operand."""
    n = m * k
    if name in ("tensor_scale", "error_energy"):
        return 2 * n
    if name == "hadamard128":
        return 2 * n + 4 * n
    if name == "softmax_24_fp8":
        return 2 * n + n // 2 + n // 8     # read the logits; write FP8 codes + metadata of P
    if name == "amax_rows":
        return 2 * n + 4 * m
    if name == "dense_int8_given_rows":
        return 2 * n + 8 * m + n
    if name == "sparse_gemm_fp8":
        raise ValueError("the GEMM is counted in FLOPs (see main)")
    pattern, fmt, bits, group = PASSES[name]
    q = n // 2 if pattern != ss24.DENSE else n
    meta = n // 8 if pattern == ss24.SPARSE_24 else (n // 16 if pattern == ss24.SPARSE_48 else 0)
    if fmt == "none":
        vals, scales = 2 * q, 0
    elif fmt == "fp8":
        vals, scales = q, 0
    elif fmt == "int":
        # int8 / int16 containers; INT4 and narrower packed two codes per byte
        vals = q // 2 if bits <= 4 else q * (2 if bits > 8 else 1)
        scales = 4 * (m if group == 0 else q // group)
    elif fmt == "nvfp4":
        vals, scales = q // 2, q // 16
    else:
        vals, scales = q // 2, q // 32
    return 2 * n + vals + scales + meta


def main():
    ap = argparse.ArgumentParser()
    extra = ["tensor_scale", "error_energy", "amax_rows", "hadamard128", "softmax_24_fp8", "dense_int8_given_rows",
             "sparse_gemm_fp8"]
    ap.add_argument("--pass", dest="name", default="fused_24_fp8", choices=sorted(PASSES) + extra)
    ap.add_argument("--m", type=int, default=4096)
    ap.add_argument("--k", type=int, default=4096)
    ap.add_argument("--n", type=int, default=4096, help="sparse_gemm_fp8: columns of the product (rows of B)")
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--seed", type=int, default=8)
    ap.add_argument("--batch", type=int, default=0, help="0: one 2-D operand; B: one launch over B operands")
    ap.add_argument("--hadamard", type=int, default=0,
                    help="passes in PASSES: rotate the operand along k in the pass (block size)")
    ap.add_argument("--dequant", action="store_true",
                    help="time the reconstruction of the pass's outputs (ss24_dequantize) instead of the pass")
    ap.add_argument("--score", default="mag", choices=["mag", "wanda"],
                    help="passes in PASSES: the selection score (wanda: column norms exp(N(0,1)))")
    ap.add_argument("--axis", type=int, default=1, choices=[0, 1],
                    help="1: k contiguous; 0: the operand stored [k][m] (rows contiguous), pruned along k")
    ap.add_argument("--derive-scale", action="store_true",
                    help="FP8 / NVFP4: let the pass compute its tensor scale (an amax launch precedes it)")
    ap.add_argument("--energy", default="fp8/int:5:128",
                    help="error_energy: the 2:4 side's and the dense side's formats, e.g. nvfp4/int:3:64 or nvfp4/int,3,64 "
                         "(FP8 and NVFP4 take the given tensor scale)")
    args = ap.parse_args()
    if args.name == "sparse_gemm_fp8":
        return gemm_case(args)
    nb = max(args.batch, 1)
    shape = (args.m, args.k) if args.axis == 1 else (args.k, args.m)
    xb = np.stack([synth.sweep_operand(*shape, seed=args.seed + i) for i in range(nb)])
    x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).cuda()
    if args.batch == 0:
        x = x[0]
    lead = None if args.batch == 0 else args.batch
    ws = ss24.Workspace()
    e = torch.zeros((nb, 4), dtype=torch.float64, device="cuda")
    if args.batch == 0:
        e = e[0]
    scale = ss24.tensor_scale(x, "fp8", ss24.SPARSE_24, ws=ws, hadamard=args.hadamard, axis=args.axis)
    out = None
    norms = None
    if args.score == "wanda":
        norms = torch.from_numpy(np.exp(np.random.default_rng(3).standard_normal(args.k)).astype(np.float32)).cuda()
    if args.name in PASSES:
        pattern, fmt, bits, group = PASSES[args.name]
        out = ss24._alloc_outputs(args.m, args.k, pattern, ss24.make_format(fmt, bits, group, fmt == "int" and bits <= 4),
                                  torch.bfloat16, "cuda", lead)
        if fmt == "nvfp4":
            scale = ss24.tensor_scale(x, "nvfp4", pattern if pattern != ss24.DENSE else ss24.DENSE, ws=ws,
                                      hadamard=args.hadamard, axis=args.axis)

    if args.name == "error_energy":
        def _parse(f):
            t = f.replace(",", ":").split(":")
            return (t[0],) + tuple(int(v) for v in t[1:])
        e_fmt = tuple(_parse(f) for f in args.energy.split("/"))
        e_scale = tuple(ss24.tensor_scale(x, f[0], ss24.SPARSE_24 if i == 0 else ss24.DENSE, ws=ws, axis=args.axis)
                        if f[0] in ("fp8", "nvfp4") else None for i, f in enumerate(e_fmt))
    row_amax = ss24.amax_rows(x, ws=ws)[0] if args.name in ("amax_rows", "dense_int8_given_rows") else None
    if args.name == "dense_int8_given_rows":
        out = ss24._alloc_outputs(args.m, args.k, ss24.DENSE, ss24.make_format("int", 8, 0), torch.bfloat16, "cuda",
                                  lead)

    rot = torch.empty(x.shape, dtype=torch.float32, device="cuda") if args.name == "hadamard128" else None
    alpha = float(np.float32(1.0 / np.sqrt(128.0)))
    p_scale = torch.full((nb,), 1.0 / 448.0, device="cuda")
    if args.name == "softmax_24_fp8":
        out = ss24._alloc_outputs(args.m, args.k, ss24.SPARSE_24, ss24.make_format("fp8"), torch.bfloat16, "cuda",
                                  lead)

    def once():
        if args.name == "amax_rows":
            ss24.amax_rows(x, scale_fmt="fp8", ws=ws, out=row_amax, scale_out=scale)
        elif args.name == "dense_int8_given_rows":
            ss24.run_int_rows(x, row_amax, bits=8, energy=e, ws=ws, out=out)
        elif args.name == "softmax_24_fp8":
            ss24.softmax_prune(x, alpha, pattern=ss24.SPARSE_24, fmt="fp8", tensor_scale=p_scale, energy=e, ws=ws,
                               out=out)
        elif args.name == "hadamard128":
            ss24.hadamard(x, 128, out=rot)
        elif args.name == "tensor_scale":
            ss24.tensor_scale(x, "fp8", ss24.SPARSE_24, ws=ws, out=scale)
        elif args.name == "error_energy":
            ss24.error_energy(x, ss24.SPARSE_24, e_fmt[0], e_fmt[1], sparse_scale=e_scale[0], dense_scale=e_scale[1],
                              ws=ws, energy=e, axis=args.axis)
        else:
            pattern, fmt, bits, group = PASSES[args.name]
            ts = scale if fmt in ("fp8", "nvfp4") and not args.derive_scale else None
            ss24.run(x, pattern=pattern, fmt=fmt, bits=bits, group=group, pack4=fmt == "int" and bits <= 4,
                     tensor_scale=ts, energy=e, ws=ws, out=out, hadamard=args.hadamard, score=args.score,
                     col_norms=norms, axis=args.axis)

    once()
    torch.cuda.synchronize()
    gb = nb * pass_bytes(args.name, args.m, args.k)
    if args.dequant:
        pattern, fmt, bits, group = PASSES[args.name]
        xhat = torch.empty(x.shape, dtype=torch.float32, device="cuda")
        # reads the stored outputs, writes fp32 x_hat: the pass's bytes less its input, plus 4 per element
        gb = gb - nb * 2 * args.m * args.k + nb * 4 * args.m * args.k

        def once():
            ss24.dequantize(out, args.m, args.k, pattern=pattern, fmt=fmt, bits=bits, group=group, batch=lead,
                            xhat=xhat)

        once()
        torch.cuda.synchronize()
    s, t = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(args.iters):
        once()
    t.record()
    t.synchronize()
    us = s.elapsed_time(t) / args.iters * 1e3
    assert ws.error() == 0
    tag = ((" dequant" if args.dequant else "") + (f" hadamard {args.hadamard}" if args.hadamard else "")
           + (" axis 0" if args.axis == 0 else ""))
    print(f"{args.name}{tag} m={args.m} k={args.k} batch={args.batch}: {us:.2f} us/launch, {gb / us / 1e3:.1f} GB/s "
          f"({gb} algorithmic bytes per launch; warm L2 between launches)")


def gemm_case(args):
    """The consumer: A = 2:4 + FP8 of an [m, k] sweep operand, B = dense FP8 of
    an [n, k] N(0, 0.02^2) operand, Y = A B^T on the sparse tensor cores."""
    x = torch.from_numpy(synth.sweep_operand(args.m, args.k, seed=args.seed).view(np.int16)).view(torch.bfloat16)
    w = torch.from_numpy(synth.gaussian_bf16(args.n, args.k, seed=args.seed + 1, std=0.02).view(np.int16))
    ws = ss24.Workspace()
    a = ss24.run(x.cuda(), pattern=ss24.SPARSE_24, fmt="fp8", ws=ws)
    b = ss24.run(w.view(torch.bfloat16).cuda(), pattern=ss24.DENSE, fmt="fp8", ws=ws)
    y = ss24.sparse_gemm_fp8(a, b, ws=ws)
    torch.cuda.synchronize()
    s, t = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(args.iters):
        ss24.sparse_gemm_fp8(a, b, y=y, ws=ws)
    t.record()
    t.synchronize()
    us = s.elapsed_time(t) / args.iters * 1e3
    assert ws.error() == 0
    flops = 2 * args.m * args.n * args.k
    print(f"sparse_gemm_fp8 m={args.m} n={args.n} k={args.k}: {us:.2f} us/launch, {flops / us / 1e6:.1f} "
          f"dense-equivalent TFLOP/s ({flops // 2} multiply-adds of kept values)")


if __name__ == "__main__":
    main()
