"""One operand split by row blocks across ranks (one process per GPU).

Rows are independent in every pass: selection, compression and all scales
except the per-tensor one stay inside a row. Sharding one operand [rows, k]
therefore needs exactly two exchanges, both a few bytes over NCCL:
  * before quantizing with a per-tensor format (FP8, NVFP4): the tensor scale
    is the maximum over ranks of the shard scales. Dividing by the positive
    constant (448 or 2688) and rounding to nearest is monotone, so
    max_r(amax_r / d) equals (max_r amax_r) / d bit for bit;
  * after the pass: the four energies are sums over rows, so their all-reduce
    (sum) gives the energies of the whole operand (binary64; the order of the
    additions differs from a single-GPU run only in the last bits).
Independent operands (a batch of layers, micro-batches) need neither exchange.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def row_block(rows: int, world: int, rank: int) -> tuple[int, int]:
    """[start, stop) of this rank's rows: contiguous blocks, sizes differing by at most one."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("rank must be in [0, world)")
    base, extra = divmod(rows, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def allreduce_tensor_scale(scale: torch.Tensor, group=None) -> torch.Tensor:
    """In place: the per-tensor scale of the whole operand from the shard scales."""
    dist.all_reduce(scale, op=dist.ReduceOp.MAX, group=group)
    return scale


def allreduce_energy(energy: torch.Tensor, group=None) -> torch.Tensor:
    """In place: the energies of the whole operand (float64[4]) from the shards'."""
    dist.all_reduce(energy, op=dist.ReduceOp.SUM, group=group)
    return energy


def sharded_prune24_quant(x_local: torch.Tensor, fmt="fp8", bits=8, group=0, pack4=False, score="mag",
                          col_norms=None, ws=None, stream=None, process_group=None):
    """The fused 2:4 pass over this rank's row block of one operand: shard
    scale, all-reduce(max), the pass with the tensor scale given, all-reduce(sum)
    of the energies. Returns the pass outputs for the local rows and the
    energies of the whole operand."""
    from . import ss24
    scale = None
    if fmt in ("fp8", "nvfp4"):
        scale = ss24.tensor_scale(x_local, fmt, ss24.SPARSE_24, score=score, col_norms=col_norms, ws=ws,
                                  stream=stream)
        allreduce_tensor_scale(scale, process_group)
    out = ss24.run(x_local, pattern=ss24.SPARSE_24, fmt=fmt, bits=bits, group=group, pack4=pack4, score=score,
                   col_norms=col_norms, tensor_scale=scale, ws=ws, stream=stream)
    allreduce_energy(out["energy"], process_group)
    return out
