"""The multi-rank logic on CPU: world size 2 over gloo.

Each rank takes its row block of one operand, computes its shard's tensor
scale and energies with the CPU oracle (standing in for the GPU pass, which
these CPU processes cannot run), and combines them with the library's
all-reduce helpers. The combined scale must equal the whole operand's scale
bit for bit, the shard codes must equal the matching rows of a whole-operand
pass, and the combined energies must match the whole operand's."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from semi_structured_sparsity_online_b200 import synth
from semi_structured_sparsity_online_b200.sharded import allreduce_energy, allreduce_tensor_scale, row_block


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, fmt, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        xh, _ = synth.linear_input(203, 256, seed=3)
        r0, r1 = row_block(xh.shape[0], world, rank)
        shard = np.ascontiguousarray(xh[r0:r1])
        scale = torch.tensor([oracle.tensor_scale(shard, fmt)], dtype=torch.float32)
        allreduce_tensor_scale(scale)
        out = oracle.run(shard, fmt=fmt, tensor_scale=float(scale.item()))
        e = torch.from_numpy(out["energy"].copy())
        allreduce_energy(e)
        results[rank] = (r0, r1, float(scale.item()), out["values"], out["meta"], e.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("fmt", ["fp8", "nvfp4"])
def test_two_rank_shards_match_whole_operand(fmt):
    world = 2
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    results = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, fmt, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    xh, _ = synth.linear_input(203, 256, seed=3)
    whole = oracle.run(xh, fmt=fmt)
    covered = []
    for rank in range(world):
        r0, r1, scale, values, meta, e = results[rank]
        covered.extend(range(r0, r1))
        assert np.float32(scale) == whole["tensor_scale"][0]
        assert np.array_equal(values, whole["values"][r0:r1])
        assert np.array_equal(meta, whole["meta"][r0:r1])
        np.testing.assert_allclose(e, whole["energy"], rtol=1e-12)
    assert covered == list(range(xh.shape[0]))


def test_row_blocks_partition():
    for rows in (0, 1, 7, 100, 4096):
        for world in (1, 2, 3, 8):
            blocks = [row_block(rows, world, r) for r in range(world)]
            assert blocks[0][0] == 0 and blocks[-1][1] == rows
            for (a, b), (c, d) in zip(blocks, blocks[1:]):
                assert b == c
            sizes = [b - a for a, b in blocks]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        row_block(10, 2, 2)
