"""Multi-rank host logic on CPU: two gloo ranks, each computing its shard with the oracle.

Checks that the shards partition the blocks (weak: disjoint id ranges; strong: every layer
exactly once), that the regulariser summed over ranks equals the single-process sum, and
that the timing reduction takes the maximum over ranks.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sparsity_mask_sampling_b200 import configs, inputs, sharding

TINY_STACK = configs.Workload(name="tiny_stack", nm=(2, 4),
                              matrices=(configs.MatrixShape("a", 8, 32), configs.MatrixShape("b", 4, 16)),
                              layers=4)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer_reg(orc, w, l, offsets, kappa=100.0, tau=1.0, seed=5, step=2):
    """Oracle regulariser of one layer with the given block offsets."""
    reg = 0.0
    for i, m in enumerate(w.matrices):
        B = m.rows * m.cols // 4
        W = inputs.weights(m.rows, m.cols, "bf16", 0.02, seed=100 * l + i).float().double().numpy().reshape(B, 4)
        pi = inputs.logits(B, 6, 0.02, seed=1000 + 100 * l + i).numpy()
        gids = np.arange(B, dtype=np.uint64) + np.uint64(offsets[l][i])
        reg += orc.sample_fwd(2, 4, W, pi, gids, kappa, tau, seed, step)["reg"]
    return reg


def _worker(rank, world, port, mode, q):
    import oracle as orc

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = TINY_STACK
        if mode == "strong":
            offs = configs.layer_block_offsets(w)
            layers = sharding.strong_layers(w, rank, world)
        else:
            offs = sharding.weak_block_offsets(w, rank)
            layers = list(range(w.layers))
        reg = torch.tensor([sum(_layer_reg(orc, w, l, offs) for l in layers)], dtype=torch.float64)
        sharding.all_reduce_sum(reg)
        tmax = sharding.max_over_ranks(10.0 + rank)
        q.put((rank, float(reg.item()), tmax, layers, offs[0][0]))
    finally:
        dist.destroy_process_group()


def _run(mode, world=2):
    import oracle

    oracle.build()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, mode, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(out)


def test_strong_split_regulariser_matches_single_process():
    import oracle as orc

    out = _run("strong")
    w = TINY_STACK
    offs = configs.layer_block_offsets(w)
    ref = sum(_layer_reg(orc, w, l, offs) for l in range(w.layers))
    for rank, reg, tmax, layers, _ in out:
        assert abs(reg - ref) <= 1e-12 * ref
        assert tmax == 11.0
    owned = sorted(l for _, _, _, layers, _ in out for l in layers)
    assert owned == list(range(w.layers))


def test_weak_split_is_disjoint_and_sums():
    import oracle as orc

    out = _run("weak")
    w = TINY_STACK
    ref = 0.0
    for r in range(2):
        offs = sharding.weak_block_offsets(w, r)
        ref += sum(_layer_reg(orc, w, l, offs) for l in range(w.layers))
    for rank, reg, tmax, _, first in out:
        assert abs(reg - ref) <= 1e-12 * ref
        assert first == rank * w.total_blocks()


def test_shard_helpers():
    w = configs.WORKLOADS["llama2_7b_stack_2of4"]
    assert w.total_blocks() == 1_619_001_344
    a, b = sharding.weak_block_offsets(w, 0), sharding.weak_block_offsets(w, 1)
    assert b[0][0] == w.total_blocks() and a[-1][-1] < b[0][0]
    for world in (1, 2, 3, 8):
        got = sorted(l for r in range(world) for l in sharding.strong_layers(w, r, world))
        assert got == list(range(32))
    with pytest.raises(ValueError):
        sharding.strong_layers(w, 2, 2)
