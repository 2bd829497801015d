"""The N-split of the layer over ranks (w4a4_hadamard_rotated_b200.nsplit):
the column partition, the all-gather of the ranks' column blocks over two
gloo ranks on the CPU, and -- with the oracle standing in for each rank's
layer -- that the gathered output equals the unsplit layer bit for bit."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from w4a4_hadamard_rotated_b200 import nsplit


@pytest.mark.parametrize("N,world", [(3072, 1), (3072, 2), (3072, 8), (12288, 8), (264, 3), (8, 4), (392, 5)])
def test_column_blocks_partition(N, world):
    blocks = nsplit.column_blocks(N, world)
    assert len(blocks) == world
    assert blocks[0][0] == 0 and blocks[-1][1] == N
    for (a, b), (c, d) in zip(blocks, blocks[1:]):
        assert b == c                                   # contiguous, disjoint
    for a, b in blocks:
        assert a % 8 == 0 and b % 8 == 0 and a <= b     # 16-byte aligned bf16 blocks
    widths = [b - a for a, b in blocks]
    assert max(widths) - min(w for w in widths) <= 8 * (-(-N // 8 // world))
    assert sum(widths) == N


def test_column_blocks_reject_bad_sizes():
    with pytest.raises(ValueError):
        nsplit.column_blocks(100, 2)
    with pytest.raises(ValueError):
        nsplit.column_blocks(64, 0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update({"WORLD_SIZE": str(world), "RANK": str(rank), "MASTER_ADDR": "127.0.0.1",
                       "MASTER_PORT": str(port)})
    import datetime
    import torch.distributed as dist
    import oracle as orc
    import workloads
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # 1) the gather: every rank's block lands in its columns on every rank
        M, N = 5, 264
        blocks = nsplit.column_blocks(N, world)
        full = torch.arange(M * N, dtype=torch.float32).view(M, N).to(torch.bfloat16)
        a, b = blocks[rank]
        got = nsplit.gather_columns(full[:, a:b].contiguous(), N, world, rank)
        ok_gather = torch.equal(got.view(torch.int16), full.view(torch.int16))
        # 2) the split layer with the oracle as each rank's layer equals the
        # unsplit oracle layer, bit for bit
        cfg = workloads.Linear("nsplit", M=7, K=256, N=392, g=64, seed=11)
        x, W, bias = cfg.make()
        wq = orc.quantize_weight(W.numpy(), cfg.g)
        Wq = torch.from_numpy(wq["packed"])
        sw = torch.from_numpy(wq["scale"])
        Wq_r, sw_r, b_r = nsplit.shard_weight(Wq, sw, bias, world, rank)
        xb = workloads.bf16_bits(x)
        if Wq_r.shape[0] > 0:
            loc = orc.linear(xb, Wq_r.numpy(), sw_r.numpy(), workloads.bf16_bits(b_r), cfg.g)["y_bits"]
            y_local = torch.from_numpy(loc.view(np.int16)).view(torch.bfloat16)
        else:
            y_local = torch.empty(cfg.M, 0, dtype=torch.bfloat16)
        y = nsplit.gather_columns(y_local, cfg.N, world, rank)
        ref = orc.linear(xb, wq["packed"], wq["scale"], workloads.bf16_bits(bias), cfg.g)["y_bits"]
        ok_layer = np.array_equal(y.view(torch.int16).numpy().view(np.uint16), ref)
        out.put((rank, ok_gather, ok_layer))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_gather_the_split_layer(world):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    res = sorted(out.get(timeout=10) for _ in range(world))
    assert [r for r, _, _ in res] == list(range(world))
    assert all(g for _, g, _ in res), res
    assert all(l for _, _, l in res), res


@pytest.mark.gpu
@pytest.mark.parametrize("M,K,N,world", [(4608, 3072, 3072, 8), (300, 1024, 392, 3), (16, 3072, 12288, 4)])
def test_column_blocks_on_the_gpu_match_the_whole_layer(cuda_lib, M, K, N, world):
    """Every rank's block, computed by the library from its weight rows on
    one GPU in turn, equals the same columns of the unsplit layer bit for
    bit (a column depends only on its weight row, its scale and its bias)."""
    import workloads
    cfg = workloads.Linear("nsplit gpu", M=M, K=K, N=N, g=128, seed=N + world)
    x, W, b = cfg.make()
    xc = x.cuda()
    Wq, sw = cuda_lib.quantize_weight(W.cuda(), cfg.g)
    bc = b.cuda()
    whole = cuda_lib.linear_fused(xc, Wq, sw, bc, cfg.g)
    blocks = nsplit.column_blocks(N, world)
    width = max(e - a for a, e in blocks)
    # what the ranks send: each block written by the layer straight into a
    # zeroed [M, width] buffer (row stride width), as NSplitLinear does
    sends = torch.zeros(world, M, width, dtype=torch.bfloat16, device="cuda")
    for rank, (a, e) in enumerate(blocks):
        if e == a:
            continue
        Wq_r, sw_r, b_r = nsplit.shard_weight(Wq, sw, bc, world, rank)
        y_r = cuda_lib.linear_fused(xc, Wq_r, sw_r, b_r, cfg.g)
        assert torch.equal(y_r.view(torch.int16), whole[:, a:e].contiguous().view(torch.int16))
        cuda_lib.linear_fused(xc, Wq_r, sw_r, b_r, cfg.g, out=sends[rank, :, : e - a])
        assert torch.equal(sends[rank, :, : e - a].view(torch.int16), y_r.view(torch.int16))
        assert not sends[rank, :, e - a:].view(torch.int16).any()   # padding untouched
    # the all-gather's result is the sends stacked along rows; placing it gives y
    y = nsplit._place_blocks(sends.view(world * M, width), torch.empty_like(whole), blocks, M, width)
    assert torch.equal(y.view(torch.int16), whole.view(torch.int16))
    # world = 1 (no process group): the split layer is the whole layer
    y = nsplit.NSplitLinear(Wq, sw, bc, cfg.g)(xc)
    assert torch.equal(y.view(torch.int16), whole.view(torch.int16))
