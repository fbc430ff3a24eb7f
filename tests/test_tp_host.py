"""Head-sharded prefill: the host logic on CPU (two and three gloo ranks).

Each rank computes the partial output of its heads with the fp64 oracle on a
head slice of the problem (a stand-in for the CUDA calls, which need a GPU),
writes it chunk by chunk through the same driver the GPU path uses, and the
chunks are summed across ranks by gloo all-reduces. The sum must equal the
oracle's output of the unsharded block: that fixes which W_kvb rows, W_o
rows, block-scale rows and query heads belong to a head, and that the partial
outputs of the ranks add up to the block (DeepSeek-V3.2-Exp "Sparse
attention": wkv_b column-parallel, wo row-parallel)."""
import dataclasses
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
import synth
from sparse_head_latent_b200.tp import head_range, reduce_chunks, row_chunks, shard_weights


def test_head_ranges_partition_the_heads():
    for H in (1, 2, 3, 7, 64, 128, 130):
        for world in (1, 2, 3, 4, 8):
            ranges = [head_range(H, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == H
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
            sizes = [h1 - h0 for h0, h1 in ranges]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        head_range(8, 2, 2)


def test_row_chunks_cover_the_rows_in_order():
    for M in (1, 255, 256, 4096, 5000):
        for c in (1, 256, 2048, 10000):
            ch = row_chunks(M, c)
            assert ch[0][0] == 0 and ch[-1][1] == M
            assert all(a[1] == b[0] for a, b in zip(ch, ch[1:]))
            assert all(r1 - r0 == c for r0, r1 in ch[:-1])


@pytest.mark.parametrize("fp8", [False, True])
def test_shard_weights_takes_the_rows_of_the_heads(fp8):
    x = synth.make_inputs(0, B=1, T=8, H=4, topk=None, seed=3, fp8=fp8)
    w = shard_weights(x.W_kvb, x.W_o, x.W_kvb_scale, x.W_o_scale, 1, 3)
    assert torch.equal(w["W_kvb"], x.W_kvb[256:768]) and torch.equal(w["W_o"], x.W_o[128:384])
    if fp8:
        assert torch.equal(w["W_kvb_scale"], x.W_kvb_scale[2:6]) and torch.equal(w["W_o_scale"], x.W_o_scale[1:3])
    else:
        assert w["W_kvb_scale"] is None and w["W_o_scale"] is None


def _head_slice(x, h0, h1):
    """The problem restricted to heads [h0, h1) (what one rank holds)."""
    w = shard_weights(x.W_kvb, x.W_o, x.W_kvb_scale, x.W_o_scale, h0, h1)
    return dataclasses.replace(x, H=h1 - h0, q=x.q[:, :, h0:h1].contiguous(), **w)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, case, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x = synth.make_inputs(0, seed=41, **case)
        h0, h1 = head_range(x.H, world, rank)
        mine = _head_slice(x, h0, h1)
        M = x.B * x.T
        partial = torch.zeros(M, 7168, dtype=torch.float64)

        def project(r0, r1):
            _, o = oracle.prefill_rows(mine, range(r0, r1))
            partial[r0:r1] = torch.from_numpy(o)

        reduce_chunks(partial, row_chunks(M, 48), project, lambda rows: dist.all_reduce(rows))
        q.put((rank, partial.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,case", [(2, dict(B=1, T=100, H=4, topk=16)),
                                        (3, dict(B=2, T=70, H=4, topk=None, fp8=True))])
def test_sharded_partials_sum_to_the_block(world, case):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=600) for _ in range(world))
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    x = synth.make_inputs(0, seed=41, **case)
    _, ref = oracle.prefill_rows(x, range(x.B * x.T))
    for r in range(world):
        d = np.abs(got[r] - ref).max() / np.abs(ref).max()
        assert d < 1e-12, (r, d)
