"""Head-sharded prefill with the CUDA kernels (needs a B200; one GPU).

Several ranks cannot run on one GPU, so the shards run one after another on
the same device ("virtual ranks"): each computes its heads' partial output
through the C ABI with its slice of the weights, and the partials are added
(in fp32, by the test). The sum must match the oracle's unsharded block at
the usual tolerances (the per-shard bf16 rounding of the partials adds about
sqrt(G) * 2^-9 of a partial's size). The driver class itself runs with no
process group and with an NCCL group of one rank, and must reproduce
mla_prefill bit for bit (its row chunks are multiples of the GEMM's 256-row
tiles, so every output element is computed the same way)."""
import os
import socket

import pytest
import torch

import oracle
import synth

mla = pytest.importorskip("sparse_head_latent_b200")

from sparse_head_latent_b200.tp import HeadShardedPrefill, head_range, shard_weights  # noqa: E402
from test_gpu_parity import _dev, _no_device_error, assert_close  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("G,case", [(2, dict(B=1, T=300, H=4, topk=40)), (4, dict(B=2, T=260, H=8, topk=None)),
                                    (3, dict(B=1, T=200, H=5, topk=24, fp8=True))])
def test_virtual_ranks_sum_to_the_block(G, case):
    x = synth.make_inputs(0, seed=71, **case)
    g = _dev(x)
    total = torch.zeros(x.B * x.T, 7168, dtype=torch.float32, device="cuda")
    for rank in range(G):
        h0, h1 = head_range(x.H, G, rank)
        w = shard_weights(g["W_kvb"], g["W_o"], g.get("W_kvb_scale"), g.get("W_o_scale"), h0, h1)
        q = g["q"][:, :, h0:h1].contiguous()
        attn = mla.mla_attend(q, g["kv_latent"], g["k_pe"], w["W_kvb"], w["W_kvb_scale"],
                              topk_idx=g.get("topk_idx"), scale=x.scale)
        part = mla.mla_out_project(attn, w["W_o"], w["W_o_scale"])
        total += part.float()
    _no_device_error()
    _, ref = oracle.prefill_rows(x, range(x.B * x.T))
    assert_close(total.cpu().numpy(), ref, f"{G} virtual ranks")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_driver_reproduces_prefill_alone_and_in_a_one_rank_nccl_group():
    import torch.distributed as dist
    x = synth.make_inputs(0, B=2, T=700, H=4, topk=64, seed=72)
    g = _dev(x)
    ref = mla.mla_prefill(g["q"], g["kv_latent"], g["k_pe"], g["W_kvb"], g["W_o"], topk_idx=g["topk_idx"],
                          scale=x.scale)
    tp = HeadShardedPrefill(x.B, x.T, x.H, g["W_kvb"], g["W_o"], topk=64, scale=x.scale, chunk_rows=512)
    out = tp(g["q"], g["kv_latent"], g["k_pe"], g["topk_idx"])
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        tp1 = HeadShardedPrefill(x.B, x.T, x.H, g["W_kvb"], g["W_o"], topk=64, scale=x.scale, chunk_rows=512)
        assert tp1.world == 1 and (tp1.h0, tp1.h1) == (0, x.H)
        out1 = tp1(g["q"], g["kv_latent"], g["k_pe"], g["topk_idx"])
        torch.cuda.synchronize()
        assert torch.equal(out1, ref)
    finally:
        dist.destroy_process_group()
    _no_device_error()
