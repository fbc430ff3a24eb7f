"""Head-sharded (tensor-parallel) prefill of one sequence batch over several GPUs.

DeepSeek-V3.2-Exp "Sparse attention" page, MLA init: wkv_b is a
ColumnParallelLinear and wo a RowParallelLinear, with n_local_heads heads per
rank. So each of G ranks owns a contiguous range of heads: the W_kvb rows of
those heads (k_nope and v, 256 rows per head), their queries, their attention,
and the W_o rows that read their outputs (128 rows per head). The selection
(top-k indices) and the shared latent and rotary key are replicated. Every
rank produces a full-width partial output [B*T, 7168] from its heads; the
block's output is the sum over ranks, the only exchange. As in the pages'
RowParallelLinear, the partial outputs are bf16 and summed by an all-reduce.

The sum is overlapped with the output projection: the rows are cut into
chunks; the W_o GEMM of chunk i+1 runs on the compute stream while chunk i is
all-reduced on a communication stream (NCCL over NVLink).

Plumbing only: every step of the computation is a C-ABI call (mla_attend,
mla_out_project); this module slices weights, orders launches and issues the
collective.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Tuple

import torch

from .mla import (MLA_ACT_BF16, MLA_ENTRY_ATTEND, MLA_ENTRY_OUT_PROJECT, MLA_PATH_AUTO, D_MODEL, D_NOPE, D_ROPE,
                  D_V, _wtype, make_dims, mla_attend, mla_out_project, mla_workspace_bytes)


def head_range(H: int, world: int, rank: int) -> Tuple[int, int]:
    """Heads [h0, h1) of `rank`: contiguous, as even as possible (the first
    H % world ranks take one more)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    base, extra = divmod(H, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def shard_weights(W_kvb, W_o, W_kvb_scale=None, W_o_scale=None, h0: int = 0, h1: int = 1):
    """The rows of heads [h0, h1): W_kvb [256 per head, 512], W_o [128 per head,
    7168] and, for e4m3 weights, their 128 x 128 block scales (2 and 1 scale
    rows per head). Returned contiguous (views of the full tensors are not)."""
    per = D_NOPE + D_V
    out = {"W_kvb": W_kvb[h0 * per:h1 * per].contiguous(), "W_o": W_o[h0 * D_V:h1 * D_V].contiguous()}
    out["W_kvb_scale"] = None if W_kvb_scale is None else W_kvb_scale[h0 * per // 128:h1 * per // 128].contiguous()
    out["W_o_scale"] = None if W_o_scale is None else W_o_scale[h0 * D_V // 128:h1 * D_V // 128].contiguous()
    return out


def row_chunks(M: int, chunk_rows: int) -> List[Tuple[int, int]]:
    """[r0, r1) ranges covering [0, M) in order; all but the last chunk_rows long."""
    if chunk_rows < 1:
        raise ValueError("chunk_rows must be positive")
    return [(r0, min(M, r0 + chunk_rows)) for r0 in range(0, M, chunk_rows)]


def reduce_chunks(partial: torch.Tensor, chunks, project: Callable[[int, int], None],
                  all_reduce: Callable[[torch.Tensor], None], wait_compute: Callable[[], None] = lambda: None):
    """Drives the overlap: for each chunk, `project(r0, r1)` writes its rows of
    `partial`; `all_reduce(rows)` then sums them across ranks (asynchronously
    on a communication stream, after `wait_compute()` has ordered it behind the
    projection)."""
    for r0, r1 in chunks:
        project(r0, r1)
        wait_compute()
        all_reduce(partial[r0:r1])


class HeadShardedPrefill:
    """mla_prefill with the heads split over the ranks of a process group.

    Each rank passes its own query heads q_local [B, T, H_local, 192] (as a
    column-parallel query projection produces them) and the replicated
    kv_latent, k_pe and topk_idx; every rank receives the full output
    [B, T, 7168]."""

    def __init__(self, B, T, H, W_kvb, W_o, W_kvb_scale=None, W_o_scale=None, topk=None, scale=192 ** -0.5,
                 group=None, chunk_rows=2048, path=MLA_PATH_AUTO, act=MLA_ACT_BF16, device=None):
        import torch.distributed as dist
        self.dist = dist if dist.is_available() and dist.is_initialized() else None
        self.group = group
        self.world = self.dist.get_world_size(group) if self.dist else 1
        self.rank = self.dist.get_rank(group) if self.dist else 0
        self.B, self.T, self.H = B, T, H
        self.h0, self.h1 = head_range(H, self.world, self.rank)
        self.Hl = self.h1 - self.h0
        self.scale, self.path, self.act = float(scale), path, act
        self.w = shard_weights(W_kvb, W_o, W_kvb_scale, W_o_scale, self.h0, self.h1)
        dev = torch.device(device) if device is not None else W_o.device
        fp8 = _wtype(W_kvb)
        M = B * T
        dims_a = make_dims(B, T, self.Hl, 0 if topk is None else topk, fp8, path, act)
        self.ws_attend = torch.empty(max(1, mla_workspace_bytes(dims_a, MLA_ENTRY_ATTEND, topk is not None)),
                                     dtype=torch.uint8, device=dev)
        self.chunks = row_chunks(M, chunk_rows)
        dims_o = make_dims(1, self.chunks[0][1] - self.chunks[0][0], self.Hl, 0, fp8, act=act)
        self.ws_out = torch.empty(max(1, mla_workspace_bytes(dims_o, MLA_ENTRY_OUT_PROJECT, False)),
                                  dtype=torch.uint8, device=dev)
        self.attn = torch.empty(B, T, self.Hl, D_V, dtype=torch.bfloat16, device=dev)
        self.comm = torch.cuda.Stream(dev) if dev.type == "cuda" else None

    def __call__(self, q_local, kv_latent, k_pe, topk_idx=None, out=None):
        B, T, Hl = self.B, self.T, self.Hl
        if tuple(q_local.shape) != (B, T, Hl, D_NOPE + D_ROPE):
            raise ValueError(f"q_local must be [B, T, {Hl}, 192] (heads {self.h0}..{self.h1 - 1})")
        M = B * T
        if out is None:
            out = torch.empty(B, T, D_MODEL, dtype=torch.bfloat16, device=q_local.device)
        compute = torch.cuda.current_stream(q_local.device)
        mla_attend(q_local, kv_latent, k_pe, self.w["W_kvb"], self.w["W_kvb_scale"], topk_idx=topk_idx,
                   scale=self.scale, attn_out=self.attn, workspace=self.ws_attend, stream=compute, path=self.path,
                   act=self.act)
        rows_attn = self.attn.view(M, Hl * D_V)
        part = out.view(M, D_MODEL)
        works = []

        def project(r0, r1):
            mla_out_project(rows_attn[r0:r1], self.w["W_o"], self.w["W_o_scale"], out=part[r0:r1],
                            workspace=self.ws_out, stream=compute, act=self.act)

        def wait_compute():
            if self.comm is not None:
                self.comm.wait_stream(compute)

        def all_reduce(rows):
            if self.dist is None or self.world == 1:
                return
            with torch.cuda.stream(self.comm):
                works.append(self.dist.all_reduce(rows, group=self.group, async_op=True))

        reduce_chunks(part, self.chunks, project, all_reduce, wait_compute)
        for w in works:
            w.wait()  # makes the current stream wait for the collectives
        if self.comm is not None:
            compute.wait_stream(self.comm)
        return out
