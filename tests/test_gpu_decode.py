"""Decode (one new position per sequence against its cache) against the
fp64 oracle (needs a B200).

Decoding the position s = T-1 of a sequence whose cache holds positions
0..T-1 computes exactly row T-1 of the prefill block for that sequence, so
the oracle's prefill rows are the reference. Same tolerances as prefill:
max-abs <= 2e-2 and relative L2 <= 5e-3 on the projected output.
"""
import pytest
import torch

import oracle
import synth

mla = pytest.importorskip("sparse_head_latent_b200")

from test_gpu_parity import _no_device_error, assert_close  # noqa: E402

pytestmark = pytest.mark.gpu

DECODE_CASES = {
    "ragged_cache": dict(B=2, T=300, H=3, topk=40),
    "heads_128": dict(B=3, T=1100, H=128, topk=300),
    "fp8_weights": dict(B=2, T=200, H=2, topk=24, fp8=True),
    "every_position": dict(B=2, T=150, H=4, topk=None),
    "one_token_cache": dict(B=3, T=1, H=2, topk=4),
    # few sequences and long selections: each query's keys are split over
    # several CTAs and the partial results combined
    "split_keys": dict(B=2, T=3000, H=4, topk=1024),
    "split_keys_64_heads": dict(B=1, T=2100, H=64, topk=1024),
    # more than 64 sequences: the per-head and output GEMMs take 128-row
    # tiles, the second one partly past the last row
    "batch_100": dict(B=100, T=40, H=4, topk=12),
}


def _decode(x, topk_last=None):
    g = {k: v.cuda() for k, v in x.tensors().items()}
    T = x.T
    q = g["q"][:, T - 1].contiguous()
    tk = None
    if x.topk_idx is not None:
        tk = (x.topk_idx[:, T - 1] if topk_last is None else topk_last).contiguous().cuda()
    out = mla.mla_decode(q, g["kv_latent"], g["k_pe"], g["W_kvb"], g["W_o"], g.get("W_kvb_scale"),
                         g.get("W_o_scale"), topk_idx=tk, scale=x.scale)
    _no_device_error()
    return out


def _reference(x):
    rows = [b * x.T + x.T - 1 for b in range(x.B)]
    _, ref_out = oracle.prefill_rows(x, rows)
    return ref_out


@pytest.mark.parametrize("case", sorted(DECODE_CASES))
def test_decode_matches_oracle(case):
    x = synth.make_inputs(0, seed=61, **dict(DECODE_CASES[case]))
    out = _decode(x)
    assert_close(out.float().cpu().numpy(), _reference(x), case)


def test_decode_ignores_order_duplicates_and_out_of_range_entries():
    x = synth.make_inputs(0, B=2, T=257, H=2, topk=32, seed=62)
    base = _decode(x)
    tk = x.topk_idx[:, x.T - 1].clone()
    messy = torch.cat([tk.flip(-1), tk, torch.tensor([[-1, x.T, 1 << 30, -7]] * x.B, dtype=torch.int32)], dim=-1)
    assert torch.equal(base, _decode(x, messy))


def test_decode_sequence_without_a_valid_key_is_zero():
    x = synth.make_inputs(0, B=2, T=64, H=2, topk=8, seed=63)
    tk = x.topk_idx[:, x.T - 1].clone()
    tk[1] = -1
    out = _decode(x, tk)
    assert not out[1].any()
    x.topk_idx[:, x.T - 1] = tk
    assert_close(out[:1].float().cpu().numpy(), _reference(x)[:1], "valid sequence")


def test_decode_split_with_empty_parts():
    # 1024 entries but about 300 distinct keys: the split is planned for 1024
    # (four parts), so the last parts of the row receive no key at all.
    x = synth.make_inputs(0, B=2, T=2000, H=4, topk=1024, seed=64)
    tk = x.topk_idx[:, x.T - 1].clone()
    tk = tk[:, :300].repeat(1, 4)[:, :1024].contiguous()
    out = _decode(x, tk)
    x.topk_idx[:, x.T - 1] = tk
    assert_close(out.float().cpu().numpy(), _reference(x), "empty parts")


def test_decode_replays_from_a_cuda_graph():
    # The decode step only enqueues kernels on the given stream, so it can be
    # captured once and replayed; the replay must reproduce the eager result
    # bit for bit, also after the inputs change in place.
    x = synth.make_inputs(0, B=4, T=2500, H=16, topk=512, seed=65)
    g = {k: v.cuda() for k, v in x.tensors().items()}
    T = x.T
    q = g["q"][:, T - 1].contiguous()
    tk = x.topk_idx[:, T - 1].contiguous().cuda()
    dims = mla.make_dims(x.B, T, x.H, tk.shape[-1], False)
    ws = torch.empty(mla.mla_workspace_bytes(dims, mla.MLA_ENTRY_DECODE, True), dtype=torch.uint8, device="cuda")
    out = torch.empty(x.B, 7168, dtype=torch.bfloat16, device="cuda")

    def step(st=None):
        mla.mla_decode(q, g["kv_latent"], g["k_pe"], g["W_kvb"], g["W_o"], topk_idx=tk, scale=x.scale,
                       out=out, workspace=ws, stream=st)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    eager = out.clone()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step(torch.cuda.current_stream())
    out.zero_()
    graph.replay()
    torch.cuda.synchronize()
    _no_device_error()
    assert torch.equal(out, eager)
    # new inputs written in place: the replay must agree with a fresh eager call
    q.mul_(-1)
    tk.copy_(torch.flip(tk, dims=[-1]) // 2)
    graph.replay()
    torch.cuda.synchronize()
    replayed = out.clone()
    step()
    torch.cuda.synchronize()
    _no_device_error()
    assert torch.equal(replayed, out)
    assert not torch.equal(replayed, eager)
    del graph
