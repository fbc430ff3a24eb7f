"""Repeated launches (needs a B200): every kernel is deterministic and its
pipeline waits are bounded, so back-to-back calls on the same inputs must
return bit-identical outputs and leave the device error word clear. A race
between pipeline stages (a barrier phase waited for out of turn, a buffer
reused early) shows up here as a timed-out wait or a changed output long
before it would in a single parity run."""
import pytest
import torch

import synth

mla = pytest.importorskip("sparse_head_latent_b200")

pytestmark = pytest.mark.gpu


def _repeat(fn, reps):
    first = fn().clone()
    for i in range(reps):
        out = fn()
        assert mla.mla_device_status() == 0, f"device error on repetition {i}"
        assert torch.equal(out, first), f"output changed on repetition {i}"


def _dev(x):
    return {k: v.cuda() for k, v in x.tensors().items()}


def test_block_dense_attention_repeats_exactly():
    x = synth.make_inputs(1, T=2048, H=16, topk=1024)
    g = _dev(x)
    out = torch.empty(x.B, x.T, x.H, 128, dtype=torch.bfloat16, device="cuda")
    _repeat(lambda: mla.mla_attend(g["q"], g["kv_latent"], g["k_pe"], g["W_kvb"], topk_idx=g["topk_idx"],
                                   scale=x.scale, attn_out=out, path=mla.MLA_PATH_BLOCK_DENSE), 40)


def test_absorbed_attention_repeats_exactly():
    x = synth.make_inputs(1, T=4096, H=16, topk=256)
    g = _dev(x)
    out = torch.empty(x.B, x.T, x.H, 128, dtype=torch.bfloat16, device="cuda")
    _repeat(lambda: mla.mla_attend(g["q"], g["kv_latent"], g["k_pe"], g["W_kvb"], topk_idx=g["topk_idx"],
                                   scale=x.scale, attn_out=out, path=mla.MLA_PATH_ABSORBED), 20)


def test_decode_repeats_exactly():
    d = synth.make_decode_inputs(16, 8192, 32, 1024, seed=3)
    g = _dev(d)
    out = torch.empty(d.B, 7168, dtype=torch.bfloat16, device="cuda")
    _repeat(lambda: mla.mla_decode(g["q"], g["kv_latent"], g["k_pe"], g["W_kvb"], g["W_o"], topk_idx=g["topk_idx"],
                                   scale=d.scale, out=out), 40)


def test_e4m3_prefill_repeats_exactly():
    x = synth.make_inputs(4, B=2, H=16)
    g = _dev(x)
    out = torch.empty(x.B, x.T, 7168, dtype=torch.bfloat16, device="cuda")
    _repeat(lambda: mla.mla_prefill(g["q"], g["kv_latent"], g["k_pe"], g["W_kvb"], g["W_o"], g["W_kvb_scale"],
                                    g["W_o_scale"], topk_idx=g["topk_idx"], scale=x.scale, out=out,
                                    act=mla.MLA_ACT_E4M3_DYNAMIC), 20)
