"""Failure detection on the GPU without a fault.

1. A bounded wait runs out: with the test hook on, the block-dense attention
   kernel's producer issues no loads, so its waits (for the loads and for
   the tensor-core work that would follow) reach the time limit, which is
   lowered to 2 ms for the test. The kernel must record a 1xx code in the
   device error word and exit (the call returns within a bounded time), and
   the next call on the same stream must succeed and reproduce the earlier
   result bit for bit.
2. The attention path stores the up-projected values v as f16. Values of v
   inside the f16 range still match the oracle (W_kvb's v rows are scaled by
   a power of two, which scales attn exactly and leaves the scores alone, so
   attn is compared after dividing by it); values that overflow f16 are
   reported with device code 301 instead of silently giving inf / NaN.
"""
import time

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.test_gpu_parity import assert_close

mla = pytest.importorskip("sparse_head_latent_b200")

pytestmark = pytest.mark.gpu


def _attend(g, x):
    return mla.mla_attend(g["q"], g["kv_latent"], g["k_pe"], g["W_kvb"], g.get("W_kvb_scale"),
                          topk_idx=g.get("topk_idx"), scale=x.scale, path=mla.MLA_PATH_BLOCK_DENSE)


def test_withheld_loads_end_in_a_wait_timeout_and_the_next_call_succeeds():
    x = synth.make_inputs(0, B=1, T=300, H=2, topk=40, seed=81)
    g = {k: v.cuda() for k, v in x.tensors().items()}
    good = _attend(g, x)
    assert mla.mla_device_status() == 0
    mla.mla_set_wait_timeout_ns(2_000_000)
    mla.mla_test_withhold_attention_loads(True)
    try:
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        _attend(g, x)
        err = mla.mla_device_status()
        dt = time.perf_counter() - t0
    finally:
        mla.mla_test_withhold_attention_loads(False)
        mla.mla_set_wait_timeout_ns(0)
    assert 100 < err < 200, err
    assert dt < 5.0, dt  # a few 2 ms limits in sequence, not the 1 s default, and no hang
    again = _attend(g, x)
    assert mla.mla_device_status() == 0
    assert torch.equal(again, good)


def _scaled_v(x, c):
    """The same problem with W_kvb's v rows multiplied by c, a power of two
    (exact in bf16 and in the fp32 block scales): v = W_v . latent scales by
    c, while the keys, and so the scores and softmax weights, do not change."""
    wk, ws = x.W_kvb.clone(), None if x.W_kvb_scale is None else x.W_kvb_scale.clone()
    if x.fp8:
        ws.view(x.H, 2, -1)[:, 1] *= c  # block-scale rows of each head's v half (128 rows each)
    else:
        wk.view(x.H, 256, 512)[:, 128:] = (wk.view(x.H, 256, 512)[:, 128:].float() * c).to(torch.bfloat16)
    return synth.MlaInputs(B=x.B, T=x.T, H=x.H, topk=x.topk, fp8=x.fp8, scale=x.scale, q=x.q,
                           kv_latent=x.kv_latent, k_pe=x.k_pe, W_kvb=wk, W_kvb_scale=ws, W_o=x.W_o,
                           W_o_scale=x.W_o_scale, topk_idx=x.topk_idx)


def _max_abs_v(x):
    rows = torch.arange(x.T)
    v = oracle.upproject_rows(x, rows.tolist()).reshape(x.T, x.H, 256)[:, :, 128:]
    return float(np.abs(v).max())


MODES = {"bf16": (False, mla.MLA_ACT_BF16), "fp8_weights": (True, mla.MLA_ACT_BF16),
         "fp8_weights_e4m3_act": (True, mla.MLA_ACT_E4M3_DYNAMIC)}


@pytest.mark.parametrize("mode", list(MODES))
def test_large_v_inside_the_f16_range_matches_the_oracle(mode):
    fp8, act = MODES[mode]
    x = synth.make_inputs(0, B=1, T=260, H=2, topk=48, seed=82, fp8=fp8)
    c = 2.0 ** 13  # v ~ N(0, c^2): the largest |v| here is a few times c, below 65504
    y = _scaled_v(x, c)
    assert 16384 < _max_abs_v(y) < 65000
    g = {k: v.cuda() for k, v in y.tensors().items()}
    got = mla.mla_attend(g["q"], g["kv_latent"], g["k_pe"], g["W_kvb"], g.get("W_kvb_scale"),
                         topk_idx=g["topk_idx"], scale=y.scale, path=mla.MLA_PATH_BLOCK_DENSE, act=act)
    assert mla.mla_device_status() == 0
    rows = list(range(y.T))
    ref = oracle.attend_rows(y, rows, act_e4m3=act != 0)
    got = got.view(y.T, y.H, 128).float().cpu().numpy()
    assert np.isfinite(got).all()
    assert_close(got / c, ref / c, f"{mode}: v x {c:g}, attn / {c:g}")


@pytest.mark.parametrize("mode", list(MODES))
def test_v_beyond_the_f16_range_is_reported(mode):
    fp8, act = MODES[mode]
    x = synth.make_inputs(0, B=1, T=260, H=2, topk=48, seed=83, fp8=fp8)
    y = _scaled_v(x, 2.0 ** 17)
    assert _max_abs_v(y) > 65520
    g = {k: v.cuda() for k, v in y.tensors().items()}
    mla.mla_attend(g["q"], g["kv_latent"], g["k_pe"], g["W_kvb"], g.get("W_kvb_scale"), topk_idx=g["topk_idx"],
                   scale=y.scale, path=mla.MLA_PATH_BLOCK_DENSE, act=act)
    assert mla.mla_device_status() == 301
    # the read cleared the error word, and the unscaled problem runs clean
    g = {k: v.cuda() for k, v in x.tensors().items()}
    mla.mla_attend(g["q"], g["kv_latent"], g["k_pe"], g["W_kvb"], g.get("W_kvb_scale"), topk_idx=g["topk_idx"],
                   scale=x.scale, path=mla.MLA_PATH_BLOCK_DENSE, act=act)
    assert mla.mla_device_status() == 0
