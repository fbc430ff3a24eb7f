"""Full-size workloads on the GPU, checked on sampled rows against the oracle.

Each workload runs through mla_prefill and mla_attend with a preallocated
workspace, exactly as the benchmark launches them. The oracle then computes
(a) the attention output of sampled query rows for a few heads and (b) the
projected output of a few whole rows (all heads, then W_o). Rows include the
sequence ends, the rows around the top-k saturation point and the edges of
the first and last 128-row tiles. Same tolerances as the small cases.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.test_gpu_parity import assert_close

mla = pytest.importorskip("sparse_head_latent_b200")

pytestmark = pytest.mark.gpu

WORKLOADS = {
    # name: (config, overrides, rows for the full output check)
    "v32_sparse_T4096": (1, {}, [(0, 0), (0, 1), (0, 4095)]),
    "k2_causal_T8192": (2, {}, [(0, 1), (0, 2500)]),
    "long_sparse_T32768": (3, {}, [(0, 0), (0, 32767)]),
    "batched_fp8_B16": (4, {}, [(0, 5), (15, 1023)]),
    "max_T65536_H1": (0, dict(T=65536, H=1, topk=256, seed=5), [(0, 65535), (0, 300)]),
}


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_full_size_sampled_rows(name):
    cfg, over, out_rows = WORKLOADS[name]
    x = synth.make_inputs(cfg, **over)
    dev = torch.device("cuda")
    g = {k: v.to(dev) for k, v in x.tensors().items()}
    dims = mla.make_dims(x.B, x.T, x.H, x.topk_idx.shape[-1] if x.topk_idx is not None else 0, x.fp8)
    ws = torch.empty(mla.mla_workspace_bytes(dims, mla.MLA_ENTRY_PREFILL, x.topk_idx is not None),
                     dtype=torch.uint8, device=dev)
    out = mla.mla_prefill(g["q"], g["kv_latent"], g["k_pe"], g["W_kvb"], g["W_o"], g.get("W_kvb_scale"),
                          g.get("W_o_scale"), topk_idx=g.get("topk_idx"), scale=x.scale, workspace=ws)
    attn = mla.mla_attend(g["q"], g["kv_latent"], g["k_pe"], g["W_kvb"], g.get("W_kvb_scale"),
                          topk_idx=g.get("topk_idx"), scale=x.scale, workspace=ws)
    assert mla.mla_device_status() == 0
    del g
    out = out.view(-1, 7168)
    attn = attn.view(x.B * x.T, x.H, 128)

    # (a) attention output: sampled rows x a few heads
    rows = synth.sample_rows(x.B, x.T, x.topk, n_random=6, seed=cfg)
    heads = sorted({0, x.H - 1, x.H // 2, (7 * cfg + 3) % x.H})
    ref = oracle.attend_rows(x, rows, heads=heads)
    got = attn[torch.tensor(rows, device=attn.device)][:, heads].float().cpu().numpy()
    assert_close(got, ref, f"{name} attn")

    # (b) projected output of whole rows
    flat = [b * x.T + s for b, s in out_rows]
    ref_attn, ref_out = oracle.prefill_rows(x, flat)
    assert_close(out[torch.tensor(flat, device=out.device)].float().cpu().numpy(), ref_out, f"{name} out")
    assert_close(attn[torch.tensor(flat, device=attn.device)].float().cpu().numpy(), ref_attn,
                 f"{name} attn rows")
    assert np.isfinite(out.float().cpu().numpy()).all()
