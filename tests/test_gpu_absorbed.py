"""The absorbed path (latent-space attention over each row's gathered keys)
against the fp64 oracle, element by element (needs a B200).

The absorbed form reaches the same result as the block-dense form up to
rounding (k_nope = W_UK c and v = W_UV c are linear in the latent row c), so
it is held to the same tolerances: max-abs <= 2e-2 and relative L2 <= 5e-3
on the attention output and on the projected output.
"""
import pytest
import torch

import oracle
import synth

mla = pytest.importorskip("sparse_head_latent_b200")

from test_gpu_parity import ATTEND_CASES, _dev, _no_device_error, assert_close  # noqa: E402

pytestmark = pytest.mark.gpu

ABS = mla.MLA_PATH_ABSORBED

ABSORBED_CASES = {
    "tiny_sparse": ATTEND_CASES["tiny_sparse"],
    "ragged_sparse": ATTEND_CASES["ragged_sparse"],
    "short_rows": ATTEND_CASES["short_rows"],
    "fp8_sparse": ATTEND_CASES["fp8_sparse"],
    "groups_lone_tile_sparse": ATTEND_CASES["groups_lone_tile_sparse"],
    # three groups of 64 heads, the last one partly empty
    "heads_130": dict(B=1, T=200, H=130, topk=24),
    # a full head count and selections longer than one 64-key gather block
    "heads_128_long_lists": dict(B=1, T=700, H=128, topk=200),
}


def _attend(x, g, topk_idx="inputs", path=ABS):
    tk = g.get("topk_idx") if isinstance(topk_idx, str) else topk_idx
    return mla.mla_attend(g["q"], g["kv_latent"], g["k_pe"], g["W_kvb"], g.get("W_kvb_scale"), topk_idx=tk,
                          scale=x.scale, path=path)


@pytest.mark.parametrize("case", sorted(ABSORBED_CASES))
def test_absorbed_matches_oracle(case):
    x = synth.make_inputs(0, seed=51, **dict(ABSORBED_CASES[case]))
    g = _dev(x)
    attn = _attend(x, g)
    _no_device_error()
    ref = oracle.attend_rows(x, range(x.B * x.T))
    assert_close(attn.float().cpu().numpy().reshape(ref.shape), ref, case)


def test_absorbed_ignores_order_duplicates_and_out_of_range_entries():
    x = synth.make_inputs(0, B=2, T=256, H=2, topk=20, seed=52)
    g = _dev(x)
    base = _attend(x, g)
    tk = x.topk_idx.clone()
    perm = torch.rand(tk.shape, generator=torch.Generator().manual_seed(5)).argsort(-1)
    doubled = torch.cat([tk.gather(-1, perm), tk.flip(-1)], dim=-1).contiguous()
    assert torch.equal(base, _attend(x, g, topk_idx=doubled.cuda()))
    s_idx = torch.arange(x.T)[None, :, None]
    bad = torch.tensor([-1, -9, x.T, 1 << 30], dtype=torch.int32)
    fill = bad[torch.arange(tk.numel()).reshape(tk.shape) % 4]
    tk_bad = torch.where(tk > s_idx, fill, tk).contiguous()
    assert torch.equal(base, _attend(x, g, topk_idx=tk_bad.cuda()))
    _no_device_error()
    x.topk_idx = tk_bad
    ref = oracle.attend_rows(x, range(x.B * x.T))
    assert_close(base.float().cpu().numpy().reshape(ref.shape), ref, "dups/out-of-range")


def test_absorbed_rows_without_any_key_are_zero():
    x = synth.make_inputs(0, B=1, T=384, H=2, topk=8, seed=53)
    tk = x.topk_idx.clone()
    tk[0, 130:260] = -1
    x.topk_idx = tk
    g = _dev(x)
    attn = _attend(x, g)
    _no_device_error()
    assert not attn[0, 130:260].any()
    ref = oracle.attend_rows(x, range(x.T))
    assert_close(attn.float().cpu().numpy().reshape(ref.shape), ref, "empty rows")


def test_absorbed_single_selected_key_returns_its_value():
    # Softmax over one key is exactly 1, so o_lat is that key's latent row and
    # the un-absorb GEMM reproduces v = W_UV c up to the final bf16 rounding.
    x = synth.make_inputs(0, B=1, T=200, H=2, topk=4, seed=54)
    x.topk_idx = torch.full_like(x.topk_idx, 150)
    g = _dev(x)
    attn = _attend(x, g)
    kvh = mla.mla_kv_upproject(g["kv_latent"], g["W_kvb"]).view(x.T, 2, 256)
    _no_device_error()
    assert not attn[0, :150].any()
    v = kvh[150, :, 128:].float()
    got = attn[0, 150:].float()
    assert torch.all((got - v).abs() <= v.abs() * 2.0 ** -7 + 1e-30)


def test_auto_hybrid_matches_oracle_and_both_paths():
    # With topk = 64 the automatic choice keeps the first 512-row group
    # block-dense and sends the later groups to the absorbed path.
    x = synth.make_inputs(0, B=1, T=2048, H=2, topk=64, seed=55)
    g = _dev(x)
    auto = _attend(x, g, path=mla.MLA_PATH_AUTO)
    dense = _attend(x, g, path=mla.MLA_PATH_BLOCK_DENSE)
    absorbed = _attend(x, g, path=ABS)
    _no_device_error()
    assert torch.equal(auto[0, :512], dense[0, :512])
    assert torch.equal(auto[0, 512:], absorbed[0, 512:])
    ref = oracle.attend_rows(x, range(x.T))
    assert_close(auto.float().cpu().numpy().reshape(ref.shape), ref, "auto")


@pytest.mark.parametrize("case", ["ragged_sparse", "fp8_sparse"])
def test_absorbed_prefill_matches_oracle(case):
    x = synth.make_inputs(0, seed=56, **dict(ATTEND_CASES[case]))
    g = _dev(x)
    out = mla.mla_prefill(g["q"], g["kv_latent"], g["k_pe"], g["W_kvb"], g["W_o"], g.get("W_kvb_scale"),
                          g.get("W_o_scale"), topk_idx=g.get("topk_idx"), scale=x.scale, path=ABS)
    _no_device_error()
    rows = list(range(x.B * x.T))
    _, ref_out = oracle.prefill_rows(x, rows)
    assert_close(out.float().cpu().numpy().reshape(len(rows), 7168), ref_out, case)
