"""CUDA path vs the fp64 oracle, element by element (needs a B200).

Every call goes through the C ABI (libmla_b200.so) via the ctypes binding.
The attention calls here use the block-dense path explicitly (the absorbed
path has its own file); the whole-block tests also run the automatic choice.
Tolerances: max-abs <= 2e-2 and relative L2 <= 5e-3 on the attention output
and on the projected output (and on the up-projected kv, which feeds both).
Small cases are compared in full; they span several 128-row tiles and a
ragged tail.
"""
import numpy as np
import pytest
import torch

import oracle
import synth

mla = pytest.importorskip("sparse_head_latent_b200")

pytestmark = pytest.mark.gpu

MAX_ABS, REL_L2 = 2e-2, 5e-3


def _dev(x):
    return {k: v.cuda() for k, v in x.tensors().items()}


def assert_close(got, ref, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    d = got - ref
    max_abs = float(np.abs(d).max()) if d.size else 0.0
    nref = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(d) / nref) if nref > 0 else float(np.linalg.norm(d))
    assert max_abs <= MAX_ABS and rel <= REL_L2, f"{what}: max_abs={max_abs:.3e} rel_l2={rel:.3e}"
    return max_abs, rel


def _no_device_error():
    assert mla.mla_device_status() == 0


DENSE = mla.MLA_PATH_BLOCK_DENSE


def _attend(x, g, topk_idx="inputs", path=DENSE):
    tk = g.get("topk_idx") if isinstance(topk_idx, str) else topk_idx
    return mla.mla_attend(g["q"], g["kv_latent"], g["k_pe"], g["W_kvb"], g.get("W_kvb_scale"),
                          topk_idx=tk, scale=x.scale, path=path)


# ---------------------------------------------------------------- GEMM stages

@pytest.mark.parametrize("fp8", [False, True])
@pytest.mark.parametrize("B,T,H", [(1, 128, 1), (2, 300, 4), (1, 1000, 2)])
def test_upprojection_matches_oracle(B, T, H, fp8):
    x = synth.make_inputs(0, B=B, T=T, H=H, topk=None, seed=21, fp8=fp8)
    g = _dev(x)
    kvh = mla.mla_kv_upproject(g["kv_latent"], g["W_kvb"], g.get("W_kvb_scale"))
    _no_device_error()
    ref = oracle.upproject_rows(x, range(B * T))
    assert_close(kvh.float().cpu().numpy(), ref, "kvh")


def test_gemms_with_a_ragged_last_row_tile_over_many_tiles():
    # 700 rows leave the last 256-row tile partly empty: the epilogue warps
    # whose 32 rows lie past the end store nothing there. Each CTA pair runs
    # several tiles, so the tile it finished before such a tile must still be
    # stored whole (its last chunk used to be overwritten while in flight).
    gen = torch.Generator().manual_seed(7)
    rows, H = 700, 128
    lat = torch.randn(rows, 512, generator=gen).to(torch.bfloat16).cuda()
    W_kvb = (torch.randn(H * 256, 512, generator=gen) * 512 ** -0.5).to(torch.bfloat16).cuda()
    kvh = mla.mla_kv_upproject(lat, W_kvb)
    attn = torch.randn(rows, H * 128, generator=gen).to(torch.bfloat16).cuda()
    W_o = (torch.randn(H * 128, 7168, generator=gen) * (H * 128) ** -0.5).to(torch.bfloat16).cuda()
    out = mla.mla_out_project(attn, W_o)
    _no_device_error()
    for got, ref in ((kvh, lat.float() @ W_kvb.float().T), (out, attn.float() @ W_o.float())):
        err = (got.float() - ref).abs()
        assert bool((err <= ref.abs() * 2.0 ** -8 + 1e-3).all()), float(err.max())


@pytest.mark.parametrize("fp8", [False, True])
@pytest.mark.parametrize("rows,H", [(128, 1), (300, 4), (517, 2)])
def test_output_projection_matches_oracle(rows, H, fp8):
    x = synth.make_inputs(0, T=8, H=H, topk=None, seed=22, fp8=fp8)
    gen = torch.Generator().manual_seed(rows)
    attn = (0.05 * torch.randn(rows, H * 128, generator=gen)).to(torch.bfloat16)
    g = _dev(x)
    out = mla.mla_out_project(attn.cuda(), g["W_o"], g.get("W_o_scale"))
    _no_device_error()
    ref = oracle.project_rows(x, attn.to(torch.float64).numpy())
    assert_close(out.float().cpu().numpy(), ref, "out")


@pytest.mark.parametrize("rows,H", [(600, 32), (1300, 128)])
def test_output_projection_with_k_split_last_wave_matches_oracle(rows, H):
    # bf16 W_o with K = H * 128 >= 4096 and a tile count that leaves the last
    # wave of CTA pairs partial (600 rows: 84 tiles of 256 x 256, 10 of them
    # in the last wave on 74 pairs; 1300 rows: 168 tiles, 20): those tiles are
    # cut along K, and a second kernel adds their fp32 partials. Whole rows
    # cover every column tile (whole and split ones), the ragged last row
    # tile included; a repeat must give the same bits.
    x = synth.make_inputs(0, T=8, H=H, topk=None, seed=23)
    gen = torch.Generator().manual_seed(rows)
    attn = (0.05 * torch.randn(rows, H * 128, generator=gen)).to(torch.bfloat16)
    g = _dev(x)
    mla.mla_profile_begin()
    out = mla.mla_out_project(attn.cuda(), g["W_o"])
    prof = mla.mla_profile_end()
    _no_device_error()
    if torch.cuda.get_device_properties(0).multi_processor_count == 148:
        assert prof["gemm_wo_split_sum"][1] == 1
    sample = sorted({0, 1, 127, 128, 255, 256, 511, 512, rows // 2, rows - 2, rows - 1})
    ref = oracle.project_rows(x, attn[sample].to(torch.float64).numpy())
    assert_close(out[sample].float().cpu().numpy(), ref, "out")
    assert torch.equal(mla.mla_out_project(attn.cuda(), g["W_o"]), out)
    _no_device_error()


def _dequant_bf16(codes, scale):
    """bf16(e4m3(code) * block scale), the fp32 product rounded to nearest even."""
    R, C = codes.shape
    f = codes.view(torch.float8_e4m3fn).to(torch.float32).view(R // 128, 128, C // 128, 128)
    return (f * scale[:, None, :, None]).view(R, C).to(torch.bfloat16)


class _OnChip:
    """Context: e4m3 weights with bf16 activations converted on chip by the
    projection GEMMs (mla_set_e4m3_weight_conversion), restored on exit."""

    def __init__(self, on):
        self.on = on

    def __enter__(self):
        mla.mla_set_e4m3_weight_conversion(self.on)

    def __exit__(self, *exc):
        mla.mla_set_e4m3_weight_conversion(False)


@pytest.mark.parametrize("onchip", [False, True], ids=["dequant", "onchip"])
@pytest.mark.parametrize("stage", ["kv_upproject", "out_project"])
def test_fp8_weight_gemms_equal_the_bf16_gemm_on_the_dequantised_weight(stage, onchip):
    # With bf16 activations each e4m3 weight becomes bf16(code * block scale),
    # the fp32 product rounded once, either in a dequantised copy or (onchip)
    # by converter warps writing the tensor-core operand; the bf16 GEMM on
    # the weight dequantised the same way on the host must give the same
    # bits. Several row tiles (ragged), column tiles and 128-deep K blocks.
    x = synth.make_inputs(0, B=1, T=600, H=4, topk=None, seed=36, fp8=True)
    g = _dev(x)
    if stage == "kv_upproject":
        with _OnChip(onchip):
            got = mla.mla_kv_upproject(g["kv_latent"], g["W_kvb"], g["W_kvb_scale"])
        ref = mla.mla_kv_upproject(g["kv_latent"], _dequant_bf16(x.W_kvb, x.W_kvb_scale).cuda())
    else:
        gen = torch.Generator().manual_seed(37)
        attn = (0.05 * torch.randn(x.T, x.H * 128, generator=gen)).to(torch.bfloat16).cuda()
        with _OnChip(onchip):
            got = mla.mla_out_project(attn, g["W_o"], g["W_o_scale"])
        ref = mla.mla_out_project(attn, _dequant_bf16(x.W_o, x.W_o_scale).cuda())
    _no_device_error()
    assert torch.equal(got, ref)


@pytest.mark.parametrize("stage", ["kv_upproject", "out_project"])
def test_fp8_weight_gemms_bit_exact_over_many_units(stage):
    # On-chip conversion with enough rows and heads that every CTA pair walks
    # several work units: up-projection pairs cross from one 256-feature tile
    # to the next inside their range (the weights converted into tensor
    # memory are replaced), output-projection pairs take several 384-token
    # units, and the last unit is ragged (4100 rows).
    x = synth.make_inputs(0, B=1, T=4100, H=16, topk=None, seed=38, fp8=True)
    g = _dev(x)
    if stage == "kv_upproject":
        with _OnChip(True):
            got = mla.mla_kv_upproject(g["kv_latent"], g["W_kvb"], g["W_kvb_scale"])
        ref = mla.mla_kv_upproject(g["kv_latent"], _dequant_bf16(x.W_kvb, x.W_kvb_scale).cuda())
    else:
        gen = torch.Generator().manual_seed(39)
        attn = (0.05 * torch.randn(x.T, x.H * 128, generator=gen)).to(torch.bfloat16).cuda()
        with _OnChip(True):
            got = mla.mla_out_project(attn, g["W_o"], g["W_o_scale"])
        ref = mla.mla_out_project(attn, _dequant_bf16(x.W_o, x.W_o_scale).cuda())
    _no_device_error()
    assert torch.equal(got, ref)


@pytest.mark.parametrize("path", [mla.MLA_PATH_BLOCK_DENSE, mla.MLA_PATH_AUTO], ids=["dense", "auto"])
def test_prefill_with_e4m3_weights_converted_on_chip_equals_dequantised(path):
    # The whole block with e4m3 weights: converting on chip must reproduce the
    # dequantise-then-bf16 result bit for bit, also when some rows take the
    # absorbed path (which keeps a bf16 copy of W_kvb for its GEMMs).
    x = synth.make_inputs(0, B=2, T=1100, H=8, topk=48, seed=40, fp8=True)
    g = _dev(x)

    def run():
        return mla.mla_prefill(g["q"], g["kv_latent"], g["k_pe"], g["W_kvb"], g["W_o"], g["W_kvb_scale"],
                               g["W_o_scale"], topk_idx=g["topk_idx"], scale=x.scale, path=path)

    ref = run()
    with _OnChip(True):
        got = run()
    _no_device_error()
    assert torch.equal(got, ref)


# ---------------------------------------------------------------- attention

ATTEND_CASES = {
    "tiny_sparse": dict(B=1, T=128, H=8, topk=32),
    "ragged_sparse": dict(B=2, T=300, H=3, topk=40),
    "ragged_causal": dict(B=1, T=300, H=2, topk=None),
    "short_rows": dict(B=1, T=77, H=2, topk=100),
    "four_tiles": dict(B=1, T=512, H=2, topk=96),
    "fp8_sparse": dict(B=2, T=200, H=2, topk=24, fp8=True),
    # Several groups of four query tiles; the last group is ragged: six tiles
    # (no second super-tile), nine tiles (a lone tile whose pair partner lies
    # past T).
    "groups_ragged_sparse": dict(B=2, T=700, H=2, topk=200),
    "groups_lone_tile_causal": dict(B=1, T=1100, H=2, topk=None),
    "groups_lone_tile_sparse": dict(B=1, T=1100, H=3, topk=300),
}


@pytest.mark.parametrize("case", sorted(ATTEND_CASES))
def test_attend_matches_oracle(case):
    c = dict(ATTEND_CASES[case])
    x = synth.make_inputs(0, seed=31, **c)
    g = _dev(x)
    attn = _attend(x, g)
    _no_device_error()
    ref = oracle.attend_rows(x, range(x.B * x.T))
    assert_close(attn.float().cpu().numpy().reshape(ref.shape), ref, case)


# The full head count of the headline workload, compared in full: the head-
# group scheduler (groups of 8 heads, heaviest tile groups first) and the
# tile-group logic at H = 128, on a sparse case and a ragged causal one.
FULL_HEAD_CASES = {
    "h128_sparse": dict(B=1, T=1024, H=128, topk=256),
    "h128_ragged_causal": dict(B=2, T=700, H=128, topk=None),
}


@pytest.mark.parametrize("case", sorted(FULL_HEAD_CASES))
def test_attend_all_128_heads_matches_oracle(case):
    x = synth.make_inputs(0, seed=35, **FULL_HEAD_CASES[case])
    g = _dev(x)
    attn = _attend(x, g)
    _no_device_error()
    ref = oracle.attend_rows_threaded(x, range(x.B * x.T))
    assert_close(attn.float().cpu().numpy().reshape(ref.shape), ref, case)


def test_topk_listing_every_key_equals_causal_only():
    x = synth.make_inputs(0, B=1, T=260, H=2, topk=260, seed=32)
    g = _dev(x)
    full = _attend(x, g)
    causal = _attend(x, g, topk_idx=None)
    _no_device_error()
    assert torch.equal(full, causal)
    ref = oracle.attend_rows(x, range(x.T))
    assert_close(causal.float().cpu().numpy().reshape(ref.shape), ref, "causal")


def test_order_duplicates_and_out_of_range_entries():
    x = synth.make_inputs(0, B=2, T=256, H=2, topk=20, seed=33)
    g = _dev(x)
    base = _attend(x, g)
    tk = x.topk_idx.clone()
    gen = torch.Generator().manual_seed(3)
    perm = torch.rand(tk.shape, generator=gen).argsort(-1)
    shuffled = tk.gather(-1, perm)
    doubled = torch.cat([shuffled, shuffled.flip(-1)], dim=-1).contiguous()
    assert torch.equal(base, _attend(x, g, topk_idx=doubled.cuda()))
    # Entries above s never survive; out-of-range values in their place change nothing.
    s_idx = torch.arange(x.T)[None, :, None]
    bad = torch.tensor([-1, -9, x.T, 1 << 30], dtype=torch.int32)
    fill = bad[torch.arange(tk.numel()).reshape(tk.shape) % 4]
    tk_bad = torch.where(tk > s_idx, fill, tk).contiguous()
    assert torch.equal(base, _attend(x, g, topk_idx=tk_bad.cuda()))
    _no_device_error()
    x.topk_idx = tk_bad
    ref = oracle.attend_rows(x, range(x.B * x.T))
    assert_close(base.float().cpu().numpy().reshape(ref.shape), ref, "dups/out-of-range")


def test_rows_without_any_key_are_zero():
    x = synth.make_inputs(0, B=1, T=384, H=2, topk=8, seed=34)
    tk = x.topk_idx.clone()
    tk[0, 130:260] = -1                      # a whole tile and parts of two more
    x.topk_idx = tk
    g = _dev(x)
    attn = _attend(x, g)
    _no_device_error()
    assert not attn[0, 130:260].any()
    ref = oracle.attend_rows(x, range(x.T))
    assert_close(attn.float().cpu().numpy().reshape(ref.shape), ref, "empty rows")


def test_single_selected_key_returns_its_value():
    x = synth.make_inputs(0, B=1, T=200, H=2, topk=4, seed=35)
    x.topk_idx = torch.full_like(x.topk_idx, 150)
    g = _dev(x)
    attn = _attend(x, g)
    kvh = mla.mla_kv_upproject(g["kv_latent"], g["W_kvb"]).view(x.T, 2, 256)
    _no_device_error()
    assert not attn[0, :150].any()
    # Softmax over one key is exactly 1, so each row is that key's v. The
    # attention path keeps v in f16 and rounds the result to bf16, so it may
    # differ from the bf16 up-projection by the last bf16 bit.
    v = kvh[150, :, 128:].float()
    got = attn[0, 150:].float()
    assert torch.all((got - v).abs() <= v.abs() * 2.0 ** -7 + 1e-30)
    ref = oracle.attend_rows(x, range(x.T))
    assert_close(attn.float().cpu().numpy().reshape(ref.shape), ref, "single key")


# ---------------------------------------------------------------- whole block

@pytest.mark.parametrize("path", [DENSE, mla.MLA_PATH_AUTO])
@pytest.mark.parametrize("case", ["tiny_sparse", "ragged_sparse", "ragged_causal", "fp8_sparse"])
def test_prefill_matches_oracle(case, path):
    c = dict(ATTEND_CASES[case])
    x = synth.make_inputs(0, seed=41, **c)
    g = _dev(x)
    out = mla.mla_prefill(g["q"], g["kv_latent"], g["k_pe"], g["W_kvb"], g["W_o"], g.get("W_kvb_scale"),
                          g.get("W_o_scale"), topk_idx=g.get("topk_idx"), scale=x.scale, path=path)
    _no_device_error()
    rows = list(range(x.B * x.T))
    ref_attn, ref_out = oracle.prefill_rows(x, rows)
    assert_close(out.float().cpu().numpy().reshape(len(rows), 7168), ref_out, case)


def test_prefill_equals_attend_then_out_project():
    x = synth.make_inputs(0, B=1, T=256, H=4, topk=32, seed=42)
    g = _dev(x)
    out = mla.mla_prefill(g["q"], g["kv_latent"], g["k_pe"], g["W_kvb"], g["W_o"], topk_idx=g["topk_idx"],
                          scale=x.scale, path=DENSE)
    attn = _attend(x, g)
    out2 = mla.mla_out_project(attn, g["W_o"])
    _no_device_error()
    assert torch.equal(out.view(-1, 7168), out2)


def test_empty_problem_is_a_noop():
    x = synth.make_inputs(0, B=1, T=4, H=2, topk=2, seed=43)
    g = _dev(x)
    q0 = g["q"][:, :0].contiguous()
    attn = mla.mla_attend(q0, g["kv_latent"][:, :0].contiguous(), g["k_pe"][:, :0].contiguous(), g["W_kvb"],
                          topk_idx=g["topk_idx"][:, :0].contiguous(), scale=x.scale)
    assert attn.shape == (1, 0, 2, 128)
    _no_device_error()


def test_pipeline_over_host_batches_equals_prefill():
    # Three different host batches through the overlapped pipeline; every
    # output equals the synchronous mla_prefill of the same batch.
    xs = [synth.make_inputs(0, B=1, T=256, H=2, topk=24, seed=90 + i) for i in range(3)]
    w = _dev(xs[0])
    pipe = mla.PrefillPipeline(1, 256, 2, w["W_kvb"], w["W_o"], topk=24, scale=xs[0].scale)
    outs = []
    for x in xs:
        host = {k: getattr(x, k).pin_memory() for k in ("q", "kv_latent", "k_pe", "topk_idx")}
        o = torch.empty(1, 256, 7168, dtype=torch.bfloat16).pin_memory()
        pipe.submit(host, o)
        outs.append(o)
    pipe.synchronize()
    for x, o in zip(xs, outs):
        g = _dev(x)
        ref = mla.mla_prefill(g["q"], g["kv_latent"], g["k_pe"], w["W_kvb"], w["W_o"], topk_idx=g["topk_idx"],
                              scale=x.scale)
        assert torch.equal(o, ref.cpu())
    _no_device_error()
