"""Pins of the fp64 oracle to facts outside itself (CPU only).

Each test ties the oracle to something the pages print, to a closed form,
to an invariant of the method, or to a library routine on a special case:
  * parameter counts printed on the pages fix the weight shapes;
  * e4m3 / bf16 decoding equals torch's float8_e4m3fn / bfloat16 casts;
  * the up-projection and W_o steps equal fp64 torch.matmul;
  * the whole block equals a dense boolean-mask restatement on tiny inputs;
  * top-k >= T (or no top-k) equals causal scaled_dot_product_attention;
  * a single selected key returns that key's value vector exactly;
  * q = 0 returns the mean of the selected value vectors;
  * the order of top-k entries and duplicate entries change nothing;
  * out-of-range top-k entries select nothing;
  * dynamic FP8 activations: the e4m3 encoder returns the nearest code (brute
    force over the format's table, ties to even, saturating at 448) and agrees
    with torch's float8_e4m3fn cast; the group scale is amax / 448 and the
    largest element maps to +-448; quantization commutes with powers of two;
    the quantized projections equal fp64 matmuls of the dequantized rows and
    the whole block equals the dense restatement with torch's casts.
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import synth
from tests._dense import dense_block, dequant, fake_quant_e4m3

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split(None, 2)
            vals[parts[0]] = parts[1]
    return vals


def _tiny(B=1, T=40, H=3, topk=12, seed=7, fp8=False):
    return synth.make_inputs(0, B=B, T=T, H=H, topk=topk, seed=seed, fp8=fp8)


def _all_rows(x):
    return list(range(x.B * x.T))


def _rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.max(np.abs(a - b)) / max(1e-300, float(np.max(np.abs(b)))))


# ---------------------------------------------------------------- printed values

def test_param_counts_printed_on_pages():
    g = {k: int(v) for k, v in _golden("param_counts.txt").items()}
    D, dv = synth.D_MODEL, synth.D_V
    # W_o is [H * d_v, d_model]: 128 heads (V3.2) and 64 heads (K2).
    assert 128 * dv * D == g["wo_v32"] == g["attend_v32"]
    assert 128 * dv * D * 58 == g["wo_v32_blocks"]
    assert 64 * dv * D == g["wo_k2"]
    assert 64 * dv * D * 60 == g["wo_k2_blocks"]
    # Query compression on the K2 page fixes qk_head_dim = d_nope + d_rope = 192
    # for 64 heads (1,536 x 12,288 = 1,536 x 64 * 192).
    q_lora = 1536
    assert D * q_lora == g["qdown_k2"]
    assert D * q_lora + q_lora == g["qcomp_k2"]
    assert D * q_lora + q_lora * 64 * (synth.D_NOPE + synth.D_ROPE) == g["qlowrank_k2"]
    assert D * 64 * (synth.D_NOPE + synth.D_ROPE) == g["qdense_k2"]


def test_weight_shapes_of_inputs_match_counts():
    g = {k: int(v) for k, v in _golden("param_counts.txt").items()}
    x = synth.make_inputs(0, T=8, H=128, topk=4)
    assert x.W_o.numel() == g["wo_v32"]
    assert tuple(x.W_kvb.shape) == (128 * (synth.D_NOPE + synth.D_V), synth.D_LATENT)
    x = synth.make_inputs(0, T=8, H=64, topk=None)
    assert x.W_o.numel() == g["wo_k2"]


def test_softmax_scale_is_qk_head_dim_rsqrt():
    # softmax_scale = qk_head_dim ** -0.5 with qk_head_dim = 128 + 64.
    assert synth.SOFTMAX_SCALE == (128 + 64) ** -0.5
    assert abs(synth.SOFTMAX_SCALE - 0.07216878364870322) < 1e-17


def test_fp8_format_fixture():
    g = _golden("fp8_format.txt")
    assert g["fmt"] == "e4m3"
    assert int(g["weight_block_rows"]) == 128 and int(g["weight_block_cols"]) == 128
    x = _tiny(H=2, fp8=True)
    assert x.W_kvb.dtype == torch.uint8
    assert tuple(x.W_kvb_scale.shape) == (2 * 256 // 128, 512 // 128)
    assert tuple(x.W_o_scale.shape) == (2 * 128 // 128, 7168 // 128)


# ---------------------------------------------------------------- decoding

def test_e4m3_decode_all_codes_match_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = np.array([oracle.e4m3_to_double(c) for c in range(256)])
    nan_ref = np.isnan(ref)
    assert np.array_equal(nan_ref, np.isnan(mine))
    assert np.array_equal(ref[~nan_ref], mine[~nan_ref])
    # Spot values of the format: max normal, smallest subnormal, smallest normal.
    assert oracle.e4m3_to_double(0x7E) == 448.0
    assert oracle.e4m3_to_double(0x01) == 2.0 ** -9
    assert oracle.e4m3_to_double(0x08) == 2.0 ** -6
    assert oracle.e4m3_to_double(0xB8) == -1.0


def test_bf16_decode_matches_torch():
    g = torch.Generator().manual_seed(3)
    bits = torch.randint(0, 1 << 16, (4096,), generator=g, dtype=torch.int32)
    bits = bits[((bits >> 7) & 0xFF) != 0xFF]  # finite values only
    ref = bits.to(torch.int16).view(torch.bfloat16).to(torch.float64).numpy()
    mine = np.array([oracle.bf16_to_double(int(b)) for b in bits])
    assert np.array_equal(ref, mine)


# ---------------------------------------------------------------- GEMM steps

@pytest.mark.parametrize("fp8", [False, True])
def test_upprojection_equals_fp64_matmul(fp8):
    x = _tiny(B=2, T=20, H=2, fp8=fp8)
    rows = [0, 5, 19, 20, 33, 39]
    got = oracle.upproject_rows(x, rows)
    lat = x.kv_latent.reshape(-1, 512).to(torch.float64)[rows]
    ref = (lat @ dequant(x.W_kvb, x.W_kvb_scale).t()).numpy()
    assert _rel(got, ref) < 1e-13


@pytest.mark.parametrize("fp8", [False, True])
def test_output_projection_equals_fp64_matmul(fp8):
    x = _tiny(H=2, fp8=fp8)
    g = torch.Generator().manual_seed(11)
    attn = torch.randn(5, 2 * 128, generator=g, dtype=torch.float64)
    got = oracle.project_rows(x, attn.numpy())
    ref = (attn @ dequant(x.W_o, x.W_o_scale)).numpy()
    assert _rel(got, ref) < 1e-13


# ---------------------------------------------------------------- whole block

def _with_duplicates(tk, seed=5):
    """Overwrite a third of each row with copies of other entries of the row."""
    g = torch.Generator().manual_seed(seed)
    tk = tk.clone()
    B, T, k = tk.shape
    src = torch.randint(0, k, (B, T, k // 3), generator=g)
    dst = torch.randint(0, k, (B, T, k // 3), generator=g)
    tk.scatter_(2, dst, tk.gather(2, src))
    return tk


@pytest.mark.parametrize("fp8", [False, True])
def test_block_equals_dense_masked_restatement(fp8):
    x = _tiny(B=2, T=48, H=3, topk=12, fp8=fp8)
    x.topk_idx = _with_duplicates(x.topk_idx)
    attn, out = oracle.prefill_rows(x, _all_rows(x))
    ref_attn, ref_out = dense_block(x)
    assert _rel(attn, ref_attn.reshape(-1, 3, 128).numpy()) < 1e-12
    assert _rel(out, ref_out.reshape(-1, 7168).numpy()) < 1e-12


def test_dense_restatement_detects_a_changed_mask():
    # Guard on the guard: dropping one selected key changes the dense result.
    x = _tiny(T=24, H=2, topk=6)
    a0, _ = dense_block(x)
    tk = x.topk_idx.clone()
    s = 20
    tk[0, s] = tk[0, s, 0]  # keep only one distinct key for row s
    a1, _ = dense_block(x, topk_idx=tk)
    assert (a0[0, s] - a1[0, s]).abs().max() > 1e-3


def test_topk_covering_all_keys_equals_causal_sdpa():
    T, H = 36, 2
    x_none = _tiny(T=T, H=H, topk=None)
    attn_none = oracle.attend_rows(x_none, _all_rows(x_none))
    x_all = _tiny(T=T, H=H, topk=T)  # every key in [0, T) listed for every row
    attn_all = oracle.attend_rows(x_all, _all_rows(x_all))
    assert np.array_equal(attn_none, attn_all)
    # Library routine: causal scaled dot-product attention in fp64.
    up = oracle.upproject_rows(x_none, _all_rows(x_none)).reshape(T, H, 256)
    k = np.concatenate([up[..., :128],
                        np.broadcast_to(x_none.k_pe.to(torch.float64).numpy()[0][:, None, :], (T, H, 64))], -1)
    q = x_none.q.to(torch.float64)[0].permute(1, 0, 2)
    kh = torch.from_numpy(np.ascontiguousarray(k)).permute(1, 0, 2)
    vh = torch.from_numpy(np.ascontiguousarray(up[..., 128:])).permute(1, 0, 2)
    ref = F.scaled_dot_product_attention(q, kh, vh, is_causal=True, scale=x_none.scale)
    assert _rel(attn_none, ref.permute(1, 0, 2).numpy()) < 1e-12


def test_single_selected_key_returns_its_value_exactly():
    T, H, t0 = 30, 3, 9
    x = _tiny(T=T, H=H, topk=5)
    x.topk_idx = torch.full_like(x.topk_idx, t0)
    attn = oracle.attend_rows(x, _all_rows(x))
    v = oracle.upproject_rows(x, [t0]).reshape(H, 256)[:, 128:]
    for s in range(T):
        if s >= t0:
            assert np.array_equal(attn[s], v), s
        else:
            assert not attn[s].any(), s  # t0 > s: nothing survives -> 0


def test_zero_query_gives_mean_of_selected_values():
    x = _tiny(T=34, H=2, topk=7)
    x.q = torch.zeros_like(x.q)
    attn = oracle.attend_rows(x, _all_rows(x))
    up = oracle.upproject_rows(x, _all_rows(x)).reshape(x.T, 2, 256)
    tk = x.topk_idx[0].numpy()
    for s in range(x.T):
        keys = sorted({int(t) for t in tk[s] if 0 <= t <= s})
        ref = up[keys][:, :, 128:].mean(axis=0)
        assert _rel(attn[s], ref) < 1e-13


def test_topk_order_and_duplicates_do_not_matter():
    x = _tiny(B=2, T=44, H=2, topk=10)
    base = oracle.attend_rows(x, _all_rows(x))
    g = torch.Generator().manual_seed(9)
    perm = torch.rand(x.topk_idx.shape, generator=g).argsort(-1)
    x.topk_idx = x.topk_idx.gather(-1, perm)
    assert np.array_equal(base, oracle.attend_rows(x, _all_rows(x)))
    x.topk_idx = torch.cat([x.topk_idx, x.topk_idx.flip(-1)], dim=-1)  # every key twice
    assert np.array_equal(base, oracle.attend_rows(x, _all_rows(x)))


def test_out_of_range_entries_select_nothing():
    x = _tiny(T=32, H=2, topk=8)
    base = oracle.attend_rows(x, _all_rows(x))
    tk = x.topk_idx.clone()
    # Entries above s never survive the causal mask; replacing them with
    # out-of-range values must change nothing.
    s_idx = torch.arange(x.T)[None, :, None]
    bad = torch.tensor([-1, -7, x.T, x.T + 100], dtype=torch.int32)
    fill = bad[torch.arange(tk.numel()).reshape(tk.shape) % 4]
    x.topk_idx = torch.where(tk > s_idx, fill, tk)
    assert np.array_equal(base, oracle.attend_rows(x, _all_rows(x)))
    # Replacing a contributing entry by -1 removes exactly that key.
    tk2 = x.topk_idx.clone()
    tk2[0, 31, :] = torch.where(tk2[0, 31] == 31, torch.tensor(-1, dtype=torch.int32), tk2[0, 31])
    x.topk_idx = tk2
    got = oracle.attend_rows(x, [31])
    ref, _ = dense_block(x)
    assert _rel(got[0], ref[0, 31].numpy()) < 1e-12


def test_empty_selection_gives_zero():
    x = _tiny(T=16, H=2, topk=4)
    x.topk_idx = torch.full_like(x.topk_idx, -1)
    attn, out = oracle.prefill_rows(x, _all_rows(x))
    assert not attn.any() and not out.any()


def test_softmax_weights_are_normalised():
    # With identical value vectors the output must equal that vector
    # whatever the scores are (weights sum to one).
    x = _tiny(T=26, H=2, topk=9)
    x.kv_latent = x.kv_latent[:, :1].expand_as(x.kv_latent).contiguous()
    attn = oracle.attend_rows(x, _all_rows(x))
    v = oracle.upproject_rows(x, [0]).reshape(2, 256)[:, 128:]
    for s in range(x.T):
        assert _rel(attn[s], v) < 1e-13


def test_scores_scale_enters_linearly():
    # Doubling the scale equals doubling q (z = scale * <q, k>).
    x = _tiny(T=20, H=2, topk=6)
    x.q = (x.q.float() * 0.5).to(torch.bfloat16)  # exact: halves the exponent
    x.scale = 2.0 * synth.SOFTMAX_SCALE
    a1 = oracle.attend_rows(x, _all_rows(x))
    x.q = (x.q.float() * 2.0).to(torch.bfloat16)
    x.scale = synth.SOFTMAX_SCALE
    a2 = oracle.attend_rows(x, _all_rows(x))
    assert _rel(a1, a2) < 1e-14


# ---------------------------------------------------------------- dynamic FP8 activations

def _e4m3_values():
    return torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _e4m3_probe_values(seed=21):
    """float32 values in [-448, 448]: random magnitudes over the whole range
    plus every midpoint between neighbouring codes (the ties)."""
    vals = _e4m3_values()
    pos = np.unique(vals[(vals >= 0) & ~np.isnan(vals)])
    mids = (pos[1:] + pos[:-1]) / 2
    rng = np.random.default_rng(seed)
    rand = rng.standard_normal(4000) * 10.0 ** rng.uniform(-4, 2.6, 4000)
    xs = np.concatenate([rand, mids, -mids, pos, -pos, mids * (1 + 2.0 ** -20), mids * (1 - 2.0 ** -20)])
    xs = xs.astype(np.float32)
    return xs[np.abs(xs) <= 448]


def test_e4m3_encode_is_the_nearest_code():
    vals = _e4m3_values()
    finite = ~np.isnan(vals)
    for x in _e4m3_probe_values():
        c = oracle.e4m3_from_float(float(x))
        sign = 0x80 if np.signbit(x) else 0
        cand = np.array([k for k in range(256) if finite[k] and (k & 0x80) == sign])
        d = np.abs(vals[cand] - np.float64(x))
        best = cand[d == d.min()]
        if len(best) > 1:  # a tie: the code with an even mantissa
            best = best[(best & 1) == 0]
        assert c == int(best[0]), (x, c, best)


def test_e4m3_encode_matches_torch_cast():
    xs = _e4m3_probe_values(seed=22)
    ref = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    mine = np.array([oracle.e4m3_from_float(float(x)) for x in xs], dtype=np.uint8)
    assert np.array_equal(mine, ref)


def test_e4m3_encode_saturates_at_448():
    for v in (448.0, 448.5, 463.9, 464.0, 480.0, 1.0e6, 3.0e38):
        assert oracle.e4m3_from_float(v) == 0x7E
        assert oracle.e4m3_from_float(-v) == 0xFE
    assert oracle.e4m3_from_float(2.0 ** -10) == 0x00       # tie between 0 and 2^-9
    assert oracle.e4m3_from_float(3 * 2.0 ** -10) == 0x02   # tie between 2^-9 and 2^-8


def test_bf16_rounding_is_nearest_and_matches_torch():
    rng = np.random.default_rng(23)
    f32 = (rng.standard_normal(3000) * 10.0 ** rng.uniform(-30, 30, 3000)).astype(np.float32)
    ref = torch.from_numpy(f32).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    mine = np.array([oracle.bf16_from_double(float(v)) for v in f32], dtype=np.uint16)
    assert np.array_equal(mine, ref)
    for v in rng.standard_normal(500) * 10.0 ** rng.uniform(-5, 5, 500):
        b = oracle.bf16_from_double(float(v))
        got = oracle.bf16_to_double(b)
        lo, hi = oracle.bf16_to_double(b - 1), oracle.bf16_to_double(b + 1)
        assert abs(got - v) <= abs(lo - v) and abs(got - v) <= abs(hi - v)


def _act_rows(seed=24, rows=6, cols=384):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols)) * 10.0 ** rng.uniform(-3, 3, (rows, 1))
    x = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    x[1, 128:256] = 0.0          # an all-zero group
    x[2, :128] = 0.0
    x[2, 17] = -3.5              # a group with a single non-zero element
    return x


def test_act_quantization_closed_forms():
    x = _act_rows()
    codes, s = oracle.quantize_act(x)
    g = x.reshape(x.shape[0], -1, 128)
    amax = np.abs(g).max(-1)
    assert np.array_equal(s, amax / np.float32(448.0))
    vals = _e4m3_values()
    deq = vals[codes].reshape(g.shape) * s[..., None].astype(np.float64)
    cg = codes.reshape(g.shape)
    for r in range(g.shape[0]):
        for j in range(g.shape[1]):
            if amax[r, j] == 0:
                assert s[r, j] == 0 and not cg[r, j].any()
                continue
            i = int(np.argmax(np.abs(g[r, j])))
            assert cg[r, j, i] in (0x7E, 0xFE)
            y = np.abs(g[r, j].astype(np.float64)) / np.float64(s[r, j])
            e = np.floor(np.log2(np.maximum(y, 2.0 ** -30)))
            half_ulp = 2.0 ** (np.maximum(e, -6) - 4)
            bound = (half_ulp + y * 2.0 ** -23) * np.float64(s[r, j])
            assert np.all(np.abs(deq[r, j] - g[r, j]) <= bound)
    assert deq[2, 0, 17] == -3.5


def test_act_quantization_commutes_with_powers_of_two():
    x = _act_rows(seed=25)
    c0, s0 = oracle.quantize_act(x)
    c1, s1 = oracle.quantize_act(x * np.float32(2.0 ** 7))
    assert np.array_equal(c0, c1) and np.array_equal(s1, s0 * np.float32(2.0 ** 7))


def test_act_quantization_matches_torch_casts():
    x = _act_rows(seed=26, rows=9)
    codes, s = oracle.quantize_act(x)
    deq = _e4m3_values()[codes] * np.repeat(s.astype(np.float64), 128, axis=1)
    ref = fake_quant_e4m3(torch.from_numpy(x)).numpy()
    assert np.array_equal(deq, ref)


@pytest.mark.parametrize("fp8", [False, True])
def test_act_e4m3_upprojection_equals_matmul_of_dequantized_latent(fp8):
    x = _tiny(B=2, T=20, H=2, fp8=fp8)
    rows = [0, 7, 19, 20, 39]
    got = oracle.upproject_rows(x, rows, act_e4m3=True)
    lat = x.kv_latent.reshape(-1, 512).to(torch.float32)[rows].numpy()
    codes, s = oracle.quantize_act(lat)
    deq = torch.from_numpy(_e4m3_values()[codes] * np.repeat(s.astype(np.float64), 128, axis=1))
    ref = (deq @ dequant(x.W_kvb, x.W_kvb_scale).t()).numpy()
    assert _rel(got, ref) < 1e-13
    assert _rel(got, oracle.upproject_rows(x, rows)) > 1e-4   # the quantization is applied


@pytest.mark.parametrize("fp8", [False, True])
def test_act_e4m3_projection_equals_matmul_of_dequantized_rows(fp8):
    x = _tiny(H=2, fp8=fp8)
    g = torch.Generator().manual_seed(12)
    attn = torch.randn(5, 2 * 128, generator=g, dtype=torch.float64)
    got = oracle.project_rows(x, attn.numpy(), act_e4m3=True)
    rounded = attn.to(torch.bfloat16).to(torch.float32).numpy()
    codes, s = oracle.quantize_act(rounded)
    deq = torch.from_numpy(_e4m3_values()[codes] * np.repeat(s.astype(np.float64), 128, axis=1))
    ref = (deq @ dequant(x.W_o, x.W_o_scale)).numpy()
    assert _rel(got, ref) < 1e-13


@pytest.mark.parametrize("fp8", [False, True])
def test_act_e4m3_block_equals_dense_restatement(fp8):
    x = _tiny(B=2, T=40, H=2, topk=10, fp8=fp8)
    attn, out = oracle.prefill_rows(x, _all_rows(x), act_e4m3=True)
    ref_attn, ref_out = dense_block(x, act_e4m3=True)
    assert _rel(attn, ref_attn.reshape(-1, 2, 128).numpy()) < 1e-12
    assert _rel(out, ref_out.reshape(-1, 7168).numpy()) < 1e-12
    _, out_bf16 = oracle.prefill_rows(x, _all_rows(x))
    d = np.linalg.norm(out - out_bf16) / np.linalg.norm(out_bf16)
    assert 1e-3 < d < 0.1   # e4m3 activations move the output by about a percent


def test_threaded_oracle_equals_the_plain_calls_bit_for_bit():
    # The tests and the benchmark's CPU leg spread the oracle's heads over
    # host threads; the shards must reassemble to exactly the plain result.
    for cfg, fp8, act in ((0, False, False), (4, True, True)):
        x = synth.make_inputs(cfg, B=2, T=200, H=5, topk=24, seed=91, fp8=fp8)
        rows = [0, 17, 199, 200, 333, 399]
        a1, o1 = oracle.prefill_rows(x, rows, act_e4m3=act)
        a2, o2 = oracle.prefill_rows_threaded(x, rows, act_e4m3=act, n_threads=3)
        assert np.array_equal(a1, a2) and np.array_equal(o1, o2)
        h = [4, 0, 2]
        assert np.array_equal(oracle.attend_rows(x, rows, heads=h), oracle.attend_rows_threaded(x, rows, heads=h,
                                                                                              n_threads=2))
