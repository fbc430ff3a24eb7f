"""mla_attend_static: the attention entry point that allocates nothing.

It serves callers that cannot hand the library device memory (a plugin in a
host framework that owns every allocation through its own pool, or a path
that cannot afford cudaMalloc's implicit synchronisation): its scratch is a
file-scope device array of MLA_STATIC_SCRATCH_BYTES inside the library.
These tests call it through the C ABI and compare it with mla_attend (the
same computation with a caller-supplied workspace). The file is named so
that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
import sparse_head_latent_b200 as mla
from sparse_head_latent_b200 import build as cuda_build
from sparse_head_latent_b200.mla import MLA_STATIC_SCRATCH_BYTES, make_dims

MAX_ABS, REL_L2 = 2e-2, 5e-3  # the tolerance every GPU parity test uses


def _static_via_abi(lib, x, g, path=mla.MLA_PATH_AUTO, act=mla.MLA_ACT_BF16):
    """One mla_attend_static call through the C ABI; returns (status, attn)."""
    tk = g.get("topk_idx")
    dims = make_dims(x.B, x.T, x.H, 0 if tk is None else tk.shape[-1], x.fp8, path, act)
    attn = torch.full((x.B, x.T, x.H, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    sc = g.get("W_kvb_scale")
    rc = lib.mla_attend_static(ctypes.byref(dims), g["q"].data_ptr(), g["kv_latent"].data_ptr(),
                               g["k_pe"].data_ptr(), g["W_kvb"].data_ptr(), None if sc is None else sc.data_ptr(),
                               None if tk is None else tk.data_ptr(), ctypes.c_float(x.scale), attn.data_ptr(),
                               ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return rc, attn


def _close(got, ref):
    d = got.float().cpu().numpy().astype(np.float64) - ref.float().cpu().numpy().astype(np.float64)
    r = ref.float().cpu().numpy().astype(np.float64)
    assert np.isfinite(d).all()
    max_abs = float(np.abs(d).max())
    rel = float(np.linalg.norm(d) / np.linalg.norm(r))
    assert max_abs <= MAX_ABS and rel <= REL_L2, (max_abs, rel)


@pytest.mark.gpu
def test_static_scratch_entry_matches_workspace_entry_on_two_calls_in_a_row():
    lib = mla.load_library()
    # Different problems back to back: each call finds the previous call's
    # contents in the shared array and must not depend on them. The cases
    # place every scratch region in the array at least once: up-projected kv,
    # bitmap and block lists (block-dense), the per-row key lists, q_abs and
    # o_lat of the absorbed rows, the dequantised e4m3 W_kvb, and the
    # quantized latent of the e4m3-activation mode.
    A, D = mla.MLA_PATH_ABSORBED, mla.MLA_PATH_BLOCK_DENSE
    cases = [(synth.make_inputs(0, B=2, T=300, H=4, topk=40, seed=71), mla.MLA_PATH_AUTO, 0),
             (synth.make_inputs(0, B=1, T=1200, H=4, topk=40, seed=73), A, 0),
             (synth.make_inputs(0, B=1, T=200, H=2, topk=None, seed=72), D, 0),
             (synth.make_inputs(0, B=1, T=1200, H=4, topk=40, seed=73), A, 0),
             (synth.make_inputs(0, B=2, T=300, H=4, topk=40, seed=74, fp8=True), D, 0),
             (synth.make_inputs(0, B=1, T=300, H=4, topk=40, seed=75, fp8=True), D, mla.MLA_ACT_E4M3_DYNAMIC)]
    for x, path, act in cases:
        g = {k: v.cuda() for k, v in x.tensors().items()}
        rc, got = _static_via_abi(lib, x, g, path, act)
        assert rc == 0, mla.mla_status_str(rc)
        ref = mla.mla_attend(g["q"], g["kv_latent"], g["k_pe"], g["W_kvb"], g.get("W_kvb_scale"),
                             topk_idx=g.get("topk_idx"), scale=x.scale, path=path, act=act)
        assert mla.mla_device_status() == 0
        _close(got, ref)
        # the same kernels on the same inputs: bit for bit
        assert torch.equal(got, ref), (x.T, path, act)


@pytest.mark.gpu
def test_static_scratch_entry_matches_the_oracle():
    # The static entry against the fp64 oracle itself (every row, every
    # head) for a block-dense and an absorbed problem, bf16 and e4m3
    # weights, the e4m3 weights also with on-chip conversion (whose scratch
    # holds no dequantised copy).
    import oracle
    lib = mla.load_library()
    A, D = mla.MLA_PATH_ABSORBED, mla.MLA_PATH_BLOCK_DENSE
    cases = [(synth.make_inputs(0, B=1, T=260, H=4, topk=40, seed=76), D, False),
             (synth.make_inputs(0, B=1, T=700, H=4, topk=40, seed=77), A, False),
             (synth.make_inputs(0, B=1, T=260, H=4, topk=40, seed=78, fp8=True), D, False),
             (synth.make_inputs(0, B=1, T=260, H=4, topk=40, seed=78, fp8=True), D, True)]
    for x, path, onchip in cases:
        g = {k: v.cuda() for k, v in x.tensors().items()}
        mla.mla_set_e4m3_weight_conversion(onchip)
        try:
            rc, got = _static_via_abi(lib, x, g, path)
        finally:
            mla.mla_set_e4m3_weight_conversion(False)
        assert rc == 0, mla.mla_status_str(rc)
        assert mla.mla_device_status() == 0
        ref = oracle.attend_rows(x, list(range(x.B * x.T)))
        _close(got.view(ref.shape), torch.from_numpy(ref))


def test_static_scratch_entry_rejects_problems_beyond_its_scratch():
    # A host-side check that runs before any device work (no GPU needed).
    cuda_build.build()
    lib = mla.load_library()
    H, T = 128, 1024  # 1024 * 128 * 512 bytes of kv alone = 64 MiB > 32 MiB
    assert T * H * 512 > MLA_STATIC_SCRATCH_BYTES
    dims = make_dims(1, T, H, 0, False)
    rc = lib.mla_attend_static(ctypes.byref(dims), 16, 16, 16, 16, None, None, ctypes.c_float(0.07), 16, None)
    assert rc == 8
    assert "MLA_STATIC_SCRATCH_BYTES" in mla.mla_status_str(rc)
    dims = make_dims(1, 0, H, 0, False)
    assert lib.mla_attend_static(ctypes.byref(dims), None, None, None, None, None, None, ctypes.c_float(0.07),
                                 None, None) == 0
