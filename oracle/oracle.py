"""ctypes front end of the C++ fp64 oracle (``mla_oracle.cpp``).

TEST INFRASTRUCTURE ONLY: called by the tests, the smoke check and the CPU
baseline of the benchmark, never by the product path. Inputs are the CPU
tensors of ``synth.MlaInputs`` (or any object with the same fields); the
oracle reads their exact stored bytes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mla_oracle.cpp")
_LIB = os.path.join(_HERE, "libmla_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into oracle/libmla_oracle.so (plain g++, -O2, no -ffast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-std=c++17", "-O2", "-fPIC", "-shared", "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


class _Problem(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int),
        ("d_nope", ctypes.c_int), ("d_rope", ctypes.c_int), ("d_v", ctypes.c_int),
        ("d_latent", ctypes.c_int), ("d_model", ctypes.c_int),
        ("topk", ctypes.c_int), ("w_fp8", ctypes.c_int),
        ("q", ctypes.c_void_p), ("kv_latent", ctypes.c_void_p), ("k_pe", ctypes.c_void_p),
        ("W_kvb", ctypes.c_void_p), ("W_kvb_scale", ctypes.c_void_p),
        ("W_o", ctypes.c_void_p), ("W_o_scale", ctypes.c_void_p),
        ("topk_idx", ctypes.c_void_p), ("scale", ctypes.c_double),
        ("act_e4m3", ctypes.c_int),
    ]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            # MLA_ORACLE_LIB points the tests' mutation check at a deliberately
            # altered copy of the oracle; normally the built library is used.
            lib = ctypes.CDLL(os.environ.get("MLA_ORACLE_LIB") or build())
            P = ctypes.POINTER(_Problem)
            i64p = ctypes.POINTER(ctypes.c_int64)
            i32p = ctypes.POINTER(ctypes.c_int32)
            dp = ctypes.POINTER(ctypes.c_double)
            lib.mlao_bf16_to_double.argtypes = [ctypes.c_uint16]
            lib.mlao_bf16_to_double.restype = ctypes.c_double
            lib.mlao_e4m3_to_double.argtypes = [ctypes.c_uint8]
            lib.mlao_e4m3_to_double.restype = ctypes.c_double
            lib.mlao_bf16_from_double.argtypes = [ctypes.c_double]
            lib.mlao_bf16_from_double.restype = ctypes.c_uint16
            lib.mlao_e4m3_from_float.argtypes = [ctypes.c_float]
            lib.mlao_e4m3_from_float.restype = ctypes.c_uint8
            lib.mlao_quantize_act.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                              ctypes.c_void_p]
            lib.mlao_quantize_act.restype = ctypes.c_int
            lib.mlao_upproject_rows.argtypes = [P, ctypes.c_int, i64p, dp]
            lib.mlao_attend_rows.argtypes = [P, ctypes.c_int, i64p, ctypes.c_int, i32p, dp]
            lib.mlao_project_rows.argtypes = [P, ctypes.c_int, dp, dp]
            lib.mlao_prefill_rows.argtypes = [P, ctypes.c_int, i64p, dp, dp]
            for f in ("mlao_upproject_rows", "mlao_attend_rows", "mlao_project_rows", "mlao_prefill_rows"):
                getattr(lib, f).restype = ctypes.c_int
            _lib = lib
    return _lib


def _cpu(t):
    if t is None:
        return None
    t = t.detach()
    if t.device.type != "cpu":
        t = t.cpu()
    return t.contiguous()


class _Bound:
    """Keeps the CPU tensors alive while the oracle reads them."""

    def __init__(self, x, d_nope=128, d_rope=64, d_v=128, d_latent=512, d_model=None, act_e4m3=False):
        self.keep = []

        def ptr(t):
            t = _cpu(t)
            if t is None:
                return None
            self.keep.append(t)
            return t.data_ptr()

        q = x.q
        H = x.H
        if d_model is None:
            d_model = int(x.W_o.shape[1])
        p = _Problem()
        p.B, p.T, p.H = int(x.B), int(x.T), int(H)
        p.d_nope, p.d_rope, p.d_v, p.d_latent, p.d_model = d_nope, d_rope, d_v, d_latent, d_model
        tk = x.topk_idx
        p.topk = 0 if tk is None else int(tk.shape[-1])
        p.w_fp8 = 1 if x.fp8 else 0
        p.q = ptr(q.view(torch.int16) if q.dtype == torch.bfloat16 else q)
        p.kv_latent = ptr(x.kv_latent.view(torch.int16))
        p.k_pe = ptr(x.k_pe.view(torch.int16))
        wk = x.W_kvb.view(torch.int16) if x.W_kvb.dtype == torch.bfloat16 else x.W_kvb
        wo = x.W_o.view(torch.int16) if x.W_o.dtype == torch.bfloat16 else x.W_o
        p.W_kvb = ptr(wk)
        p.W_kvb_scale = ptr(x.W_kvb_scale)
        p.W_o = ptr(wo)
        p.W_o_scale = ptr(x.W_o_scale)
        p.topk_idx = ptr(tk.to(torch.int32) if tk is not None else None)
        p.scale = float(x.scale)
        p.act_e4m3 = 1 if act_e4m3 else 0
        self.p = p
        self.H, self.d_v, self.d_model = H, d_v, d_model
        self.per_head = d_nope + d_v


def _rows_arr(rows):
    return np.ascontiguousarray(np.asarray(rows, dtype=np.int64))


def upproject_rows(x, rows, **dims) -> np.ndarray:
    """fp64 [n, H*(d_nope+d_v)]: latent rows times W_kvb (stored row order).

    Every entry point takes ``act_e4m3=True`` for dynamic FP8 activations: the
    latent and the attention output are quantized per row in groups of 128
    before W_kvb and W_o (see ``quantize_act``)."""
    lib = _load()
    bd = _Bound(x, **dims)
    r = _rows_arr(rows)
    out = np.zeros((len(r), bd.H * bd.per_head), dtype=np.float64)
    rc = lib.mlao_upproject_rows(ctypes.byref(bd.p), len(r),
                                 r.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                 out.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    assert rc == 0
    return out


def attend_rows(x, rows, heads=None, **dims) -> np.ndarray:
    """fp64 [n, len(heads), d_v] attention output of the given rows and heads."""
    lib = _load()
    bd = _Bound(x, **dims)
    r = _rows_arr(rows)
    if heads is None:
        hs, hp, nh = None, None, bd.H
    else:
        hs = np.ascontiguousarray(np.asarray(heads, dtype=np.int32))
        hp, nh = hs.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), len(hs)
    out = np.zeros((len(r), nh, bd.d_v), dtype=np.float64)
    rc = lib.mlao_attend_rows(ctypes.byref(bd.p), len(r),
                              r.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), nh, hp,
                              out.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    assert rc == 0
    return out


def project_rows(x, attn, **dims) -> np.ndarray:
    """fp64 [n, d_model] = attn [n, H*d_v] (fp64) times W_o."""
    lib = _load()
    bd = _Bound(x, **dims)
    a = np.ascontiguousarray(np.asarray(attn, dtype=np.float64)).reshape(-1, bd.H * bd.d_v)
    out = np.zeros((a.shape[0], bd.d_model), dtype=np.float64)
    rc = lib.mlao_project_rows(ctypes.byref(bd.p), a.shape[0],
                               a.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
                               out.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    assert rc == 0
    return out


def prefill_rows(x, rows, **dims):
    """(attn fp64 [n, H, d_v], out fp64 [n, d_model]) for the given rows."""
    lib = _load()
    bd = _Bound(x, **dims)
    r = _rows_arr(rows)
    attn = np.zeros((len(r), bd.H, bd.d_v), dtype=np.float64)
    out = np.zeros((len(r), bd.d_model), dtype=np.float64)
    rc = lib.mlao_prefill_rows(ctypes.byref(bd.p), len(r),
                               r.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                               attn.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
                               out.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    assert rc == 0
    return attn, out


def host_threads() -> int:
    """Threads the *_threaded helpers use by default (the host's cores, at most 32)."""
    return max(1, min(32, os.cpu_count() or 1))


def attend_rows_threaded(x, rows, heads=None, act_e4m3=False, n_threads=None) -> np.ndarray:
    """attend_rows with the heads spread over host threads.

    The oracle computes every head on its own (each call up-projects the keys
    its heads need), so a call's heads can be split into shards that run at
    once; ctypes releases the GIL while the C++ code runs. Each thread runs
    the same plain single-threaded function on its shard and the shards are
    put back in head order, so the result equals one call bit for bit."""
    hs = list(range(int(x.H))) if heads is None else list(heads)
    rows = list(rows)
    n = max(1, min(n_threads or host_threads(), len(hs)))
    shards = [hs[i::n] for i in range(n)]
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(n) as ex:
        parts = list(ex.map(lambda sh: attend_rows(x, rows, heads=sh, act_e4m3=act_e4m3), shards))
    out = np.zeros((len(rows), len(hs), 128), dtype=np.float64)
    for i in range(n):
        out[:, i::n] = parts[i]
    return out


def prefill_rows_threaded(x, rows, act_e4m3=False, n_threads=None):
    """prefill_rows with the attention's heads spread over host threads and
    the output projection run once on the assembled rows (equal to
    prefill_rows bit for bit)."""
    attn = attend_rows_threaded(x, rows, act_e4m3=act_e4m3, n_threads=n_threads)
    out = project_rows(x, attn.reshape(attn.shape[0], -1), act_e4m3=act_e4m3)
    return attn, out


def bf16_to_double(bits: int) -> float:
    return _load().mlao_bf16_to_double(int(bits) & 0xFFFF)


def e4m3_to_double(code: int) -> float:
    return _load().mlao_e4m3_to_double(int(code) & 0xFF)


def bf16_from_double(v: float) -> int:
    """bf16 bits of the value nearest to v (ties to even)."""
    return int(_load().mlao_bf16_from_double(float(v)))


def e4m3_from_float(v: float) -> int:
    """E4M3FN code nearest to the fp32 value v (ties to even), saturating at +-448."""
    return int(_load().mlao_e4m3_from_float(float(v)))


def quantize_act(x):
    """Dynamic activation quantization of x (float32 [rows, cols], cols % 128 == 0):
    (codes uint8 [rows, cols], scales float32 [rows, cols // 128]), s = amax / 448 per group."""
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    rows, cols = a.shape
    codes = np.zeros((rows, cols), dtype=np.uint8)
    scales = np.zeros((rows, cols // 128), dtype=np.float32)
    rc = _load().mlao_quantize_act(a.ctypes.data, rows, cols, codes.ctypes.data, scales.ctypes.data)
    assert rc == 0
    return codes, scales
