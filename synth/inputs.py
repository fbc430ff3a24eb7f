"""Seeded synthetic workloads for the sparse MLA prefill attend block.

Shapes follow the DeepSeek-V3.2-Exp "Sparse attention" page (prefill,
empty cache: q, k and v per head with 192 = 128 content + 64 rotary
dimensions, 128 value dimensions, output width 7168) and the Kimi K2
"Output projection" page (64 heads, 8,192 -> 7,168). The FP8 weight format
(e4m3, one scale per 128 x 128 block) is the one the Kimi K2 "Down
projection" page quotes from its quantization config.

Every tensor is drawn on the CPU from a torch.Generator seeded with
``(config seed << 8) | tensor id`` so that a given config always yields the
same bytes. Nothing here computes attention; the module only draws numbers,
rounds them to the storage type and lays them out.

Distributions (the workload recipe):
  * q, kv_latent, k_pe: N(0, 1), rounded to bf16.
  * W_kvb [H*256, 512]: N(0, 1/512); W_o [H*128, 7168]: N(0, 1/(H*128)).
    The second argument of N is the variance.
  * FP8 weights: per 128 x 128 block, s = u * absmax / 448 with
    u ~ U[0.5, 2]; code = e4m3_rne(clamp(W / s, -448, 448)).
  * topk_idx [B, T, k] (int32): for query s, n = min(k, s + 1) distinct keys
    from [0, s] -- s itself plus n - 1 uniform draws without replacement
    from [0, s - 1] -- then k - n padding keys s + 1, ..., s + k - n (all
    > s, so the causal mask removes them). Each row is stored in a random
    order.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

D_NOPE = 128
D_ROPE = 64
D_QK = D_NOPE + D_ROPE
D_V = 128
D_LATENT = 512
D_MODEL = 7168
# qk_head_dim ** -0.5 with qk_head_dim = 128 + 64 (DeepSeek-V3.2-Exp MLA init).
SOFTMAX_SCALE = float(D_QK) ** -0.5

# The five workloads. topk None means "top-k >= T": causal mask only.
CONFIGS = {
    0: dict(name="tiny_sparse", B=1, T=128, H=8, topk=32, fp8=False, seed=0),
    1: dict(name="v32_sparse_T4096", B=1, T=4096, H=128, topk=2048, fp8=False, seed=1),
    2: dict(name="k2_causal_T8192", B=1, T=8192, H=64, topk=None, fp8=False, seed=2),
    3: dict(name="long_sparse_T32768", B=1, T=32768, H=128, topk=2048, fp8=False, seed=3),
    4: dict(name="batched_fp8_B16", B=16, T=1024, H=128, topk=512, fp8=True, seed=4),
}

_CHUNK = 1 << 24

_TID_Q, _TID_LAT, _TID_KPE, _TID_WKVB, _TID_WO, _TID_TOPK, _TID_SKVB, _TID_SWO = range(1, 9)


def _gen(seed: int, tid: int) -> torch.Generator:
    g = torch.Generator()
    g.manual_seed((int(seed) << 8) | tid)
    return g


def _randn_f32(shape, g: torch.Generator, std: float = 1.0) -> torch.Tensor:
    n = 1
    for d in shape:
        n *= int(d)
    out = torch.empty(n, dtype=torch.float32)
    for lo in range(0, n, _CHUNK):
        hi = min(n, lo + _CHUNK)
        out[lo:hi] = torch.randn(hi - lo, generator=g, dtype=torch.float32)
    if std != 1.0:
        out.mul_(std)
    return out.view(*shape)


def _randn_bf16(shape, g: torch.Generator, std: float = 1.0) -> torch.Tensor:
    n = 1
    for d in shape:
        n *= int(d)
    out = torch.empty(n, dtype=torch.bfloat16)
    for lo in range(0, n, _CHUNK):
        hi = min(n, lo + _CHUNK)
        x = torch.randn(hi - lo, generator=g, dtype=torch.float32)
        if std != 1.0:
            x.mul_(std)
        out[lo:hi] = x.to(torch.bfloat16)
    return out.view(*shape)


def quantize_e4m3_block128(w: torch.Tensor, g: torch.Generator):
    """Block-scaled e4m3 storage of a float32 matrix [R, C] (R, C multiples of 128).

    Returns (codes uint8 [R, C], scales float32 [R/128, C/128]) with
    w ~= e4m3(codes) * scale[row/128, col/128].
    """
    R, C = w.shape
    assert R % 128 == 0 and C % 128 == 0
    blocks = w.view(R // 128, 128, C // 128, 128)
    absmax = blocks.abs().amax(dim=(1, 3))
    u = 0.5 + 1.5 * torch.rand(absmax.shape, generator=g, dtype=torch.float32)
    s = (u * absmax / 448.0).to(torch.float32)
    codes = torch.empty(R, C, dtype=torch.uint8)
    cv = codes.view(R // 128, 128, C // 128, 128)
    for rb in range(R // 128):
        x = (blocks[rb] / s[rb][None, :, None]).clamp_(-448.0, 448.0)
        cv[rb] = x.to(torch.float8_e4m3fn).view(torch.uint8)
    return codes, s.contiguous()


def make_topk(B: int, T: int, k: int, seed: int, rows_per_chunk: int = 256) -> torch.Tensor:
    """topk_idx int32 [B, T, k] by the selection rule in the module docstring.

    With k > T the rows hold every key of [0, T) and then the k - T
    positions T, T+1, ... (out of range, so they select nothing)."""
    assert k >= 1
    if k > T:
        base = make_topk(B, T, T, seed, rows_per_chunk)
        extra = torch.arange(T, k, dtype=torch.int32).expand(B, T, k - T)
        return torch.cat([base, extra], dim=-1).contiguous()
    g = _gen(seed, _TID_TOPK)
    out = torch.empty(B, T, k, dtype=torch.int32)
    t = torch.arange(T, dtype=torch.int64)
    pad_key = t.to(torch.float64) + 2.0  # ascending, distinct, above every draw
    for b in range(B):
        for s0 in range(0, T, rows_per_chunk):
            s1 = min(T, s0 + rows_per_chunk)
            s = torch.arange(s0, s1, dtype=torch.int64)[:, None]
            u = torch.rand(s1 - s0, T, generator=g, dtype=torch.float64)
            key = torch.where(t[None, :] < s, u, pad_key[None, :].expand(s1 - s0, T))
            key = torch.where(t[None, :] == s, torch.full_like(key, -1.0), key)
            idx = torch.topk(key, k, dim=1, largest=False, sorted=True).indices
            perm = torch.rand(s1 - s0, k, generator=g, dtype=torch.float32).argsort(dim=1)
            out[b, s0:s1] = idx.gather(1, perm).to(torch.int32)
    return out


@dataclasses.dataclass
class MlaInputs:
    B: int
    T: int
    H: int
    topk: Optional[int]            # None: causal mask only
    fp8: bool
    scale: float
    q: torch.Tensor                # bf16 [B, T, H, 192], nope then rope
    kv_latent: torch.Tensor        # bf16 [B, T, 512]
    k_pe: torch.Tensor             # bf16 [B, T, 64]
    W_kvb: torch.Tensor            # bf16 or uint8(e4m3) [H*256, 512]
    W_kvb_scale: Optional[torch.Tensor]  # f32 [2H, 4]
    W_o: torch.Tensor              # bf16 or uint8(e4m3) [H*128, 7168]
    W_o_scale: Optional[torch.Tensor]    # f32 [H, 56]
    topk_idx: Optional[torch.Tensor]     # int32 [B, T, k]
    name: str = ""

    def tensors(self):
        return {k: v for k, v in dataclasses.asdict(self).items() if isinstance(v, torch.Tensor)}


def make_inputs(cfg, *, T: Optional[int] = None, B: Optional[int] = None,
                H: Optional[int] = None, topk="cfg", seed: Optional[int] = None,
                fp8: Optional[bool] = None) -> MlaInputs:
    """Build one workload. ``cfg`` is a CONFIGS key or a dict with the same keys;
    keyword overrides give the small and ragged variants the tests use."""
    c = dict(CONFIGS[cfg]) if isinstance(cfg, int) else dict(cfg)
    if T is not None:
        c["T"] = T
    if B is not None:
        c["B"] = B
    if H is not None:
        c["H"] = H
    if topk != "cfg":
        c["topk"] = topk
    if seed is not None:
        c["seed"] = seed
    if fp8 is not None:
        c["fp8"] = fp8
    B_, T_, H_, k_, sd = c["B"], c["T"], c["H"], c["topk"], c["seed"]
    q = _randn_bf16((B_, T_, H_, D_QK), _gen(sd, _TID_Q))
    lat = _randn_bf16((B_, T_, D_LATENT), _gen(sd, _TID_LAT))
    kpe = _randn_bf16((B_, T_, D_ROPE), _gen(sd, _TID_KPE))
    std_kvb = (1.0 / D_LATENT) ** 0.5
    std_o = (1.0 / (H_ * D_V)) ** 0.5
    if c.get("fp8", False):
        wk, sk = quantize_e4m3_block128(
            _randn_f32((H_ * (D_NOPE + D_V), D_LATENT), _gen(sd, _TID_WKVB), std_kvb),
            _gen(sd, _TID_SKVB))
        wo, so = quantize_e4m3_block128(
            _randn_f32((H_ * D_V, D_MODEL), _gen(sd, _TID_WO), std_o), _gen(sd, _TID_SWO))
    else:
        wk = _randn_bf16((H_ * (D_NOPE + D_V), D_LATENT), _gen(sd, _TID_WKVB), std_kvb)
        wo = _randn_bf16((H_ * D_V, D_MODEL), _gen(sd, _TID_WO), std_o)
        sk = so = None
    tk = None if k_ is None else make_topk(B_, T_, int(k_), sd)
    return MlaInputs(B=B_, T=T_, H=H_, topk=k_, fp8=bool(c.get("fp8", False)),
                     scale=SOFTMAX_SCALE, q=q, kv_latent=lat, k_pe=kpe,
                     W_kvb=wk, W_kvb_scale=sk, W_o=wo, W_o_scale=so, topk_idx=tk,
                     name=c.get("name", ""))


@dataclasses.dataclass
class DecodeInputs:
    B: int
    T: int                         # cache length including the new position (s = T - 1)
    H: int
    topk: Optional[int]
    fp8: bool
    scale: float
    q: torch.Tensor                # bf16 [B, H, 192] of the new position
    kv_latent: torch.Tensor        # bf16 [B, T, 512] latent cache
    k_pe: torch.Tensor             # bf16 [B, T, 64]
    W_kvb: torch.Tensor
    W_kvb_scale: Optional[torch.Tensor]
    W_o: torch.Tensor
    W_o_scale: Optional[torch.Tensor]
    topk_idx: Optional[torch.Tensor]     # int32 [B, k]

    def tensors(self):
        return {k: v for k, v in dataclasses.asdict(self).items() if isinstance(v, torch.Tensor)}


def make_decode_inputs(B: int, T: int, H: int, topk: Optional[int], seed: int, fp8: bool = False) -> DecodeInputs:
    """One new position per sequence and its cache, with the distributions of
    make_inputs (without the [B, T, H, 192] queries of the whole prefill).
    The selection of the new query s = T - 1 follows the same rule: s itself
    plus min(k, T) - 1 distinct positions of [0, s), in a shuffled order."""
    g = lambda tid: _gen(seed, tid)  # noqa: E731
    q = _randn_bf16((B, H, D_QK), g(_TID_Q))
    lat = _randn_bf16((B, T, D_LATENT), g(_TID_LAT))
    kpe = _randn_bf16((B, T, D_ROPE), g(_TID_KPE))
    std_kvb = (1.0 / D_LATENT) ** 0.5
    std_o = (1.0 / (H * D_V)) ** 0.5
    if fp8:
        wk, sk = quantize_e4m3_block128(_randn_f32((H * (D_NOPE + D_V), D_LATENT), g(_TID_WKVB), std_kvb),
                                        g(_TID_SKVB))
        wo, so = quantize_e4m3_block128(_randn_f32((H * D_V, D_MODEL), g(_TID_WO), std_o), g(_TID_SWO))
    else:
        wk = _randn_bf16((H * (D_NOPE + D_V), D_LATENT), g(_TID_WKVB), std_kvb)
        wo = _randn_bf16((H * D_V, D_MODEL), g(_TID_WO), std_o)
        sk = so = None
    tk = decode_topk(B, T, topk, seed) if topk is not None else None
    return DecodeInputs(B=B, T=T, H=H, topk=topk, fp8=fp8, scale=SOFTMAX_SCALE, q=q, kv_latent=lat, k_pe=kpe,
                        W_kvb=wk, W_kvb_scale=sk, W_o=wo, W_o_scale=so, topk_idx=tk)


def decode_topk(B: int, T: int, topk: int, seed: int) -> torch.Tensor:
    """The selection of make_decode_inputs (same seed, same bytes): per
    sequence, s = T - 1 plus min(k, T) - 1 distinct positions of [0, s) in a
    shuffled order, padded with out-of-range fillers when k > T. int32 [B, k]."""
    gt = _gen(seed, _TID_TOPK)
    n = min(int(topk), T)
    rows = []
    for _ in range(B):
        others = torch.randperm(T - 1, generator=gt)[: n - 1] if n > 1 else torch.empty(0, dtype=torch.int64)
        sel = torch.cat([torch.tensor([T - 1]), others])
        sel = sel[torch.randperm(n, generator=gt)]
        if int(topk) > n:  # more entries than positions: out-of-range fillers select nothing
            sel = torch.cat([sel, torch.arange(T, T + int(topk) - n)])
        rows.append(sel)
    return torch.stack(rows).to(torch.int32).contiguous()


def sample_rows(B: int, T: int, k: Optional[int], n_random: int, seed: int,
                batches=None) -> list:
    """Query rows (flattened b*T + s) for sampled parity: the sequence ends,
    the rows around the top-k saturation point, the edges of the first and
    last 128-row tiles, and seeded random rows."""
    g = torch.Generator()
    g.manual_seed(0x5EED0000 + int(seed))
    kk = T if k is None else int(k)
    fixed = {0, 1, kk - 2, kk - 1, kk, T - 1, 127, 128, T - 128, T - 129}
    if batches is None:
        batches = sorted({0, B - 1})
    rows = set()
    for b in batches:
        for s in fixed:
            if 0 <= s < T:
                rows.add(b * T + s)
        for s in torch.randint(0, T, (n_random,), generator=g).tolist():
            rows.add(b * T + int(s))
    return sorted(rows)
