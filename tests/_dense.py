"""Dense fp64 restatement of the attend block for tiny inputs (test helper).

It builds the full [T, T] selection as a boolean matrix and runs a dense
masked softmax with torch library routines, so it shares no loop structure
with the oracle's per-row key lists. Used only on inputs small enough that
the dense [B, H, T, T] logits fit comfortably in memory.
"""
import torch


def dequant(w, scale):
    """Stored weight -> float64 (bf16 directly; e4m3 codes times block scale)."""
    if scale is None:
        return w.to(torch.float64)
    codes = w.view(torch.float8_e4m3fn).to(torch.float64)
    s = scale.to(torch.float64).repeat_interleave(128, 0).repeat_interleave(128, 1)
    return codes * s


def fake_quant_e4m3(x):
    """Dynamic activation quantization restated with torch casts: per row, groups
    of 128 channels, s = amax / 448 in float32, codes = float8_e4m3fn(x / s);
    returns the float64 values code * s. x is float32 (or exactly convertible)."""
    xf = x.to(torch.float32)
    g = xf.reshape(*xf.shape[:-1], xf.shape[-1] // 128, 128)
    s = g.abs().amax(-1, keepdim=True) / 448.0
    safe = torch.where(s > 0, s, torch.ones_like(s))
    codes = (g / safe).to(torch.float8_e4m3fn)
    deq = codes.to(torch.float64) * s.to(torch.float64)
    return deq.reshape(x.shape)


def selection_matrix(B, T, topk_idx):
    """bool [B, T, T]: key t is selected for query s and t <= s."""
    allowed = torch.ones(T, T, dtype=torch.bool).tril()
    if topk_idx is None:
        return allowed.expand(B, T, T).clone()
    idx = topk_idx.to(torch.int64)
    valid = (idx >= 0) & (idx < T)
    chosen = torch.zeros(B, T, T + 1, dtype=torch.bool)
    # Out-of-range entries land in the extra column T and are dropped.
    chosen.scatter_(2, torch.where(valid, idx, torch.full_like(idx, T)), True)
    return chosen[:, :, :T] & allowed


def dense_block(x, topk_idx="inputs", act_e4m3=False):
    """(attn fp64 [B, T, H, 128], out fp64 [B, T, 7168]). With act_e4m3 the latent
    and the bf16-rounded attention output are fake-quantized before the projections."""
    B, T, H = x.B, x.T, x.H
    tk = x.topk_idx if isinstance(topk_idx, str) else topk_idx
    wk = dequant(x.W_kvb, x.W_kvb_scale)
    wo = dequant(x.W_o, x.W_o_scale)
    latent = x.kv_latent.to(torch.float64)
    if act_e4m3:
        latent = fake_quant_e4m3(x.kv_latent.to(torch.float32))
    up = torch.matmul(latent, wk.t()).reshape(B, T, H, 256)
    k_nope, v = up[..., :128], up[..., 128:]
    rope = x.k_pe.to(torch.float64).unsqueeze(2).expand(B, T, H, 64)
    keys = torch.cat([k_nope, rope], dim=-1)                      # [B, T, H, 192]
    qh = x.q.to(torch.float64).permute(0, 2, 1, 3)                # [B, H, T, 192]
    kh = keys.permute(0, 2, 1, 3)
    vh = v.permute(0, 2, 1, 3)
    logits = torch.matmul(qh, kh.transpose(-1, -2)) * x.scale     # [B, H, S, T]
    keep = selection_matrix(B, T, tk).unsqueeze(1)
    logits = logits.masked_fill(~keep, float("-inf"))
    probs = torch.softmax(logits, dim=-1)
    probs = torch.nan_to_num(probs, nan=0.0)                      # empty rows -> 0
    attn = torch.matmul(probs, vh).permute(0, 2, 1, 3).contiguous()  # [B, T, H, 128]
    a = attn.reshape(B, T, H * 128)
    if act_e4m3:
        a = fake_quant_e4m3(a.to(torch.bfloat16).to(torch.float32))
    out = torch.matmul(a, wo)
    return attn, out
