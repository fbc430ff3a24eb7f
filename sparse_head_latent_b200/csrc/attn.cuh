// attn.cuh -- fused sparse-causal MLA attention for sm_100a (tcgen05 + TMA).
//
// For one batch b, one head h and one tile of 128 queries s, over the key
// blocks (128 keys each) in which some query of the tile selected a key
// (DeepSeek-V3.2-Exp "Sparse attention", prefill):
//   S   = q_h . [k_nope_h | k_pe]^T              (UMMA, K = 192, S in tensor memory)
//   S   = -inf where bit(s, t) = 0                (top-k + causal selection)
//   m,l = running max / sum of exp2(S*scale*log2e - m) per query row (fp32)
//   O  += P . v_h                                 (UMMA, P f16 in tensor memory, O in tensor memory)
//   l  += P . 1                                   (UMMA against a constant block of ones)
//   attn[b, s, h, :] = O / l                      (bf16)
// P is exp2 of the scaled scores, computed two at a time in f16
// (ex2.approx.f16x2); v is stored as f16 by the up-projection, so PV is an
// f16 x f16 UMMA with fp32 accumulation and the row sums come from the
// tensor core, never from the softmax warps.
// Neither the [T, T] scores nor a float mask is ever materialised: the
// selection arrives as one bit per causal (query, key) pair.
//
// CTA = 192 threads:
//   warp 0      TMA producer: Q once; K (k_nope from the up-projected kv
//               plus the shared k_pe) and V into 2-deep rings
//   warp 1      tensor-memory allocator and UMMA issuer; issues QK^T of the
//               next block before PV of the current one so the tensor core
//               works while the softmax runs
//   warps 2..5  softmax: one query row per thread (tensor-memory lane)
// Tensor memory: S0 cols [0,128), S1 [128,256), O [256,384), l [384,400),
// P [416,480) (P: 128 f16 per row packed in 64 columns; the PV UMMA reads it
// as its A operand, so P never touches shared memory).
#pragma once

#include "prepass.cuh"
#include "ptx.cuh"

namespace mla {

struct AttnParams {
  int B, T, H, nq;
  int hgroup;                   // heads per scheduling group (divides H)
  float scale_log2;             // softmax scale * log2(e)
  const uint4* bitmap;          // selection bitmap, NULL = causal mask only
  const int32_t* blocks;        // active key blocks per tile (with bitmap)
  __nv_bfloat16* attn;          // [B, T, H, 128]
  int* err;
};

struct AttnSmem {
  static constexpr int Q = 0;              // 3 x [128 x 64] bf16, 128B-swizzled
  static constexpr int K0 = 49152;         // stage 0: k_nope 0-63, 64-127, k_pe
  static constexpr int K1 = 98304;         // stage 1
  static constexpr int V0 = 147456;        // stage 0: 2 x [128 keys x 64 dv]
  static constexpr int V1 = 180224;        // stage 1
  static constexpr int ONES = 212992;      // [16 x 128] f16 ones (row-sum operand)
  static constexpr int BARS = 217088;
  static constexpr int NUM_BARS = 16;
  static constexpr int BLIST = BARS + 256;  // active key-block ids of this tile (<= MLA_MAX_T / 128)
  static constexpr int BYTES = 1024 + BLIST + (MLA_MAX_T / 128) * 4;
};

// Tensor-memory columns.
constexpr uint32_t kTmemS0 = 0, kTmemO = 256, kTmemL = 384, kTmemP = 416;

// Barrier slots.
enum : int {
  kBarQFull = 0, kBarKFull0 = 1, kBarKEmpty0 = 3, kBarVFull0 = 5, kBarVEmpty0 = 7, kBarSFull0 = 9,
  kBarSFree0 = 11, kBarPFull = 13, kBarPvDone = 14, kBarDrain = 15
};

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// (x0, x1) <- (x0 * c + b, x1 * c + b) as one packed f32x2 FMA.
__device__ __forceinline__ void fma2_scalar(float& x0, float& x1, float c, float b) {
  asm("{\n\t.reg .b64 t, u, v;\n\t"
      "mov.b64 t, {%0, %1};\n\t"
      "mov.b64 u, {%2, %2};\n\t"
      "mov.b64 v, {%3, %3};\n\t"
      "fma.rn.f32x2 t, t, u, v;\n\t"
      "mov.b64 {%0, %1}, t;\n\t}"
      : "+f"(x0), "+f"(x1)
      : "f"(c), "f"(b));
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// exp2 of two f16 values at once (MUFU ex2.approx on an f16 pair).
__device__ __forceinline__ uint32_t ex2_f16x2(uint32_t x) {
  uint32_t y;
  asm("ex2.approx.f16x2 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

__global__ void __launch_bounds__(192, 1)
sparse_mla_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKV,
                       const __grid_constant__ CUtensorMap tmKpe, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + AttnSmem::BARS);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + AttnSmem::NUM_BARS);
  int* abort_word = reinterpret_cast<int*>(tmem_slot + 1);
  const uint32_t bar0 = smem_u32(bars);
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };

  const int warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31;

  // Work item. CTAs are ordered by groups of `hgroup` heads, so that the
  // CTAs resident at any time read the K/V of a few heads and those stay in
  // L2; within a group, heavy (late) query tiles come first.
  const int per_group = p.nq * p.B * p.hgroup;
  const int hg = static_cast<int>(blockIdx.x) / per_group;
  const int rem0 = static_cast<int>(blockIdx.x) % per_group;
  const int qt = p.nq - 1 - rem0 / (p.B * p.hgroup);
  const int rem = rem0 % (p.B * p.hgroup);
  const int b = rem / p.hgroup, h = hg * p.hgroup + rem % p.hgroup;
  const int32_t* gblist = p.blocks ? p.blocks + (static_cast<int64_t>(b) * p.nq + qt) * (p.nq + 1) : nullptr;
  const int n = gblist ? gblist[0] : qt + 1;
  // Key-block ids in shared memory (read by every role once per block).
  int32_t* blist = gblist ? reinterpret_cast<int32_t*>(smem + AttnSmem::BLIST) : nullptr;
  if (gblist) {
    for (int i = threadIdx.x; i < n; i += blockDim.x) blist[i] = gblist[1 + i];
  }
  {
    uint4* ones = reinterpret_cast<uint4*>(smem + AttnSmem::ONES);
    for (int i = threadIdx.x; i < 4096 / 16; i += blockDim.x) ones[i] = make_uint4(0x3C003C00u, 0x3C003C00u, 0x3C003C00u, 0x3C003C00u);
    fence_proxy_async_smem();  // read by the tensor core through a descriptor
  }

  if (threadIdx.x == 0) {
    mbar_init(bar(kBarQFull), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(kBarKFull0 + i), 1);
      mbar_init(bar(kBarKEmpty0 + i), 1);
      mbar_init(bar(kBarVFull0 + i), 1);
      mbar_init(bar(kBarVEmpty0 + i), 1);
      mbar_init(bar(kBarSFull0 + i), 1);
      mbar_init(bar(kBarSFree0 + i), 4);
    }
    mbar_init(bar(kBarPFull), 4);
    mbar_init(bar(kBarPvDone), 1);
    mbar_init(bar(kBarDrain), 1);
    *abort_word = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmKV);
    prefetch_tmap(&tmKpe);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Abort ab{abort_word, p.err};
  const uint32_t sQ = smem_u32(smem + AttnSmem::Q);

  if (warp == 0) {
    if (lane == 0 && n > 0) {
      // ---------------- TMA producer
      int nk = 0, nv = 0;
      bool ok = true;
      mbar_arrive_expect_tx(bar(kBarQFull), 3 * 16384);
      for (int c = 0; c < 3; ++c) tma_load_3d(sQ + c * 16384, &tmQ, bar(kBarQFull), h * 192 + 64 * c, qt * 128, b);
      auto load_k = [&](int j) -> bool {
        const int ks = j & 1;
        if (!mbar_wait(bar(kBarKEmpty0 + ks), ((j >> 1) & 1) ^ 1, ab, kErrWaitMma)) return false;
        const int t0 = (blist ? blist[j] : j) * 128;
        const uint32_t dst = smem_u32(smem + (ks ? AttnSmem::K1 : AttnSmem::K0));
        const uint32_t fb = bar(kBarKFull0 + ks);
        mbar_arrive_expect_tx(fb, 3 * 16384);
        tma_load_3d(dst, &tmKV, fb, h * 256, t0, b);
        tma_load_3d(dst + 16384, &tmKV, fb, h * 256 + 64, t0, b);
        tma_load_3d(dst + 32768, &tmKpe, fb, 0, t0, b);
        ++nk;
        return true;
      };
      ok = load_k(0);
      for (int j = 0; j < n && ok; ++j) {
        if (j + 1 < n && !(ok = load_k(j + 1))) break;
        const int vs = j & 1;
        if (!(ok = mbar_wait(bar(kBarVEmpty0 + vs), ((j >> 1) & 1) ^ 1, ab, kErrWaitMma))) break;
        const int t0 = (blist ? blist[j] : j) * 128;
        const uint32_t dst = smem_u32(smem + (vs ? AttnSmem::V1 : AttnSmem::V0));
        const uint32_t fb = bar(kBarVFull0 + vs);
        mbar_arrive_expect_tx(fb, 2 * 16384);
        tma_load_3d(dst, &tmKV, fb, h * 256 + 128, t0, b);
        tma_load_3d(dst + 16384, &tmKV, fb, h * 256 + 192, t0, b);
        ++nv;
      }
      if (!ok) {
        mbar_wait_drain(bar(kBarQFull), 0);
        for (int i = (nk > 2 ? nk - 2 : 0); i < nk; ++i) mbar_wait_drain(bar(kBarKFull0 + (i & 1)), (i >> 1) & 1);
        for (int i = (nv > 2 ? nv - 2 : 0); i < nv; ++i) mbar_wait_drain(bar(kBarVFull0 + (i & 1)), (i >> 1) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && n > 0) {
      // ---------------- UMMA issuer
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idesc_pv = idesc_f16_f32(128, 128, 0, 1);
      constexpr uint32_t idesc_l = idesc_f16_f32(128, 16, 0, 0);
      const uint32_t sOnes = smem_u32(smem + AttnSmem::ONES);
      bool ok = mbar_wait(bar(kBarQFull), 0, ab, kErrWaitTma);
      int issued = 0;
      auto issue_qk = [&](int j) -> bool {
        const int st = j & 1;
        if (!mbar_wait(bar(kBarKFull0 + st), (j >> 1) & 1, ab, kErrWaitTma)) return false;
        if (!mbar_wait(bar(kBarSFree0 + st), ((j >> 1) & 1) ^ 1, ab, kErrWaitSoftmax)) return false;
        tc_fence_after();
        const uint32_t sK = smem_u32(smem + (st ? AttnSmem::K1 : AttnSmem::K0));
        const uint32_t d = tmem + kTmemS0 + st * 128;
#pragma unroll
        for (int k = 0; k < 12; ++k) {
          const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
          umma_ss(d, smem_desc_sw128(sQ + off, 16, 1024), smem_desc_sw128(sK + off, 16, 1024), idesc_qk,
                  k > 0 ? 1u : 0u);
        }
        ++issued;
        umma_commit(bar(kBarKEmpty0 + st));
        umma_commit(bar(kBarSFull0 + st));
        return true;
      };
      if (ok) ok = issue_qk(0);
      for (int j = 0; j < n && ok; ++j) {
        if (j + 1 < n && !(ok = issue_qk(j + 1))) break;
        const int vs = j & 1;
        if (!(ok = mbar_wait(bar(kBarPFull), j & 1, ab, kErrWaitSoftmax))) break;
        if (!(ok = mbar_wait(bar(kBarVFull0 + vs), (j >> 1) & 1, ab, kErrWaitTma))) break;
        tc_fence_after();
        const uint32_t sV = smem_u32(smem + (vs ? AttnSmem::V1 : AttnSmem::V0));
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint64_t bdesc = smem_desc_sw128(sV + k * 2048, 16384, 1024);
          umma_ts(tmem + kTmemO, tmem + kTmemP + k * 8, bdesc, idesc_pv, (j > 0 || k > 0) ? 1u : 0u);
        }
        // Row sums: l += P . ones (every one of the 16 columns gets the sum).
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint64_t odesc = smem_desc_sw128(sOnes + (k >> 2) * 2048 + (k & 3) * 32, 16, 1024);
          umma_ts(tmem + kTmemL, tmem + kTmemP + k * 8, odesc, idesc_l, (j > 0 || k > 0) ? 1u : 0u);
        }
        ++issued;
        umma_commit(bar(kBarVEmpty0 + vs));
        umma_commit(bar(kBarPvDone));
      }
      if (!ok && issued > 0) {
        umma_commit(bar(kBarDrain));
        mbar_wait_drain(bar(kBarDrain), 0);
      }
    }
  } else {
    // ---------------- softmax warps: thread = query row r of the tile
    const int q4 = warp & 3;
    const int r = q4 * 32 + static_cast<int>(lane);
    const int s = qt * 128 + r;
    const uint32_t trow = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const int64_t tri_total = tri_index(p.nq, 0);
    const float c = p.scale_log2;
    float m_run = -INFINITY;  // running max (scaled log2 domain); the sums live in tensor memory
    bool ok = true;

    // Selection words of this row, fetched one block ahead.
    const uint4* bm_row = p.bitmap ? p.bitmap + (static_cast<int64_t>(b) * tri_total + tri_index(qt, 0)) * 128 + r
                                   : nullptr;
    uint4 bits_next = make_uint4(0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu);
    if (bm_row && n > 0) bits_next = __ldg(bm_row + static_cast<int64_t>(blist ? blist[0] : 0) * 128);
    for (int j = 0; j < n; ++j) {
      const int kb = blist ? blist[j] : j;
      const uint32_t bw[4] = {bits_next.x, bits_next.y, bits_next.z, bits_next.w};
      if (bm_row && j + 1 < n) bits_next = __ldg(bm_row + static_cast<int64_t>(blist ? blist[j + 1] : j + 1) * 128);
      const int st = j & 1;
      if (!(ok = warp_wait(bar(kBarSFull0 + st), (j >> 1) & 1, ab, kErrWaitMma))) break;
      tc_fence_after();
      float x[128];
      {
        uint32_t a0[32], a1[32];
        tmem_ld32x2(trow + kTmemS0 + st * 128, trow + kTmemS0 + st * 128 + 32, a0, a1);
#pragma unroll
        for (int i = 0; i < 32; ++i) { x[i] = __uint_as_float(a0[i]); x[32 + i] = __uint_as_float(a1[i]); }
        tmem_ld32x2(trow + kTmemS0 + st * 128 + 64, trow + kTmemS0 + st * 128 + 96, a0, a1);
#pragma unroll
        for (int i = 0; i < 32; ++i) { x[64 + i] = __uint_as_float(a0[i]); x[96 + i] = __uint_as_float(a1[i]); }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kBarSFree0 + st));

      // Selection: unselected scores become -inf (raw domain; the scale is
      // positive, so the max commutes with it).
      const bool all_sel = (bw[0] & bw[1] & bw[2] & bw[3]) == 0xffffffffu;
      const bool causal_diag = (p.bitmap == nullptr) && (kb == qt);
      if (causal_diag) {
#pragma unroll
        for (int i = 0; i < 128; ++i) x[i] = (i <= r) ? x[i] : -INFINITY;
      } else if (!__all_sync(0xffffffffu, all_sel)) {
#pragma unroll
        for (int i = 0; i < 128; ++i) x[i] = ((bw[i >> 5] >> (i & 31)) & 1u) ? x[i] : -INFINITY;
      }
      // Row max: 8 independent chains of 3-input max.
      float mx[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx[i] = max3(x[i], x[8 + i], x[16 + i]);
#pragma unroll
      for (int k0 = 24; k0 < 120; k0 += 16) {
#pragma unroll
        for (int i = 0; i < 8; ++i) mx[i] = max3(mx[i], x[k0 + i], x[k0 + 8 + i]);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) mx[i] = fmaxf(mx[i], x[120 + i]);
      const float mblk = fmaxf(max3(mx[0], mx[1], mx[2]), max3(mx[3], max3(mx[4], mx[5], mx[6]), mx[7])) * c;
      // Lazy rescaling: keep the running max unless the block max exceeds it
      // by more than 8 (a factor of 256), so O and l are rarely touched and P
      // stays below 2^8 (well inside f16).
      const float m_new = fmaxf(m_run, mblk);
      const bool resc = (m_new - m_run) > 8.f;
      float alpha = 1.f;
      if (resc) {
        alpha = ex2_approx(m_run - m_new);
        m_run = m_new;
      }
      const float nb = (m_run == -INFINITY) ? 0.f : -m_run;
      // P = exp2(S*c - m): the argument in fp32 (packed FMA), the exp2 on f16
      // pairs; masked entries are -inf and give 0.
      uint32_t pk[64];
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        fma2_scalar(x[2 * i], x[2 * i + 1], c, nb);
        pk[i] = ex2_f16x2(pack_f16x2(x[2 * i], x[2 * i + 1]));
      }

      // PV of the previous block must be complete before O and l are
      // rescaled and before P is overwritten.
      if (j >= 1) {
        if (!(ok = warp_wait(bar(kBarPvDone), (j - 1) & 1, ab, kErrWaitMma))) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, resc)) {
#pragma unroll 1
          for (int c0 = 0; c0 < 160; c0 += 32) {  // O (128 columns), then l (16) and 16 spare
            uint32_t o[32];
            tmem_ld32(trow + kTmemO + c0, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(trow + kTmemO + c0, o);
          }
        }
      }
      // P (f16 pairs) into tensor memory, row r = lane r.
      {
        uint32_t (&p0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&pk[0]);
        uint32_t (&p1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&pk[32]);
        tmem_st32(trow + kTmemP, p0);
        tmem_st32(trow + kTmemP + 32, p1);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kBarPFull));
    }

    if (ok) {
      __nv_bfloat16* dst = p.attn + ((static_cast<int64_t>(b) * p.T + s) * p.H + h) * 128;
      if (n > 0) {
        ok = warp_wait(bar(kBarPvDone), (n - 1) & 1, ab, kErrWaitMma);
        if (ok) {
          tc_fence_after();
          uint32_t lv[32];
          tmem_ld32(trow + kTmemL, lv);
          const float l_row = __uint_as_float(lv[0]);
          const float inv = l_row > 0.f ? 1.f / l_row : 0.f;
#pragma unroll 1
          for (int c0 = 0; c0 < 128; c0 += 64) {
            uint32_t a0[32], a1[32];
            tmem_ld32x2(trow + kTmemO + c0, trow + kTmemO + c0 + 32, a0, a1);
            if (s < p.T) {
              uint4* d4 = reinterpret_cast<uint4*>(dst + c0);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                d4[i] = make_uint4(pack_bf16x2(__uint_as_float(a0[8 * i + 0]) * inv, __uint_as_float(a0[8 * i + 1]) * inv),
                                   pack_bf16x2(__uint_as_float(a0[8 * i + 2]) * inv, __uint_as_float(a0[8 * i + 3]) * inv),
                                   pack_bf16x2(__uint_as_float(a0[8 * i + 4]) * inv, __uint_as_float(a0[8 * i + 5]) * inv),
                                   pack_bf16x2(__uint_as_float(a0[8 * i + 6]) * inv, __uint_as_float(a0[8 * i + 7]) * inv));
                d4[4 + i] = make_uint4(pack_bf16x2(__uint_as_float(a1[8 * i + 0]) * inv, __uint_as_float(a1[8 * i + 1]) * inv),
                                       pack_bf16x2(__uint_as_float(a1[8 * i + 2]) * inv, __uint_as_float(a1[8 * i + 3]) * inv),
                                       pack_bf16x2(__uint_as_float(a1[8 * i + 4]) * inv, __uint_as_float(a1[8 * i + 5]) * inv),
                                       pack_bf16x2(__uint_as_float(a1[8 * i + 6]) * inv, __uint_as_float(a1[8 * i + 7]) * inv));
              }
            }
          }
        }
      } else if (s < p.T) {
        uint4* d4 = reinterpret_cast<uint4*>(dst);
        for (int i = 0; i < 16; ++i) d4[i] = make_uint4(0, 0, 0, 0);  // no surviving key
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace mla
