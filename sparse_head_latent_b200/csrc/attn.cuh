// attn.cuh -- fused sparse-causal MLA attention for sm_100a (tcgen05 + TMA).
//
// For one batch b, one head h and two consecutive tiles of 128 queries (the
// "A" tile 2p and the "B" tile 2p+1), over every 128-key block in which a
// query of either tile selected a key (DeepSeek-V3.2-Exp "Sparse attention",
// prefill):
//   S_t = q_h[tile t] . [k_nope_h | k_pe]^T      (UMMA, K = 192, S in tensor memory)
//   S_t = -inf where bit(s, t) = 0                (top-k + causal selection)
//   m   = running max of S*scale*log2e per row   (fp32)
//   P_t = exp2(S_t*scale*log2e - m)              (MUFU ex2, fp32; sums in fp32)
//   O_t += P_t . v_h                             (UMMA, P f16 from tensor memory, v f16)
//   attn[b, s, h, :] = O_t / l                   (bf16)
// Neither the [T, T] scores nor a float mask is ever materialised: the
// selection arrives as one bit per causal (query, key) pair.
//
// The two tiles share every K and V block and alternate on the tensor core:
// while the softmax warpgroup of tile A works on block j, the tensor core
// runs PV of tile B's block j-1 and QK^T of tile B's block j, and vice versa
// ("ping-pong"), so the softmax of one tile hides behind the other's UMMAs.
//
// CTA = 320 threads:
//   warp 0      TMA producer: both Q tiles once; K (k_nope from the
//               up-projected kv plus the shared k_pe) into a 2-deep ring;
//               V single-buffered
//   warp 1      tensor-memory allocator and UMMA issuer
//   warps 2..5  softmax of tile A, warps 6..9 softmax of tile B: one query
//               row per thread (tensor-memory lane = row)
// Tensor memory: S_A [0,128), O_A [128,256), S_B [256,384), O_B [384,512).
// P_t (f16 pairs, 64 columns) overwrites the first half of S_t once the
// softmax has read S_t; the PV UMMA reads it from there as its A operand.
#pragma once

#include "prepass.cuh"
#include "ptx.cuh"

namespace mla {

struct AttnParams {
  int B, T, H, nq;
  int npairs;                   // ceil(nq / 2) query-tile pairs
  int hgroup;                   // heads per scheduling group (divides H)
  float scale_log2;             // softmax scale * log2(e)
  const uint4* bitmap;          // selection bitmap, NULL = causal mask only
  const int32_t* blocks;        // active key blocks per tile pair (with bitmap)
  __nv_bfloat16* attn;          // [B, T, H, 128]
  int* err;
};

struct AttnSmem {
  static constexpr int QA = 0;             // 3 x [128 x 64] bf16, 128B-swizzled
  static constexpr int QB = 49152;
  static constexpr int K0 = 98304;         // stage 0: k_nope 0-63, 64-127, k_pe
  static constexpr int K1 = 147456;        // stage 1
  static constexpr int V = 196608;         // 2 x [128 keys x 64 dv] (f16)
  static constexpr int BARS = 229376;
  static constexpr int NUM_BARS = 15;
  static constexpr int BYTES = 1024 + BARS + 256;
};

constexpr int kAttnThreads = 320;

// Tensor-memory columns of tile t: S at 256t, O at 256t + 128.
__host__ __device__ constexpr uint32_t tmem_s(int t) { return 256u * t; }
__host__ __device__ constexpr uint32_t tmem_o(int t) { return 256u * t + 128u; }

// Barrier slots.
enum : int {
  kBarQFull = 0, kBarKFull0 = 1, kBarKEmpty0 = 3, kBarVFull = 5, kBarVEmpty = 6,
  kBarSFull0 = 7,   // per tile: S of the current block is in tensor memory
  kBarPFull0 = 9,   // per tile: P of the current block is in tensor memory (4 warps)
  kBarODone = 11,   // every UMMA of the CTA has completed
  kBarDrain = 12
};

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// (x0, x1) <- (x0 * c + b, x1 * c + b): one packed f32x2 FMA (one issue
// slot for two elements).
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

// (a0, a1) += (x0, x1): one packed f32x2 add.
__device__ __forceinline__ void add2(float& a0, float& a1, float x0, float x1) {
  asm("{\n\t.reg .b64 t, u;\n\t"
      "mov.b64 t, {%0, %1};\n\t"
      "mov.b64 u, {%2, %3};\n\t"
      "add.f32x2 t, t, u;\n\t"
      "mov.b64 {%0, %1}, t;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(x0), "f"(x1));
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__global__ void __launch_bounds__(kAttnThreads, 1)
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
  if (blockDim.x != kAttnThreads) {  // every role below assumes this block size
    if (threadIdx.x == 0) atomicCAS(p.err, 0, kErrGeometry);
    return;
  }

  // Work item: (batch, head, tile pair). CTAs are ordered by groups of
  // `hgroup` heads, so that the CTAs resident at any time read the K/V of a
  // few heads and those stay in L2; within a group, heavy (late) pairs first.
  const int per_group = p.npairs * p.B * p.hgroup;
  const int hg = static_cast<int>(blockIdx.x) / per_group;
  const int rem0 = static_cast<int>(blockIdx.x) % per_group;
  const int pair = p.npairs - 1 - rem0 / (p.B * p.hgroup);
  const int rem = rem0 % (p.B * p.hgroup);
  const int b = rem / p.hgroup, h = hg * p.hgroup + rem % p.hgroup;
  const bool has_b = 2 * pair + 1 < p.nq;      // an odd tile count leaves the last pair with one tile
  const int ntiles = has_b ? 2 : 1;
  const int32_t* blist = p.blocks ? p.blocks + (static_cast<int64_t>(b) * p.nq + pair) * (p.nq + 1) : nullptr;
  const int n = blist ? blist[0] : 2 * pair + ntiles;  // key blocks to visit (union of both tiles)
  auto kblock = [&](int j) { return blist ? blist[1 + j] : j; };

  if (threadIdx.x == 0) {
    mbar_init(bar(kBarQFull), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(kBarKFull0 + i), 1);
      mbar_init(bar(kBarKEmpty0 + i), 1);
      mbar_init(bar(kBarSFull0 + i), 1);
      mbar_init(bar(kBarPFull0 + i), 4);
    }
    mbar_init(bar(kBarVFull), 1);
    mbar_init(bar(kBarVEmpty), 1);
    mbar_init(bar(kBarODone), 1);
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

  if (warp == 0) {
    if (lane == 0 && n > 0) {
      // ---------------- TMA producer
      int nk = 0, nv = 0;
      bool ok = true;
      mbar_arrive_expect_tx(bar(kBarQFull), ntiles * 3 * 16384);
      for (int t = 0; t < ntiles; ++t) {
        const uint32_t sq = smem_u32(smem + (t ? AttnSmem::QB : AttnSmem::QA));
        for (int c = 0; c < 3; ++c)
          tma_load_3d(sq + c * 16384, &tmQ, bar(kBarQFull), h * 192 + 64 * c, (2 * pair + t) * 128, b);
      }
      auto load_k = [&](int j) -> bool {
        const int ks = j & 1;
        if (!mbar_wait(bar(kBarKEmpty0 + ks), ((j >> 1) & 1) ^ 1, ab, kErrWaitMma)) return false;
        const int t0 = kblock(j) * 128;
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
        if (!(ok = mbar_wait(bar(kBarVEmpty), (j & 1) ^ 1, ab, kErrWaitMma))) break;
        const int t0 = kblock(j) * 128;
        const uint32_t dst = smem_u32(smem + AttnSmem::V);
        mbar_arrive_expect_tx(bar(kBarVFull), 2 * 16384);
        tma_load_3d(dst, &tmKV, bar(kBarVFull), h * 256 + 128, t0, b);
        tma_load_3d(dst + 16384, &tmKV, bar(kBarVFull), h * 256 + 192, t0, b);
        ++nv;
      }
      if (!ok) {
        mbar_wait_drain(bar(kBarQFull), 0);
        for (int i = (nk > 2 ? nk - 2 : 0); i < nk; ++i) mbar_wait_drain(bar(kBarKFull0 + (i & 1)), (i >> 1) & 1);
        if (nv > 0) mbar_wait_drain(bar(kBarVFull), (nv - 1) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && n > 0) {
      // ---------------- UMMA issuer
      // Order per key block j: for each tile t, O_t += P_t(j) . V_j as soon as
      // the softmax has written P_t(j), then S_t(j+1) = Q_t . K_{j+1}^T. The
      // tensor core therefore runs tile B's PV/QK^T while tile A's softmax
      // works and vice versa. Every commit covers all earlier UMMAs of this
      // thread, so "S_t(j+1) is ready" also means "PV_t(j) is done".
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idesc_pv = idesc_f16_f32(128, 128, 0, 1);
      // Shared-memory descriptors are built once; a K step only moves the
      // start address (bits 0-13, in 16-byte units), which never carries.
      const uint64_t dQ[2] = {smem_desc_sw128(smem_u32(smem + AttnSmem::QA), 16, 1024),
                              smem_desc_sw128(smem_u32(smem + AttnSmem::QB), 16, 1024)};
      const uint64_t dK[2] = {smem_desc_sw128(smem_u32(smem + AttnSmem::K0), 16, 1024),
                              smem_desc_sw128(smem_u32(smem + AttnSmem::K1), 16, 1024)};
      const uint64_t dV = smem_desc_sw128(smem_u32(smem + AttnSmem::V), 16384, 1024);
      int issued = 0;
      auto qk = [&](int t, int j) {
        const uint64_t q0 = t ? dQ[1] : dQ[0];
        const uint64_t k0 = (j & 1) ? dK[1] : dK[0];
#pragma unroll
        for (int k = 0; k < 12; ++k) {
          const uint32_t off = ((k >> 2) * 16384 + (k & 3) * 32) >> 4;
          umma_ss(tmem + tmem_s(t), q0 + off, k0 + off, idesc_qk, k > 0 ? 1u : 0u);
        }
        umma_commit(bar(kBarSFull0 + t));
        ++issued;
      };
      auto pv = [&](int t, int j) {
#pragma unroll
        for (int k = 0; k < 8; ++k)
          umma_ts(tmem + tmem_o(t), tmem + tmem_s(t) + k * 8, dV + ((k * 2048) >> 4), idesc_pv,
                  (j > 0 || k > 0) ? 1u : 0u);
        ++issued;
      };
      bool ok = mbar_wait(bar(kBarQFull), 0, ab, kErrWaitTma) && mbar_wait(bar(kBarKFull0), 0, ab, kErrWaitTma);
      if (ok) {
        tc_fence_after();
        for (int t = 0; t < ntiles; ++t) qk(t, 0);
        umma_commit(bar(kBarKEmpty0));
      }
      for (int j = 0; j < n && ok; ++j) {
        const bool next = j + 1 < n;
        if (!(ok = mbar_wait(bar(kBarVFull), j & 1, ab, kErrWaitTma))) break;
        for (int t = 0; t < ntiles && ok; ++t) {
          if (!(ok = mbar_wait(bar(kBarPFull0 + t), j & 1, ab, kErrWaitSoftmax))) break;
          tc_fence_after();
          pv(t, j);
          if (t == ntiles - 1) umma_commit(bar(kBarVEmpty));  // V_j is no longer read
          if (next) {
            if (t == 0 && !(ok = mbar_wait(bar(kBarKFull0 + ((j + 1) & 1)), ((j + 1) >> 1) & 1, ab, kErrWaitTma)))
              break;
            tc_fence_after();
            qk(t, j + 1);
          }
        }
        if (ok && next) umma_commit(bar(kBarKEmpty0 + ((j + 1) & 1)));
      }
      if (ok) umma_commit(bar(kBarODone));
      if (!ok && issued > 0) {
        umma_commit(bar(kBarDrain));
        mbar_wait_drain(bar(kBarDrain), 0);
      }
    }
  } else {
    // ---------------- softmax: warpgroup t = (warp - 2) / 4 owns query tile t;
    // thread = query row r of the tile (tensor-memory lane r)
    const int t = (warp - 2) >> 2;
    if (t < ntiles) {
      const int q4 = warp & 3;
      const int r = q4 * 32 + static_cast<int>(lane);
      const int qt = 2 * pair + t;
      const int s = qt * 128 + r;
      const uint32_t trow = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
      const uint32_t tS = trow + tmem_s(t), tO = trow + tmem_o(t);
      const int64_t tri_total = tri_index(p.nq, 0);
      const uint4* bm_row = p.bitmap ? p.bitmap + (static_cast<int64_t>(b) * tri_total + tri_index(qt, 0)) * 128 + r
                                     : nullptr;
      // Selection words of block j for this row; blocks past this tile's
      // causal range select nothing.
      auto bits_of = [&](int j) -> uint4 {
        const int kb = kblock(j);
        if (kb > qt) return make_uint4(0u, 0u, 0u, 0u);
        if (!bm_row) return make_uint4(0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu);
        return __ldg(bm_row + static_cast<int64_t>(kb) * 128);
      };
      const float c = p.scale_log2;
      float m_run = -INFINITY, l_run = 0.f;  // running max (scaled log2 domain) and row sum
      bool ok = true;
      uint4 bits_next = n > 0 ? bits_of(0) : make_uint4(0u, 0u, 0u, 0u);

      for (int j = 0; j < n; ++j) {
        const int kb = kblock(j);
        const uint32_t bw[4] = {bits_next.x, bits_next.y, bits_next.z, bits_next.w};
        if (j + 1 < n) bits_next = bits_of(j + 1);
        if (!(ok = warp_wait(bar(kBarSFull0 + t), j & 1, ab, kErrWaitMma))) break;
        tc_fence_after();
        uint32_t pk[64];
        float alpha = 1.f;
        bool resc = false;
        if (kb > qt) {
          // Block beyond this tile's causal range (visited for the other tile).
#pragma unroll
          for (int i = 0; i < 64; ++i) pk[i] = 0u;
        } else {
          float x[128];
          tmem_ld128(tS, *reinterpret_cast<uint32_t(*)[128]>(x));
          // Selection: unselected scores become -inf (raw domain; the scale is
          // positive, so the max commutes with it).
          const bool all_sel = (bw[0] & bw[1] & bw[2] & bw[3]) == 0xffffffffu;
          if (p.bitmap == nullptr && kb == qt) {
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
          // Lazy rescaling: keep the running max unless the block max exceeds
          // it by more than 8 (a factor of 256), so O is rarely touched and P
          // stays below 2^8 (well inside f16).
          const float m_new = fmaxf(m_run, mblk);
          resc = (m_new - m_run) > 8.f;
          if (resc) {
            alpha = ex2_approx(m_run - m_new);
            m_run = m_new;
          }
          const float nb = (m_run == -INFINITY) ? 0.f : -m_run;
          float sm[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) sm[i] = 0.f;
          // The argument and the row sums use packed f32x2 FMA/add (one issue
          // slot per two elements); the softmax is bound by issue slots.
#pragma unroll
          for (int i = 0; i < 64; ++i) {
            fma2_scalar(x[2 * i], x[2 * i + 1], c, nb);
            const float p0 = ex2_approx(x[2 * i]);
            const float p1 = ex2_approx(x[2 * i + 1]);
            add2(sm[2 * (i & 3)], sm[2 * (i & 3) + 1], p0, p1);
            pk[i] = pack_f16x2(p0, p1);
          }
          l_run = l_run * alpha + (((sm[0] + sm[1]) + (sm[2] + sm[3])) + ((sm[4] + sm[5]) + (sm[6] + sm[7])));
        }
        // O holds PV of blocks < j (complete: S_t(j) was committed after
        // them); rescale it before PV of block j is issued.
        if (j >= 1 && __any_sync(0xffffffffu, resc)) {
#pragma unroll 1
          for (int c0 = 0; c0 < 128; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(tO + c0, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tO + c0, o);
          }
        }
        // P (f16 pairs) over the first half of S_t.
        tmem_st64(tS, pk);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBarPFull0 + t));
      }

      if (ok) {
        __nv_bfloat16* dst = p.attn + ((static_cast<int64_t>(b) * p.T + s) * p.H + h) * 128;
        if (n > 0) {
          ok = warp_wait(bar(kBarODone), 0, ab, kErrWaitMma);
          if (ok) {
            tc_fence_after();
            const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll 1
            for (int c0 = 0; c0 < 128; c0 += 64) {
              uint32_t a0[32], a1[32];
              tmem_ld32x2(tO + c0, tO + c0 + 32, a0, a1);
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
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace mla
